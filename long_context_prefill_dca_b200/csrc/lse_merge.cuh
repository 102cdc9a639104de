// lse_merge.cuh — log-sum-exp merge of the partial attention results of DCA's three
// patterns ("Qwen2.5-1M Technical Report" paper review, section 四 "Dual Chunk
// Attention": intra-chunk, successive-chunk and inter-chunk attention of one softmax).
// For each row: lse = log2 sum_x 2^lse_x and out = sum_x 2^(lse_x - lse) o_x, over the
// patterns x (0 intra, 1 successive, 2 inter) that exist for the row (successive from the
// second DCA chunk on, inter from the third) and are not empty (lse_x = -inf).
#pragma once

#include "q1m_device.cuh"

namespace q1m {

template <typename TO, int D>
__global__ void lse_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                 int n_parts, int64_t ld_rows, int64_t s0, int64_t e, int hq,
                                 int64_t L, TO* __restrict__ out, float* __restrict__ lse,
                                 int64_t seq_len) {
  constexpr int PER = D / 32;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (e - s0) * hq) return;
  const int h = (int)(wid % hq);
  const int64_t rl = wid / hq;
  const int64_t i = s0 + rl;
  const int64_t cb = L > 0 ? i / L : 0;
  float lx[3];
  float M = -INFINITY;
  for (int x = 0; x < 3; ++x) {
    // with the DCA chunk length known, a pattern's partial exists only where the row has
    // such keys; otherwise every part is read and empty ones carry -inf
    bool exists = x < n_parts;
    if (exists && L > 0 && n_parts == 3) exists = (x == 0) || (x == 1 && cb >= 1) || (x == 2 && cb >= 2);
    lx[x] = exists ? lse_part[((int64_t)x * hq + h) * ld_rows + rl] : -INFINITY;
    M = fmaxf(M, lx[x]);
  }
  float acc[PER];
#pragma unroll
  for (int c = 0; c < PER; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  for (int x = 0; x < 3; ++x) {
    if (lx[x] == -INFINITY) continue;
    const float w = ex2(lx[x] - M);
    wsum += w;
    const float* src = o_part + (((int64_t)x * hq + h) * ld_rows + rl) * D;
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[c] += w * src[lane + 32 * c];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  TO* dst = out + (i * hq + h) * D;
#pragma unroll
  for (int c = 0; c < PER; ++c) {
    const float y = acc[c] * inv;
    if constexpr (sizeof(TO) == 2) dst[lane + 32 * c] = __float2bfloat16_rn(y);
    else dst[lane + 32 * c] = y;
  }
  if (lse && lane == 0)
    lse[(int64_t)h * seq_len + i] = wsum > 0.f ? (M + __log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace q1m
