// rope_dca.cuh — RoPE table and DCA position remap (rotation of keys and query views).
//
// "Qwen2.5-1M Technical Report" paper review (xllm-io), section 三: RoPE; section 四
// "Dual Chunk Attention": intra-chunk, successive-chunk and inter-chunk patterns keep
// remapped relative positions inside the trained range; "YaRN 注意力缩放": logits are
// scaled by (0.1 ln s + 1)^2 / sqrt(D).
//
// Positions (one DCA chunk holds L = c - w tokens, c = dca_chunk, w = local_window):
//   key j                         -> j mod L
//   query i, intra pattern        -> i mod L
//   query i, successive pattern   -> min(i mod L + L, c - 1)
//   query i, inter pattern        -> c - 1
// RoPE is the rotate-half form on pairs (f, f + D/2), theta_f = base^(-2f/D).
// Query views carry the whole logit scale (1/t) / sqrt(D) * log2(e), so the attention
// kernels work in base-2 exponentials directly.
#pragma once

#include "q1m_device.cuh"

namespace q1m {

enum : int { VIEW_INTRA = 0, VIEW_SUCC = 1, VIEW_INTER = 2 };

template <typename T>
__device__ __forceinline__ float load_as_f32(const T* p);
template <>
__device__ __forceinline__ float load_as_f32<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_as_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// The rotate-half pair (x1, x2) by the angle with (cos, sin) = cs, with one fixed rounding
// (explicit fused multiply-adds), so that every kernel that rotates the same values (the
// prefill's keys and views, the decode step's) produces the same bits.
__device__ __forceinline__ float rot_lo(float x1, float x2, float2 cs) { return __fmaf_rn(x1, cs.x, -(x2 * cs.y)); }
__device__ __forceinline__ float rot_hi(float x1, float x2, float2 cs) { return __fmaf_rn(x2, cs.x, x1 * cs.y); }

__device__ __forceinline__ uint16_t to_f16_checked(float x) {
  if (!(fabsf(x) <= 65504.f)) latch(Q1M_ERR_RANGE);   // also catches NaN
  return __half_as_ushort(__float2half_rn(x));
}

// table[pos][f] = (cos, sin)(pos * base^(-2f/D)), angle in fp64.
__global__ void rope_table_kernel(float2* table, int64_t n_pos, int half_d, double base) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pos * half_d) return;
  const int64_t pos = idx / half_d;
  const int f = (int)(idx % half_d);
  const double theta = pow(base, -2.0 * (double)f / (double)(2 * half_d));
  double s, c;
  sincos((double)pos * theta, &s, &c);
  table[idx] = make_float2((float)c, (float)s);
}

// Eight consecutive elements of one row as fp32 (16 bytes of bf16 or 32 bytes of fp32).
__device__ __forceinline__ void load8_f32(const __nv_bfloat16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    x[2 * k] = __uint_as_float(w[k] << 16);
    x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8_f32(const float* p, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Keys [s0, e): k_rot[g][j] = R(j mod L) k[j][g]; v16[g][j] = v[j][g]; fp16. grid.x = e - s0
// (one block per token); each thread rotates 8 pairs (f, f + D/2) of one KV head with 16-byte
// loads and stores, and converts the same 16 elements of v.
template <typename T>
__global__ void rope_keys_kernel(const T* __restrict__ k, const T* __restrict__ v, int64_t s0,
                                 int64_t e, int hkv, int d, int64_t L,
                                 const float2* __restrict__ table, uint16_t* __restrict__ k_rot,
                                 uint16_t* __restrict__ v16, int64_t ld_tokens) {
  const int hd = d >> 1, n8 = hd >> 3;
  const int64_t j = s0 + blockIdx.x;
  if (j >= e) return;
  const float2* trow = table + (j % L) * hd;
  for (int w = threadIdx.x; w < hkv * n8; w += blockDim.x) {
    const int g = w / n8, f0 = (w - g * n8) * 8;
    const int64_t src = (j * hkv + g) * d;
    const int64_t dst = ((int64_t)g * ld_tokens + j) * d;
    float x1[8], x2[8], v1[8], v2[8];
    load8_f32(k + src + f0, x1);
    load8_f32(k + src + f0 + hd, x2);
    load8_f32(v + src + f0, v1);
    load8_f32(v + src + f0 + hd, v2);
    const float4* cs4 = reinterpret_cast<const float4*>(trow + f0);
    uint32_t lo[4], hi[4], vl[4], vh[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 t4 = __ldg(cs4 + q);                 // (cos, sin) of pairs 2q, 2q + 1
      const float2 ca = make_float2(t4.x, t4.y), cb = make_float2(t4.z, t4.w);
      lo[q] = (uint32_t)to_f16_checked(rot_lo(x1[2 * q], x2[2 * q], ca)) |
              ((uint32_t)to_f16_checked(rot_lo(x1[2 * q + 1], x2[2 * q + 1], cb)) << 16);
      hi[q] = (uint32_t)to_f16_checked(rot_hi(x1[2 * q], x2[2 * q], ca)) |
              ((uint32_t)to_f16_checked(rot_hi(x1[2 * q + 1], x2[2 * q + 1], cb)) << 16);
      vl[q] = (uint32_t)to_f16_checked(v1[2 * q]) | ((uint32_t)to_f16_checked(v1[2 * q + 1]) << 16);
      vh[q] = (uint32_t)to_f16_checked(v2[2 * q]) | ((uint32_t)to_f16_checked(v2[2 * q + 1]) << 16);
    }
    *reinterpret_cast<uint4*>(k_rot + dst + f0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(k_rot + dst + f0 + hd) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(v16 + dst + f0) = make_uint4(vl[0], vl[1], vl[2], vl[3]);
    *reinterpret_cast<uint4*>(v16 + dst + f0 + hd) = make_uint4(vh[0], vh[1], vh[2], vh[3]);
  }
}

__device__ __forceinline__ int64_t dca_query_pos(int64_t i, int view, int64_t L, int64_t c) {
  const int64_t t = i % L;
  if (view == VIEW_INTRA) return t;
  if (view == VIEW_SUCC) return t + L < c - 1 ? t + L : c - 1;
  return c - 1;
}

// Query views for rows [s0, e): qv[x][h][i - s0] = scale * R(pos_x(i)) q[i][h]; rows
// e - s0 .. ld_rows-1 are zero. grid.x = ld_rows (one block per row, whose three view
// positions are then uniform); each thread rotates 8 pairs (f, f + D/2) of one head with
// 16-byte loads and stores.
template <typename T>
__global__ void rope_queries_kernel(const T* __restrict__ q, int64_t s0, int64_t e, int hq,
                                    int d, int64_t L, int64_t c, float scale,
                                    const float2* __restrict__ table, uint16_t* __restrict__ qv,
                                    int64_t ld_rows) {
  const int hd = d >> 1, n8 = hd >> 3;
  const int64_t r = blockIdx.x;
  const int64_t i = s0 + r;
  const bool in = i < e;
  int64_t pos[3] = {0, 0, 0};
  if (in) {
#pragma unroll
    for (int x = 0; x < 3; ++x) pos[x] = dca_query_pos(i, x, L, c);
  }
  for (int w = threadIdx.x; w < hq * n8; w += blockDim.x) {
    const int h = w / n8, f0 = (w - h * n8) * 8;
    float x1[8], x2[8];
    if (in) {
      const int64_t src = (i * hq + h) * d;
      load8_f32(q + src + f0, x1);
      load8_f32(q + src + f0 + hd, x2);
#pragma unroll
      for (int k = 0; k < 8; ++k) { x1[k] *= scale; x2[k] *= scale; }
    }
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const int64_t dst = (((int64_t)x * hq + h) * ld_rows + r) * d;
      uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
      if (in) {
        const float4* cs4 = reinterpret_cast<const float4*>(table + pos[x] * hd + f0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 t4 = __ldg(cs4 + k);                 // (cos, sin) of pairs 2k, 2k + 1
          const float2 ca = make_float2(t4.x, t4.y), cb = make_float2(t4.z, t4.w);
          lo[k] = (uint32_t)to_f16_checked(rot_lo(x1[2 * k], x2[2 * k], ca)) |
                  ((uint32_t)to_f16_checked(rot_lo(x1[2 * k + 1], x2[2 * k + 1], cb)) << 16);
          hi[k] = (uint32_t)to_f16_checked(rot_hi(x1[2 * k], x2[2 * k], ca)) |
                  ((uint32_t)to_f16_checked(rot_hi(x1[2 * k + 1], x2[2 * k + 1], cb)) << 16);
        }
      }
      *reinterpret_cast<uint4*>(qv + dst + f0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(qv + dst + f0 + hd) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
  }
}

// Estimator query operand. Rows R = [r_lo, e) (n_r <= 64 rows) of the Q heads of each KV
// group g are laid out as m = hh * 64 + r (hh < G). For a key block whose DCA chunk is
// kc, let cls = min(C_hi - kc, 3) with C_hi the chunk of row e - 1; row i then uses the
// view of pattern chunk(i) - kc = chunk(i) - C_hi + cls (no view, zero row, when that is
// negative: every key of the block is then in the row's future). Output
// est_q[cls][g][m][D] fp16, rows m >= G*64 padded with zeros up to m_pad.
template <typename T>
__global__ void est_queries_kernel(const T* __restrict__ q, int64_t r_lo, int64_t e, int hq,
                                   int hkv, int d, int64_t L, int64_t c, float scale,
                                   const float2* __restrict__ table, uint16_t* __restrict__ est_q,
                                   int m_pad) {
  const int hd = d >> 1;
  const int G = hq / hkv;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)4 * hkv * m_pad * hd;
  if (idx >= total) return;
  const int f = (int)(idx % hd);
  const int m = (int)((idx / hd) % m_pad);
  const int g = (int)((idx / ((int64_t)hd * m_pad)) % hkv);
  const int cls = (int)(idx / ((int64_t)hd * m_pad * hkv));
  const int hh = m / 64, r = m % 64;
  const int64_t i = r_lo + r;
  uint16_t y1 = 0, y2 = 0;
  if (hh < G && i < e) {
    const int64_t c_hi = (e - 1) / L;
    const int64_t rel = i / L - c_hi + cls;
    if (rel >= 0) {
      const int view = rel == 0 ? VIEW_INTRA : (rel == 1 ? VIEW_SUCC : VIEW_INTER);
      const int h = g * G + hh;
      const int64_t src = (i * hq + h) * d;
      const float x1 = load_as_f32(q + src + f) * scale;
      const float x2 = load_as_f32(q + src + f + hd) * scale;
      const float2 cs = table[dca_query_pos(i, view, L, c) * hd + f];
      y1 = to_f16_checked(rot_lo(x1, x2, cs));
      y2 = to_f16_checked(rot_hi(x1, x2, cs));
    }
  }
  const int64_t dst = (((int64_t)cls * hkv + g) * m_pad + m) * d;
  est_q[dst + f] = y1;
  est_q[dst + f + hd] = y2;
}

}  // namespace q1m
