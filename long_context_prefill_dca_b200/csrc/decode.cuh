// decode.cuh — DCA decode attention: the token at position pos attends keys [0, pos] with the
// same DCA logits as the prefill ("Qwen2.5-1M Technical Report" paper review, section 四
// "Dual Chunk Attention": intra, successive and inter chunk patterns; YaRN scaling; section
// 三: generation up to 8K tokens after a context of up to 1M).
//
// The step is HBM-bound: it reads every cached K/V row once (2 x n x Hkv x D x 2 bytes, 2 GB
// at 1M tokens for 4 KV heads) for G = Hq / Hkv query heads, about 7 FLOP per byte. FP32 FMA
// on the CUDA cores would take ~1.6x the HBM time, so the contraction runs on mma.sync
// (m16n8k16, fp16 in, fp32 accumulate) with the G heads of a KV group as the M rows (padded
// to 16): S = Q K^T, then P (from the accumulator fragments, no shuffles) times V.
//
//  * Split-KV: a CTA owns one KV group and a contiguous key range; its four warps take
//    32-key tiles round-robin, each with its own 3-stage TMA pipeline (128-byte-swizzled
//    tiles, read with ldmatrix; V through ldmatrix.trans) and its own online softmax. The
//    warps' partials are merged in shared memory, the CTAs' partials by dec_merge_kernel.
//  * A 32-key tile never straddles a DCA chunk (L is a multiple of 128), so each tile uses
//    one of the token's three query views: the key's chunk equal to the token's (intra),
//    one before it (successive) or older (inter).
#pragma once

#include "q1m_device.cuh"
#include "rope_dca.cuh"

namespace q1m {

constexpr int DEC_WARPS = 4;
constexpr int DEC_TILE = 32;       // keys per tile
constexpr int DEC_STAGES = 3;
constexpr int DEC_MAX_SPLIT = 256;  // CTAs per KV group at most (scratch is sized for it)

template <int D>
struct DecSmem {
  static constexpr int TILE = DEC_TILE * D * 2;   // bytes of one K (or V) tile
  static constexpr int HALF = DEC_TILE * 128;     // bytes of one 64-dim half of a tile
  alignas(1024) uint8_t k[DEC_WARPS][DEC_STAGES][TILE];
  alignas(1024) uint8_t v[DEC_WARPS][DEC_STAGES][TILE];
  float o[DEC_WARPS][8][D];                       // per-warp partials for the CTA merge
  float m[DEC_WARPS][8], l[DEC_WARPS][8];
  uint64_t full[DEC_WARPS][DEC_STAGES];
};

struct DecArgs {
  const uint16_t* qv;    // [3][hq][D] fp16: the token's views, scale folded in (log2 domain)
  int64_t pos, L, n_keys;
  int hq, G;
  int64_t ld_tokens;
  int nsplit;
  int64_t tiles_per_split, n_tiles;
  float* o_part;         // [nsplit][hq][D], normalised per split
  float* lse_part;       // [nsplit][hq], log2-sum-exp2 per split (-inf: empty)
};

__device__ __forceinline__ void mma_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// Shared-memory address of the 16-byte chunk c (8 dims) of key row r in a 128-byte-swizzled
// 32-row tile made of 64-dim halves HALF bytes apart.
template <int D>
__device__ __forceinline__ uint32_t dec_addr(uint32_t base, int r, int c) {
  return base + (uint32_t)(c >> 3) * DecSmem<D>::HALF + sw128_offset((uint32_t)r, (uint32_t)(c & 7));
}

template <int D>
__global__ void __launch_bounds__(32 * DEC_WARPS, 1)
dca_decode_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                  const DecArgs a) {
  extern __shared__ uint8_t dec_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(dec_raw) + 1023) & ~uintptr_t(1023));
  constexpr int KS = D / 16;   // k-steps of S = Q K^T
  constexpr int DN = D / 8;    // 8-dim n-tiles of O
  const int w = warp_id(), lane = lane_id(), gid = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x, g = blockIdx.y;
  const int64_t t_begin = (int64_t)split * a.tiles_per_split;
  const int64_t t_end = t_begin + a.tiles_per_split < a.n_tiles ? t_begin + a.tiles_per_split : a.n_tiles;
  if (lane == 0) {
    for (int s = 0; s < DEC_STAGES; ++s) mbar_init(&sm.full[w][s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int64_t cq = a.pos / a.L;
  // this warp's tiles: t_begin + w + DEC_WARPS i
  const int64_t n_mine = t_end - t_begin > w ? (t_end - t_begin - w + DEC_WARPS - 1) / DEC_WARPS : 0;
  auto issue = [&](int64_t i) {
    const int s = (int)(i % DEC_STAGES);
    const int64_t t = t_begin + w + DEC_WARPS * i;
    const int y = (int)((int64_t)g * a.ld_tokens + t * DEC_TILE);
    mbar_expect_tx(&sm.full[w][s], 2 * DecSmem<D>::TILE);
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
      tma_load_2d(sm.k[w][s] + hf * DecSmem<D>::HALF, &mk, &sm.full[w][s], 64 * hf, y);
      tma_load_2d(sm.v[w][s] + hf * DecSmem<D>::HALF, &mv, &sm.full[w][s], 64 * hf, y);
    }
  };
  if (lane == 0)
    for (int64_t i = 0; i < n_mine && i < DEC_STAGES; ++i) issue(i);
  float m_run = -INFINITY, l_run = 0.f;        // row gid (head gid of the group)
  float oacc[DN][4];
#pragma unroll
  for (int n = 0; n < DN; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  uint32_t qa[KS][4];
  int cur_view = -1;
  bool ok = true;
  for (int64_t i = 0; i < n_mine && ok; ++i) {
    const int s = (int)(i % DEC_STAGES);
    const int64_t t = t_begin + w + DEC_WARPS * i;
    const int64_t key0 = t * DEC_TILE;
    const int64_t ck = key0 / a.L;
    const int view = ck == cq ? 0 : (ck == cq - 1 ? 1 : 2);
    if (view != cur_view) {
      // A fragments of the view: rows = heads of the group (gid < G), cols = dims
      const bool live = gid < a.G;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          a.qv + ((int64_t)view * a.hq + (int64_t)g * a.G + (live ? gid : 0)) * D);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = live ? qrow[8 * kk + tig] : 0u;       // dims 16kk + 2tig, +1
        qa[kk][1] = 0u;                                    // rows 8..15: no heads
        qa[kk][2] = live ? qrow[8 * kk + 4 + tig] : 0u;   // dims 16kk + 8 + 2tig, +1
        qa[kk][3] = 0u;
      }
      cur_view = view;
    }
    ok = mbar_wait_warp(&sm.full[w][s], (uint32_t)((i / DEC_STAGES) & 1));
    if (!ok) break;
    const uint32_t kb = smem_u32(sm.k[w][s]), vb = smem_u32(sm.v[w][s]);
    // S = Q K^T: 4 n-tiles of 8 keys
    float sc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        // matrices j: keys 8 (2np + (j >> 1)) + r, dim chunk 2kk + (j & 1)
        const int j = lane >> 3, r = lane & 7;
        uint32_t b[4];
        ldsm_x4(dec_addr<D>(kb, 8 * (2 * np + (j >> 1)) + r, 2 * kk + (j & 1)), b);
        mma_16816(sc[2 * np], qa[kk], b[0], b[1]);
        mma_16816(sc[2 * np + 1], qa[kk], b[2], b[3]);
      }
    }
    // keys past the token are masked (only in the last tile)
    if (key0 + DEC_TILE > a.n_keys) {
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          if (key0 + 8 * nt + 2 * tig + c >= a.n_keys) sc[nt][c] = -INFINITY;
    }
    // online softmax of row gid over the tile (the 4 threads of a group share the row)
    float mx = fmaxf(fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])),
                     fmaxf(fmaxf(sc[2][0], sc[2][1]), fmaxf(sc[3][0], sc[3][1])));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = ex2(m_run - m_new);   // 0 on the first tile (m_run = -inf)
    m_run = m_new;
    float p[4][2];
    float ps = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      p[nt][0] = ex2(sc[nt][0] - m_new);
      p[nt][1] = ex2(sc[nt][1] - m_new);
      ps += p[nt][0] + p[nt][1];
    }
    l_run = l_run * alpha + ps;               // this thread's columns; summed per row at the end
#pragma unroll
    for (int n = 0; n < DN; ++n) { oacc[n][0] *= alpha; oacc[n][1] *= alpha; }
    // O += P V: 2 k-steps of 16 keys; P from the accumulator fragments of n-tiles 2ks, 2ks+1
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t pa[4] = {pack_f16x2(p[2 * ks][0], p[2 * ks][1]), 0u,
                              pack_f16x2(p[2 * ks + 1][0], p[2 * ks + 1][1]), 0u};
#pragma unroll
      for (int dp = 0; dp < DN / 2; ++dp) {
        // matrices j: keys 16ks + 8 (j & 1) + r, dim chunk 2dp + (j >> 1), transposed
        const int j = lane >> 3, r = lane & 7;
        uint32_t b[4];
        ldsm_x4_t(dec_addr<D>(vb, 16 * ks + 8 * (j & 1) + r, 2 * dp + (j >> 1)), b);
        mma_16816(oacc[2 * dp], pa, b[0], b[1]);
        mma_16816(oacc[2 * dp + 1], pa, b[2], b[3]);
      }
    }
    // the stage is free once every lane's ldmatrix reads are done: refill it
    __syncwarp();
    if (lane == 0 && i + DEC_STAGES < n_mine) {
      fence_async_smem();
      issue(i + DEC_STAGES);
    }
  }
  // per-warp partial of each head of the group
  float lt = l_run;
  lt += __shfl_xor_sync(0xFFFFFFFFu, lt, 1);
  lt += __shfl_xor_sync(0xFFFFFFFFu, lt, 2);
  if (gid < 8) {
#pragma unroll
    for (int n = 0; n < DN; ++n) {
      sm.o[w][gid][8 * n + 2 * tig] = oacc[n][0];
      sm.o[w][gid][8 * n + 2 * tig + 1] = oacc[n][1];
    }
    if (tig == 0) { sm.m[w][gid] = m_run; sm.l[w][gid] = lt; }
  }
  if (!ok) {
    // let copies already issued land before the CTA exits
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
  __syncthreads();
  if (!ok) return;
  // CTA merge over the warps: thread -> (head r, dims)
  for (int idx = threadIdx.x; idx < a.G * D; idx += blockDim.x) {
    const int r = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < DEC_WARPS; ++ww) M = fmaxf(M, sm.m[ww][r]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < DEC_WARPS; ++ww) {
        if (sm.m[ww][r] == -INFINITY) continue;
        const float f = ex2(sm.m[ww][r] - M);
        L += f * sm.l[ww][r];
        O += f * sm.o[ww][r][d];
      }
    }
    const int h = g * a.G + r;
    a.o_part[((int64_t)split * a.hq + h) * D + d] = L > 0.f ? O / L : 0.f;
    if (d == 0) a.lse_part[(int64_t)split * a.hq + h] = L > 0.f ? M + __log2f(L) : -INFINITY;
  }
}

// out[h] = sum over splits of 2^(lse_s - lse) o_s, lse = log2 sum 2^lse_s (one warp per head).
template <typename TO, int D>
__global__ void dec_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                 int nsplit, int hq, TO* __restrict__ out, float* __restrict__ lse) {
  constexpr int PER = D / 32;
  const int h = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= hq) return;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, lse_part[(int64_t)s * hq + h]);
  float acc[PER];
#pragma unroll
  for (int c = 0; c < PER; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < nsplit && M != -INFINITY; ++s) {
    const float ls = lse_part[(int64_t)s * hq + h];
    if (ls == -INFINITY) continue;
    const float wgt = ex2(ls - M);
    wsum += wgt;
    const float* src = o_part + ((int64_t)s * hq + h) * D;
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[c] += wgt * src[lane + 32 * c];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int c = 0; c < PER; ++c) {
    const float y = acc[c] * inv;
    if constexpr (sizeof(TO) == 2) out[(int64_t)h * D + lane + 32 * c] = __float2bfloat16_rn(y);
    else out[(int64_t)h * D + lane + 32 * c] = y;
  }
  if (lse && lane == 0) lse[h] = wsum > 0.f ? (M + __log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

// The token's three query views: rotation at its intra / successive / inter positions
// (the same remap as the prefill), times (1/t)/sqrt(D) log2 e, in fp16: qv [3][hq][D].
template <typename T>
__global__ void dec_queries_kernel(const T* __restrict__ q, int hq, int d, int64_t pos, int64_t L,
                                   int64_t c, const float2* __restrict__ table, float scale,
                                   uint16_t* __restrict__ qv) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int hd = d / 2;
  if (idx >= (int64_t)3 * hq * hd) return;
  const int f = (int)(idx % hd);
  const int h = (int)((idx / hd) % hq);
  const int x = (int)(idx / ((int64_t)hd * hq));
  const float2 cs = table[dca_query_pos(pos, x, L, c) * hd + f];
  const float x1 = load_as_f32(q + (int64_t)h * d + f) * scale;
  const float x2 = load_as_f32(q + (int64_t)h * d + f + hd) * scale;
  uint16_t* dst = qv + ((int64_t)x * hq + h) * d;
  dst[f] = to_f16_checked(rot_lo(x1, x2, cs));
  dst[f + hd] = to_f16_checked(rot_hi(x1, x2, cs));
}

// Appends the token's key (rotated at pos mod L) and value to the fp16 cache at row pos and
// zeroes the rest of that 32-key tile (rows the decode tile reads but masks), so that masked
// keys never meet non-finite V values. Latches Q1M_ERR_RANGE on fp16 overflow.
template <typename T>
__global__ void dec_append_kernel(const T* __restrict__ k, const T* __restrict__ v, int hkv, int d,
                                  int64_t pos, int64_t L, int64_t ld_tokens,
                                  const float2* __restrict__ table, uint16_t* __restrict__ k_rot,
                                  uint16_t* __restrict__ v16) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int hd = d / 2;
  const int64_t rows = (pos / DEC_TILE + 1) * DEC_TILE - pos;   // pos .. end of its tile
  if (idx >= (int64_t)hkv * rows * hd) return;
  const int f = (int)(idx % hd);
  const int64_t r = (idx / hd) % rows;
  const int g = (int)(idx / ((int64_t)hd * rows));
  const int64_t row = pos + r;
  if (row >= ld_tokens) return;
  uint16_t* kd = k_rot + ((int64_t)g * ld_tokens + row) * d;
  uint16_t* vd = v16 + ((int64_t)g * ld_tokens + row) * d;
  if (r > 0) {
    kd[f] = kd[f + hd] = 0;
    vd[f] = vd[f + hd] = 0;
    return;
  }
  const float2 cs = table[(pos % L) * hd + f];
  const float x1 = load_as_f32(k + (int64_t)g * d + f), x2 = load_as_f32(k + (int64_t)g * d + f + hd);
  kd[f] = to_f16_checked(rot_lo(x1, x2, cs));
  kd[f + hd] = to_f16_checked(rot_hi(x1, x2, cs));
  vd[f] = to_f16_checked(load_as_f32(v + (int64_t)g * d + f));
  vd[f + hd] = to_f16_checked(load_as_f32(v + (int64_t)g * d + f + hd));
}

}  // namespace q1m
