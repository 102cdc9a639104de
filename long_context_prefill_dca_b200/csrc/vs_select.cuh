// vs_select.cuh — vertical-slash index selection and block-mask construction.
//
// "Qwen2.5-1M Technical Report" paper review (xllm-io), section 四 "稀疏注意力机制":
// MInference's vertical-slash pattern with key tokens chosen per prefill chunk. Per Q head
// the vertical budget keeps the columns with the largest vertical score and the slash
// budget the offsets with the largest slash score (offsets below vs_force_local always
// kept); larger score first, equal scores by the smaller index; results ascending.
// Then, for 128 x 128 blocks, key block kb of query block b (rows r0..r1) is computed when
// a selected slash line i - j = o with o <= r1 crosses it:
//   floor(max(0, r0 - o) / 128) <= kb <= floor((r1 - o) / 128),
// and selected columns outside computed blocks remain as residual single columns.
// All of this is integer work and matches the oracle bit for bit on equal scores.
#pragma once

#include "q1m_device.cuh"

namespace q1m {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_BITS0 = 11, SEL_BITS1 = 11, SEL_BITS2 = 10;

// Order key of a score: non-negative floats order like their bit patterns; forced entries
// get the largest key. Negative or NaN scores latch Q1M_ERR_RANGE.
__device__ __forceinline__ uint32_t sel_key(float v, bool forced) {
  if (forced) return 0xFFFFFFFFu;
  uint32_t b = __float_as_uint(v);
  if (b == 0x80000000u) return 0u;                 // -0
  if (b > 0x7F800000u) { latch(Q1M_ERR_RANGE); return 0u; }  // NaN or negative
  return b;
}

__device__ __forceinline__ int block_excl_scan(int v, int* tmp, int* total) {
  // tmp: SEL_THREADS/32 ints of shared memory
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int t = lane < (int)(blockDim.x >> 5) ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, t, o);
      if (lane >= o) t += y;
    }
    tmp[lane] = t;  // inclusive prefix over warps
  }
  __syncthreads();
  const int warp_before = wid > 0 ? tmp[wid - 1] : 0;
  *total = tmp[(blockDim.x >> 5) - 1];
  const int res = warp_before + x - v;
  __syncthreads();
  return res;
}

// Order keys of scores j0 .. j0 + 3 (j0 a multiple of 4; beyond e: key 0, valid false), with
// one 16-byte load when the row is 16-byte aligned.
__device__ __forceinline__ void sel_keys4(const float* __restrict__ sc, int64_t j0, int64_t e, int fl,
                                          bool vec, uint32_t (&key)[4], bool (&valid)[4]) {
  float v[4];
  if (vec && j0 + 3 < e) {
    const float4 x = *reinterpret_cast<const float4*>(sc + j0);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = j0 + k < e ? sc[j0 + k] : 0.f;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    valid[k] = j0 + k < e;
    key[k] = valid[k] ? sel_key(v[k], j0 + k < fl) : 0u;
  }
}

// grid (hq, 2): y = 0 vertical, y = 1 slash. One CTA selects one list of one head. Every pass
// reads the list with 16-byte loads, several in flight per thread: the passes are bound by
// the memory-level parallelism of one SM.
__global__ void __launch_bounds__(SEL_THREADS)
vs_select_kernel(const float* __restrict__ vert, const float* __restrict__ slash, int64_t ld,
                 int64_t e, int nv, int ns, int force_local, int32_t* __restrict__ V,
                 int32_t* __restrict__ S) {
  __shared__ int hist[1 << SEL_BITS0];
  __shared__ int scan_tmp[32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  const int h = blockIdx.x;
  const bool is_slash = blockIdx.y == 1;
  const float* sc = (is_slash ? slash : vert) + (int64_t)h * ld;
  const int k = is_slash ? ns : nv;
  const int kk = (int64_t)k < e ? k : (int)e;
  int32_t* out = (is_slash ? S : V) + (int64_t)h * kk;
  const int fl = is_slash ? force_local : 0;
  if (k == 0) return;
  if ((int64_t)k >= e) {
    for (int64_t j = threadIdx.x; j < e; j += blockDim.x) out[j] = (int32_t)j;
    return;
  }
  if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_remaining = k; }
  const bool vec = (reinterpret_cast<uintptr_t>(sc) & 15) == 0;
  const int bits[3] = {SEL_BITS0, SEL_BITS1, SEL_BITS2};
  int shift = 32;
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = bits[pass];
    shift -= nb;
    for (int b = threadIdx.x; b < (1 << nb); b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t pre = s_prefix, pm = s_mask;
    // thread t takes elements 4 (t + i blockDim) .. + 3, four groups per iteration
    for (int64_t base = 4 * (int64_t)threadIdx.x; base < e; base += 16 * (int64_t)blockDim.x) {
      uint32_t key[4][4];
      bool valid[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) sel_keys4(sc, base + 4 * (int64_t)u * blockDim.x, e, fl, vec, key[u], valid[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (valid[u][k] && (key[u][k] & pm) == pre) atomicAdd(&hist[(key[u][k] >> shift) & ((1u << nb) - 1u)], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = s_remaining;
      int b = (1 << nb) - 1;
      for (; b > 0; --b) {
        if (hist[b] >= rem) break;
        rem -= hist[b];
      }
      s_remaining = rem;
      s_prefix = pre | ((uint32_t)b << shift);
      s_mask = pm | (((1u << nb) - 1u) << shift);
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int need_eq = s_remaining;  // elements equal to T to take, smallest indices first
  // ascending compaction: warp w owns the contiguous range [w*seg, (w+1)*seg) and reads it 128
  // consecutive elements at a time (4 per lane); a first pass counts the keys above T and
  // equal to T, a block scan gives each warp its output offset, a second pass writes in index
  // order
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int64_t seg = ((e + nw - 1) / nw + 127) / 128 * 128;
  const int64_t w0 = (int64_t)wid * seg, w1 = w0 + seg < e ? w0 + seg : e;
  int n_gt = 0, n_eq = 0;
  for (int64_t base = w0; base < w1; base += 128) {
    uint32_t key[4];
    bool valid[4];
    sel_keys4(sc, base + 4 * lane, w1, fl, vec, key, valid);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      n_gt += valid[k] && key[k] > T;
      n_eq += valid[k] && key[k] == T;
    }
  }
  n_gt = __reduce_add_sync(0xFFFFFFFFu, (unsigned)n_gt);
  n_eq = __reduce_add_sync(0xFFFFFFFFu, (unsigned)n_eq);
  // warp totals -> exclusive prefix over warps (lane 0 of each warp carries the totals)
  int tot;
  const int gt_before = block_excl_scan(lane == 0 ? n_gt : 0, scan_tmp, &tot);
  const int eq_before = block_excl_scan(lane == 0 ? n_eq : 0, scan_tmp, &tot);
  int gt_run = __shfl_sync(0xFFFFFFFFu, gt_before, 0);   // keys above T before this step
  int eq_run = __shfl_sync(0xFFFFFFFFu, eq_before, 0);   // keys equal to T before this step
  for (int64_t base = w0; base < w1; base += 128) {
    uint32_t key[4];
    bool valid[4];
    sel_keys4(sc, base + 4 * lane, w1, fl, vec, key, valid);
    int c_gt = 0, c_eq = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      c_gt += valid[k] && key[k] > T;
      c_eq += valid[k] && key[k] == T;
    }
    // exclusive prefix of the lanes' counts (lane order is index order)
    int p_gt = c_gt, p_eq = c_eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xFFFFFFFFu, p_gt, o), b = __shfl_up_sync(0xFFFFFFFFu, p_eq, o);
      if (lane >= o) { p_gt += a; p_eq += b; }
    }
    int g_before = gt_run + p_gt - c_gt, e_before = eq_run + p_eq - c_eq;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!valid[k]) continue;
      if (key[k] > T) {
        out[g_before + (e_before < need_eq ? e_before : need_eq)] = (int32_t)(base + 4 * lane + k);
        ++g_before;
      } else if (key[k] == T) {
        if (e_before < need_eq) out[g_before + e_before] = (int32_t)(base + 4 * lane + k);
        ++e_before;
      }
    }
    gt_run += __shfl_sync(0xFFFFFFFFu, p_gt, 31);
    eq_run += __shfl_sync(0xFFFFFFFFu, p_eq, 31);
  }
}

// --------------------------------------------------------------------------------------
// Mask builder. grid (hq, ceil(nqb / MB_QB)), MB_THREADS threads; warp w < MB_QB owns
// query block qb = blockIdx.y * MB_QB + w for the per-block counts and residual list.
// --------------------------------------------------------------------------------------
constexpr int MB_QB = 8;
constexpr int MB_THREADS = 256;
constexpr int MB_MAX_NKW = 320;   // up to 40,960 key blocks (5.2M tokens)

__global__ void __launch_bounds__(MB_THREADS)
vs_mask_kernel(const int32_t* __restrict__ V, const int32_t* __restrict__ S, int64_t s0,
               int64_t e, int nv, int ns, int64_t L, uint32_t* __restrict__ mask,
               int32_t* __restrict__ resid, int32_t* __restrict__ cnt) {
  __shared__ uint32_t delta[MB_MAX_NKW + 1];     // block-diagonal offsets crossed by S
  __shared__ uint32_t words[MB_QB][MB_MAX_NKW];
  const int h = blockIdx.x;
  const int64_t nkb = (e + 127) / 128;
  const int nkw = (int)((nkb + 31) / 32);
  const int nqb = (int)((e - s0 + 127) / 128);
  const int32_t* Sh = S + (int64_t)h * ns;
  const int32_t* Vh = V + (int64_t)h * nv;
  for (int i = threadIdx.x; i <= nkw; i += blockDim.x) delta[i] = 0;
  __syncthreads();
  // For a full block (r1 = r0 + 127), o crosses key blocks b - floor(o/128) and
  // b - ceil(o/128): mark both block diagonals.
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int o = Sh[i];
    const int d0 = o >> 7, d1 = (o + 127) >> 7;
    if (d0 <= nkb) atomicOr(&delta[d0 >> 5], 1u << (d0 & 31));
    if (d1 <= nkb) atomicOr(&delta[d1 >> 5], 1u << (d1 & 31));
  }
  __syncthreads();
  const int qb0 = blockIdx.y * MB_QB;
  for (int idx = threadIdx.x; idx < MB_QB * nkw; idx += blockDim.x) {
    const int lq = idx / nkw, w = idx % nkw;
    const int qb = qb0 + lq;
    uint32_t bitsw = 0;
    if (qb < nqb) {
      const int64_t B = s0 / 128 + qb;
      const int64_t r0 = B * 128, r1 = r0 + 127 < e - 1 ? r0 + 127 : e - 1;
      if (r1 == r0 + 127) {
        for (int b = 0; b < 32; ++b) {
          const int64_t kb = 32 * w + b;
          if (kb > B) break;
          const int64_t dd = B - kb;
          if ((delta[dd >> 5] >> (dd & 31)) & 1u) bitsw |= 1u << b;
        }
      } else {
        // ragged last block: the definition per offset
        for (int i = 0; i < ns; ++i) {
          const int64_t o = Sh[i];
          if (o > r1) continue;
          const int64_t lo = (r0 - o > 0 ? r0 - o : 0) >> 7, hi = (r1 - o) >> 7;
          for (int64_t kb = lo; kb <= hi; ++kb)
            if (kb >= 32 * w && kb < 32 * w + 32) bitsw |= 1u << (kb - 32 * w);
        }
      }
    }
    words[lq][w] = bitsw;
    if (qb < nqb) mask[((int64_t)h * nqb + qb) * nkw + w] = bitsw;
  }
  __syncthreads();
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (wid >= MB_QB) return;
  const int qb = qb0 + wid;
  if (qb >= nqb) return;
  const int64_t B = s0 / 128 + qb;
  const int64_t r1 = B * 128 + 127 < e - 1 ? B * 128 + 127 : e - 1;
  const int64_t Lb = L / 128, cb = B / Lb;
  // computed blocks per DCA pattern: intra = [cb Lb, B], successive = chunk cb - 1,
  // inter = chunks <= cb - 2
  const int64_t seg_lo[3] = {cb * Lb, cb >= 1 ? (cb - 1) * Lb : 0, 0};
  const int64_t seg_hi[3] = {B, cb >= 1 ? cb * Lb - 1 : -1, cb >= 2 ? (cb - 1) * Lb - 1 : -1};
  int c3[3] = {0, 0, 0};
  for (int w = lane; w < nkw; w += 32) {
    const uint32_t bw = words[wid][w];
    for (int x = 0; x < 3; ++x) {
      if (seg_hi[x] < seg_lo[x]) continue;
      const int64_t b0 = 32 * w;
      const int64_t lo = seg_lo[x] > b0 ? seg_lo[x] - b0 : 0;
      const int64_t hi = seg_hi[x] < b0 + 31 ? seg_hi[x] - b0 : 31;
      if (hi < lo) continue;
      const uint32_t upto = hi == 31 ? 0xFFFFFFFFu : ((1u << (hi + 1)) - 1u);
      c3[x] += __popc(bw & upto & ~((1u << lo) - 1u));
    }
  }
  for (int x = 0; x < 3; ++x)
    for (int o = 16; o > 0; o >>= 1) c3[x] += __shfl_xor_sync(0xFFFFFFFFu, c3[x], o);
  // residual verticals in ascending order (so grouped: inter, successive, intra)
  int32_t* rdst = resid + ((int64_t)h * nqb + qb) * nv;
  int pos = 0;
  int r3[3] = {0, 0, 0};
  for (int i0 = 0; i0 < nv; i0 += 32) {
    const int i = i0 + lane;
    int j = -1;
    bool keep = false;
    if (i < nv) {
      j = Vh[i];
      if (j <= r1) {
        const int kb = j >> 7;
        keep = !((words[wid][kb >> 5] >> (kb & 31)) & 1u);
      }
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) {
      rdst[pos + __popc(bal & ((1u << lane) - 1u))] = j;
      const int64_t cj = (int64_t)j / L;
      r3[cj == cb ? 0 : (cj == cb - 1 ? 1 : 2)] += 1;
    }
    pos += __popc(bal);
  }
  for (int x = 0; x < 3; ++x)
    for (int o = 16; o > 0; o >>= 1) r3[x] += __shfl_xor_sync(0xFFFFFFFFu, r3[x], o);
  if (lane == 0) {
    int32_t* c = cnt + ((int64_t)h * nqb + qb) * 8;
    c[0] = c3[0]; c[1] = c3[1]; c[2] = c3[2];
    c[3] = r3[0]; c[4] = r3[1]; c[5] = r3[2];
    c[6] = pos; c[7] = 0;
  }
}

}  // namespace q1m
