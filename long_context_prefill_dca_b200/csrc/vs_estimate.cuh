// vs_estimate.cuh — vertical-slash score estimator on the tensor cores.
//
// "Qwen2.5-1M Technical Report" paper review (xllm-io), section 四 "稀疏注意力机制":
// MInference's vertical-slash pattern; key tokens chosen per prefill chunk while keeping
// relative positions continuous. For the last rows R of a prefill chunk [s0, e) and every
// Q head, p_ij = softmax over keys j <= i of the DCA logits, and
//   vert[h][j]  = sum_{i in R} p_ij,     slash[h][o] = sum_{i in R} p_{i, i-o}.
//
// The G Q heads of a KV group share keys, so the G * |R| (<= 448) estimator rows of a group
// form one operand ("est rows", m = hh * 64 + r). Each key block picks the rows' query view
// by its DCA chunk class (see est_queries_kernel).
//  pass A: rows as M (128 rows per tile), keys as N; online max/sum per row over a range of
//          key tiles; partial (max, sum) per split, merged into the row's log2-sum-exp2.
//  pass B: keys as M (128 keys per tile), est rows as N (<= 448 TMEM columns). Each thread
//          owns one key: its vertical score is a thread-local sum over rows. Slash sums go
//          through shared memory along diagonals (192 offsets per key tile, written per tile
//          and summed over the two tiles that touch each offset in a fixed order), so the
//          scores are deterministic.
#pragma once

#include "q1m_device.cuh"

namespace q1m {

constexpr int EA_THREADS = 192;   // warps 0-3 softmax, 4 loader, 5 MMA
constexpr int EA_NK = 2;
constexpr int EB_THREADS = 576;   // warps 0-15 epilogue (4 groups), 16 loader, 17 MMA
constexpr int EB_GROUPS = 4;      // epilogue groups of 4 warps (one per TMEM lane quarter)
constexpr int EB_STEP = 16;       // est rows per epilogue step
constexpr int EB_NK = 2;
constexpr int EB_MAX_ROWS = 448;
constexpr int EB_U = 192;         // offsets per key tile (64 + 128 - 1 used)

struct EstArgs {
  int64_t r_lo, e;     // estimator rows [r_lo, e)
  int hq, hkv, G;
  int64_t L, ld_tokens;
  int m_pad;           // est rows per (class, group), multiple of 128
  int nkt;             // key tiles over [0, e)
  int n_mt;            // 128-row tiles of est rows
  int nsplit;          // pass A key-range splits
  int64_t c_hi;        // DCA chunk of row e - 1
  float2* part;        // pass A partials [hkv][n_mt*128][nsplit]
  float* lse2;         // [hkv][m_pad]
  float* vert;         // [hq][ld]
  float* slash_part;   // [hq][nkt][EB_U]
  int64_t ld;
};

__device__ __forceinline__ int est_class(const EstArgs& a, int kt) {
  const int64_t kc = (int64_t)kt * 128 / a.L;
  const int64_t d = a.c_hi - kc;
  return d >= 3 ? 3 : (int)d;
}

// --------------------------------------------------------------------------------------
// Pass A. grid = hkv * n_mt * nsplit; CTA -> (g, mt, split) over key tiles [t0, t1).
// --------------------------------------------------------------------------------------
template <int D>
struct EASmem {
  static constexpr int TILE = 128 * D * 2;
  alignas(1024) uint8_t q[TILE];
  alignas(1024) uint8_t k[EA_NK][TILE];
  uint64_t k_full[EA_NK], k_empty[EA_NK], q_full, q_empty, s_full[2], s_free[2], drain;
  uint32_t tmem_base;
};

template <int D>
__global__ void __launch_bounds__(EA_THREADS, 2)
est_pass_a_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const EstArgs a) {
  extern __shared__ uint8_t ea_raw[];
  EASmem<D>& sm = *reinterpret_cast<EASmem<D>*>((reinterpret_cast<uintptr_t>(ea_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t TILE = EASmem<D>::TILE;
  const int w = warp_id();
  const int split = blockIdx.x % a.nsplit;
  const int mt = (blockIdx.x / a.nsplit) % a.n_mt;
  const int g = blockIdx.x / (a.nsplit * a.n_mt);
  const int per = (a.nkt + a.nsplit - 1) / a.nsplit;
  const int t0 = split * per, t1 = min(a.nkt, t0 + per);
  if (threadIdx.x == 0) {
    for (int i = 0; i < EA_NK; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 1); }
    mbar_init(&sm.q_full, 1); mbar_init(&sm.q_empty, 1);
    for (int b = 0; b < 2; ++b) { mbar_init(&sm.s_full[b], 1); mbar_init(&sm.s_free[b], 128); }
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
  }
  if (w == 5) { tmem_alloc(&sm.tmem_base, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = sm.tmem_base;
  if (w == 4) {
    if (lane_id() == 0) {
      bool ok = true;
      int cls_cur = -1, qn = 0;
      for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
        const int cls = est_class(a, kt);
        if (cls != cls_cur) {
          ok = mbar_wait(&sm.q_empty, (qn & 1) ^ 1);
          if (!ok) break;
          mbar_expect_tx(&sm.q_full, TILE);
          const int y = (int)(((int64_t)cls * a.hkv + g) * a.m_pad + mt * 128);
          for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.q + hf * 16384, &mq, &sm.q_full, 64 * hf, y);
          ++qn;
          cls_cur = cls;
        }
        const int st = n % EA_NK;
        ok = mbar_wait(&sm.k_empty[st], ((n / EA_NK) & 1) ^ 1);
        if (!ok) break;
        mbar_expect_tx(&sm.k_full[st], TILE);
        const int y = (int)((int64_t)g * a.ld_tokens + (int64_t)kt * 128);
        for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.k[st] + hf * 16384, &mk, &sm.k_full[st], 64 * hf, y);
      }
      if (!ok) { const long long c0 = clock64(); while (clock64() - c0 < 2000000) __nanosleep(1000); }
    }
  } else if (w == 5) {
    if (lane_id() == 0) {
      constexpr uint32_t IDESC = idesc_f16(128, 128, 0);
      bool ok = true;
      int cls_cur = -1, qn = 0;
      for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
        const int cls = est_class(a, kt);
        if (cls != cls_cur) {
          ok = mbar_wait(&sm.q_full, qn & 1);
          if (!ok) break;
          ++qn;
          cls_cur = cls;
        }
        const int st = n % EA_NK, b = n & 1;
        ok = mbar_wait(&sm.k_full[st], (n / EA_NK) & 1) && mbar_wait(&sm.s_free[b], ((n >> 1) & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
          mma_ss(tb + 128u * b, sdesc_sw128(smem_u32(sm.q) + off, 16u, 1024u),
                 sdesc_sw128(smem_u32(sm.k[st]) + off, 16u, 1024u), IDESC, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[b]);
        mma_commit(&sm.k_empty[st]);
        if (kt + 1 >= t1 || est_class(a, kt + 1) != cls) mma_commit(&sm.q_empty);
      }
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0);
    }
  } else {
    // softmax: thread t owns est row m = mt * 128 + t
    const int t = threadIdx.x;
    const int m = mt * 128 + t;
    const int hh = m / 64, r = m % 64;
    const int64_t i = a.r_lo + r;
    const bool live = hh < a.G && i < a.e;
    const uint32_t lb = tb + ((32u * (warp_id() & 3u)) << 16);
    float mx = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
      const int b = n & 1;
      ok = mbar_wait_warp(&sm.s_full[b], (n >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lb + 128u * b + 32u * c, reinterpret_cast<uint32_t*>(x) + 32 * c);
      tc_fence_before();
      mbar_arrive(&sm.s_free[b]);
      const int64_t lim = i - (int64_t)kt * 128;   // keys c <= lim are causal
#pragma unroll
      for (int c = 0; c < 128; ++c) if (c > lim) x[c] = -INFINITY;
      float tmax = x[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) tmax = fmaxf(tmax, x[c]);
      const float mn = fmaxf(mx, tmax);
      if (mn == -INFINITY) continue;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) sum += ex2(x[c] - mn);
      l = l * ex2(mx - mn) + sum;
      mx = mn;
    }
    if (ok) a.part[((int64_t)g * a.n_mt * 128 + m) * a.nsplit + split] = make_float2(live ? mx : -INFINITY, live ? l : 0.f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 5) { __syncwarp(); tmem_dealloc(tb, 256); }
}

// lse2[g][m] = log2 sum over splits of l * 2^max
__global__ void est_merge_a_kernel(const EstArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)a.hkv * a.m_pad) return;
  const int g = (int)(idx / a.m_pad), m = (int)(idx % a.m_pad);
  float M = -INFINITY;
  if (m < a.n_mt * 128) {
    const float2* p = a.part + ((int64_t)g * a.n_mt * 128 + m) * a.nsplit;
    for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, p[s].x);
    if (M != -INFINITY) {
      float sum = 0.f;
      for (int s = 0; s < a.nsplit; ++s) if (p[s].y > 0.f) sum += p[s].y * ex2(p[s].x - M);
      M = M + __log2f(sum);
    }
  }
  a.lse2[idx] = M;
}

// --------------------------------------------------------------------------------------
// Pass B. grid = number of SMs; CTA c processes work units [c*W/grid, (c+1)*W/grid) of
// W = hkv * nkt (group-major), reloading the est-row operand when (group, class) changes.
// --------------------------------------------------------------------------------------
template <int D>
struct EBSmem {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int EST = EB_MAX_ROWS * D * 2;
  alignas(1024) uint8_t est[EST];         // est rows, [half][row][64 halfs] swizzled
  alignas(1024) uint8_t k[EB_NK][TILE];
  float pbuf[EB_GROUPS][EB_STEP][128];    // per epilogue group: EB_STEP rows x 128 keys
  float lse[EB_GROUPS][EB_MAX_ROWS];      // per epilogue group
  uint64_t k_full[EB_NK], k_empty[EB_NK], e_full, e_empty, acc_full, acc_free, drain;
  uint32_t tmem_base;
};

template <int D>
__global__ void __launch_bounds__(EB_THREADS, 1)
est_pass_b_kernel(const __grid_constant__ CUtensorMap me, const __grid_constant__ CUtensorMap mk,
                  const EstArgs a) {
  extern __shared__ uint8_t eb_raw[];
  EBSmem<D>& sm = *reinterpret_cast<EBSmem<D>*>((reinterpret_cast<uintptr_t>(eb_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t TILE = EBSmem<D>::TILE;
  const int w = warp_id();
  const int Mr = a.G * 64;                                  // est rows used as N
  const int64_t W = (int64_t)a.hkv * a.nkt;
  const int64_t u0 = W * blockIdx.x / gridDim.x, u1 = W * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < EB_NK; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 1); }
    mbar_init(&sm.e_full, 1); mbar_init(&sm.e_empty, 1);
    mbar_init(&sm.acc_full, 1); mbar_init(&sm.acc_free, 32 * 4 * EB_GROUPS);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
  }
  constexpr int W_LOAD = 4 * EB_GROUPS, W_MMA = 4 * EB_GROUPS + 1;
  if (w == W_MMA) { tmem_alloc(&sm.tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = sm.tmem_base;
  // the est-row operand is [half][row] with rows of 128 bytes; a 64-row-aligned row offset
  // keeps the 1024-byte swizzle atoms intact
  const uint32_t EST_HALF = (uint32_t)EB_MAX_ROWS * 128u;
  if (w == W_LOAD) {
    if (lane_id() == 0) {
      bool ok = true;
      int key_cur = -1, en = 0;
      for (int64_t u = u0, n = 0; u < u1 && ok; ++u, ++n) {
        const int g = (int)(u / a.nkt), kt = (int)(u % a.nkt);
        const int key = g * 4 + est_class(a, kt);
        if (key != key_cur) {
          ok = mbar_wait(&sm.e_empty, (en & 1) ^ 1);
          if (!ok) break;
          mbar_expect_tx(&sm.e_full, (uint32_t)Mr * D * 2u);
          const int cls = key & 3;
          for (int r0 = 0; r0 < Mr; r0 += 64) {
            const int y = (int)(((int64_t)cls * a.hkv + g) * a.m_pad + r0);
            for (int hf = 0; hf < D / 64; ++hf)
              tma_load_2d(sm.est + hf * EST_HALF + r0 * 128, &me, &sm.e_full, 64 * hf, y);
          }
          ++en;
          key_cur = key;
        }
        const int st = (int)(n % EB_NK);
        ok = mbar_wait(&sm.k_empty[st], ((n / EB_NK) & 1) ^ 1);
        if (!ok) break;
        mbar_expect_tx(&sm.k_full[st], TILE);
        const int y = (int)((int64_t)g * a.ld_tokens + (int64_t)kt * 128);
        for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.k[st] + hf * 16384, &mk, &sm.k_full[st], 64 * hf, y);
      }
      if (!ok) { const long long c0 = clock64(); while (clock64() - c0 < 2000000) __nanosleep(1000); }
    }
  } else if (w == W_MMA) {
    if (lane_id() == 0) {
      bool ok = true;
      int key_cur = -1, en = 0;
      for (int64_t u = u0, n = 0; u < u1 && ok; ++u, ++n) {
        const int g = (int)(u / a.nkt), kt = (int)(u % a.nkt);
        const int key = g * 4 + est_class(a, kt);
        if (key != key_cur) {
          ok = mbar_wait(&sm.e_full, en & 1);
          if (!ok) break;
          ++en;
          key_cur = key;
        }
        const int st = (int)(n % EB_NK);
        ok = mbar_wait(&sm.k_full[st], (n / EB_NK) & 1) && mbar_wait(&sm.acc_free, (n & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        for (int n0 = 0; n0 < Mr; n0 += 256) {
          const int N = Mr - n0 < 256 ? Mr - n0 : 256;
          const uint32_t idesc = idesc_f16(128, N, 0);
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
            const uint32_t eoff = (uint32_t)(kk >> 2) * EST_HALF + (uint32_t)n0 * 128u + (uint32_t)(kk & 3) * 32u;
            mma_ss(tb + (uint32_t)n0, sdesc_sw128(smem_u32(sm.k[st]) + koff, 16u, 1024u),
                   sdesc_sw128(smem_u32(sm.est) + eoff, 16u, 1024u), idesc, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&sm.acc_full);
        mma_commit(&sm.k_empty[st]);
        if (u + 1 >= u1) mma_commit(&sm.e_empty);
        else {
          const int64_t un = u + 1;
          const int keyn = (int)(un / a.nkt) * 4 + est_class(a, (int)(un % a.nkt));
          if (keyn != key) mma_commit(&sm.e_empty);
        }
      }
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0);
    }
  } else {
    // epilogue: group eg = w / 4 handles heads hh = eg, eg + EB_GROUPS, ...; thread owns key
    // lane kl (its warp's TMEM lane quarter)
    const int eg = w >> 2;
    const int kl = 32 * (w & 3) + (int)lane_id();
    const uint32_t lb = tb + ((32u * (w & 3)) << 16);
    const int nR = (int)(a.e - a.r_lo);
    int g_cur = -1;
    bool ok = true;
    for (int64_t u = u0, n = 0; u < u1 && ok; ++u, ++n) {
      const int g = (int)(u / a.nkt), kt = (int)(u % a.nkt);
      if (g != g_cur) {
        // est rows' lse of this group (each epilogue group keeps its own copy)
        named_bar_sync(1 + eg, 128);
        for (int m = kl; m < Mr; m += 128) sm.lse[eg][m] = a.lse2[(int64_t)g * a.m_pad + m];
        named_bar_sync(1 + eg, 128);
        g_cur = g;
      }
      ok = named_bar_and(1 + eg, 128, mbar_wait(&sm.acc_full, n & 1));
      if (!ok) break;
      tc_fence_after();
      const int64_t j = (int64_t)kt * 128 + kl;              // this thread's key
      for (int hh = eg; hh < a.G; hh += EB_GROUPS) {
        float vsum = 0.f;
        float acc0 = 0.f, acc1 = 0.f;   // slash sums for U = kl and U = kl + 128
        for (int rh = 0; rh < 64 / EB_STEP; ++rh) {
          uint32_t rr[EB_STEP];
          tmem_ld16(lb + (uint32_t)(hh * 64 + rh * EB_STEP), rr);
#pragma unroll
          for (int c = 0; c < EB_STEP; ++c) {
            const int r = rh * EB_STEP + c;
            const int64_t i = a.r_lo + r;
            float p = 0.f;
            if (r < nR && j <= i) p = ex2(__uint_as_float(rr[c]) - sm.lse[eg][hh * 64 + r]);
            vsum += p;
            sm.pbuf[eg][c][kl] = p;
          }
          named_bar_sync(1 + eg, 128);
          // U = EB_STEP rh + c - k + 127 for row c of this step and key k of the tile
#pragma unroll 4
          for (int c = 0; c < EB_STEP; ++c) {
            const int k0 = EB_STEP * rh + c + 127 - kl;
            if (k0 >= 0 && k0 < 128) acc0 += sm.pbuf[eg][c][k0];
            const int k1 = k0 - 128;
            if (k1 >= 0 && k1 < 128) acc1 += sm.pbuf[eg][c][k1];
          }
          named_bar_sync(1 + eg, 128);
        }
        const int h = g * a.G + hh;
        if (j < a.e) a.vert[(int64_t)h * a.ld + j] = vsum;
        float* sp = a.slash_part + ((int64_t)h * a.nkt + kt) * EB_U;
        sp[kl] = acc0;
        if (kl + 128 < EB_U) sp[kl + 128] = acc1;
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == W_MMA) { __syncwarp(); tmem_dealloc(tb, 512); }
}

// slash[h][o] = sum of the (at most two) key tiles' partials that contain offset o, in
// ascending tile order.
__global__ void est_slash_reduce_kernel(const EstArgs a, float* __restrict__ slash) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)a.hq * a.e) return;
  const int h = (int)(idx / a.e);
  const int64_t o = idx % a.e;
  // tile kt holds U = o - (r_lo - 128 kt - 127) in [0, 190]
  int64_t kmin = a.r_lo - 127 - o;
  kmin = kmin <= 0 ? 0 : (kmin + 127) / 128;
  int64_t kmax = a.r_lo + 63 - o;
  if (kmax < 0) { slash[(int64_t)h * a.ld + o] = 0.f; return; }
  kmax = kmax / 128;
  if (kmax > a.nkt - 1) kmax = a.nkt - 1;
  float s = 0.f;
  for (int64_t kt = kmin; kt <= kmax; ++kt) {
    const int64_t U = o - (a.r_lo - 128 * kt - 127);
    if (U >= 0 && U < 191) s += a.slash_part[((int64_t)h * a.nkt + kt) * EB_U + U];
  }
  slash[(int64_t)h * a.ld + o] = s;
}

}  // namespace q1m
