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
//  pass A: rows as M (128 rows per tile), keys as N; per row a sum l of 2^(x - m) against a
//          reference m kept from the row's first tile, over a range of key tiles; partial
//          (m, l) per split, merged into the row's log2-sum-exp2.
//  pass B: keys as M (128 keys per tile), est rows as N (<= 448 TMEM columns, in two
//          accumulators: heads 0..3 and heads 4..6, so the MMA of one overlaps the epilogue
//          of the other). One epilogue warp per (pair of heads, 32-key quarter), the two
//          heads' values packed in float2 so that every add, shuffle and exponential
//          argument serves both; each thread owns one key, so its vertical scores are
//          thread-local sums over rows. Slash sums are sums along diagonals: for each group of
//          8 rows, every lane fetches by warp shuffles the values of its two diagonals from
//          the warp's 32 keys and sums them; the four quarters' diagonal partials are added
//          per tile (192 offsets) and the two tiles that touch each offset are summed later,
//          always in the same order, so the scores are deterministic.
#pragma once

#include "q1m_device.cuh"

namespace q1m {

constexpr int EA_THREADS = 320;   // warps 0-7 softmax (two per TMEM lane quarter), 8 loader, 9 MMA
constexpr int EA_NK = 2;
constexpr int EB_PAIRS = 4;                            // head pairs (0,1) (2,3) (4,5) (6)
constexpr int EB_THREADS = 32 * (4 * EB_PAIRS + 2);    // warps 0-15 epilogue, 16 loader, 17 MMA
constexpr int EB_STEP = 8;        // est rows per epilogue step
constexpr int EB_ACC0_HEADS = 4;  // accumulator 0 holds heads 0..3, accumulator 1 heads 4..6
constexpr int EB_MAX_ROWS = 448;
constexpr int EB_U = 192;         // offsets per key tile (64 + 128 - 1 used)
constexpr int EB_DQ = 96;         // diagonal partials of one key quarter (32 + 64 - 1 used)

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

// 64 keys of a pass A row: the log2-sum-exp2 of row values x[0..63] (log2-scaled logits)
// added into (mx, l), which stands for l * 2^mx. MASKED: keys c > lim are not causal for the
// row.
//
// The sums are fp32, so the reference mx need not be the running maximum: any mx with every
// 2^(x - mx) in range gives the same l * 2^mx up to rounding. The values are therefore
// exponentiated against the current mx first. The tile is redone against its own maximum
// only when that sum is infinite, NaN or above 2^64: on a row's first tile, where mx = -inf,
// or when values lie far above mx. A row's accumulated l then stays below 2^77, far inside
// fp32.
template <bool MASKED>
__device__ __forceinline__ void est_a_half(float (&x)[64], int64_t lim, float& mx, float& l) {
  if (MASKED) {
#pragma unroll
    for (int c = 0; c < 64; ++c) if (c > lim) x[c] = -INFINITY;
  }
  if (mx != -INFINITY) {
    const uint64_t nm = f2_pack(-mx, -mx);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float d0, d1;
      f2_unpack(f2_add(f2_pack(x[2 * c], x[2 * c + 1]), nm), d0, d1);
      acc[c & 3] = f2_add(acc[c & 3], f2_pack(ex2(d0), ex2(d1)));
    }
    float s0, s1, s2, s3;
    f2_unpack(f2_add(acc[0], acc[1]), s0, s1);
    f2_unpack(f2_add(acc[2], acc[3]), s2, s3);
    const float sum = (s0 + s1) + (s2 + s3);
    if (sum <= 0x1p64f) {                                    // false for +inf and NaN
      l += sum;
      return;
    }
  }
  // maximum: eight independent chains, then a tree
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
  for (int c = 8; c < 64; c += 8)
#pragma unroll
    for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], x[c + k]);
#pragma unroll
  for (int wdt = 4; wdt >= 1; wdt /= 2)
#pragma unroll
    for (int k = 0; k < wdt; ++k) m8[k] = fmaxf(m8[k], m8[k + wdt]);
  const float mn = fmaxf(mx, m8[0]);
  if (mn == -INFINITY) return;
  // 2^(x - mn): packed subtractions, four independent packed sums
  const uint64_t nmn = f2_pack(-mn, -mn);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    float d0, d1;
    f2_unpack(f2_add(f2_pack(x[2 * c], x[2 * c + 1]), nmn), d0, d1);
    acc[c & 3] = f2_add(acc[c & 3], f2_pack(ex2(d0), ex2(d1)));
  }
  float s0, s1, s2, s3;
  f2_unpack(f2_add(acc[0], acc[1]), s0, s1);
  f2_unpack(f2_add(acc[2], acc[3]), s2, s3);
  l = l * ex2(mx - mn) + ((s0 + s1) + (s2 + s3));
  mx = mn;
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
  float2 half_part[128];                  // (max, sum) of each row over the key columns 64..127
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
    for (int b = 0; b < 2; ++b) { mbar_init(&sm.s_full[b], 1); mbar_init(&sm.s_free[b], 256); }
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
  }
  if (w == 9) { tmem_alloc(&sm.tmem_base, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = sm.tmem_base;
  if (w == 8) {
    if (lane_id() == 0) {
      bool ok = true;
      int cls_cur = -1, qn = 0;
      for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
        const int cls = est_class(a, kt);
        if (cls != cls_cur) {
          ok = mbar_wait_sleep(&sm.q_empty, (qn & 1) ^ 1);
          if (!ok) break;
          mbar_expect_tx(&sm.q_full, TILE);
          const int y = (int)(((int64_t)cls * a.hkv + g) * a.m_pad + mt * 128);
          for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.q + hf * 16384, &mq, &sm.q_full, 64 * hf, y);
          ++qn;
          cls_cur = cls;
        }
        const int st = n % EA_NK;
        ok = mbar_wait_sleep(&sm.k_empty[st], ((n / EA_NK) & 1) ^ 1);
        if (!ok) break;
        mbar_expect_tx(&sm.k_full[st], TILE);
        const int y = (int)((int64_t)g * a.ld_tokens + (int64_t)kt * 128);
        for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.k[st] + hf * 16384, &mk, &sm.k_full[st], 64 * hf, y);
      }
      if (!ok) { const long long c0 = clock64(); while (clock64() - c0 < 2000000) __nanosleep(1000); }
    }
  } else if (w == 9) {
    if (lane_id() == 0) {
      constexpr uint32_t IDESC = idesc_f16(128, 128, 0);
      bool ok = true;
      int cls_cur = -1, qn = 0;
      for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
        const int cls = est_class(a, kt);
        if (cls != cls_cur) {
          ok = mbar_wait_sleep(&sm.q_full, qn & 1);
          if (!ok) break;
          ++qn;
          cls_cur = cls;
        }
        const int st = n % EA_NK, b = n & 1;
        ok = mbar_wait_sleep(&sm.k_full[st], (n / EA_NK) & 1) && mbar_wait_sleep(&sm.s_free[b], ((n >> 1) & 1) ^ 1);
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
      mbar_wait_sleep(&sm.drain, 0);
    }
  } else {
    // softmax: warp w takes the rows of TMEM lane quarter w & 3 (thread t owns est row
    // m = mt * 128 + t) and the key columns [64 ch, 64 ch + 64) of each tile, ch = w >> 2; the
    // two column halves' (max, sum) of a row are merged once at the end
    const int ch = w >> 2;
    const int t = threadIdx.x & 127;
    const int m = mt * 128 + t;
    const int hh = m / 64, r = m % 64;
    const int64_t i = a.r_lo + r;
    const bool live = hh < a.G && i < a.e;
    const uint32_t lb = tb + ((32u * (warp_id() & 3u)) << 16) + 64u * (uint32_t)ch;
    float mx = -INFINITY, l = 0.f;
    bool ok = true;
    // a warp whose 32 est rows are all padding (past the group's G x 64 rows) only frees the
    // accumulator buffers
    const bool warp_live = (mt * 128 + 32 * (int)(warp_id() & 3u)) / 64 < a.G;
    for (int kt = t0, n = 0; kt < t1 && ok; ++kt, ++n) {
      const int b = n & 1;
      ok = mbar_wait_sleep_warp(&sm.s_full[b], (n >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (!warp_live) {
        tc_fence_before();
        mbar_arrive(&sm.s_free[b]);
        continue;
      }
      float x[64];
      tmem_ld64(lb + 128u * b, reinterpret_cast<uint32_t*>(x));
      tc_fence_before();
      mbar_arrive(&sm.s_free[b]);
      const int64_t k0 = (int64_t)kt * 128 + 64 * ch;           // first key of this half
      if (k0 + 63 > a.r_lo) est_a_half<true>(x, i - k0, mx, l);
      else est_a_half<false>(x, 0, mx, l);
    }
    // merge the two column halves of each row: warps 4-7 hand theirs to warps 0-3
    if (ch == 1) sm.half_part[t] = make_float2(mx, l);
    ok = named_bar_and(1, 256, ok);
    if (ok && ch == 0) {
      const float2 o = sm.half_part[t];
      const float M = fmaxf(mx, o.x);
      float L = 0.f;
      if (M != -INFINITY) L = (l > 0.f ? l * ex2(mx - M) : 0.f) + (o.y > 0.f ? o.y * ex2(o.x - M) : 0.f);
      a.part[((int64_t)g * a.n_mt * 128 + m) * a.nsplit + split] = make_float2(live ? M : -INFINITY, live ? L : 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 9) { __syncwarp(); tmem_dealloc(tb, 256); }
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
  alignas(1024) uint8_t k[TILE];          // one key tile (the epilogue covers its reload)
  float2 dsum[EB_PAIRS][4][EB_DQ];        // per head pair and key quarter: diagonal partials
  float nlse[2 * EB_PAIRS][64];           // per head and est row: -(log2-sum-exp2)
  uint64_t k_full, k_empty, e_full, e_empty, acc_full[2], acc_free[2], drain;
  uint32_t tmem_base;
};

// One element of a diagonal sum: v (a packed pair of row C of another lane's key) goes into
// da when C <= l, else into db (predicated, no branch).
template <int C>
__device__ __forceinline__ void diag_add(uint64_t& da, uint64_t& db, uint64_t v, int l) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.le.s32 q, %3, %4;\n\t"
      "@q add.rn.f32x2 %0, %0, %2;\n\t"
      "@!q add.rn.f32x2 %1, %1, %2;\n\t}"
      : "+l"(da), "+l"(db)
      : "l"(v), "n"(C), "r"(l));
}

// Row C of the key of lane (C - 1 - l) mod 32, fetched by a shuffle into lane l: it lies on
// warp diagonal d = C - key + 31, which is d = l when C <= l and d = l + 32 when C > l.
template <int C>
__device__ __forceinline__ void diag_fetch_add(uint64_t& da, uint64_t& db, uint64_t p, int l) {
  float x, y;
  f2_unpack(p, x, y);
  const int src = (C - 1 - l) & 31;
  x = __shfl_sync(0xffffffffu, x, src);
  y = __shfl_sync(0xffffffffu, y, src);
  diag_add<C>(da, db, f2_pack(x, y), l);
}

template <int C>
__device__ __forceinline__ void diag_all(uint64_t& da, uint64_t& db, const uint64_t* pp, int l) {
  if constexpr (C < EB_STEP) {
    diag_fetch_add<C>(da, db, pp[C], l);
    diag_all<C + 1>(da, db, pp, l);
  }
}

// One key tile of a pass B epilogue warp: p = 2^(s - lse) for the warp's 32 keys and its
// head pair's 64 est rows, their vertical sums (returned packed (A, B)) and the diagonal
// partials added into ds. MASKED: the tile reaches the estimator rows (keys after a row are
// not causal) or the chunk has fewer than 64 rows.
template <int D, bool TWO, bool MASKED>
__device__ __forceinline__ uint64_t est_b_tile(EBSmem<D>& sm, const EstArgs& a, int pi, int hA, int half,
                                               uint32_t lbA, float2* ds, int l, int64_t j, int nR) {
  uint64_t vs = 0ull;                                       // vertical sums (A, B)
#pragma unroll 1
  for (int s = 0; s < 64 / EB_STEP; ++s) {
    uint32_t ra[EB_STEP], rb[EB_STEP];
    static_assert(EB_STEP == 8, "one 8-column TMEM load per head and step");
    tmem_ld8(lbA + (uint32_t)(s * EB_STEP), ra);
    if (TWO) tmem_ld8(lbA + 64u + (uint32_t)(s * EB_STEP), rb);
    if (s == 64 / EB_STEP - 1) {
      // every TMEM read of this tile is done: the MMA may overwrite the accumulator
      tc_fence_before();
      __syncwarp();
      if (l == 0) mbar_arrive(&sm.acc_free[half]);
    }
    // row pairs (c, c + 1) of one head are adjacent registers: packed adds on them, then
    // each exponential's result is paired with the other head's for the shuffles
    const float4* nA4 = reinterpret_cast<const float4*>(&sm.nlse[hA][s * EB_STEP]);
    const float4* nB4 = reinterpret_cast<const float4*>(&sm.nlse[hA + 1][s * EB_STEP]);
    uint64_t pp[EB_STEP];
#pragma unroll
    for (int c4 = 0; c4 < EB_STEP / 4; ++c4) {
      const float4 na = nA4[c4];
      float dA[4], dB[4];
      f2_unpack(f2_add(f2_pack(__uint_as_float(ra[4 * c4]), __uint_as_float(ra[4 * c4 + 1])), f2_pack(na.x, na.y)), dA[0], dA[1]);
      f2_unpack(f2_add(f2_pack(__uint_as_float(ra[4 * c4 + 2]), __uint_as_float(ra[4 * c4 + 3])), f2_pack(na.z, na.w)), dA[2], dA[3]);
      if (TWO) {
        const float4 nb = nB4[c4];
        f2_unpack(f2_add(f2_pack(__uint_as_float(rb[4 * c4]), __uint_as_float(rb[4 * c4 + 1])), f2_pack(nb.x, nb.y)), dB[0], dB[1]);
        f2_unpack(f2_add(f2_pack(__uint_as_float(rb[4 * c4 + 2]), __uint_as_float(rb[4 * c4 + 3])), f2_pack(nb.z, nb.w)), dB[2], dB[3]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = 4 * c4 + k;
        float pA = ex2(dA[k]);
        float pB = TWO ? ex2(dB[k]) : 0.f;
        if (MASKED) {
          const int r = s * EB_STEP + c;
          if (r >= nR || j > a.r_lo + r) { pA = 0.f; pB = 0.f; }
        }
        pp[c] = f2_pack(pA, pB);
        vs = f2_add(vs, pp[c]);
      }
    }
    // diagonal sums across the warp's 32 keys: lane l sums warp diagonal l (rows c <= l)
    // and l + 32 (rows c > l), rows in ascending order
    uint64_t da = 0ull, db = 0ull;
    diag_all<0>(da, db, pp, l);
    // warp diagonal d of step s is quarter offset EB_STEP s + d (tile offset
    // U = that + 96 - 32 q)
    uint64_t* dsa = reinterpret_cast<uint64_t*>(&ds[s * EB_STEP + l]);
    *dsa = f2_add(*dsa, da);
    if (l < EB_STEP - 1) {
      uint64_t* dsb = reinterpret_cast<uint64_t*>(&ds[s * EB_STEP + l + 32]);
      *dsb = f2_add(*dsb, db);
    }
    __syncwarp();
  }
  return vs;
}

// Pass B epilogue warp: heads hA = 2 pi and, when TWO, hB = 2 pi + 1, key quarter q (the
// warp's TMEM lane quarter); lane l owns key 32 q + l and keeps the two heads' values packed
// (A, B), so one packed add, shared-memory access or exponential argument serves both.
template <int D, bool TWO>
__device__ __forceinline__ void est_b_epilogue(EBSmem<D>& sm, const EstArgs& a, int w, uint32_t tb,
                                               int64_t u0, int64_t u1) {
  const int pi = w >> 2, q = w & 3;
  const int l = (int)lane_id();
  const int hA = 2 * pi;
  const int half = hA < EB_ACC0_HEADS ? 0 : 1;
  const int bar = 1 + pi;                                   // named barrier of the pair's 4 warps
  const uint32_t lbA = tb + ((32u * (uint32_t)q) << 16) + (uint32_t)(hA * 64);
  float2* ds = sm.dsum[pi][q];
  const int nR = (int)(a.e - a.r_lo);
  int g = (int)(u0 / a.nkt), kt = (int)(u0 % a.nkt);
  int g_cur = -1;
  bool ok = true;
  for (int i = l; i < EB_DQ; i += 32) ds[i] = make_float2(0.f, 0.f);
  for (int64_t u = u0, n = 0; u < u1 && ok; ++u, ++n) {
    if (g != g_cur) {
      // -lse of the pair's est rows, (A, B) per row (each pair keeps its own copy)
      named_bar_sync(bar, 128);
      {
        const int t = 32 * q + l, hh = hA + (t >> 6), m = t & 63;
        sm.nlse[hh][m] = hh < a.G ? -a.lse2[(int64_t)g * a.m_pad + hh * 64 + m] : 0.f;
      }
      named_bar_sync(bar, 128);
      g_cur = g;
    }
    const bool okw = mbar_wait_sleep_warp(&sm.acc_full[half], (uint32_t)(n & 1));
    const int64_t j = (int64_t)kt * 128 + 32 * q + l;       // this thread's key
    if (okw) {
      tc_fence_after();
      // the tile reaches the estimator rows (causal mask), or the chunk has fewer rows
      const bool masked = (int64_t)kt * 128 + 127 >= a.r_lo || nR < 64;
      const uint64_t vs = masked ? est_b_tile<D, TWO, true>(sm, a, pi, hA, half, lbA, ds, l, j, nR)
                                 : est_b_tile<D, TWO, false>(sm, a, pi, hA, half, lbA, ds, l, j, nR);
      const int64_t hgA = (int64_t)g * a.G + hA;
      float vA, vB;
      f2_unpack(vs, vA, vB);
      if (j < a.e) {
        a.vert[hgA * a.ld + j] = vA;
        if (TWO) a.vert[(hgA + 1) * a.ld + j] = vB;
      }
    }
    // the four quarters' partials of this pair, in quarter order, into the tile's offsets
    ok = named_bar_and(bar, 128, okw);
    if (!ok) break;
    const int64_t hgA = (int64_t)g * a.G + hA;
    float* spA = a.slash_part + (hgA * a.nkt + kt) * EB_U;
    float* spB = spA + (int64_t)a.nkt * EB_U;
    for (int U = 32 * q + l; U < EB_U; U += 128) {
      uint64_t acc = 0ull;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int idx = U - 96 + 32 * qq;
        if (idx >= 0 && idx < EB_DQ - 1)
          acc = f2_add(acc, *reinterpret_cast<const uint64_t*>(&sm.dsum[pi][qq][idx]));
      }
      float xA, xB;
      f2_unpack(acc, xA, xB);
      spA[U] = xA;
      if (TWO) spB[U] = xB;
    }
    named_bar_sync(bar, 128);
    for (int i = l; i < EB_DQ; i += 32) ds[i] = make_float2(0.f, 0.f);
    if (++kt == a.nkt) { kt = 0; ++g; }
  }
}

template <int D>
__global__ void __launch_bounds__(EB_THREADS, 1)
est_pass_b_kernel(const __grid_constant__ CUtensorMap me, const __grid_constant__ CUtensorMap mk,
                  const EstArgs a) {
  extern __shared__ uint8_t eb_raw[];
  EBSmem<D>& sm = *reinterpret_cast<EBSmem<D>*>((reinterpret_cast<uintptr_t>(eb_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t TILE = EBSmem<D>::TILE;
  constexpr int W_LOAD = 4 * EB_PAIRS, W_MMA = 4 * EB_PAIRS + 1;
  const int w = warp_id();
  const int Mr = a.G * 64;                                  // est rows used as N
  const int h0 = a.G < EB_ACC0_HEADS ? a.G : EB_ACC0_HEADS;  // heads in accumulator 0
  const int h1 = a.G - h0;                                  // heads in accumulator 1
  const int p0 = (h0 + 1) / 2, p1 = (h1 + 1) / 2;           // head pairs per accumulator
  const int64_t W = (int64_t)a.hkv * a.nkt;
  const int64_t u0 = W * blockIdx.x / gridDim.x, u1 = W * (blockIdx.x + 1) / gridDim.x;
  if (threadIdx.x == 0) {
    mbar_init(&sm.k_full, 1); mbar_init(&sm.k_empty, 1);
    mbar_init(&sm.e_full, 1); mbar_init(&sm.e_empty, 1);
    mbar_init(&sm.acc_full[0], 1); mbar_init(&sm.acc_full[1], 1);
    mbar_init(&sm.acc_free[0], 4 * p0); mbar_init(&sm.acc_free[1], p1 > 0 ? 4 * p1 : 1);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
  }
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
          ok = mbar_wait_sleep(&sm.e_empty, (en & 1) ^ 1);
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
        ok = mbar_wait_sleep(&sm.k_empty, (uint32_t)(n & 1) ^ 1u);
        if (!ok) break;
        mbar_expect_tx(&sm.k_full, TILE);
        const int y = (int)((int64_t)g * a.ld_tokens + (int64_t)kt * 128);
        for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.k + hf * 16384, &mk, &sm.k_full, 64 * hf, y);
      }
      if (!ok) { const long long c0 = clock64(); while (clock64() - c0 < 2000000) __nanosleep(1000); }
    }
  } else if (w == W_MMA) {
    if (lane_id() == 0) {
      bool ok = true;
      int key_cur = -1, en = 0;
      // S[key][row] for est rows [r0, r0 + N) into TMEM columns [r0, r0 + N)
      auto issue = [&](int r0, int N) {
        const uint32_t idesc = idesc_f16(128, N, 0);
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
          const uint32_t eoff = (uint32_t)(kk >> 2) * EST_HALF + (uint32_t)r0 * 128u + (uint32_t)(kk & 3) * 32u;
          mma_ss(tb + (uint32_t)r0, sdesc_sw128(smem_u32(sm.k) + koff, 16u, 1024u),
                 sdesc_sw128(smem_u32(sm.est) + eoff, 16u, 1024u), idesc, kk > 0 ? 1u : 0u);
        }
      };
      for (int64_t u = u0, n = 0; u < u1 && ok; ++u, ++n) {
        const int g = (int)(u / a.nkt), kt = (int)(u % a.nkt);
        const int key = g * 4 + est_class(a, kt);
        if (key != key_cur) {
          ok = mbar_wait_sleep(&sm.e_full, en & 1);
          if (!ok) break;
          ++en;
          key_cur = key;
        }
        const uint32_t par = (uint32_t)(n & 1);
        ok = mbar_wait_sleep(&sm.k_full, par) && mbar_wait_sleep(&sm.acc_free[0], par ^ 1u);
        if (!ok) break;
        tc_fence_after();
        issue(0, h0 * 64);
        mma_commit(&sm.acc_full[0]);
        if (h1 > 0) {
          ok = mbar_wait_sleep(&sm.acc_free[1], par ^ 1u);
          if (!ok) break;
          tc_fence_after();
          issue(h0 * 64, h1 * 64);
          mma_commit(&sm.acc_full[1]);
        }
        mma_commit(&sm.k_empty);
        if (u + 1 >= u1) mma_commit(&sm.e_empty);
        else {
          const int64_t un = u + 1;
          const int keyn = (int)(un / a.nkt) * 4 + est_class(a, (int)(un % a.nkt));
          if (keyn != key) mma_commit(&sm.e_empty);
        }
      }
      mma_commit(&sm.drain);
      mbar_wait_sleep(&sm.drain, 0);
    }
  } else if (2 * (w >> 2) < a.G) {
    if (2 * (w >> 2) + 1 < a.G) est_b_epilogue<D, true>(sm, a, w, tb, u0, u1);
    else est_b_epilogue<D, false>(sm, a, w, tb, u0, u1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == W_MMA) { __syncwarp(); tmem_dealloc(tb, 512); }
}

// slash[h][o] = sum of the (at most two) key tiles' partials that contain offset o, in
// ascending tile order. Tile kt holds offset o at U = o - r_lo + 128 kt + 127 in [0, 190], so
// the tiles are kt1 = floor((r_lo + 63 - o) / 128) and kt1 - 1. grid = (ceil(e / 256), hq).
__global__ void est_slash_reduce_kernel(const EstArgs a, float* __restrict__ slash) {
  const int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y;
  if (o >= a.e) return;
  const int64_t kt1 = (a.r_lo + 63 - o) >> 7;               // r_lo + 63 - o >= 0 (o <= e - 1)
  const int64_t U1 = o - a.r_lo + 128 * kt1 + 127;          // in [63, 190]
  const float* part = a.slash_part + (int64_t)h * a.nkt * EB_U;
  float s = 0.f;
  if (kt1 >= 1 && kt1 - 1 < a.nkt && U1 >= 128) s += part[(kt1 - 1) * EB_U + (U1 - 128)];
  if (kt1 < a.nkt && U1 < 191) s += part[kt1 * EB_U + U1];
  slash[(int64_t)h * a.ld + o] = s;
}

}  // namespace q1m
