// attn_tc.cuh — block-sparse DCA flash attention on the 5th-generation tensor cores.
//
// "Qwen2.5-1M Technical Report" paper review (xllm-io), section 四: DCA's three patterns
// (intra / successive / inter chunk), MInference vertical-slash sparse attention with key
// tokens chosen per prefill chunk, and the sparse attention kernel (Figure 7). That
// kernel was written for A100; this one is designed for sm_100a:
//
//  * A work item is (Q head h, a pair of adjacent 128-row query blocks, DCA pattern x).
//    Pattern x (0 intra, 1 successive, 2 inter) selects the key blocks of that pattern; all
//    of them use the same rotated query view x, so each item loads one Q view per query
//    block, and the item writes a partial result (o, log2-sum-exp2) that a separate kernel
//    merges.
//  * The two query blocks of an item ("slots") share one stream of K/V tiles: the union of
//    their key-block lists, each tile flagged with the slots that use it. Slot 1 is the
//    block right after slot 0, so in dense mode the lists coincide and in sparse mode
//    (Toeplitz block masks) they mostly do.
//  * Each item walks its key blocks from a start taken from a global count of the tiles all
//    CTAs have issued (wrapping around its range; for intra items the count is first taken
//    modulo the DCA chunk's block count), so CTAs that stream the same K/V range stay at
//    about the same tile and share it in L2 (see g_k3_cursor); deterministic mode starts
//    every walk at its first block.
//  * Warp roles: warps 0-3 softmax of slot 0, warps 4-7 softmax of slot 1, warp 8 loads
//    (TMA for key blocks, cp.async gathers for residual vertical columns), warp 9 issues
//    tcgen05.mma and owns tensor memory, warp 10 loads V tiles, warp 11 idles; the softmax
//    warpgroups take registers from the third warpgroup (setmaxnreg) to hold a whole S row.
//  * Tensor memory per slot: S (128 fp32 columns), O (D fp32 columns); the softmax writes
//    P as packed fp16 over the first 64 columns of S and the PV product reads it from
//    tensor memory (A operand), with V as an MN-major shared-memory operand.
//  * The MMA warp issues, per tile: [PV of the slot's previous tile] then QK^T of this
//    tile, alternating slots, so one slot's softmax overlaps the other slot's MMAs.
//  * Online softmax in base 2 with a lazy rescale: O (in TMEM) and l are rescaled only
//    when a row's running maximum grows by more than 2^8.
#pragma once

#include "q1m_device.cuh"

namespace q1m {

constexpr int K3_NK = 2;        // K stages
constexpr int K3_NV = 2;        // V stages
constexpr int K3_THREADS = 384;   // 3 warpgroups: softmax slot 0, softmax slot 1, loader + MMA
// register split (setmaxnreg): launch 384 x 168 = 64,512 = 2 x 128 x 192 + 128 x 120 (no spills)
constexpr int K3_REGS_SOFTMAX = 192;
constexpr int K3_REGS_OTHER = 120;
constexpr float K3_RESCALE_THRESHOLD = 8.0f;
// exponentials of K3_POLY_PAIRS_OF_8 of every 8 pairs run on the FMA pipe (ex2_poly2), the
// rest on the MUFU; measured on B200 with both slots' softmax warps active, 2 to 4 of 8 on the
// FMA pipe made the kernel 10-35% slower, so the default is 0
constexpr int K3_POLY_PAIRS_OF_8 = 0;
// P overwrites the first half of S (columns 0..63), so the slot's next QK^T must not write
// S before the PV MMA that reads P has completed. The PTX ISA guarantees that two
// tcgen05.mma execute in issue order only when they share the accumulator and the shape
// (its tcgen05 "pipelined instructions" pairs); QK^T (accumulator S) and PV (accumulator O)
// do not, so the MMA warp waits for the PV's commit before it issues the next QK^T of the
// slot. Measured on B200 this wait costs 3.5-4% of the kernel's time; issuing QK^T as two
// N = 64 halves, the half clear of P first, to hide it was 15-17% slower (N = 64 MMAs re-read
// the Q tile from shared memory for each half).

struct K3Args {
  int64_t s0, e;
  int hq, hkv, G;
  int64_t L;             // DCA chunk length in tokens (multiple of 128)
  int nqb, npair;
  int64_t ld_rows, ld_tokens;
  const uint32_t* mask;  // [hq][nqb][nkw] or null (dense)
  const int32_t* resid;  // [hq][nqb][nvcap]
  const int32_t* cnt;    // [hq][nqb][8]
  int nkw, nvcap;
  const uint16_t* k_rot;
  const uint16_t* v16;
  float* o_part;         // [3][hq][ld_rows][D]
  float* lse_part;       // [3][hq][ld_rows]
  const int32_t* units;  // sorted (pair << 2 | pattern)
  const int32_t* n_units;
  int aligned;           // 1: walks start at the global cursor; 0: at lo (deterministic order)
};

struct K3Item {
  int h, g, x;
  int qb[2];
  int64_t B[2];
  int lo[2], hi[2];      // key-block range of each slot in segment x (lo > hi: empty)
  int ntiles[2];
  int nres[2], res_off[2];
  bool valid[2];
};

// Key-block range of DCA pattern x for global query block B (Lb blocks per DCA chunk,
// cb = B / Lb): intra (0) = chunk cb up to the diagonal block B, successive (1) = chunk
// cb - 1, inter (2) = chunks <= cb - 2. Empty ranges have lo > hi.
__device__ __forceinline__ void seg_range(int64_t B, int x, int64_t Lb, int* lo, int* hi) {
  const int64_t cb = B / Lb;
  if (x == 0) { *lo = (int)(cb * Lb); *hi = (int)B; }
  else if (x == 1) { if (cb >= 1) { *lo = (int)((cb - 1) * Lb); *hi = (int)(cb * Lb - 1); } else { *lo = 1; *hi = 0; } }
  else { if (cb >= 2) { *lo = 0; *hi = (int)((cb - 1) * Lb - 1); } else { *lo = 1; *hi = 0; } }
}

__device__ __forceinline__ K3Item k3_item(const K3Args& a, int it) {
  K3Item r;
  const int u = a.units[it / a.hq];
  r.h = it % a.hq;
  r.g = r.h / a.G;
  r.x = u & 3;
  const int m = u >> 2;
  const int64_t Lb = a.L / 128;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    r.qb[s] = 2 * m + s;
    r.valid[s] = r.qb[s] < a.nqb;
    r.B[s] = a.s0 / 128 + r.qb[s];
    r.lo[s] = 1; r.hi[s] = 0; r.ntiles[s] = 0; r.nres[s] = 0; r.res_off[s] = 0;
    if (!r.valid[s]) continue;
    seg_range(r.B[s], r.x, Lb, &r.lo[s], &r.hi[s]);
    if (a.mask == nullptr) {
      r.ntiles[s] = r.hi[s] >= r.lo[s] ? r.hi[s] - r.lo[s] + 1 : 0;
    } else {
      const int32_t* c = a.cnt + ((int64_t)r.h * a.nqb + r.qb[s]) * 8;
      r.nres[s] = c[3 + r.x];
      // the ascending residual list holds inter columns, then successive, then intra
      r.res_off[s] = (r.x < 2 ? c[5] : 0) + (r.x < 1 ? c[4] : 0);
      r.ntiles[s] = c[r.x] + (r.nres[s] + 127) / 128;
    }
  }
  return r;
}

__device__ __forceinline__ uint32_t range_bits(int w, int lo, int hi) {
  if (hi < lo) return 0u;
  const int b0 = 32 * w, b1 = b0 + 31;
  if (hi < b0 || lo > b1) return 0u;
  const int l = lo > b0 ? lo - b0 : 0;
  const int h = hi < b1 ? hi - b0 : 31;
  const uint32_t upto = h == 31 ? 0xFFFFFFFFu : ((1u << (h + 1)) - 1u);
  return upto & ~((1u << l) - 1u);
}

template <int D>
struct K3Smem {
  static constexpr int TILE = 128 * D * 2;  // bytes of one 128-row fp16 tile
  alignas(1024) uint8_t q[2][TILE];
  alignas(1024) uint8_t k[K3_NK][TILE];
  alignas(1024) uint8_t v[K3_NV][TILE];
  int desc[K3_NK][4];       // flags, diag mask, ncols (gathers; 128 for blocks), unused (K stages)
  int meta[2];              // per-slot mailbox written by the MMA warp before its arrive
  uint64_t k_full[K3_NK], k_empty[K3_NK], v_full[K3_NV], v_empty[K3_NV];
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_done[2], pv_done[2];
  uint64_t drain;
  int walk_start[2];        // first key block of each item's walk (K loader -> V loader)
  uint64_t start_full[2], start_empty[2];
  uint32_t tmem_base;
};

// Free-running count of the K tiles all CTAs have issued. An item's walk over its key blocks
// starts at the block this count divided by the number of CTAs points to (wrapping around
// its range): every CTA's position then follows the same global clock, so CTAs that stream
// the same K/V range read about the same tile at the same time and it is fetched from DRAM
// about once and served from L2 after that. Measured on B200 at 7B@1M under the power cap:
// 8-12% faster per prefill chunk, the DRAM power saved going to the SM clock. The online
// softmax is exact in any tile order up to rounding, but the rounding (fp32 sums, and P in
// fp16 against the running maximum) follows the order, which now depends on timing: runs can
// differ at that level (about 1e-4 relative). With `aligned` off every walk starts at lo and
// runs are bit-identical.
__device__ unsigned long long g_k3_cursor;

// --------------------------------------------------------------------------------------
// Loader warps. Two warps walk the same tile sequence: ROLE 0 loads the Q views and the K
// tiles (and publishes each tile's descriptor), ROLE 1 loads the V tiles, so a K tile can
// be fetched ahead of the V tiles still in use.
// --------------------------------------------------------------------------------------
template <int D>
__device__ void k3_gather(uint8_t* dst, const uint16_t* src_base, const K3Args& a, int g,
                          const int32_t* cols, int n) {
  // 128 rows x D fp16 gathered by column index into the 128-byte-swizzled tile layout
  const uint32_t lane = lane_id();
  constexpr int CHUNKS = D / 8;  // 16-byte chunks per row
  for (int r = (int)lane; r < 128; r += 32) {
    const int j = cols[r < n ? r : 0];
    const uint16_t* src = src_base + ((int64_t)g * a.ld_tokens + j) * D;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const uint32_t off = (uint32_t)(c >> 3) * 16384u + sw128_offset((uint32_t)r, (uint32_t)(c & 7));
      cp_async16(dst + off, src + c * 8);
    }
  }
  cp_async_wait_all();
  fence_async_smem();
  __syncwarp();
}

template <int D, int ROLE>
__device__ void k3_producer(K3Smem<D>& sm, const K3Args& a, const CUtensorMap* mq,
                            const CUtensorMap* mk, const CUtensorMap* mv, int nitems) {
  constexpr uint32_t TILE = K3Smem<D>::TILE;
  constexpr int NS = ROLE == 0 ? K3_NK : K3_NV;
  uint64_t* full = ROLE == 0 ? sm.k_full : sm.v_full;
  uint64_t* empty = ROLE == 0 ? sm.k_empty : sm.v_empty;
  const CUtensorMap* map = ROLE == 0 ? mk : mv;
  const uint16_t* src = ROLE == 0 ? a.k_rot : a.v16;
  const bool leader = lane_id() == 0;
  uint32_t kt = 0;             // tiles produced by this CTA
  uint32_t wn = 0;             // key-block walks started (items with key blocks)
  uint32_t qn[2] = {0, 0};     // Q loads per slot
  bool ok = true;
  auto stage_buf = [&](int st) -> uint8_t* { return ROLE == 0 ? sm.k[st] : sm.v[st]; };
  for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
    const K3Item I = k3_item(a, it);
    if (ROLE == 0) {
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (!ok || I.ntiles[s] == 0) continue;
        ok = mbar_wait_warp(&sm.q_empty[s], (qn[s] & 1) ^ 1);
        if (!ok) continue;
        if (leader) {
          mbar_expect_tx(&sm.q_full[s], TILE);
          const int y = (int)(((int64_t)I.x * a.hq + I.h) * a.ld_rows + (int64_t)I.qb[s] * 128);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(sm.q[s] + hf * 16384, mq, &sm.q_full[s], 64 * hf, y);
        }
        ++qn[s];
      }
    }
    // residual vertical columns, per slot, 128 per gathered tile
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (!ok || I.nres[s] == 0) continue;
      const int32_t* cols = a.resid + ((int64_t)I.h * a.nqb + I.qb[s]) * a.nvcap + I.res_off[s];
      for (int t0 = 0; t0 < I.nres[s] && ok; t0 += 128) {
        const int st = kt % NS;
        ok = mbar_wait_warp(&empty[st], ((kt / NS) & 1) ^ 1);
        if (!ok) break;
        const int n = I.nres[s] - t0 < 128 ? I.nres[s] - t0 : 128;
        if (ROLE == 0 && leader) {
          sm.desc[st][0] = 1 << s;
          sm.desc[st][1] = 0;
          sm.desc[st][2] = n;
        }
        k3_gather<D>(stage_buf(st), src, a, I.g, cols + t0, n);
        if (leader) mbar_arrive(&full[st]);
        ++kt;
      }
    }
    // key blocks: union of both slots' lists, walked from a start block taken from the
    // global tile count (the K loader picks it and hands it to the V loader) and wrapping
    int lo = 1 << 30, hi = -1;
#pragma unroll
    for (int s = 0; s < 2; ++s)
      if (I.ntiles[s] > 0 && I.hi[s] >= I.lo[s]) { lo = min(lo, I.lo[s]); hi = max(hi, I.hi[s]); }
    auto walk = [&](int a0, int b0) {
      for (int w = a0 >> 5; w <= (b0 >> 5) && b0 >= a0 && ok; ++w) {
        uint32_t m0 = (I.ntiles[0] > 0) ? range_bits(w, max(I.lo[0], a0), min(I.hi[0], b0)) : 0u;
        uint32_t m1 = (I.ntiles[1] > 0) ? range_bits(w, max(I.lo[1], a0), min(I.hi[1], b0)) : 0u;
        if (a.mask) {
          if (m0) m0 &= a.mask[((int64_t)I.h * a.nqb + I.qb[0]) * a.nkw + w];
          if (m1) m1 &= a.mask[((int64_t)I.h * a.nqb + I.qb[1]) * a.nkw + w];
        }
        uint32_t u = m0 | m1;
        while (u && ok) {
          const int b = __ffs(u) - 1;
          u &= u - 1;
          const int kb = 32 * w + b;
          const int st = kt % NS;
          ok = mbar_wait_warp(&empty[st], ((kt / NS) & 1) ^ 1);
          if (!ok) break;
          const int y = (int)((int64_t)I.g * a.ld_tokens + (int64_t)kb * 128);
          if (leader) {
            if (ROLE == 0) {
              sm.desc[st][0] = (int)((m0 >> b) & 1u) | (int)(((m1 >> b) & 1u) << 1);
              sm.desc[st][1] = (int)(kb == I.B[0]) | ((int)(kb == I.B[1]) << 1);
              sm.desc[st][2] = 128;
            }
            mbar_expect_tx(&full[st], TILE);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(stage_buf(st) + hf * 16384, map, &full[st], 64 * hf, y);
            if (ROLE == 0 && a.aligned) atomicAdd(&g_k3_cursor, 1ull);
          }
          ++kt;
        }
      }
    };
    if (ok && hi >= lo) {
      const int slot = (int)(wn & 1u);
      int start = lo;
      if (ROLE == 0) {
        ok = mbar_wait_warp(&sm.start_empty[slot], ((wn >> 1) & 1u) ^ 1u);
        if (ok && a.aligned) {
          unsigned long long c = 0;
          if (leader) c = *(volatile unsigned long long*)&g_k3_cursor;
          c = __shfl_sync(0xFFFFFFFFu, c, 0);
          // intra items' ranges share lo but differ in length: taking the clock modulo the
          // DCA chunk's block count first puts every intra item whose range reaches that
          // phase on the same block
          unsigned long long ph = c / gridDim.x;
          if (I.x == 0) ph %= (unsigned long long)(a.L / 128);
          start = lo + (int)(ph % (unsigned long long)(hi - lo + 1));
        }
        if (ok) {
          if (leader) { sm.walk_start[slot] = start; mbar_arrive(&sm.start_full[slot]); }
        }
      } else {
        ok = mbar_wait_warp(&sm.start_full[slot], (wn >> 1) & 1u);
        if (ok) {
          start = sm.walk_start[slot];
          __syncwarp();
          if (leader) mbar_arrive(&sm.start_empty[slot]);
        }
      }
      ++wn;
      if (ok) {
        walk(start, hi);
        walk(lo, start - 1);
      }
    }
  }
  if (!ok) {
    // give copies already issued time to land before the CTA exits (TMA completes in
    // microseconds and depends on nothing else)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) __nanosleep(1000);
  }
}

// --------------------------------------------------------------------------------------
// MMA warp. The whole warp runs the loop (waits, bookkeeping and descriptors are warp-
// uniform); one elected lane issues each tcgen05.mma / commit / arrive.
// --------------------------------------------------------------------------------------
struct K3Slot {
  int pend_v = -1;            // V stage of the slot's pending PV (-1: none)
  uint32_t pend_kt = 0;       // tile index of that PV
  bool pend_last = false;     // it is the slot's last tile of the item
  bool o_started = false;     // O holds a partial sum of the current item
  uint32_t qn = 0, pn = 0, pvd_issued = 0, pvd_waited = 0;
};

struct K3Desc {
  uint64_t q[2], k[K3_NK], v[K3_NV];   // 128B-swizzle descriptors of the tile bases
  // stage selection by value (no dynamically indexed local arrays)
  __device__ __forceinline__ uint64_t kd(int st) const {
    static_assert(K3_NK == 2, "two K stages");
    return st ? k[1] : k[0];
  }
  __device__ __forceinline__ uint64_t vd(int st) const {
    static_assert(K3_NV == 2, "two V stages");
    return st ? v[1] : v[0];
  }
};

// PV of the slot's pending tile: O (+)= P V, P read from tensor memory.
template <int D, int S>
__device__ __forceinline__ bool k3_pv(K3Smem<D>& sm, const K3Desc& dsc, K3Slot& sl, uint32_t tb,
                                      uint32_t& v_users) {
  constexpr uint32_t IDESC_PV = idesc_f16(128, D, 1);
  if (!mbar_wait_warp(&sm.p_full[S], sl.pn & 1)) return false;
  ++sl.pn;
  const int vst = sl.pend_v;
  if (!mbar_wait_warp(&sm.v_full[vst], (sl.pend_kt / K3_NV) & 1)) return false;
  tc_fence_after();
  const uint32_t o_t = tb + 256u * S + 128u, p_t = tb + 256u * S;
  const uint64_t vd = dsc.vd(vst);
  const uint32_t sh = 4u * (uint32_t)vst;
  const uint32_t u = ((v_users >> sh) & 0xFu) - 1u;
  if (elect_one()) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)   // 16 keys = 16 rows of 128 B per step (2048 B, >> 4 = 128)
      mma_ts(o_t, p_t + kk * 8u, vd + (uint64_t)(kk * 128), IDESC_PV,
             (sl.o_started || kk > 0) ? 1u : 0u);
    // P lives in S's columns 0..63: the slot's next QK^T is issued only after this commit
    mma_commit(&sm.pv_done[S]);
    if (sl.pend_last) mma_commit(&sm.o_done[S]);
    if (u == 0) mma_commit(&sm.v_empty[vst]);
  }
  __syncwarp();
  sl.o_started = !sl.pend_last;
  ++sl.pvd_issued;
  v_users = (v_users & ~(0xFu << sh)) | (u << sh);
  sl.pend_v = -1;
  return true;
}

// S = Q K^T for the slot on K stage kst.
template <int D, int S>
__device__ __forceinline__ bool k3_qk(K3Smem<D>& sm, const K3Desc& dsc, K3Slot& sl, int& rem,
                                      bool& first, int kst, int vst, uint32_t kt, int diag,
                                      int ncols, uint32_t tb) {
  constexpr uint32_t IDESC_QK = idesc_f16(128, 128, 0);
  if (first) {
    if (!mbar_wait_warp(&sm.q_full[S], sl.qn & 1)) return false;
    ++sl.qn;
    first = false;
    tc_fence_after();
  }
  if (sl.pvd_waited < sl.pvd_issued) {   // the slot's previous PV still reads P (S columns)
    if (!mbar_wait_warp(&sm.pv_done[S], sl.pvd_waited & 1)) return false;
    ++sl.pvd_waited;
    tc_fence_after();
  }
  --rem;
  const bool last = rem == 0;
  const uint32_t s_t = tb + 256u * S;
  const uint64_t qd = dsc.q[S], kd = dsc.kd(kst);
  if (elect_one()) {
    sm.meta[S] = ((diag >> S) & 1) | (ncols << 8) | ((int)last << 16);
    mbar_arrive(&sm.s_full[S]);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      // 16 fp16 of K = 32 B inside a 128 B swizzle row (>> 4 = 2); halves 16 KB apart
      const uint64_t off = (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2);
      mma_ss(s_t, qd + off, kd + off, IDESC_QK, kk > 0 ? 1u : 0u);
    }
    mma_commit(&sm.s_full[S]);
    if (last) mma_commit(&sm.q_empty[S]);
  }
  __syncwarp();
  sl.pend_v = vst;
  sl.pend_kt = kt;
  sl.pend_last = last;
  return true;
}

template <int D>
__device__ void k3_mma(K3Smem<D>& sm, const K3Args& a, int nitems) {
  const uint32_t tb = sm.tmem_base;
  K3Desc dsc;
  dsc.q[0] = sdesc_sw128(smem_u32(sm.q[0]), 16u, 1024u);
  dsc.q[1] = sdesc_sw128(smem_u32(sm.q[1]), 16u, 1024u);
#pragma unroll
  for (int i = 0; i < K3_NK; ++i) dsc.k[i] = sdesc_sw128(smem_u32(sm.k[i]), 16u, 1024u);
#pragma unroll
  for (int i = 0; i < K3_NV; ++i) dsc.v[i] = sdesc_sw128(smem_u32(sm.v[i]), 16384u, 1024u);
  uint32_t kt = 0;
  K3Slot s0, s1;
  uint32_t v_users = 0;       // 4 bits per V stage: PVs still to issue on it
  bool ok = true;
  for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
    const K3Item I = k3_item(a, it);
    int rem0 = I.ntiles[0], rem1 = I.ntiles[1];
    bool first0 = true, first1 = true;
    while ((rem0 > 0 || rem1 > 0) && ok) {
      const int kst = kt % K3_NK, vst = kt % K3_NV;
      // slot 0's pending PV does not need the next K tile: issue it first
      if (s0.pend_v >= 0) ok = k3_pv<D, 0>(sm, dsc, s0, tb, v_users);
      if (!ok) break;
      ok = mbar_wait_warp(&sm.k_full[kst], (kt / K3_NK) & 1);
      if (!ok) break;
      tc_fence_after();
      const int flags = sm.desc[kst][0], diag = sm.desc[kst][1], ncols = sm.desc[kst][2];
      uint32_t users = 0;
      if (ok && (flags & 1)) { ok = k3_qk<D, 0>(sm, dsc, s0, rem0, first0, kst, vst, kt, diag, ncols, tb); ++users; }
      if (ok && s1.pend_v >= 0) ok = k3_pv<D, 1>(sm, dsc, s1, tb, v_users);
      if (ok && (flags & 2)) { ok = k3_qk<D, 1>(sm, dsc, s1, rem1, first1, kst, vst, kt, diag, ncols, tb); ++users; }
      if (!ok) break;
      const uint32_t sh = 4u * (uint32_t)vst;
      v_users = (v_users & ~(0xFu << sh)) | (users << sh);
      if (elect_one()) mma_commit(&sm.k_empty[kst]);
      __syncwarp();
      ++kt;
    }
  }
  if (ok && s0.pend_v >= 0) ok = k3_pv<D, 0>(sm, dsc, s0, tb, v_users);
  if (ok && s1.pend_v >= 0) ok = k3_pv<D, 1>(sm, dsc, s1, tb, v_users);
  if (elect_one()) mma_commit(&sm.drain);
  __syncwarp();
  mbar_wait_warp(&sm.drain, 0);
}

// --------------------------------------------------------------------------------------
// Softmax warpgroup of slot S: thread t owns row t of the slot's query block.
// --------------------------------------------------------------------------------------
template <int D, int S>
__device__ void k3_softmax(K3Smem<D>& sm, const K3Args& a, int nitems) {
  const int t = threadIdx.x - 128 * S;          // row within the query block
  const uint32_t wq = warp_id() & 3u;           // TMEM lane quarter of this warp
  const uint32_t tb = sm.tmem_base + ((32u * wq) << 16) + 256u * S;
  uint32_t sn = 0, on = 0;
  bool ok = true;
  for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
    const K3Item I = k3_item(a, it);
    if (!I.valid[S]) continue;
    const int64_t row = I.B[S] * 128 + t;       // global row
    const int64_t rl = row - a.s0;              // row within the chunk
    const bool live = row < a.e;
    float* lse_out = a.lse_part + ((int64_t)I.x * a.hq + I.h) * a.ld_rows + rl;
    if (I.ntiles[S] == 0) {
      if (live) *lse_out = -INFINITY;
      continue;
    }
    float m = -INFINITY, l = 0.f;
    bool o_valid = false;
    for (int tt = 0; tt < I.ntiles[S]; ++tt) {
      ok = mbar_wait_warp(&sm.s_full[S], sn & 1);
      if (!ok) break;
      ++sn;
      tc_fence_after();
      const int meta = sm.meta[S];
      const bool diag = meta & 1;
      const int ncols = (meta >> 8) & 0xFF;
      // the whole 128-column S row in registers: one tensor-memory load and wait per tile
      uint32_t xr[128];
      tmem_ld128(tb, xr);
      float* x = reinterpret_cast<float*>(xr);
      if (diag || ncols < 128) {
        const int lim = diag ? t : ncols - 1;
#pragma unroll
        for (int c = 0; c < 128; ++c) if (c > lim) x[c] = -INFINITY;
      }
      // row maximum: eight independent chains of 2-input max (the 3-input max.f32 is far
      // slower on sm_100: measured 550 vs 115 cycles per 128-column row)
      float a8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) a8[k] = x[k];
#pragma unroll
      for (int c = 8; c < 128; c += 8)
#pragma unroll
        for (int k = 0; k < 8; ++k) a8[k] = fmaxf(a8[k], x[c + k]);
#pragma unroll
      for (int wdt = 4; wdt >= 1; wdt /= 2)
#pragma unroll
        for (int k = 0; k < wdt; ++k) a8[k] = fmaxf(a8[k], a8[k + wdt]);
      const float mx = a8[0];
      const bool need = mx > m + K3_RESCALE_THRESHOLD;
      if (__any_sync(0xFFFFFFFFu, need)) {
        const float m_new = need ? mx : m;
        const float alpha = need ? ex2(m - m_new) : 1.f;
        l *= alpha;
        if (o_valid) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tb + 128u + 32u * c, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
            tmem_st32(tb + 128u + 32u * c, r);
          }
        }
        m = m_new;
      }
      const float mu = m == -INFINITY ? 0.f : m;
      // p = 2^(x - mu) in packed pairs, four independent packed sums; P goes to tensor
      // memory 32 keys (16 packed words) at a time
      const uint64_t nmu = f2_pack(-mu, -mu);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int j = 32 * ch + 2 * c;
          const uint64_t dx = f2_add(f2_pack(x[j], x[j + 1]), nmu);
          float p0, p1;
          if ((c & 7) < K3_POLY_PAIRS_OF_8) {
            f2_unpack(ex2_poly2(dx), p0, p1);       // FMA pipe
          } else {
            float d0, d1;
            f2_unpack(dx, d0, d1);
            p0 = ex2(d0);                           // multi-function unit
            p1 = ex2(d1);
          }
          acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
          pk[c] = pack_f16x2(p0, p1);
        }
        tmem_st16(tb + 16u * ch, pk);
      }
      float s0, s1, s2, s3;
      f2_unpack(f2_add(acc[0], acc[1]), s0, s1);
      f2_unpack(f2_add(acc[2], acc[3]), s2, s3);
      l += (s0 + s1) + (s2 + s3);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[S]);
      o_valid = true;
    }
    if (!ok) break;
    ok = mbar_wait_warp(&sm.o_done[S], on & 1);
    if (!ok) break;
    ++on;
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* dst = a.o_part + (((int64_t)I.x * a.hq + I.h) * a.ld_rows + rl) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tb + 128u + 32u * c, r);
      if (live) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 v4 = make_float4(__uint_as_float(r[j]) * inv, __uint_as_float(r[j + 1]) * inv,
                                  __uint_as_float(r[j + 2]) * inv, __uint_as_float(r[j + 3]) * inv);
          *reinterpret_cast<float4*>(dst + 32 * c + j) = v4;
        }
      }
    }
    if (live) *lse_out = l > 0.f ? m + __log2f(l) : -INFINITY;
    tc_fence_before();
  }
}

template <int D>
__global__ void __launch_bounds__(K3_THREADS, 1)
block_sparse_attn_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                         const __grid_constant__ CUtensorMap mv, const K3Args a) {
  extern __shared__ uint8_t k3_raw[];
  K3Smem<D>& sm = *reinterpret_cast<K3Smem<D>*>((reinterpret_cast<uintptr_t>(k3_raw) + 1023) & ~uintptr_t(1023));
  const int w = warp_id();
  const int nitems = (*a.n_units) * a.hq;
  if (threadIdx.x == 0) {
    for (int i = 0; i < K3_NK; ++i) { mbar_init(&sm.k_full[i], 1); mbar_init(&sm.k_empty[i], 1); }
    for (int i = 0; i < K3_NV; ++i) { mbar_init(&sm.v_full[i], 1); mbar_init(&sm.v_empty[i], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1); mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.s_full[s], 2); mbar_init(&sm.p_full[s], 128); mbar_init(&sm.o_done[s], 1);
      mbar_init(&sm.pv_done[s], 1);
    }
    mbar_init(&sm.drain, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&sm.start_full[i], 1); mbar_init(&sm.start_empty[i], 1); }
    fence_mbar_init();
  }
  if (w == 9) { tmem_alloc(&sm.tmem_base, 512); tmem_relinquish(); }
  if (w == 8 && lane_id() == 0) { tma_prefetch(&mq); tma_prefetch(&mk); tma_prefetch(&mv); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w < 8) {
    regs_increase<K3_REGS_SOFTMAX>();
    if (w < 4) k3_softmax<D, 0>(sm, a, nitems);
    else k3_softmax<D, 1>(sm, a, nitems);
  } else {
    regs_decrease<K3_REGS_OTHER>();
    if (w == 8) k3_producer<D, 0>(sm, a, &mq, &mk, &mv, nitems);
    else if (w == 9) k3_mma<D>(sm, a, nitems);
    else if (w == 10) k3_producer<D, 1>(sm, a, &mq, &mk, &mv, nitems);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (w == 9) { __syncwarp(); tmem_dealloc(sm.tmem_base, 512); }
}

// --------------------------------------------------------------------------------------
// Work units: (pair m, pattern x) sorted by dense tile count, largest first, so the
// static round-robin over (unit, head) items starts with the longest items.
// --------------------------------------------------------------------------------------
__global__ void k3_units_kernel(int64_t s0, int nqb, int64_t L, int32_t* units, int32_t* n_units) {
  const int npair = (nqb + 1) / 2;
  const int U = 3 * npair;
  const int64_t Lb = L / 128;
  extern __shared__ int32_t ucost[];
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int m = u / 3, x = u % 3;
    int c = 0;
    for (int s = 0; s < 2; ++s) {
      const int qb = 2 * m + s;
      if (qb >= nqb) continue;
      int lo, hi;
      seg_range(s0 / 128 + qb, x, Lb, &lo, &hi);
      if (hi >= lo) c = max(c, hi - lo + 1);
    }
    ucost[u] = c;
  }
  __syncthreads();
  int nz = 0;
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int c = ucost[u];
    if (c == 0) continue;
    int rank = 0;
    for (int v = 0; v < U; ++v) {
      const int cv = ucost[v];
      rank += (cv > c) || (cv == c && v < u);
    }
    units[rank] = ((u / 3) << 2) | (u % 3);
    ++nz;
  }
  __shared__ int total;
  if (threadIdx.x == 0) total = 0;
  __syncthreads();
  atomicAdd(&total, nz);
  __syncthreads();
  if (threadIdx.x == 0) *n_units = total;
}

}  // namespace q1m
