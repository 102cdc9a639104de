// q1m_api.cu — the C ABI declared in include/q1m.h: argument validation, workspace layout,
// TMA tensor maps, kernel launches and the chunked-prefill driver. The whole library is
// this one translation unit (the kernels are headers), so the device status word is shared
// without relocatable device code.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "q1m_device.cuh"
#include "rope_dca.cuh"
#include "vs_select.cuh"
#include "vs_estimate.cuh"
#include "attn_tc.cuh"
#include "lse_merge.cuh"
#include "decode.cuh"

using namespace q1m;

namespace {

thread_local std::string t_err;

q1m_status fail(q1m_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

#define Q1M_CUDA(call)                                                                 \
  do {                                                                                 \
    cudaError_t err_ = (call);                                                         \
    if (err_ != cudaSuccess)                                                           \
      return fail(Q1M_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(err_));     \
  } while (0)

std::atomic<uint64_t> g_launches{0};

#define Q1M_LAUNCHED()                                                                 \
  do {                                                                                 \
    g_launches.fetch_add(1, std::memory_order_relaxed);                                \
    cudaError_t err_ = cudaGetLastError();                                             \
    if (err_ != cudaSuccess)                                                           \
      return fail(Q1M_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(err_)); \
  } while (0)

#define Q1M_TRY(expr)                       \
  do {                                      \
    q1m_status st_ = (expr);                \
    if (st_ != Q1M_OK) return st_;          \
  } while (0)

// ---- per-stage event timers (opt-in, per thread) -------------------------------------------
struct ProfRec {
  int stage;
  cudaEvent_t a, b;
};
struct StageTimer {
  bool on = false;
  std::vector<cudaEvent_t> pool;   // events are reused across reads
  size_t used = 0;
  std::vector<ProfRec> recs;
};
thread_local StageTimer t_prof;

cudaEvent_t prof_event() {
  if (t_prof.used == t_prof.pool.size()) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return nullptr;
    t_prof.pool.push_back(ev);
  }
  return t_prof.pool[t_prof.used++];
}

// Opens a timed interval of `stage` on stream `st`; returns its index (-1: timing off).
int prof_begin(int stage, cudaStream_t st) {
  if (!t_prof.on) return -1;
  cudaEvent_t a = prof_event(), b = prof_event();
  if (!a || !b) return -1;
  cudaEventRecord(a, st);
  t_prof.recs.push_back(ProfRec{stage, a, b});
  return (int)t_prof.recs.size() - 1;
}

void prof_end(int idx, cudaStream_t st) {
  if (idx >= 0) cudaEventRecord(t_prof.recs[idx].b, st);
}

inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
inline size_t align_up(size_t x) { return (x + 1023) & ~size_t(1023); }
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D fp16 tensor map with 128-byte swizzle: rows of `inner` elements, `rows` rows.
q1m_status make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint32_t box_inner, uint32_t box_rows) {
  auto enc = tmap_encode();
  if (!enc) return fail(Q1M_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return fail(Q1M_ERR_INVALID, "tensor base not 16-byte aligned");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(Q1M_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return Q1M_OK;
}

struct Dev {
  int sms = 0;
  bool sm100 = false;
};

q1m_status device_info(Dev* d) {
  int dev = 0;
  Q1M_CUDA(cudaGetDevice(&dev));
  int major = 0, minor = 0;
  Q1M_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  Q1M_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  Q1M_CUDA(cudaDeviceGetAttribute(&d->sms, cudaDevAttrMultiProcessorCount, dev));
  d->sm100 = (major == 10 && minor == 0);
  if (!d->sm100) return fail(Q1M_ERR_UNSUPPORTED, "device is sm_%d%d; this library runs on sm_100a only", major, minor);
  return Q1M_OK;
}

bool sparse(const q1m_params* p) { return p->vs_vertical != 0 || p->vs_slash != 0; }

q1m_status check_shape(int64_t n, int hq, int hkv, int d, const q1m_params* p) {
  if (!p) return fail(Q1M_ERR_INVALID, "params is NULL");
  if (n <= 0) return fail(Q1M_ERR_INVALID, "seq_len must be positive");
  if (hq <= 0 || hkv <= 0 || hq % hkv != 0) return fail(Q1M_ERR_INVALID, "n_q_heads must be a positive multiple of n_kv_heads");
  if (d != 64 && d != 128) return fail(Q1M_ERR_UNSUPPORTED, "head_dim %d (64 or 128 supported)", d);
  if (p->in_dtype != Q1M_BF16 && p->in_dtype != Q1M_F32) return fail(Q1M_ERR_INVALID, "bad in_dtype");
  if (p->out_dtype != Q1M_BF16 && p->out_dtype != Q1M_F32) return fail(Q1M_ERR_INVALID, "bad out_dtype");
  if (!(p->rope_base > 1.0) || !std::isfinite(p->rope_base)) return fail(Q1M_ERR_INVALID, "rope_base must be > 1");
  if (!std::isfinite(p->yarn_s)) return fail(Q1M_ERR_INVALID, "yarn_s must be finite");
  if (p->local_window < 0 || p->dca_chunk <= p->local_window) return fail(Q1M_ERR_INVALID, "need 0 <= local_window < dca_chunk");
  if ((p->dca_chunk - p->local_window) % 128 != 0) return fail(Q1M_ERR_UNSUPPORTED, "dca_chunk - local_window must be a multiple of 128");
  if (p->dca_chunk > (int64_t)1 << 30) return fail(Q1M_ERR_UNSUPPORTED, "dca_chunk too large");
  if (p->equal_cost_chunks < 0) return fail(Q1M_ERR_INVALID, "equal_cost_chunks must be >= 0");
  if (p->equal_cost_chunks == 0 && (p->prefill_chunk <= 0 || p->prefill_chunk % 128 != 0))
    return fail(Q1M_ERR_INVALID, "prefill_chunk must be a positive multiple of 128");
  if (n > ((int64_t)1 << 31) / 8) return fail(Q1M_ERR_UNSUPPORTED, "seq_len too large");
  if ((int64_t)hkv * round_up(n, 128) >= ((int64_t)1 << 31)) return fail(Q1M_ERR_UNSUPPORTED, "n_kv_heads * seq_len too large");
  if (sparse(p)) {
    if (p->vs_vertical < 0 || p->vs_slash < 1) return fail(Q1M_ERR_INVALID, "sparse mode needs vs_slash >= 1 and vs_vertical >= 0");
    if (p->vs_force_local < 1) return fail(Q1M_ERR_INVALID, "sparse mode needs vs_force_local >= 1 (every row keeps its diagonal)");
    if (p->vs_last_q < 1 || p->vs_last_q > 64) return fail(Q1M_ERR_INVALID, "vs_last_q must be in [1, 64]");
    if ((hq / hkv) * 64 > EB_MAX_ROWS) return fail(Q1M_ERR_UNSUPPORTED, "estimator supports at most 7 Q heads per KV head");
    if ((round_up(n, 128) / 128 + 31) / 32 > MB_MAX_NKW) return fail(Q1M_ERR_UNSUPPORTED, "seq_len too large for the block mask");
  }
  return Q1M_OK;
}

// Exclusive end rows of the prefill chunks (see q1m_prefill_bounds in the header).
std::vector<int64_t> chunk_ends(int64_t n, const q1m_params* p) {
  std::vector<int64_t> ends;
  if (p->equal_cost_chunks == 0) {
    for (int64_t s0 = 0; s0 < n; s0 += p->prefill_chunk)
      ends.push_back(s0 + p->prefill_chunk < n ? s0 + p->prefill_chunk : n);
    return ends;
  }
  using u128 = unsigned __int128;
  const int64_t nb = (n + 127) / 128, K = p->equal_cost_chunks;
  auto C = [](int64_t m) { return (u128)m * (u128)(m + 1) / 2; };
  const u128 T = C(nb);
  int64_t m = 0, prev = 0;
  for (int64_t k = 1; k < K; ++k) {
    while (m < nb && (u128)K * C(m) < (u128)k * T) ++m;   // smallest m with K C(m) >= k T
    if (m > prev) { ends.push_back(128 * m < n ? 128 * m : n); prev = m; }
  }
  if (prev < nb) ends.push_back(n);
  return ends;
}

int64_t max_chunk_rows(int64_t n, const q1m_params* p) {
  int64_t s0 = 0, mx = 0;
  for (int64_t e : chunk_ends(n, p)) { mx = e - s0 > mx ? e - s0 : mx; s0 = e; }
  return mx;
}

// The attention stage sorts a chunk's work units in one CTA's shared memory, so a prefill
// chunk may hold at most Q1M_MAX_CHUNK_QUERY_BLOCKS query blocks.
q1m_status check_chunks(int64_t n, const q1m_params* p) {
  const int64_t rows = max_chunk_rows(n, p);
  if (rows > (int64_t)128 * Q1M_MAX_CHUNK_QUERY_BLOCKS)
    return fail(Q1M_ERR_UNSUPPORTED, "a prefill chunk of %lld rows exceeds %d query blocks",
                (long long)rows, Q1M_MAX_CHUNK_QUERY_BLOCKS);
  return Q1M_OK;
}

float view_scale(const q1m_params* p, int d) {
  const double s = p->yarn_s;
  double inv_t = 1.0;
  if (s > 1.0) { const double r = 0.1 * std::log(s) + 1.0; inv_t = r * r; }
  return (float)(inv_t / std::sqrt((double)d) * 1.4426950408889634);  // * log2(e)
}

// ---- estimator scratch layout --------------------------------------------------------------
struct EstLayout {
  int m_pad, n_mt, nsplit, nkt;
  size_t est_q, part, lse2, slash_part, total;
};

EstLayout est_layout(int64_t e, int hq, int hkv, int d) {
  EstLayout L{};
  const int G = hq / hkv;
  L.n_mt = (G * 64 + 127) / 128;
  L.m_pad = L.n_mt * 128;
  L.nkt = (int)((e + 127) / 128);
  // pass A runs two CTAs per SM: split the key range so every CTA is resident in one wave
  // of 2 x 148
  int ns = 296 / (hkv * L.n_mt);
  L.nsplit = ns < 1 ? 1 : (ns > L.nkt ? L.nkt : ns);
  size_t off = 0;
  L.est_q = off; off = align_up(off + (size_t)4 * hkv * L.m_pad * d * 2);
  L.part = off; off = align_up(off + (size_t)hkv * L.m_pad * L.nsplit * sizeof(float2));
  L.lse2 = off; off = align_up(off + (size_t)hkv * L.m_pad * 4);
  L.slash_part = off; off = align_up(off + (size_t)hq * L.nkt * EB_U * 4);
  L.total = off;
  return L;
}

// ---- whole-layer workspace layout ---------------------------------------------------------
// ---- debug mode: guard regions after every workspace buffer, index-list validation -------
constexpr size_t GUARD_BYTES = 4096;
constexpr uint32_t GUARD_WORD = 0xA5A5A5A5u;
constexpr int MAX_GUARDS = 32;
std::atomic<int> g_debug{-1};
std::atomic<int> g_determ{-1};

bool deterministic_on() {
  int v = g_determ.load();
  if (v < 0) {
    const char* e = std::getenv("Q1M_DETERMINISTIC");
    v = (e && *e && std::strcmp(e, "0") != 0) ? 1 : 0;
    g_determ.store(v);
  }
  return v == 1;
}
std::atomic<int> g_inject{-1};

bool debug_on() {
  int v = g_debug.load();
  if (v < 0) {
    const char* e = std::getenv("Q1M_DEBUG");
    v = (e && *e && std::strcmp(e, "0") != 0) ? 1 : 0;
    g_debug.store(v);
  }
  return v == 1;
}

__device__ int g_check_info = -1;   // first failing guard (0..) or list check (1000 + kind)

struct GuardSet {
  uint64_t off[MAX_GUARDS];
  int n;
};

__global__ void guard_check_kernel(const uint8_t* __restrict__ base, GuardSet gs) {
  const int gi = blockIdx.x;
  if (gi >= gs.n) return;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(base + gs.off[gi]);
  for (int i = threadIdx.x; i < (int)(GUARD_BYTES / 4); i += blockDim.x)
    if (w[i] != GUARD_WORD) { atomicCAS(&g_check_info, -1, gi); latch(Q1M_ERR_CHECK); }
}

// One thread per head: V ascending in [0, e); S ascending in [0, e) starting with the forced
// diagonals 0 .. fl - 1; then, per (head, query block), block counts within the key-block
// count and residual columns ascending in [0, e).
__global__ void index_check_kernel(const int32_t* __restrict__ V, int nv, const int32_t* __restrict__ Sx,
                                   int ns, int64_t e, int hq, int fl, const int32_t* __restrict__ cnt,
                                   const int32_t* __restrict__ resid, int nqb, int nvcap, int64_t nkb) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= hq) return;
  auto bad = [](int kind) { atomicCAS(&g_check_info, -1, 1000 + kind); latch(Q1M_ERR_CHECK); };
  for (int i = 0; i < nv; ++i) {
    const int64_t c = V[(int64_t)h * nv + i];
    if (c < 0 || c >= e || (i > 0 && c <= V[(int64_t)h * nv + i - 1])) { bad(1); return; }
  }
  for (int i = 0; i < ns; ++i) {
    const int64_t o = Sx[(int64_t)h * ns + i];
    if (o < 0 || o >= e || (i > 0 && o <= Sx[(int64_t)h * ns + i - 1])) { bad(2); return; }
    if (i < fl && i < e && o != i) { bad(3); return; }
  }
  for (int b = 0; b < nqb; ++b) {
    const int32_t* c = cnt + ((int64_t)h * nqb + b) * 8;
    if (c[0] < 0 || c[1] < 0 || c[2] < 0 || c[0] + c[1] + c[2] > nkb) { bad(4); return; }
    const int nres = c[6];
    if (nres < 0 || nres > nvcap || c[3] + c[4] + c[5] != nres) { bad(5); return; }
    const int32_t* r = resid + ((int64_t)h * nqb + b) * nvcap;
    for (int i = 0; i < nres; ++i)
      if (r[i] < 0 || r[i] >= e || (i > 0 && r[i] <= r[i - 1])) { bad(6); return; }
  }
}

struct Layout {
  int64_t ld_tokens, ld_rows, nqb_max, nkw_max;
  int nv, ns;
  size_t table, k_rot, v16, qv, o_part, lse_part, units, vert, slash, est, V, Sx, mask, resid,
      cnt, total;
  GuardSet guards{};
};

Layout layout(int64_t n, int hq, int hkv, int d, const q1m_params* p) {
  Layout L{};
  L.ld_tokens = round_up(n, 128);
  L.ld_rows = round_up(max_chunk_rows(n, p), 128);
  L.nqb_max = L.ld_rows / 128;
  L.nkw_max = (L.ld_tokens / 128 + 31) / 32;
  L.nv = (int)(p->vs_vertical < n ? p->vs_vertical : n);
  L.ns = (int)(p->vs_slash < n ? p->vs_slash : n);
  size_t off = 0;
  const bool dbg = debug_on();
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes);
    if (dbg && L.guards.n < MAX_GUARDS) { L.guards.off[L.guards.n++] = off; off += GUARD_BYTES; }
    return o;
  };
  L.table = take((size_t)p->dca_chunk * (d / 2) * sizeof(float2));
  L.k_rot = take((size_t)hkv * L.ld_tokens * d * 2);
  L.v16 = take((size_t)hkv * L.ld_tokens * d * 2);
  L.qv = take((size_t)3 * hq * L.ld_rows * d * 2);
  L.o_part = take((size_t)3 * hq * L.ld_rows * d * 4);
  L.lse_part = take((size_t)3 * hq * L.ld_rows * 4);
  L.units = take((size_t)(3 * (L.nqb_max + 1) / 2 + 8) * 4);
  if (sparse(p)) {
    L.vert = take((size_t)hq * L.ld_tokens * 4);
    L.slash = take((size_t)hq * L.ld_tokens * 4);
    L.est = take(est_layout(n, hq, hkv, d).total);
    L.V = take((size_t)hq * (L.nv > 0 ? L.nv : 1) * 4);
    L.Sx = take((size_t)hq * L.ns * 4);
    L.mask = take((size_t)hq * L.nqb_max * L.nkw_max * 4);
    L.resid = take((size_t)hq * L.nqb_max * (L.nv > 0 ? L.nv : 1) * 4);
    L.cnt = take((size_t)hq * L.nqb_max * 8 * 4);
  }
  L.total = off;
  return L;
}

template <typename T>
T* at(void* base, size_t off) { return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off); }

int blocks_for(int64_t n, int threads) { return (int)((n + threads - 1) / threads); }

// Debug mode: checks every guard after `stage` (and first plays the armed injection, once).
q1m_status debug_after(const Layout& L, void* ws, int stage, bool first_chunk, cudaStream_t st) {
  if (L.guards.n == 0) return Q1M_OK;
  if (first_chunk && g_inject.load() == stage) {
    g_inject.store(-1);
    Q1M_CUDA(cudaMemsetAsync(at<uint8_t>(ws, L.guards.off[0]), 0, 1, st));
  }
  guard_check_kernel<<<L.guards.n, 256, 0, st>>>(static_cast<const uint8_t*>(ws), L.guards);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

// ---- stage launchers (arguments already validated) ------------------------------------------
q1m_status run_rope_table(float* table, int64_t n_pos, int d, double base, cudaStream_t st) {
  const int64_t n = n_pos * (d / 2);
  rope_table_kernel<<<blocks_for(n, 256), 256, 0, st>>>(reinterpret_cast<float2*>(table), n_pos, d / 2, base);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

q1m_status run_rope_keys(const void* k, const void* v, int64_t s0, int64_t e, int hkv, int d,
                         const q1m_params* p, const float* table, uint16_t* k_rot, uint16_t* v16,
                         int64_t ld_tokens, cudaStream_t st) {
  const int64_t L = p->dca_chunk - p->local_window;
  const float2* tb = reinterpret_cast<const float2*>(table);
  // one block per token; hkv * D / 16 threads of work per token
  const int work = hkv * (d / 16);
  const int threads = work >= 128 ? 128 : (work + 31) / 32 * 32;
  if (p->in_dtype == Q1M_BF16)
    rope_keys_kernel<__nv_bfloat16><<<(unsigned)(e - s0), threads, 0, st>>>(
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, s0, e, hkv, d, L, tb, k_rot, v16, ld_tokens);
  else
    rope_keys_kernel<float><<<(unsigned)(e - s0), threads, 0, st>>>(
        (const float*)k, (const float*)v, s0, e, hkv, d, L, tb, k_rot, v16, ld_tokens);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

q1m_status run_rope_queries(const void* q, int64_t s0, int64_t e, int hq, int d, const q1m_params* p,
                            const float* table, uint16_t* qv, int64_t ld_rows, cudaStream_t st) {
  const int64_t L = p->dca_chunk - p->local_window;
  const float sc = view_scale(p, d);
  const float2* tb = reinterpret_cast<const float2*>(table);
  // one block per row; hq * D / 16 threads of work per row
  const int work = hq * (d / 16);
  const int threads = work >= 256 ? 256 : (work + 31) / 32 * 32;
  if (p->in_dtype == Q1M_BF16)
    rope_queries_kernel<__nv_bfloat16><<<(unsigned)ld_rows, threads, 0, st>>>(
        (const __nv_bfloat16*)q, s0, e, hq, d, L, p->dca_chunk, sc, tb, qv, ld_rows);
  else
    rope_queries_kernel<float><<<(unsigned)ld_rows, threads, 0, st>>>(
        (const float*)q, s0, e, hq, d, L, p->dca_chunk, sc, tb, qv, ld_rows);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

template <int D>
q1m_status run_estimate_d(const void* q, const uint16_t* k_rot, int64_t ld_tokens, int64_t s0,
                          int64_t e, int hq, int hkv, const q1m_params* p, const float* table,
                          float* vert, float* slash, int64_t ld, void* scratch, const Dev& dev,
                          cudaStream_t st) {
  const EstLayout EL = est_layout(e, hq, hkv, D);
  EstArgs a{};
  a.r_lo = e - p->vs_last_q > s0 ? e - p->vs_last_q : s0;
  a.e = e;
  a.hq = hq; a.hkv = hkv; a.G = hq / hkv;
  a.L = p->dca_chunk - p->local_window;
  a.ld_tokens = ld_tokens;
  a.m_pad = EL.m_pad; a.nkt = EL.nkt; a.n_mt = EL.n_mt; a.nsplit = EL.nsplit;
  a.c_hi = (e - 1) / a.L;
  a.part = at<float2>(scratch, EL.part);
  a.lse2 = at<float>(scratch, EL.lse2);
  a.vert = vert;
  a.slash_part = at<float>(scratch, EL.slash_part);
  a.ld = ld;
  uint16_t* est_q = at<uint16_t>(scratch, EL.est_q);
  {
    const int64_t n = (int64_t)4 * hkv * EL.m_pad * (D / 2);
    const float sc = view_scale(p, D);
    const float2* tb = reinterpret_cast<const float2*>(table);
    if (p->in_dtype == Q1M_BF16)
      est_queries_kernel<__nv_bfloat16><<<blocks_for(n, 256), 256, 0, st>>>(
          (const __nv_bfloat16*)q, a.r_lo, e, hq, hkv, D, a.L, p->dca_chunk, sc, tb, est_q, EL.m_pad);
    else
      est_queries_kernel<float><<<blocks_for(n, 256), 256, 0, st>>>(
          (const float*)q, a.r_lo, e, hq, hkv, D, a.L, p->dca_chunk, sc, tb, est_q, EL.m_pad);
    Q1M_LAUNCHED();
  }
  CUtensorMap m_est128, m_est64, m_k;
  const uint64_t est_rows = (uint64_t)4 * hkv * EL.m_pad;
  Q1M_TRY(make_map(&m_est128, est_q, D, est_rows, 64, 128));
  Q1M_TRY(make_map(&m_est64, est_q, D, est_rows, 64, 64));
  Q1M_TRY(make_map(&m_k, k_rot, D, (uint64_t)hkv * ld_tokens, 64, 128));
  {
    const size_t smem = sizeof(EASmem<D>) + 1024;
    Q1M_CUDA(cudaFuncSetAttribute(est_pass_a_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    est_pass_a_kernel<D><<<hkv * EL.n_mt * EL.nsplit, EA_THREADS, smem, st>>>(m_est128, m_k, a);
    Q1M_LAUNCHED();
    est_merge_a_kernel<<<blocks_for((int64_t)hkv * EL.m_pad, 256), 256, 0, st>>>(a);
    Q1M_LAUNCHED();
  }
  {
    const size_t smem = sizeof(EBSmem<D>) + 1024;
    Q1M_CUDA(cudaFuncSetAttribute(est_pass_b_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    const int64_t W = (int64_t)hkv * EL.nkt;
    const int grid = (int)(W < dev.sms ? W : dev.sms);
    est_pass_b_kernel<D><<<grid, EB_THREADS, smem, st>>>(m_est64, m_k, a);
    Q1M_LAUNCHED();
    est_slash_reduce_kernel<<<dim3(blocks_for(e, 256), hq), 256, 0, st>>>(a, slash);
    Q1M_LAUNCHED();
  }
  return Q1M_OK;
}

q1m_status run_select(const float* vert, const float* slash, int64_t ld, int64_t e, int hq,
                      const q1m_params* p, int32_t* V, int32_t* Sx, cudaStream_t st) {
  vs_select_kernel<<<dim3(hq, 2), SEL_THREADS, 0, st>>>(vert, slash, ld, e, p->vs_vertical,
                                                       p->vs_slash, p->vs_force_local, V, Sx);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

q1m_status run_masks(const int32_t* V, const int32_t* Sx, int64_t s0, int64_t e, int hq,
                     const q1m_params* p, uint32_t* mask, int32_t* resid, int32_t* cnt,
                     cudaStream_t st) {
  const int nqb = (int)((e - s0 + 127) / 128);
  const int nv = (int)(p->vs_vertical < e ? p->vs_vertical : e);
  const int ns = (int)(p->vs_slash < e ? p->vs_slash : e);
  vs_mask_kernel<<<dim3(hq, (nqb + MB_QB - 1) / MB_QB), MB_THREADS, 0, st>>>(
      V, Sx, s0, e, nv, ns, p->dca_chunk - p->local_window, mask, resid, cnt);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

template <int D>
q1m_status run_attn_d(const uint16_t* qv, int64_t ld_rows, const uint16_t* k_rot, const uint16_t* v16,
                      int64_t ld_tokens, const uint32_t* mask, const int32_t* resid, const int32_t* cnt,
                      int64_t s0, int64_t e, int hq, int hkv, const q1m_params* p, float* o_part,
                      float* lse_part, int32_t* units, const Dev& dev, cudaStream_t st) {
  K3Args a{};
  a.s0 = s0; a.e = e; a.hq = hq; a.hkv = hkv; a.G = hq / hkv;
  a.L = p->dca_chunk - p->local_window;
  a.nqb = (int)((e - s0 + 127) / 128);
  a.npair = (a.nqb + 1) / 2;
  a.ld_rows = ld_rows; a.ld_tokens = ld_tokens;
  a.mask = mask; a.resid = resid; a.cnt = cnt;
  a.nkw = (int)(((e + 127) / 128 + 31) / 32);
  a.nvcap = (int)(p->vs_vertical < e ? p->vs_vertical : e);
  a.k_rot = k_rot; a.v16 = v16;
  a.o_part = o_part; a.lse_part = lse_part;
  a.units = units + 8;
  a.n_units = units;
  a.aligned = deterministic_on() ? 0 : 1;
  const int U = 3 * a.npair;
  Q1M_CUDA(cudaFuncSetAttribute(k3_units_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, U * 4));
  k3_units_kernel<<<1, 1024, (size_t)U * 4, st>>>(s0, a.nqb, a.L, units + 8, units);
  Q1M_LAUNCHED();
  CUtensorMap mq, mk, mv;
  Q1M_TRY(make_map(&mq, qv, D, (uint64_t)3 * hq * ld_rows, 64, 128));
  Q1M_TRY(make_map(&mk, k_rot, D, (uint64_t)hkv * ld_tokens, 64, 128));
  Q1M_TRY(make_map(&mv, v16, D, (uint64_t)hkv * ld_tokens, 64, 128));
  const size_t smem = sizeof(K3Smem<D>) + 1024;
  Q1M_CUDA(cudaFuncSetAttribute(block_sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int64_t items_max = (int64_t)U * hq;
  const int grid = (int)(items_max < dev.sms ? items_max : dev.sms);
  const int pr = prof_begin(Q1M_STAGE_ATTN, st);
  block_sparse_attn_kernel<D><<<grid, K3_THREADS, smem, st>>>(mq, mk, mv, a);
  prof_end(pr, st);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

q1m_status run_merge(const float* o_part, const float* lse_part, int n_parts, int64_t ld_rows,
                     int64_t s0, int64_t e, int64_t n, int hq, int d, int out_dtype, int64_t L,
                     void* out, float* lse, cudaStream_t st) {
  const int64_t warps = (e - s0) * hq;
  const int grid = blocks_for(warps * 32, 256);
  if (out_dtype == Q1M_BF16) {
    if (d == 128) lse_merge_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(o_part, lse_part, n_parts, ld_rows, s0, e, hq, L, (__nv_bfloat16*)out, lse, n);
    else lse_merge_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(o_part, lse_part, n_parts, ld_rows, s0, e, hq, L, (__nv_bfloat16*)out, lse, n);
  } else {
    if (d == 128) lse_merge_kernel<float, 128><<<grid, 256, 0, st>>>(o_part, lse_part, n_parts, ld_rows, s0, e, hq, L, (float*)out, lse, n);
    else lse_merge_kernel<float, 64><<<grid, 256, 0, st>>>(o_part, lse_part, n_parts, ld_rows, s0, e, hq, L, (float*)out, lse, n);
  }
  Q1M_LAUNCHED();
  return Q1M_OK;
}

struct DecScratch {
  size_t qv, o_part, lse_part, total;
};

DecScratch dec_scratch(int hq, int d) {
  DecScratch L{};
  size_t off = 0;
  L.qv = off; off = align_up(off + (size_t)3 * hq * d * 2);
  L.o_part = off; off = align_up(off + (size_t)DEC_MAX_SPLIT * hq * d * 4);
  L.lse_part = off; off = align_up(off + (size_t)DEC_MAX_SPLIT * hq * 4);
  L.total = off;
  return L;
}

template <int D, typename T>
q1m_status run_decode_d(const T* q, const T* k, const T* v, int64_t pos, uint16_t* k_rot,
                        uint16_t* v16, int64_t ld_tokens, int hq, int hkv, const q1m_params* p,
                        const float* table, void* out, float* lse, void* scratch, const Dev& dev,
                        cudaStream_t st) {
  const DecScratch SL = dec_scratch(hq, D);
  const int64_t L = p->dca_chunk - p->local_window;
  uint16_t* qv = at<uint16_t>(scratch, SL.qv);
  float* o_part = at<float>(scratch, SL.o_part);
  float* lse_part = at<float>(scratch, SL.lse_part);
  const float2* tab = reinterpret_cast<const float2*>(table);
  const int64_t rows = (pos / DEC_TILE + 1) * DEC_TILE - pos;
  dec_append_kernel<T><<<blocks_for((int64_t)hkv * rows * (D / 2), 256), 256, 0, st>>>(
      k, v, hkv, D, pos, L, ld_tokens, tab, k_rot, v16);
  Q1M_LAUNCHED();
  dec_queries_kernel<T><<<blocks_for((int64_t)3 * hq * (D / 2), 256), 256, 0, st>>>(
      q, hq, D, pos, L, p->dca_chunk, tab, view_scale(p, D), qv);
  Q1M_LAUNCHED();
  DecArgs a{};
  a.qv = qv; a.pos = pos; a.L = L; a.n_keys = pos + 1;
  a.hq = hq; a.G = hq / hkv; a.ld_tokens = ld_tokens;
  a.n_tiles = (pos + 1 + DEC_TILE - 1) / DEC_TILE;
  int64_t ns = (dev.sms + hkv - 1) / hkv;
  const int64_t by_tiles = (a.n_tiles + DEC_WARPS - 1) / DEC_WARPS;   // at least a tile per warp
  ns = ns < by_tiles ? ns : by_tiles;
  ns = ns < DEC_MAX_SPLIT ? ns : DEC_MAX_SPLIT;
  ns = ns < 1 ? 1 : ns;
  a.tiles_per_split = (a.n_tiles + ns - 1) / ns;
  a.nsplit = (int)((a.n_tiles + a.tiles_per_split - 1) / a.tiles_per_split);
  a.o_part = o_part; a.lse_part = lse_part;
  CUtensorMap mk, mv;
  Q1M_TRY(make_map(&mk, k_rot, D, (uint64_t)hkv * ld_tokens, 64, DEC_TILE));
  Q1M_TRY(make_map(&mv, v16, D, (uint64_t)hkv * ld_tokens, 64, DEC_TILE));
  const size_t smem = sizeof(DecSmem<D>) + 1024;
  Q1M_CUDA(cudaFuncSetAttribute(dca_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int pr = prof_begin(Q1M_STAGE_DECODE, st);
  dca_decode_kernel<D><<<dim3(a.nsplit, hkv), 32 * DEC_WARPS, smem, st>>>(mk, mv, a);
  prof_end(pr, st);
  Q1M_LAUNCHED();
  const int grid = blocks_for((int64_t)hq * 32, 256);
  if (p->out_dtype == Q1M_BF16)
    dec_merge_kernel<__nv_bfloat16, D><<<grid, 256, 0, st>>>(o_part, lse_part, a.nsplit, hq, (__nv_bfloat16*)out, lse);
  else
    dec_merge_kernel<float, D><<<grid, 256, 0, st>>>(o_part, lse_part, a.nsplit, hq, (float*)out, lse);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

}  // namespace

// =============================================================================================
// C ABI
// =============================================================================================
extern "C" {

const char* q1m_version(void) { return "q1m 0.1 (sm_100a)"; }

const char* q1m_last_error(void) { return t_err.c_str(); }

size_t q1m_workspace_bytes(int64_t n, int hq, int hkv, int d, const q1m_params* p) {
  if (check_shape(n, hq, hkv, d, p) != Q1M_OK || check_chunks(n, p) != Q1M_OK) return 0;
  return layout(n, hq, hkv, d, p).total;
}

size_t q1m_host_workspace_bytes(int64_t n, int hq, int hkv, int d, const q1m_params* p) {
  if (check_shape(n, hq, hkv, d, p) != Q1M_OK || check_chunks(n, p) != Q1M_OK) return 0;
  const size_t ein = p->in_dtype == Q1M_BF16 ? 2 : 4, eout = p->out_dtype == Q1M_BF16 ? 2 : 4;
  return align_up((size_t)n * hq * d * ein) + 2 * align_up((size_t)n * hkv * d * ein) +
         align_up((size_t)n * hq * d * eout) + align_up((size_t)n * hq * 4) +
         layout(n, hq, hkv, d, p).total;
}

q1m_status q1m_rope_table(float* table, int64_t n_pos, int d, double base, void* stream) {
  if (!table || n_pos <= 0) return fail(Q1M_ERR_INVALID, "bad table arguments");
  if (d != 64 && d != 128) return fail(Q1M_ERR_UNSUPPORTED, "head_dim %d", d);
  if (!(base > 1.0)) return fail(Q1M_ERR_INVALID, "rope_base must be > 1");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  return run_rope_table(table, n_pos, d, base, S(stream));
}

q1m_status q1m_rope_dca_keys(const void* k, const void* v, int64_t s0, int64_t e, int hkv, int d,
                             const q1m_params* p, const float* table, uint16_t* k_rot, uint16_t* v16,
                             int64_t ld_tokens, void* stream) {
  Q1M_TRY(check_shape(e > 0 ? e : 1, hkv, hkv, d, p));
  if (!k || !v || !table || !k_rot || !v16) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(table) |
        reinterpret_cast<uintptr_t>(k_rot) | reinterpret_cast<uintptr_t>(v16)) & 15) != 0)
    return fail(Q1M_ERR_INVALID, "k, v, table, k_rot and v16 must be 16-byte aligned");
  if (s0 < 0 || e <= s0 || ld_tokens < e || ld_tokens % 128) return fail(Q1M_ERR_INVALID, "bad token range");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  return run_rope_keys(k, v, s0, e, hkv, d, p, table, k_rot, v16, ld_tokens, S(stream));
}

q1m_status q1m_rope_dca_queries(const void* q, int64_t s0, int64_t e, int hq, int d,
                                const q1m_params* p, const float* table, uint16_t* qv,
                                int64_t ld_rows, void* stream) {
  Q1M_TRY(check_shape(e > 0 ? e : 1, hq, hq, d, p));
  if (!q || !table || !qv) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(table) | reinterpret_cast<uintptr_t>(qv)) & 15) != 0)
    return fail(Q1M_ERR_INVALID, "q, table and qv must be 16-byte aligned");
  if (s0 < 0 || e <= s0 || ld_rows < e - s0 || ld_rows % 128) return fail(Q1M_ERR_INVALID, "bad row range");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  return run_rope_queries(q, s0, e, hq, d, p, table, qv, ld_rows, S(stream));
}

size_t q1m_vs_estimate_scratch_bytes(int64_t e, int hq, int hkv, int d) {
  if (e <= 0 || hq <= 0 || hkv <= 0 || hq % hkv || (d != 64 && d != 128)) return 0;
  return est_layout(e, hq, hkv, d).total;
}

q1m_status q1m_vs_estimate(const void* q, const uint16_t* k_rot, int64_t ld_tokens, int64_t s0,
                           int64_t e, int hq, int hkv, int d, const q1m_params* p, const float* table,
                           float* vert, float* slash, int64_t ld, void* scratch, size_t scratch_bytes,
                           void* stream) {
  Q1M_TRY(check_shape(e > 0 ? e : 1, hq, hkv, d, p));
  if (!sparse(p)) return fail(Q1M_ERR_INVALID, "estimator needs a sparse budget");
  if (!q || !k_rot || !table || !vert || !slash || !scratch) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (s0 < 0 || e <= s0 || ld < e || ld_tokens < e || ld_tokens % 128) return fail(Q1M_ERR_INVALID, "bad range");
  if (scratch_bytes < q1m_vs_estimate_scratch_bytes(e, hq, hkv, d)) return fail(Q1M_ERR_WORKSPACE, "estimator scratch too small");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  if (d == 128) return run_estimate_d<128>(q, k_rot, ld_tokens, s0, e, hq, hkv, p, table, vert, slash, ld, scratch, dev, S(stream));
  return run_estimate_d<64>(q, k_rot, ld_tokens, s0, e, hq, hkv, p, table, vert, slash, ld, scratch, dev, S(stream));
}

size_t q1m_vs_select_scratch_bytes(int64_t e, int hq) { (void)e; (void)hq; return 0; }

q1m_status q1m_vs_select(const float* vert, const float* slash, int64_t ld, int64_t e, int hq,
                         const q1m_params* p, int32_t* V, int32_t* Sx, void* scratch,
                         size_t scratch_bytes, void* stream) {
  (void)scratch; (void)scratch_bytes;
  if (!p || !vert || !slash || !Sx || (p->vs_vertical > 0 && !V)) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (e <= 0 || ld < e || hq <= 0) return fail(Q1M_ERR_INVALID, "bad sizes");
  if (p->vs_vertical < 0 || p->vs_slash < 1 || p->vs_force_local < 0) return fail(Q1M_ERR_INVALID, "bad budgets");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  return run_select(vert, slash, ld, e, hq, p, V, Sx, S(stream));
}

q1m_status q1m_vs_build_masks(const int32_t* V, const int32_t* Sx, int64_t s0, int64_t e, int hq,
                              const q1m_params* p, uint32_t* mask, int32_t* resid, int32_t* cnt,
                              void* stream) {
  if (!p || !Sx || !mask || !cnt || (p->vs_vertical > 0 && (!V || !resid))) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (s0 < 0 || e <= s0 || s0 % 128 || hq <= 0) return fail(Q1M_ERR_INVALID, "bad range");
  if (p->dca_chunk <= p->local_window || (p->dca_chunk - p->local_window) % 128) return fail(Q1M_ERR_UNSUPPORTED, "DCA chunk length must be a multiple of 128");
  if (((e + 127) / 128 + 31) / 32 > MB_MAX_NKW) return fail(Q1M_ERR_UNSUPPORTED, "too many key blocks");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  return run_masks(V, Sx, s0, e, hq, p, mask, resid, cnt, S(stream));
}

size_t q1m_attn_scratch_bytes(int64_t s0, int64_t e, int hq, int d) {
  (void)hq; (void)d;
  if (e <= s0) return 0;
  const int64_t nqb = (e - s0 + 127) / 128;
  return (size_t)(3 * (nqb + 1) / 2 + 8) * 4;
}

q1m_status q1m_block_sparse_attn(const uint16_t* qv, int64_t ld_rows, const uint16_t* k_rot,
                                 const uint16_t* v16, int64_t ld_tokens, const uint32_t* mask,
                                 const int32_t* resid, const int32_t* cnt, int64_t s0, int64_t e,
                                 int hq, int hkv, int d, const q1m_params* p, float* o_part,
                                 float* lse_part, void* scratch, size_t scratch_bytes, void* stream) {
  Q1M_TRY(check_shape(e > 0 ? e : 1, hq, hkv, d, p));
  if (!qv || !k_rot || !v16 || !o_part || !lse_part || !scratch) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (mask && (!cnt || (p->vs_vertical > 0 && !resid))) return fail(Q1M_ERR_INVALID, "mask without counts/residuals");
  if (s0 < 0 || e <= s0 || s0 % 128 || ld_rows < e - s0 || ld_rows % 128 || ld_tokens < e || ld_tokens % 128)
    return fail(Q1M_ERR_INVALID, "bad range");
  if ((e - s0 + 127) / 128 > Q1M_MAX_CHUNK_QUERY_BLOCKS)
    return fail(Q1M_ERR_UNSUPPORTED, "a chunk of %lld query blocks exceeds %d", (long long)((e - s0 + 127) / 128),
                Q1M_MAX_CHUNK_QUERY_BLOCKS);
  if (scratch_bytes < q1m_attn_scratch_bytes(s0, e, hq, d)) return fail(Q1M_ERR_WORKSPACE, "attention scratch too small");
  if (reinterpret_cast<uintptr_t>(scratch) & 3) return fail(Q1M_ERR_INVALID, "scratch misaligned");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  int32_t* units = static_cast<int32_t*>(scratch);
  if (d == 128) return run_attn_d<128>(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, S(stream));
  return run_attn_d<64>(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, S(stream));
}

q1m_status q1m_lse_merge(const float* o_part, const float* lse_part, int n_parts, int64_t ld_rows,
                         int64_t s0, int64_t e, int64_t n, int hq, int d, int out_dtype,
                         const q1m_params* p, void* out, float* lse, void* stream) {
  if (!o_part || !lse_part || !out) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (n_parts < 1 || n_parts > 3) return fail(Q1M_ERR_INVALID, "n_parts must be 1..3");
  if (s0 < 0 || e <= s0 || e > n || ld_rows < e - s0 || hq <= 0) return fail(Q1M_ERR_INVALID, "bad range");
  if (d != 64 && d != 128) return fail(Q1M_ERR_UNSUPPORTED, "head_dim %d", d);
  if (out_dtype != Q1M_BF16 && out_dtype != Q1M_F32) return fail(Q1M_ERR_INVALID, "bad out_dtype");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  const int64_t Ld = p ? p->dca_chunk - p->local_window : 0;
  if (p && Ld <= 0) return fail(Q1M_ERR_INVALID, "bad DCA chunk length");
  return run_merge(o_part, lse_part, n_parts, ld_rows, s0, e, n, hq, d, out_dtype, Ld, out, lse, S(stream));
}

q1m_status q1m_dca_sparse_prefill(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int64_t n, int hq, int hkv, int d,
                                  const q1m_params* p, void* ws, size_t ws_bytes, void* stream) {
  return q1m_dca_sparse_prefill_chunks(q, k, v, out, lse, n, hq, hkv, d, p, 0, INT64_MAX, ws,
                                       ws_bytes, stream);
}

// Host-side hooks around each prefill chunk of prefill_range, called when the chunk's work
// is enqueued (before its first stage and after its merge).
struct ChunkHooks {
  virtual q1m_status before(int64_t s0, int64_t e) = 0;
  virtual q1m_status after(int64_t s0, int64_t e) = 0;
};

static q1m_status prefill_range(const void* q, const void* k, const void* v, void* out,
                                float* lse, int64_t n, int hq, int hkv, int d,
                                const q1m_params* p, int64_t first_chunk, int64_t last_chunk,
                                void* ws, size_t ws_bytes, void* stream, ChunkHooks* hooks);

q1m_status q1m_dca_sparse_prefill_chunks(const void* q, const void* k, const void* v, void* out,
                                         float* lse, int64_t n, int hq, int hkv, int d,
                                         const q1m_params* p, int64_t first_chunk,
                                         int64_t last_chunk, void* ws, size_t ws_bytes,
                                         void* stream) {
  return prefill_range(q, k, v, out, lse, n, hq, hkv, d, p, first_chunk, last_chunk, ws, ws_bytes,
                       stream, nullptr);
}

static q1m_status prefill_range(const void* q, const void* k, const void* v, void* out,
                                float* lse, int64_t n, int hq, int hkv, int d,
                                const q1m_params* p, int64_t first_chunk, int64_t last_chunk,
                                void* ws, size_t ws_bytes, void* stream, ChunkHooks* hooks) {
  Q1M_TRY(check_shape(n, hq, hkv, d, p));
  Q1M_TRY(check_chunks(n, p));
  if (first_chunk < 0 || last_chunk < first_chunk) return fail(Q1M_ERR_INVALID, "bad chunk range");
  if (!q || !k || !v || !out || !ws) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(Q1M_ERR_INVALID, "workspace must be 256-byte aligned");
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) != 0)
    return fail(Q1M_ERR_INVALID, "q, k and v must be 16-byte aligned");
  const Layout L = layout(n, hq, hkv, d, p);
  if (ws_bytes < L.total) return fail(Q1M_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  Dev dev;
  Q1M_TRY(device_info(&dev));
  cudaStream_t st = S(stream);
  float* table = at<float>(ws, L.table);
  uint16_t* k_rot = at<uint16_t>(ws, L.k_rot);
  uint16_t* v16 = at<uint16_t>(ws, L.v16);
  uint16_t* qv = at<uint16_t>(ws, L.qv);
  float* o_part = at<float>(ws, L.o_part);
  float* lse_part = at<float>(ws, L.lse_part);
  int32_t* units = at<int32_t>(ws, L.units);
  const int64_t Ld = p->dca_chunk - p->local_window;
  // debug mode: guard regions get their pattern at the start of every call
  for (int gi = 0; gi < L.guards.n; ++gi)
    Q1M_CUDA(cudaMemsetAsync(at<uint8_t>(ws, L.guards.off[gi]), 0xA5, GUARD_BYTES, st));
  int pr = prof_begin(Q1M_STAGE_TABLE, st);
  Q1M_TRY(run_rope_table(table, p->dca_chunk, d, p->rope_base, st));
  prof_end(pr, st);
  Q1M_TRY(debug_after(L, ws, Q1M_STAGE_TABLE, true, st));
  if (L.ld_tokens > n) {
    // zero the padded key rows once so tiles past the end read finite values
    for (int g = 0; g < hkv; ++g) {
      Q1M_CUDA(cudaMemsetAsync(k_rot + ((int64_t)g * L.ld_tokens + n) * d, 0, (size_t)(L.ld_tokens - n) * d * 2, st));
      Q1M_CUDA(cudaMemsetAsync(v16 + ((int64_t)g * L.ld_tokens + n) * d, 0, (size_t)(L.ld_tokens - n) * d * 2, st));
    }
  }
  const std::vector<int64_t> ends = chunk_ends(n, p);
  for (int64_t ci = first_chunk; ci < (int64_t)ends.size() && ci < last_chunk; ++ci) {
    const int64_t s0 = ci == 0 ? 0 : ends[ci - 1], e = ends[ci];
    const bool first = ci == first_chunk;
    if (hooks) Q1M_TRY(hooks->before(s0, e));
    pr = prof_begin(Q1M_STAGE_KEYS, st);
    Q1M_TRY(run_rope_keys(k, v, s0, e, hkv, d, p, table, k_rot, v16, L.ld_tokens, st));
    prof_end(pr, st);
    Q1M_TRY(debug_after(L, ws, Q1M_STAGE_KEYS, first, st));
    pr = prof_begin(Q1M_STAGE_QUERIES, st);
    Q1M_TRY(run_rope_queries(q, s0, e, hq, d, p, table, qv, L.ld_rows, st));
    prof_end(pr, st);
    Q1M_TRY(debug_after(L, ws, Q1M_STAGE_QUERIES, first, st));
    const uint32_t* mask = nullptr;
    const int32_t *resid = nullptr, *cnt = nullptr;
    if (sparse(p)) {
      float* vert = at<float>(ws, L.vert);
      float* slash = at<float>(ws, L.slash);
      int32_t* V = at<int32_t>(ws, L.V);
      int32_t* Sx = at<int32_t>(ws, L.Sx);
      pr = prof_begin(Q1M_STAGE_ESTIMATE, st);
      if (d == 128) Q1M_TRY(run_estimate_d<128>(q, k_rot, L.ld_tokens, s0, e, hq, hkv, p, table, vert, slash, L.ld_tokens, at<void>(ws, L.est), dev, st));
      else Q1M_TRY(run_estimate_d<64>(q, k_rot, L.ld_tokens, s0, e, hq, hkv, p, table, vert, slash, L.ld_tokens, at<void>(ws, L.est), dev, st));
      prof_end(pr, st);
      Q1M_TRY(debug_after(L, ws, Q1M_STAGE_ESTIMATE, first, st));
      pr = prof_begin(Q1M_STAGE_SELECT, st);
      Q1M_TRY(run_select(vert, slash, L.ld_tokens, e, hq, p, V, Sx, st));
      prof_end(pr, st);
      Q1M_TRY(debug_after(L, ws, Q1M_STAGE_SELECT, first, st));
      pr = prof_begin(Q1M_STAGE_MASKS, st);
      Q1M_TRY(run_masks(V, Sx, s0, e, hq, p, at<uint32_t>(ws, L.mask), at<int32_t>(ws, L.resid), at<int32_t>(ws, L.cnt), st));
      prof_end(pr, st);
      Q1M_TRY(debug_after(L, ws, Q1M_STAGE_MASKS, first, st));
      if (L.guards.n > 0) {
        const int nv_e = (int)(p->vs_vertical < e ? p->vs_vertical : e);
        const int ns_e = (int)(p->vs_slash < e ? p->vs_slash : e);
        index_check_kernel<<<blocks_for(hq, 32), 32, 0, st>>>(
            V, nv_e, Sx, ns_e, e, hq, p->vs_force_local, at<int32_t>(ws, L.cnt), at<int32_t>(ws, L.resid),
            (int)((e - s0 + 127) / 128), nv_e, (e + 127) / 128);
        Q1M_LAUNCHED();
      }
      mask = at<uint32_t>(ws, L.mask);
      resid = at<int32_t>(ws, L.resid);
      cnt = at<int32_t>(ws, L.cnt);
    }
    if (d == 128) Q1M_TRY(run_attn_d<128>(qv, L.ld_rows, k_rot, v16, L.ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, st));
    else Q1M_TRY(run_attn_d<64>(qv, L.ld_rows, k_rot, v16, L.ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, st));
    Q1M_TRY(debug_after(L, ws, Q1M_STAGE_ATTN, first, st));
    pr = prof_begin(Q1M_STAGE_MERGE, st);
    Q1M_TRY(run_merge(o_part, lse_part, 3, L.ld_rows, s0, e, n, hq, d, p->out_dtype, Ld, out, lse, st));
    prof_end(pr, st);
    Q1M_TRY(debug_after(L, ws, Q1M_STAGE_MERGE, first, st));
    if (hooks) Q1M_TRY(hooks->after(s0, e));
  }
  return Q1M_OK;
}

// The host-buffer path's copies, one prefill chunk at a time on two copy streams of the
// call's own: chunk c's rows of q, k and v go up on `up` while earlier chunks compute, and
// its rows of out and lse come down on `down` while later chunks compute. A chunk reads
// only its own rows of q, k and v (the rotated keys of earlier chunks are in the workspace),
// so the compute stream waits only for that chunk's upload.
struct HostCopies final : ChunkHooks {
  const uint8_t *q_h = nullptr, *k_h = nullptr, *v_h = nullptr;
  uint8_t* out_h = nullptr;
  float* lse_h = nullptr;
  uint8_t *dq = nullptr, *dk = nullptr, *dv = nullptr, *dout = nullptr;
  float* dlse = nullptr;
  size_t row_q = 0, row_k = 0, row_o = 0;   // bytes per token of q, of k (and v), of out
  int64_t n = 0;
  int hq = 0;
  cudaStream_t st = nullptr, up = nullptr, down = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr, ev_edge = nullptr;

  q1m_status open() {
    Q1M_CUDA(cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking));
    Q1M_CUDA(cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking));
    Q1M_CUDA(cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming));
    Q1M_CUDA(cudaEventCreateWithFlags(&ev_out, cudaEventDisableTiming));
    Q1M_CUDA(cudaEventCreateWithFlags(&ev_edge, cudaEventDisableTiming));
    // the uploads start after the work already queued on the caller's stream
    Q1M_CUDA(cudaEventRecord(ev_edge, st));
    Q1M_CUDA(cudaStreamWaitEvent(up, ev_edge, 0));
    return Q1M_OK;
  }
  q1m_status before(int64_t s0, int64_t e) override {
    const size_t r = (size_t)(e - s0);
    Q1M_CUDA(cudaMemcpyAsync(dq + s0 * row_q, q_h + s0 * row_q, r * row_q, cudaMemcpyHostToDevice, up));
    Q1M_CUDA(cudaMemcpyAsync(dk + s0 * row_k, k_h + s0 * row_k, r * row_k, cudaMemcpyHostToDevice, up));
    Q1M_CUDA(cudaMemcpyAsync(dv + s0 * row_k, v_h + s0 * row_k, r * row_k, cudaMemcpyHostToDevice, up));
    Q1M_CUDA(cudaEventRecord(ev_in, up));
    Q1M_CUDA(cudaStreamWaitEvent(st, ev_in, 0));
    return Q1M_OK;
  }
  q1m_status after(int64_t s0, int64_t e) override {
    const size_t r = (size_t)(e - s0);
    Q1M_CUDA(cudaEventRecord(ev_out, st));
    Q1M_CUDA(cudaStreamWaitEvent(down, ev_out, 0));
    Q1M_CUDA(cudaMemcpyAsync(out_h + s0 * row_o, dout + s0 * row_o, r * row_o, cudaMemcpyDeviceToHost, down));
    if (lse_h)   // rows [s0, e) of every head of the [Hq][N] array
      Q1M_CUDA(cudaMemcpy2DAsync(lse_h + s0, (size_t)n * 4, dlse + s0, (size_t)n * 4, r * 4, hq,
                                 cudaMemcpyDeviceToHost, down));
    return Q1M_OK;
  }
  // the caller's stream then follows the downloads
  q1m_status close() {
    Q1M_CUDA(cudaEventRecord(ev_edge, down));
    Q1M_CUDA(cudaStreamWaitEvent(st, ev_edge, 0));
    return Q1M_OK;
  }
  ~HostCopies() {
    if (up) { cudaStreamSynchronize(up); cudaStreamDestroy(up); }
    if (down) { cudaStreamSynchronize(down); cudaStreamDestroy(down); }
    if (ev_in) cudaEventDestroy(ev_in);
    if (ev_out) cudaEventDestroy(ev_out);
    if (ev_edge) cudaEventDestroy(ev_edge);
  }
};

q1m_status q1m_dca_sparse_prefill_host(const void* q_h, const void* k_h, const void* v_h, void* out_h,
                                       float* lse_h, int64_t n, int hq, int hkv, int d,
                                       const q1m_params* p, void* ws, size_t ws_bytes, void* stream) {
  Q1M_TRY(check_shape(n, hq, hkv, d, p));
  Q1M_TRY(check_chunks(n, p));
  if (!q_h || !k_h || !v_h || !out_h || !ws) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(Q1M_ERR_INVALID, "workspace must be 256-byte aligned");
  if (ws_bytes < q1m_host_workspace_bytes(n, hq, hkv, d, p)) return fail(Q1M_ERR_WORKSPACE, "host-path workspace too small");
  const size_t ein = p->in_dtype == Q1M_BF16 ? 2 : 4, eout = p->out_dtype == Q1M_BF16 ? 2 : 4;
  const size_t bq = (size_t)n * hq * d * ein, bk = (size_t)n * hkv * d * ein, bo = (size_t)n * hq * d * eout;
  size_t off = 0;
  void* dq = at<void>(ws, off); off += align_up(bq);
  void* dk = at<void>(ws, off); off += align_up(bk);
  void* dv = at<void>(ws, off); off += align_up(bk);
  void* dout = at<void>(ws, off); off += align_up(bo);
  float* dlse = at<float>(ws, off); off += align_up((size_t)n * hq * 4);
  HostCopies hc;
  hc.q_h = static_cast<const uint8_t*>(q_h);
  hc.k_h = static_cast<const uint8_t*>(k_h);
  hc.v_h = static_cast<const uint8_t*>(v_h);
  hc.out_h = static_cast<uint8_t*>(out_h);
  hc.lse_h = lse_h;
  hc.dq = static_cast<uint8_t*>(dq);
  hc.dk = static_cast<uint8_t*>(dk);
  hc.dv = static_cast<uint8_t*>(dv);
  hc.dout = static_cast<uint8_t*>(dout);
  hc.dlse = dlse;
  hc.row_q = (size_t)hq * d * ein;
  hc.row_k = (size_t)hkv * d * ein;
  hc.row_o = (size_t)hq * d * eout;
  hc.n = n;
  hc.hq = hq;
  hc.st = S(stream);
  Q1M_TRY(hc.open());
  Q1M_TRY(prefill_range(dq, dk, dv, dout, lse_h ? dlse : nullptr, n, hq, hkv, d, p, 0, INT64_MAX,
                        at<void>(ws, off), ws_bytes - off, stream, &hc));
  Q1M_TRY(hc.close());
  return q1m_status_poll(stream);
}

size_t q1m_dca_decode_scratch_bytes(int hq, int d) {
  if (hq <= 0 || (d != 64 && d != 128)) return 0;
  return dec_scratch(hq, d).total;
}

q1m_status q1m_dca_decode(const void* q, const void* k, const void* v, int64_t pos, uint16_t* k_rot,
                          uint16_t* v16, int64_t ld_tokens, int hq, int hkv, int d,
                          const q1m_params* p, const float* table, void* out, float* lse,
                          void* scratch, size_t scratch_bytes, void* stream) {
  if (pos < 0) return fail(Q1M_ERR_INVALID, "pos must be >= 0");
  Q1M_TRY(check_shape(pos + 1, hq, hkv, d, p));
  if (hq / hkv > 8) return fail(Q1M_ERR_UNSUPPORTED, "decode supports at most 8 Q heads per KV head");
  if (!q || !k || !v || !k_rot || !v16 || !table || !out || !scratch) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (ld_tokens <= pos || ld_tokens % 128) return fail(Q1M_ERR_INVALID, "ld_tokens must be a multiple of 128 and > pos");
  if ((int64_t)hkv * ld_tokens >= ((int64_t)1 << 31)) return fail(Q1M_ERR_UNSUPPORTED, "n_kv_heads * ld_tokens too large");
  if (scratch_bytes < q1m_dca_decode_scratch_bytes(hq, d)) return fail(Q1M_ERR_WORKSPACE, "decode scratch too small");
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return fail(Q1M_ERR_INVALID, "scratch must be 256-byte aligned");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  cudaStream_t st = S(stream);
  if (p->in_dtype == Q1M_BF16) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    if (d == 128) return run_decode_d<128>(qq, kk, vv, pos, k_rot, v16, ld_tokens, hq, hkv, p, table, out, lse, scratch, dev, st);
    return run_decode_d<64>(qq, kk, vv, pos, k_rot, v16, ld_tokens, hq, hkv, p, table, out, lse, scratch, dev, st);
  }
  auto* qq = static_cast<const float*>(q);
  auto* kk = static_cast<const float*>(k);
  auto* vv = static_cast<const float*>(v);
  if (d == 128) return run_decode_d<128>(qq, kk, vv, pos, k_rot, v16, ld_tokens, hq, hkv, p, table, out, lse, scratch, dev, st);
  return run_decode_d<64>(qq, kk, vv, pos, k_rot, v16, ld_tokens, hq, hkv, p, table, out, lse, scratch, dev, st);
}

int64_t q1m_prefill_bounds(int64_t n, const q1m_params* p, int64_t* ends, int64_t max_chunks) {
  if (!p || !ends || n <= 0 || max_chunks <= 0) return fail(Q1M_ERR_INVALID, "bad arguments");
  if (p->equal_cost_chunks < 0) return fail(Q1M_ERR_INVALID, "equal_cost_chunks must be >= 0");
  if (p->equal_cost_chunks == 0 && (p->prefill_chunk <= 0 || p->prefill_chunk % 128 != 0))
    return fail(Q1M_ERR_INVALID, "prefill_chunk must be a positive multiple of 128");
  const std::vector<int64_t> e = chunk_ends(n, p);
  if ((int64_t)e.size() > max_chunks) return fail(Q1M_ERR_WORKSPACE, "%zu chunks > max_chunks", e.size());
  for (size_t i = 0; i < e.size(); ++i) ends[i] = e[i];
  return (int64_t)e.size();
}

q1m_status q1m_status_poll(void* stream) {
  cudaError_t e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return fail(Q1M_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
  int st = 0;
  Q1M_CUDA(cudaMemcpyFromSymbol(&st, g_status, sizeof(int)));
  if (st != 0) {
    const int zero = 0, none = -1;
    int info = -1;
    Q1M_CUDA(cudaMemcpyFromSymbol(&info, g_check_info, sizeof(int)));
    Q1M_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)));
    Q1M_CUDA(cudaMemcpyToSymbol(g_check_info, &none, sizeof(int)));
    if (st == Q1M_ERR_CHECK) {
      static const char* lists[] = {"", "vertical columns", "slash offsets", "forced diagonals",
                                    "block counts", "residual counts", "residual columns"};
      if (info >= 1000 && info < 1007) return fail(Q1M_ERR_CHECK, "debug check: malformed %s", lists[info - 1000]);
      return fail(Q1M_ERR_CHECK, "debug check: workspace guard region %d overwritten", info);
    }
    return fail((q1m_status)st, st == Q1M_ERR_TIMEOUT ? "a device-side wait ran out" : "device-side range/NaN check failed");
  }
  return Q1M_OK;
}

q1m_status q1m_set_deterministic(int on) {
  g_determ.store(on ? 1 : 0);
  return Q1M_OK;
}

int q1m_deterministic(void) { return deterministic_on() ? 1 : 0; }

q1m_status q1m_set_debug(int on) {
  g_debug.store(on ? 1 : 0);
  return Q1M_OK;
}

int q1m_debug_enabled(void) { return debug_on() ? 1 : 0; }

q1m_status q1m_debug_inject(int stage) {
  if (stage < -1 || stage >= Q1M_NUM_STAGES) return fail(Q1M_ERR_INVALID, "bad stage %d", stage);
  g_inject.store(stage);
  return Q1M_OK;
}

q1m_status q1m_profile_enable(int on) {
  t_prof.on = on != 0;
  t_prof.used = 0;
  t_prof.recs.clear();
  return Q1M_OK;
}

q1m_status q1m_profile_read(double* ms, int64_t* launches) {
  if (!ms) return fail(Q1M_ERR_INVALID, "ms is NULL");
  for (int i = 0; i < Q1M_NUM_STAGES; ++i) { ms[i] = 0.0; if (launches) launches[i] = 0; }
  for (const ProfRec& r : t_prof.recs) {
    Q1M_CUDA(cudaEventSynchronize(r.b));
    float t = 0.f;
    Q1M_CUDA(cudaEventElapsedTime(&t, r.a, r.b));
    ms[r.stage] += t;
    if (launches) launches[r.stage] += 1;
  }
  t_prof.used = 0;
  t_prof.recs.clear();
  return Q1M_OK;
}

uint64_t q1m_launch_count(void) { return g_launches.load(); }

q1m_status q1m_set_wait_budget(uint64_t cycles) {
  unsigned long long v = cycles ? (unsigned long long)cycles : 2000000000ull;
  Q1M_CUDA(cudaMemcpyToSymbol(g_wait_cycles, &v, sizeof v));
  return Q1M_OK;
}

}  // extern "C"

namespace {
__global__ void recall_kernel(const float* __restrict__ ls, const float* __restrict__ ld, int64_t n,
                              float* __restrict__ r) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float d = ls[i] - ld[i];
  r[i] = d >= 0.f ? 1.f : expf(d);
}

__global__ void selftest_exp2_kernel(const float* x, float* yp, float* ym, float* yr, int64_t n) {
  const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (i + 1 >= n + 1) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  float pa, pb;
  f2_unpack(ex2_poly2(f2_pack(a, b)), pa, pb);
  yp[i] = pa; ym[i] = ex2(a); yr[i] = exp2f(a);
  if (i + 1 < n) { yp[i + 1] = pb; ym[i + 1] = ex2(b); yr[i + 1] = exp2f(b); }
}

// one warp waits on a barrier that no thread and no copy ever arrives on
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
  __syncwarp();
  mbar_wait(&bar, 0);
}
}  // namespace

extern "C" q1m_status q1m_attention_recall(const float* ls, const float* ld, int64_t n, float* r,
                                           void* stream) {
  if (!ls || !ld || !r || n <= 0) return fail(Q1M_ERR_INVALID, "bad arguments");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  recall_kernel<<<blocks_for(n, 256), 256, 0, S(stream)>>>(ls, ld, n, r);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

extern "C" q1m_status q1m_selftest_exp2(const float* x, float* yp, float* ym, float* yr, int64_t n,
                                        void* stream) {
  if (!x || !yp || !ym || !yr || n <= 0) return fail(Q1M_ERR_INVALID, "bad arguments");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  selftest_exp2_kernel<<<blocks_for((n + 1) / 2, 256), 256, 0, S(stream)>>>(x, yp, ym, yr, n);
  Q1M_LAUNCHED();
  return Q1M_OK;
}

extern "C" q1m_status q1m_selftest_wait_timeout(uint64_t cycles, void* stream) {
  Dev dev;
  Q1M_TRY(device_info(&dev));
  Q1M_TRY(q1m_status_poll(stream));
  Q1M_TRY(q1m_set_wait_budget(cycles ? cycles : 1000000ull));
  selftest_wait_kernel<<<1, 32, 0, S(stream)>>>();
  Q1M_LAUNCHED();
  const q1m_status st = q1m_status_poll(stream);
  Q1M_TRY(q1m_set_wait_budget(0));
  return st;
}

// =============================================================================================
// Allocation-free attention entry point: the work-unit list in a static device array.
// =============================================================================================
namespace {
static __device__ __align__(256) int32_t g_noalloc_units[Q1M_NOALLOC_UNITS];
static_assert(3 * (Q1M_NOALLOC_MAX_QUERY_BLOCKS + 1) / 2 + 8 <= Q1M_NOALLOC_UNITS,
              "the static work list holds the largest chunk it admits");
static_assert(Q1M_NOALLOC_MAX_QUERY_BLOCKS <= Q1M_MAX_CHUNK_QUERY_BLOCKS, "within the stage limit");
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
struct NoallocSlot {
  void* ctx = nullptr;       // the device's context when ptr was looked up
  int32_t* ptr = nullptr;
};
NoallocSlot g_noalloc_slot[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of g_noalloc_units on the current device. In host code the array's name is
// only a stand-in for the symbol, so the address is looked up with cudaGetSymbolAddress the
// first time a device is used, and again whenever that device's context differs from the one
// the address was taken in (a cudaDeviceReset reloads the module at another address).
q1m_status noalloc_units(int32_t** out) {
  int dev = 0;
  Q1M_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(Q1M_ERR_UNSUPPORTED, "device ordinal %d", dev);
  auto get = ctx_get_current();
  if (!get) return fail(Q1M_ERR_CUDA, "cuCtxGetCurrent unavailable");
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return fail(Q1M_ERR_CUDA, "cuCtxGetCurrent failed");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot& sl = g_noalloc_slot[dev];
  if (!sl.ptr || !ctx || sl.ctx != static_cast<void*>(ctx)) {
    void* ptr = nullptr;
    Q1M_CUDA(cudaGetSymbolAddress(&ptr, g_noalloc_units));   // binds the context if needed
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return fail(Q1M_ERR_CUDA, "no current CUDA context");
    sl.ptr = static_cast<int32_t*>(ptr);
    sl.ctx = ctx;
  }
  *out = sl.ptr;
  return Q1M_OK;
}
}  // namespace

extern "C" q1m_status q1m_block_sparse_attn_noalloc(
    const uint16_t* qv, int64_t ld_rows, const uint16_t* k_rot, const uint16_t* v16,
    int64_t ld_tokens, const uint32_t* mask, const int32_t* resid, const int32_t* cnt, int64_t s0,
    int64_t e, int hq, int hkv, int d, const q1m_params* p, float* o_part, float* lse_part,
    void* stream) {
  // the size limit first: a chunk the static list cannot hold is refused whatever else is passed
  if (e > s0 && s0 >= 0) {
    const int64_t nqb = (e - s0 + 127) / 128;
    if (nqb > Q1M_NOALLOC_MAX_QUERY_BLOCKS)
      return fail(Q1M_ERR_UNSUPPORTED, "chunk of %lld query blocks exceeds the static work list (%d blocks)",
                  (long long)nqb, Q1M_NOALLOC_MAX_QUERY_BLOCKS);
  }
  Q1M_TRY(check_shape(e > 0 ? e : 1, hq, hkv, d, p));
  if (!qv || !k_rot || !v16 || !o_part || !lse_part) return fail(Q1M_ERR_INVALID, "NULL pointer");
  if (mask && (!cnt || (p->vs_vertical > 0 && !resid))) return fail(Q1M_ERR_INVALID, "mask without counts/residuals");
  if (s0 < 0 || e <= s0 || s0 % 128 || ld_rows < e - s0 || ld_rows % 128 || ld_tokens < e || ld_tokens % 128)
    return fail(Q1M_ERR_INVALID, "bad range");
  Dev dev;
  Q1M_TRY(device_info(&dev));
  int32_t* units = nullptr;
  Q1M_TRY(noalloc_units(&units));
  if (d == 128) return run_attn_d<128>(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, S(stream));
  return run_attn_d<64>(qv, ld_rows, k_rot, v16, ld_tokens, mask, resid, cnt, s0, e, hq, hkv, p, o_part, lse_part, units, dev, S(stream));
}
