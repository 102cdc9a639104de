/*
 * q1m.h — C ABI of the B200 (sm_100a) library for long-context prefill attention of one
 * grouped-query attention layer: Dual Chunk Attention (DCA) position remapping, YaRN logit
 * scaling and vertical-slash sparse attention under chunked prefill.
 *
 * Sources (page title, section):
 *   [P2] "Qwen2.5-1M Technical Report" paper review (xllm-io): section 三 (GQA 28/4 and 40/8
 *        heads, RoPE), section 四 "Dual Chunk Attention" (intra-chunk, inter-chunk and
 *        successive-chunk patterns; Figure 2: remapped relative positions stay in the trained
 *        range), "YaRN 注意力缩放" (softmax(q^T k / (t sqrt(D))), sqrt(1/t) = 0.1 ln s + 1),
 *        "稀疏注意力机制" (MInference vertical-slash; Figure 4: key tokens chosen per prefill
 *        chunk; continuous relative positions).
 *   [P5] "Qwen2.5-1M リリース" (agentlenshq): "Sparse Attention" (chunked prefill, 32,768) and
 *        "Deploy Qwen2.5-1M Models Locally" (--max-num-batched-tokens 131072 = prefill chunk).
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned device memory; the library never allocates, frees or
 *     keeps them. Host pointers are named *_host.
 *   - Tensors are contiguous; q, k and v (and the rotation stages' table, qv, k_rot and v16)
 *     must be 16-byte aligned: the rotations read and write 16 bytes at a time. q / out are
 *     token-major [seq_len][n_q_heads][head_dim]; k / v are [seq_len][n_kv_heads][head_dim];
 *     lse is [n_q_heads][seq_len].
 *   - Arguments are validated synchronously; on failure nothing is launched and a negative
 *     q1m_status is returned (q1m_last_error() gives a message). Otherwise the work is
 *     queued on `stream` (a cudaStream_t, NULL = legacy default stream) and the call returns
 *     Q1M_OK at once. Device-side faults detected by the kernels (a bounded wait that ran
 *     out, an fp16 range overflow, a NaN score, and in debug mode an overwritten guard region
 *     or a malformed index list) are latched on the device and returned by q1m_status_poll().
 *   - Calls are thread-safe as long as concurrent calls use distinct workspaces/outputs.
 *   - head_dim is 64 or 128; n_q_heads is a multiple of n_kv_heads; (dca_chunk - local_window)
 *     and prefill_chunk are multiples of 128. Sparse mode takes at most 7 Q heads per KV head
 *     (the estimator's 7 x 64 rows per group fill its tensor-memory accumulator), decode at
 *     most 8; larger groups return Q1M_ERR_UNSUPPORTED. A prefill chunk holds at most
 *     Q1M_MAX_CHUNK_QUERY_BLOCKS query blocks of 128 rows; a layer or attention call with a
 *     larger chunk returns Q1M_ERR_UNSUPPORTED before anything is launched. Only sm_100a
 *     devices are supported; there is no CPU fallback.
 */
#ifndef Q1M_H_
#define Q1M_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  Q1M_OK = 0,
  Q1M_ERR_INVALID = -1,      /* a bad argument (null pointer, bad size or shape)          */
  Q1M_ERR_UNSUPPORTED = -2,  /* a valid case the library does not handle (head_dim, GPU) */
  Q1M_ERR_WORKSPACE = -3,    /* workspace too small                                        */
  Q1M_ERR_CUDA = -4,         /* a CUDA runtime call failed                                 */
  Q1M_ERR_TIMEOUT = -5,      /* a device-side bounded wait ran out (latched on the device) */
  Q1M_ERR_RANGE = -6,        /* fp16 overflow in the rotation stage, or a NaN score        */
  Q1M_ERR_CHECK = -7         /* debug mode: a workspace guard region was overwritten or an
                              * index list is malformed (q1m_set_debug)                      */
} q1m_status;

typedef enum { Q1M_BF16 = 0, Q1M_F32 = 1 } q1m_dtype;

/* Largest prefill chunk the attention stage takes, in 128-row query blocks (4,194,304 rows):
 * its work-unit sort keeps 3 x ceil(blocks / 2) costs in one CTA's shared memory. */
#define Q1M_MAX_CHUNK_QUERY_BLOCKS 32768

/* Layer parameters. Mirrors the pages' deployment knobs: dca_chunk / local_window (DCA),
 * yarn_s (YaRN ratio s), prefill_chunk (--max-num-batched-tokens) and the vertical-slash
 * budgets of the sparse estimator. */
typedef struct {
  int32_t in_dtype;        /* q1m_dtype of q, k, v                                         */
  int32_t out_dtype;       /* q1m_dtype of out                                             */
  double rope_base;        /* RoPE base, theta_f = base^(-2f/D), rotate-half pairing       */
  double yarn_s;           /* inference/training length ratio; <= 1 disables the scale     */
  int64_t dca_chunk;       /* c: trained length; one DCA chunk holds c - local_window tokens */
  int64_t local_window;    /* w: 0 <= w < c                                                */
  int32_t vs_vertical;     /* vertical budget per head (columns); 0 and 0 => dense         */
  int32_t vs_slash;        /* slash budget per head (diagonals)                            */
  int32_t vs_last_q;       /* estimator rows: the last vs_last_q rows of a chunk (1..64)   */
  int32_t vs_force_local;  /* diagonals 0 .. vs_force_local-1 always kept (>= 1 if sparse) */
  int64_t prefill_chunk;   /* query rows per chunked-prefill step (multiple of 128)        */
  int32_t equal_cost_chunks; /* 0: fixed chunks of prefill_chunk rows. K > 0: K chunks of
                              * equal dense attention cost instead (q1m_prefill_bounds);
                              * prefill_chunk is then unused                               */
} q1m_params;

/* Chunked-prefill boundaries of the layer (host function; no GPU needed). Writes the
 * exclusive end row of each prefill chunk to ends[0 .. m-1] (chunk i covers rows
 * [ends[i-1], ends[i]), ends[-1] = 0, ends[m-1] = seq_len) and returns m, or a negative
 * q1m_status (Q1M_ERR_INVALID for bad arguments, Q1M_ERR_WORKSPACE when m > max_chunks).
 *  - equal_cost_chunks == 0: chunks of prefill_chunk rows, the last one ragged.
 *  - equal_cost_chunks == K > 0: the pages size chunks by the attention kernel's cost so
 *    that every chunk takes about the same time ([P2] 四, pipeline-parallel optimisation,
 *    DCPP, Figure 9); here the same sizing on one GPU. With nb = ceil(seq_len / 128) query
 *    blocks, block b costs b + 1 key blocks (dense causal), the first m blocks cost
 *    C(m) = m (m + 1) / 2 and T = C(nb). Chunk k (1 <= k < K) ends at block
 *    m_k = min{ m : K C(m) >= k T } (exact integers), the last at nb; a chunk left empty
 *    (m_k = m_{k-1}) is dropped, so m <= K. Row boundaries are 128 m_k, the last seq_len. */
int64_t q1m_prefill_bounds(int64_t seq_len, const q1m_params* p, int64_t* ends, int64_t max_chunks);

/* ---------------------------------------------------------------------------------------
 * Whole layer
 * ------------------------------------------------------------------------------------- */

/* Bytes of device workspace q1m_dca_sparse_prefill needs for this shape (0 on bad input). */
size_t q1m_workspace_bytes(int64_t seq_len, int n_q_heads, int n_kv_heads, int head_dim,
                           const q1m_params* p);

/* The layer: for every prefill chunk [s0, e) (the bounds q1m_prefill_bounds lists: fixed
 * chunks of prefill_chunk rows, or equal-cost chunks when equal_cost_chunks > 0), rotate the chunk's keys and queries (DCA views), estimate vertical/slash scores from the
 * chunk's last vs_last_q rows over keys [0, e), select the per-head budgets, build the
 * 128 x 128 block mask, run block-sparse DCA attention for rows [s0, e) and merge the three
 * DCA patterns' partial results ([P2] 四; [P5] Sparse Attention).
 * q: [N][Hq][D], k, v: [N][Hkv][D] in p->in_dtype; out: [N][Hq][D] in p->out_dtype;
 * lse (nullable): [Hq][N] fp32, natural-log log-sum-exp of each row's scaled logits.
 * workspace: device memory of at least q1m_workspace_bytes(...) bytes, 256-byte aligned.
 * The call only enqueues work on `stream` (no host synchronization, no allocation), so it may
 * be captured into a CUDA graph and replayed, with the stage timers (q1m_profile_enable)
 * off; the key-block order follows q1m_set_deterministic as it stood at capture. */
q1m_status q1m_dca_sparse_prefill(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int64_t seq_len, int n_q_heads, int n_kv_heads,
                                  int head_dim, const q1m_params* p, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* The layer restricted to prefill chunks [first_chunk, last_chunk) (chunk numbers as
 * q1m_prefill_bounds lists them; last_chunk past the end means "to the end"): a prefill
 * resumed at chunk granularity. Chunk c attends the rotated keys of chunks 0..c, which live
 * in the workspace, so chunks before first_chunk must have run on the same workspace (same
 * shapes and params) with nothing else written to it in between; the rows of out and lse
 * of the chunks that run are written, the others are left as they are. Running [0, a) and
 * then [a, end) gives the same result as one q1m_dca_sparse_prefill call (which is this
 * call with [0, end)): bit for bit in deterministic mode (q1m_set_deterministic), up to the
 * rounding differences of the aligned tile order otherwise. */
q1m_status q1m_dca_sparse_prefill_chunks(const void* q, const void* k, const void* v, void* out,
                                         float* lse, int64_t seq_len, int n_q_heads,
                                         int n_kv_heads, int head_dim, const q1m_params* p,
                                         int64_t first_chunk, int64_t last_chunk,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace q1m_dca_sparse_prefill_host needs (staging for q, k, v, out
 * and lse plus q1m_workspace_bytes). */
size_t q1m_host_workspace_bytes(int64_t seq_len, int n_q_heads, int n_kv_heads, int head_dim,
                                const q1m_params* p);

/* The same layer from host buffers, with the copies overlapping the compute one prefill
 * chunk at a time: chunk c's rows of q, k and v go host->device on a copy stream of the
 * call's own while earlier chunks compute (chunk c reads only its own rows of them; earlier
 * keys are in the workspace already rotated), and its rows of out (and of lse, if non-null)
 * go device->host on a second copy stream while later chunks compute. One cudaMemcpyAsync
 * per tensor and chunk (cudaMemcpy2DAsync for the [Hq][N] lse rows). The copies start after
 * the work already queued on `stream`; the call creates its two copy streams and three
 * events, makes `stream` wait for the last download, synchronizes `stream` and destroys them
 * before it returns. Results are those of q1m_dca_sparse_prefill on the same inputs. Host
 * buffers should be pinned (page-locked) for full copy bandwidth and for the overlap.
 * Returns the device-side status of the run. */
q1m_status q1m_dca_sparse_prefill_host(const void* q_host, const void* k_host,
                                       const void* v_host, void* out_host, float* lse_host,
                                       int64_t seq_len, int n_q_heads, int n_kv_heads,
                                       int head_dim, const q1m_params* p, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Stages (the same kernels the layer runs; exported for tests and measurement)
 * ------------------------------------------------------------------------------------- */

/* Cosine/sine table for RoPE positions 0 .. n_pos-1 ([P2] 三 RoPE): table[pos][f] =
 * (cos, sin)(pos * base^(-2f/D)) as float2, f < D/2, angles formed in fp64.
 * table: device, n_pos * D/2 float2. */
q1m_status q1m_rope_table(float* table, int64_t n_pos, int head_dim, double rope_base,
                          void* stream);

/* DCA key rotation ([P2] 四 DCA: keys sit at position j mod (c - w)) for tokens [s0, e):
 * k_rot[g][j][:] = fp16(R(j mod L) k[j][g][:]), v16[g][j][:] = fp16(v[j][g][:]).
 * k_rot, v16: device [Hkv][ld_tokens][D] fp16 (ld_tokens >= e, a multiple of 128).
 * table: q1m_rope_table output for n_pos >= dca_chunk. Values beyond fp16 range latch
 * Q1M_ERR_RANGE. */
q1m_status q1m_rope_dca_keys(const void* k, const void* v, int64_t s0, int64_t e,
                             int n_kv_heads, int head_dim, const q1m_params* p,
                             const float* table, uint16_t* k_rot, uint16_t* v16,
                             int64_t ld_tokens, void* stream);

/* DCA query views for rows [s0, e) ([P2] 四 DCA and YaRN): for pattern x in
 * {0 intra, 1 successive, 2 inter}, qv[x][h][i - s0][:] = fp16(R(pos_x(i)) q[i][h][:] *
 * (1/t) / sqrt(D) * log2(e)) with pos_0 = i mod L, pos_1 = min(i mod L + L, c - 1),
 * pos_2 = c - 1, L = c - w. qv: device [3][Hq][ld_rows][D] fp16 (ld_rows >= e - s0,
 * multiple of 128; rows e - s0 .. ld_rows-1 are zeroed). */
q1m_status q1m_rope_dca_queries(const void* q, int64_t s0, int64_t e, int n_q_heads,
                                int head_dim, const q1m_params* p, const float* table,
                                uint16_t* qv, int64_t ld_rows, void* stream);

/* Bytes of scratch q1m_vs_estimate needs for a chunk ending at e. */
size_t q1m_vs_estimate_scratch_bytes(int64_t e, int n_q_heads, int n_kv_heads, int head_dim);

/* Vertical-slash estimator ([P2] 四 稀疏注意力机制; MInference vertical-slash): for the rows
 * R = [max(s0, e - vs_last_q), e) and each Q head h, p_ij = softmax over j <= i of the DCA
 * logits; vert[h][j] = sum_{i in R} p_ij and slash[h][o] = sum_{i in R} p_{i,i-o} for
 * j, o in [0, e). q: raw queries [N][Hq][D] (in_dtype); k_rot: q1m_rope_dca_keys output
 * covering [0, e). vert, slash: device fp32 [Hq][ld] (ld >= e). scratch: device memory of
 * q1m_vs_estimate_scratch_bytes(...) bytes. */
q1m_status q1m_vs_estimate(const void* q, const uint16_t* k_rot, int64_t ld_tokens, int64_t s0,
                           int64_t e, int n_q_heads, int n_kv_heads, int head_dim,
                           const q1m_params* p, const float* table, float* vert, float* slash,
                           int64_t ld, void* scratch, size_t scratch_bytes, void* stream);

/* Bytes of scratch q1m_vs_select needs for candidates [0, e). */
size_t q1m_vs_select_scratch_bytes(int64_t e, int n_q_heads);

/* Budget selection: per head, the vs_vertical columns with the largest vert score and the
 * vs_slash offsets with the largest slash score, offsets < vs_force_local always kept;
 * larger score first, equal scores by smaller index; a budget >= e keeps all. Results are
 * written in ascending order: V [Hq][min(vs_vertical, e)] and S [Hq][min(vs_slash, e)]
 * int32 (device). Scores must be >= 0 (NaN latches Q1M_ERR_RANGE). */
q1m_status q1m_vs_select(const float* vert, const float* slash, int64_t ld, int64_t e,
                         int n_q_heads, const q1m_params* p, int32_t* V, int32_t* S,
                         void* scratch, size_t scratch_bytes, void* stream);

/* Block mask and residual verticals for query blocks b of rows [s0, e) (128 x 128 blocks):
 * key block kb of query block b (rows r0 = 128b .. r1 = min(128b+127, e-1)) is computed when
 * some o in S has o <= r1 and floor(max(0, r0-o)/128) <= kb <= floor((r1-o)/128); residual
 * verticals are the j in V with j <= r1 whose block is not computed (ascending).
 * Outputs (device), nqb = ceil((e - s0)/128), nkw = ceil(ceil(e/128)/32):
 *   mask  [Hq][nqb][nkw] uint32, bit kb%32 of word kb/32;
 *   resid [Hq][nqb][nv] int32 (nv = min(vs_vertical, e)), entries past the count undefined;
 *   cnt   [Hq][nqb][8] int32: computed blocks per DCA pattern (0 intra, 1 successive,
 *         2 inter), then residual columns per pattern (same order), then total residuals,
 *         then 0. The ascending residual list holds inter, then successive, then intra. */
q1m_status q1m_vs_build_masks(const int32_t* V, const int32_t* S, int64_t s0, int64_t e,
                              int n_q_heads, const q1m_params* p, uint32_t* mask,
                              int32_t* resid, int32_t* cnt, void* stream);

/* Bytes of scratch q1m_block_sparse_attn needs for rows [s0, e). */
size_t q1m_attn_scratch_bytes(int64_t s0, int64_t e, int n_q_heads, int head_dim);

/* Block-sparse DCA attention on the tensor cores for rows [s0, e), one partial result per
 * DCA pattern x (0 intra, 1 successive, 2 inter; query view x): over the keys of that pattern in
 * A(i) (computed blocks and residual verticals; every causal key when mask == NULL),
 *   o_part[x][h][i - s0][:] = softmax-weighted sum of v (fp32), lse_part[x][h][i - s0] =
 *   log2-sum-exp2 of the log2-scaled logits (-inf when the segment is empty for the row).
 * qv, k_rot, v16: stage outputs above; mask/resid/cnt: q1m_vs_build_masks output or NULL.
 * o_part: device fp32 [3][Hq][ld_rows][D]; lse_part: device fp32 [3][Hq][ld_rows].
 * The order in which a work item visits its key blocks follows a global tile count unless
 * deterministic mode is on (q1m_set_deterministic); results agree up to rounding either way. */
q1m_status q1m_block_sparse_attn(const uint16_t* qv, int64_t ld_rows, const uint16_t* k_rot,
                                 const uint16_t* v16, int64_t ld_tokens, const uint32_t* mask,
                                 const int32_t* resid, const int32_t* cnt, int64_t s0,
                                 int64_t e, int n_q_heads, int n_kv_heads, int head_dim,
                                 const q1m_params* p, float* o_part, float* lse_part,
                                 void* scratch, size_t scratch_bytes, void* stream);

/* Allocation-free variant of q1m_block_sparse_attn, for callers that cannot call cudaMalloc
 * and cannot hand the library a scratch buffer: for example code that runs under a strict
 * memory planner or pool that owns every device allocation, or a host thread on a latency
 * path that must never wait on the allocator. The pages have no counterpart to this entry
 * point; it exists only for such callers.
 * Same arguments and results as q1m_block_sparse_attn, without scratch: the work-unit list
 * lives in a static device array of Q1M_NOALLOC_UNITS int32 (64 KiB) that every GPU which
 * loads the library holds until the process exits. A chunk may therefore have at most
 * Q1M_NOALLOC_MAX_QUERY_BLOCKS query blocks of 128 rows (1,397,248 rows); larger chunks are
 * rejected with Q1M_ERR_UNSUPPORTED before anything is launched. The call allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine). The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress) with that device current, so
 * make that first call before any stream capture; the address is looked up again when the
 * device's context has changed (after cudaDeviceReset), and that call, too, must come
 * before any capture. All calls share the one array, and each
 * call rewrites every entry it reads; calls that can overlap on the GPU (different
 * streams, or devices sharing it) race on it and must be serialised by the caller. */
#define Q1M_NOALLOC_UNITS 16384
#define Q1M_NOALLOC_MAX_QUERY_BLOCKS 10916
q1m_status q1m_block_sparse_attn_noalloc(const uint16_t* qv, int64_t ld_rows,
                                         const uint16_t* k_rot, const uint16_t* v16,
                                         int64_t ld_tokens, const uint32_t* mask,
                                         const int32_t* resid, const int32_t* cnt, int64_t s0,
                                         int64_t e, int n_q_heads, int n_kv_heads, int head_dim,
                                         const q1m_params* p, float* o_part, float* lse_part,
                                         void* stream);

/* Log-sum-exp merge of the DCA patterns' partial results for rows [s0, e)
 * (lse = log2 sum_x 2^lse_x, out = sum_x 2^(lse_x - lse) o_x):
 * out[i][h][:] in out_dtype ([N][Hq][D] layout) and lse[h][i] (natural log, nullable).
 * n_parts partials laid out as q1m_block_sparse_attn writes them. With p non-NULL and
 * n_parts == 3, a row reads only the patterns it has keys in (inter from the third DCA
 * chunk on, successive from the second), which is what q1m_block_sparse_attn writes;
 * with p NULL every part is read and an empty part must hold lse = -inf. */
q1m_status q1m_lse_merge(const float* o_part, const float* lse_part, int n_parts,
                         int64_t ld_rows, int64_t s0, int64_t e, int64_t seq_len,
                         int n_q_heads, int head_dim, int out_dtype, const q1m_params* p,
                         void* out, float* lse, void* stream);

/* Attention recall of the sparse selection ([P2] 四 稀疏注意力机制: sparsity refinement keeps
 * the accuracy loss of the sparse configuration small): for every row, the share of the
 * dense softmax mass that the attended set A(i) keeps,
 *   recall_i = sum_{j in A(i)} softmax_j(l(i, .)) = exp(lse_sparse_i - lse_dense_i),
 * from the natural-log lse outputs of a sparse and a dense run of the same layer (n values,
 * device fp32). recall: device fp32 [n], in [0, 1]. */
q1m_status q1m_attention_recall(const float* lse_sparse, const float* lse_dense, int64_t n,
                                float* recall, void* stream);

/* ---------------------------------------------------------------------------------------
 * Status
 * ------------------------------------------------------------------------------------- */

/* Synchronizes `stream`, then returns and clears the device-side status latched by the
 * kernels on the current device (Q1M_OK, Q1M_ERR_TIMEOUT, Q1M_ERR_RANGE or, in debug mode,
 * Q1M_ERR_CHECK), or Q1M_ERR_CUDA if the stream reported an error. */
q1m_status q1m_status_poll(void* stream);

/* The message of the last failing call on this thread ("" if none). */
const char* q1m_last_error(void);

/* Library version string. */
const char* q1m_version(void);

/* ---------------------------------------------------------------------------------------
 * Decode
 * ------------------------------------------------------------------------------------- */

/* Bytes of device scratch q1m_dca_decode needs (the token's query views and the split-KV
 * partials; independent of the position). 0 on bad input. */
size_t q1m_dca_decode_scratch_bytes(int n_q_heads, int head_dim);

/* One decode step of the layer ([P2] 四 "Dual Chunk Attention": the token's logits against
 * every cached key use the same intra / successive / inter remap and YaRN scale as the
 * prefill; [P2] 三: generation up to 8K tokens after the long context). The token sits at
 * position pos and attends keys [0, pos], densely.
 *  - q: [Hq][D], k, v: [Hkv][D] in p->in_dtype: the token's projections (device).
 *  - k_rot, v16: the fp16 cache [Hkv][ld_tokens][D] (ld_tokens a multiple of 128, > pos).
 *    Rows [0, pos) hold the earlier tokens' keys rotated at j mod L and their values, as
 *    q1m_rope_dca_keys or earlier q1m_dca_decode calls write them. The call rotates the
 *    token's key (position pos mod L), stores it and its value at row pos, and zeroes rows
 *    (pos, round_up(pos + 1, 32)) of both.
 *  - table: the RoPE table of q1m_rope_table for (rope_base, dca_chunk, D).
 *  - out: [Hq][D] in p->out_dtype; lse (nullable): [Hq] fp32, natural log.
 *  - The budgets and prefill_chunk of p are not used (decode is dense).
 * Asynchronous on `stream`; fp16 overflow of the token's key, value or query views latches
 * Q1M_ERR_RANGE (q1m_status_poll). */
q1m_status q1m_dca_decode(const void* q, const void* k, const void* v, int64_t pos,
                          uint16_t* k_rot, uint16_t* v16, int64_t ld_tokens, int n_q_heads,
                          int n_kv_heads, int head_dim, const q1m_params* p, const float* table,
                          void* out, float* lse, void* scratch, size_t scratch_bytes,
                          void* stream);

/* ---------------------------------------------------------------------------------------
 * Determinism
 * ------------------------------------------------------------------------------------- */

/* By default the attention kernel starts each work item's walk over its key blocks at a
 * position taken from a global count of the tiles all CTAs have issued, so that CTAs
 * streaming the same K/V range stay at about the same tile and share it in L2 (less DRAM
 * traffic, and under the power cap a higher clock). The result does not depend on the tile
 * order beyond rounding (fp32 sums and the fp16 rounding of P against the running maximum),
 * but the order then depends on timing, so repeated runs can differ at that level (about
 * 1e-4 relative). Deterministic mode (process-wide; initially on when the
 * environment variable Q1M_DETERMINISTIC is set to a non-zero value) starts every walk at
 * its first block: repeated runs, and the layer against its stages, are then bit-identical. */
q1m_status q1m_set_deterministic(int on);
int q1m_deterministic(void);

/* ---------------------------------------------------------------------------------------
 * Debug mode
 * ------------------------------------------------------------------------------------- */

/* Debug mode for the whole process (initially on when the environment variable Q1M_DEBUG is
 * set to a non-zero value). In debug mode q1m_dca_sparse_prefill(_chunks) lays out its
 * workspace with a 4 KiB guard region after every buffer (so q1m_workspace_bytes grows:
 * query it after switching), fills the guards with a pattern at the start of each call,
 * checks every guard after each stage and validates the selected index lists (ascending,
 * inside [0, e), the forced diagonals present) and the block counts after the mask stage.
 * A failed check latches Q1M_ERR_CHECK, which q1m_status_poll returns with the failing
 * guard or list in q1m_last_error. Results are unchanged; the checks cost time. */
q1m_status q1m_set_debug(int on);
int q1m_debug_enabled(void);

/* Test hook of the debug mode: on the next layer call, right after the given stage
 * (Q1M_STAGE_*) of the first prefill chunk, the library overwrites one byte of the first
 * guard region from the host side (cudaMemsetAsync), so that the following check reports
 * Q1M_ERR_CHECK. -1 disarms it. Has no effect outside debug mode. */
q1m_status q1m_debug_inject(int stage);

/* ---------------------------------------------------------------------------------------
 * Measurement
 * ------------------------------------------------------------------------------------- */

/* Stages timed by the per-stage event timers of q1m_dca_sparse_prefill. */
enum {
  Q1M_STAGE_TABLE = 0,     /* RoPE table                              */
  Q1M_STAGE_KEYS = 1,      /* DCA key rotation                        */
  Q1M_STAGE_QUERIES = 2,   /* DCA query views                         */
  Q1M_STAGE_ESTIMATE = 3,  /* vertical-slash estimator                */
  Q1M_STAGE_SELECT = 4,    /* budget selection                        */
  Q1M_STAGE_MASKS = 5,     /* block masks and residual columns        */
  Q1M_STAGE_ATTN = 6,      /* block-sparse attention kernel           */
  Q1M_STAGE_MERGE = 7,     /* LSE merge of the DCA patterns           */
  Q1M_STAGE_DECODE = 8,    /* decode attention kernel (q1m_dca_decode) */
  Q1M_NUM_STAGES = 9
};

/* Enables (1) or disables (0) per-stage CUDA-event timing inside q1m_dca_sparse_prefill on
 * this thread; enabling also clears the accumulated times. Events are recorded on the call's
 * stream around each stage's launches. */
q1m_status q1m_profile_enable(int on);

/* Synchronizes the recorded events and writes, per stage, the accumulated milliseconds
 * (ms[Q1M_NUM_STAGES]) and the number of timed launches of that stage's main kernel
 * (launches[Q1M_NUM_STAGES], nullable) since the last enable. */
q1m_status q1m_profile_read(double* ms, int64_t* launches);

/* Self-test of the attention kernel's FMA-pipe exponential: for x[0..n) (device, fp32)
 * writes y_poly = the kernel's polynomial 2^x, y_mufu = the multi-function-unit 2^x
 * (ex2.approx) and y_ref = CUDA's exp2f(x), so a caller can check the error bound. */
q1m_status q1m_selftest_exp2(const float* x, float* y_poly, float* y_mufu, float* y_ref, int64_t n,
                             void* stream);

/* Number of kernels this library has launched in the process so far. */
uint64_t q1m_launch_count(void);

/* Sets the budget, in SM clock cycles, of the kernels' bounded waits on the current device
 * (default 2e9, about one second); 0 restores the default. */
q1m_status q1m_set_wait_budget(uint64_t cycles);

/* Self-test of the bounded waits: launches one warp that waits on a barrier nothing ever
 * arrives on, with a budget of `cycles`, and returns what q1m_status_poll then reports
 * (Q1M_ERR_TIMEOUT when the wait gave up as designed). The default budget is restored. */
q1m_status q1m_selftest_wait_timeout(uint64_t cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q1M_H_ */
