/*
 * kvc.h - C ABI of the attention-score-driven KV eviction and ragged decode
 * attention library (libkvc.so, sm_100a).
 *
 * The hot path, in call order:
 *   kvc_score          window scoring (token keys or chunk keys)
 *   kvc_select         per-head budget selection (top-B, LMBA mass count, FastGen
 *                      local / special / full, ChunkLLM chunk selection)
 *   kvc_alloc_budgets  ZigZagKV bounded per-layer budgets from the LMBA counts
 *   kvc_layout         packed-cache offsets and capacities
 *   kvc_compact        gather of the kept rows into the packed per-head cache
 *   kvc_layout_compact the two above in one launch
 *   kvc_append         one new token per slot per decode step
 *   kvc_decode_attn    split-K GQA decode attention over the ragged packed cache
 *   kvc_append_decode  the two above fused into one launch (the per-step call)
 *   kvc_append_decode_chain  the same for the loop's later steps, overlapping the
 *                      previous step's tail
 *
 * Sources: "ZigZagKV: Dynamic KV Cache Compression for Long-context Modeling based
 * on Layer Uncertainty" (arXiv 2412.09036) Eq. 3-7; "Model Tells You What to
 * Discard: Adaptive KV Cache Compression for LLMs" (FastGen, arXiv 2310.01801),
 * abstract and Section 1; "ChunkLLM: A Lightweight Pluggable Framework for
 * Accelerating LLMs Inference" (arXiv 2510.02361) Section 2.2, Eq. 3.
 *
 * Conventions (all calls):
 *  - A slot is one (layer, batch row, KV head). Slots are numbered row-major in
 *    that order; query head j of slot s is global query row s*G + j (GQA group G).
 *  - Every tensor pointer is DEVICE memory owned by the caller; tensors are
 *    contiguous, row-major, and 16-byte aligned. The library allocates no device
 *    memory and keeps no state besides a per-device error word (read by
 *    kvc_get_status) and a thread-local message (kvc_last_error).
 *  - Calls are asynchronous on `stream`. Shapes and arguments are validated on the
 *    host before any launch; a failed validation returns a non-zero kvc_status,
 *    launches nothing, and sets the message. Device-side range checks never trap:
 *    they skip the offending access and set a bit of the error word.
 *  - Workspaces: `ws`/`ws_bytes` is caller-owned scratch of at least
 *    kvc_workspace_size(...) bytes. It must be zero-filled before its first use;
 *    every call leaves it zero-filled again, so one allocation serves many calls.
 *    Calls that share a workspace must be ordered on one stream.
 *  - Supported: head_dim d in {64, 128}; K/V/Q in bf16 or fp32
 *    (the same type for all three); decode needs G <= 8 (bf16) or G in {1, 2, 4}
 *    (fp32); scoring needs G*w <= 256;
 *    all accumulation in fp32.
 */
#ifndef KVC_H_
#define KVC_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
  KVC_ERR_SHAPE = 2,         /* inconsistent sizes */
  KVC_ERR_UNSUPPORTED = 3,   /* valid but not implemented (e.g. d = 96) */
  KVC_ERR_CAPACITY = 4,      /* an output buffer is too small */
  KVC_ERR_CUDA = 5,          /* a CUDA runtime call failed */
  KVC_ERR_WORKSPACE = 6,     /* workspace missing or too small */
  KVC_ERR_DEVICE = 7         /* kvc_get_status: a kernel reported a range/timeout fault */
} kvc_status;

typedef enum { KVC_BF16 = 0, KVC_FP32 = 1 } kvc_dtype;

typedef enum {
  KVC_POL_TOPB = 0,        /* keep the B highest-scoring tokens (B = budget[s]) */
  KVC_POL_MASS_COUNT = 1,  /* LMBA count only: smallest k whose top-k mass >= mass * total */
  KVC_POL_LOCAL = 2,       /* FastGen local head: keep [L - W, L), W = budget[s] */
  KVC_POL_SPECIAL = 3,     /* FastGen special-token head: keep positions set in special_mask */
  KVC_POL_FULL = 4,        /* FastGen global head: keep [0, L) */
  KVC_POL_CHUNK = 5        /* ChunkLLM: keep the top chunks until >= budget[s] tokens */
} kvc_policy;

/* Bit values of the device error word returned through kvc_get_status. */
#define KVC_DEVERR_APPEND_OVERFLOW 0x1u  /* append found len == cap: token dropped */
#define KVC_DEVERR_INDEX_RANGE     0x2u  /* compact/select met an out-of-range index or row */
#define KVC_DEVERR_WAIT_TIMEOUT    0x4u  /* a pipeline wait hit its iteration limit */
#define KVC_DEVERR_WORKSPACE       0x8u  /* a kernel's work list exceeded its workspace */

typedef struct {
  int32_t n_slots;   /* S = n_layers * batch * n_kv_heads */
  int32_t G;         /* query heads per KV head */
  int32_t d;         /* head dim */
  int32_t L;         /* context length (keys per slot before compaction) */
  int32_t w;         /* observation window (window queries per query head); 0 if unused */
  int32_t n_kv_heads;/* KV heads per (layer, batch row): slot s has batch row (s / n_kv_heads) % batch */
  int32_t batch;     /* batch rows per layer */
  int32_t dtype;     /* kvc_dtype of Q, K, V */
} kvc_shape;

/* Workspace selectors for kvc_workspace_size. */
#define KVC_WS_SCORE  0
#define KVC_WS_SELECT 1
#define KVC_WS_DECODE 2

/*
 * kvc_score - observation-window importance scores (ZigZagKV Eq. 7, after SnapKV).
 *   For slot s, query head j < G and window row i < w (row position L - w + i),
 *   p_{j,i,.} = softmax over the keys the row sees (key position <= L - w + i) of
 *   q_{j,i} . k / sqrt(d); score[s][n] = sum_{j,i} p_{j,i,n}.
 *   Token keys (chunk_end == NULL): key n is k[s][n], position n, n < L.
 *   Chunk keys (ChunkLLM Eq. 3): key n < C is k[s][chunk_end[n]] (the chunk's last
 *   token), position chunk_end[n]; chunk_end strictly increasing, last = L - 1.
 *
 *   q_win     [S*G, w, d]  window queries (dtype)
 *   k         [S, L, d]    keys (dtype)
 *   chunk_end [C] int32 or NULL; C its length (ignored when NULL)
 *   row_lse   [S*G*w] fp32 or NULL: natural-log softmax normaliser of each window
 *             row (log sum_n exp(q.k_n/sqrt(d)) over visible keys) if the caller has
 *             it from prefill; NULL: computed here (one extra pass over K).
 *   score     [S, N] fp32 out, N = L (tokens) or C (chunks)
 * Errors: UNSUPPORTED for d not in {64,128} or G*w > 256; WORKSPACE if ws_bytes <
 * kvc_workspace_size(KVC_WS_SCORE, shape, C).
 */
kvc_status kvc_score(const kvc_shape* shape, const void* q_win, const void* k,
                     const int32_t* chunk_end, int32_t C, const float* row_lse,
                     float* score, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * kvc_select - per-slot selection; each slot follows policy[s].
 *   TOPB       keep budget[s] tokens with the highest score (ties: lower index first)
 *   MASS_COUNT count[s] = LMBA of the slot (ZigZagKV Eq. 3): smallest k whose k
 *              highest scores hold >= mass * (sum of scores); idx not written
 *   LOCAL      keep [L - budget[s], L)
 *   SPECIAL    keep n where special_mask[b][n] != 0, b the slot's batch row
 *   FULL       keep [0, L)
 *   CHUNK      `score` holds chunk scores [S, C]; keep the highest-scoring chunks
 *              (ties: lower chunk index) until they hold >= budget[s] tokens,
 *              emitting every token of the kept chunks
 *   Kept indices are written to idx[s][0 .. count[s]) in ascending position order.
 *
 *   score        [S, N] fp32 (N = L, or C for CHUNK); may be NULL if no slot needs it
 *   policy       [S] int8 kvc_policy, device
 *   budget       [S] int32, device (B, W or token target; unused for MASS/SPECIAL/FULL)
 *   special_mask [batch, L] uint8 or NULL (required if any slot is SPECIAL)
 *   chunk_end    [C] int32 or NULL (required if any slot is CHUNK)
 *   idx          [S, max_sel] int32 out; max_sel >= every count (else the kernel
 *                clips, sets KVC_DEVERR_INDEX_RANGE)
 *   count        [S] int32 out
 */
kvc_status kvc_select(const kvc_shape* shape, const float* score, const int8_t* policy,
                      const int32_t* budget, float mass, const uint8_t* special_mask,
                      const int32_t* chunk_end, int32_t C, int32_t* idx, int32_t max_sel,
                      int32_t* count, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * kvc_alloc_budgets - ZigZagKV bounded per-layer budgets (Eq. 4-6).
 *   C_l = sum of counts[l][0 .. spl); u_l = C_l / sum C; exact rational
 *   B_l = floor_B + (avg_B - floor_B) * n_layers * u_l, made integer by floor plus
 *   largest remainder (ties to the lower layer) so that sum B_l = n_layers * avg_B;
 *   layers whose B_l exceeds L are fixed at L and the rest re-split the same way;
 *   all-zero counts split uniformly.
 *   counts       [n_layers * spl] int32 (MASS_COUNT of every slot), device
 *   budgets      [n_layers] int32 out, device
 *   slot_budgets [n_layers * spl] int32 out or NULL: B_l broadcast to each slot
 * Errors: SHAPE unless 0 <= floor_B <= avg_B <= L.
 */
kvc_status kvc_alloc_budgets(const int32_t* counts, int32_t n_layers, int32_t spl, int32_t L,
                             int32_t avg_B, int32_t floor_B, int32_t* budgets,
                             int32_t* slot_budgets, cudaStream_t stream);

/*
 * kvc_layout - packed-cache layout: cap[s] = round_up(count[s] + reserve, 16);
 *   off[0] = 0, off[s+1] = off[s] + cap[s] (rows). Slot s owns rows [off[s], off[s+1]).
 *   count [S] int32 in; off [S+1] int64 out; cap [S] int32 out. All device.
 */
kvc_status kvc_layout(const int32_t* count, int32_t n_slots, int32_t reserve,
                      int64_t* off, int32_t* cap, cudaStream_t stream);

/*
 * kvc_compact - kp[off[s] + r] = k[s][idx[s][r]], vp likewise, for r < count[s];
 *   len[s] = count[s]. Rows [off[s] + count[s], off[s+1]) are not written.
 *   k, v [S, L, d]; idx [S, max_sel]; kp, vp [kp_rows, d]; len [S] int32 out.
 *   Rows outside [0, kp_rows) or indices outside [0, L) are skipped and flagged.
 */
kvc_status kvc_compact(const kvc_shape* shape, const void* k, const void* v,
                       const int32_t* idx, int32_t max_sel, const int32_t* count,
                       const int64_t* off, void* kp, void* vp, int64_t kp_rows,
                       int32_t* len, cudaStream_t stream);

/*
 * kvc_layout_compact - kvc_layout followed by kvc_compact, in one launch when
 *   n_slots <= 512 (every CTA of the compaction scans the capacities itself), else
 *   as those two launches. Same arguments and results as the two calls: off [S+1]
 *   int64 and cap [S] int32 are outputs here, with reserve >= 0 as in kvc_layout;
 *   the rows written, len and the flags are those of kvc_compact.
 */
kvc_status kvc_layout_compact(const kvc_shape* shape, const void* k, const void* v,
                              const int32_t* idx, int32_t max_sel, const int32_t* count,
                              int32_t reserve, int64_t* off, int32_t* cap, void* kp, void* vp,
                              int64_t kp_rows, int32_t* len, cudaStream_t stream);

/*
 * kvc_append - one new token per slot: kp[off[s] + len[s]] = k_new[s], vp
 *   likewise, len[s] += 1. A slot with len[s] == cap[s] (or whose next row would
 *   fall outside the kp_rows rows of kp/vp) keeps its cache, leaves len unchanged
 *   and sets KVC_DEVERR_APPEND_OVERFLOW.
 *   k_new, v_new [S, d] (dtype); off [S+1]; cap, len [S]; kp, vp [kp_rows, d].
 */
kvc_status kvc_append(const kvc_shape* shape, const void* k_new, const void* v_new,
                      const int64_t* off, const int32_t* cap, int32_t* len,
                      void* kp, void* vp, int64_t kp_rows, cudaStream_t stream);

/*
 * kvc_decode_attn - for query head h of slot s = h / G:
 *   out[h] = sum_{r < len[s]} softmax_r(q[h] . kp[off[s]+r] / sqrt(d)) vp[off[s]+r]
 *   (fp32 accumulation and output; bf16 dot products on the tensor cores, fp32 on
 *   the CUDA cores). Work is split evenly over the GPU by token
 *   ranges that may cross slot boundaries; partial results are merged by the last
 *   CTA to finish a slot. A slot with len 0 yields zeros.
 *   q [S*G, d] (dtype); kp, vp packed cache [kp_rows, d]; off [S+1]; len [S];
 *   out [S*G, d] fp32. Rows past kp_rows are never read: a slot whose len runs past
 *   them is cut short and KVC_DEVERR_INDEX_RANGE is set.
 */
kvc_status kvc_decode_attn(const kvc_shape* shape, const void* q, const void* kp,
                           const void* vp, const int64_t* off, const int32_t* len,
                           int64_t kp_rows, float* out, void* ws, size_t ws_bytes,
                           cudaStream_t stream);

/*
 * kvc_append_decode - kvc_append followed by kvc_decode_attn, fused into one launch
 *   for bf16 (G <= 8): slot s with room gets its new token (k_new[s], v_new[s]) at
 *   row off[s] + len[s], decode attends over len[s] + 1 rows including it, and len[s]
 *   is incremented once every CTA has read it (by the last CTA to finish). A slot
 *   without room (len == cap) is decoded over its old rows and flagged
 *   KVC_DEVERR_APPEND_OVERFLOW, as with kvc_append. Other dtypes / G run the two calls.
 *   Same workspace as kvc_decode_attn.
 */
kvc_status kvc_append_decode(const kvc_shape* shape, const void* k_new, const void* v_new,
                             const void* q, void* kp, void* vp, const int64_t* off,
                             const int32_t* cap, int32_t* len, int64_t kp_rows, float* out,
                             void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * kvc_append_decode_chain - kvc_append_decode for the steps of a decode loop after its
 *   first: same arguments and results, plus `stable` [n_slots] int32 (device), a row
 *   count per slot that the caller guarantees is not written by the kernel issued just
 *   before this call on `stream`, nor by this call: the kept rows of a compacted cache
 *   (its count from kvc_select) while the loop only appends. The caller also guarantees
 *   that this previous kernel writes none of off, cap and stable. The launch then plans
 *   its work split from cap and starts loading the rows below stable[s] before the
 *   previous kernel has finished (programmatic dependent launch), which shortens a step
 *   by the prologue and the first load's latency. The first step after kvc_compact (or
 *   anything else that rewrites those rows) must use kvc_append_decode. A slot whose
 *   length turns out below stable[s] breaks the promise: it gets no new token, is
 *   attended over stable[s] rows, and KVC_DEVERR_INDEX_RANGE is set. stable == NULL:
 *   KVC_ERR_INVALID_ARG. Other dtypes / G behave
 *   as kvc_append_decode (the promise is then unused).
 */
kvc_status kvc_append_decode_chain(const kvc_shape* shape, const void* k_new, const void* v_new,
                                   const void* q, void* kp, void* vp, const int64_t* off,
                                   const int32_t* cap, const int32_t* stable, int32_t* len,
                                   int64_t kp_rows, float* out, void* ws, size_t ws_bytes,
                                   cudaStream_t stream);

/*
 * kvc_decode_attn_noalloc - kvc_decode_attn for callers that cannot allocate
 *   device memory: code that runs inside a runtime owning every device buffer
 *   (a plugin or operator that is handed only its inputs and outputs at enqueue
 *   time, with no allocator and no workspace handle), or loops where a
 *   cudaMalloc's implicit device synchronisation is not acceptable. The paper has
 *   no counterpart; this is a property of the library, not of the method.
 *   Same arguments as kvc_decode_attn minus the workspace: the scratch lives in a
 *   fixed 4 MiB array inside the library (held by every GPU that loads it, until
 *   exit). It always takes the token-range work split (the per-slot cluster form
 *   kvc_decode_attn picks for few slots merges through shared memory, not the
 *   scratch), so for shapes where kvc_decode_attn runs clusters the two sum the
 *   partials in a different order: results agree within the decode tolerance, not
 *   bit for bit. Scratch needed: 256-byte rounded (S + 1) * 4 B of tickets plus
 *   (SMs + S) * round_up(G * (d + 2), 4) * 4 B of partials, 256-byte rounded
 *   (= kvc_workspace_size(KVC_WS_DECODE, ...)); shapes needing more than 4 MiB are
 *   rejected with KVC_ERR_WORKSPACE (G = 4, d = 128 on 148 SMs: up to 1864 slots).
 *   The first successful call on each device looks up the array's device address
 *   (make it before any stream capture); a failed lookup is retried on the next
 *   call. All calls share the array and each call clears the part that must start
 *   at zero: calls that overlap on the GPU (for example on two streams) race and
 *   must not be issued.
 */
kvc_status kvc_decode_attn_noalloc(const kvc_shape* shape, const void* q, const void* kp,
                                   const void* vp, const int64_t* off, const int32_t* len,
                                   int64_t kp_rows, float* out, cudaStream_t stream);

/*
 * kvc_append_window - kvc_append with sliding-window eviction (the local-window variant
 *   of FastGen's local heads - the policy keeps the most recent tokens - applied while
 *   decoding): a slot with window[s] > 0 whose cache already holds window[s] rows keeps
 *   exactly those rows; the new token overwrites row head[s] (the oldest) and head[s]
 *   advances cyclically, len[s] unchanged. Every other slot appends at row len[s] and
 *   increments len[s] (overflow past cap[s] is flagged, the row is not written).
 *   Decode attention does not depend on the order of a slot's rows, so kvc_decode_attn
 *   over [off[s], off[s] + len[s]) sees exactly the window. Compaction stores a local
 *   slot's rows oldest first, so head[s] starts at 0.
 *   k_new, v_new [S, d]; window [S] int32 (0: no eviction); head [S] int32, in/out.
 */
kvc_status kvc_append_window(const kvc_shape* shape, const void* k_new, const void* v_new, const int64_t* off,
                             const int32_t* cap, int32_t* len, const int32_t* window, int32_t* head,
                             void* kp, void* vp, int64_t kp_rows, cudaStream_t stream);

/*
 * kvc_select_chunks - ChunkLLM chunk selection with always-kept local chunks (ChunkLLM
 *   Section 3.2 keeps the 15 or 16 most recent chunks): for every slot, the last
 *   n_local chunks are kept, then the other chunks in descending chunk-score order
 *   (ties: lower chunk index) until the kept chunks hold >= target[s] tokens; every
 *   token of the kept chunks is written to idx[s] in ascending order. With n_local = 0
 *   this is kvc_select's KVC_POL_CHUNK.
 *   chunk_score [S, C] fp32; chunk_end [C]; target [S] int32; idx [S, max_sel]; count [S].
 */
kvc_status kvc_select_chunks(const kvc_shape* shape, const float* chunk_score, const int32_t* chunk_end,
                             int32_t C, const int32_t* target, int32_t n_local, int32_t* idx,
                             int32_t max_sel, int32_t* count, cudaStream_t stream);

/*
 * kvc_retained_mass - share of each slot's window-attention mass its kept tokens hold:
 *   retained[s] = sum_{r < count[s]} score[s][idx[s][r]] / sum_n score[s][n] (0 if no
 *   mass). ZigZagKV's attention loss (Section 5.5, Table 3) is max(0, 0.9 - retained).
 *   score [S, N] fp32; idx [S, max_sel]; count [S]; retained [S] fp32 out (fp64 sums).
 */
kvc_status kvc_retained_mass(const kvc_shape* shape, const float* score, int32_t N, const int32_t* idx,
                             int32_t max_sel, const int32_t* count, float* retained, cudaStream_t stream);

/*
 * kvc_profile_heads - FastGen-style head profiling from the window scores (FastGen
 *   abstract / Section 1: profile the heads, then give local heads a recent window,
 *   special-token heads the special tokens, broad heads the full cache). The pages
 *   give no criterion; this one keeps the policy (local: the last `window` tokens;
 *   special: the batch row's special tokens) that keeps fewer tokens (ties: local)
 *   among those whose share of the head's window-attention mass is >= tau, else full.
 *   policy [S] int8 out (feeds kvc_select); shares [S][2] fp32 out or NULL: the local
 *   and special mass shares. special_mask [batch, L] or NULL (no special policy).
 */
kvc_status kvc_profile_heads(const kvc_shape* shape, const float* score, const uint8_t* special_mask,
                             int32_t window, float tau, int8_t* policy, float* shares,
                             cudaStream_t stream);

/* Bytes of workspace the call `which` (KVC_WS_*) needs for this shape (C: chunks, 0 if none). */
size_t kvc_workspace_size(int which, const kvc_shape* shape, int32_t C);

/* Synchronises `stream`, reads and clears the current device's error word.
 * Returns KVC_ERR_DEVICE (message names the bits) if it was non-zero. */
kvc_status kvc_get_status(cudaStream_t stream);

/* Message of the last failure on this host thread ("" if none). */
const char* kvc_last_error(void);

/* Library version string. */
const char* kvc_version(void);

/* Number of kernels this library has launched in this process so far (diagnostic). */
unsigned long long kvc_launch_count(void);

/*
 * kvc_check_wait_limit - diagnostic of the library's failure path: launches one CTA whose
 *   thread waits on an mbarrier that nothing arrives on, with the bounded wait every
 *   pipeline in the library uses (they give up after 2 s; here after limit_us). The wait
 *   gives up, sets KVC_DEVERR_WAIT_TIMEOUT and the kernel returns, so kvc_get_status then
 *   reports the timeout and the context stays usable. limit_us in [1, 1e6], else
 *   KVC_ERR_INVALID_ARG.
 */
kvc_status kvc_check_wait_limit(int32_t limit_us, cudaStream_t stream);

/*
 * kvc_diag_set_path - diagnostic, for cross-checks only: force one of the library's
 *   alternate kernel paths for every later call in this process (all threads), so a
 *   test can run the same inputs through both forms of a step and compare. Production
 *   callers never call it: with every knob at 0 (the state at load) each call takes
 *   the path its shape selects. Nothing else (no environment variable) changes a path.
 *   knob (KVC_DIAG_*) and choice:
 *     KVC_DIAG_SCORE        0 auto, 1 two-launch tensor-core form, 2 CUDA-core kernels,
 *                           3 the earlier slot-cluster form with 128-key tiles (one launch;
 *                           two-launch where the slots do not fill the GPU in clusters)
 *     KVC_DIAG_SCORE_K      0 auto, 1..16: CTAs per slot of the default scoring form
 *     KVC_DIAG_SELECT       0 auto, 1 one CTA per slot
 *     KVC_DIAG_COMPACT      0 auto, 1 grid-stride compaction kernel
 *     KVC_DIAG_DECODE       0 auto, 1 CUDA-core decode, 2 tcgen05 decode (bf16, d = 128)
 *     KVC_DIAG_DECODE_SPLIT 0 auto, 1 token-range split even for few slots
 *   Unknown knob or choice: KVC_ERR_INVALID_ARG, nothing changed. Set it between calls,
 *   not while another thread launches or a stream is being captured.
 * kvc_diag_get_path - the current choice of `knob` (-1 for an unknown knob).
 */
#define KVC_DIAG_SCORE 0
#define KVC_DIAG_SELECT 1
#define KVC_DIAG_COMPACT 2
#define KVC_DIAG_DECODE 3
#define KVC_DIAG_DECODE_SPLIT 4
#define KVC_DIAG_SCORE_K 5
#define KVC_DIAG_KNOBS 6
#define KVC_DIAG_SCORE_TWO_PASS 1
#define KVC_DIAG_SCORE_SIMT 2
#define KVC_DIAG_SCORE_CLUSTER 3
#define KVC_DIAG_SELECT_CTA 1
#define KVC_DIAG_COMPACT_GRID 1
#define KVC_DIAG_DECODE_SIMT 1
#define KVC_DIAG_DECODE_TC 2
#define KVC_DIAG_SPLIT_TOKENS 1
kvc_status kvc_diag_set_path(int32_t knob, int32_t choice);
int32_t kvc_diag_get_path(int32_t knob);

#ifdef __cplusplus
}
#endif
#endif /* KVC_H_ */
