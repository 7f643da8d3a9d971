/*
 * jca.h — C ABI of libjca.so: jagged, candidate-isolated softmax attention on NVIDIA B200 (sm_100a).
 *
 * A jagged batch holds B user rows laid out as [user prefix | history | candidates]
 * (候选隔离注意力掩码, section 为什么需要它), packed back to back and described by offsets
 * ('HSTU scale' tutorial, section 手算 padding 的浪费与 offset). Every token carries a segment ID:
 * 1 = prefix/history, -1 = candidate, 0 = padding (候选隔离注意力掩码, section 段 ID：掩码的表达方式).
 * Prefix and history attend to each other bidirectionally and never to candidates; each candidate
 * attends to its user's prefix, history and itself; no position reads across a user boundary.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.     Every pointer argument is DEVICE memory owned by the caller; the library never
 *             allocates device memory and never frees what it is given. Scratch space, where an
 *             entry point needs it, is the caller's `workspace` of at least
 *             jca_workspace_bytes(...) bytes, 256-byte aligned.
 * Layout.     Q/K/V/out are token-major [rows, H, d_head] (row stride H*d_head elements), bf16
 *             unless stated; offsets/lengths/candidate starts/bounds are int32 or int64 as chosen
 *             by `idx_bits` (32 or 64); segment IDs are int8; the padding mask is uint8 (1 = real).
 * Streams.    Every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *             stream) and returns without synchronising the host.
 * Host errors.  Argument errors are detected before anything is enqueued and returned as a
 *             negative JCA_ERR_* code; nothing is written then.
 * Device errors. Data errors found on the device (bad offsets, bad candidate starts, a history
 *             token after a candidate, a pipeline wait that timed out) are recorded as a positive
 *             JCA_STATUS_* code in *status (int32, device memory). The first error wins. Every
 *             kernel of the library reads *status when it starts and does nothing when it is
 *             non-zero, so an error stops every later call that shares the status word. The caller
 *             zeroes *status before the first call and reads it back when convenient.
 * Limits.     rows < 2^31 per tensor; H >= 1; d_head in {16, 32, 64, 128}; pointers of Q/K/V/out
 *             16-byte aligned.
 * Numerics.   bf16 inputs, fp32 accumulation and fp32 online softmax; `scale` <= 0 selects
 *             1/sqrt(d_head). Inputs are assumed finite.
 * Device.     sm_100a (B200). On another device the attention entry points return JCA_ERR_DEVICE.
 */
#ifndef JCA_H_
#define JCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* jca_stream_t;

enum jca_code {
  JCA_OK = 0,
  /* host-side argument errors (return values) */
  JCA_ERR_NULL = -1,        /* a required pointer is NULL */
  JCA_ERR_SHAPE = -2,       /* B < 0, rows < 0, H < 1, or a size beyond the limits */
  JCA_ERR_HEAD_DIM = -3,    /* d_head not in {16, 32, 64, 128} */
  JCA_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned (workspace: 256-byte) */
  JCA_ERR_IDX_BITS = -5,    /* idx_bits not 32 or 64 */
  JCA_ERR_WORKSPACE = -6,   /* workspace smaller than jca_workspace_bytes(...) */
  JCA_ERR_CUDA = -7,        /* a CUDA runtime/driver call failed (launch, tensor map, ...) */
  JCA_ERR_DEVICE = -8,      /* current device is not sm_100 */
  JCA_ERR_SCRATCH_LIMIT = -9, /* jagged_cand_attn_fwd_noalloc: problem needs more scratch than
                                 the library's static array (jca_noalloc_scratch_bytes()) */
  /* device-side data errors (written to *status) */
  JCA_STATUS_BAD_LENGTH = 1,     /* a sequence length is negative, or offsets overflow int32 */
  JCA_STATUS_BAD_OFFSETS = 2,    /* offsets[0] != 0, offsets decrease, or offsets[B] != rows */
  JCA_STATUS_BAD_CAND_START = 3, /* candidate_start[b] outside [0, row length] */
  JCA_STATUS_BAD_SEG_LAYOUT = 4, /* a segment-1 token follows a candidate inside a row */
  JCA_STATUS_BAD_SEG_VALUE = 5,  /* a segment ID outside {-1, 0, 1} */
  JCA_STATUS_QUEUE_OVERFLOW = 6, /* more work items than the workspace bound (internal) */
  JCA_STATUS_BAD_SPLIT = 7,      /* jca_stack_fwd: the segment IDs hold a different number of
                                    history or candidate tokens than the caller's Th / Nc */
  JCA_STATUS_TIMEOUT = 16        /* a pipeline wait in the attention kernel gave up */
};

/* Text of a JCA_ERR_* or JCA_STATUS_* code (static storage; never NULL). */
const char* jca_status_string(int code);

/*
 * Offsets of a ragged batch: offsets[0] = 0 and offsets[b+1] = offsets[b] + lengths[b]
 * ('HSTU scale' tutorial, section 手算 padding 的浪费与 offset: sequence b is
 * values[offsets[b]:offsets[b+1]]).
 *   lengths  [B] int32/int64 (idx_bits), read;   offsets [B+1] same type, written.
 *   B >= 0 (B = 0 writes offsets[0] = 0).
 * Device errors: a negative length, or (idx_bits = 32) a total beyond INT32_MAX ->
 * JCA_STATUS_BAD_LENGTH; offsets are then unspecified.
 */
int jca_offsets_from_lengths(const void* lengths, void* offsets, int64_t B, int idx_bits,
                             int32_t* status, jca_stream_t stream);

/*
 * Segment IDs of every packed token (候选隔离注意力掩码, section 段 ID：掩码的表达方式):
 * for position idx of user row b (row-relative), is_candidate = idx >= candidate_start[b];
 * valid = valid_mask[token] (or valid_mask[token] OR NOT is_candidate when
 * attend_padded_history != 0); seg = valid ? (is_candidate ? -1 : 1) : 0.
 *   offsets [B+1] and candidate_start [B] (row-relative) in the idx_bits type, read.
 *   valid_mask [T] uint8 or NULL (NULL = every token is real), read.
 *   seg [T] int8, written.
 * Device errors: offsets not starting at 0, decreasing or not ending at T ->
 * JCA_STATUS_BAD_OFFSETS; candidate_start[b] outside [0, offsets[b+1]-offsets[b]] ->
 * JCA_STATUS_BAD_CAND_START.
 */
int jca_build_segment_ids(const void* offsets, const void* candidate_start,
                          const uint8_t* valid_mask, int attend_padded_history,
                          int64_t B, int64_t T, int idx_bits, int8_t* seg,
                          int32_t* status, jca_stream_t stream);

/*
 * Per-user history and candidate intervals (候选隔离注意力掩码, section 段 ID：掩码的表达方式,
 * bounds_from_segment_ids): [hist_lo, hist_hi) runs from the first to one past the last
 * segment-1 token of the row, [cand_lo, cand_hi) from the first to one past the last
 * segment -1 token; indices are absolute packed positions. An empty history gives
 * hist_lo = hist_hi = offsets[b]; no candidate gives cand_lo = cand_hi = offsets[b+1]
 * (a reading: the pages do not state the empty convention).
 *   seg [T] int8 and offsets [B+1] (idx_bits type), read.
 *   hist_lo, hist_hi, cand_lo, cand_hi [B] in the idx_bits type, written.
 * Device errors: bad offsets -> JCA_STATUS_BAD_OFFSETS; a segment ID outside {-1,0,1} ->
 * JCA_STATUS_BAD_SEG_VALUE; a segment-1 token after a candidate inside one row ->
 * JCA_STATUS_BAD_SEG_LAYOUT.
 */
int jca_bounds_from_segment_ids(const int8_t* seg, const void* offsets, int64_t B, int64_t T,
                                int idx_bits, void* hist_lo, void* hist_hi, void* cand_lo,
                                void* cand_hi, int32_t* status, jca_stream_t stream);

/*
 * Work queue of the attention kernels: one item per (user b, head h, 256-row query block t),
 * ordered by cost (the number of 128-key tiles over the user's key interval), largest first,
 * so that a persistent kernel taking items in order approximates longest-processing-time-first.
 * Items of equal cost may come in any order.
 *   q_offsets [B+1], kv_lo [B], kv_hi [B] in the idx_bits type, read (absolute rows; the key
 *   interval of user b is [kv_lo[b], kv_hi[b])).
 *   kv_count [B] int32 or NULL: number of valid keys inside the interval; when it differs from
 *   kv_hi - kv_lo the user's key tiles are masked key by key.
 *   items [max_items * 4] int32, written; item i = {first query row, (h << 9) | rows in the
 *   block (1..256), kv_lo, (kv_hi - kv_lo) | (holes << 31)}.
 *   n_items [1] int32, written.
 *   q_rows / kv_rows: rows of the query and key tensors (q_offsets[B] must equal q_rows;
 *   every key interval must lie inside [0, kv_rows)).
 * Device errors: bad q_offsets or a key interval outside [0, kv_rows) -> JCA_STATUS_BAD_OFFSETS;
 * more than max_items items -> JCA_STATUS_QUEUE_OVERFLOW. n_items is 0 after any error.
 */
int jca_build_work_queue(const void* q_offsets, const void* kv_lo, const void* kv_hi,
                         const int32_t* kv_count, int64_t B, int64_t q_rows, int64_t kv_rows,
                         int H, int idx_bits, int32_t* items, int64_t max_items,
                         int32_t* n_items, int32_t* status, jca_stream_t stream);

/* Upper bound on the work items of B users with `rows` query rows in total and H heads. */
int64_t jca_max_work_items(int64_t B, int64_t rows, int H);

/*
 * Workspace bytes needed by jagged_cand_attn_fwd (rows = T) or cand_only_attn_fwd
 * (rows = Nc) for B users, H heads and head size d_head. Returns 0 for invalid sizes.
 */
size_t jca_workspace_bytes(int64_t B, int64_t rows, int H, int d_head);

/*
 * Jagged candidate-isolated attention forward (候选隔离注意力掩码, sections 段 ID：掩码的表达方式
 * and 掩码长什么样): for every user row and head, softmax(scale * Q K^T + mask) V with
 *   mask[q, kv] = (kv is history AND (q is history OR q is a candidate))
 *              OR (q and kv are the same candidate position),
 * evaluated from segment intervals inside the kernel; no [L, L] mask is materialised
 * (section 设计决策). Query rows of padding (segment 0) output 0.
 *   q, k, v  [T, H, d_head] bf16, read.
 *   out      [T, H, d_head] bf16 (out_fp32 = 0) or fp32 (out_fp32 != 0), written.
 *   offsets  [B+1] (idx_bits type), read.
 *   candidate_start [B] row-relative (idx_bits type), read when seg == NULL.
 *   seg      [T] int8 or NULL. When given it replaces candidate_start (this is how padding
 *            enters: build it with jca_build_segment_ids); when NULL no token is padding.
 *   scale    softmax scale; <= 0 selects 1/sqrt(d_head).
 *   workspace / workspace_bytes: >= jca_workspace_bytes(B, T, H, d_head).
 * Runs on `stream`: segment IDs (when seg == NULL), bounds, work queue, attention kernel.
 * Device errors: as the builders above, plus JCA_STATUS_TIMEOUT.
 */
int jagged_cand_attn_fwd(const void* q, const void* k, const void* v, void* out, int out_fp32,
                         const void* offsets, const void* candidate_start, const int8_t* seg,
                         int64_t B, int64_t T, int H, int d_head, float scale, int idx_bits,
                         void* workspace, size_t workspace_bytes, int32_t* status,
                         jca_stream_t stream);

/*
 * The two halves of jagged_cand_attn_fwd, for callers that run several attention layers over one
 * batch layout (the ranker's full layers all share it):
 *   jagged_cand_attn_plan  derives everything that depends only on the layout — segment IDs
 *                          (when seg == NULL), bounds and the work queue — into `workspace`;
 *   jagged_cand_attn_run   launches only the attention kernel, reading that plan. It may be called
 *                          any number of times after one plan, as long as `workspace` and the
 *                          layout arguments (seg, B, T, H, d_head) are the same as at plan time.
 * Arguments, errors and workspace size are as for jagged_cand_attn_fwd.
 * Sharing a workspace: the attention kernel claims its work items at run time from a counter in
 * the workspace (zeroed by the plan, reset by the kernel's last block for the next run). Calls that
 * use one workspace must therefore not overlap on the GPU: order them on one stream (or with
 * events). Runs that may overlap, e.g. on two streams, each need their own workspace (and plan).
 * The same holds for every entry point below that takes a workspace.
 */
int jagged_cand_attn_plan(const void* offsets, const void* candidate_start, const int8_t* seg,
                          int64_t B, int64_t T, int H, int d_head, int idx_bits, void* workspace,
                          size_t workspace_bytes, int32_t* status, jca_stream_t stream);

int jagged_cand_attn_run(const void* q, const void* k, const void* v, void* out, int out_fp32,
                         const int8_t* seg, int64_t B, int64_t T, int H, int d_head, float scale,
                         void* workspace, size_t workspace_bytes, int32_t* status,
                         jca_stream_t stream);

/*
 * Candidate-only attention layer (候选隔离注意力掩码, section 只更新候选的末尾层; the arguments mirror
 * the page's operator inputs candidate_q, history_k, history_v, own_k, own_v): each candidate of
 * user b attends to the frozen history keys/values of user b and to its own key/value only.
 * Its result equals the candidate rows of jagged_cand_attn_fwd on the same K/V: bit for bit at
 * d_head <= 32; at d_head 64 and 128 the candidate's own key and value go through the tensor core
 * (its own weight rounded to bf16 like every other weight), and the two agree within the parity
 * tolerance (max-abs 1e-2, rel-L2 5e-3).
 *   cand_q, own_k, own_v [Nc, H, d_head] bf16, read; cand_offsets [B+1] (idx_bits type).
 *   hist_k, hist_v [Th, H, d_head] bf16, read; hist_offsets [B+1] (idx_bits type).
 *   hist_seg [Th] int8 or NULL: 1 = valid history row, 0 = padding (NULL = all valid).
 *   out [Nc, H, d_head] bf16 or fp32 (out_fp32), written.
 *   workspace / workspace_bytes: >= jca_workspace_bytes(B, Nc, H, d_head).
 * Device errors: bad offsets -> JCA_STATUS_BAD_OFFSETS; hist_seg values other than 0/1 ->
 * JCA_STATUS_BAD_SEG_VALUE; JCA_STATUS_TIMEOUT.
 */
int cand_only_attn_fwd(const void* cand_q, const void* own_k, const void* own_v,
                       const void* cand_offsets, const void* hist_k, const void* hist_v,
                       const void* hist_offsets, const int8_t* hist_seg, void* out, int out_fp32,
                       int64_t B, int64_t Nc, int64_t Th, int H, int d_head, float scale,
                       int idx_bits, void* workspace, size_t workspace_bytes, int32_t* status,
                       jca_stream_t stream);

/*
 * The two halves of cand_only_attn_fwd (see jagged_cand_attn_plan/run): the plan holds the key
 * intervals and the work queue of the candidate/history layout; `hist_seg` given to run must be the
 * one given to plan.
 */
int cand_only_attn_plan(const void* cand_offsets, const void* hist_offsets, const int8_t* hist_seg,
                        int64_t B, int64_t Nc, int64_t Th, int H, int d_head, int idx_bits,
                        void* workspace, size_t workspace_bytes, int32_t* status,
                        jca_stream_t stream);

int cand_only_attn_run(const void* cand_q, const void* own_k, const void* own_v,
                       const void* hist_k, const void* hist_v, const int8_t* hist_seg, void* out,
                       int out_fp32, int64_t B, int64_t Nc, int64_t Th, int H, int d_head,
                       float scale, void* workspace, size_t workspace_bytes, int32_t* status,
                       jca_stream_t stream);

/*
 * jagged_cand_attn_fwd without a workspace argument. (No counterpart on the source pages: this is
 * an interface for callers, not part of the method.)
 *
 * For callers that cannot allocate device memory when they call: a serving loop whose memory is
 * fixed up front, a plugin that is handed only its input and output tensors, or code that must not
 * pay cudaMalloc's implicit device synchronisation on the request path. The scratch this call
 * needs (segment IDs, per-user bounds, the work queue) lives in one static device array inside the
 * library, jca_noalloc_scratch_bytes() = 8 MiB, which every GPU that loads the library holds until
 * the process exits. The call allocates and frees nothing.
 *
 *   Arguments, results and device-side errors: as jagged_cand_attn_fwd.
 *   Size limit: when jca_workspace_bytes(B, T, H, d_head) exceeds jca_noalloc_scratch_bytes(),
 *   the call returns JCA_ERR_SCRATCH_LIMIT before enqueuing anything (use jagged_cand_attn_fwd
 *   with a workspace then). Roughly: T + 44 B + 16 H (T/128 + B + 1) bytes must fit in 8 MiB.
 *   First use per device: the array's device address is looked up (cudaGetSymbolAddress, with
 *   that device current) and cached, by jca_noalloc_prepare() or else by the first call. Call
 *   jca_noalloc_prepare() with each device current before any stream capture (inside a capture
 *   the lookup may fail, and the call then returns JCA_ERR_CUDA).
 *   Sharing: all calls on a device use the same array, which keeps the last call's contents (no
 *   part of it needs to start at zero). Calls whose execution overlaps on the GPU — on different
 *   streams without ordering between them, or from several host threads — race on it; order them
 *   on one stream or with events.
 */
size_t jca_noalloc_scratch_bytes(void);

/* Looks up and caches the static array's device address for the current device, so that later
 * jagged_cand_attn_fwd_noalloc calls on it do no CUDA runtime call beyond their launches.
 * Returns JCA_OK, or JCA_ERR_CUDA when the lookup fails (no usable device). Enqueues nothing. */
int jca_noalloc_prepare(void);

int jagged_cand_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                 int out_fp32, const void* offsets, const void* candidate_start,
                                 const int8_t* seg, int64_t B, int64_t T, int H, int d_head,
                                 float scale, int idx_bits, int32_t* status, jca_stream_t stream);

/* Self-test of the failure path (no counterpart on the pages): launches one block whose thread runs
 * the library's bounded pipeline wait on a barrier that nothing completes. After the wait's limit
 * (2 s) it records JCA_STATUS_TIMEOUT in *status (if *status was 0) and the block returns, as a
 * kernel whose pipeline stalls does; the context stays usable. Enqueues one kernel on `stream`.
 * Errors: JCA_ERR_NULL, JCA_ERR_DEVICE, JCA_ERR_CUDA. */
int jca_selftest_wait_timeout(int32_t* status, jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Several GPUs: users are independent (no position reads across a user boundary: 候选隔离注意力掩码,
 * section 段 ID：掩码的表达方式; 'HSTU scale' tutorial, section 手算 padding 的浪费与 offset), so one
 * batch's users are split over the GPUs with no exchange in the forward pass; each GPU plans and
 * runs its own users and keeps its outputs. These two calls are HOST functions on HOST memory: they
 * enqueue nothing and need no GPU.
 * ------------------------------------------------------------------------------------------- */

/* Tile cost of one user as the attention kernel sees it: ceil(row_len / 128) query tiles times
 * max(1, ceil(n_keys / 128)) key tiles (n_keys = the user's segment-1 keys); 0 for an empty row. */
int64_t jca_user_tile_cost(int64_t row_len, int64_t n_keys);

/* Longest-processing-time-first split of B users over n_shards GPUs: users in order of decreasing
 * jca_user_tile_cost (ties in user order), each to the least-loaded shard so far (ties to the lowest
 * shard index). Deterministic, so every rank computes the same split from the same lengths. The
 * largest shard load stays within Graham's list-scheduling bound, total / n_shards + (1 - 1 /
 * n_shards) * max cost, and within 4/3 - 1/(3 n_shards) of the best split.
 *   row_len [B], n_keys [B]  int64, host memory, read (0 <= n_keys <= row_len).
 *   shard   [B] int32, host memory, written: the shard of each user, in [0, n_shards).
 *   load    [n_shards] int64, host memory, written (nullable): total cost per shard.
 * Errors: JCA_ERR_SHAPE (B < 0, n_shards < 1, a negative length, n_keys > row_len), JCA_ERR_NULL. */
int jca_shard_users(const int64_t* row_len, const int64_t* n_keys, int64_t B, int n_shards,
                    int32_t* shard, int64_t* load);

/* ---------------------------------------------------------------------------------------------
 * Right-anchored rotary position embedding (候选隔离注意力掩码, section 位置编码：候选共用一个位置):
 * the history is right-aligned so that the newest history record of every user sits at
 * history_end - 1 whatever its length, and every candidate sits at history_end; candidate order
 * therefore never enters a score. Applied to the queries and keys before jagged_cand_attn_fwd or
 * cand_only_attn_fwd (scores depend only on position differences, so any constant history_end
 * gives the same attention output).
 * ------------------------------------------------------------------------------------------- */

/* Positions of the packed tokens of a segment-ID array. Per user row [offsets[b], offsets[b+1]):
 * the k-th segment-1 token (prefix and history, in row order) of a row with n of them gets
 * history_end - n + k; a candidate (segment -1) gets history_end; a padding token (segment 0)
 * gets history_end - n + (segment-1 tokens before it), a value no score reads.
 *   seg        device int8 [T]; offsets device [B+1] (idx_bits 32 or 64);
 *   positions  device int32 [T] (written; values are clamped to the int32 range).
 * Errors: as jca_bounds_from_segment_ids for the arguments; JCA_STATUS_BAD_OFFSETS in *status for
 * offsets that are not monotone or do not end at T (then nothing further is written). */
int jca_rope_positions(const int8_t* seg, const void* offsets, int64_t B, int64_t T,
                       int64_t history_end, int idx_bits, int32_t* positions, int32_t* status,
                       jca_stream_t stream);

/* Rotates every row of a token-major [T, H, d_head] bf16 tensor by its token's position: for each
 * head and each pair (j, j + d_head/2), (a, b) -> (a cos(p t_j) - b sin(p t_j),
 * a sin(p t_j) + b cos(p t_j)) with t_j = base^(-2j/d_head), computed in fp32 and rounded once to
 * bf16. out may equal x (in place); both 16-byte aligned, caller-owned device memory.
 *   positions  device int32 [T], e.g. from jca_rope_positions; base > 1 (10000 in the usual form).
 * Errors: JCA_ERR_HEAD_DIM, JCA_ERR_SHAPE (T < 0, H < 1, base <= 1), JCA_ERR_NULL, JCA_ERR_ALIGN,
 * JCA_ERR_CUDA. Nothing is reported through a status word: every input is valid. */
int jca_apply_rope(const void* x, void* out, const int32_t* positions, int64_t T, int H,
                   int d_head, float base, jca_stream_t stream);

/* jagged_cand_attn_fwd with right-anchored RoPE applied inside the attention kernel: q and k are
 * given UNROTATED and are left unchanged; each Q and K tile is rotated in shared memory, after it
 * lands and before the tensor core reads it, by the positions jca_rope_positions gives the batch's
 * segment IDs (history_end as there) and base rope_base. The rotated values are those
 * jca_apply_rope would store (the same cosines and sines, rotation in fp32, one rounding to bf16),
 * so the output equals jca_apply_rope on q and k followed by jagged_cand_attn_fwd, up to the
 * summation order of the candidates' own scores. Saves that pre-pass's read and write of q and k.
 *   Other arguments as jagged_cand_attn_fwd; rope_base > 1; positions must fit int32
 *   (history_end <= INT32_MAX and history_end - T >= INT32_MIN, else JCA_ERR_SHAPE).
 *   workspace >= jca_rope_attn_workspace_bytes(B, T, H, d_head) bytes, 256-byte aligned.
 * Device errors: as jagged_cand_attn_fwd. */
size_t jca_rope_attn_workspace_bytes(int64_t B, int64_t T, int H, int d_head);

int jagged_cand_attn_rope_fwd(const void* q, const void* k, const void* v, void* out, int out_fp32,
                              const void* offsets, const void* candidate_start, const int8_t* seg,
                              int64_t B, int64_t T, int H, int d_head, float scale,
                              int64_t history_end, float rope_base, int idx_bits, void* workspace,
                              size_t workspace_bytes, int32_t* status, jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Variant: per-user causal attention on the packed layout (prior art on the pages: the early
 * demo ranker's lower-triangular mask, noted in the FAQ of 候选隔离注意力掩码, and the
 * block-diagonal causal varlen attention of the contest repository). Row i of user b attends to
 * rows j <= i of user b; no segment IDs (every row is real).
 *   q, k, v [T, H, d_head] bf16, read; out [T, H, d_head] bf16 or fp32 (out_fp32), written.
 *   offsets [B+1] (idx_bits type), read. workspace >= jca_workspace_bytes(B, T, H, d_head).
 * Device errors: bad offsets -> JCA_STATUS_BAD_OFFSETS (nothing written); JCA_STATUS_TIMEOUT.
 * ------------------------------------------------------------------------------------------- */
int jagged_causal_attn_fwd(const void* q, const void* k, const void* v, void* out, int out_fp32,
                           const void* offsets, int64_t B, int64_t T, int H, int d_head,
                           float scale, int idx_bits, void* workspace, size_t workspace_bytes,
                           int32_t* status, jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Variant: UG-Sep's masked cross-attention, the separated residual of a pyramid TokenMixer (UG-Sep
 * page, "Compute Only Once: UG-Separated TokenMixer", sections 分离残差连接 and UG-Separated
 * Mixup 与 mask). Per sample and head, the T_out output tokens (queries) attend to the T_in input
 * tokens (keys and values) under M_UG: an output i < c_u (a U-token) reads only the inputs
 * j < n_u (the U-tokens), every other output reads all T_in inputs. The page's formulas for R and
 * Y were lost in extraction; the op computes R = softmax(scale Q K^T under M_UG) V and, with a
 * residual, Y = residual + R. A U output with n_u = 0 sees no key: R = 0 there.
 *   q, residual  [B, T_out, H, d_head] bf16, read (residual nullable: then out = R).
 *   k, v         [B, T_in, H, d_head] bf16, read (may be the same tensor).
 *   out          [B, T_out, H, d_head], written: bf16, or fp32 when out_fp32 != 0. With a bf16
 *                output, out may be the residual tensor itself (Y = X + R in place: each row is
 *                read before the same thread writes it, and no other thread touches it).
 *   All caller-owned device memory, 16-byte aligned, token-major with row stride H * d_head.
 *   0 <= T_out, T_in <= 128 (TokenMixer token counts), 0 <= c_u <= T_out, 0 <= n_u <= T_in;
 *   scale <= 0 means 1/sqrt(d_head).
 * Errors: JCA_ERR_SHAPE (a size outside those ranges, H < 1, or B * max(T_out, T_in) beyond the
 * 32-bit row range), JCA_ERR_HEAD_DIM, JCA_ERR_NULL, JCA_ERR_ALIGN, JCA_ERR_DEVICE, JCA_ERR_CUDA.
 * The launch is a no-op when *status is already nonzero; a pipeline wait that gives up records
 * JCA_STATUS_TIMEOUT. No workspace.
 * ------------------------------------------------------------------------------------------- */
int ug_masked_cross_attn_fwd(const void* q, const void* k, const void* v, const void* residual,
                             void* out, int out_fp32, int64_t B, int T_out, int T_in, int c_u,
                             int n_u, int H, int d_head, float scale, int32_t* status,
                             jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Training: the forward with its log-sum-exp, and the backward pass. The pages train on the same
 * packed layout they serve (候选隔离注意力掩码, section 训练时的序列打包: several users' sequences
 * in one packed matrix, split at cu_seqlens = the offsets here), under the same mask.
 * ------------------------------------------------------------------------------------------- */

/* jagged_cand_attn_fwd that also writes lse [T, H] fp32 (4-byte aligned): per row and head, the
 * natural log of the row's softmax denominator, log sum_j exp(scale q.k_j) over the keys the mask
 * lets it see (its own key included for a candidate); -inf for a padding row. The backward pass
 * rebuilds the probabilities from it. Other arguments and errors as jagged_cand_attn_fwd. */
int jagged_cand_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, int out_fp32,
                             float* lse, const void* offsets, const void* candidate_start,
                             const int8_t* seg, int64_t B, int64_t T, int H, int d_head,
                             float scale, int idx_bits, void* workspace, size_t workspace_bytes,
                             int32_t* status, jca_stream_t stream);

/* Workspace bytes of jagged_cand_attn_bwd (0 for invalid sizes). */
size_t jca_bwd_workspace_bytes(int64_t B, int64_t T, int H, int d_head);

/*
 * Gradients of jagged_cand_attn_fwd for the upstream gradient dout: per user and head, with P the
 * forward's probabilities, dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)), dQ = scale dS K,
 * dK = scale dS^T Q. Rows of padding get zero gradients; a candidate's own key and value receive
 * gradient from that candidate only.
 *   q, k, v, dout [T, H, d_head] bf16, read; out [T, H, d_head] bf16 or fp32 (out_fp32), the
 *   forward's output, read; lse [T, H] fp32 from jagged_cand_attn_fwd_lse, read.
 *   dq, dk, dv [T, H, d_head] bf16 or fp32 (grad_fp32), written (every row).
 *   offsets, candidate_start, seg, B, T, H, d_head, scale, idx_bits: as for the forward (the same
 *   values the forward was called with).
 *   workspace >= jca_bwd_workspace_bytes(B, T, H, d_head) bytes, 256-byte aligned.
 * Device errors: as jagged_cand_attn_fwd (the layout is validated again), plus
 * JCA_STATUS_QUEUE_OVERFLOW (internal) and JCA_STATUS_TIMEOUT.
 */
int jagged_cand_attn_bwd(const void* q, const void* k, const void* v, const void* out, int out_fp32,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         int grad_fp32, const void* offsets, const void* candidate_start,
                         const int8_t* seg, int64_t B, int64_t T, int H, int d_head, float scale,
                         int idx_bits, void* workspace, size_t workspace_bytes, int32_t* status,
                         jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Training with candidate packing (候选隔离注意力掩码, section 训练时的序列打包: users' sequences are
 * packed into one matrix split at cu_seqlens, and the candidates are stored apart, all in one
 * block, each candidate's representation read back at its candidate_positions entry). Packing
 * changes where rows sit, not what they compute: the mask is the serving one.
 *
 * Layout (a reading; the pages name it without drawing it): one packed matrix of T = Th + Nc rows.
 * Rows [0, Th) hold every user's prefix + history run back to back, split at hist_offsets [B+1]
 * (hist_offsets[0] = 0, hist_offsets[B] = Th: the cu_seqlens). Rows [Th, T) hold every user's
 * candidate run back to back, split at cand_offsets [B+1], relative to the block (cand_offsets[0]
 * = 0, cand_offsets[B] = Nc). Candidate c therefore sits at row Th + c: candidate_positions is
 * Th + [0, Nc). User b's history rows see the segment-1 rows of its own history run, and its
 * candidates see those plus themselves.
 *   seg [T] int8 or NULL: NULL means history rows 1 and candidate rows -1; when given, history
 *       rows hold 1 or 0 (padding) and candidate rows -1 or 0 (an empty candidate slot).
 * ------------------------------------------------------------------------------------------- */

/* Workspace bytes of jagged_cand_attn_seqpack_fwd (0 for invalid sizes). */
size_t jca_seqpack_workspace_bytes(int64_t B, int64_t Th, int64_t Nc, int H, int d_head);

/*
 * Forward over the candidate-packed matrix.
 *   q, k, v [T, H, d_head] bf16, read; out [T, H, d_head] bf16 or fp32 (out_fp32), written.
 *   lse [T, H] fp32 or NULL: when given, the natural-log softmax denominator of every row and head
 *       (as jagged_cand_attn_fwd_lse; -inf for padding rows), for the backward pass.
 *   hist_offsets, cand_offsets [B+1] (idx_bits type), read; seg as above.
 *   workspace >= jca_seqpack_workspace_bytes(B, Th, Nc, H, d_head) bytes, 256-byte aligned.
 * Device errors: bad hist_offsets or cand_offsets -> JCA_STATUS_BAD_OFFSETS (nothing written); a
 * segment ID outside the values above -> JCA_STATUS_BAD_SEG_VALUE; JCA_STATUS_TIMEOUT.
 */
int jagged_cand_attn_seqpack_fwd(const void* q, const void* k, const void* v, void* out,
                                 int out_fp32, float* lse, const void* hist_offsets,
                                 const void* cand_offsets, const int8_t* seg, int64_t B,
                                 int64_t Th, int64_t Nc, int H, int d_head, float scale,
                                 int idx_bits, void* workspace, size_t workspace_bytes,
                                 int32_t* status, jca_stream_t stream);

/* Workspace bytes of jagged_cand_attn_seqpack_bwd (0 for invalid sizes). */
size_t jca_seqpack_bwd_workspace_bytes(int64_t B, int64_t Th, int64_t Nc, int H, int d_head);

/*
 * Gradients over the candidate-packed matrix, as jagged_cand_attn_bwd: dq, dk, dv [T, H, d_head]
 * (bf16, or fp32 with grad_fp32), every row written; a history key's dK and dV collect the
 * gradient of its user's history rows and candidate rows, a candidate's own key and value that of
 * the candidate alone, padding rows get 0.
 *   out and lse from jagged_cand_attn_seqpack_fwd on the same inputs; other arguments as the
 *   forward. workspace >= jca_seqpack_bwd_workspace_bytes(B, Th, Nc, H, d_head) bytes.
 * Device errors: as the forward, plus JCA_STATUS_QUEUE_OVERFLOW (internal).
 */
int jagged_cand_attn_seqpack_bwd(const void* q, const void* k, const void* v, const void* out,
                                 int out_fp32, const void* dout, const float* lse, void* dq,
                                 void* dk, void* dv, int grad_fp32, const void* hist_offsets,
                                 const void* cand_offsets, const int8_t* seg, int64_t B,
                                 int64_t Th, int64_t Nc, int H, int d_head, float scale,
                                 int idx_bits, void* workspace, size_t workspace_bytes,
                                 int32_t* status, jca_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Layer stack with candidate-only tail layers (候选隔离注意力掩码, section 只更新候选的末尾层 and its
 * flowchart): the first n_layers - n_cand_only layers run over whole rows [prefix | history |
 * candidates] under the isolation mask; then the states are split into the frozen history
 * (segment 1, prefix included) and the candidates (segment -1), and each of the last n_cand_only
 * layers updates only the candidates: their queries attend to the frozen history's keys/values
 * (projected with that layer's weights) and to their own key/value. Padding rows (segment 0) and
 * history rows keep the states they had at the split.
 *
 * A layer is x <- x + Attn(x Wq, x Wk, x Wv) Wo with square D x D weights, D = H * d_head, no bias
 * and no normalisation (the pages describe only the attention part of a layer); with
 * history_end >= 0, right-anchored RoPE (jca_rope_positions / jca_apply_rope, base rope_base) is
 * applied to the queries and keys of every layer. Projections are bf16 GEMMs with fp32
 * accumulation (cuBLASLt); every projection, RoPE output, attention output and residual sum is
 * rounded once to bf16.
 * ------------------------------------------------------------------------------------------- */

/* Workspace bytes of jca_stack_fwd (0 for invalid sizes). */
size_t jca_stack_workspace_bytes(int64_t B, int64_t T, int64_t Nc, int64_t Th, int H, int d_head);

/*
 *   x        [T, D] bf16, read (the first layer's input); x_out [T, D] bf16, written (may equal x).
 *   weights  [n_layers, 4, D, D] bf16, read: per layer Wq, Wk, Wv, Wo, each row-major [D_in, D_out]
 *            so that a projection is x @ W.
 *   n_cand_only  number of candidate-only tail layers, 0 <= n_cand_only <= n_layers.
 *   offsets [B+1], candidate_start [B] (row-relative) and seg [T] (nullable) as for
 *            jagged_cand_attn_fwd.
 *   Nc, Th   total candidate (segment -1) and history (segment 1) tokens of the batch; the host
 *            needs them to size the tail layers without reading device memory. When they disagree
 *            with the segment IDs, *status gets JCA_STATUS_BAD_SPLIT and the tail layers do not run.
 *            Ignored (may be 0) when n_cand_only = 0. Nc + Th <= T.
 *   scale    softmax scale (<= 0: 1/sqrt(d_head)); history_end < 0 turns RoPE off.
 *   workspace >= jca_stack_workspace_bytes(B, T, Nc, Th, H, d_head) bytes, 256-byte aligned
 *            (about (4 T + 2 (Nc + Th)) D bf16 elements plus 32 MiB for the GEMMs).
 * Errors: the host errors of jagged_cand_attn_fwd; device errors in *status as the builders and
 * attention kernels report them. After a device error x_out is unspecified (the GEMMs do not read
 * the status word); the other kernels do nothing further.
 */
int jca_stack_fwd(const void* x, void* x_out, const void* weights, int n_layers, int n_cand_only,
                  const void* offsets, const void* candidate_start, const int8_t* seg, int64_t B,
                  int64_t T, int64_t Nc, int64_t Th, int H, int d_head, float scale,
                  int64_t history_end, float rope_base, int idx_bits, void* workspace,
                  size_t workspace_bytes, int32_t* status, jca_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JCA_H_ */
