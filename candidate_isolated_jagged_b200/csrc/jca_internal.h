// Host-side pieces shared by the translation units of libjca.so (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "jca.h"

namespace jca {

constexpr int kTileM = 128;          // query rows per MMA tile (one softmax group)
constexpr int kItemRows = 256;       // query rows per work item: two tiles sharing every K/V load
constexpr int kTileN = 128;          // keys per key tile
constexpr int kQueueBuckets = 1024;  // cost buckets of the work-queue counting sort

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

int64_t max_work_items(int64_t B, int64_t rows, int H);

// TMA map over a token-major [rows, H, D] bf16 tensor (3-D: D, H, rows), box = {swizzle span,
// 1 head, box_rows}; swizzle span = min(128, 2 D) bytes. Rows past the end read as zeros. Returns
// false when the driver's encoder is unavailable or rejects the map.
bool make_rows_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int H, int D,
                        int box_rows);

// The current device (index < 64) and its multiprocessor count, cached per device. Returns
// JCA_ERR_DEVICE on a device that is not sm_100, JCA_ERR_CUDA when a query fails.
int current_device(int* dev, int* sms);

// Carve-up of the caller's workspace (all offsets 256-byte aligned).
struct WorkspaceLayout {
  size_t seg = 0;        // int8  [rows]   segment IDs built from candidate starts
  size_t hist_lo = 0;    // int64 [B]      (entries in the caller's idx type)
  size_t hist_hi = 0;
  size_t cand_lo = 0;
  size_t cand_hi = 0;
  size_t kv_count = 0;   // int32 [B]      segment-1 tokens per user
  size_t items = 0;      // int4  [max_items]
  size_t n_items = 0;    // int32 [1]
  size_t queue = 0;      // int32 [2]: next item to claim, CTAs finished (the attention kernel's
                         // run-time queue; zeroed by the plan, reset by the kernel's last CTA)
  size_t total = 0;
  int64_t max_items = 0;
};

WorkspaceLayout workspace_layout(int64_t B, int64_t rows, int H);

// Builder launches (no argument checks; callers validate first).
cudaError_t launch_segment_ids(const void* offsets, const void* cand_start, const uint8_t* valid,
                               int attend_padded_history, int64_t B, int64_t T, int idx_bits,
                               int8_t* seg, int32_t* status, cudaStream_t stream);

// history_only != 0: segment -1 is invalid (a frozen history may hold only 1 and 0). With
// cand_start non-null the segment IDs are built from it (every token valid) into seg_out in the
// same pass, and seg is not read.
cudaError_t launch_bounds(const int8_t* seg, const void* offsets, int64_t B, int64_t T,
                          int idx_bits, void* hist_lo, void* hist_hi, void* cand_lo,
                          void* cand_hi, int32_t* kv_count, int history_only, int32_t* status,
                          cudaStream_t stream, const void* cand_start = nullptr,
                          int8_t* seg_out = nullptr);

// queue_ctl non-null: also zero the attention kernel's two run-time queue counters.
cudaError_t launch_work_queue(const void* q_offsets, const void* kv_lo, const void* kv_hi,
                              const int32_t* kv_count, int64_t B, int64_t q_rows,
                              int64_t kv_rows, int H, int idx_bits, int32_t* items,
                              int64_t max_items, int32_t* n_items, int32_t* status,
                              cudaStream_t stream, int32_t* queue_ctl = nullptr);

// Work queue of the per-user causal variant (also zeroes the two run-time queue counters).
cudaError_t launch_causal_queue(const void* offsets, int64_t B, int64_t rows, int H,
                                int idx_bits, int32_t* items, int64_t max_items, int32_t* n_items,
                                int32_t* status, cudaStream_t stream, int32_t* queue_ctl);

// Training with candidate packing: the packed matrix [history runs | candidate runs] as 2B query
// runs over B key intervals. `L` is workspace_layout(2B, Th + Nc, H); q_off2 is the byte offset of
// 2B + 1 offsets (idx_bits type) in the workspace. Writes the segment IDs (when seg is NULL), the
// bounds of the history block, the runs and the work queue.
cudaError_t launch_seqpack_plan(const void* hist_off, const void* cand_off, const int8_t* seg,
                                int64_t B, int64_t Th, int64_t Nc, int H, int idx_bits, char* ws,
                                const WorkspaceLayout& L, size_t q_off2, int32_t* status,
                                cudaStream_t stream);

// Factor tables of the attention kernel's in-tile RoPE rotation (rope_device.cuh): positions lie in
// [history_end - T, history_end], i.e. 128-position blocks q in [qmax - n_coarse + 1, qmax].
struct RopeTables {
  int64_t qmax = 0;
  int64_t n_coarse = 0;
};
RopeTables rope_tables(int64_t T, int64_t history_end);
cudaError_t launch_rope_tables(float2* coarse, float2* fine, int d, const RopeTables& t,
                               float base, cudaStream_t stream);

// Workspace of the candidate-packing entry points: workspace_layout(2B, T, H) followed by the
// 2B + 1 query-run offsets.
struct SeqpackLayout {
  WorkspaceLayout base;
  size_t q_off2 = 0;
  size_t total = 0;
};

inline SeqpackLayout seqpack_layout(int64_t B, int64_t T, int H) {
  SeqpackLayout s;
  s.base = workspace_layout(2 * B, T, H);
  s.q_off2 = align_up(s.base.total, 256);
  s.total = align_up(s.q_off2 + 8 * (size_t)(2 * B + 1), 256);
  return s;
}

}  // namespace jca
