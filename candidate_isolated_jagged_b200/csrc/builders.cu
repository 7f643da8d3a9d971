// Builder kernels of the jagged batch: offsets from lengths, segment IDs, per-user bounds, and the
// cost-sorted work queue consumed by the attention kernels. All of them are sync-free: errors go
// to the device status word and every kernel returns at once when that word is already non-zero.
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "jca_internal.h"

namespace jca {
namespace {

__device__ __forceinline__ void set_status(int32_t* status, int code) {
  atomicCAS(status, 0, (int32_t)code);
}

// ---------------------------------------------------------------------------------------------
// Offsets: exclusive prefix sum of lengths ('HSTU scale' tutorial, section 手算 padding 的浪费与
// offset). One block walks the lengths in chunks of blockDim.x, carrying the running total.
// ---------------------------------------------------------------------------------------------
template <typename IdxT>
__global__ void __launch_bounds__(1024) offsets_kernel(const IdxT* __restrict__ len,
                                                       IdxT* __restrict__ off, int64_t B,
                                                       int32_t* status) {
  if (*status != 0) return;
  __shared__ long long warp_incl[32];
  __shared__ long long carry;
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nwarps = blockDim.x >> 5;
  if (tid == 0) {
    carry = 0;
    bad = 0;
    off[0] = (IdxT)0;
  }
  __syncthreads();
  for (int64_t base = 0; base < B; base += blockDim.x) {
    const int64_t i = base + tid;
    long long x = 0;
    if (i < B) {
      x = (long long)len[i];
      if (x < 0) bad = 1;
    }
    long long v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) warp_incl[wid] = v;
    __syncthreads();
    if (wid == 0) {
      long long w = lane < nwarps ? warp_incl[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += n;
      }
      if (lane < nwarps) warp_incl[lane] = w;
    }
    __syncthreads();
    const long long incl = v + (wid > 0 ? warp_incl[wid - 1] : 0) + carry;
    if (i < B) {
      off[i + 1] = (IdxT)incl;
      if (sizeof(IdxT) == 4 && incl > (long long)INT_MAX) bad = 1;
    }
    __syncthreads();
    if (tid == (int)blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (tid == 0 && bad) set_status(status, JCA_STATUS_BAD_LENGTH);
}

// Offsets of user b must satisfy 0 <= off[b] <= off[b+1] <= rows, off[0] = 0, off[B] = rows.
__device__ __forceinline__ bool row_ok(long long s, long long e, int64_t b, int64_t B,
                                       int64_t rows) {
  return s >= 0 && s <= e && e <= rows && (b > 0 || s == 0) && (b < B - 1 || e == rows);
}

// ---------------------------------------------------------------------------------------------
// Segment IDs (候选隔离注意力掩码, section 段 ID：掩码的表达方式): one block per user row.
// ---------------------------------------------------------------------------------------------
template <typename IdxT>
__global__ void segment_ids_kernel(const IdxT* __restrict__ off, const IdxT* __restrict__ cs,
                                   const uint8_t* __restrict__ valid, int attend_padded_history,
                                   int64_t B, int64_t T, int8_t* __restrict__ seg,
                                   int32_t* status) {
  if (*status != 0) return;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    if (!row_ok(s, e, b, B, T)) {
      if (threadIdx.x == 0) set_status(status, JCA_STATUS_BAD_OFFSETS);
      continue;
    }
    const long long c = (long long)cs[b];
    if (c < 0 || c > e - s) {
      if (threadIdx.x == 0) set_status(status, JCA_STATUS_BAD_CAND_START);
      continue;
    }
    for (long long i = threadIdx.x; i < e - s; i += blockDim.x) {
      const bool is_candidate = i >= c;
      bool ok = valid ? (valid[s + i] != 0) : true;
      if (attend_padded_history) ok = ok || !is_candidate;
      seg[s + i] = ok ? (is_candidate ? (int8_t)-1 : (int8_t)1) : (int8_t)0;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Bounds (候选隔离注意力掩码, section 段 ID：掩码的表达方式, bounds_from_segment_ids): one block per
// user row reduces first/last positions of segment 1 and -1 and counts the segment-1 tokens, with
// warp reductions and one shared-memory combine. With FUSED, the block also builds the row's
// segment IDs from its candidate start (all tokens valid) and writes them, so that the plan makes
// one pass over the rows instead of two.
// ---------------------------------------------------------------------------------------------
template <typename IdxT, bool FUSED>
__global__ void __launch_bounds__(256) bounds_kernel(
    int8_t* __restrict__ seg, const IdxT* __restrict__ off, const IdxT* __restrict__ cs, int64_t B,
    int64_t T, IdxT* __restrict__ hist_lo, IdxT* __restrict__ hist_hi, IdxT* __restrict__ cand_lo,
    IdxT* __restrict__ cand_hi, int32_t* __restrict__ kv_count, int history_only,
    int32_t* status) {
  if (*status != 0) return;
  __shared__ int s_red[8][6];   // per warp: hmin, hmax, cmin, cmax, count, bad
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    if (!row_ok(s, e, b, B, T)) {
      if (threadIdx.x == 0) set_status(status, JCA_STATUS_BAD_OFFSETS);
      continue;
    }
    const int L = (int)(e - s);   // rows < 2^31 (checked on the host)
    int c = L;
    if (FUSED) {
      const long long cb = (long long)cs[b];
      if (cb < 0 || cb > L) {
        if (threadIdx.x == 0) set_status(status, JCA_STATUS_BAD_CAND_START);
        continue;
      }
      c = (int)cb;
    }
    int hmin = INT_MAX, hmax = -1, cmin = INT_MAX, cmax = -1, count = 0, bad = 0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      int x;
      if (FUSED) {
        x = i >= c ? -1 : 1;
        seg[s + i] = (int8_t)x;
      } else {
        x = seg[s + i];
      }
      if (x == 1) {
        hmin = min(hmin, i);
        hmax = max(hmax, i);
        ++count;
      } else if (x == -1) {
        bad |= history_only;
        cmin = min(cmin, i);
        cmax = max(cmax, i);
      } else if (x != 0) {
        bad = 1;
      }
    }
    hmin = __reduce_min_sync(0xffffffffu, hmin);
    hmax = __reduce_max_sync(0xffffffffu, hmax);
    cmin = __reduce_min_sync(0xffffffffu, cmin);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    count = __reduce_add_sync(0xffffffffu, count);
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) {
      s_red[wid][0] = hmin;
      s_red[wid][1] = hmax;
      s_red[wid][2] = cmin;
      s_red[wid][3] = cmax;
      s_red[wid][4] = count;
      s_red[wid][5] = bad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < nw; ++w) {
        hmin = min(hmin, s_red[w][0]);
        hmax = max(hmax, s_red[w][1]);
        cmin = min(cmin, s_red[w][2]);
        cmax = max(cmax, s_red[w][3]);
        count += s_red[w][4];
        bad |= s_red[w][5];
      }
      if (bad) {
        set_status(status, JCA_STATUS_BAD_SEG_VALUE);
      } else if (hmax >= 0 && cmax >= 0 && hmax > cmin) {
        set_status(status, JCA_STATUS_BAD_SEG_LAYOUT);
      }
      const bool has_h = hmax >= 0, has_c = cmax >= 0;
      hist_lo[b] = (IdxT)(has_h ? s + hmin : s);
      hist_hi[b] = (IdxT)(has_h ? s + hmax + 1 : s);
      if (cand_lo) cand_lo[b] = (IdxT)(has_c ? s + cmin : e);
      if (cand_hi) cand_hi[b] = (IdxT)(has_c ? s + cmax + 1 : e);
      if (kv_count) kv_count[b] = count;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Work queue: counting sort of (user, head, 256-row query pair) items by key-tile count,
// descending.
// A single block: pass 1 validates and histograms, a block scan turns bucket sizes into start
// positions (largest cost first), pass 2 emits each user's items contiguously (head-major, then
// query tile) at a position claimed with an atomic on its bucket cursor.
// ---------------------------------------------------------------------------------------------
template <typename IdxT>
__global__ void __launch_bounds__(1024) work_queue_kernel(
    const IdxT* __restrict__ qoff, const IdxT* __restrict__ kvlo, const IdxT* __restrict__ kvhi,
    const int32_t* __restrict__ kv_count, int64_t B, int64_t q_rows, int64_t kv_rows, int H,
    int4* __restrict__ items, int64_t max_items, int32_t* n_items, int32_t* status,
    int32_t* queue_ctl) {
  __shared__ unsigned long long s_cnt[kQueueBuckets];
  __shared__ unsigned long long s_cursor[kQueueBuckets];
  __shared__ unsigned long long s_warp[32];
  __shared__ unsigned long long s_total;
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (queue_ctl != nullptr && tid == 0) {
    queue_ctl[0] = 0;
    queue_ctl[1] = 0;
  }
  if (*status != 0) {
    if (tid == 0) *n_items = 0;
    return;
  }
  for (int i = tid; i < kQueueBuckets; i += blockDim.x) s_cnt[i] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int64_t b = tid; b < B; b += blockDim.x) {
    const long long s = (long long)qoff[b], e = (long long)qoff[b + 1];
    const long long lo = (long long)kvlo[b], hi = (long long)kvhi[b];
    if (!row_ok(s, e, b, B, q_rows) || lo < 0 || lo > hi || hi > kv_rows) {
      s_bad = 1;
      continue;
    }
    const long long nq = (e - s + kItemRows - 1) / kItemRows;
    const long long nkv = (hi - lo + kTileN - 1) / kTileN;
    const int key = (int)min(nkv, (long long)(kQueueBuckets - 1));
    if (nq) atomicAdd(&s_cnt[key], (unsigned long long)(nq * H));
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      set_status(status, JCA_STATUS_BAD_OFFSETS);
      *n_items = 0;
    }
    return;
  }
  // Exclusive scan over buckets in descending key order (thread t <-> bucket NB-1-t).
  static_assert(kQueueBuckets == 1024, "scan assumes one bucket per thread");
  const int kb = kQueueBuckets - 1 - tid;
  const unsigned long long val = s_cnt[kb];
  unsigned long long v = val;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[wid] = v;
  __syncthreads();
  if (wid == 0) {
    unsigned long long w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const unsigned long long incl = v + (wid > 0 ? s_warp[wid - 1] : 0ull);
  s_cursor[kb] = incl - val;
  if (tid == kQueueBuckets - 1) s_total = incl;
  __syncthreads();
  if (s_total > (unsigned long long)max_items) {
    if (tid == 0) {
      set_status(status, JCA_STATUS_QUEUE_OVERFLOW);
      *n_items = 0;
    }
    return;
  }
  // Pass 2, per chunk of 1024 users: one thread per user claims the user's run of nq * H slots
  // (all users at once, so that no user's loads wait behind another's), then one thread per
  // (user, head) writes that head's nq items, so that no thread writes more than one head's run.
  __shared__ unsigned long long s_pos[1024];
  __shared__ int s_nq[1024];
  for (int64_t b0 = 0; b0 < B; b0 += blockDim.x) {
    const int64_t b = b0 + tid;
    int nq_b = 0;
    if (b < B) {
      const long long s = (long long)qoff[b], e = (long long)qoff[b + 1];
      const long long lo = (long long)kvlo[b], hi = (long long)kvhi[b];
      nq_b = (int)((e - s + kItemRows - 1) / kItemRows);
      if (nq_b > 0) {
        const long long nkv = (hi - lo + kTileN - 1) / kTileN;
        const int key = (int)min(nkv, (long long)(kQueueBuckets - 1));
        s_pos[tid] = atomicAdd(&s_cursor[key], (unsigned long long)nq_b * (unsigned long long)H);
      }
    }
    s_nq[tid] = nq_b;
    __syncthreads();
    const int nb = (int)min((int64_t)blockDim.x, B - b0);
    for (int p = tid; p < nb * H; p += blockDim.x) {
      const int ub = p / H, h = p - ub * H;
      const int nq = s_nq[ub];
      if (nq == 0) continue;
      const int64_t bb = b0 + ub;
      const long long s = (long long)qoff[bb], e = (long long)qoff[bb + 1];
      const long long lo = (long long)kvlo[bb], hi = (long long)kvhi[bb];
      const int holes = (kv_count != nullptr && (long long)kv_count[bb] != hi - lo) ? 1 : 0;
      const int w = (int)(hi - lo) | (holes << 31);
      const unsigned long long pos = s_pos[ub] + (unsigned long long)h * (unsigned long long)nq;
      for (int t = 0; t < nq; ++t) {
        const long long row0 = s + (long long)t * kItemRows;
        const int rows = (int)min((long long)kItemRows, e - row0);
        items[pos + (unsigned long long)t] = make_int4((int)row0, (h << 9) | rows, (int)lo, w);
      }
    }
    __syncthreads();
  }
  if (tid == 0) *n_items = (int32_t)s_total;
}

// ---------------------------------------------------------------------------------------------
// Work queue of the per-user causal variant: one item per (user, head, 256-row query block); the
// keys of a block are the user's rows up to the block's last row, so the cost (128-key tiles)
// grows with the block's position. Same counting sort as above, keyed per item.
// ---------------------------------------------------------------------------------------------
template <typename IdxT>
__global__ void __launch_bounds__(1024) causal_queue_kernel(
    const IdxT* __restrict__ off, int64_t B, int64_t rows, int H, int4* __restrict__ items,
    int64_t max_items, int32_t* n_items, int32_t* status, int32_t* queue_ctl) {
  __shared__ unsigned long long s_cnt[kQueueBuckets];
  __shared__ unsigned long long s_cursor[kQueueBuckets];
  __shared__ unsigned long long s_warp[32];
  __shared__ unsigned long long s_total;
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) {
    queue_ctl[0] = 0;
    queue_ctl[1] = 0;
  }
  if (*status != 0) {
    if (tid == 0) *n_items = 0;
    return;
  }
  for (int i = tid; i < kQueueBuckets; i += blockDim.x) s_cnt[i] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  auto key_of = [](long long kv_len) {
    return (int)min((kv_len + kTileN - 1) / kTileN, (long long)(kQueueBuckets - 1));
  };
  for (int64_t b = tid; b < B; b += blockDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    if (!row_ok(s, e, b, B, rows)) {
      s_bad = 1;
      continue;
    }
    for (long long r0 = s; r0 < e; r0 += kItemRows)
      atomicAdd(&s_cnt[key_of(min(r0 + kItemRows, e) - s)], (unsigned long long)H);
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      set_status(status, JCA_STATUS_BAD_OFFSETS);
      *n_items = 0;
    }
    return;
  }
  static_assert(kQueueBuckets == 1024, "scan assumes one bucket per thread");
  const int kb = kQueueBuckets - 1 - tid;
  const unsigned long long val = s_cnt[kb];
  unsigned long long v = val;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[wid] = v;
  __syncthreads();
  if (wid == 0) {
    unsigned long long w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const unsigned long long incl = v + (wid > 0 ? s_warp[wid - 1] : 0ull);
  s_cursor[kb] = incl - val;
  if (tid == kQueueBuckets - 1) s_total = incl;
  __syncthreads();
  if (s_total > (unsigned long long)max_items) {
    if (tid == 0) {
      set_status(status, JCA_STATUS_QUEUE_OVERFLOW);
      *n_items = 0;
    }
    return;
  }
  // One warp per user: per query block, lane 0 claims H slots, the lanes write them (one per head).
  const int nwarps = blockDim.x >> 5;
  for (int64_t b = wid; b < B; b += nwarps) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    for (long long r0 = s; r0 < e; r0 += kItemRows) {
      const long long kv_len = min(r0 + kItemRows, e) - s;
      unsigned long long pos = 0;
      if (lane == 0) pos = atomicAdd(&s_cursor[key_of(kv_len)], (unsigned long long)H);
      pos = __shfl_sync(0xffffffffu, pos, 0);
      const int nrows = (int)(min(r0 + kItemRows, e) - r0);
      for (int h = lane; h < H; h += 32)
        items[pos + (unsigned long long)h] =
            make_int4((int)r0, (h << 9) | nrows, (int)s, (int)kv_len);
    }
  }
  if (tid == 0) *n_items = (int32_t)s_total;
}

inline int grid_for_rows(int64_t B) { return (int)(B < (1 << 20) ? B : (1 << 20)); }

// ---------------------------------------------------------------------------------------------
// Training with candidate packing (候选隔离注意力掩码, section 训练时的序列打包): the packed matrix
// holds every user's prefix + history run in rows [0, Th) (split at hist_off) and every user's
// candidate run in rows [Th, Th + Nc) (split at cand_off, relative to Th). The attention kernels
// take it as 2B "query runs" over B key intervals: run b < B is user b's history run, run B + b
// its candidate run, and both read user b's history keys.
// ---------------------------------------------------------------------------------------------

// Segment IDs of the packed matrix when the caller gives none (history rows 1, candidate rows -1),
// or a check of the caller's candidate rows (only -1 or 0 there; the history rows are checked by
// the bounds pass, which admits only 1 and 0).
__global__ void __launch_bounds__(256) seqpack_seg_kernel(int8_t* __restrict__ seg_out,
                                                          const int8_t* __restrict__ seg_in,
                                                          int64_t Th, int64_t T,
                                                          int32_t* status) {
  if (*status != 0) return;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (seg_out) {
      seg_out[i] = i < Th ? (int8_t)1 : (int8_t)-1;
    } else if (i >= Th) {
      const int x = seg_in[i];
      if (x != -1 && x != 0) set_status(status, JCA_STATUS_BAD_SEG_VALUE);
    }
  }
}

// Checks the candidate offsets and writes the 2B query runs: q_off2[0..B] = hist_off,
// q_off2[B + b] = Th + cand_off[b]; the key interval and key count of run B + b are user b's,
// copied from entry b (written by the bounds pass over the history block).
template <typename IdxT>
__global__ void __launch_bounds__(256) seqpack_runs_kernel(
    const IdxT* __restrict__ hist_off, const IdxT* __restrict__ cand_off, int64_t B, int64_t Th,
    int64_t Nc, IdxT* __restrict__ q_off2, IdxT* __restrict__ kv_lo, IdxT* __restrict__ kv_hi,
    int32_t* __restrict__ kv_count, int32_t* status) {
  if (*status != 0) return;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b <= B;
       b += (int64_t)gridDim.x * blockDim.x) {
    const long long c = (long long)cand_off[b];
    const bool bad = (b == 0 && c != 0) || (b == B && c != Nc) ||
                     (b < B && (long long)cand_off[b + 1] < c) || c < 0 || c > Nc;
    if (bad) set_status(status, JCA_STATUS_BAD_OFFSETS);
    q_off2[b] = hist_off[b];
    if (b > 0) q_off2[B + b] = (IdxT)(Th + c);
    if (b < B) {
      kv_lo[B + b] = kv_lo[b];
      kv_hi[B + b] = kv_hi[b];
      kv_count[B + b] = kv_count[b];
    }
  }
}

}  // namespace

int64_t max_work_items(int64_t B, int64_t rows, int H) {
  return ((rows + kItemRows - 1) / kItemRows + B) * (int64_t)H;
}

WorkspaceLayout workspace_layout(int64_t B, int64_t rows, int H) {
  WorkspaceLayout w;
  size_t p = 0;
  w.seg = p;
  p = align_up(p + (size_t)rows, 256);
  w.hist_lo = p;
  p = align_up(p + 8 * (size_t)B, 256);
  w.hist_hi = p;
  p = align_up(p + 8 * (size_t)B, 256);
  w.cand_lo = p;
  p = align_up(p + 8 * (size_t)B, 256);
  w.cand_hi = p;
  p = align_up(p + 8 * (size_t)B, 256);
  w.kv_count = p;
  p = align_up(p + 4 * (size_t)B, 256);
  w.max_items = max_work_items(B, rows, H);
  w.items = p;
  p = align_up(p + 16 * (size_t)w.max_items, 256);
  w.n_items = p;
  w.queue = p + 16;
  p = align_up(p + 32, 256);
  w.total = p;
  return w;
}

cudaError_t launch_segment_ids(const void* offsets, const void* cand_start, const uint8_t* valid,
                               int attend_padded_history, int64_t B, int64_t T, int idx_bits,
                               int8_t* seg, int32_t* status, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const int grid = grid_for_rows(B);
  if (idx_bits == 32)
    segment_ids_kernel<int32_t><<<grid, 256, 0, stream>>>(
        (const int32_t*)offsets, (const int32_t*)cand_start, valid, attend_padded_history, B, T,
        seg, status);
  else
    segment_ids_kernel<int64_t><<<grid, 256, 0, stream>>>(
        (const int64_t*)offsets, (const int64_t*)cand_start, valid, attend_padded_history, B, T,
        seg, status);
  return cudaGetLastError();
}

cudaError_t launch_bounds(const int8_t* seg, const void* offsets, int64_t B, int64_t T,
                          int idx_bits, void* hist_lo, void* hist_hi, void* cand_lo,
                          void* cand_hi, int32_t* kv_count, int history_only, int32_t* status,
                          cudaStream_t stream, const void* cand_start, int8_t* seg_out) {
  if (B == 0) return cudaSuccess;
  const int grid = grid_for_rows(B);
  if (idx_bits == 32) {
    if (cand_start)
      bounds_kernel<int32_t, true><<<grid, 256, 0, stream>>>(
          seg_out, (const int32_t*)offsets, (const int32_t*)cand_start, B, T, (int32_t*)hist_lo,
          (int32_t*)hist_hi, (int32_t*)cand_lo, (int32_t*)cand_hi, kv_count, history_only, status);
    else
      bounds_kernel<int32_t, false><<<grid, 256, 0, stream>>>(
          const_cast<int8_t*>(seg), (const int32_t*)offsets, nullptr, B, T, (int32_t*)hist_lo,
          (int32_t*)hist_hi, (int32_t*)cand_lo, (int32_t*)cand_hi, kv_count, history_only, status);
  } else {
    if (cand_start)
      bounds_kernel<int64_t, true><<<grid, 256, 0, stream>>>(
          seg_out, (const int64_t*)offsets, (const int64_t*)cand_start, B, T, (int64_t*)hist_lo,
          (int64_t*)hist_hi, (int64_t*)cand_lo, (int64_t*)cand_hi, kv_count, history_only, status);
    else
      bounds_kernel<int64_t, false><<<grid, 256, 0, stream>>>(
          const_cast<int8_t*>(seg), (const int64_t*)offsets, nullptr, B, T, (int64_t*)hist_lo,
          (int64_t*)hist_hi, (int64_t*)cand_lo, (int64_t*)cand_hi, kv_count, history_only, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_causal_queue(const void* offsets, int64_t B, int64_t rows, int H,
                                int idx_bits, int32_t* items, int64_t max_items, int32_t* n_items,
                                int32_t* status, cudaStream_t stream, int32_t* queue_ctl) {
  if (idx_bits == 32)
    causal_queue_kernel<int32_t><<<1, kQueueBuckets, 0, stream>>>(
        (const int32_t*)offsets, B, rows, H, (int4*)items, max_items, n_items, status, queue_ctl);
  else
    causal_queue_kernel<int64_t><<<1, kQueueBuckets, 0, stream>>>(
        (const int64_t*)offsets, B, rows, H, (int4*)items, max_items, n_items, status, queue_ctl);
  return cudaGetLastError();
}

cudaError_t launch_work_queue(const void* q_offsets, const void* kv_lo, const void* kv_hi,
                              const int32_t* kv_count, int64_t B, int64_t q_rows,
                              int64_t kv_rows, int H, int idx_bits, int32_t* items,
                              int64_t max_items, int32_t* n_items, int32_t* status,
                              cudaStream_t stream, int32_t* queue_ctl) {
  if (idx_bits == 32)
    work_queue_kernel<int32_t><<<1, kQueueBuckets, 0, stream>>>(
        (const int32_t*)q_offsets, (const int32_t*)kv_lo, (const int32_t*)kv_hi, kv_count, B,
        q_rows, kv_rows, H, (int4*)items, max_items, n_items, status, queue_ctl);
  else
    work_queue_kernel<int64_t><<<1, kQueueBuckets, 0, stream>>>(
        (const int64_t*)q_offsets, (const int64_t*)kv_lo, (const int64_t*)kv_hi, kv_count, B,
        q_rows, kv_rows, H, (int4*)items, max_items, n_items, status, queue_ctl);
  return cudaGetLastError();
}

cudaError_t launch_seqpack_plan(const void* hist_off, const void* cand_off, const int8_t* seg,
                                int64_t B, int64_t Th, int64_t Nc, int H, int idx_bits, char* ws,
                                const WorkspaceLayout& L, size_t q_off2, int32_t* status,
                                cudaStream_t stream) {
  const int64_t T = Th + Nc;
  int8_t* seg_ws = reinterpret_cast<int8_t*>(ws + L.seg);
  const int8_t* segp = seg ? seg : seg_ws;
  if (T > 0) {
    const int64_t blocks = (T + 255) / 256;
    seqpack_seg_kernel<<<(int)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, stream>>>(
        seg ? nullptr : seg_ws, seg, Th, T, status);
    if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
  }
  cudaError_t e = launch_bounds(segp, hist_off, B, Th, idx_bits, ws + L.hist_lo, ws + L.hist_hi,
                                nullptr, nullptr, reinterpret_cast<int32_t*>(ws + L.kv_count), 1,
                                status, stream);
  if (e != cudaSuccess) return e;
  const int grid = (int)((B + 1 + 255) / 256);
  if (idx_bits == 32)
    seqpack_runs_kernel<int32_t><<<grid, 256, 0, stream>>>(
        (const int32_t*)hist_off, (const int32_t*)cand_off, B, Th, Nc, (int32_t*)(ws + q_off2),
        (int32_t*)(ws + L.hist_lo), (int32_t*)(ws + L.hist_hi),
        reinterpret_cast<int32_t*>(ws + L.kv_count), status);
  else
    seqpack_runs_kernel<int64_t><<<grid, 256, 0, stream>>>(
        (const int64_t*)hist_off, (const int64_t*)cand_off, B, Th, Nc, (int64_t*)(ws + q_off2),
        (int64_t*)(ws + L.hist_lo), (int64_t*)(ws + L.hist_hi),
        reinterpret_cast<int32_t*>(ws + L.kv_count), status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_work_queue(ws + q_off2, ws + L.hist_lo, ws + L.hist_hi,
                           reinterpret_cast<int32_t*>(ws + L.kv_count), 2 * B, T, T, H, idx_bits,
                           reinterpret_cast<int32_t*>(ws + L.items), L.max_items,
                           reinterpret_cast<int32_t*>(ws + L.n_items), status, stream,
                           reinterpret_cast<int32_t*>(ws + L.queue));
}

}  // namespace jca

using namespace jca;

extern "C" int jca_offsets_from_lengths(const void* lengths, void* offsets, int64_t B,
                                        int idx_bits, int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (B < 0 || B >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  if (!offsets || !status || (B > 0 && !lengths)) return JCA_ERR_NULL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (idx_bits == 32)
    offsets_kernel<int32_t><<<1, 1024, 0, s>>>((const int32_t*)lengths, (int32_t*)offsets, B,
                                                status);
  else
    offsets_kernel<int64_t><<<1, 1024, 0, s>>>((const int64_t*)lengths, (int64_t*)offsets, B,
                                                status);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

extern "C" int jca_build_segment_ids(const void* offsets, const void* candidate_start,
                                     const uint8_t* valid_mask, int attend_padded_history,
                                     int64_t B, int64_t T, int idx_bits, int8_t* seg,
                                     int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (B < 0 || T < 0 || T >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  if (B == 0 && T != 0) return JCA_ERR_SHAPE;
  if (!status || !offsets || (B > 0 && !candidate_start) || (T > 0 && !seg)) return JCA_ERR_NULL;
  cudaError_t e = launch_segment_ids(offsets, candidate_start, valid_mask, attend_padded_history,
                                     B, T, idx_bits, seg, status,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

extern "C" int jca_bounds_from_segment_ids(const int8_t* seg, const void* offsets, int64_t B,
                                           int64_t T, int idx_bits, void* hist_lo, void* hist_hi,
                                           void* cand_lo, void* cand_hi, int32_t* status,
                                           jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (B < 0 || T < 0 || T >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  if (B == 0 && T != 0) return JCA_ERR_SHAPE;
  if (!status || !offsets || (T > 0 && !seg)) return JCA_ERR_NULL;
  if (B > 0 && (!hist_lo || !hist_hi || !cand_lo || !cand_hi)) return JCA_ERR_NULL;
  cudaError_t e = launch_bounds(seg, offsets, B, T, idx_bits, hist_lo, hist_hi, cand_lo, cand_hi,
                                nullptr, 0, status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

extern "C" int jca_build_work_queue(const void* q_offsets, const void* kv_lo, const void* kv_hi,
                                    const int32_t* kv_count, int64_t B, int64_t q_rows,
                                    int64_t kv_rows, int H, int idx_bits, int32_t* items,
                                    int64_t max_items, int32_t* n_items, int32_t* status,
                                    jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (B < 0 || q_rows < 0 || kv_rows < 0 || H < 1 || H >= 65536 || max_items < 0 ||
      max_items >= (int64_t)INT_MAX || q_rows >= (int64_t)INT_MAX ||
      kv_rows >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX)
    return JCA_ERR_SHAPE;
  if (B == 0 && q_rows != 0) return JCA_ERR_SHAPE;
  if (!q_offsets || !n_items || !status || (B > 0 && (!kv_lo || !kv_hi)) ||
      (max_items > 0 && !items))
    return JCA_ERR_NULL;
  if (items && !aligned(items, 16)) return JCA_ERR_ALIGN;
  cudaError_t e = launch_work_queue(q_offsets, kv_lo, kv_hi, kv_count, B, q_rows, kv_rows, H,
                                    idx_bits, items, max_items, n_items, status,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

extern "C" int64_t jca_max_work_items(int64_t B, int64_t rows, int H) {
  if (B < 0 || rows < 0 || H < 1) return 0;
  return max_work_items(B, rows, H);
}
