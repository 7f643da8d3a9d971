// Layer stack of a ranker over one jagged batch, with candidate-only tail layers
// (候选隔离注意力掩码, section 只更新候选的末尾层): the first n_layers - n_cand_only layers run over whole
// rows [prefix | history | candidates] under the isolation mask; the states are then split into the
// frozen history (segment 1) and the candidates (segment -1), and each tail layer updates only the
// candidates, whose queries attend to the frozen history's keys/values and to their own.
//
// A layer is x <- x + Attn(x Wq, x Wk, x Wv) Wo (square weights, no bias), with right-anchored RoPE
// on the queries and keys when a history_end is given (section 位置编码：候选共用一个位置). The
// projections are plain dense GEMMs and run on cuBLASLt (bf16 in, fp32 accumulation, bf16 out;
// the residual enters as the GEMM's C operand, so x + a Wo is rounded once). Everything else runs
// in this library's kernels: the split into history and candidates (count, scan, compaction,
// row gather), RoPE, the two attention kernels, and the final scatter of the candidate rows.
#include <climits>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>

#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "jca_internal.h"

namespace jca {
namespace {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ void set_status(int32_t* status, int code) {
  atomicCAS(status, 0, (int32_t)code);
}

// ---------------------------------------------------------------------------------------------
// Split of the packed rows into history (segment 1) and candidates (segment -1).
// ---------------------------------------------------------------------------------------------

// cnt[b] = segment-1 tokens of user b, cnt[B + b] = its segment -1 tokens. One block per user.
// Offsets and segment IDs were validated by the attention plan that ran before on the stream.
template <typename IdxT>
__global__ void __launch_bounds__(256) split_count_kernel(const int8_t* __restrict__ seg,
                                                          const IdxT* __restrict__ off, int64_t B,
                                                          int32_t* __restrict__ cnt,
                                                          const int32_t* status) {
  if (*status != 0) return;
  __shared__ int s_h[8], s_c[8];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    int h = 0, c = 0;
    for (long long i = s + threadIdx.x; i < e; i += blockDim.x) {
      const int g = seg[i];
      h += g == 1;
      c += g == -1;
    }
    h = __reduce_add_sync(0xffffffffu, h);
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
      s_h[wid] = h;
      s_c[wid] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int th = 0, tc = 0;
      for (int w = 0; w < 8; ++w) {
        th += s_h[w];
        tc += s_c[w];
      }
      cnt[b] = th;
      cnt[B + b] = tc;
    }
    __syncthreads();
  }
}

// hoff/coff = exclusive scans of the two count arrays (B + 1 entries each); the totals must equal
// the caller's Th and Nc, otherwise JCA_STATUS_BAD_SPLIT and nothing later runs. One block.
template <typename IdxT>
__global__ void __launch_bounds__(1024) split_scan_kernel(const int32_t* __restrict__ cnt,
                                                          int64_t B, int64_t Th, int64_t Nc,
                                                          IdxT* __restrict__ hoff,
                                                          IdxT* __restrict__ coff,
                                                          int32_t* status) {
  if (*status != 0) return;
  __shared__ long long w_h[32], w_c[32];
  __shared__ long long carry_h, carry_c;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) {
    carry_h = 0;
    carry_c = 0;
    hoff[0] = (IdxT)0;
    coff[0] = (IdxT)0;
  }
  __syncthreads();
  for (int64_t base = 0; base < B; base += blockDim.x) {
    const int64_t i = base + tid;
    long long h = i < B ? cnt[i] : 0, c = i < B ? cnt[B + i] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long nh = __shfl_up_sync(0xffffffffu, h, o);
      const long long nc = __shfl_up_sync(0xffffffffu, c, o);
      if (lane >= o) {
        h += nh;
        c += nc;
      }
    }
    if (lane == 31) {
      w_h[wid] = h;
      w_c[wid] = c;
    }
    __syncthreads();
    if (wid == 0) {
      long long a = lane < nw ? w_h[lane] : 0, b2 = lane < nw ? w_c[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long na = __shfl_up_sync(0xffffffffu, a, o);
        const long long nb = __shfl_up_sync(0xffffffffu, b2, o);
        if (lane >= o) {
          a += na;
          b2 += nb;
        }
      }
      if (lane < nw) {
        w_h[lane] = a;
        w_c[lane] = b2;
      }
    }
    __syncthreads();
    const long long ih = h + (wid > 0 ? w_h[wid - 1] : 0) + carry_h;
    const long long ic = c + (wid > 0 ? w_c[wid - 1] : 0) + carry_c;
    if (i < B) {
      hoff[i + 1] = (IdxT)ih;
      coff[i + 1] = (IdxT)ic;
    }
    __syncthreads();
    if (tid == (int)blockDim.x - 1) {
      carry_h = ih;
      carry_c = ic;
    }
    __syncthreads();
  }
  if (tid == 0 && (carry_h != Th || carry_c != Nc)) set_status(status, JCA_STATUS_BAD_SPLIT);
}

// sidx[hoff[b] + k] = packed row of the k-th segment-1 token of user b, and
// sidx[Th + coff[b] + k] = that of its k-th candidate. One block (256 threads) per user; rows are
// taken in chunks of 256 with ballot-based exclusive scans, so the order within a user is kept.
template <typename IdxT>
__global__ void __launch_bounds__(256) split_index_kernel(const int8_t* __restrict__ seg,
                                                          const IdxT* __restrict__ off,
                                                          const IdxT* __restrict__ hoff,
                                                          const IdxT* __restrict__ coff,
                                                          int64_t B, int64_t Th,
                                                          int32_t* __restrict__ sidx,
                                                          const int32_t* status) {
  if (*status != 0) return;
  __shared__ int s_h[8], s_c[8];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    long long dh = (long long)hoff[b], dc = Th + (long long)coff[b];
    for (long long base = s; base < e; base += blockDim.x) {
      const long long i = base + threadIdx.x;
      const int g = i < e ? seg[i] : 0;
      const unsigned bh = __ballot_sync(0xffffffffu, g == 1);
      const unsigned bc = __ballot_sync(0xffffffffu, g == -1);
      if (lane == 0) {
        s_h[wid] = __popc(bh);
        s_c[wid] = __popc(bc);
      }
      __syncthreads();
      int ph = 0, pc = 0, th = 0, tc = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const int a = s_h[w], c = s_c[w];
        if (w < wid) {
          ph += a;
          pc += c;
        }
        th += a;
        tc += c;
      }
      if (g == 1) sidx[dh + ph + __popc(bh & lt)] = (int32_t)i;
      if (g == -1) sidx[dc + pc + __popc(bc & lt)] = (int32_t)i;
      dh += th;
      dc += tc;
      __syncthreads();
    }
  }
}

// Row copies between the packed states and the split buffer: gather (to_split != 0) copies
// x[sidx[r]] to xs[r] for r in [0, n) (and pos[sidx[r]] to spos[r] when pos is given); scatter
// copies xs[r0 + r] to x[sidx[r0 + r]]. One warp per row, 16-byte accesses (D is a multiple of 16).
__global__ void __launch_bounds__(256) split_rows_kernel(bf16* __restrict__ x,
                                                         bf16* __restrict__ xs, int64_t D,
                                                         const int32_t* __restrict__ sidx,
                                                         int64_t r0, int64_t n, int to_split,
                                                         const int32_t* __restrict__ pos,
                                                         int32_t* __restrict__ spos,
                                                         const int32_t* status) {
  if (*status != 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t chunks = D / 8;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n;
       r += warps) {
    const int64_t row = sidx[r0 + r];
    uint4* packed = reinterpret_cast<uint4*>(x + row * D);
    uint4* split = reinterpret_cast<uint4*>(xs + (r0 + r) * D);
    if (to_split) {
      for (int64_t c = lane; c < chunks; c += 32) split[c] = packed[c];
      if (pos && lane == 0) spos[r0 + r] = pos[row];
    } else {
      for (int64_t c = lane; c < chunks; c += 32) packed[c] = split[c];
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Projections on cuBLASLt: Y[M, N] = X[M, K] W[K, N] (+ R[M, N]), all row-major bf16, fp32
// accumulation, one rounding to bf16. In cuBLASLt's column-major terms this is
// Y^T (N x M) = W^T (N x K) * X^T (K x M) with no transposes.
// ---------------------------------------------------------------------------------------------
constexpr size_t kLtWorkspace = size_t(32) << 20;
constexpr int kMaxDevices = 64;

struct LtDevice {
  cublasLtHandle_t handle = nullptr;
  std::map<std::tuple<int64_t, int, int, int>, cublasLtMatmulAlgo_t> algos;
};
LtDevice g_lt[kMaxDevices];
std::mutex g_lt_mu;

struct LtDescs {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t a = nullptr, b = nullptr, c = nullptr;
  ~LtDescs() {
    if (a) cublasLtMatrixLayoutDestroy(a);
    if (b) cublasLtMatrixLayoutDestroy(b);
    if (c) cublasLtMatrixLayoutDestroy(c);
    if (op) cublasLtMatmulDescDestroy(op);
  }
};

int gemm_bf16(const bf16* X, const bf16* W, const bf16* R, bf16* Y, int64_t M, int N, int K,
              void* lt_ws, cudaStream_t stream) {
  if (M == 0) return JCA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return JCA_ERR_CUDA;
  LtDescs d;
  const cublasOperation_t opn = CUBLAS_OP_N;
  if (cublasLtMatmulDescCreate(&d.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(d.op, CUBLASLT_MATMUL_DESC_TRANSA, &opn, sizeof(opn)) !=
          CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(d.op, CUBLASLT_MATMUL_DESC_TRANSB, &opn, sizeof(opn)) !=
          CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&d.a, CUDA_R_16BF, N, K, N) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&d.b, CUDA_R_16BF, K, M, K) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&d.c, CUDA_R_16BF, N, M, N) != CUBLAS_STATUS_SUCCESS)
    return JCA_ERR_CUDA;
  cublasLtHandle_t handle;
  cublasLtMatmulAlgo_t algo;
  {
    std::lock_guard<std::mutex> lock(g_lt_mu);
    LtDevice& L = g_lt[dev];
    if (!L.handle && cublasLtCreate(&L.handle) != CUBLAS_STATUS_SUCCESS) {
      L.handle = nullptr;
      return JCA_ERR_CUDA;
    }
    handle = L.handle;
    const auto key = std::make_tuple(M, N, K, R ? 1 : 0);
    auto it = L.algos.find(key);
    if (it == L.algos.end()) {
      cublasLtMatmulPreference_t pref = nullptr;
      if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) return JCA_ERR_CUDA;
      const uint64_t wsb = kLtWorkspace;
      const uint32_t align = 16;   // every operand is only promised 16-byte alignment
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsb,
                                           sizeof(wsb));
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_A_BYTES,
                                           &align, sizeof(align));
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_B_BYTES,
                                           &align, sizeof(align));
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_C_BYTES,
                                           &align, sizeof(align));
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MIN_ALIGNMENT_D_BYTES,
                                           &align, sizeof(align));
      cublasLtMatmulHeuristicResult_t res;
      int found = 0;
      const cublasStatus_t hs = cublasLtMatmulAlgoGetHeuristic(handle, d.op, d.a, d.b, d.c, d.c,
                                                               pref, 1, &res, &found);
      cublasLtMatmulPreferenceDestroy(pref);
      if (hs != CUBLAS_STATUS_SUCCESS || found < 1) return JCA_ERR_CUDA;
      it = L.algos.emplace(key, res.algo).first;
    }
    algo = it->second;
  }
  const float alpha = 1.f, beta = R ? 1.f : 0.f;
  const cublasStatus_t st = cublasLtMatmul(handle, d.op, &alpha, W, d.a, X, d.b, &beta,
                                           R ? R : Y, d.c, Y, d.c, &algo, lt_ws, kLtWorkspace,
                                           stream);
  return st == CUBLAS_STATUS_SUCCESS ? JCA_OK : JCA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// Workspace of the stack (256-byte aligned sections).
// ---------------------------------------------------------------------------------------------
struct StackLayout {
  size_t attn = 0, cand = 0, pos = 0, spos = 0, cnt = 0, hoff = 0, coff = 0, sidx = 0;
  size_t qkv = 0, a = 0, xs = 0, lt = 0, total = 0;
};

StackLayout stack_layout(int64_t B, int64_t T, int64_t Nc, int64_t Th, int H, int d_head) {
  StackLayout L;
  const int64_t D = (int64_t)H * d_head;
  const int64_t S = Nc + Th;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.attn = take(jca_workspace_bytes(B, T, H, d_head));
  L.cand = take(jca_workspace_bytes(B, Nc, H, d_head));
  L.pos = take((size_t)T * 4);
  L.spos = take((size_t)S * 4);
  L.cnt = take((size_t)2 * B * 4);
  L.hoff = take((size_t)(B + 1) * 8);
  L.coff = take((size_t)(B + 1) * 8);
  L.sidx = take((size_t)S * 4);
  L.qkv = take((size_t)3 * T * D * 2);
  L.a = take((size_t)T * D * 2);
  L.xs = take((size_t)S * D * 2);
  L.lt = take(kLtWorkspace);
  L.total = o;
  return L;
}

int grid_for(int64_t want, int cap) { return (int)(want < cap ? (want > 0 ? want : 1) : cap); }

}  // namespace
}  // namespace jca

using namespace jca;

extern "C" size_t jca_stack_workspace_bytes(int64_t B, int64_t T, int64_t Nc, int64_t Th, int H,
                                            int d_head) {
  if (B < 0 || T < 0 || Nc < 0 || Th < 0 || Nc + Th > T || H < 1 || !head_dim_ok(d_head))
    return 0;
  return stack_layout(B, T, Nc, Th, H, d_head).total;
}

extern "C" int jca_stack_fwd(const void* x, void* x_out, const void* weights, int n_layers,
                             int n_cand_only, const void* offsets, const void* candidate_start,
                             const int8_t* seg, int64_t B, int64_t T, int64_t Nc, int64_t Th,
                             int H, int d_head, float scale, int64_t history_end,
                             float rope_base, int idx_bits, void* workspace,
                             size_t workspace_bytes, int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (n_layers < 0 || n_cand_only < 0 || n_cand_only > n_layers || B < 0 || T < 0 || Nc < 0 ||
      Th < 0 || Nc + Th > T || H < 1 || H >= 65536 || T >= (int64_t)INT_MAX ||
      (int64_t)H * d_head >= 65536 || (B == 0 && T != 0))
    return JCA_ERR_SHAPE;
  const bool rope = history_end >= 0;
  if (rope && !(rope_base > 1.f)) return JCA_ERR_SHAPE;
  if (!status || !offsets || !workspace) return JCA_ERR_NULL;
  if (T > 0 && (!x || !x_out || (n_layers > 0 && !weights))) return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(x, 16) || !aligned(x_out, 16) || !aligned(weights, 16)))
    return JCA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  const StackLayout L = stack_layout(B, T, Nc, Th, H, d_head);
  if (workspace_bytes < L.total) return JCA_ERR_WORKSPACE;
  if (T == 0) return JCA_OK;

  const int D = H * d_head;
  const int64_t DD = (int64_t)D * D;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  void* attn_ws = ws + L.attn;
  const size_t attn_bytes = L.cand - L.attn;
  void* cand_ws = ws + L.cand;
  const size_t cand_bytes = L.pos - L.cand;
  int32_t* pos = reinterpret_cast<int32_t*>(ws + L.pos);
  int32_t* spos = reinterpret_cast<int32_t*>(ws + L.spos);
  bf16* q = reinterpret_cast<bf16*>(ws + L.qkv);
  bf16* a = reinterpret_cast<bf16*>(ws + L.a);
  bf16* xs = reinterpret_cast<bf16*>(ws + L.xs);
  void* lt_ws = ws + L.lt;
  const bf16* Wt = static_cast<const bf16*>(weights);
  bf16* xo = static_cast<bf16*>(x_out);

  // Layout of the whole rows: segment IDs (unless given), bounds and the attention work queue.
  int rc = jagged_cand_attn_plan(offsets, candidate_start, seg, B, T, H, d_head, idx_bits,
                                 attn_ws, attn_bytes, status, stream);
  if (rc) return rc;
  const int8_t* segp =
      seg ? seg
          : reinterpret_cast<const int8_t*>(static_cast<char*>(attn_ws) +
                                            workspace_layout(B, T, H).seg);
  if (rope) {
    rc = jca_rope_positions(segp, offsets, B, T, history_end, idx_bits, pos, status, stream);
    if (rc) return rc;
  }

  // Full layers over whole rows.
  const int n_full = n_layers - n_cand_only;
  const bf16* cur = static_cast<const bf16*>(x);
  bf16* k = q + (int64_t)T * D;
  bf16* v = k + (int64_t)T * D;
  for (int l = 0; l < n_full; ++l) {
    const bf16* W = Wt + (int64_t)l * 4 * DD;
    // Q, K and V as three GEMMs: one batched GEMM over the three consecutive weights measured
    // slower (0.1 ms per layer on users256), cuBLASLt's heuristic picking a slower kernel for it.
    if ((rc = gemm_bf16(cur, W, nullptr, q, T, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(cur, W + DD, nullptr, k, T, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(cur, W + 2 * DD, nullptr, v, T, D, D, lt_ws, st)))
      return rc;
    // RoPE as a pre-pass over Q and K: each key row is rotated once here, whereas the kernel's
    // in-tile rotation (jagged_cand_attn_rope_fwd) rotates a key tile again for every query block
    // of its user and head, which measured slower on this workload.
    if (rope && ((rc = jca_apply_rope(q, q, pos, T, H, d_head, rope_base, stream)) ||
                 (rc = jca_apply_rope(k, k, pos, T, H, d_head, rope_base, stream))))
      return rc;
    rc = jagged_cand_attn_run(q, k, v, a, 0, seg, B, T, H, d_head, scale, attn_ws, attn_bytes,
                              status, stream);
    if (rc) return rc;
    if ((rc = gemm_bf16(a, W + 3 * DD, cur, xo, T, D, D, lt_ws, st))) return rc;
    cur = xo;
  }
  if (n_full == 0 && x_out != x &&
      cudaMemcpyAsync(x_out, x, (size_t)T * D * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return JCA_ERR_CUDA;
  if (n_cand_only == 0 || Nc == 0) return JCA_OK;

  // Split: frozen history rows first, then the candidate rows, in row order within each user.
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  void* hoff = ws + L.hoff;
  void* coff = ws + L.coff;
  int32_t* sidx = reinterpret_cast<int32_t*>(ws + L.sidx);
  const int ub = grid_for(B, 1 << 20);
  if (idx_bits == 32) {
    split_count_kernel<int32_t><<<ub, 256, 0, st>>>(segp, (const int32_t*)offsets, B, cnt, status);
    split_scan_kernel<int32_t><<<1, 1024, 0, st>>>(cnt, B, Th, Nc, (int32_t*)hoff,
                                                   (int32_t*)coff, status);
    split_index_kernel<int32_t><<<ub, 256, 0, st>>>(segp, (const int32_t*)offsets,
                                                    (const int32_t*)hoff, (const int32_t*)coff,
                                                    B, Th, sidx, status);
  } else {
    split_count_kernel<int64_t><<<ub, 256, 0, st>>>(segp, (const int64_t*)offsets, B, cnt, status);
    split_scan_kernel<int64_t><<<1, 1024, 0, st>>>(cnt, B, Th, Nc, (int64_t*)hoff,
                                                   (int64_t*)coff, status);
    split_index_kernel<int64_t><<<ub, 256, 0, st>>>(segp, (const int64_t*)offsets,
                                                    (const int64_t*)hoff, (const int64_t*)coff,
                                                    B, Th, sidx, status);
  }
  const int64_t S = Th + Nc;
  split_rows_kernel<<<grid_for((S + 7) / 8, 148 * 16), 256, 0, st>>>(
      xo, xs, D, sidx, 0, S, 1, rope ? pos : nullptr, spos, status);
  if (cudaGetLastError() != cudaSuccess) return JCA_ERR_CUDA;

  rc = cand_only_attn_plan(coff, hoff, nullptr, B, Nc, Th, H, d_head, idx_bits, cand_ws,
                           cand_bytes, status, stream);
  if (rc) return rc;
  bf16* xh = xs;
  bf16* xc = xs + Th * D;
  bf16* cq = q;
  bf16* ck = cq + Nc * D;
  bf16* cv = ck + Nc * D;
  bf16* hk = cv + Nc * D;
  bf16* hv = hk + Th * D;
  for (int l = n_full; l < n_layers; ++l) {
    const bf16* W = Wt + (int64_t)l * 4 * DD;
    if ((rc = gemm_bf16(xc, W, nullptr, cq, Nc, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(xc, W + DD, nullptr, ck, Nc, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(xc, W + 2 * DD, nullptr, cv, Nc, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(xh, W + DD, nullptr, hk, Th, D, D, lt_ws, st)) ||
        (rc = gemm_bf16(xh, W + 2 * DD, nullptr, hv, Th, D, D, lt_ws, st)))
      return rc;
    if (rope && ((rc = jca_apply_rope(cq, cq, spos + Th, Nc, H, d_head, rope_base, stream)) ||
                 (rc = jca_apply_rope(ck, ck, spos + Th, Nc, H, d_head, rope_base, stream)) ||
                 (rc = jca_apply_rope(hk, hk, spos, Th, H, d_head, rope_base, stream))))
      return rc;
    rc = cand_only_attn_run(cq, ck, cv, hk, hv, nullptr, a, 0, B, Nc, Th, H, d_head, scale,
                            cand_ws, cand_bytes, status, stream);
    if (rc) return rc;
    if ((rc = gemm_bf16(a, W + 3 * DD, xc, xc, Nc, D, D, lt_ws, st))) return rc;
  }
  // The candidates' new states go back to their rows; history and padding rows keep the states
  // they had at the split.
  split_rows_kernel<<<grid_for((Nc + 7) / 8, 148 * 16), 256, 0, st>>>(
      xo, xs, D, sidx, Th, Nc, 0, nullptr, nullptr, status);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}
