// jagged_cand_attn_fwd_noalloc: the full jagged attention call for callers that cannot hand the
// library a workspace.
//
// Some callers have no way to obtain device scratch memory at call time: a serving loop whose
// memory is reserved up front and must not change while requests are in flight, a plugin that is
// given only its input and output tensors by a host framework, or code for which cudaMalloc's
// implicit device synchronisation is not acceptable on the request path. For them this entry point
// keeps its scratch (segment IDs, per-user bounds, the work queue) in one fixed-size array that
// lives in the library's own device memory, so a call needs nothing beyond its inputs and outputs.
//
// The array is a file-scope static __device__ object: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits. Host code cannot use its name as a device
// address; jca_noalloc_prepare(), or else the first call on each device, looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it.
#include <climits>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "jca_internal.h"

namespace jca {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxScratchDevices = 64;
void* g_scratch_addr[kMaxScratchDevices] = {};
std::mutex g_scratch_mu;

// Device address of the static scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices)
    return JCA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return JCA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return JCA_OK;
}

}  // namespace
}  // namespace jca

extern "C" size_t jca_noalloc_scratch_bytes(void) { return jca::kNoAllocScratchBytes; }

extern "C" int jca_noalloc_prepare(void) {
  void* scratch = nullptr;
  return jca::scratch_address(&scratch);
}

extern "C" int jagged_cand_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                            void* out, int out_fp32, const void* offsets,
                                            const void* candidate_start, const int8_t* seg,
                                            int64_t B, int64_t T, int H, int d_head, float scale,
                                            int idx_bits, int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (!jca::head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (B < 0 || T < 0 || H < 1 || H >= 65536 || T >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX)
    return JCA_ERR_SHAPE;
  const size_t need = jca::workspace_layout(B, T, H).total;
  if (need > jca::kNoAllocScratchBytes) return JCA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int rc = jca::scratch_address(&scratch);
  if (rc != JCA_OK) return rc;
  // No byte of the scratch has to start at zero: the plan kernels write everything the attention
  // kernel reads (segment IDs, bounds, the queue and its length) before it runs.
  return jagged_cand_attn_fwd(q, k, v, out, out_fp32, offsets, candidate_start, seg, B, T, H,
                              d_head, scale, idx_bits, scratch, jca::kNoAllocScratchBytes, status,
                              stream);
}
