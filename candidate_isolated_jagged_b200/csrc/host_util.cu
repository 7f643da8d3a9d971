// Host-side helpers shared by the kernel launchers: TMA tensor maps over the token-major bf16
// tensors of the ABI, and the current device's multiprocessor count and architecture.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "jca_internal.h"

namespace jca {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no libcuda link).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

struct DeviceProps {
  int sms = 0;
  bool sm100 = false;
};
constexpr int kMaxDevices = 64;
DeviceProps g_props[kMaxDevices];
std::mutex g_props_mu;

}  // namespace

bool make_rows_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int H, int D,
                        int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int sw = D * 2 >= 128 ? 128 : D * 2;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)(sw / 2), 1u, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle swz = sw == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : sw == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int current_device(int* dev, int* sms) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return JCA_ERR_CUDA;
  DeviceProps* p = &g_props[d];
  std::lock_guard<std::mutex> lock(g_props_mu);
  if (p->sms == 0) {
    int major = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess)
      return JCA_ERR_CUDA;
    p->sm100 = major == 10;
    p->sms = n;
  }
  if (!p->sm100) return JCA_ERR_DEVICE;
  *dev = d;
  *sms = p->sms;
  return JCA_OK;
}

}  // namespace jca
