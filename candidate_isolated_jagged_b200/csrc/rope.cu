// Right-anchored rotary position embedding (候选隔离注意力掩码, section 位置编码：候选共用一个位置):
// the newest history record of every user sits at history_end - 1 and every candidate at
// history_end, so candidate order carries no information. Two kernels:
//   * positions: one block per user row; the segment-1 run (prefix + history) is numbered so that
//     it ends at history_end - 1 (padding takes the position the next segment-1 token would take,
//     candidates take history_end);
//   * rotation: rows of a [T, H, d] bf16 tensor rotated pairwise (element j with j + d/2) by
//     pos * base^(-2j/d) (cos/sin as rope_device.cuh forms them, rotation in fp32), rounded once
//     to bf16. Memory-bound: one read and one write of the tensor, 16-byte accesses.
// and the cos/sin factor tables that the attention kernel's in-tile rotation reads.
#include <climits>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "jca_internal.h"
#include "rope_device.cuh"

namespace jca {
namespace {

__device__ __forceinline__ void set_status(int32_t* status, int code) {
  atomicCAS(status, 0, (int32_t)code);
}

template <typename IdxT>
__global__ void __launch_bounds__(256) rope_positions_kernel(const int8_t* __restrict__ seg,
                                                             const IdxT* __restrict__ off,
                                                             int64_t B, int64_t T,
                                                             int64_t history_end,
                                                             int32_t* __restrict__ pos,
                                                             int32_t* status) {
  if (*status != 0) return;
  __shared__ int s_warp[8];
  __shared__ int s_carry;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    if (s < 0 || s > e || e > T || (b == 0 && s != 0) || (b == B - 1 && e != T)) {
      if (threadIdx.x == 0) set_status(status, JCA_STATUS_BAD_OFFSETS);
      continue;
    }
    const int L = (int)(e - s);
    // Pass 1: n = segment-1 tokens of the row.
    int cnt = 0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) cnt += seg[s + i] == 1;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) s_warp[wid] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
      int n = 0;
      for (int w = 0; w < nw; ++w) n += s_warp[w];
      s_carry = n;   // reused below as the running count, after this block-wide read
    }
    __syncthreads();
    const long long first = history_end - s_carry;   // position of the row's first segment-1 token
    __syncthreads();
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    // Pass 2: exclusive scan of the segment-1 flags, chunk by chunk.
    for (int base = 0; base < L; base += blockDim.x) {
      const int i = base + threadIdx.x;
      const int x = i < L ? (int)seg[s + i] : 0;
      const int f = x == 1;
      const unsigned ball = __ballot_sync(0xffffffffu, f);
      const int in_warp = __popc(ball & ((1u << lane) - 1u));
      if (lane == 0) s_warp[wid] = __popc(ball);
      __syncthreads();
      int before = s_carry;
      for (int w = 0; w < wid; ++w) before += s_warp[w];
      before += in_warp;
      if (i < L) {
        const long long p = x == -1 ? history_end : first + before;
        pos[s + i] = (int32_t)max((long long)INT_MIN, min((long long)INT_MAX, p));
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int tot = 0;
        for (int w = 0; w < nw; ++w) tot += s_warp[w];
        s_carry += tot;
      }
      __syncthreads();
    }
  }
}

// One thread rotates 8 pairs (16 bytes of each half) of one (row, head) per step. The grid stride
// is a multiple of the units per (row, head), so a thread always handles the same 8 frequencies
// and computes them once.
template <int D>
__global__ void __launch_bounds__(256) rope_rotate_kernel(const __nv_bfloat16* __restrict__ x,
                                                          __nv_bfloat16* __restrict__ out,
                                                          const int32_t* __restrict__ pos,
                                                          int64_t T, int H, double log2_base) {
  constexpr int HALF = D / 2;
  constexpr int UNITS = HALF / 8;   // 8-pair units per (row, head)
  static_assert(256 % UNITS == 0, "stride keeps each thread on one set of frequencies");
  const int64_t total = T * (int64_t)H * UNITS;
  const int64_t u0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int j0 = (int)(u0 % UNITS) * 8;
  double inv_freq[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) inv_freq[t] = rope_inv_freq(j0 + t, D, log2_base);
  for (int64_t u = u0; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rh = u / UNITS;
    const int64_t row = rh / H;
    const size_t base = (size_t)rh * D;
    int64_t q;
    int r;
    rope_split((int64_t)pos[row], q, r);
    const uint4 va = *reinterpret_cast<const uint4*>(x + base + j0);
    const uint4 vb = *reinterpret_cast<const uint4*>(x + base + HALF + j0);
    const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
    uint32_t ra[4], rb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a2[2], b2[2], oa[2], ob[2];
      a2[0] = __uint_as_float(wa[k] << 16);
      a2[1] = __uint_as_float(wa[k] & 0xffff0000u);
      b2[0] = __uint_as_float(wb[k] << 16);
      b2[1] = __uint_as_float(wb[k] & 0xffff0000u);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const double f = inv_freq[2 * k + t];
        const float2 cs = rope_compose(rope_cs((double)(q * kRopeFine), f), rope_cs((double)r, f));
        rope_rotate(a2[t], b2[t], cs, oa[t], ob[t]);
      }
      __nv_bfloat162 ha = __floats2bfloat162_rn(oa[0], oa[1]);
      __nv_bfloat162 hb = __floats2bfloat162_rn(ob[0], ob[1]);
      ra[k] = *reinterpret_cast<uint32_t*>(&ha);
      rb[k] = *reinterpret_cast<uint32_t*>(&hb);
    }
    *reinterpret_cast<uint4*>(out + base + j0) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
    *reinterpret_cast<uint4*>(out + base + HALF + j0) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
  }
}

// The factor tables of the in-tile rotation: coarse[i][j] = (cos, sin)(128 (qmax - i) theta_j) for
// i in [0, n_coarse), fine[r][j] = (cos, sin)(r theta_j) for r in [0, 128); theta_j as above.
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ coarse,
                                                         float2* __restrict__ fine, int half,
                                                         int d, int64_t qmax, int64_t n_coarse,
                                                         double log2_base) {
  const int64_t n = (n_coarse + kRopeFine) * half;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / half;
    const int j = (int)(e - i * half);
    const double f = rope_inv_freq(j, d, log2_base);
    if (i < n_coarse)
      coarse[e] = rope_cs((double)((qmax - i) * kRopeFine), f);
    else
      fine[e - n_coarse * half] = rope_cs((double)(i - n_coarse), f);
  }
}

int sm_count() {
  static int sms = [] {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 148;
    return n;
  }();
  return sms;
}

}  // namespace

RopeTables rope_tables(int64_t T, int64_t history_end) {
  RopeTables t;
  // Positions lie in [history_end - T, history_end]: a row's segment-1 run is at most T long.
  auto fl = [](int64_t p) { return p >= 0 ? p / kRopeFine : -((-p + kRopeFine - 1) / kRopeFine); };
  const int64_t qmax = fl(history_end), qmin = fl(history_end - T);
  t.qmax = qmax;
  t.n_coarse = qmax - qmin + 1;
  return t;
}

cudaError_t launch_rope_tables(float2* coarse, float2* fine, int d, const RopeTables& t,
                               float base, cudaStream_t stream) {
  const int half = d / 2;
  const int64_t n = (t.n_coarse + kRopeFine) * half;
  const int64_t want = (n + 255) / 256;
  const int grid = (int)(want < (int64_t)sm_count() * 8 ? want : (int64_t)sm_count() * 8);
  rope_table_kernel<<<grid, 256, 0, stream>>>(coarse, fine, half, d, t.qmax, t.n_coarse,
                                              log2((double)base));
  return cudaGetLastError();
}

}  // namespace jca

using namespace jca;

extern "C" int jca_rope_positions(const int8_t* seg, const void* offsets, int64_t B, int64_t T,
                                  int64_t history_end, int idx_bits, int32_t* positions,
                                  int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (B < 0 || T < 0 || T >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  if (B == 0 && T != 0) return JCA_ERR_SHAPE;
  if (!status || !offsets || (T > 0 && (!seg || !positions))) return JCA_ERR_NULL;
  if (B == 0) return JCA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int grid = (int)(B < (1 << 20) ? B : (1 << 20));
  if (idx_bits == 32)
    rope_positions_kernel<int32_t><<<grid, 256, 0, st>>>(seg, (const int32_t*)offsets, B, T,
                                                         history_end, positions, status);
  else
    rope_positions_kernel<int64_t><<<grid, 256, 0, st>>>(seg, (const int64_t*)offsets, B, T,
                                                         history_end, positions, status);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

extern "C" int jca_apply_rope(const void* x, void* out, const int32_t* positions, int64_t T, int H,
                              int d_head, float base, jca_stream_t stream) {
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (T < 0 || H < 1 || T >= (int64_t)INT_MAX || !(base > 1.f)) return JCA_ERR_SHAPE;
  if (T == 0) return JCA_OK;
  if (!x || !out || !positions) return JCA_ERR_NULL;
  if (!aligned(x, 16) || !aligned(out, 16)) return JCA_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t units = T * (int64_t)H * (d_head / 16);
  const int64_t want = (units + 255) / 256;
  const int grid = (int)(want < (int64_t)sm_count() * 16 ? want : (int64_t)sm_count() * 16);
  const double log2_base = log2((double)base);
  const __nv_bfloat16* xi = static_cast<const __nv_bfloat16*>(x);
  __nv_bfloat16* xo = static_cast<__nv_bfloat16*>(out);
  switch (d_head) {
    case 16: rope_rotate_kernel<16><<<grid, 256, 0, st>>>(xi, xo, positions, T, H, log2_base); break;
    case 32: rope_rotate_kernel<32><<<grid, 256, 0, st>>>(xi, xo, positions, T, H, log2_base); break;
    case 64: rope_rotate_kernel<64><<<grid, 256, 0, st>>>(xi, xo, positions, T, H, log2_base); break;
    default: rope_rotate_kernel<128><<<grid, 256, 0, st>>>(xi, xo, positions, T, H, log2_base); break;
  }
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}
