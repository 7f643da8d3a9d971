// UG-Sep masked cross-attention (the separated residual) on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (UG-Sep page, sections 分离残差连接 and UG-Separated Mixup 与 mask): for each
// sample and head, R = softmax(scale * Q K^T under M_UG) V, where Q holds the sample's T_out output
// tokens and K, V its T_in input tokens. M_UG keeps the U outputs (the first c_u) from reading the
// G inputs: output i < c_u attends to inputs j < n_u only, every other output to all T_in inputs.
// With a residual, Y = residual + R. A U output with n_u = 0 sees no key and yields 0 (+ residual).
//
// Design. A sample holds a few dozen tokens, so each input byte feeds only a few FLOPs and the op
// is bound by HBM. Samples are streamed in packs: P consecutive samples whose P * T_out query rows
// fit one 128-row MMA tile and whose P * T_in keys fit one key tile of at most 128 (rounded up to
// 16). Because the samples of a pack are consecutive rows of the packed tensors, each pack is one
// TMA box of Q, one of K and one of V. One tcgen05 MMA computes the pack's scores; the blocks that
// pair a query with another sample's keys are computed and ignored (the tensor core has an order
// of magnitude more throughput than this op needs). The softmax thread of a row reads only its
// sample's block of S, writes P over S (zeros outside its block) and a second MMA forms O = P V.
//
// CTA: one persistent CTA per SM, 10 warps; units (pack, head) in a static stride over the grid.
//   warp 0      TMA producer (lane 0): Q, K and V of a unit into one of STAGES shared stages
//   warp 1      TMEM allocator and MMA issuer (lane 0), order QK(0), [QK(i+1), PV(i)] for i = 0..
//   warps 2-5   softmax + epilogue group 0 (the CTA's even units), one query row per thread
//   warps 6-9   group 1 (odd units)
// TMEM columns: S_0 | O_0 | S_1 | O_1 (128 each).
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "jca_device.cuh"
#include "jca_internal.h"

namespace jca {
namespace {

struct UgArgs {
  const __nv_bfloat16* residual;   // [B * T_out, H, D] or null
  void* out;                       // [B * T_out, H, D] bf16 or fp32
  int32_t* status;
  int64_t B;
  int64_t n_units;                 // packs * H
  int T_out, T_in, c_u, n_u, H;
  int per_pack;                    // samples per pack
  int rows_q;                      // query rows per pack: per_pack * T_out (<= 128)
  int keys;                        // key rows per pack, rounded up to 16 (<= 128)
  float scale_log2;
  int out_fp32;
  int out_v8;                      // out rows may be written with 32-byte stores
};

constexpr int kUgThreads = 320;
constexpr int kUgGroupThreads = 128;

template <int D>
struct UgCfg {
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int SW = ROW_BYTES >= 128 ? 128 : ROW_BYTES;   // swizzle span (bytes)
  static constexpr int NBLK = ROW_BYTES / SW;                     // column blocks per tile
  static constexpr int BOX_X = SW / 2;
  static constexpr int TILE_BYTES = 128 * ROW_BYTES;              // a 128-row tile
  static constexpr int BLK_BYTES = 128 * SW;
  static constexpr uint32_t LAYOUT = SW == 128 ? 2u : (SW == 64 ? 4u : 6u);
  static constexpr int KSTEPS_QK = D / 16;
  static constexpr int KSTEPS_PER_BLK = SW / 32;
  static constexpr int STAGE_BYTES = 3 * TILE_BYTES;              // Q | K | V
  static constexpr int STAGES_FIT = (192 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;  // 2, 4, 8, 8 for D = 128..16
  static constexpr int OFF_Q = 0, OFF_K = TILE_BYTES, OFF_V = 2 * TILE_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int B_FULL = 0;                  // [STAGES] a unit's Q, K, V landed
  static constexpr int B_EMPTY = B_FULL + STAGES;   // [STAGES] the unit's MMAs are done
  static constexpr int B_SFULL = B_EMPTY + STAGES;  // [group] S written by QK
  static constexpr int B_PFULL = B_SFULL + 2;       // [group] P written over S
  static constexpr int B_OFULL = B_PFULL + 2;       // [group] O written by PV
  static constexpr int B_DRAIN = B_OFULL + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_USED = OFF_MISC + 16;
  static constexpr int SMEM_RAW = SMEM_USED + 1024;   // slack for 1 KB alignment
  // At least 120 KB so that a second CTA never shares the SM (and its 512 TMEM columns).
  static constexpr int SMEM_ALLOC = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(TILE_BYTES % 1024 == 0, "swizzled tiles start on 1 KB boundaries");
};

// Units of this CTA under the static stride (unit u = blockIdx.x + i * gridDim.x).
__device__ __forceinline__ int local_units(int64_t n_units) {
  const int64_t b = blockIdx.x;
  return b < n_units ? (int)((n_units - b + gridDim.x - 1) / gridDim.x) : 0;
}

// Non-blocking test of an mbarrier phase (the MMA thread polls two barriers).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D>
__device__ void ug_producer(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const UgArgs& a, uint32_t sbase,
                            uint32_t bars, volatile int* abort_flag) {
  using C = UgCfg<D>;
  const int n_local = local_units(a.n_units);
  const uint32_t tx = (uint32_t)(D * 2 * (a.rows_q + 2 * a.keys));
  int issued = 0;
  bool ok = true;
  for (int i = 0; i < n_local; ++i) {
    const int64_t u = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
    const int64_t pack = u / a.H;
    const int h = (int)(u - pack * a.H);
    const int s = i % C::STAGES;
    ok = mbar_wait(bars + 8 * (C::B_EMPTY + s), ((i / C::STAGES) & 1) ^ 1, abort_flag, a.status);
    if (!ok) break;
    const uint32_t full = bars + 8 * (C::B_FULL + s);
    mbar_arrive_expect_tx(full, tx);
    ++issued;
    const int qrow = (int)(pack * a.rows_q);
    const int krow = (int)(pack * a.per_pack * a.T_in);
    const uint32_t st = sbase + s * C::STAGE_BYTES;
#pragma unroll
    for (int c = 0; c < C::NBLK; ++c) {
      tma_load_3d(st + C::OFF_Q + c * C::BLK_BYTES, tmQ, full, c * C::BOX_X, h, qrow);
      tma_load_3d(st + C::OFF_K + c * C::BLK_BYTES, tmK, full, c * C::BOX_X, h, krow);
      tma_load_3d(st + C::OFF_V + c * C::BLK_BYTES, tmV, full, c * C::BOX_X, h, krow);
    }
  }
  if (!ok) {
    // Aborting: let the copies already issued land before the CTA exits (load n of a stage
    // completes phase n of its full barrier).
    for (int n = issued > C::STAGES ? issued - C::STAGES : 0; n < issued; ++n)
      mbar_wait_drain(bars + 8 * (C::B_FULL + n % C::STAGES), (n / C::STAGES) & 1);
  }
}

template <int D>
__device__ void ug_mma(const UgArgs& a, uint32_t sbase, uint32_t bars, uint32_t tmem,
                       volatile int* abort_flag) {
  using C = UgCfg<D>;
  const int n_local = local_units(a.n_units);
  const uint32_t idesc_qk = idesc_bf16_f32(128, a.keys, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
  const uint64_t dq = smem_desc(sbase + C::OFF_Q, 16, 8 * C::SW, C::LAYOUT);
  const uint64_t dk = smem_desc(sbase + C::OFF_K, 16, 8 * C::SW, C::LAYOUT);
  const uint64_t dv = smem_desc(sbase + C::OFF_V, C::BLK_BYTES, 8 * C::SW, C::LAYOUT);
  const int kpv = a.keys >> 4;
  // S_g = Q K^T of unit i (group g = i & 1) once its operands landed. It is issued after PV(i - 2),
  // the last reader of S_g (the P of the group's previous unit), and MMAs from one thread execute
  // in issue order; the group reads this S only after its SFULL, so the QK may run while the group
  // still finishes its previous unit. O_g is overwritten only by PV(i), which waits for the
  // group's P of unit i, written after the group read the previous O_g.
  auto issue_qk = [&](int i) {
    const int s = i % C::STAGES, g = i & 1;
    tc_fence_after();
    const uint64_t so = (uint64_t)((s * C::STAGE_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < C::KSTEPS_QK; ++kk) {
      const uint32_t off =
          ((kk / C::KSTEPS_PER_BLK) * C::BLK_BYTES + (kk % C::KSTEPS_PER_BLK) * 32) >> 4;
      tc_mma(tmem + (uint32_t)(g * 256), dq + so + off, dk + so + off, idesc_qk,
             kk > 0 ? 1u : 0u);
    }
    tc_commit(bars + 8 * (C::B_SFULL + g));
  };
  // O_g = P_g V of unit i; P_g is read from the first keys / 2 columns of S_g (bf16 pairs).
  auto issue_pv = [&](int i) {
    const int s = i % C::STAGES, g = i & 1;
    tc_fence_after();
    const uint64_t vb = dv + (uint64_t)((s * C::STAGE_BYTES) >> 4);
    constexpr uint32_t kStep = (16 * C::SW) >> 4;   // 16 key rows of V per k-step
    const uint32_t p_tmem = tmem + (uint32_t)(g * 256);
    const uint32_t o_tmem = p_tmem + 128u;
    for (int kk = 0; kk < kpv; ++kk)
      tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, vb + (uint64_t)(kk * kStep), kIdescPV,
                kk > 0 ? 1u : 0u);
    tc_commit(bars + 8 * (C::B_EMPTY + s));
    tc_commit(bars + 8 * (C::B_OFULL + g));
  };
  auto full_bar = [&](int i) { return bars + 8 * (C::B_FULL + i % C::STAGES); };
  auto full_par = [&](int i) { return (uint32_t)((i / C::STAGES) & 1); };
  bool ok = true;
  if (n_local > 0) {
    ok = mbar_wait(full_bar(0), full_par(0), abort_flag, a.status);
    if (ok) issue_qk(0);
  }
  // After PV(i - 1), both QK(i + 1) (the other group's S, last read by PV(i - 1)) and PV(i) may be
  // issued; whichever becomes ready first goes first, PV(i) when both are, so that a late load of
  // unit i + 1 never holds back the PV that releases unit i's stage.
  for (int i = 0; ok && i < n_local; ++i) {
    bool qk_done = i + 1 >= n_local, pv_done = false;
    const uint32_t pbar = bars + 8 * (C::B_PFULL + (i & 1)), ppar = (uint32_t)((i >> 1) & 1);
    const uint64_t t0 = global_timer_ns();
    while (!(qk_done && pv_done)) {
      if (!qk_done && mbar_test(full_bar(i + 1), full_par(i + 1))) {
        issue_qk(i + 1);
        qk_done = true;
      } else if (!pv_done && mbar_test(pbar, ppar)) {
        issue_pv(i);
        pv_done = true;
      } else if (*abort_flag) {
        ok = false;
        break;
      } else if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        atomicCAS(a.status, 0, (int32_t)JCA_STATUS_TIMEOUT);
        ok = false;
        break;
      }
    }
  }
  if (!ok) {
    // Aborting: wait until every MMA this thread issued has completed.
    tc_commit(bars + 8 * C::B_DRAIN);
    mbar_wait_drain(bars + 8 * C::B_DRAIN, 0);
  }
}

// Writes 8 consecutive output values (bf16 or fp32).
__device__ __forceinline__ void ug_store8(const UgArgs& a, size_t idx, const float* o) {
  if (a.out_fp32) {
    float* op = reinterpret_cast<float*>(a.out) + idx;
    if (a.out_v8) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(o[i]);
      st_global_v8(op, w);
    } else {
      reinterpret_cast<float4*>(op)[0] = make_float4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<float4*>(op)[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  } else {
    reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + idx)[0] =
        make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                   pack_bf16x2(o[6], o[7]));
  }
}

__device__ __forceinline__ void ug_store16_bf16(const UgArgs& a, size_t idx, const float* o) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
  __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.out) + idx;
  if (a.out_v8) {
    st_global_v8(op, w);
  } else {
    reinterpret_cast<uint4*>(op)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(op)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

template <int D>
__device__ void ug_softmax(const UgArgs& a, uint32_t bars, uint32_t tmem,
                           volatile int* abort_flag, int warp, int lane) {
  using C = UgCfg<D>;
  const int grp = (warp - 2) >> 2;
  const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
  const int r = quarter * 32 + lane;            // query row of this thread inside a pack
  const uint32_t t_s = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(grp * 256);
  const uint32_t t_o = t_s + 128u;
  // The row's place in every pack: sample sl of the pack, token ti of the sample. Its keys are
  // the columns [col0, col0 + ncols) of S: its own sample's block, cut to the U inputs for a U
  // output.
  const bool in_pack = r < a.rows_q;
  const int sl = in_pack ? r / a.T_out : 0;
  const int ti = in_pack ? r - sl * a.T_out : 0;
  const int col0 = sl * a.T_in;
  const int ncols = in_pack ? (ti < a.c_u ? a.n_u : a.T_in) : 0;
  const int kchunks = (a.keys + 31) >> 5;       // 32-key chunks of P the PV reads
  // The warp's rows lie in samples [w_first, w_last] of a pack, whose blocks of S fill the 32-key
  // chunks [ch_lo, ch_hi]; a warp without a row in the pack reads no chunk (its lanes' P and O
  // rows feed no output).
  const int r0 = quarter * 32;
  const bool warp_in = r0 < a.rows_q;
  const int w_first = warp_in ? r0 / a.T_out : 0;
  const int w_last = warp_in ? min(r0 + 31, a.rows_q - 1) / a.T_out : 0;
  const int ch_lo = warp_in ? (w_first * a.T_in) >> 5 : 4;
  const int ch_hi = warp_in ? ((w_last + 1) * a.T_in - 1) >> 5 : -1;
  const float sl2 = a.scale_log2;
  const int n_local = local_units(a.n_units);
  bool ok = true;
  for (int i = grp; i < n_local; i += 2) {
    const int64_t u = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
    const int64_t pack = u / a.H;
    const int h = (int)(u - pack * a.H);
    const int64_t sample = pack * a.per_pack + sl;
    const bool row_ok = in_pack && sample < a.B;
    const int nc = row_ok ? ncols : 0;
    const size_t base =
        ((size_t)(row_ok ? sample * a.T_out + ti : 0) * (size_t)a.H + (size_t)h) * D;
    // The residual row starts moving towards L2 while the scores are computed.
    if (a.residual != nullptr && row_ok) {
#pragma unroll
      for (int c = 0; c < D * 2; c += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.residual + base + c / 2));
    }
    ok = __all_sync(0xffffffffu,
                    mbar_wait(bars + 8 * (C::B_SFULL + grp), (i >> 1) & 1, abort_flag, a.status));
    if (!ok) break;
    tc_fence_after();
    // Only the 32-key chunks of S that hold the blocks of the warp's samples are read (twice: the
    // row max, then the probabilities), 32 columns at a time; inside a chunk a bit mask keeps the
    // row's own columns [col0, col0 + nc).
    const int hi = col0 + nc;
    auto chunk_bits = [&](int c) -> uint32_t {
      const int lo_c = min(max(col0 - 32 * c, 0), 32), hi_c = min(max(hi - 32 * c, 0), 32);
      return (hi_c >= 32 ? 0xffffffffu : ((1u << hi_c) - 1u)) &
             ~(lo_c >= 32 ? 0xffffffffu : ((1u << lo_c) - 1u));
    };
    float mx0 = -INFINITY, mx1 = -INFINITY;
    for (int c = ch_lo; c <= ch_hi; ++c) {
      uint32_t x[32];
      tmem_ld_x32(t_s + 32 * c, x);
      tmem_wait_ld();
      reg_fence16(x);
      reg_fence16(x + 16);
      const uint32_t bits = chunk_bits(c);
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const uint32_t b = bits >> j;
        mx0 = fmax3(mx0, (b & 1u) ? __uint_as_float(x[j]) : -INFINITY,
                    (b & 2u) ? __uint_as_float(x[j + 1]) : -INFINITY);
        mx1 = fmax3(mx1, (b & 4u) ? __uint_as_float(x[j + 2]) : -INFINITY,
                    (b & 8u) ? __uint_as_float(x[j + 3]) : -INFINITY);
      }
    }
    const float m = fmaxf(mx0, mx1) * sl2;
    const float neg_m = (nc == 0) ? 0.f : -m;
    float l0 = 0.f, l1 = 0.f;
    for (int c = 0; c < kchunks; ++c) {
      uint32_t pk[16];
      if (c >= ch_lo && c <= ch_hi) {
        uint32_t x[32];
        tmem_ld_x32(t_s + 32 * c, x);
        tmem_wait_ld();
        reg_fence16(x);
        reg_fence16(x + 16);
        const uint32_t bits = chunk_bits(c);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t b = bits >> (2 * k);
          const float p0 = (b & 1u) ? fast_exp2(fmaf(__uint_as_float(x[2 * k]), sl2, neg_m)) : 0.f;
          const float p1 =
              (b & 2u) ? fast_exp2(fmaf(__uint_as_float(x[2 * k + 1]), sl2, neg_m)) : 0.f;
          l0 += p0;
          l1 += p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = 0u;
      }
      tmem_st_x16(t_s + 16 * c, pk);
    }
    const float l = l0 + l1;
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bars + 8 * (C::B_PFULL + grp));

    const float inv = l > 0.f ? 1.f / l : 0.f;   // no visible key: R = 0
    // The residual row is read into registers while the PV runs.
    uint4 rv[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c)
      rv[c] = (a.residual != nullptr && row_ok)
                  ? ld_global_nc_v4(reinterpret_cast<const uint4*>(a.residual + base) + c)
                  : make_uint4(0u, 0u, 0u, 0u);
    ok = __all_sync(0xffffffffu,
                    mbar_wait(bars + 8 * (C::B_OFULL + grp), (i >> 1) & 1, abort_flag, a.status));
    if (!ok) break;
    tc_fence_after();
    constexpr int CW = D < 32 ? D : 32;   // columns per TMEM load
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += CW) {
      uint32_t w[CW];
      if constexpr (CW == 32) tmem_ld_x32(t_o + c0, w);
      else tmem_ld_x16(t_o + c0, w);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < CW; k += 16) reg_fence16(w + k);
      if (!row_ok) continue;
      float o[CW];
#pragma unroll
      for (int k = 0; k < CW / 8; ++k) {
        const uint4 rr = rv[c0 / 8 + k];
        const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[8 * k + 2 * e] = fmaf(__uint_as_float(w[8 * k + 2 * e]), inv, bf16_lo(rw[e]));
          o[8 * k + 2 * e + 1] = fmaf(__uint_as_float(w[8 * k + 2 * e + 1]), inv, bf16_hi(rw[e]));
        }
      }
      if (a.out_fp32) {
#pragma unroll
        for (int k = 0; k < CW; k += 8) ug_store8(a, base + c0 + k, o + k);
      } else {
#pragma unroll
        for (int k = 0; k < CW; k += 16) ug_store16_bf16(a, base + c0 + k, o + k);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kUgThreads, 1)
    ug_cross_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const UgArgs a) {
  using C = UgCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* skip = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // An error recorded earlier on the stream makes the launch a no-op.
  if (threadIdx.x == 0) {
    *skip = *a.status != 0;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(bars + 8 * (C::B_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_EMPTY + i), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bars + 8 * (C::B_SFULL + g), 1);
      mbar_init(bars + 8 * (C::B_PFULL + g), kUgGroupThreads);
      mbar_init(bars + 8 * (C::B_OFULL + g), 1);
    }
    mbar_init(bars + 8 * C::B_DRAIN, 1);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (!*skip) {
    if (warp == 0) {
      if (lane == 0) ug_producer<D>(&tmQ, &tmK, &tmV, a, sbase, bars, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) ug_mma<D>(a, sbase, bars, tmem, abort_flag);
    } else {
      ug_softmax<D>(a, bars, tmem, abort_flag, warp, lane);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Degenerate layer without input tokens (T_in = 0): every output sees no key, so Y = residual
// (or 0). One thread per 8 output values.
__global__ void ug_no_keys_kernel(const __nv_bfloat16* __restrict__ residual, void* out,
                                  int out_fp32, int64_t n8, const int32_t* status) {
  if (*status != 0) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 r = residual ? reinterpret_cast<const uint4*>(residual)[i]
                             : make_uint4(0u, 0u, 0u, 0u);
    if (out_fp32) {
      float4* op = reinterpret_cast<float4*>(out) + 2 * i;
      op[0] = make_float4(bf16_lo(r.x), bf16_hi(r.x), bf16_lo(r.y), bf16_hi(r.y));
      op[1] = make_float4(bf16_lo(r.z), bf16_hi(r.z), bf16_lo(r.w), bf16_hi(r.w));
    } else {
      reinterpret_cast<uint4*>(out)[i] = r;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
// Kernel attributes set so far, per device and head size.
constexpr int kUgMaxDevices = 64;
bool g_ug_attr[kUgMaxDevices][4];
std::mutex g_ug_mu;

template <int D>
int launch_ug(const void* q, const void* k, const void* v, UgArgs a, int64_t B, int T_out,
              int T_in, cudaStream_t stream) {
  using C = UgCfg<D>;
  int dev = 0, sms = 0;
  const int rc = current_device(&dev, &sms);
  if (rc) return rc;
  const int di = D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : 3;
  {
    std::lock_guard<std::mutex> lock(g_ug_mu);
    if (!g_ug_attr[dev][di]) {
      if (cudaFuncSetAttribute(ug_cross_attn_kernel<D>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess)
        return JCA_ERR_CUDA;
      g_ug_attr[dev][di] = true;
    }
  }
  CUtensorMap tmQ, tmK, tmV;
  if (!make_rows_map_bf16(&tmQ, q, B * T_out, a.H, D, a.rows_q) ||
      !make_rows_map_bf16(&tmK, k, B * T_in, a.H, D, a.keys) ||
      !make_rows_map_bf16(&tmV, v, B * T_in, a.H, D, a.keys))
    return JCA_ERR_CUDA;
  const int64_t grid64 = a.n_units < sms ? a.n_units : sms;
  ug_cross_attn_kernel<D><<<(int)grid64, kUgThreads, C::SMEM_ALLOC, stream>>>(tmQ, tmK, tmV, a);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

}  // namespace
}  // namespace jca

using namespace jca;

extern "C" int ug_masked_cross_attn_fwd(const void* q, const void* k, const void* v,
                                        const void* residual, void* out, int out_fp32, int64_t B,
                                        int T_out, int T_in, int c_u, int n_u, int H, int d_head,
                                        float scale, int32_t* status, cudaStream_t stream) {
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (B < 0 || T_out < 0 || T_in < 0 || T_out > 128 || T_in > 128 || H < 1 || H >= 65536 ||
      c_u < 0 || c_u > T_out || n_u < 0 || n_u > T_in)
    return JCA_ERR_SHAPE;
  // TMA row coordinates are 32-bit.
  if (B * (int64_t)(T_out > T_in ? T_out : T_in) + 128 >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  // Tensors without elements may be null (empty tensors often have no storage).
  const bool has_q = B > 0 && T_out > 0, has_kv = B > 0 && T_in > 0;
  if (!status || (has_q && (!q || !out)) || (has_kv && (!k || !v))) return JCA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (residual && !aligned(residual, 16)))
    return JCA_ERR_ALIGN;
  if (B == 0 || T_out == 0) return JCA_OK;
  if (T_in == 0) {
    const int64_t n8 = B * T_out * (int64_t)H * d_head / 8;
    const int64_t blocks64 = (n8 + 255) / 256;
    const int blocks = (int)(blocks64 < 4096 ? blocks64 : 4096);
    ug_no_keys_kernel<<<blocks, 256, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(residual), out, out_fp32, n8, status);
    return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
  }
  UgArgs a{};
  a.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  a.out = out;
  a.status = status;
  a.B = B;
  a.T_out = T_out;
  a.T_in = T_in;
  a.c_u = c_u;
  a.n_u = n_u;
  a.H = H;
  const int by_q = 128 / T_out, by_k = 128 / T_in;
  a.per_pack = by_q < by_k ? by_q : by_k;
  a.rows_q = a.per_pack * T_out;
  a.keys = (a.per_pack * T_in + 15) & ~15;
  const int64_t packs = (B + a.per_pack - 1) / a.per_pack;
  a.n_units = packs * H;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d_head);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.out_fp32 = out_fp32 ? 1 : 0;
  a.out_v8 = aligned(out, 32) ? 1 : 0;
  switch (d_head) {
    case 16: return launch_ug<16>(q, k, v, a, B, T_out, T_in, stream);
    case 32: return launch_ug<32>(q, k, v, a, B, T_out, T_in, stream);
    case 64: return launch_ug<64>(q, k, v, a, B, T_out, T_in, stream);
    default: return launch_ug<128>(q, k, v, a, B, T_out, T_in, stream);
  }
}
