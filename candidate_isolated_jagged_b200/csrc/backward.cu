// Backward pass of jagged candidate-isolated attention on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes: the gradients of the forward's masked softmax attention (候选隔离注意力掩码,
// sections 段 ID：掩码的表达方式 and 掩码长什么样), trained on the same packed layout the forward
// serves (section 训练时的序列打包). Per user and head, with P the forward's probabilities,
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D) with D = rowsum(dO * O),
//   dQ = scale dS K,   dK = scale dS^T Q.
// P is rebuilt tile by tile from the forward's log-sum-exp, so no [L, L] matrix exists anywhere.
// The mask splits the work in three parts with no overlap and no atomics:
//   * keys with segment 1 (prefix + history) are seen by every non-padding query of their user:
//     a key-outer kernel (mode dKV) takes one 128-key tile of a user's history interval and walks
//     all of the user's query tiles, accumulating dV = P^T dO and dK = dS^T Q in TMEM;
//   * every query reads only the segment-1 keys plus, for a candidate, itself: a query-outer
//     kernel (mode dQ) takes one 128-row query tile and walks the history key tiles,
//     accumulating dQ = dS K in TMEM;
//   * a candidate's own key and value are seen by that candidate alone, so their gradients (and
//     the candidate's diagonal share of dQ) are scalar work done in the dQ kernel's epilogue on
//     CUDA cores, like the forward's diagonal term.
// Both modes share one kernel body. With O1/O2 the two "outer" tiles loaded once per unit and
// I1/I2 the two "inner" tiles streamed through a ring, every inner step issues
//   S = O1 I1^T and dP = O2 I2^T (SS MMAs, M = N = 128, K = d, fp32 in TMEM),
// the compute warps (one TMEM lane = one outer row per thread) turn them into bf16 dS (and, for
// dKV, bf16 P) written back over S / dP, and the MMA thread issues the TS MMAs that read them
// from TMEM as the A operand:
//   mode dQ  (O1 = Q, O2 = dO, I1 = K, I2 = V):   acc0 += dS I1
//   mode dKV (O1 = K, O2 = V, I1 = Q, I2 = dO):   acc0 (dV) += P^T I2,  acc1 (dK) += dS^T I1.
// Each 128-row inner tile is consumed as two 64-row half steps, so that S and dP fit twice in
// TMEM: while the compute warps work on half step t, the tensor core computes S and dP of t + 1.
// TMEM columns: S0 | dP0 | S1 | dP1 (64 each) | acc0 | acc1 (128 each); 512 allocated.
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

using bf16 = __nv_bfloat16;

constexpr int kModeDQ = 0;
constexpr int kModeDKV = 1;
constexpr int kBwdThreads = 320;     // warp 0 producer, warp 1 MMA, warps 2..9 compute
constexpr int kBwdCompute = 256;
constexpr int kBwdStages = 2;        // inner ring depth
constexpr int kHalf = 64;            // inner rows per half step

struct BwdArgs {
  const bf16* q;
  const bf16* k;
  const bf16* v;
  const bf16* dout;
  void* dq;
  void* dk;
  void* dv;
  const int8_t* seg;       // [T]
  const float* lse2;       // [H][T]: log2-units log-sum-exp of each row; +inf = row sees no key
  const float* dsum;       // [H][T]: rowsum(dO * O)
  const int4* items;
  const int2* items2;      // dKV only, or null: a second query run {row start, rows} per item
  const int32_t* n_items;
  int32_t* status;
  int64_t T;
  int H;
  int grad_fp32;
  float scale;
  float scale_log2;
};

template <int D>
struct BCfg {
  static constexpr int BM = kTileM;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int SW = ROW_BYTES >= 128 ? 128 : ROW_BYTES;
  static constexpr int NBLK = ROW_BYTES / SW;
  static constexpr int BOX_X = SW / 2;
  static constexpr int TILE_BYTES = BM * ROW_BYTES;
  static constexpr int BLK_BYTES = BM * SW;
  static constexpr uint32_t LAYOUT = SW == 128 ? 2u : (SW == 64 ? 4u : 6u);
  static constexpr int KSTEPS_QK = D / 16;
  static constexpr int KSTEPS_PER_BLK = SW / 32;
  static constexpr int OFF_OUT = 0;                                   // 2 tiles
  static constexpr int OFF_IN = 2 * TILE_BYTES;                       // kBwdStages x 2 tiles
  static constexpr int OFF_BAR = OFF_IN + kBwdStages * 2 * TILE_BYTES;
  static constexpr int B_OUTFULL = 0;
  static constexpr int B_OUTEMPTY = 1;
  static constexpr int B_INFULL = 2;                                  // [kBwdStages]
  static constexpr int B_INEMPTY = B_INFULL + kBwdStages;             // [kBwdStages]
  static constexpr int B_SPFULL = B_INEMPTY + kBwdStages;             // [2] S and dP written
  // [2] dS (and P) of the half step in buffer b written back. One barrier per buffer: with
  // S/dP of step t + 1 already computed, a warp may finish step t + 1 before another warp
  // finishes step t, and its arrival must not count toward step t.
  static constexpr int B_DSFULL = B_SPFULL + 2;
  static constexpr int B_ACCFULL = B_DSFULL + 2;                      // unit's last TS MMA done
  static constexpr int B_ACCFREE = B_ACCFULL + 1;                     // accumulators read
  static constexpr int B_COLS = B_ACCFREE + 1;                        // [2] column stats (dKV)
  static constexpr int B_DRAIN = B_COLS + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_COLS = OFF_MISC + 16;                      // [2][2][128] floats
  static constexpr int SMEM_USED = OFF_COLS + 2 * 2 * BM * 4;
  static constexpr int SMEM_RAW = SMEM_USED + 1024;
  // At least 120 KB so that a second CTA never shares the SM (and its TMEM).
  static constexpr int SMEM_ALLOC = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
  // Half-step buffer b: S at 128 b, dP at 128 b + 64.
  static constexpr uint32_t TMEM_S = 0, TMEM_P = 64, TMEM_BUF = 128, TMEM_A0 = 256,
                            TMEM_A1 = 384, TMEM_COLS = 512;
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
};

// One unit of work: `orows` outer rows starting at `orow0` for head h, against the inner rows
// [in_lo, in_lo + in_len) and then [in_lo2, in_lo2 + in_len2), walked in tiles of 128 (n_in1
// tiles over the first run, n_in in all). The second run is empty except for dKV units of the
// candidate-packed layout, where a user's candidate queries sit apart from its history.
struct Unit {
  int orow0, orows, h, in_lo, in_len, holes, n_in, in_lo2, in_len2, n_in1;
};

// First row and valid rows of inner tile i of a unit.
__device__ __forceinline__ int in_row(const Unit& u, int i) {
  return i < u.n_in1 ? u.in_lo + i * kTileN : u.in_lo2 + (i - u.n_in1) * kTileN;
}

__device__ __forceinline__ int in_valid(const Unit& u, int i) {
  return i < u.n_in1 ? min(kTileN, u.in_len - i * kTileN)
                     : min(kTileN, u.in_len2 - (i - u.n_in1) * kTileN);
}

// Units of an item. dQ items are the forward's work items (up to 256 query rows: two units);
// dKV items hold one key tile.
template <int MODE>
__device__ __forceinline__ int unit_count(int4 v) {
  if (MODE == kModeDKV) return 1;
  return ((v.y & 511) + kTileM - 1) / kTileM;
}

template <int MODE>
__device__ __forceinline__ Unit decode_unit(int4 v, int t, const int2* items2, int it) {
  Unit u;
  u.h = v.y >> 9;
  const int rows = v.y & 511;
  u.orow0 = v.x + t * kTileM;
  u.orows = min(kTileM, rows - t * kTileM);
  u.in_lo = v.z;
  if (MODE == kModeDQ) {
    u.in_len = v.w & 0x7fffffff;
    u.holes = (int)((unsigned)v.w >> 31);
  } else {
    u.in_len = v.w;
    u.holes = 0;
  }
  u.n_in1 = (u.in_len + kTileN - 1) / kTileN;
  u.in_lo2 = 0;
  u.in_len2 = 0;
  if (MODE == kModeDKV && items2 != nullptr) {
    const int2 w = items2[it];
    u.in_lo2 = w.x;
    u.in_len2 = w.y;
  }
  u.n_in = u.n_in1 + (u.in_len2 + kTileN - 1) / kTileN;
  return u;
}

// ------------------------------------------------------------------------------------------
// Producer: outer tiles once per unit, inner tile pairs through a kBwdStages ring.
// ------------------------------------------------------------------------------------------
template <int D, int MODE>
__device__ void bwd_producer(const CUtensorMap* tmO1, const CUtensorMap* tmO2,
                             const CUtensorMap* tmI1, const CUtensorMap* tmI2, const BwdArgs& a,
                             uint32_t sbase, uint32_t bars, int n_items,
                             volatile int* abort_flag) {
  using C = BCfg<D>;
  uint32_t u_count = 0, g = 0;
  bool ok = true;
  for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
    const int4 raw = a.items[it];
    const int nu = unit_count<MODE>(raw);
    for (int t = 0; ok && t < nu; ++t) {
      const Unit u = decode_unit<MODE>(raw, t, a.items2, it);
      if (u.n_in == 0) continue;
      ok = mbar_wait(bars + 8 * C::B_OUTEMPTY, (u_count & 1) ^ 1, abort_flag, a.status);
      if (!ok) break;
      mbar_arrive_expect_tx(bars + 8 * C::B_OUTFULL, 2 * C::TILE_BYTES);
      ++u_count;
#pragma unroll
      for (int c = 0; c < C::NBLK; ++c) {
        tma_load_3d(sbase + C::OFF_OUT + c * C::BLK_BYTES, tmO1, bars + 8 * C::B_OUTFULL,
                    c * C::BOX_X, u.h, u.orow0);
        tma_load_3d(sbase + C::OFF_OUT + C::TILE_BYTES + c * C::BLK_BYTES, tmO2,
                    bars + 8 * C::B_OUTFULL, c * C::BOX_X, u.h, u.orow0);
      }
      for (int i = 0; i < u.n_in; ++i, ++g) {
        const int s = (int)(g % kBwdStages);
        ok = mbar_wait(bars + 8 * (C::B_INEMPTY + s), ((g / kBwdStages) & 1) ^ 1, abort_flag,
                       a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bars + 8 * (C::B_INFULL + s), 2 * C::TILE_BYTES);
        const uint32_t dst = sbase + C::OFF_IN + s * 2 * C::TILE_BYTES;
        const int row = in_row(u, i);
#pragma unroll
        for (int c = 0; c < C::NBLK; ++c) {
          tma_load_3d(dst + c * C::BLK_BYTES, tmI1, bars + 8 * (C::B_INFULL + s), c * C::BOX_X,
                      u.h, row);
          tma_load_3d(dst + C::TILE_BYTES + c * C::BLK_BYTES, tmI2, bars + 8 * (C::B_INFULL + s),
                      c * C::BOX_X, u.h, row);
        }
      }
    }
  }
  if (!ok) {
    // Aborting: let the copies this thread started land before the CTA exits.
    if (u_count > 0) mbar_wait_drain(bars + 8 * C::B_OUTFULL, (u_count - 1) & 1);
    for (uint32_t n = g > (uint32_t)kBwdStages ? g - kBwdStages : 0; n < g; ++n)
      mbar_wait_drain(bars + 8 * (C::B_INFULL + (int)(n % kBwdStages)), (n / kBwdStages) & 1);
  }
}

// ------------------------------------------------------------------------------------------
// MMA issuer
// ------------------------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b,
                                           uint32_t idesc) {
  using C = BCfg<D>;
#pragma unroll
  for (int kk = 0; kk < C::KSTEPS_QK; ++kk) {
    const uint32_t off =
        ((kk / C::KSTEPS_PER_BLK) * C::BLK_BYTES + (kk % C::KSTEPS_PER_BLK) * 32) >> 4;
    tc_mma(d_tmem, a + off, b + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A[tmem, bf16 pairs, M = 128 lanes x K = 16 ksteps] * B[smem, MN-major, K rows x N = D].
// The A pairs of a half step sit in two 16-column runs, columns [0, 16) for inner rows 0..31 and
// [32, 48) for rows 32..63 (one run per compute warp of a lane quarter).
template <int D>
__device__ __forceinline__ void bwd_mma_ts(uint32_t acc, uint32_t a_tmem, uint64_t b, int ksteps,
                                           bool overwrite) {
  using C = BCfg<D>;
  constexpr uint32_t kIdesc = idesc_bf16_f32(C::BM, D, false, true);
  constexpr uint32_t kStep = (16 * C::SW) >> 4;
  for (int kk = 0; kk < ksteps; ++kk)
    tc_mma_ts(acc, a_tmem + (uint32_t)(kk >> 1) * 32u + (uint32_t)(kk & 1) * 8u,
              b + (uint64_t)(kk * kStep), kIdesc, (overwrite && kk == 0) ? 0u : 1u);
}

// Half steps of a unit: inner tile i is split into rows [0, 64) and [64, 128) of the tile; the
// second half exists only when the tile holds more than 64 valid rows.
struct HalfStep {
  int i, hh, valid;   // inner tile, half (0 / 1), valid rows of the half (1..64)
};

__device__ __forceinline__ bool next_half(const Unit& u, HalfStep& h) {
  const int tile_valid = in_valid(u, h.i);
  if (h.hh == 0 && tile_valid > kHalf) {
    h.hh = 1;
  } else {
    if (h.i + 1 >= u.n_in) return false;
    ++h.i;
    h.hh = 0;
  }
  h.valid = min(kHalf, in_valid(u, h.i) - h.hh * kHalf);
  return true;
}

template <int D, int MODE>
__device__ void bwd_mma(const BwdArgs& a, uint32_t sbase, uint32_t bars, uint32_t tmem,
                        int n_items, volatile int* abort_flag) {
  using C = BCfg<D>;
  constexpr uint32_t kIdescHalf = idesc_bf16_f32(C::BM, kHalf, false, false);
  constexpr uint32_t kIdesc0 = kIdescHalf & ~(0x3Fu << 17);
  constexpr uint32_t kHalfRows = (kHalf * C::SW) >> 4;   // descriptor offset of row 64
  const uint64_t o1 = smem_desc(sbase + C::OFF_OUT, 16, 8 * C::SW, C::LAYOUT);
  const uint64_t o2 = o1 + (uint64_t)(C::TILE_BYTES >> 4);
  const uint64_t in_k = smem_desc(sbase + C::OFF_IN, 16, 8 * C::SW, C::LAYOUT);
  const uint64_t in_mn = smem_desc(sbase + C::OFF_IN, C::BLK_BYTES, 8 * C::SW, C::LAYOUT);
  uint32_t u_count = 0, g = 0, steps = 0, ts_steps = 0, acc_units = 0;
  bool ok = true;
  // S = O1 I1^T and dP = O2 I2^T of one half step, into TMEM buffer (step & 1).
  auto issue_sp = [&](const HalfStep& h, uint32_t stage) {
    const uint32_t idesc =
        h.valid == kHalf ? kIdescHalf
                         : (kIdesc0 | ((uint32_t)(((h.valid + 15) & ~15) >> 3) << 17));
    const uint64_t i1 = in_k + (uint64_t)((stage * 2 * C::TILE_BYTES) >> 4) +
                        (uint64_t)(h.hh * kHalfRows);
    const uint64_t i2 = i1 + (uint64_t)(C::TILE_BYTES >> 4);
    const uint32_t buf = (steps & 1) * C::TMEM_BUF;
    bwd_mma_ss<D>(tmem + buf + C::TMEM_S, o1, i1, idesc);
    bwd_mma_ss<D>(tmem + buf + C::TMEM_P, o2, i2, idesc);
    tc_commit(bars + 8 * (C::B_SPFULL + (int)(steps & 1)));
    ++steps;
  };
  // The TS MMAs of a half step, once the compute warps wrote its dS (and P).
  auto issue_ts = [&](const HalfStep& h, uint32_t stage, bool first, bool last_half) -> bool {
    if (!mbar_wait(bars + 8 * (C::B_DSFULL + (int)(ts_steps & 1)), (ts_steps >> 1) & 1,
                   abort_flag, a.status))
      return false;
    const uint32_t buf = (ts_steps & 1) * C::TMEM_BUF;
    ++ts_steps;
    if (first && acc_units > 0 &&
        !mbar_wait(bars + 8 * C::B_ACCFREE, (acc_units - 1) & 1, abort_flag, a.status))
      return false;
    tc_fence_after();
    const int ksteps = (h.valid + 15) >> 4;
    const uint64_t m1 = in_mn + (uint64_t)((stage * 2 * C::TILE_BYTES) >> 4) +
                        (uint64_t)(h.hh * kHalfRows);
    const uint64_t m2 = m1 + (uint64_t)(C::TILE_BYTES >> 4);
    if (MODE == kModeDQ) {
      bwd_mma_ts<D>(tmem + C::TMEM_A0, tmem + buf + C::TMEM_P, m1, ksteps, first);
    } else {
      bwd_mma_ts<D>(tmem + C::TMEM_A0, tmem + buf + C::TMEM_S, m2, ksteps, first);
      bwd_mma_ts<D>(tmem + C::TMEM_A1, tmem + buf + C::TMEM_P, m1, ksteps, first);
    }
    if (last_half) tc_commit(bars + 8 * (C::B_INEMPTY + (int)stage));
    return true;
  };
  for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
    const int4 raw = a.items[it];
    const int nu = unit_count<MODE>(raw);
    for (int t = 0; ok && t < nu; ++t) {
      const Unit u = decode_unit<MODE>(raw, t, a.items2, it);
      if (u.n_in == 0) continue;
      ok = mbar_wait(bars + 8 * C::B_OUTFULL, u_count & 1, abort_flag, a.status);
      if (!ok) break;
      ++u_count;
      // One half step of lookahead: S/dP of step t + 1 are issued before the TS MMAs of step t.
      HalfStep cur{0, 0, min(kHalf, in_valid(u, 0))};
      uint32_t cur_stage = g % kBwdStages;
      ok = mbar_wait(bars + 8 * (C::B_INFULL + (int)cur_stage), (g / kBwdStages) & 1, abort_flag,
                     a.status);
      if (!ok) break;
      tc_fence_after();
      issue_sp(cur, cur_stage);
      bool first = true;
      for (;;) {
        HalfStep nxt = cur;
        const bool more = next_half(u, nxt);
        uint32_t nxt_stage = cur_stage;
        if (more && nxt.hh == 0) {
          ++g;
          nxt_stage = g % kBwdStages;
          ok = mbar_wait(bars + 8 * (C::B_INFULL + (int)nxt_stage), (g / kBwdStages) & 1,
                         abort_flag, a.status);
          if (!ok) break;
          tc_fence_after();
        }
        if (more) issue_sp(nxt, nxt_stage);
        // The current half closes its inner tile unless the next step is the tile's second half.
        const bool last_half = !(more && nxt.hh == 1);
        ok = issue_ts(cur, cur_stage, first, last_half);
        if (!ok) break;
        first = false;
        if (!more) break;
        cur = nxt;
        cur_stage = nxt_stage;
      }
      if (!ok) break;
      ++g;
      tc_commit(bars + 8 * C::B_OUTEMPTY);
      tc_commit(bars + 8 * C::B_ACCFULL);
      ++acc_units;
    }
  }
  if (!ok) {
    tc_commit(bars + 8 * C::B_DRAIN);
    mbar_wait_drain(bars + 8 * C::B_DRAIN, 0);
  }
}

// ------------------------------------------------------------------------------------------
// Compute warps
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void store_row8(void* base, int fp32, size_t idx, const float* o) {
  if (fp32) {
    float* p = reinterpret_cast<float*>(base) + idx;
    reinterpret_cast<float4*>(p)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(o[4], o[5], o[6], o[7]);
  } else {
    reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(base) + idx)[0] =
        make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                   pack_bf16x2(o[6], o[7]));
  }
}

// Dot product of two bf16 rows of D elements.
template <int D>
__device__ __forceinline__ float row_dot(const bf16* x, const bf16* y) {
  const uint4* xp = reinterpret_cast<const uint4*>(x);
  const uint4* yp = reinterpret_cast<const uint4*>(y);
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 xv = ld_global_nc_v4(xp + c), yv = ld_global_nc_v4(yp + c);
    acc0 = fmaf(bf16_lo(xv.x), bf16_lo(yv.x), acc0);
    acc1 = fmaf(bf16_hi(xv.x), bf16_hi(yv.x), acc1);
    acc0 = fmaf(bf16_lo(xv.y), bf16_lo(yv.y), acc0);
    acc1 = fmaf(bf16_hi(xv.y), bf16_hi(yv.y), acc1);
    acc0 = fmaf(bf16_lo(xv.z), bf16_lo(yv.z), acc0);
    acc1 = fmaf(bf16_hi(xv.z), bf16_hi(yv.z), acc1);
    acc0 = fmaf(bf16_lo(xv.w), bf16_lo(yv.w), acc0);
    acc1 = fmaf(bf16_hi(xv.w), bf16_hi(yv.w), acc1);
  }
  return acc0 + acc1;
}

__device__ __forceinline__ void unpack8(uint4 w, float* o) {
  o[0] = bf16_lo(w.x); o[1] = bf16_hi(w.x); o[2] = bf16_lo(w.y); o[3] = bf16_hi(w.y);
  o[4] = bf16_lo(w.z); o[5] = bf16_hi(w.z); o[6] = bf16_lo(w.w); o[7] = bf16_hi(w.w);
}

template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t t, uint32_t* r) {
  if constexpr (N == 8) {
    tmem_ld_x8(t, r);
  } else if constexpr (N == 16) {
    tmem_ld_x16(t, r);
  } else {
    tmem_ld_x32(t, r);
  }
}

template <int N>
__device__ __forceinline__ void reg_fence_n(uint32_t* r) {
  if constexpr (N == 8) {
    reg_fence8(r);
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 16) reg_fence16(r + i);
  }
}

// Compute warps 2..9: warp w serves TMEM lane quarter w % 4 (one outer row per thread) and column
// half ch = (w - 2) / 4, i.e. 32 of the 64 inner columns of every half step and half of the D
// columns of the accumulators in the epilogue.
template <int D, int MODE>
__device__ void bwd_compute(const BwdArgs& a, uint32_t bars, uint32_t tmem, float* cols,
                            int n_items, volatile int* abort_flag, int warp, int lane) {
  using C = BCfg<D>;
  const int quarter = warp & 3;
  const int ch = (warp - 2) >> 2;
  const int r = quarter * 32 + lane;            // outer row of this thread inside its tile
  const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
  const uint32_t t_s = t_lane + C::TMEM_S + 32 * ch, t_p = t_lane + C::TMEM_P + 32 * ch;
  // The bf16 pairs of a chunk go to the first 16 columns of the chunk itself, so that a warp
  // never writes columns the other warp of its lane quarter still has to read.
  const uint32_t t_ps = t_s, t_ds = t_p;
  constexpr int HD = D / 2;                     // accumulator columns of this warp
  constexpr int CW = HD < 32 ? HD : 32;
  const uint32_t t_a0 = t_lane + C::TMEM_A0 + ch * HD, t_a1 = t_lane + C::TMEM_A1 + ch * HD;
  const float sl2 = a.scale_log2;
  const float2 sl2v = make_float2(sl2, sl2);
  const int64_t T = a.T;
  uint32_t sp_seen = 0, acc_seen = 0, cols_n = 0;
  bool ok = true;
  for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
    const int4 raw = a.items[it];
    const int nu = unit_count<MODE>(raw);
    for (int t = 0; ok && t < nu; ++t) {
      const Unit u = decode_unit<MODE>(raw, t, a.items2, it);
      const bool row_ok = r < u.orows;
      const int64_t row = (int64_t)u.orow0 + (row_ok ? r : 0);
      const int seg = row_ok ? (int)a.seg[row] : 0;
      const size_t base = ((size_t)row * (size_t)a.H + (size_t)u.h) * D;
      const size_t stat = (size_t)u.h * (size_t)T + (size_t)row;
      // dQ: this row's statistics (padding rows: lse2 = +inf, so P = 0). dKV: a key row that is
      // not a segment-1 key only pollutes its own accumulator row, which is never stored.
      const float lse2 = (MODE == kModeDQ && row_ok) ? a.lse2[stat] : INFINITY;
      const float dsum = (MODE == kModeDQ && row_ok) ? a.dsum[stat] : 0.f;
      const float2 nlv = make_float2(-lse2, -lse2), ndv = make_float2(-dsum, -dsum);
      // dQ: the diagonal term of a candidate row (its score against its own key, P_ii from the
      // forward's log-sum-exp, dS_ii = P_ii (dO_i . v_i - D_i)), computed while the unit's first
      // tiles load, so that the epilogue can release the accumulator at once.
      float pd = 0.f, dsd = 0.f;
      if (MODE == kModeDQ && row_ok && seg == -1) {
        const float sd = row_dot<D>(a.q + base, a.k + base) * sl2;
        pd = fast_exp2(sd - lse2);
        dsd = pd * (row_dot<D>(a.dout + base, a.v + base) - dsum);
      }
      // dKV: column statistics of the query tiles (lse2 = +inf, D = 0 past the user's rows, so
      // that those columns get P = 0), stored negated in shared memory (warps of column half 0
      // fill -lse2, half 1 -D). The value for tile i + 1 is fetched while tile i is computed.
      auto col_stat = [&](int i) -> float {
        const int v = in_valid(u, i);
        if (r >= v) return ch == 0 ? -INFINITY : 0.f;
        const size_t qs = (size_t)u.h * (size_t)T + (size_t)((int64_t)in_row(u, i) + r);
        return ch == 0 ? -a.lse2[qs] : -a.dsum[qs];
      };
      float next_stat = (MODE == kModeDKV && u.n_in > 0) ? col_stat(0) : 0.f;
      for (int i = 0; i < u.n_in; ++i) {
        const int valid = in_valid(u, i);
        float* cl = cols + (cols_n & 1) * 2 * kTileN;   // dKV: -lse2 | -dsum of the 128 columns
        if (MODE == kModeDKV) {
          cl[ch * kTileN + r] = next_stat;
          mbar_arrive(bars + 8 * (C::B_COLS + (cols_n & 1)));
          if (i + 1 < u.n_in) next_stat = col_stat(i + 1);
          ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_COLS + (cols_n & 1)),
                                                 (cols_n >> 1) & 1, abort_flag, a.status));
          ++cols_n;
          if (!ok) break;
        }
        for (int hh = 0; hh < 2; ++hh) {
          const int hvalid = min(kHalf, valid - hh * kHalf);
          if (hvalid <= 0) break;
          const int b = (int)(sp_seen & 1);
          ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (C::B_SPFULL + b),
                                                 (sp_seen >> 1) & 1, abort_flag, a.status));
          if (!ok) break;
          ++sp_seen;
          tc_fence_after();
          const int cvalid = hvalid - 32 * ch;          // valid columns of this warp's chunk
          if (cvalid > 0) {
            const uint32_t buf = b * C::TMEM_BUF;
            uint32_t sv[32], dp[32];
            tmem_ld_x32(t_s + buf, sv);
            tmem_ld_x32(t_p + buf, dp);
            uint32_t bits = 0xffffffffu;
            if (MODE == kModeDQ && (cvalid < 32 || u.holes)) {
              // Key columns past the interval or on padding holes are masked.
              const int c = 32 * ch + lane;
              bool keep = lane < cvalid;
              if (keep && u.holes) keep = a.seg[in_row(u, i) + hh * kHalf + c] == 1;
              bits = __ballot_sync(0xffffffffu, keep);
            }
            tmem_wait_ld();
            reg_fence16(sv);
            reg_fence16(sv + 16);
            reg_fence16(dp);
            reg_fence16(dp + 16);
            if (MODE == kModeDQ && bits != 0xffffffffu) {
#pragma unroll
              for (int j = 0; j < 32; ++j) sv[j] = ((bits >> j) & 1u) ? sv[j] : 0xff800000u;
            }
            const float* cln = cl + hh * kHalf + 32 * ch;
            uint32_t pk_ds[16], pk_p[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float2 nl = nlv, nd = ndv;
              if (MODE == kModeDKV) {
                nl = *reinterpret_cast<const float2*>(cln + j);
                nd = *reinterpret_cast<const float2*>(cln + kTileN + j);
              }
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[j]),
                                                      __uint_as_float(sv[j + 1])), sl2v, nl);
              const float2 pp = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              const float2 dd = __fadd2_rn(make_float2(__uint_as_float(dp[j]),
                                                       __uint_as_float(dp[j + 1])), nd);
              const float2 ds = __fmul2_rn(pp, dd);
              pk_ds[j / 2] = pack_bf16x2(ds.x, ds.y);
              if (MODE == kModeDKV) pk_p[j / 2] = pack_bf16x2(pp.x, pp.y);
            }
            tmem_st_x16(t_ds + buf, pk_ds);
            if (MODE == kModeDKV) tmem_st_x16(t_ps + buf, pk_p);
            tmem_wait_st();
          }
          tc_fence_before();
          mbar_arrive(bars + 8 * (C::B_DSFULL + b));
        }
        if (!ok) break;
      }
      if (!ok) break;

      // ---- epilogue: this warp's half of the D accumulator columns ----
      const bool has_acc = u.n_in > 0;
      if (has_acc) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bars + 8 * C::B_ACCFULL, acc_seen & 1, abort_flag, a.status));
        if (!ok) break;
        ++acc_seen;
        tc_fence_after();
      }
      const size_t cbase = base + (size_t)(ch * HD);
      if (MODE == kModeDKV) {
        const bool kvalid = row_ok && seg == 1;
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += CW) {
          uint32_t dvv[CW], dkv[CW];
          tmem_ld_n<CW>(t_a0 + c0, dvv);
          tmem_ld_n<CW>(t_a1 + c0, dkv);
          tmem_wait_ld();
          reg_fence_n<CW>(dvv);
          reg_fence_n<CW>(dkv);
          if (c0 + CW >= HD) {
            tc_fence_before();
            mbar_arrive(bars + 8 * C::B_ACCFREE);
          }
          if (!kvalid) continue;
#pragma unroll
          for (int x = 0; x < CW; x += 8) {
            float ov[8], ok8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              ov[e] = __uint_as_float(dvv[x + e]);
              ok8[e] = __uint_as_float(dkv[x + e]) * a.scale;
            }
            store_row8(a.dv, a.grad_fp32, cbase + c0 + x, ov);
            store_row8(a.dk, a.grad_fp32, cbase + c0 + x, ok8);
          }
        }
      } else {
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += CW) {
          uint32_t acc[CW];
          if (has_acc) {
            tmem_ld_n<CW>(t_a0 + c0, acc);
            tmem_wait_ld();
            reg_fence_n<CW>(acc);
            if (c0 + CW >= HD) {
              tc_fence_before();
              mbar_arrive(bars + 8 * C::B_ACCFREE);
            }
          } else {
#pragma unroll
            for (int x = 0; x < CW; ++x) acc[x] = 0u;
          }
          if (!row_ok) continue;
#pragma unroll
          for (int x = 0; x < CW; x += 8) {
            float kv8[8], o[8];
            unpack8(ld_global_nc_v4(a.k + cbase + c0 + x), kv8);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o[e] = a.scale * fmaf(dsd, kv8[e], __uint_as_float(acc[x + e]));
            store_row8(a.dq, a.grad_fp32, cbase + c0 + x, o);
            if (seg != 1) {
              // Candidate rows: their key and value are seen by themselves only. Padding rows:
              // pd = dsd = 0, so their gradients are written as 0.
              float qv8[8], dov8[8], dk8[8], dv8[8];
              unpack8(ld_global_nc_v4(a.q + cbase + c0 + x), qv8);
              unpack8(ld_global_nc_v4(a.dout + cbase + c0 + x), dov8);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                dk8[e] = a.scale * dsd * qv8[e];
                dv8[e] = pd * dov8[e];
              }
              store_row8(a.dk, a.grad_fp32, cbase + c0 + x, dk8);
              store_row8(a.dv, a.grad_fp32, cbase + c0 + x, dv8);
            }
          }
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Kernel
// ------------------------------------------------------------------------------------------
template <int D, int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    jagged_attn_bwd_kernel(const __grid_constant__ CUtensorMap tmO1,
                           const __grid_constant__ CUtensorMap tmO2,
                           const __grid_constant__ CUtensorMap tmI1,
                           const __grid_constant__ CUtensorMap tmI2, const BwdArgs a) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* skip = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    *skip = *a.status != 0;
    // Every barrier slot is initialised: the ones the compute warps arrive on count one arrival
    // per compute thread, all others (TMA transactions, MMA commits) one.
    for (int i = 0; i < C::NUM_BARS; ++i) {
      const bool by_compute = i == C::B_DSFULL || i == C::B_DSFULL + 1 || i == C::B_ACCFREE ||
                              i == C::B_COLS || i == C::B_COLS + 1;
      mbar_init(bars + 8 * i, by_compute ? kBwdCompute : 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmO1);
    tma_prefetch_map(&tmO2);
    tma_prefetch_map(&tmI1);
    tma_prefetch_map(&tmI2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = *a.n_items;
  if (!*skip) {
    if (warp == 0) {
      if (lane == 0)
        bwd_producer<D, MODE>(&tmO1, &tmO2, &tmI1, &tmI2, a, sbase, bars, n_items, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) bwd_mma<D, MODE>(a, sbase, bars, tmem, n_items, abort_flag);
    } else {
      bwd_compute<D, MODE>(a, bars, tmem, reinterpret_cast<float*>(smem + C::OFF_COLS), n_items,
                           abort_flag, warp, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// Per-row statistics: lse2 = lse * log2(e) (+inf for a row with no key) and D = rowsum(dO * O),
// both transposed to [H][T] so that a tile's 128 consecutive rows of one head are contiguous.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const void* __restrict__ out, int out_fp32,
                                                       const bf16* __restrict__ dout,
                                                       const float* __restrict__ lse, int64_t T,
                                                       int H, float* __restrict__ lse2,
                                                       float* __restrict__ dsum,
                                                       const int32_t* status) {
  if (*status != 0) return;
  const int64_t n = T * H;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / H;
    const int h = (int)(idx - row * H);
    const size_t base = (size_t)idx * D;
    const uint4* dp = reinterpret_cast<const uint4*>(dout + base);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      float g[8], o[8];
      unpack8(ld_global_nc_v4(dp + c), g);
      if (out_fp32) {
        const float4* op = reinterpret_cast<const float4*>(static_cast<const float*>(out) + base);
        const float4 a0 = op[2 * c], a1 = op[2 * c + 1];
        o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
        o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
      } else {
        unpack8(ld_global_nc_v4(reinterpret_cast<const uint4*>(static_cast<const bf16*>(out) +
                                                               base) + c), o);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(g[e], o[e], acc);
    }
    const float l = lse[idx];
    lse2[(size_t)h * T + row] = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
    dsum[(size_t)h * T + row] = acc;
  }
}

// ------------------------------------------------------------------------------------------
// Work queue of the dKV kernel: one item per (user, head, 128-key tile of the history interval),
// sorted by the number of the user's 128-row query tiles, largest first (counting sort in one
// block, as the forward's queue). Item = {first key row, (h << 9) | key rows, row start, row
// length}. With `coff` (the candidate-packed layout) the user's queries are its run
// [off[b], off[b+1]) plus its candidate run [cbase + coff[b], cbase + coff[b+1]), which goes to
// items2 = {row start, rows}.
// ------------------------------------------------------------------------------------------
template <typename IdxT>
__global__ void __launch_bounds__(1024) dkv_queue_kernel(const IdxT* __restrict__ off,
                                                         const IdxT* __restrict__ hlo,
                                                         const IdxT* __restrict__ hhi, int64_t B,
                                                         int H, int4* __restrict__ items,
                                                         int64_t max_items, int32_t* n_items,
                                                         int32_t* status,
                                                         const IdxT* __restrict__ coff,
                                                         int64_t cbase, int2* __restrict__ items2) {
  __shared__ unsigned long long s_cnt[kQueueBuckets];
  __shared__ unsigned long long s_cursor[kQueueBuckets];
  __shared__ unsigned long long s_warp[32];
  __shared__ unsigned long long s_total;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (*status != 0) {
    if (tid == 0) *n_items = 0;
    return;
  }
  for (int i = tid; i < kQueueBuckets; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  for (int64_t b = tid; b < B; b += blockDim.x) {
    const long long nk = ((long long)hhi[b] - (long long)hlo[b] + kTileN - 1) / kTileN;
    long long nq = ((long long)off[b + 1] - (long long)off[b] + kTileM - 1) / kTileM;
    if (coff) nq += ((long long)coff[b + 1] - (long long)coff[b] + kTileM - 1) / kTileM;
    const int key = (int)min(nq, (long long)(kQueueBuckets - 1));
    if (nk) atomicAdd(&s_cnt[key], (unsigned long long)(nk * H));
  }
  __syncthreads();
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
      atomicCAS(status, 0, (int32_t)JCA_STATUS_QUEUE_OVERFLOW);
      *n_items = 0;
    }
    return;
  }
  const int nwarps = blockDim.x >> 5;
  for (int64_t b = wid; b < B; b += nwarps) {
    const long long lo = (long long)hlo[b], hi = (long long)hhi[b];
    const long long s = (long long)off[b], e = (long long)off[b + 1];
    const long long nk = (hi - lo + kTileN - 1) / kTileN;
    if (nk == 0) continue;
    long long nq = (e - s + kTileM - 1) / kTileM;
    long long c0 = 0, c1 = 0;
    if (coff) {
      c0 = cbase + (long long)coff[b];
      c1 = cbase + (long long)coff[b + 1];
      nq += (c1 - c0 + kTileM - 1) / kTileM;
    }
    const int key = (int)min(nq, (long long)(kQueueBuckets - 1));
    unsigned long long pos = 0;
    if (lane == 0) pos = atomicAdd(&s_cursor[key], (unsigned long long)(nk * H));
    pos = __shfl_sync(0xffffffffu, pos, 0);
    for (long long i = lane; i < nk * H; i += 32) {
      const int h = (int)(i / nk);
      const long long t = i - (long long)h * nk;
      const long long k0 = lo + t * kTileN;
      const int rows = (int)min((long long)kTileN, hi - k0);
      items[pos + (unsigned long long)i] = make_int4((int)k0, (h << 9) | rows, (int)s, (int)(e - s));
      if (items2) items2[pos + (unsigned long long)i] = make_int2((int)c0, (int)(c1 - c0));
    }
  }
  if (tid == 0) *n_items = (int32_t)s_total;
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
// Kernel attributes set so far, per device, head size and mode.
constexpr int kMaxDevices = 64;
bool g_bwd_attr[kMaxDevices][4][2];
std::mutex g_bwd_mu;

int d_slot(int d) { return d == 16 ? 0 : d == 32 ? 1 : d == 64 ? 2 : 3; }

template <int D, int MODE>
int launch_bwd_mode(const BwdArgs& a, const void* o1, const void* o2, const void* i1,
                    const void* i2, int64_t T, cudaStream_t stream) {
  using C = BCfg<D>;
  int dev = 0, sms = 0;
  const int rc = current_device(&dev, &sms);
  if (rc) return rc;
  {
    std::lock_guard<std::mutex> lock(g_bwd_mu);
    if (!g_bwd_attr[dev][d_slot(D)][MODE]) {
      if (cudaFuncSetAttribute(jagged_attn_bwd_kernel<D, MODE>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess)
        return JCA_ERR_CUDA;
      g_bwd_attr[dev][d_slot(D)][MODE] = true;
    }
  }
  CUtensorMap m1, m2, m3, m4;
  if (!make_rows_map_bf16(&m1, o1, T, a.H, D, C::BM) ||
      !make_rows_map_bf16(&m2, o2, T, a.H, D, C::BM) ||
      !make_rows_map_bf16(&m3, i1, T, a.H, D, C::BM) ||
      !make_rows_map_bf16(&m4, i2, T, a.H, D, C::BM))
    return JCA_ERR_CUDA;
  jagged_attn_bwd_kernel<D, MODE><<<sms, kBwdThreads, C::SMEM_ALLOC, stream>>>(m1, m2, m3,
                                                                                      m4, a);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

// Workspace of the backward pass: the forward's plan (segment IDs, bounds, dQ work queue), then
// the dKV queue (with its second query runs for the candidate-packed layout) and the transposed
// row statistics.
struct BwdLayout {
  size_t plan = 0, dkv_items = 0, dkv_items2 = 0, dkv_n = 0, lse2 = 0, dsum = 0, total = 0;
  int64_t dkv_max = 0;
};

// plan_bytes: size of the forward plan at the start of the workspace; key_rows: rows that can hold
// history keys (T, or Th for the candidate-packed layout).
BwdLayout bwd_layout_after(size_t plan_bytes, int64_t B, int64_t T, int64_t key_rows, int H,
                           bool runs2) {
  BwdLayout L;
  size_t o = align_up(plan_bytes, 256);
  L.plan = 0;
  L.dkv_max = (key_rows / kTileN + B + 1) * (int64_t)H;
  L.dkv_items = o;
  o = align_up(o + 16 * (size_t)L.dkv_max, 256);
  if (runs2) {
    L.dkv_items2 = o;
    o = align_up(o + 8 * (size_t)L.dkv_max, 256);
  }
  L.dkv_n = o;
  o = align_up(o + 16, 256);
  L.lse2 = o;
  o = align_up(o + 4 * (size_t)T * H, 256);
  L.dsum = o;
  o = align_up(o + 4 * (size_t)T * H, 256);
  L.total = o;
  return L;
}

BwdLayout bwd_layout(int64_t B, int64_t T, int H) {
  return bwd_layout_after(workspace_layout(B, T, H).total, B, T, T, H, false);
}

template <int D>
int launch_backward(const BwdArgs& base_args, const void* out, int out_fp32, const float* lse,
                    int64_t T, void* ws, const WorkspaceLayout& W, const BwdLayout& L,
                    cudaStream_t st, bool runs2 = false) {
  char* w = static_cast<char*>(ws);
  const int64_t n = T * base_args.H;
  const int64_t want = (n + 255) / 256;
  const int grid = (int)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  bwd_prep_kernel<D><<<grid, 256, 0, st>>>(out, out_fp32, base_args.dout, lse, T, base_args.H,
                                           reinterpret_cast<float*>(w + L.lse2),
                                           reinterpret_cast<float*>(w + L.dsum),
                                           base_args.status);
  if (cudaGetLastError() != cudaSuccess) return JCA_ERR_CUDA;
  BwdArgs a = base_args;
  a.lse2 = reinterpret_cast<const float*>(w + L.lse2);
  a.dsum = reinterpret_cast<const float*>(w + L.dsum);
  // Keys of segment 1: dK, dV.
  a.items = reinterpret_cast<const int4*>(w + L.dkv_items);
  a.items2 = runs2 ? reinterpret_cast<const int2*>(w + L.dkv_items2) : nullptr;
  a.n_items = reinterpret_cast<const int32_t*>(w + L.dkv_n);
  int rc = launch_bwd_mode<D, kModeDKV>(a, a.k, a.v, a.q, a.dout, T, st);
  if (rc) return rc;
  // Every query: dQ, plus dK, dV of the other rows (candidates' diagonal terms; padding zeros).
  a.items2 = nullptr;
  a.items = reinterpret_cast<const int4*>(w + W.items);
  a.n_items = reinterpret_cast<const int32_t*>(w + W.n_items);
  return launch_bwd_mode<D, kModeDQ>(a, a.q, a.dout, a.k, a.v, T, st);
}

}  // namespace
}  // namespace jca

using namespace jca;

extern "C" size_t jca_bwd_workspace_bytes(int64_t B, int64_t T, int H, int d_head) {
  if (B < 0 || T < 0 || H < 1 || !head_dim_ok(d_head)) return 0;
  return bwd_layout(B, T, H).total;
}

extern "C" int jagged_cand_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                                    int out_fp32, const void* dout, const float* lse, void* dq,
                                    void* dk, void* dv, int grad_fp32, const void* offsets,
                                    const void* candidate_start, const int8_t* seg, int64_t B,
                                    int64_t T, int H, int d_head, float scale, int idx_bits,
                                    void* workspace, size_t workspace_bytes, int32_t* status,
                                    jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (B < 0 || T < 0 || H < 1 || H >= 65536 || T >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX ||
      (B == 0 && T != 0))
    return JCA_ERR_SHAPE;
  if (!status || !offsets || !workspace) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv))
    return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
                !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
                !aligned(lse, 4)))
    return JCA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  const BwdLayout L = bwd_layout(B, T, H);
  if (workspace_bytes < L.total) return JCA_ERR_WORKSPACE;
  if (T == 0) return JCA_OK;
  const WorkspaceLayout W = workspace_layout(B, T, H);
  int rc = jagged_cand_attn_plan(offsets, candidate_start, seg, B, T, H, d_head, idx_bits,
                                 workspace, W.total, status, stream);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  if (idx_bits == 32)
    dkv_queue_kernel<int32_t><<<1, kQueueBuckets, 0, st>>>(
        (const int32_t*)offsets, (const int32_t*)(w + W.hist_lo), (const int32_t*)(w + W.hist_hi),
        B, H, reinterpret_cast<int4*>(w + L.dkv_items), L.dkv_max,
        reinterpret_cast<int32_t*>(w + L.dkv_n), status, nullptr, 0, nullptr);
  else
    dkv_queue_kernel<int64_t><<<1, kQueueBuckets, 0, st>>>(
        (const int64_t*)offsets, (const int64_t*)(w + W.hist_lo), (const int64_t*)(w + W.hist_hi),
        B, H, reinterpret_cast<int4*>(w + L.dkv_items), L.dkv_max,
        reinterpret_cast<int32_t*>(w + L.dkv_n), status, nullptr, 0, nullptr);
  if (cudaGetLastError() != cudaSuccess) return JCA_ERR_CUDA;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_head);
  BwdArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k = static_cast<const bf16*>(k);
  a.v = static_cast<const bf16*>(v);
  a.dout = static_cast<const bf16*>(dout);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.seg = seg ? seg : reinterpret_cast<const int8_t*>(w + W.seg);
  a.lse2 = nullptr;
  a.dsum = nullptr;
  a.items = nullptr;
  a.items2 = nullptr;
  a.n_items = nullptr;
  a.status = status;
  a.T = T;
  a.H = H;
  a.grad_fp32 = grad_fp32 ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  switch (d_head) {
    case 16: return launch_backward<16>(a, out, out_fp32, lse, T, workspace, W, L, st);
    case 32: return launch_backward<32>(a, out, out_fp32, lse, T, workspace, W, L, st);
    case 64: return launch_backward<64>(a, out, out_fp32, lse, T, workspace, W, L, st);
    default: return launch_backward<128>(a, out, out_fp32, lse, T, workspace, W, L, st);
  }
}

extern "C" size_t jca_seqpack_bwd_workspace_bytes(int64_t B, int64_t Th, int64_t Nc, int H,
                                                  int d_head) {
  if (B < 0 || Th < 0 || Nc < 0 || H < 1 || !head_dim_ok(d_head)) return 0;
  const SeqpackLayout S = seqpack_layout(B, Th + Nc, H);
  return bwd_layout_after(S.total, B, Th + Nc, Th, H, true).total;
}

extern "C" int jagged_cand_attn_seqpack_bwd(
    const void* q, const void* k, const void* v, const void* out, int out_fp32, const void* dout,
    const float* lse, void* dq, void* dk, void* dv, int grad_fp32, const void* hist_offsets,
    const void* cand_offsets, const int8_t* seg, int64_t B, int64_t Th, int64_t Nc, int H,
    int d_head, float scale, int idx_bits, void* workspace, size_t workspace_bytes,
    int32_t* status, jca_stream_t stream) {
  if (idx_bits != 32 && idx_bits != 64) return JCA_ERR_IDX_BITS;
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  const int64_t T = Th + Nc;
  if (B < 0 || Th < 0 || Nc < 0 || H < 1 || H >= 65536 || T >= (int64_t)INT_MAX ||
      2 * B >= (int64_t)INT_MAX || (B == 0 && T != 0))
    return JCA_ERR_SHAPE;
  if (!status || !hist_offsets || !cand_offsets || !workspace) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv))
    return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
                !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
                !aligned(lse, 4)))
    return JCA_ERR_ALIGN;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  const SeqpackLayout S = seqpack_layout(B, T, H);
  if (S.base.max_items >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  const BwdLayout L = bwd_layout_after(S.total, B, T, Th, H, true);
  if (workspace_bytes < L.total) return JCA_ERR_WORKSPACE;
  if (T == 0) return JCA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  if (launch_seqpack_plan(hist_offsets, cand_offsets, seg, B, Th, Nc, H, idx_bits, w, S.base,
                          S.q_off2, status, st) != cudaSuccess)
    return JCA_ERR_CUDA;
  // dK, dV of each history key tile come from the user's history run and its candidate run.
  if (idx_bits == 32)
    dkv_queue_kernel<int32_t><<<1, kQueueBuckets, 0, st>>>(
        (const int32_t*)hist_offsets, (const int32_t*)(w + S.base.hist_lo),
        (const int32_t*)(w + S.base.hist_hi), B, H, reinterpret_cast<int4*>(w + L.dkv_items),
        L.dkv_max, reinterpret_cast<int32_t*>(w + L.dkv_n), status,
        (const int32_t*)cand_offsets, Th, reinterpret_cast<int2*>(w + L.dkv_items2));
  else
    dkv_queue_kernel<int64_t><<<1, kQueueBuckets, 0, st>>>(
        (const int64_t*)hist_offsets, (const int64_t*)(w + S.base.hist_lo),
        (const int64_t*)(w + S.base.hist_hi), B, H, reinterpret_cast<int4*>(w + L.dkv_items),
        L.dkv_max, reinterpret_cast<int32_t*>(w + L.dkv_n), status,
        (const int64_t*)cand_offsets, Th, reinterpret_cast<int2*>(w + L.dkv_items2));
  if (cudaGetLastError() != cudaSuccess) return JCA_ERR_CUDA;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_head);
  BwdArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k = static_cast<const bf16*>(k);
  a.v = static_cast<const bf16*>(v);
  a.dout = static_cast<const bf16*>(dout);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.seg = seg ? seg : reinterpret_cast<const int8_t*>(w + S.base.seg);
  a.lse2 = nullptr;
  a.dsum = nullptr;
  a.items = nullptr;
  a.items2 = nullptr;
  a.n_items = nullptr;
  a.status = status;
  a.T = T;
  a.H = H;
  a.grad_fp32 = grad_fp32 ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  switch (d_head) {
    case 16: return launch_backward<16>(a, out, out_fp32, lse, T, workspace, S.base, L, st, true);
    case 32: return launch_backward<32>(a, out, out_fp32, lse, T, workspace, S.base, L, st, true);
    case 64: return launch_backward<64>(a, out, out_fp32, lse, T, workspace, S.base, L, st, true);
    default: return launch_backward<128>(a, out, out_fp32, lse, T, workspace, S.base, L, st, true);
  }
}
