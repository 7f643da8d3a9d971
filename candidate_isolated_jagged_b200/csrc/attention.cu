// Jagged candidate-isolated attention on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (候选隔离注意力掩码, sections 段 ID：掩码的表达方式 and 掩码长什么样): every
// non-padding query of user b attends to the segment-1 keys of its own row (prefix + history),
// and each candidate also attends to itself; padding queries output 0. The mask is never
// materialised: per user, the keys a query can see (besides itself) are exactly the segment-1
// positions inside [hist_lo, hist_hi), so the work of a user is a dense, non-causal rectangle of
// (row tiles) x (history key tiles). Key tiles over the candidate range are never visited
// (history x candidate and candidate x other-candidate pairs are skipped wholesale), and the
// candidate's self term is merged into the online softmax as a diagonal epilogue on CUDA cores.
//
// Kernel structure (one persistent CTA per SM, 12 warps). A work item is a block of up to 256 query
// rows of one (user, head): two 128-row query tiles A and B that share every K/V tile load.
//   warp 0       two TMA producer threads: lane 0 claims the CTA's items and loads their Q tiles
//                and the K tiles, lane 1 loads the V tiles (rings of stages).
//   warp 1       TMEM allocator and single-thread MMA issuer.
//   warps 2..9   two softmax warpgroups, one per query tile, one query row per thread (TMEM lane =
//                row). Each group owns an S buffer in TMEM (P is written back over S as bf16 pairs
//                and read from there by the PV MMA), an fp32 O accumulator and its rows' running
//                max / sum, and finalises its own rows (diagonal term, 1/l, store).
//   warps 10..11 diagonal scores of candidate rows, one item ahead of the softmax warps.
// TMEM columns: S_A | S_B | O_A | O_B (128 each). MMA order per key tile j, one stream over all the
// CTA's items:
//   QK_A(j), PV_B(j-1), QK_B(j), PV_A(j)
// so each group's chain (softmax -> PV -> next QK) is short and the tensor core works for one
// group while the other runs its softmax. An MMA that overwrites S_w is issued after the PV that
// reads the P stored there, and MMAs from one thread execute in issue order; a commit fires only
// when every earlier MMA has completed, so once a group sees S_w full its previous PV into O_w is
// done and O_w may be rescaled in place.
// Work items (user, head, 256-row query block) come from the cost-sorted queue and are claimed at
// run time from a global counter, so the longest items start first and a CTA that finishes early
// takes the next one; the claiming thread passes each item's descriptor to every role through a
// shared ring. Heads of up to 32 release each key tile's P to the MMA thread in two halves, so
// that the first half of the PV overlaps the softmax of the second. The kernel is instantiated
// per mode: the main path, the per-user causal variant (CAUSAL), the training forward that also
// writes each row's log-sum-exp (LSE), the in-kernel RoPE rotation (ROPE), and the candidate-only
// layer with heads of 64 or more (DT), where every row is a candidate: there each query tile's own
// keys and values arrive as TMA tiles and go through the tensor core as one more "diagonal" key
// step after the history tiles (QK against the own keys, of which each row keeps its own score;
// P zero off the diagonal; PV against the own values), instead of per-row loads on CUDA cores;
// the diagonal warps then only follow the item ring.
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "jca_device.cuh"
#include "jca_internal.h"
#include "rope_device.cuh"

namespace jca {
namespace {

struct AttnArgs {
  const __nv_bfloat16* q;   // [Tq, H, D] query rows (read again for the diagonal term)
  const __nv_bfloat16* dk;  // [Tq, H, D] diagonal keys: the query row's own key
  const __nv_bfloat16* dv;  // [Tq, H, D] diagonal values
  const int8_t* q_seg;      // [Tq] segment of each query row, or null = every row is a candidate
  const int8_t* kv_seg;     // [Tkv] segment of each key row (read only for users with holes)
  void* out;                // [Tq, H, D] bf16 or fp32
  const int4* items;
  const int32_t* n_items;
  int32_t* queue;           // [2]: next item to claim, CTAs finished
  int32_t* status;
  int H;
  int out_fp32;
  int out_v8;               // out is 32-byte aligned: rows are written with 32-byte stores
  float scale_log2;         // softmax scale * log2(e)
  float* lse = nullptr;     // [Tq, H] natural-log softmax denominators, or null (not written);
                            // non-null selects the LSE instantiation of the kernel
  int causal = 0;           // per-user causal variant: row i sees the keys j <= i of its user,
                            // no candidate or padding rows (items come from the causal queue);
                            // selects the CAUSAL instantiation of the kernel
  // Right-anchored RoPE applied inside the kernel (the ROPE instantiation): every Q and K tile is
  // rotated in shared memory after it lands and before the tensor core reads it.
  const int32_t* q_pos = nullptr;      // [Tq] position of each query row
  const int32_t* kv_pos = nullptr;     // [Tkv] position of each key row
  const float2* rope_coarse = nullptr; // [n_coarse][D/2] (cos, sin)(128 (qmax - i) theta_j)
  const float2* rope_fine = nullptr;   // [128][D/2] (cos, sin)(r theta_j)
  long long rope_qmax = 0;
  int rope = 0;                        // selects the ROPE instantiation
};

// Depth of the shared ring through which every role receives the claimed work items.
constexpr int kRing = 4;

template <int D>
struct Cfg {
  static constexpr int BM = kTileM;
  static constexpr int BN = kTileN;
  static constexpr int ROW_BYTES = D * 2;                          // one head of one token
  static constexpr int SW = ROW_BYTES >= 128 ? 128 : ROW_BYTES;    // swizzle span (bytes)
  static constexpr int NBLK = ROW_BYTES / SW;                      // column blocks per tile
  static constexpr int BOX_X = SW / 2;                             // elements per TMA box row
  static constexpr int TILE_BYTES = BM * ROW_BYTES;
  static constexpr int BLK_BYTES = BM * SW;
  static constexpr uint32_t LAYOUT = SW == 128 ? 2u : (SW == 64 ? 4u : 6u);
  static constexpr int KSTEPS_QK = D / 16;
  static constexpr int KSTEPS_PER_BLK = SW / 32;
  static constexpr int KSTEPS_PV = BN / 16;
  // Heads of up to 32: P of a key tile is released to the MMA thread in two halves (keys 0..63,
  // then the rest), so the first half of the PV runs while the softmax computes the second. At
  // d = 32 a PV is eight MMAs of N = 32, whose issue takes about as long as the softmax half
  // (retrieval 0.358 -> 0.338 ms); at d = 128 the extra barrier round trip costs more than it
  // hides (users256 0.70 -> 0.76 ms), so larger heads release P whole.
  static constexpr bool SPLIT_P = D <= 32;
  static constexpr int PV_FIRST = KSTEPS_PV / 2;                 // k-steps of the first half
  // Ring depths: query-tile buffers per group and K / V stages. Small heads make short items
  // (a few key tiles) whose loads must be issued an item ahead to hide HBM latency; their tiles are
  // small, so the rings are deeper there. D = 128 fills shared memory with one Q buffer per group.
  static constexpr int QS = D >= 128 ? 1 : (D == 64 ? 2 : 4);
  static constexpr int KVS = D >= 128 ? 2 : (D == 64 ? 3 : 4);
  static constexpr int OFF_Q = 0;                          // [group][QS] tiles
  static constexpr int OFF_K = OFF_Q + 2 * QS * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KVS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + KVS * TILE_BYTES;
  // Barrier slots.
  static constexpr int B_QFULL = 0;                        // [group][QS]
  static constexpr int B_QEMPTY = B_QFULL + 2 * QS;        // [group][QS]
  static constexpr int B_KFULL = B_QEMPTY + 2 * QS;        // [KVS]
  static constexpr int B_KEMPTY = B_KFULL + KVS;
  static constexpr int B_VFULL = B_KEMPTY + KVS;
  static constexpr int B_VEMPTY = B_VFULL + KVS;
  static constexpr int B_SFULL = B_VEMPTY + KVS;           // [group]: S_w written by a QK
  static constexpr int B_PFULL = B_SFULL + 2;              // [group]: P_w written, S_w read
  static constexpr int B_OREADY = B_PFULL + 2;             // [group]: item's last PV complete
  static constexpr int B_OFREE = B_OREADY + 2;             // [group]: O_w read by the group
  static constexpr int B_DRAIN = B_OFREE + 2;
  static constexpr int B_DIAGFULL = B_DRAIN + 1;           // [slot]: scores written
  static constexpr int B_DIAGEMPTY = B_DIAGFULL + 2;       // [slot]: scores taken
  static constexpr int B_RINGFULL = B_DIAGEMPTY + 2;       // [kRing]: claimed item index written
  static constexpr int B_RINGEMPTY = B_RINGFULL + kRing;   // [kRing]: index read by every role
  // ROPE instantiation: a landed Q / K tile has been rotated in place (the MMA waits on these
  // instead of the TMA's full barriers).
  static constexpr int B_QREADY = B_RINGEMPTY + kRing;     // [group][QS]
  static constexpr int B_KREADY = B_QREADY + 2 * QS;       // [KVS]
  // [group]: keys 0..63 of P_w written (SPLIT_P: the PV may start on them).
  static constexpr int B_PHALF = B_KREADY + KVS;
  static constexpr int NUM_BARS = B_PHALF + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // Diagonal scores of the candidate rows: two item slots of kItemRows floats.
  static constexpr int OFF_RING = OFF_MISC + 16;           // kRing claimed item descriptors
  static constexpr int OFF_DIAG = OFF_RING + 16 * kRing;
  static constexpr int SMEM_USED = OFF_DIAG + 2 * kItemRows * 4;
  static constexpr int SMEM_RAW = SMEM_USED + 1024;                // slack for 1 KB alignment
  // At least 120 KB so that a second CTA never shares the SM (and its TMEM).
  static constexpr int SMEM_ALLOC = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
  // TMEM columns: S_A | S_B (fp32 scores, then bf16 P over their first 64 columns) | O_A | O_B.
  static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 384,
                            TMEM_COLS = 512;
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
};

// Warps: 0 TMA producers, 1 TMEM allocator + MMA issuer, 2..9 softmax/epilogue, 10..11 diagonal
// scores. Softmax warp w belongs to group (w - 2) / 4 (query tile A or B) and owns TMEM lane
// quarter w % 4 (rows 32 (w % 4) .. +31 of its tile).
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
constexpr int kDiagThreads = 64;
// Readers of the item ring: V producer lane, MMA thread, softmax and diagonal threads.
constexpr int kRingReaders = 1 + 1 + kSoftmaxThreads + kDiagThreads;

struct Item {
  int q_row0, h, nrows, kv_lo, kv_len, holes, n_kv;
};

__device__ __forceinline__ Item decode_item(int4 v) {
  Item w;
  w.q_row0 = v.x;
  w.h = v.y >> 9;
  w.nrows = v.y & 511;
  w.kv_lo = v.z;
  w.kv_len = v.w & 0x7fffffff;
  w.holes = (int)((unsigned)v.w >> 31);
  w.n_kv = (w.kv_len + kTileN - 1) / kTileN;
  return w;
}

// Work items are claimed at run time from a global counter, so that a CTA that finishes early
// takes the next item (the queue is sorted by cost, largest first). The claiming thread (producer
// lane 0) reads each claimed item's descriptor from the queue and writes it (or an end marker once
// the queue is exhausted) into a shared ring; every other role reads the same sequence of
// descriptors from the ring and releases each slot after reading it. The claimer runs up to kRing
// items ahead, so no role waits on the global queue at an item boundary.
struct ItemRing {
  volatile int* slot;   // kRing shared entries of 4 ints (the item descriptor)
  uint32_t full;        // address of full barrier 0 (kRing consecutive barriers)
  uint32_t empty;       // address of empty barrier 0
  uint32_t k;           // entries taken so far
};

constexpr int kEndOfQueue = -1;   // q_row0 of the end marker (real items start at row >= 0)

__device__ __forceinline__ int4 ring_claim(ItemRing& r, const int4* items, int32_t* head,
                                           int n_items, volatile int* abort_flag, int32_t* status,
                                           bool& ok) {
  const int s = (int)(r.k % kRing);
  ok = mbar_wait(r.empty + 8 * s, ((r.k / kRing) & 1) ^ 1, abort_flag, status);
  if (!ok) return make_int4(kEndOfQueue, 0, 0, 0);
  const int v = atomicAdd(head, 1);
  const int4 d = v < n_items ? items[v] : make_int4(kEndOfQueue, 0, 0, 0);
  r.slot[4 * s + 0] = d.x;
  r.slot[4 * s + 1] = d.y;
  r.slot[4 * s + 2] = d.z;
  r.slot[4 * s + 3] = d.w;
  mbar_arrive(r.full + 8 * s);
  ++r.k;
  return d;
}

// Every thread of a consuming role calls this (warps stay converged: `ok` is made warp-uniform
// by the caller where warp-collective operations follow).
__device__ __forceinline__ int4 ring_take(ItemRing& r, volatile int* abort_flag, int32_t* status,
                                          bool& ok) {
  const int s = (int)(r.k % kRing);
  ok = mbar_wait(r.full + 8 * s, (r.k / kRing) & 1, abort_flag, status);
  if (!ok) return make_int4(kEndOfQueue, 0, 0, 0);
  const int4 d = make_int4(r.slot[4 * s + 0], r.slot[4 * s + 1], r.slot[4 * s + 2],
                           r.slot[4 * s + 3]);
  mbar_arrive(r.empty + 8 * s);
  ++r.k;
  return d;
}

// ------------------------------------------------------------------------------------------
// Producer
// ------------------------------------------------------------------------------------------
// Two producer threads in warp 0 walk the same item sequence: lane 0 loads the Q tiles (a ring of
// QS buffers per query tile, each refilled once the last QK of the item that used it completed)
// and the K tiles (stages freed by QK completions), lane 1 loads the V tiles (stages freed by PV
// completions), so a slow PV never holds back the next K. With DT each item also gets its query
// tiles' own keys (lane 0) and values (lane 1), one stage per query tile, after its key tiles.
template <int D, bool DT>
__device__ void producer_role(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                              const CUtensorMap* tmV, const CUtensorMap* tmDK,
                              const CUtensorMap* tmDV, const AttnArgs& a, uint32_t sbase,
                              uint32_t bars, int n_items, volatile int* abort_flag, bool loads_v,
                              ItemRing ring) {
  using C = Cfg<D>;
  uint32_t nq[2] = {0, 0};   // Q loads per query tile
  uint32_t g = 0;            // K (or V) loads
  bool ok = true;
  for (;;) {
    // Lane 0 claims the CTA's next item; lane 1 reads the claims from the ring.
    const int4 desc = loads_v ? ring_take(ring, abort_flag, a.status, ok)
                              : ring_claim(ring, a.items, a.queue, n_items, abort_flag, a.status, ok);
    if (!ok || desc.x == kEndOfQueue) break;
    const Item w = decode_item(desc);
    if (!DT && w.n_kv == 0) continue;
    const int empty = loads_v ? C::B_VEMPTY : C::B_KEMPTY;
    const int full = loads_v ? C::B_VFULL : C::B_KFULL;
    const CUtensorMap* map = loads_v ? tmV : tmK;
    const int off = loads_v ? C::OFF_V : C::OFF_K;
    auto load_kv = [&](int j) -> bool {
      const int s = (int)(g % C::KVS);
      const uint32_t ph = (g / C::KVS) & 1;
      const int row = w.kv_lo + j * C::BN;
      if (!mbar_wait(bars + 8 * (empty + s), ph ^ 1, abort_flag, a.status)) return false;
      mbar_arrive_expect_tx(bars + 8 * (full + s), C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < C::NBLK; ++c)
        tma_load_3d(sbase + off + s * C::TILE_BYTES + c * C::BLK_BYTES, map,
                    bars + 8 * (full + s), c * C::BOX_X, w.h, row);
      ++g;
      return true;
    };
    int j0 = 0;
    if (!loads_v) {
      // The item's first K tile goes out before its Q tiles: its stage was freed by a QK of the
      // previous item's second-to-last key tile, while the Q buffers wait for the last, so the
      // load is issued a key tile earlier and lands before the item's first QK needs it
      // (users256 0.714 -> 0.702 ms). Every earlier K tile's item had its Q tiles issued by
      // then, so no release this wait depends on is held up by it.
      if (!DT || w.n_kv > 0) {
        ok = load_kv(0);
        if (!ok) break;
        j0 = 1;
      }
      const int ntiles = w.nrows > C::BM ? 2 : 1;
      for (int t = 0; ok && t < ntiles; ++t) {
        // Load n of a buffer waits for the release of load n - 1 (immediate the first time).
        const int slot = t * C::QS + (int)(nq[t] % C::QS);
        ok = mbar_wait(bars + 8 * (C::B_QEMPTY + slot), ((nq[t] / C::QS) & 1) ^ 1, abort_flag,
                       a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bars + 8 * (C::B_QFULL + slot), C::TILE_BYTES);
        ++nq[t];
#pragma unroll
        for (int c = 0; c < C::NBLK; ++c)
          tma_load_3d(sbase + C::OFF_Q + slot * C::TILE_BYTES + c * C::BLK_BYTES, tmQ,
                      bars + 8 * (C::B_QFULL + slot), c * C::BOX_X, w.h, w.q_row0 + t * C::BM);
      }
      if (!ok) break;
    }
    for (int j = j0; j < w.n_kv; ++j) {
      ok = load_kv(j);
      if (!ok) break;
    }
    if (DT && ok) {
      // Diagonal step: each query tile's own keys (lane 0) or values (lane 1), one stage each,
      // in the order the MMA thread consumes the stages (tile A's, then tile B's).
      const CUtensorMap* dmap = loads_v ? tmDV : tmDK;
      const int ntiles = w.nrows > C::BM ? 2 : 1;
      for (int t = 0; t < ntiles; ++t) {
        const int s = (int)(g % C::KVS);
        const uint32_t ph = (g / C::KVS) & 1;
        ok = mbar_wait(bars + 8 * (empty + s), ph ^ 1, abort_flag, a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bars + 8 * (full + s), C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::NBLK; ++c)
          tma_load_3d(sbase + off + s * C::TILE_BYTES + c * C::BLK_BYTES, dmap,
                      bars + 8 * (full + s), c * C::BOX_X, w.h, w.q_row0 + t * C::BM);
        ++g;
      }
    }
  }
  if (!ok) {
    // Aborting: let every copy this thread started land before the CTA exits. Load n of a slot
    // completes phase n of its full barrier; the last one issued is the newest.
    if (!loads_v) {
      for (int t = 0; t < 2; ++t)
        for (uint32_t n = nq[t] > (uint32_t)C::QS ? nq[t] - C::QS : 0; n < nq[t]; ++n)
          mbar_wait_drain(bars + 8 * (C::B_QFULL + t * C::QS + (int)(n % C::QS)),
                          (n / C::QS) & 1);
    }
    const int full = loads_v ? C::B_VFULL : C::B_KFULL;
    for (uint32_t n = g > (uint32_t)C::KVS ? g - C::KVS : 0; n < g; ++n)
      mbar_wait_drain(bars + 8 * (full + (int)(n % C::KVS)), (n / C::KVS) & 1);
  }
}

// ------------------------------------------------------------------------------------------
// MMA issuer
// ------------------------------------------------------------------------------------------
struct MmaState {
  uint32_t p_seen[2];   // P-full completions consumed, per softmax group
  uint32_t o_items[2];  // items whose O_w was written, per group (O-free completions expected)
  uint32_t q_seen[2];   // Q-full completions consumed, per query tile
  uint32_t v_seen;      // global key tiles whose V stage was seen full (the second PV skips it)
  // Operand descriptors of Q buffer 0 and of K / V stage 0 (start address of the first k-step);
  // a buffer, stage or k-step adds an offset to the low bits (shared addresses stay below 256 KB,
  // so the 14-bit field never carries).
  uint64_t q, k, v;
};

// Tensor-core issue is paced by execution (one 128x128x16 MMA takes about 64 cycles), so the issue
// paths below keep the work between two MMAs minimal: precomputed descriptors, compile-time
// offsets, and straight-line code for full tiles.
template <int D>
__device__ __forceinline__ void mma_qk(uint32_t d_tmem, uint64_t qa, uint64_t kb, uint32_t idesc) {
  using C = Cfg<D>;
#pragma unroll
  for (int kk = 0; kk < C::KSTEPS_QK; ++kk) {
    const uint32_t off = ((kk / C::KSTEPS_PER_BLK) * C::BLK_BYTES +
                          (kk % C::KSTEPS_PER_BLK) * 32) >> 4;
    tc_mma(d_tmem, qa + off, kb + off, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t vb, int ksteps,
                                       bool overwrite) {
  using C = Cfg<D>;
  constexpr uint32_t kIdescPV = idesc_bf16_f32(C::BM, D, false, true);
  constexpr uint32_t kStep = (16 * C::SW) >> 4;   // 16 key rows of V per k-step
  if (ksteps == C::KSTEPS_PV) {
#pragma unroll
    for (int kk = 0; kk < C::KSTEPS_PV; ++kk)
      tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, vb + (uint64_t)(kk * kStep), kIdescPV,
                (overwrite && kk == 0) ? 0u : 1u);
  } else {
    for (int kk = 0; kk < ksteps; ++kk)
      tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, vb + (uint64_t)(kk * kStep), kIdescPV,
                (overwrite && kk == 0) ? 0u : 1u);
  }
}

// k-steps [k0, k1) of O_w += P_w V (SPLIT_P halves); a range of N k-steps is straight-line code.
template <int D, int N>
__device__ __forceinline__ void mma_pv_range(uint32_t o_tmem, uint32_t p_tmem, uint64_t vb, int k0,
                                             int k1, bool overwrite) {
  using C = Cfg<D>;
  constexpr uint32_t kIdescPV = idesc_bf16_f32(C::BM, D, false, true);
  constexpr uint32_t kStep = (16 * C::SW) >> 4;   // 16 key rows of V per k-step
  if (k1 - k0 == N) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int kk = k0 + i;
      tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, vb + (uint64_t)(kk * kStep), kIdescPV,
                (overwrite && i == 0) ? 0u : 1u);
    }
  } else {
    for (int kk = k0; kk < k1; ++kk)
      tc_mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8u, vb + (uint64_t)(kk * kStep), kIdescPV,
                (overwrite && kk == k0) ? 0u : 1u);
  }
}

// O_w += P_w V for key tile jj of the item (global tile gg: V stage), whose first `valid` keys are
// real: only ceil(valid / 16) k-steps are issued. P_w is read from the first 64 TMEM columns of
// S_w (bf16 pairs: 16 keys = 8 columns per k-step). The first PV of an item overwrites O_w, so it
// waits until the group has read the previous item's O_w.
template <int D>
__device__ __forceinline__ bool issue_pv(int grp, uint32_t gg, int jj, int valid, MmaState& st,
                                         uint32_t bars, uint32_t tmem, const AttnArgs& a,
                                         volatile int* abort_flag) {
  using C = Cfg<D>;
  const int s = (int)(gg % C::KVS);
  if (gg + 1 != st.v_seen) {
    if (!mbar_wait(bars + 8 * (C::B_VFULL + s), (gg / C::KVS) & 1, abort_flag, a.status))
      return false;
    st.v_seen = gg + 1;
  }
  const uint32_t par = st.p_seen[grp] & 1;
  ++st.p_seen[grp];
  if (!mbar_wait(bars + 8 * ((C::SPLIT_P ? C::B_PHALF : C::B_PFULL) + grp), par, abort_flag,
                 a.status))
    return false;
  if (jj == 0 && st.o_items[grp] > 0 &&
      !mbar_wait(bars + 8 * (C::B_OFREE + grp), (st.o_items[grp] - 1) & 1, abort_flag, a.status))
    return false;
  tc_fence_after();
  const uint32_t o_t = tmem + (grp ? C::TMEM_O1 : C::TMEM_O0);
  const uint32_t p_t = tmem + (grp ? C::TMEM_S1 : C::TMEM_S0);
  const uint64_t vb = st.v + (uint64_t)((s * C::TILE_BYTES) >> 4);
  const int ksteps = (valid + 15) >> 4;
  if (!C::SPLIT_P) {
    mma_pv<D>(o_t, p_t, vb, ksteps, jj == 0);
    return true;
  }
  const int first = ksteps < C::PV_FIRST ? ksteps : C::PV_FIRST;
  mma_pv_range<D, C::PV_FIRST>(o_t, p_t, vb, 0, first, jj == 0);
  if (!mbar_wait(bars + 8 * (C::B_PFULL + grp), par, abort_flag, a.status)) return false;
  tc_fence_after();
  mma_pv_range<D, C::KSTEPS_PV - C::PV_FIRST>(o_t, p_t, vb, first, ksteps, false);
  return true;
}

// The issue order is one stream over the key tiles of all the CTA's items: per key tile t,
//   QK_A(t), PV_B(t-1), QK_B(t), PV_A(t),
// where t-1 may be the last tile of the previous item. The next item's first QK therefore starts
// while the previous item's tile-B softmax is still running, and the two groups stay a half tile
// apart across item boundaries instead of starting every item in step.
struct PendingPV {
  uint32_t gg;   // global key tile (V stage)
  int jj;        // key tile within its item (0: overwrite O)
  int valid;     // real keys in the tile; 0 = nothing pending
  bool last;     // the item's last key tile: its completion makes O ready
};

template <int D, bool CAUSAL, bool ROPE, bool DT>
__device__ void mma_role(const AttnArgs& a, uint32_t sbase, uint32_t bars, uint32_t tmem,
                         volatile int* abort_flag, ItemRing ring) {
  using C = Cfg<D>;
  // With in-kernel RoPE a landed tile is usable only once the diagonal warps have rotated it.
  constexpr int QF = ROPE ? C::B_QREADY : C::B_QFULL;
  constexpr int KF = ROPE ? C::B_KREADY : C::B_KFULL;
  constexpr uint32_t kIdescQKFull = idesc_bf16_f32(C::BM, C::BN, false, false);
  // QK^T of a trimmed tile: N = keys of the tile rounded up to 16.
  constexpr uint32_t kIdescQK0 = kIdescQKFull & ~(0x3Fu << 17);
  MmaState st;
  st.p_seen[0] = st.p_seen[1] = 0;
  st.o_items[0] = st.o_items[1] = 0;
  st.q_seen[0] = st.q_seen[1] = 0;
  st.v_seen = 0;
  st.q = smem_desc(sbase + C::OFF_Q, 16, 8 * C::SW, C::LAYOUT);
  st.k = smem_desc(sbase + C::OFF_K, 16, 8 * C::SW, C::LAYOUT);
  st.v = smem_desc(sbase + C::OFF_V, C::BLK_BYTES, 8 * C::SW, C::LAYOUT);
  uint32_t g = 0;
  PendingPV pend{0, 0, 0, false};
  bool ok = true;
  // PV_B of the pending tile, its V-stage release and, for an item's last tile, O_B ready.
  auto flush_b = [&]() -> bool {
    if (pend.valid == 0) return true;
    if (!issue_pv<D>(1, pend.gg, pend.jj, pend.valid, st, bars, tmem, a, abort_flag)) return false;
    tc_commit(bars + 8 * (C::B_VEMPTY + (int)(pend.gg % C::KVS)));
    if (pend.last) {
      tc_commit(bars + 8 * (C::B_OREADY + 1));
      ++st.o_items[1];
    }
    pend.valid = 0;
    return true;
  };
  for (;;) {
    const int4 desc = ring_take(ring, abort_flag, a.status, ok);
    if (!ok || desc.x == kEndOfQueue) break;
    const Item w = decode_item(desc);
    if (!DT && w.n_kv == 0) continue;
    const bool has_b = w.nrows > C::BM;
    // This item's Q buffers (one per query tile) in the per-group rings.
    const int qslot_a = (int)(st.q_seen[0] % C::QS);
    const int qslot_b = C::QS + (int)(st.q_seen[1] % C::QS);
    const uint64_t qa = st.q + (uint64_t)((qslot_a * C::TILE_BYTES) >> 4);
    const uint64_t qb = st.q + (uint64_t)((qslot_b * C::TILE_BYTES) >> 4);
    ok = mbar_wait(bars + 8 * (QF + qslot_a), (st.q_seen[0] / C::QS) & 1, abort_flag,
                   a.status);
    if (!ok) break;
    ++st.q_seen[0];
    tc_fence_after();
    for (int j = 0; j < w.n_kv; ++j, ++g) {
      const int s = (int)(g % C::KVS);
      const uint32_t ph = (g / C::KVS) & 1;
      // With the diagonal step the item's last QK and PV come after its key tiles.
      const bool last = !DT && j == w.n_kv - 1;
      // Causal variant: an item's key tiles end at its last row, which tile B holds; tile A's
      // rows end 128 rows earlier and see none of the last key tile, so A stops one tile early.
      const bool a_skips = CAUSAL && has_b && last;
      const bool last_a = (CAUSAL && has_b) ? j == w.n_kv - 2 : last;
      const int valid = min(C::BN, w.kv_len - j * C::BN);
      const uint32_t idesc_qk =
          valid == C::BN ? kIdescQKFull
                         : (kIdescQK0 | ((uint32_t)(((valid + 15) & ~15) >> 3) << 17));
      const uint64_t kb = st.k + (uint64_t)((s * C::TILE_BYTES) >> 4);
      ok = mbar_wait(bars + 8 * (KF + s), ph, abort_flag, a.status);
      if (!ok) break;
      tc_fence_after();
      // QK_A(t)
      if (!a_skips) {
        mma_qk<D>(tmem + C::TMEM_S0, qa, kb, idesc_qk);
        tc_commit(bars + 8 * C::B_SFULL);
        if (last_a) tc_commit(bars + 8 * (C::B_QEMPTY + qslot_a));
      }
      // PV_B(t-1), possibly of the previous item
      ok = flush_b();
      if (!ok) break;
      if (has_b) {
        // QK_B(t)
        if (j == 0) {
          ok = mbar_wait(bars + 8 * (QF + qslot_b), (st.q_seen[1] / C::QS) & 1,
                         abort_flag, a.status);
          if (!ok) break;
          ++st.q_seen[1];
          tc_fence_after();
        }
        mma_qk<D>(tmem + C::TMEM_S1, qb, kb, idesc_qk);
        tc_commit(bars + 8 * (C::B_SFULL + 1));
        if (last) tc_commit(bars + 8 * (C::B_QEMPTY + qslot_b));
      }
      tc_commit(bars + 8 * (C::B_KEMPTY + s));
      // PV_A(t); the V stage is released here when the item has no tile B, else after PV_B(t).
      if (!a_skips) {
        ok = issue_pv<D>(0, g, j, valid, st, bars, tmem, a, abort_flag);
        if (!ok) break;
        if (!has_b) tc_commit(bars + 8 * (C::B_VEMPTY + s));
        if (last_a) {
          tc_commit(bars + 8 * C::B_OREADY);
          ++st.o_items[0];
        }
      }
      if (has_b) pend = PendingPV{g, j, valid, last};
    }
    if (DT) {
      if (!ok) break;
      // Diagonal step: S_w = Q_w K_own,w^T against the query tile's own keys (only the diagonal
      // is used), then O_w += P_w V_own,w with P_w zero off the diagonal. Group A's own keys and
      // values occupy one K / V stage, group B's the next.
      const int sa = (int)(g % C::KVS), sb = (int)((g + 1) % C::KVS);
      ok = mbar_wait(bars + 8 * (KF + sa), (g / C::KVS) & 1, abort_flag, a.status);
      if (!ok) break;
      tc_fence_after();
      mma_qk<D>(tmem + C::TMEM_S0, qa, st.k + (uint64_t)((sa * C::TILE_BYTES) >> 4), kIdescQKFull);
      tc_commit(bars + 8 * C::B_SFULL);
      tc_commit(bars + 8 * (C::B_QEMPTY + qslot_a));
      tc_commit(bars + 8 * (C::B_KEMPTY + sa));
      ok = flush_b();
      if (!ok) break;
      if (has_b) {
        if (w.n_kv == 0) {
          ok = mbar_wait(bars + 8 * (QF + qslot_b), (st.q_seen[1] / C::QS) & 1, abort_flag,
                         a.status);
          if (!ok) break;
          ++st.q_seen[1];
        }
        ok = mbar_wait(bars + 8 * (KF + sb), ((g + 1) / C::KVS) & 1, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        mma_qk<D>(tmem + C::TMEM_S1, qb, st.k + (uint64_t)((sb * C::TILE_BYTES) >> 4),
                  kIdescQKFull);
        tc_commit(bars + 8 * (C::B_SFULL + 1));
        tc_commit(bars + 8 * (C::B_QEMPTY + qslot_b));
        tc_commit(bars + 8 * (C::B_KEMPTY + sb));
      }
      ok = issue_pv<D>(0, g, w.n_kv == 0 ? 0 : 1, C::BN, st, bars, tmem, a, abort_flag);
      if (!ok) break;
      tc_commit(bars + 8 * (C::B_VEMPTY + sa));
      tc_commit(bars + 8 * C::B_OREADY);
      ++st.o_items[0];
      if (has_b) pend = PendingPV{g + 1, w.n_kv == 0 ? 0 : 1, C::BN, true};
      g += has_b ? 2u : 1u;
    }
  }
  if (ok) ok = flush_b();
  if (!ok) {
    // Aborting: wait until every MMA this thread issued has completed.
    tc_commit(bars + 8 * C::B_DRAIN);
    mbar_wait_drain(bars + 8 * C::B_DRAIN, 0);
  }
}

// ------------------------------------------------------------------------------------------
// Softmax + epilogue
// ------------------------------------------------------------------------------------------
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t t, uint32_t* r) {
  if constexpr (N == 8) {
    tmem_ld_x8(t, r);
  } else if constexpr (N == 16) {
    tmem_ld_x16(t, r);
  } else {
    tmem_ld_x32(t, r);
  }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t t, const uint32_t* r) {
  if constexpr (N == 8) {
    tmem_st_x8(t, r);
  } else if constexpr (N == 16) {
    tmem_st_x16(t, r);
  } else {
    tmem_st_x32(t, r);
  }
}

template <int N>
__device__ __forceinline__ void reg_fence_cols(uint32_t* r) {
  if constexpr (N == 8) {
    reg_fence8(r);
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 16) reg_fence16(r + i);
  }
}

// One O row (D columns) of this group, multiplied by alpha in place in TMEM.
template <int D>
__device__ __forceinline__ void rescale_o_row(uint32_t t_o, float alpha) {
  constexpr int CW = D < 32 ? D : 32;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += CW) {
    uint32_t u[CW];
    tmem_ld_cols<CW>(t_o + c0, u);
    tmem_wait_ld();
    reg_fence_cols<CW>(u);
#pragma unroll
    for (int i = 0; i < CW; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
    tmem_st_cols<CW>(t_o + c0, u);
  }
  tmem_wait_st();
}


// Score of a candidate row against its own key, scaled to log2 units (the diagonal term of the
// mask). Plain CUDA-core dot product over 16-byte loads, half a row at a time.
template <int D>
__device__ __forceinline__ float diag_score(const AttnArgs& a, size_t base) {
  const uint4* qp = reinterpret_cast<const uint4*>(a.q + base);
  const uint4* kp = reinterpret_cast<const uint4*>(a.dk + base);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  constexpr int HV = D / 16 > 0 ? D / 16 : 1;   // 16-byte vectors per half row (at least 1)
#pragma unroll
  for (int h0 = 0; h0 < D / 8; h0 += HV) {
    uint4 qv[HV], kv[HV];
#pragma unroll
    for (int c = 0; c < HV; ++c) {
      qv[c] = ld_global_nc_v4(qp + h0 + c);
      kv[c] = ld_global_nc_v4(kp + h0 + c);
    }
#pragma unroll
    for (int c = 0; c < HV; ++c) {
      acc[0] = fmaf(bf16_lo(qv[c].x), bf16_lo(kv[c].x), fmaf(bf16_hi(qv[c].x), bf16_hi(kv[c].x), acc[0]));
      acc[1] = fmaf(bf16_lo(qv[c].y), bf16_lo(kv[c].y), fmaf(bf16_hi(qv[c].y), bf16_hi(kv[c].y), acc[1]));
      acc[2] = fmaf(bf16_lo(qv[c].z), bf16_lo(kv[c].z), fmaf(bf16_hi(qv[c].z), bf16_hi(kv[c].z), acc[2]));
      acc[3] = fmaf(bf16_lo(qv[c].w), bf16_lo(kv[c].w), fmaf(bf16_hi(qv[c].w), bf16_hi(kv[c].w), acc[3]));
    }
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) * a.scale_log2;
}

// Writes 8 consecutive output values of a row (bf16 or fp32 per a.out_fp32), already normalised.
__device__ __forceinline__ void store8(const AttnArgs& a, size_t idx, const float* o) {
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

// Writes 16 consecutive bf16 output values of a row with one 32-byte store when allowed.
__device__ __forceinline__ void store16_bf16(const AttnArgs& a, size_t idx, const float* o) {
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

// Epilogue of one query row (every thread of a group calls this; the TMEM loads are collective and
// rows outside the tile only skip their memory accesses). The diagonal score sd and the row's own
// value vv were fetched before O_w was complete, so that after it completes only the TMEM reads,
// the merge, the normalisation and the stores remain: read O_w, release it to the MMA warp, merge
// the diagonal term of a candidate row, normalise and store.
template <int D, bool LSE>
__device__ __forceinline__ void finish_row(const AttnArgs& a, bool row_ok, int seg, size_t base,
                                           uint32_t t_o, bool has_o, float m, float l, float sd,
                                           const uint4 (&vv)[D / 8], uint32_t o_free_bar) {
  const bool cand = seg == -1;
  float alpha = 1.f, beta = 0.f;
  if (cand) {
    const float m_new = fmaxf(m, sd);
    alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
    beta = fast_exp2(sd - m_new);
    l = l * alpha + beta;
  }
  // Padding queries (segment 0) see no key and output 0.
  const float inv = (seg != 0 && l > 0.f) ? 1.f / l : 0.f;
  if (LSE && row_ok) {
    // log of the row's softmax denominator: l is relative to the reference max (log2 units),
    // which the diagonal merge moved to max(m, sd) for a candidate; -inf for a padding row.
    const float ref = cand ? fmaxf(m, sd) : m;
    a.lse[base / D] = seg == 0 ? -INFINITY : (ref + log2f(l)) * 0.69314718055994531f;
  }
  const float scale_o = alpha * inv, scale_v = beta * inv;
  constexpr int CW = D < 32 ? D : 32;            // columns per TMEM load
  constexpr int PER = (D / CW) >= 2 ? 2 : 1;     // loads per TMEM wait
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += CW * PER) {
    uint32_t u[CW * PER];
    if (has_o) {
#pragma unroll
      for (int p = 0; p < PER; ++p) tmem_ld_cols<CW>(t_o + c0 + p * CW, u + p * CW);
      tmem_wait_ld();
#pragma unroll
      for (int p = 0; p < PER; ++p) reg_fence_cols<CW>(u + p * CW);
      if (c0 + CW * PER >= D) {
        // O_w has been read: the next item's first PV may overwrite it.
        tc_fence_before();
        mbar_arrive(o_free_bar);
      }
    } else {
#pragma unroll
      for (int i = 0; i < CW * PER; ++i) u[i] = 0u;
    }
    if (!row_ok) continue;
    float o[CW * PER];
#pragma unroll
    for (int i = 0; i < CW * PER; ++i) o[i] = __uint_as_float(u[i]) * scale_o;
    if (cand) {
#pragma unroll
      for (int c = 0; c < CW * PER / 8; ++c) {
        const uint4 va = vv[c0 / 8 + c];
        const uint32_t vw[4] = {va.x, va.y, va.z, va.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[8 * c + 2 * i] = fmaf(scale_v, bf16_lo(vw[i]), o[8 * c + 2 * i]);
          o[8 * c + 2 * i + 1] = fmaf(scale_v, bf16_hi(vw[i]), o[8 * c + 2 * i + 1]);
        }
      }
    }
    if (a.out_fp32) {
#pragma unroll
      for (int c = 0; c < CW * PER; c += 8) store8(a, base + c0 + c, o + c);
    } else {
#pragma unroll
      for (int c = 0; c < CW * PER; c += 16) store16_bf16(a, base + c0 + c, o + c);
    }
  }
}

// ------------------------------------------------------------------------------------------
// In-kernel right-anchored RoPE (ROPE instantiation)
// ------------------------------------------------------------------------------------------
// Swizzled shared-memory address of byte `byte_in_row` of row r of a landed tile: column block
// byte_in_row / SW, and inside it the TMA's swizzle, which XORs the 16-byte chunk index with the
// address bits three above it (tiles start on 1 KB boundaries).
template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int r, int byte_in_row) {
  using C = Cfg<D>;
  constexpr uint32_t kSwz = (uint32_t)(C::SW / 16 - 1) << 4;
  const uint32_t a = tile + (uint32_t)((byte_in_row / C::SW) * C::BLK_BYTES + r * C::SW +
                                       (byte_in_row % C::SW));
  return a ^ ((a >> 3) & kSwz);
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// (cos, sin) of the 8 pairs j = 8 cp .. 8 cp + 7 at position p, from the factor tables.
template <int D>
__device__ __forceinline__ void rope_factors(const AttnArgs& a, int p, int cp, float2 (&cs)[8]) {
  constexpr int HALF = D / 2;
  int64_t q;
  int r;
  rope_split((int64_t)p, q, r);
  const float4* cq = reinterpret_cast<const float4*>(a.rope_coarse +
                                                     (size_t)(a.rope_qmax - q) * HALF + 8 * cp);
  const float4* cf = reinterpret_cast<const float4*>(a.rope_fine + (size_t)r * HALF + 8 * cp);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 c4 = __ldg(cq + e), f4 = __ldg(cf + e);
    cs[2 * e] = rope_compose(make_float2(c4.x, c4.y), make_float2(f4.x, f4.y));
    cs[2 * e + 1] = rope_compose(make_float2(c4.z, c4.w), make_float2(f4.z, f4.w));
  }
}

// Rotates 8 pairs held as bf16 in (wa, wb) (first-half and second-half chunks of a row) and
// rounds them to bf16 again, as the rotation pre-pass does.
__device__ __forceinline__ void rope_chunk(uint4& va, uint4& vb, const float2 (&cs)[8]) {
  uint32_t wa[4] = {va.x, va.y, va.z, va.w};
  uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float oa0, ob0, oa1, ob1;
    rope_rotate(bf16_lo(wa[k]), bf16_lo(wb[k]), cs[2 * k], oa0, ob0);
    rope_rotate(bf16_hi(wa[k]), bf16_hi(wb[k]), cs[2 * k + 1], oa1, ob1);
    wa[k] = pack_bf16x2(oa0, oa1);
    wb[k] = pack_bf16x2(ob0, ob1);
  }
  va = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  vb = make_uint4(wb[0], wb[1], wb[2], wb[3]);
}

// Rotates rows [0, rows) of a landed 128-row tile in place (kDiagThreads threads, index t): thread
// t takes chunk pair cp = t % CP (pairs 8 cp .. 8 cp + 7, whose elements sit at bytes 16 cp and
// 16 cp + D of the row) on every (kDiagThreads / CP)-th row. The rows of a tile belong to one user
// and their positions rise by at most one per row, so they span fewer than 128 positions: two
// coarse blocks q0, q0 + 1 at most, whose factors the thread loads once; the fine factors are
// loaded for two rows at a time, so that their latencies overlap. Then the thread makes its
// writes visible to the tensor core's reads.
template <int D>
__device__ __forceinline__ void rope_tile(const AttnArgs& a, uint32_t tile, const int32_t* pos,
                                          int row0, int rows, int t) {
  constexpr int CP = D / 16;
  constexpr int STEP = kDiagThreads / CP;
  constexpr int HALF = D / 2;
  const int cp = t % CP;
  if (rows > 0) {
    int64_t q0;
    int r_unused;
    rope_split((int64_t)pos[row0], q0, r_unused);
    float4 co[2][4];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      // Block q0 + 1 lies past the table when q0 is the last block; no position reaches it then.
      const long long ci = a.rope_qmax - q0 - k;
      const float4* cq = reinterpret_cast<const float4*>(
          a.rope_coarse + (size_t)(ci < 0 ? 0 : ci) * HALF + 8 * cp);
#pragma unroll
      for (int e = 0; e < 4; ++e) co[k][e] = __ldg(cq + e);
    }
    for (int r = t / CP; r < rows; r += 2 * STEP) {
      const bool two = r + STEP < rows;
      int64_t qq[2];
      int rr[2];
      rope_split((int64_t)pos[row0 + r], qq[0], rr[0]);
      rope_split((int64_t)pos[row0 + (two ? r + STEP : r)], qq[1], rr[1]);
      float4 fi[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float4* cf = reinterpret_cast<const float4*>(a.rope_fine + (size_t)rr[u] * HALF +
                                                           8 * cp);
#pragma unroll
        for (int e = 0; e < 4; ++e) fi[u][e] = __ldg(cf + e);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        const int row = r + u * STEP;
        const uint32_t pa = tile_addr<D>(tile, row, 16 * cp);
        const uint32_t pb = tile_addr<D>(tile, row, 16 * cp + D);
        uint4 va = lds_v4(pa), vb = lds_v4(pb);
        const int k = qq[u] == q0 ? 0 : 1;
        float2 cs[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 c4 = k ? co[1][e] : co[0][e];
          cs[2 * e] = rope_compose(make_float2(c4.x, c4.y), make_float2(fi[u][e].x, fi[u][e].y));
          cs[2 * e + 1] =
              rope_compose(make_float2(c4.z, c4.w), make_float2(fi[u][e].z, fi[u][e].w));
        }
        rope_chunk(va, vb, cs);
        st_shared_v4(pa, va.x, va.y, va.z, va.w);
        st_shared_v4(pb, vb.x, vb.y, vb.z, vb.w);
      }
    }
  }
  fence_proxy_async_smem();
}

// Score of a candidate row against its own key with both rotated to the row's position and
// rounded to bf16 (the values the pre-pass would store), scaled to log2 units.
template <int D>
__device__ __forceinline__ float diag_score_rope(const AttnArgs& a, size_t base, int p) {
  constexpr int CP = D / 16;
  const uint4* qp = reinterpret_cast<const uint4*>(a.q + base);
  const uint4* kp = reinterpret_cast<const uint4*>(a.dk + base);
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int cp = 0; cp < CP; ++cp) {
    float2 cs[8];
    rope_factors<D>(a, p, cp, cs);
    uint4 qa = ld_global_nc_v4(qp + cp), qb = ld_global_nc_v4(qp + CP + cp);
    uint4 ka = ld_global_nc_v4(kp + cp), kb = ld_global_nc_v4(kp + CP + cp);
    rope_chunk(qa, qb, cs);
    rope_chunk(ka, kb, cs);
    const uint32_t q4[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const uint32_t k4[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc0 = fmaf(bf16_lo(q4[e]), bf16_lo(k4[e]), acc0);
      acc1 = fmaf(bf16_hi(q4[e]), bf16_hi(k4[e]), acc1);
    }
  }
  return (acc0 + acc1) * a.scale_log2;
}

// Diagonal scores, computed by two warps up to one item ahead of the softmax warps so that no
// softmax thread waits on the q / k loads: thread t covers rows t, t + 64, t + 128 and t + 192 of
// each item and deposits the score (-inf for a row without a diagonal term) in the item's slot of
// a two-slot shared array; it also starts moving each candidate row's own value towards L2 for
// the epilogue. Slot s is reused for the item after next once all 256 softmax threads have taken
// the scores out of it.
template <int D, bool CAUSAL, bool ROPE, bool DT>
__device__ void diag_role(const AttnArgs& a, float* sd_buf, uint32_t sbase, uint32_t bars,
                          volatile int* abort_flag, int t, ItemRing ring) {
  using C = Cfg<D>;
  if (DT) {
    // The diagonal terms go through the tensor core: these warps only follow the item ring.
    bool ok = true;
    for (;;) {
      const int4 desc = ring_take(ring, abort_flag, a.status, ok);
      if (!ok || desc.x == kEndOfQueue) return;
    }
  }
  uint32_t n = 0;
  uint32_t nq[2] = {0, 0};   // ROPE: Q tiles rotated per query tile (mirrors the producer)
  uint32_t g = 0;            // ROPE: K tiles rotated
  bool ok = true;
  // ROPE: rotates the next landed K tile of the item (key tile j).
  auto rotate_k = [&](const Item& w, int j) -> bool {
    const int s = (int)(g % C::KVS);
    if (!mbar_wait(bars + 8 * (C::B_KFULL + s), (g / C::KVS) & 1, abort_flag, a.status))
      return false;
    const int valid = min(C::BN, w.kv_len - j * C::BN);
    rope_tile<D>(a, sbase + C::OFF_K + s * C::TILE_BYTES, a.kv_pos, w.kv_lo + j * C::BN, valid, t);
    mbar_arrive(bars + 8 * (C::B_KREADY + s));
    ++g;
    return true;
  };
  for (;; ++n) {
    const int4 desc = ring_take(ring, abort_flag, a.status, ok);
    if (!ok || desc.x == kEndOfQueue) return;
    const Item w = decode_item(desc);
    if (ROPE && w.n_kv > 0) {
      // The item's query tiles, then its first key tile, are rotated before anything else: the
      // tensor core waits on them. The remaining key tiles follow the diagonal scores.
      const int ntiles = w.nrows > C::BM ? 2 : 1;
      for (int tt = 0; tt < ntiles; ++tt) {
        const int slot = tt * C::QS + (int)(nq[tt] % C::QS);
        if (!mbar_wait(bars + 8 * (C::B_QFULL + slot), (nq[tt] / C::QS) & 1, abort_flag,
                       a.status))
          return;
        rope_tile<D>(a, sbase + C::OFF_Q + slot * C::TILE_BYTES, a.q_pos, w.q_row0 + tt * C::BM,
                     min(C::BM, w.nrows - tt * C::BM), t);
        mbar_arrive(bars + 8 * (C::B_QREADY + slot));
        ++nq[tt];
      }
      if (!rotate_k(w, 0)) return;
    }
    const int slot = n & 1;
    // Candidate-only layer (every row a candidate) with heads of 64 or more: first every row's own
    // query, key and value towards L2, so that the score loads below wait about one memory
    // latency in all instead of one per row (3 % on the 512-candidate workload; on the full
    // layer, where few rows are candidates, and at d = 32 it measured slightly slower).
    const bool bulk_prefetch = !CAUSAL && a.q_seg == nullptr && D >= 64;
    if (bulk_prefetch) {
      for (int rr = t; rr < w.nrows; rr += kDiagThreads) {
        const size_t base = ((size_t)(w.q_row0 + rr) * (size_t)a.H + (size_t)w.h) * D;
#pragma unroll
        for (int c = 0; c < D * 2; c += 128) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.q + base + c / 2));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.dk + base + c / 2));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.dv + base + c / 2));
        }
      }
    }
    if (!mbar_wait(bars + 8 * (C::B_DIAGEMPTY + slot), ((n >> 1) & 1) ^ 1, abort_flag, a.status))
      return;
    for (int rr = t; rr < kItemRows; rr += kDiagThreads) {
      float sd = -INFINITY;
      if (rr < w.nrows) {
        const int row = w.q_row0 + rr;
        if (!CAUSAL && (!a.q_seg || a.q_seg[row] == -1)) {
          const size_t base = ((size_t)row * (size_t)a.H + (size_t)w.h) * D;
          if (!bulk_prefetch) {
#pragma unroll
            for (int c = 0; c < D * 2; c += 128)
              asm volatile("prefetch.global.L2 [%0];" ::"l"(a.dv + base + c / 2));
          }
          sd = ROPE ? diag_score_rope<D>(a, base, a.q_pos[row]) : diag_score<D>(a, base);
        }
      }
      sd_buf[slot * kItemRows + rr] = sd;
    }
    mbar_arrive(bars + 8 * (C::B_DIAGFULL + slot));
    if (ROPE)
      for (int j = 1; j < w.n_kv; ++j)
        if (!rotate_k(w, j)) return;
  }
}

template <int D, bool CAUSAL, bool LSE, bool DT>
__device__ void softmax_role(const AttnArgs& a, uint32_t bars, uint32_t tmem,
                             const float* sd_buf, volatile int* abort_flag, int warp, int lane,
                             ItemRing ring) {
  using C = Cfg<D>;
  const int grp = (warp - 2) >> 2;            // query tile A (0) or B (1) of each item
  const int quarter = warp & 3;               // TMEM lane quarter this warp may access
  const int r = quarter * 32 + lane;          // query row of this thread inside its tile
  const int row_in_item = grp * C::BM + r;
  const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
  const uint32_t t_s = t_lane + (grp ? C::TMEM_S1 : C::TMEM_S0);
  const uint32_t t_o = t_lane + (grp ? C::TMEM_O1 : C::TMEM_O0);
  const float sl2 = a.scale_log2;
  uint32_t lt = 0, oi = 0;                    // S_w fills and O_w-ready completions seen
  bool ok = true;
  uint32_t n = 0;                             // items walked (diagonal-score slot sequence)
  for (;; ++n) {
    const int4 desc = ring_take(ring, abort_flag, a.status, ok);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok || desc.x == kEndOfQueue) break;
    const Item w = decode_item(desc);
    const int slot = n & 1;
    if (DT && grp == 1 && w.nrows <= C::BM) continue;
    if (grp == 1 && w.nrows <= C::BM) {
      // The item has no tile B; its diagonal-score slot is still released (after it was filled,
      // so that this release cannot count toward the slot's previous use).
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bars + 8 * (C::B_DIAGFULL + slot), (n >> 1) & 1, abort_flag, a.status));
      if (ok) mbar_arrive(bars + 8 * (C::B_DIAGEMPTY + slot));
      continue;
    }
    const bool row_ok = row_in_item < w.nrows;
    const int row = w.q_row0 + (row_ok ? row_in_item : 0);
    const size_t base = ((size_t)row * (size_t)a.H + (size_t)w.h) * D;
    const int seg = row_ok ? (CAUSAL ? 1 : (a.q_seg ? (int)a.q_seg[row] : -1)) : 0;
    float m = -INFINITY, l = 0.f;             // running max (log2 units) and row sum
    // Causal variant: tile A of a two-tile item sees none of the item's last key tile.
    const int n_kv_g = (CAUSAL && grp == 0 && w.nrows > C::BM) ? w.n_kv - 1 : w.n_kv;
    for (int j = 0; j < n_kv_g; ++j, ++lt) {
      const int valid = min(C::BN, w.kv_len - j * C::BN);
      const int nchunks = (valid + 31) >> 5;
      // Edge tiles (the trimmed last tile, or any tile of a user with padding holes) are masked
      // column by column; interior tiles take the unmasked path.
      // Causal variant: columns past the diagonal of this group's rows are masked; key and query
      // tiles both start at the user's first row, so the offset is a multiple of the tile size
      // (a whole tile of this group's rows sees the whole key tile, or none of it, or the lower
      // triangle of it).
      const int diag_off = CAUSAL ? (w.q_row0 + grp * C::BM) - (w.kv_lo + j * C::BN) : C::BN;
      const bool edge = valid < C::BN || w.holes || (CAUSAL && diag_off < C::BN - 1);
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bars + 8 * (C::B_SFULL + grp), lt & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();

      // Pass 1: the whole S row in registers (four 32-column TMEM loads, one wait), then the
      // max of the raw scores (the scale is positive, so it commutes with max).
      uint32_t x[128];
      tmem_ld_x32(t_s + 0, x);
      tmem_ld_x32(t_s + 32, x + 32);
      tmem_ld_x32(t_s + 64, x + 64);
      tmem_ld_x32(t_s + 96, x + 96);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 128; c += 16) reg_fence16(x + c);
      if (edge) {
        // Every row of the tile sees the same key columns: the warp builds the tile's 128-bit
        // column mask with one ballot per 32 columns (lane i tests column 32k + i).
        const int8_t* kseg = w.holes ? a.kv_seg + (w.kv_lo + j * C::BN) : nullptr;
        uint32_t bits[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = 32 * k + lane;
          bool keep = c < valid;
          if (keep && kseg != nullptr) keep = kseg[c] == 1;
          bits[k] = __ballot_sync(0xffffffffu, keep);
        }
        if (CAUSAL) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            x[c] = (((bits[c >> 5] >> (c & 31)) & 1u) && c <= r + diag_off) ? x[c] : 0xff800000u;
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            x[c] = ((bits[c >> 5] >> (c & 31)) & 1u) ? x[c] : 0xff800000u;   // -inf
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const float m_new = fmaxf(m, m_tile);
      // Lazy rescaling: keep the stale reference unless the max grew by more than 2^8.
      const bool rescale = m_new > m + 8.0f;
      const float m_use = rescale ? m_new : m;
      const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;

      // Pass 2: p = 2^(scale_log2 * s - m), written back over S_w as bf16 pairs (TMEM column k
      // holds keys 2k, 2k+1) 32 keys at a time; chunks past the last real key are never read
      // by the trimmed PV and are skipped. Arithmetic runs on key pairs (packed fp32 FMA/add).
      // TMEM loads and stores are warp-collective: the warp rescales O_w (after pass 2) when any
      // of its rows must. With SPLIT_P such a warp releases the first half of P only after the
      // rescale, since the first PV k-step already adds into every row of O_w.
      const float alpha = (rescale && m != -INFINITY) ? fast_exp2(m - m_use) : 1.f;
      const bool warp_rescale = __any_sync(0xffffffffu, rescale && j >= 1);
      const float2 sl2v = make_float2(sl2, sl2), negv = make_float2(neg_m, neg_m);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (C::SPLIT_P && 32 * c == 16 * C::PV_FIRST && !warp_rescale) {
          // Keys 0..63 of P_w are written: the PV may start on them.
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bars + 8 * (C::B_PHALF + grp));
        }
        if (c >= nchunks) continue;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 xs = __ffma2_rn(make_float2(__uint_as_float(x[32 * c + 2 * i]),
                                                   __uint_as_float(x[32 * c + 2 * i + 1])),
                                       sl2v, negv);
          float2 p;
          p.x = fast_exp2(xs.x);
          p.y = fast_exp2(xs.y);
          if ((i & 3) == 0) acc0 = __fadd2_rn(acc0, p);
          if ((i & 3) == 1) acc1 = __fadd2_rn(acc1, p);
          if ((i & 3) == 2) acc2 = __fadd2_rn(acc2, p);
          if ((i & 3) == 3) acc3 = __fadd2_rn(acc3, p);
          pk[i] = pack_bf16x2(p.x, p.y);
        }
        tmem_st_x16(t_s + 16 * c, pk);
      }
      const float2 acc01 = __fadd2_rn(acc0, acc1), acc23 = __fadd2_rn(acc2, acc3);
      const float tile_sum = (acc01.x + acc01.y) + (acc23.x + acc23.y);
      // O_w is stable here: its last PV was issued before the QK that filled S_w, and that
      // QK's commit fired only after every earlier MMA completed.
      if (warp_rescale) rescale_o_row<D>(t_o, alpha);
      l = l * alpha + tile_sum;
      m = m_use;
      tmem_wait_st();
      tc_fence_before();
      if (C::SPLIT_P && warp_rescale) mbar_arrive(bars + 8 * (C::B_PHALF + grp));
      mbar_arrive(bars + 8 * (C::B_PFULL + grp));
    }
    if (!ok) break;
    if (DT) {
      // Diagonal step: S holds this tile's rows against their own keys; each row keeps only its
      // own score (column r), merged like a key tile's, and P is zero off the diagonal.
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bars + 8 * (C::B_SFULL + grp), lt & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      ++lt;
      uint32_t xs[32];
      tmem_ld_x32(t_s + (uint32_t)(quarter * 32), xs);
      tmem_wait_ld();
      reg_fence16(xs);
      reg_fence16(xs + 16);
      float sraw = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) sraw = c == lane ? __uint_as_float(xs[c]) : sraw;
      const float s2 = sraw * sl2;
      const float m_new = fmaxf(m, s2);
      const bool rescale = m_new > m + 8.0f;
      const float m_use = rescale ? m_new : m;
      const float alpha = (rescale && m != -INFINITY) ? fast_exp2(m - m_use) : 1.f;
      const uint32_t pb = pack_bf16x2(fast_exp2(s2 - m_use), 0.f) & 0xFFFFu;
      // The row sum takes the weight exactly as the PV applies it (bf16), so that a row whose own
      // term dominates is normalised by that same weight.
      const float p = __uint_as_float(pb << 16);
      const uint32_t pw = (r & 1) ? (pb << 16) : pb;
      const int pcol = r >> 1;   // TMEM column of P holding keys 2 pcol, 2 pcol + 1
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = (16 * c + i == pcol) ? pw : 0u;
        tmem_st_x16(t_s + 16 * c, pk);
      }
      // O_w is stable here (as for a key tile); the item's first step needs no rescale.
      if (__any_sync(0xffffffffu, rescale && w.n_kv > 0)) rescale_o_row<D>(t_o, alpha);
      l = l * alpha + p;
      m = m_use;
      tmem_wait_st();
      tc_fence_before();
      // The whole diagonal P is written at once: with SPLIT_P (heads of up to 32, where the host
      // does not select this step) both of its releases go out here.
      if (C::SPLIT_P) mbar_arrive(bars + 8 * (C::B_PHALF + grp));
      mbar_arrive(bars + 8 * (C::B_PFULL + grp));
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bars + 8 * (C::B_OREADY + grp), oi & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      ++oi;
      const uint4 vz[D / 8] = {};
      finish_row<D, LSE>(a, row_ok, row_ok ? 1 : 0, base, t_o, true, m, l, -INFINITY, vz,
                         bars + 8 * (C::B_OFREE + grp));
      continue;
    }
    // The row's own value is fetched while the item's last PV runs.
    uint4 vv[D / 8];
    {
      const uint4* vp = reinterpret_cast<const uint4*>(a.dv + base);
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        vv[c] = seg == -1 ? ld_global_nc_v4(vp + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    ok = __all_sync(0xffffffffu,
                    mbar_wait(bars + 8 * (C::B_DIAGFULL + slot), (n >> 1) & 1, abort_flag, a.status));
    if (!ok) break;
    const float sd = sd_buf[slot * kItemRows + row_in_item];   // diagonal score (candidates)
    mbar_arrive(bars + 8 * (C::B_DIAGEMPTY + slot));
    if (w.n_kv > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bars + 8 * (C::B_OREADY + grp), oi & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      ++oi;
    }
    finish_row<D, LSE>(a, row_ok, seg, base, t_o, w.n_kv > 0, m, l, sd, vv,
                       bars + 8 * (C::B_OFREE + grp));
  }
}

// ------------------------------------------------------------------------------------------
// Kernel
// ------------------------------------------------------------------------------------------
template <int D, bool CAUSAL, bool LSE, bool ROPE, bool DT>
__global__ void __launch_bounds__(kThreads, 1)
    jagged_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDK,
                       const __grid_constant__ CUtensorMap tmDV, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* skip = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // An error recorded earlier on the stream makes the launch a no-op; one thread reads the status
  // so that the whole CTA takes the same decision.
  if (threadIdx.x == 0) *skip = *a.status != 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * C::QS; ++i) {
      mbar_init(bars + 8 * (C::B_QFULL + i), 1);
      mbar_init(bars + 8 * (C::B_QEMPTY + i), 1);
    }
    for (int i = 0; i < C::KVS; ++i) {
      mbar_init(bars + 8 * (C::B_KFULL + i), 1);
      mbar_init(bars + 8 * (C::B_KEMPTY + i), 1);
      mbar_init(bars + 8 * (C::B_VFULL + i), 1);
      mbar_init(bars + 8 * (C::B_VEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + 8 * (C::B_SFULL + i), 1);
      mbar_init(bars + 8 * (C::B_PFULL + i), kSoftmaxThreads / 2);
      mbar_init(bars + 8 * (C::B_OREADY + i), 1);
      mbar_init(bars + 8 * (C::B_OFREE + i), kSoftmaxThreads / 2);
      mbar_init(bars + 8 * (C::B_DIAGFULL + i), kDiagThreads);
      mbar_init(bars + 8 * (C::B_DIAGEMPTY + i), kSoftmaxThreads);
    }
    mbar_init(bars + 8 * C::B_DRAIN, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(bars + 8 * (C::B_RINGFULL + i), 1);
      mbar_init(bars + 8 * (C::B_RINGEMPTY + i), kRingReaders);
    }
    for (int i = 0; i < 2 * C::QS; ++i) mbar_init(bars + 8 * (C::B_QREADY + i), kDiagThreads);
    for (int i = 0; i < C::KVS; ++i) mbar_init(bars + 8 * (C::B_KREADY + i), kDiagThreads);
    for (int i = 0; i < 2; ++i) mbar_init(bars + 8 * (C::B_PHALF + i), kSoftmaxThreads / 2);
    *abort_flag = 0;
    mbar_fence_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    if (DT) {
      tma_prefetch_map(&tmDK);
      tma_prefetch_map(&tmDV);
    }
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
  ItemRing ring{reinterpret_cast<volatile int*>(smem + C::OFF_RING), bars + 8 * C::B_RINGFULL,
                bars + 8 * C::B_RINGEMPTY, 0u};

  if (!*skip) {
    if (warp == 0) {
      if (lane < 2)
        producer_role<D, DT>(&tmQ, &tmK, &tmV, &tmDK, &tmDV, a, sbase, bars, n_items, abort_flag,
                             lane == 1, ring);
    } else if (warp == 1) {
      if (lane == 0) mma_role<D, CAUSAL, ROPE, DT>(a, sbase, bars, tmem, abort_flag, ring);
    } else if (warp < 10) {
      softmax_role<D, CAUSAL, LSE, DT>(a, bars, tmem, reinterpret_cast<const float*>(smem + C::OFF_DIAG),
                      abort_flag, warp, lane, ring);
    } else {
      diag_role<D, CAUSAL, ROPE, DT>(a, reinterpret_cast<float*>(smem + C::OFF_DIAG), sbase, bars,
                                 abort_flag,
                   threadIdx.x - 320, ring);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // The last CTA to finish resets the run-time queue for the next launch on the stream.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&a.queue[1], 1) == (int)gridDim.x - 1) {
      a.queue[0] = 0;
      a.queue[1] = 0;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
// Kernel attributes set so far, per device and head size.
constexpr int kMaxDevices = 64;
bool g_attr_set[kMaxDevices][4];
std::mutex g_attr_mu;

int d_index(int d) { return d == 16 ? 0 : d == 32 ? 1 : d == 64 ? 2 : 3; }

template <int D>
int launch_attention_d(const AttnArgs& a, const void* q, int64_t Tq, const void* k,
                       const void* v, int64_t Tkv, cudaStream_t stream) {
  using C = Cfg<D>;
  int dev = 0, sms = 0;
  const int rc = current_device(&dev, &sms);
  if (rc) return rc;
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!g_attr_set[dev][d_index(D)]) {
      if (cudaFuncSetAttribute(jagged_attn_kernel<D, false, false, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess ||
          cudaFuncSetAttribute(jagged_attn_kernel<D, true, false, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess ||
          cudaFuncSetAttribute(jagged_attn_kernel<D, false, true, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess ||
          cudaFuncSetAttribute(jagged_attn_kernel<D, false, false, true, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_ALLOC) != cudaSuccess ||
          (D >= 64 && cudaFuncSetAttribute(jagged_attn_kernel<D, false, false, false, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::SMEM_ALLOC) != cudaSuccess))
        return JCA_ERR_CUDA;
      g_attr_set[dev][d_index(D)] = true;
    }
  }
  CUtensorMap tmQ, tmK, tmV;
  if (!make_rows_map_bf16(&tmQ, q, Tq, a.H, D, C::BM) ||
      !make_rows_map_bf16(&tmK, k, Tkv, a.H, D, C::BM) ||
      !make_rows_map_bf16(&tmV, v, Tkv, a.H, D, C::BM))
    return JCA_ERR_CUDA;
  AttnArgs args = a;
  args.out_v8 = aligned(a.out, 32) ? 1 : 0;
  // Candidate-only layer with heads of 64 or more: the rows' own keys and values go through the
  // tensor core as a diagonal step (two more maps over them); elsewhere those maps are unused.
  const bool dt = D >= 64 && a.q_seg == nullptr && !a.causal && a.lse == nullptr && !a.rope;
  CUtensorMap tmDK = tmK, tmDV = tmV;
  if (dt && (!make_rows_map_bf16(&tmDK, a.dk, Tq, a.H, D, C::BM) ||
             !make_rows_map_bf16(&tmDV, a.dv, Tq, a.H, D, C::BM)))
    return JCA_ERR_CUDA;
  // Instantiations: the main path, the causal variant, the training forward (log-sum-exp
  // output), the in-kernel RoPE rotation and the candidate-only diagonal step; each mode is
  // compile-time so that the main path carries none of the others' code.
  if (a.causal)
    jagged_attn_kernel<D, true, false, false, false><<<sms, kThreads, C::SMEM_ALLOC, stream>>>(
        tmQ, tmK, tmV, tmDK, tmDV, args);
  else if (a.lse != nullptr)
    jagged_attn_kernel<D, false, true, false, false><<<sms, kThreads, C::SMEM_ALLOC, stream>>>(
        tmQ, tmK, tmV, tmDK, tmDV, args);
  else if (a.rope)
    jagged_attn_kernel<D, false, false, true, false><<<sms, kThreads, C::SMEM_ALLOC, stream>>>(
        tmQ, tmK, tmV, tmDK, tmDV, args);
  else if (dt)
    jagged_attn_kernel<D, false, false, false, (D >= 64)><<<sms, kThreads, C::SMEM_ALLOC, stream>>>(
        tmQ, tmK, tmV, tmDK, tmDV, args);
  else
    jagged_attn_kernel<D, false, false, false, false><<<sms, kThreads, C::SMEM_ALLOC, stream>>>(
        tmQ, tmK, tmV, tmDK, tmDV, args);
  return cudaGetLastError() == cudaSuccess ? JCA_OK : JCA_ERR_CUDA;
}

int launch_attention(int d, const AttnArgs& a, const void* q, int64_t Tq, const void* k,
                     const void* v, int64_t Tkv, cudaStream_t stream) {
  switch (d) {
    case 16: return launch_attention_d<16>(a, q, Tq, k, v, Tkv, stream);
    case 32: return launch_attention_d<32>(a, q, Tq, k, v, Tkv, stream);
    case 64: return launch_attention_d<64>(a, q, Tq, k, v, Tkv, stream);
    case 128: return launch_attention_d<128>(a, q, Tq, k, v, Tkv, stream);
    default: return JCA_ERR_HEAD_DIM;
  }
}

bool idx_ok(int idx_bits) { return idx_bits == 32 || idx_bits == 64; }

}  // namespace
}  // namespace jca

using namespace jca;

namespace jca {
namespace {

// Checks shared by the plan/run entry points; returns JCA_OK or a negative code.
int check_sizes(int idx_bits, int d_head, int64_t B, int64_t rows, int64_t kv_rows, int H) {
  if (!idx_ok(idx_bits)) return JCA_ERR_IDX_BITS;
  if (!head_dim_ok(d_head)) return JCA_ERR_HEAD_DIM;
  if (B < 0 || rows < 0 || kv_rows < 0 || H < 1 || H >= 65536 || rows >= (int64_t)INT_MAX ||
      kv_rows >= (int64_t)INT_MAX || B >= (int64_t)INT_MAX)
    return JCA_ERR_SHAPE;
  if (B == 0 && (rows != 0 || kv_rows != 0)) return JCA_ERR_SHAPE;
  if (workspace_layout(B, rows, H).max_items >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  return JCA_OK;
}

int check_workspace(const void* workspace, size_t workspace_bytes, int64_t B, int64_t rows, int H) {
  if (!workspace) return JCA_ERR_NULL;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  if (workspace_bytes < workspace_layout(B, rows, H).total) return JCA_ERR_WORKSPACE;
  return JCA_OK;
}

}  // namespace
}  // namespace jca

extern "C" size_t jca_workspace_bytes(int64_t B, int64_t rows, int H, int d_head) {
  if (B < 0 || rows < 0 || H < 1 || !head_dim_ok(d_head)) return 0;
  return workspace_layout(B, rows, H).total;
}

extern "C" int jagged_cand_attn_plan(const void* offsets, const void* candidate_start,
                                     const int8_t* seg, int64_t B, int64_t T, int H, int d_head,
                                     int idx_bits, void* workspace, size_t workspace_bytes,
                                     int32_t* status, jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, T, T, H);
  if (rc) return rc;
  if (!status || !offsets) return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  rc = check_workspace(workspace, workspace_bytes, B, T, H);
  if (rc) return rc;
  const WorkspaceLayout L = workspace_layout(B, T, H);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int8_t* segp = seg ? const_cast<int8_t*>(seg) : reinterpret_cast<int8_t*>(ws + L.seg);
  int32_t* kv_count = reinterpret_cast<int32_t*>(ws + L.kv_count);
  // Without a caller's segment IDs, one pass builds them from the candidate starts and reduces
  // the bounds.
  if (launch_bounds(segp, offsets, B, T, idx_bits, ws + L.hist_lo, ws + L.hist_hi, ws + L.cand_lo,
                    ws + L.cand_hi, kv_count, 0, status, st, seg ? nullptr : candidate_start,
                    seg ? nullptr : segp) != cudaSuccess)
    return JCA_ERR_CUDA;
  if (launch_work_queue(offsets, ws + L.hist_lo, ws + L.hist_hi, kv_count, B, T, T, H, idx_bits,
                        reinterpret_cast<int32_t*>(ws + L.items), L.max_items,
                        reinterpret_cast<int32_t*>(ws + L.n_items), status, st,
                        reinterpret_cast<int32_t*>(ws + L.queue)) != cudaSuccess)
    return JCA_ERR_CUDA;
  return JCA_OK;
}

namespace jca {
namespace {

// In-kernel RoPE for run_full: positions of the rows and the factor tables (rope_device.cuh).
struct RopeRun {
  const int32_t* pos = nullptr;
  const float2* coarse = nullptr;
  const float2* fine = nullptr;
  long long qmax = 0;
};

int run_full(const void* q, const void* k, const void* v, void* out, int out_fp32, float* lse,
             const int8_t* seg, int64_t B, int64_t T, int H, int d_head, float scale,
             void* workspace, size_t workspace_bytes, int32_t* status, jca_stream_t stream,
             const RopeRun* rope = nullptr) {
  int rc = check_sizes(32, d_head, B, T, T, H);
  if (rc) return rc;
  if (!status) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out)) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  rc = check_workspace(workspace, workspace_bytes, B, T, H);
  if (rc) return rc;
  if (T == 0) return JCA_OK;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_head);
  const WorkspaceLayout L = workspace_layout(B, T, H);
  char* ws = static_cast<char*>(workspace);
  const int8_t* segp = seg ? seg : reinterpret_cast<const int8_t*>(ws + L.seg);
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.dk = static_cast<const __nv_bfloat16*>(k);
  a.dv = static_cast<const __nv_bfloat16*>(v);
  a.q_seg = segp;
  a.kv_seg = segp;
  a.out = out;
  a.items = reinterpret_cast<const int4*>(ws + L.items);
  a.n_items = reinterpret_cast<const int32_t*>(ws + L.n_items);
  a.queue = reinterpret_cast<int32_t*>(ws + L.queue);
  a.status = status;
  a.H = H;
  a.out_fp32 = out_fp32 ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse = lse;
  if (rope != nullptr) {
    a.rope = 1;
    a.q_pos = rope->pos;
    a.kv_pos = rope->pos;
    a.rope_coarse = rope->coarse;
    a.rope_fine = rope->fine;
    a.rope_qmax = rope->qmax;
  }
  return launch_attention(d_head, a, q, T, k, v, T, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace jca

extern "C" int jagged_cand_attn_run(const void* q, const void* k, const void* v, void* out,
                                    int out_fp32, const int8_t* seg, int64_t B, int64_t T, int H,
                                    int d_head, float scale, void* workspace,
                                    size_t workspace_bytes, int32_t* status,
                                    jca_stream_t stream) {
  return run_full(q, k, v, out, out_fp32, nullptr, seg, B, T, H, d_head, scale, workspace,
                  workspace_bytes, status, stream);
}

extern "C" int jagged_cand_attn_fwd_lse(const void* q, const void* k, const void* v, void* out,
                                        int out_fp32, float* lse, const void* offsets,
                                        const void* candidate_start, const int8_t* seg, int64_t B,
                                        int64_t T, int H, int d_head, float scale, int idx_bits,
                                        void* workspace, size_t workspace_bytes, int32_t* status,
                                        jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, T, T, H);
  if (rc) return rc;
  if (!status || !offsets || (T > 0 && (!q || !k || !v || !out || !lse))) return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
                !aligned(lse, 4)))
    return JCA_ERR_ALIGN;
  rc = jagged_cand_attn_plan(offsets, candidate_start, seg, B, T, H, d_head, idx_bits, workspace,
                             workspace_bytes, status, stream);
  if (rc) return rc;
  return run_full(q, k, v, out, out_fp32, lse, seg, B, T, H, d_head, scale, workspace,
                  workspace_bytes, status, stream);
}

extern "C" int jagged_cand_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                    int out_fp32, const void* offsets,
                                    const void* candidate_start, const int8_t* seg, int64_t B,
                                    int64_t T, int H, int d_head, float scale, int idx_bits,
                                    void* workspace, size_t workspace_bytes, int32_t* status,
                                    jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, T, T, H);
  if (rc) return rc;
  if (!status || !offsets) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out)) return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  rc = jagged_cand_attn_plan(offsets, candidate_start, seg, B, T, H, d_head, idx_bits, workspace,
                             workspace_bytes, status, stream);
  if (rc) return rc;
  return jagged_cand_attn_run(q, k, v, out, out_fp32, seg, B, T, H, d_head, scale, workspace,
                              workspace_bytes, status, stream);
}

extern "C" int jagged_causal_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                      int out_fp32, const void* offsets, int64_t B, int64_t T,
                                      int H, int d_head, float scale, int idx_bits,
                                      void* workspace, size_t workspace_bytes, int32_t* status,
                                      jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, T, T, H);
  if (rc) return rc;
  if (!status || !offsets) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out)) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  rc = check_workspace(workspace, workspace_bytes, B, T, H);
  if (rc) return rc;
  const WorkspaceLayout L = workspace_layout(B, T, H);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (launch_causal_queue(offsets, B, T, H, idx_bits, reinterpret_cast<int32_t*>(ws + L.items),
                          L.max_items, reinterpret_cast<int32_t*>(ws + L.n_items), status, st,
                          reinterpret_cast<int32_t*>(ws + L.queue)) != cudaSuccess)
    return JCA_ERR_CUDA;
  if (T == 0) return JCA_OK;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_head);
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.dk = static_cast<const __nv_bfloat16*>(k);
  a.dv = static_cast<const __nv_bfloat16*>(v);
  a.q_seg = nullptr;
  a.kv_seg = nullptr;
  a.out = out;
  a.items = reinterpret_cast<const int4*>(ws + L.items);
  a.n_items = reinterpret_cast<const int32_t*>(ws + L.n_items);
  a.queue = reinterpret_cast<int32_t*>(ws + L.queue);
  a.status = status;
  a.H = H;
  a.out_fp32 = out_fp32 ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.causal = 1;
  return launch_attention(d_head, a, q, T, k, v, T, st);
}

extern "C" int cand_only_attn_plan(const void* cand_offsets, const void* hist_offsets,
                                   const int8_t* hist_seg, int64_t B, int64_t Nc, int64_t Th,
                                   int H, int d_head, int idx_bits, void* workspace,
                                   size_t workspace_bytes, int32_t* status,
                                   jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, Nc, Th, H);
  if (rc) return rc;
  if (!status || !cand_offsets || !hist_offsets) return JCA_ERR_NULL;
  rc = check_workspace(workspace, workspace_bytes, B, Nc, H);
  if (rc) return rc;
  const WorkspaceLayout L = workspace_layout(B, Nc, H);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const void* kv_lo;
  const void* kv_hi;
  const int32_t* kv_count = nullptr;
  if (hist_seg) {
    int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.kv_count);
    if (launch_bounds(hist_seg, hist_offsets, B, Th, idx_bits, ws + L.hist_lo, ws + L.hist_hi,
                      nullptr, nullptr, cnt, 1, status, st) != cudaSuccess)
      return JCA_ERR_CUDA;
    kv_lo = ws + L.hist_lo;
    kv_hi = ws + L.hist_hi;
    kv_count = cnt;
  } else {
    // Every history row is valid: the key interval of user b is [hist_off[b], hist_off[b+1]).
    kv_lo = hist_offsets;
    kv_hi = static_cast<const char*>(hist_offsets) + idx_bits / 8;
  }
  if (launch_work_queue(cand_offsets, kv_lo, kv_hi, kv_count, B, Nc, Th, H, idx_bits,
                        reinterpret_cast<int32_t*>(ws + L.items), L.max_items,
                        reinterpret_cast<int32_t*>(ws + L.n_items), status, st,
                        reinterpret_cast<int32_t*>(ws + L.queue)) != cudaSuccess)
    return JCA_ERR_CUDA;
  return JCA_OK;
}

extern "C" int cand_only_attn_run(const void* cand_q, const void* own_k, const void* own_v,
                                  const void* hist_k, const void* hist_v, const int8_t* hist_seg,
                                  void* out, int out_fp32, int64_t B, int64_t Nc, int64_t Th,
                                  int H, int d_head, float scale, void* workspace,
                                  size_t workspace_bytes, int32_t* status,
                                  jca_stream_t stream) {
  int rc = check_sizes(32, d_head, B, Nc, Th, H);
  if (rc) return rc;
  if (!status) return JCA_ERR_NULL;
  if (Nc > 0 && (!cand_q || !own_k || !own_v || !out)) return JCA_ERR_NULL;
  if (Th > 0 && (!hist_k || !hist_v)) return JCA_ERR_NULL;
  if (Nc > 0 && (!aligned(cand_q, 16) || !aligned(own_k, 16) || !aligned(own_v, 16) ||
                 !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  if (Th > 0 && (!aligned(hist_k, 16) || !aligned(hist_v, 16))) return JCA_ERR_ALIGN;
  rc = check_workspace(workspace, workspace_bytes, B, Nc, H);
  if (rc) return rc;
  if (Nc == 0) return JCA_OK;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_head);
  const WorkspaceLayout L = workspace_layout(B, Nc, H);
  char* ws = static_cast<char*>(workspace);
  AttnArgs a;
  a.q = static_cast<const __nv_bfloat16*>(cand_q);
  a.dk = static_cast<const __nv_bfloat16*>(own_k);
  a.dv = static_cast<const __nv_bfloat16*>(own_v);
  a.q_seg = nullptr;
  a.kv_seg = hist_seg;
  a.out = out;
  a.items = reinterpret_cast<const int4*>(ws + L.items);
  a.n_items = reinterpret_cast<const int32_t*>(ws + L.n_items);
  a.queue = reinterpret_cast<int32_t*>(ws + L.queue);
  a.status = status;
  a.H = H;
  a.out_fp32 = out_fp32 ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  // With no history rows at all, the key maps are never read; they point at the candidates.
  const void* kp = Th > 0 ? hist_k : own_k;
  const void* vp = Th > 0 ? hist_v : own_v;
  return launch_attention(d_head, a, cand_q, Nc, kp, vp, Th > 0 ? Th : Nc,
                          reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int cand_only_attn_fwd(const void* cand_q, const void* own_k, const void* own_v,
                                  const void* cand_offsets, const void* hist_k,
                                  const void* hist_v, const void* hist_offsets,
                                  const int8_t* hist_seg, void* out, int out_fp32, int64_t B,
                                  int64_t Nc, int64_t Th, int H, int d_head, float scale,
                                  int idx_bits, void* workspace, size_t workspace_bytes,
                                  int32_t* status, jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, Nc, Th, H);
  if (rc) return rc;
  if (!status || !cand_offsets || !hist_offsets) return JCA_ERR_NULL;
  if (Nc > 0 && (!cand_q || !own_k || !own_v || !out)) return JCA_ERR_NULL;
  if (Th > 0 && (!hist_k || !hist_v)) return JCA_ERR_NULL;
  if (Nc > 0 && (!aligned(cand_q, 16) || !aligned(own_k, 16) || !aligned(own_v, 16) ||
                 !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  if (Th > 0 && (!aligned(hist_k, 16) || !aligned(hist_v, 16))) return JCA_ERR_ALIGN;
  rc = cand_only_attn_plan(cand_offsets, hist_offsets, hist_seg, B, Nc, Th, H, d_head, idx_bits,
                           workspace, workspace_bytes, status, stream);
  if (rc) return rc;
  return cand_only_attn_run(cand_q, own_k, own_v, hist_k, hist_v, hist_seg, out, out_fp32, B, Nc,
                            Th, H, d_head, scale, workspace, workspace_bytes, status, stream);
}

namespace jca {
namespace {

// Workspace of jagged_cand_attn_rope_fwd: the plan, then the positions and the factor tables.
struct RopeLayout {
  WorkspaceLayout base;
  size_t pos = 0, coarse = 0, fine = 0, total = 0;
};

RopeLayout rope_layout(int64_t B, int64_t T, int H, int d) {
  RopeLayout L;
  L.base = workspace_layout(B, T, H);
  size_t o = align_up(L.base.total, 256);
  L.pos = o;
  o = align_up(o + 4 * (size_t)T, 256);
  L.coarse = o;
  o = align_up(o + 8 * (size_t)(d / 2) * (size_t)(T / kRopeFine + 3), 256);
  L.fine = o;
  o = align_up(o + 8 * (size_t)(d / 2) * kRopeFine, 256);
  L.total = o;
  return L;
}

}  // namespace
}  // namespace jca

extern "C" size_t jca_rope_attn_workspace_bytes(int64_t B, int64_t T, int H, int d_head) {
  if (B < 0 || T < 0 || H < 1 || !head_dim_ok(d_head)) return 0;
  return rope_layout(B, T, H, d_head).total;
}

extern "C" int jagged_cand_attn_rope_fwd(const void* q, const void* k, const void* v, void* out,
                                         int out_fp32, const void* offsets,
                                         const void* candidate_start, const int8_t* seg, int64_t B,
                                         int64_t T, int H, int d_head, float scale,
                                         int64_t history_end, float rope_base, int idx_bits,
                                         void* workspace, size_t workspace_bytes,
                                         int32_t* status, jca_stream_t stream) {
  int rc = check_sizes(idx_bits, d_head, B, T, T, H);
  if (rc) return rc;
  if (!(rope_base > 1.f) || history_end > (int64_t)INT_MAX || history_end - T < (int64_t)INT_MIN)
    return JCA_ERR_SHAPE;
  if (!status || !offsets) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out)) return JCA_ERR_NULL;
  if (B > 0 && !seg && !candidate_start) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)))
    return JCA_ERR_ALIGN;
  if (!workspace) return JCA_ERR_NULL;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  const RopeLayout L = rope_layout(B, T, H, d_head);
  if (workspace_bytes < L.total) return JCA_ERR_WORKSPACE;
  rc = jagged_cand_attn_plan(offsets, candidate_start, seg, B, T, H, d_head, idx_bits, workspace,
                             workspace_bytes, status, stream);
  if (rc) return rc;
  if (T == 0) return JCA_OK;
  char* ws = static_cast<char*>(workspace);
  const int8_t* segp = seg ? seg : reinterpret_cast<const int8_t*>(ws + L.base.seg);
  int32_t* pos = reinterpret_cast<int32_t*>(ws + L.pos);
  rc = jca_rope_positions(segp, offsets, B, T, history_end, idx_bits, pos, status, stream);
  if (rc) return rc;
  const RopeTables tabs = rope_tables(T, history_end);
  float2* coarse = reinterpret_cast<float2*>(ws + L.coarse);
  float2* fine = reinterpret_cast<float2*>(ws + L.fine);
  if (launch_rope_tables(coarse, fine, d_head, tabs, rope_base,
                         reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JCA_ERR_CUDA;
  RopeRun rr;
  rr.pos = pos;
  rr.coarse = coarse;
  rr.fine = fine;
  rr.qmax = tabs.qmax;
  return run_full(q, k, v, out, out_fp32, nullptr, seg, B, T, H, d_head, scale, workspace,
                  workspace_bytes, status, stream, &rr);
}

extern "C" size_t jca_seqpack_workspace_bytes(int64_t B, int64_t Th, int64_t Nc, int H,
                                              int d_head) {
  if (B < 0 || Th < 0 || Nc < 0 || H < 1 || !head_dim_ok(d_head)) return 0;
  return seqpack_layout(B, Th + Nc, H).total;
}

extern "C" int jagged_cand_attn_seqpack_fwd(const void* q, const void* k, const void* v,
                                            void* out, int out_fp32, float* lse,
                                            const void* hist_offsets, const void* cand_offsets,
                                            const int8_t* seg, int64_t B, int64_t Th, int64_t Nc,
                                            int H, int d_head, float scale, int idx_bits,
                                            void* workspace, size_t workspace_bytes,
                                            int32_t* status, jca_stream_t stream) {
  if (Th < 0 || Nc < 0 || 2 * B >= (int64_t)INT_MAX) return JCA_ERR_SHAPE;
  const int64_t T = Th + Nc;
  int rc = check_sizes(idx_bits, d_head, 2 * B, T, T, H);
  if (rc) return rc;
  if (!status || !hist_offsets || !cand_offsets) return JCA_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !out)) return JCA_ERR_NULL;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
                (lse && !aligned(lse, 4))))
    return JCA_ERR_ALIGN;
  if (!workspace) return JCA_ERR_NULL;
  if (!aligned(workspace, 256)) return JCA_ERR_ALIGN;
  const SeqpackLayout S = seqpack_layout(B, T, H);
  if (workspace_bytes < S.total) return JCA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_seqpack_plan(hist_offsets, cand_offsets, seg, B, Th, Nc, H, idx_bits,
                          static_cast<char*>(workspace), S.base, S.q_off2, status,
                          st) != cudaSuccess)
    return JCA_ERR_CUDA;
  // The 2B query runs go through the attention kernel as 2B "users" of the packed matrix; without
  // a caller's segment IDs the kernel reads the ones the plan wrote into the workspace.
  return run_full(q, k, v, out, out_fp32, lse, seg, 2 * B, T, H, d_head, scale, workspace,
                  workspace_bytes, status, stream);
}

extern "C" const char* jca_status_string(int code) {
  switch (code) {
    case JCA_OK: return "ok";
    case JCA_ERR_NULL: return "a required pointer is NULL";
    case JCA_ERR_SHAPE: return "invalid or unsupported size (B, rows, H)";
    case JCA_ERR_HEAD_DIM: return "d_head must be 16, 32, 64 or 128";
    case JCA_ERR_ALIGN: return "pointer not aligned (tensors: 16 bytes, workspace: 256 bytes)";
    case JCA_ERR_IDX_BITS: return "idx_bits must be 32 or 64";
    case JCA_ERR_WORKSPACE: return "workspace smaller than jca_workspace_bytes()";
    case JCA_ERR_CUDA: return "a CUDA call failed";
    case JCA_ERR_DEVICE: return "the current device is not sm_100 (B200)";
    case JCA_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the library's static array holds";
    case JCA_STATUS_BAD_LENGTH: return "negative length or offsets overflow the index type";
    case JCA_STATUS_BAD_OFFSETS: return "offsets do not start at 0, decrease, or do not end at rows";
    case JCA_STATUS_BAD_CAND_START: return "candidate_start outside [0, row length]";
    case JCA_STATUS_BAD_SEG_LAYOUT: return "a history token follows a candidate inside a row";
    case JCA_STATUS_BAD_SEG_VALUE: return "segment ID outside the allowed values";
    case JCA_STATUS_QUEUE_OVERFLOW: return "work queue overflow";
    case JCA_STATUS_BAD_SPLIT:
      return "history/candidate token counts differ from the totals given to the stack";
    case JCA_STATUS_TIMEOUT: return "an attention pipeline wait timed out";
    default: return "unknown code";
  }
}
