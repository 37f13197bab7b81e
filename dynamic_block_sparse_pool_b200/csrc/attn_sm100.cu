// Block-sparse attention forward on Blackwell tensor cores (sm_100a):
// TMA loads of the indexed K/V blocks, tcgen05 MMAs with fp32 accumulators
// in tensor memory, online softmax on CUDA cores, warp-specialised and
// persistent.
//
// GSRS (arXiv 2610.21129), abstract: exact attention over the selected
// blocks inside a FlashAttention-style pass that also yields the exact
// per-block attention weights.  DSV (arXiv 2502.07590), abstract: the work
// per query block is skewed, so every query block is its own work item and
// the work items are handed out dynamically.
//
// One CTA per SM.  Each CTA takes CSR rows (one query block of 128 rows
// each) from a ticket counter shared by the launch until none are left, so
// a CTA that drew short rows takes more of them (the balance of one CTA per
// row, without a CTA's start-up and tear-down cost per row).  Ticket t is
// row row_order[t] when an order is given: each head's rows longest first
// put the short rows at the end of the launch, where they fill the gaps
// the last long rows leave.  384 threads:
//   warps 0-7  softmax: warp w owns the 16 query rows (TMEM lanes)
//              32*(w%4) + 16*(w/4) .. +15; thread t of it owns two rows
//              (t/4 and t/4 + 8 of those) and, in every 8-key chunk, keys
//              2*(t%4) and 2*(t%4)+1 (the tcgen05.ld 16x256b layout), so the
//              four threads of a quad share two rows and a row reduction is
//              two quad shuffles; no warp waits for another
//   warp  8    MMA issuer (one thread) and TMEM allocation (whole warp)
//   warp  9    TMA loader of Q and K (one thread)
//   warp 10    TMA loader of V and TMA store of O (one thread)
//   warp 11    row scheduler: draws the next row, checks its column indices
//              and marks its ragged key block while the current row runs
//   warps 8-11 also write each row's O out, one tensor-memory lane quarter
//              (32 rows) each: O / l as bf16 into the V slot of the row's
//              last block (no MMA reads it once that block's PV is done),
//              which warp 10 stores with TMA before the slot takes its next
//              V tile.  The softmax warps only leave 1/l in shared memory
//              and go on to the next row.
// Tensor memory (512 columns): three S buffers at columns 0, 128, 256 and O
// at column 384.  Shared memory: Q, a 3-deep K ring and a 3-deep V ring of
// [128 x D] tiles (a V slot doubles as the staging tile of a row's O), two
// row-descriptor slots, 1/l of two rows.
//
// Blocks are numbered g = 0, 1, 2, ... across all the rows a CTA takes, in
// order; block g uses K/V ring stage g % 3 and S buffer g % 3, so the rings
// and the MMA pipeline run on across row boundaries: the next row's Q and
// first K tiles load while the current row's last blocks are still in the
// softmax.  Within a row the MMA thread issues S(0), S(1), S(2), then for
// every block PV(it) [after P(it) is ready], S(it+3); the next row's S(0..2)
// follow its last PV.  tcgen05 MMAs from one thread execute in order, so
// S(g+3) overwrites buffer g % 3 only after PV(g) has read P(g) from it.  A
// row's first PV overwrites O, so the MMA warp issues it only once warps
// 8-11 have read the previous row's O (OFree); each of them does so at a
// point where it waits for nothing that the next row's PVs produce (the MMA
// warp after the next row's first S products, the Q/K loader after its first
// K tiles, the scheduler once the softmax warps are done with the row, the V
// loader before it refills the staging slot or waits for a descriptor two
// rows on).  The softmax warps can finish the next row before that (a row of
// at most three blocks needs no PV of its own), so 1/l and its LReady
// barrier alternate by row parity; they cannot get two rows ahead, because
// the MMA warp issues the S products of the row after next only after that
// OFree wait.  Q of a row loads once every S of the previous rows is done.
// (A CPU model of this protocol, with random timing, checks that no wait
// skips a phase, nothing deadlocks and no buffer is overwritten early.)
//
// Online softmax with a lazy reference: the first block's row maxima set the
// reference m_ref; later blocks form P = 2^(S*scale*log2e - m_ref) without
// computing their maxima.  P up to 2^64 is harmless (bf16 and fp32 carry it
// as precisely as small values), so only a block whose partial row sums
// reach 2^64 (or overflow) is redone: its maxima become the new reference,
// and O (after PV(it-1) has finished) and the running sums are rescaled.
// O / l and lse use the same reference, so the result is exact.  P is
// written back with the 16x128b layout, which puts each thread's packed key
// pairs exactly where the MMA reads row-major P.
//
// Each selected block's log-sum (for the exact block mass) is
// m_ref + log2(sum of that block's P row), written per query row.
//
// K/V tile of block j: one 3-D TMA box {64 cols, 128 rows, 1 head} per 64
// columns of D over the tensor {D, N, B*H}: rows past N are zero-filled and
// masked to -inf.  No multicast.  Every mbarrier wait is bounded; a timeout
// sets the device error word and the CTA winds down (rows it drew and did
// not finish are left unwritten; the error word reports it).
#include <type_traits>

#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int BM = 128;         // query rows per block row
constexpr int BN = 128;         // keys per key block
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
constexpr int kMmaWarp = 8, kKLoadWarp = 9, kVLoadWarp = 10, kSchedWarp = 11;
constexpr int kStages = 3;      // depth of the K ring and of the V ring
constexpr int kSBufs = 3;       // S/P buffers in tensor memory
constexpr int kRowSlots = 2;    // row descriptors in flight (current, next)
// warps that read a row descriptor: 8 softmax, the MMA issuer, two loaders
constexpr int kRowUsers = kSoftmaxThreads / 32 + 3;
// warps 8-11 also write O out: their tensor-memory lane quarters are 0-3
constexpr int kEpilogueWarps = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 384;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kPMax = 0x1p64f;  // partial row sums at or above this redo the block

// mbarrier slots.  Block g uses stage g % 3 of the K and V rings and S
// buffer g % 3, so one barrier per event serves both the ring and the
// buffer.  Each tcgen05.commit and each fence costs the tensor pipe a few
// dozen cycles, so a block signals only two events:
//   SFull:  S(g) is done -- S is ready for the softmax and K slot is free
//   PVDone: PV(g) is done -- V slot is free, O holds the row through g
static_assert(kStages == kSBufs, "ring stages and S buffers share barriers");
enum : int {
  kBarQ = 0,
  kBarKFull = 1,                        // + stage: K tile landed
  kBarVFull = kBarKFull + kStages,      // + stage: V tile landed
  kBarSFull = kBarVFull + kStages,      // + stage: S(g) done
  kBarPFull = kBarSFull + kStages,      // + stage: P(g) written (one arrival per softmax warp)
  kBarPVDone = kBarPFull + kStages,     // + stage: PV(g) done
  kBarRowFull = kBarPVDone + kStages,   // + slot: row descriptor written
  kBarRowFree = kBarRowFull + kRowSlots,  // + slot: every user is done with it
  kBarOStaged = kBarRowFree + kRowSlots,  // + (row % 3): the row's O is in shared memory
  kBarLReady = kBarOStaged + kStages,   // + (row % 2): the row's 1/l is in shared memory (8 softmax warps)
  kBarOFree = kBarLReady + 2,           // the row's O is read out of tensor memory (4 warps)
  kBarDrain = kBarOFree + 1,            // teardown after an abort: every MMA issued is done
  kNumBars = kBarDrain + 1
};

// A row handed to the CTA.  r < 0: no rows left.  n = 0 for an empty row
// and for a malformed one (flagged in the error word; O = 0, lse = -inf).
struct RowDesc {
  int r;               // CSR row (b*H + h)*nB + i
  int s0;              // its first list position
  int n;               // its number of blocks
  int pad;
  uint32_t ragged[32]; // bit e: list position e (< 1024) holds the ragged last key block
};

template <int D>
struct SmemLayout {
  static constexpr int kTile = BM * D * 2;                // one [128 x D] bf16 tile
  static constexpr int kSub = BM * 64 * 2;                // one 128B-swizzled [128 x 64] sub-tile
  static constexpr int kQ = 0;
  static constexpr int kK = kTile;                        // K ring
  static constexpr int kV = kK + kStages * kTile;         // V ring
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kRow = kBar + 8 * kNumBars;        // RowDesc [kRowSlots]
  static constexpr int kInvL = kRow + kRowSlots * (int)sizeof(RowDesc);  // float [2][128]: 1/l by row parity
  static constexpr int kSlot = kInvL + 2 * BM * 4;                      // TMEM base, abort flag
  static constexpr int kBytes = kSlot + 16;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// log2(x) on the multi-function unit (the PTX approximate base-2 logarithm;
// one instruction, absolute error ~1e-7 for the row sums it is used on).
__device__ __forceinline__ float lg2_mufu(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the multi-function unit (the PTX approximate base-2 exponential).
__device__ __forceinline__ float exp2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Number of the 16 eight-key chunks of each thread's S row pair whose
// exponentials run on the FMA pipe (exp2_poly_x2) instead of the MUFU.  Per
// block the softmax needs 128 x 128 exponentials, 1024 MUFU cycles per SM at
// 16 per clock: as much as the block's MMAs at D = 128 and twice theirs at
// D = 64.  Measured, the MUFU is not what bounds this kernel (moving a
// quarter or half of the exponentials to the FMA pipe made it slower at
// both D), so by default every exponential runs on the MUFU.
#ifndef DSA_POLY_CHUNKS_D64
#define DSA_POLY_CHUNKS_D64 0
#endif
#ifndef DSA_POLY_CHUNKS_D128
#define DSA_POLY_CHUNKS_D128 0
#endif
// Warps 4-7 start their first block once S(1) is ready (half a block behind
// warps 0-3), so the two softmax warps of each SM sub-partition are out of
// phase.
#ifndef DSA_SOFTMAX_LAG
#define DSA_SOFTMAX_LAG 1
#endif
// sleep between polls of the MMA issuer's and the loader's waits (ns)
#ifndef DSA_IDLE_SLEEP_NS
#define DSA_IDLE_SLEEP_NS 0
#endif
constexpr uint32_t kIdleSleepNs = DSA_IDLE_SLEEP_NS;
template <int D>
constexpr int poly_chunks() { return D == 64 ? DSA_POLY_CHUNKS_D64 : DSA_POLY_CHUNKS_D128; }
// chunk k of 16 takes the polynomial path: the kPoly chunks are spread evenly
__host__ __device__ constexpr bool poly_chunk(int k, int kPoly) {
  return (k + 1) * kPoly / 16 != k * kPoly / 16;
}

template <int D>
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int row, int bh,
                                         uint32_t bar) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c)
    tma_load_3d(dst + c * SmemLayout<D>::kSub, map, c * 64, row, bh, bar);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmO, int N, int nB, int rows,
                      float scale_log2, const int32_t* __restrict__ row_ptr,
                      const int32_t* __restrict__ col_idx,
                      const int32_t* __restrict__ row_order, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse, float* __restrict__ blk_lse,
                      unsigned* __restrict__ tickets, unsigned* err) {
  using L = SmemLayout<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, true);
  constexpr uint32_t kTileBytes = L::kTile;
  constexpr int kPoly = poly_chunks<D>();

  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) {
      flag_error(err, kErrAlign);
      // this CTA draws no rows; it still counts as finished
      if (atomicAdd(&tickets[1], 1u) == gridDim.x - 1) {
        atomicExch(&tickets[0], 0u);
        atomicExch(&tickets[1], 0u);
      }
    }
    return;
  }
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  const uint32_t bars = base + L::kBar;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  RowDesc* rdesc = reinterpret_cast<RowDesc*>(smem + L::kRow);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv_last = N - (nB - 1) * BN;  // keys in the last (possibly ragged) block

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int i = 0; i < kNumBars; ++i) {
        uint32_t count = 1;
        if (i >= kBarPFull && i < kBarPFull + kStages) count = kSoftmaxThreads / 32;
        if (i >= kBarRowFree && i < kBarRowFree + kRowSlots) count = kRowUsers;
        if (i >= kBarOStaged && i < kBarOStaged + kStages) count = kEpilogueWarps;
        if (i == kBarLReady || i == kBarLReady + 1) count = kSoftmaxThreads / 32;
        if (i == kBarOFree) count = kEpilogueWarps;
        mbar_init(bar(i), count);
      }
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kKLoadWarp && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
  }
  if (warp == kVLoadWarp && lane == 0) {
    prefetch_tensormap(&tmV);
    prefetch_tensormap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Row descriptor k sits in slot k % 2; RowFull(slot) completes its phase
  // (k / 2) % 2 when the scheduler has written it, RowFree(slot) when its
  // kRowUsers readers are done with it.
  auto row_wait = [&](int k) {
    return mbar_wait_idle(bar(kBarRowFull + (k & 1)), (uint32_t)(k >> 1) & 1u, kIdleSleepNs);
  };
  // The O epilogue of one row, shared by warps 8-11 (each takes the 32 rows
  // of its tensor-memory lane quarter, one row per thread, so the softmax
  // warps go on to the next row at once): O / l as bf16 into the V slot of
  // the row's last block gl (its PV is done, so no MMA reads that slot any
  // more), in the O tensor map's 128-byte-swizzled layout (16-byte chunk k
  // of row r of each 64-column sub-tile at chunk k ^ (r % 8)).  Then the
  // warp arrives on OFree (it has read O: the next row's first PV may
  // overwrite it) and on the row's OStaged (the V loader stores the tile).
  // orow counts the rows with blocks; 1/l comes from the softmax warps
  // (LReady).
  float* inv_l = reinterpret_cast<float*>(smem + L::kInvL);
  auto o_epilogue = [&](uint32_t orow, uint32_t gl) -> bool {
    if (!warp_all(mbar_wait(bar(kBarLReady + (orow & 1u)), (orow >> 1) & 1u))) return false;
    const int row = 32 * (warp & 3) + lane;
    const float inv = inv_l[(orow & 1u) * BM + row];
    if (!warp_all(mbar_wait(bar(kBarPVDone + gl % kStages), (gl / kStages) & 1u))) return false;
    tc_fence_after();
    uint8_t* stage = smem + L::kV + (gl % kStages) * kTileBytes + row * 128;
    const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kTmemO;
#pragma unroll
    for (int c32 = 0; c32 < D / 32; ++c32) {
      uint32_t o[32];  // columns 32 c32 .. 32 c32 + 31 of the thread's row
      tmem_ld32(taddr + 32 * c32, o);
      tmem_wait_ld_regs(o);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = 4 * c32 + j;  // 8-column chunk of the row
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(o[8 * j + 2 * u]) * inv,
                                                          __uint_as_float(o[8 * j + 2 * u + 1]) * inv);
          w[u] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(stage + (ch >> 3) * L::kSub + (((ch & 7) ^ (row & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    fence_proxy_async_smem();  // visible to the TMA store
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(bar(kBarOFree));
      mbar_arrive(bar(kBarOStaged + orow % kStages));
    }
    return true;
  };

  // Blocks issued by the loaders (for the teardown after an abort).
  uint32_t k_issued = 0, v_issued = 0, q_issued = 0;
  bool had_rows = false;  // the MMA issuer issued at least one MMA

  if (warp == kSchedWarp) {
    // -------------------------------------------------------------- scheduler
    bool ok = true;
    uint32_t g = 0, orow = 0;  // blocks and rows with blocks published so far
    // the epilogue share this warp still owes for the row in each slot
    bool owe0 = false, owe1 = false;
    uint32_t orow0 = 0, orow1 = 0, gl0 = 0, gl1 = 0;
    int k = 0;
    for (;; ++k) {
      const int slot = k & 1;
      // slot is free once row k - 2's readers are done with it
      // (a row lasts microseconds: poll every quarter microsecond)
      if (k >= kRowSlots)
        ok = warp_all(mbar_wait_idle(bar(kBarRowFree + slot), (uint32_t)((k - kRowSlots) >> 1) & 1u,
                                     256u));
      // the softmax warps are done with row k - 2: write out its O (this
      // warp's quarter)
      if (ok && (slot ? owe1 : owe0)) ok = o_epilogue(slot ? orow1 : orow0, slot ? gl1 : gl0);
      if (slot) owe1 = false; else owe0 = false;
      if (*abort_flag) ok = false;
      // ticket t is row row_order[t] (t itself without an order); an entry
      // outside [0, rows) is reported and passed over for the next ticket
      int r = rows;
      if (lane == 0 && ok) {
        for (;;) {
          const unsigned t = atomicAdd(&tickets[0], 1u);
          if (t >= (unsigned)rows) break;
          const int o = row_order ? row_order[t] : (int)t;
          if ((unsigned)o < (unsigned)rows) {
            r = o;
            break;
          }
          flag_error(err, kErrRowOrder);
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      RowDesc* d = rdesc + slot;
      if (r >= rows) {
        if (lane == 0) {
          d->r = -1;
          mbar_arrive(bar(kBarRowFull + slot));
        }
        break;
      }
      int s0 = row_ptr[r], s1 = row_ptr[r + 1];
      bool bad = s0 < 0 || s1 < s0;
      if (!bad) {
        for (int e0 = s0; e0 < s1; e0 += 32) {
          const int e = e0 + lane;
          const int j = e < s1 ? col_idx[e] : 0;
          bad |= j < 0 || j >= nB;
          const uint32_t rag = __ballot_sync(0xffffffffu, e < s1 && j == nB - 1 && kv_last < BN);
          const int w = (e0 - s0) >> 5;
          if (lane == 0 && w < 32) d->ragged[w] = rag;
        }
      }
      bad = __any_sync(0xffffffffu, bad);
      const int n = bad ? 0 : s1 - s0;
      if (lane == 0) {
        if (bad) flag_error(err, kErrCsrIndex | kErrRowPtr);
        d->r = r;
        d->s0 = bad ? 0 : s0;
        d->n = n;
        mbar_arrive(bar(kBarRowFull + slot));  // release: the descriptor is visible to the readers
        // the row's Q tile into L2 now: its load then has the current row's
        // time to come from HBM, and the MMA warp can start the row's first
        // S products before the current row's last PV
        if (n > 0) {
          const int bh = r / nB, q0 = (r - bh * nB) * BM;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) tma_prefetch_l2_3d(&tmQ, c * 64, q0, bh);
        }
      }
      if (n > 0) {
        if (slot) {
          owe1 = true;
          orow1 = orow;
          gl1 = g + n - 1;
        } else {
          owe0 = true;
          orow0 = orow;
          gl0 = g + n - 1;
        }
        ++orow;
        g += n;
      }
    }
    // the row before the end marker may still owe its share
    if (ok && k >= 1 && (((k - 1) & 1) ? owe1 : owe0))
      ok = o_epilogue(((k - 1) & 1) ? orow1 : orow0, ((k - 1) & 1) ? gl1 : gl0);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) flag_error(err, kErrTimeout);
    }
  } else if (warp == kKLoadWarp) {
    // ------------------------------------------------------------ Q/K loader
    // The whole warp runs the loop (it also writes out a quarter of each
    // row's O); lane 0 issues the copies.
    const bool leader = lane == 0;
    bool ok = true;
    uint32_t g = 0, orow = 0;  // blocks and rows with blocks so far
    bool owe = false;          // the previous row's epilogue share
    uint32_t owe_orow = 0, owe_gl = 0;
    for (int k = 0; ok; ++k) {
      ok = warp_all(row_wait(k) && !*abort_flag);
      if (!ok) break;
      const RowDesc* d = rdesc + (k & 1);
      const int r = d->r, s0 = d->s0, n = d->n;
      if (r < 0) break;
      __syncwarp();
      if (leader) mbar_arrive(bar(kBarRowFree + (k & 1)));
      if (n == 0) continue;
      const int bh = r / nB, q0 = (r - bh * nB) * BM;
      // Q's buffer is free once every S of the earlier rows is done
      if (g > 0) {
        ok = warp_all(mbar_wait_idle(bar(kBarSFull + (g - 1) % kStages), ((g - 1) / kStages) & 1u,
                                     kIdleSleepNs) && !*abort_flag);
        if (!ok) break;
      }
      if (leader) {
        mbar_expect_tx(bar(kBarQ), kTileBytes);
        tma_tile<D>(sQ, &tmQ, q0, bh, bar(kBarQ));
      }
      ++q_issued;
      for (int it = 0; it < n; ++it, ++g) {
        const uint32_t s = g % kStages;
        // K slot s is free once S(g - 3) is done
        ok = warp_all(mbar_wait_idle(bar(kBarSFull + s), ((g / kStages) & 1u) ^ 1u, kIdleSleepNs) &&
                      !*abort_flag);
        if (!ok) break;
        if (leader) {
          const int j = col_idx[s0 + it];
          mbar_expect_tx(bar(kBarKFull + s), kTileBytes);
          tma_tile<D>(sK + s * kTileBytes, &tmK, j * BN, bh, bar(kBarKFull + s));
        }
        k_issued = g + 1;
        // with this row's first K tiles on their way, write out the
        // previous row's O (the next K tile waits for this row's S(0))
        if (owe && (it == 2 || it == n - 1)) {
          owe = false;
          if (!(ok = o_epilogue(owe_orow, owe_gl))) break;
        }
      }
      if (!ok) break;
      owe = true;
      owe_orow = orow++;
      owe_gl = g - 1;
    }
    if (ok && owe) ok = o_epilogue(owe_orow, owe_gl);
    if (!ok) {
      *abort_flag = 1;
      if (leader) flag_error(err, kErrTimeout);
    }
  } else if (warp == kVLoadWarp) {
    // -------------------------------------------------------------- V loader
    // Also stores O: warps 8-11 leave a row's O (bf16, in the tensor map's
    // 128-byte-swizzled layout) in the V slot of the row's last block, which
    // no MMA reads any more, and this warp stores it with TMA before it loads
    // the next V tile into that slot (or at the end).  The whole warp runs
    // the loop (it writes out a quarter of each row's O); lane 0 issues the
    // copies.
    const bool leader = lane == 0;
    bool ok = true;
    uint32_t g = 0;      // blocks of the rows so far
    uint32_t orows = 0;  // rows with blocks so far
    // rows whose O is not stored yet, oldest first: at most three (their
    // last blocks are among the three blocks before the next V load)
    struct Pending {
      uint32_t last, idx;  // the row's last block; its number among rows with blocks
      int bh, q0, k;       // where its O goes; its descriptor number
      bool shared;         // this warp's quarter of its O is staged
    };
    Pending p0{}, p1{}, p2{};
    int np = 0;
    auto share = [&](Pending& p) -> bool {
      if (p.shared) return true;
      p.shared = true;
      return o_epilogue(p.idx, p.last);
    };
    auto store_o = [&]() -> bool {  // the oldest pending row
      if (!share(p0)) return false;
      if (!warp_all(mbar_wait(bar(kBarOStaged + p0.idx % kStages), (p0.idx / kStages) & 1u)))
        return false;
      if (leader) {
        const uint32_t src = sV + (p0.last % kStages) * kTileBytes;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_store_3d(&tmO, src + c * L::kSub, c * 64, p0.q0, p0.bh);
        tma_store_commit();
        tma_store_wait_read();  // the slot may be refilled now
      }
      __syncwarp();
      p0 = p1;
      p1 = p2;
      --np;
      return true;
    };
    for (int k = 0; ok; ++k) {
      // A row's share of O is written before this warp waits for the
      // descriptor two rows on: that descriptor comes only once the softmax
      // warps are done with the row between, whose first PV waits for the
      // share (OFree).
      if (np > 0 && p0.k <= k - 2 && !(ok = share(p0))) break;
      if (np > 1 && p1.k <= k - 2 && !(ok = share(p1))) break;
      if (np > 2 && p2.k <= k - 2 && !(ok = share(p2))) break;
      ok = warp_all(row_wait(k) && !*abort_flag);
      if (!ok) break;
      const RowDesc* d = rdesc + (k & 1);
      const int r = d->r, s0 = d->s0, n = d->n;
      if (r < 0) break;
      __syncwarp();
      if (leader) mbar_arrive(bar(kBarRowFree + (k & 1)));
      if (n == 0) continue;
      const int bh = r / nB;
      for (int it = 0; it < n; ++it, ++g) {
        const uint32_t s = g % kStages;
        // slot s last held V(g - 3); if that was a row's last block, the
        // row's O is staged there
        if (np > 0 && p0.last + kStages == g && !(ok = store_o())) break;
        // V slot s is free once PV(g - 3) is done
        ok = warp_all(mbar_wait_idle(bar(kBarPVDone + s), ((g / kStages) & 1u) ^ 1u, kIdleSleepNs) &&
                      !*abort_flag);
        if (!ok) break;
        if (leader) {
          const int j = col_idx[s0 + it];
          mbar_expect_tx(bar(kBarVFull + s), kTileBytes);
          tma_tile<D>(sV + s * kTileBytes, &tmV, j * BN, bh, bar(kBarVFull + s));
        }
        v_issued = g + 1;
      }
      if (!ok) break;
      const Pending pr{g - 1, orows++, bh, (r - bh * nB) * BM, k, false};
      if (np == 0) p0 = pr;
      else if (np == 1) p1 = pr;
      else p2 = pr;
      ++np;
    }
    while (ok && np > 0) ok = store_o();
    if (!ok) {
      *abort_flag = 1;
      if (leader) flag_error(err, kErrTimeout);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so the waits, descriptors and addresses
    // stay warp-uniform; lane 0 issues each MMA and commit.  Each ring stage
    // has its own copy of the block step, so stage indices and descriptor
    // offsets are compile-time constants; a switch on g % 3 picks the copy.
    const bool leader = lane == 0;
    // three base descriptors; every other one differs only in its start
    // address field (address >> 4, 14 bits, no carry below 256 KB)
    const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(sK, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(sV, L::kSub, 1024);
    auto kdesc = [](int kk) -> uint64_t {  // K step kk of a K-major tile
      return (uint64_t)(((kk >> 2) * L::kSub + (kk & 3) * 32) >> 4);
    };
    bool ok = true;
    // S(g) = Q K^T into buffer g % 3.  The TMA load and the MMA both act in
    // the async proxy and are ordered by the mbarrier alone.
    auto issue_s = [&](uint32_t gs, auto stage) {
      constexpr int s = decltype(stage)::value;
      if (!(ok = ok && warp_all(mbar_wait_idle(bar(kBarKFull + s), (gs / kStages) & 1u, kIdleSleepNs))))
        return;
      if (leader) {
        const uint32_t d = tmem + 128u * s;
        const uint64_t k0 = dk0 + (uint64_t)((s * kTileBytes) >> 4);
        mma_ss(d, dq0 + kdesc(0), k0 + kdesc(0), kIdescS, 0u);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) mma_ss_acc(d, dq0 + kdesc(kk), k0 + kdesc(kk), kIdescS);
        mma_commit(bar(kBarSFull + s));
      }
      __syncwarp();
    };
    // O (+)= P(g) V(g), P from tensor memory (the row's first block
    // overwrites O); then S(g + 3) into the same buffer if the row has it
    auto block = [&](uint32_t gb, bool first, bool more, auto stage) {
      constexpr int s = decltype(stage)::value;
      const uint32_t ph = (gb / kStages) & 1u;
      if (!(ok = ok && warp_all(mbar_wait_idle(bar(kBarPFull + s), ph, kIdleSleepNs)) &&
                 warp_all(mbar_wait_idle(bar(kBarVFull + s), ph, kIdleSleepNs))))
        return;
      tc_fence_after();
      if (leader) {
        const uint32_t p = tmem + 128u * s;
        const uint64_t v0 = dv0 + (uint64_t)((s * kTileBytes) >> 4);
        if (first)
          mma_ts(tmem + kTmemO, p, v0, kIdescO, 0u);
        else
          mma_ts_acc(tmem + kTmemO, p, v0, kIdescO);
#pragma unroll
        for (int kk = 1; kk < BN / 16; ++kk)
          mma_ts_acc(tmem + kTmemO, p + kk * 8, v0 + (uint64_t)((kk * 2048) >> 4), kIdescO);
        mma_commit(bar(kBarPVDone + s));
      }
      __syncwarp();
      if (more) issue_s(gb + kStages, stage);
    };
    using S0 = std::integral_constant<int, 0>;
    using S1 = std::integral_constant<int, 1>;
    using S2 = std::integral_constant<int, 2>;
    uint32_t g = 0, qrows = 0;
    bool owe = false;  // the previous row's epilogue share
    uint32_t owe_orow = 0, owe_gl = 0;
    int ahead = 0;     // S products of this row issued during the previous one
    uint32_t orow = 0; // rows with blocks so far
    auto issue_s_any = [&](uint32_t gs) {
      switch (gs % kStages) {
        case 0: issue_s(gs, S0{}); break;
        case 1: issue_s(gs, S1{}); break;
        default: issue_s(gs, S2{}); break;
      }
    };
    for (int k = 0; ok; ++k) {
      ok = warp_all(row_wait(k));
      if (!ok) break;
      const RowDesc* d = rdesc + (k & 1);
      const int r = d->r, n = d->n;
      if (r < 0) break;
      __syncwarp();
      if (leader) mbar_arrive(bar(kBarRowFree + (k & 1)));
      if (n == 0) continue;
      const uint32_t this_orow = orow++;
      if (ahead == 0) {
        ok = warp_all(mbar_wait(bar(kBarQ), qrows & 1u));
        ++qrows;
      }
      had_rows = true;
      for (int it = ahead; it < 3 && it < n && ok; ++it) issue_s_any(g + it);
      ahead = 0;
      // With this row's first S products queued, write out the previous
      // row's O (this warp's quarter); this row's first PV overwrites O, so
      // it waits until all four quarters are read (OFree).
      if (ok && owe) {
        owe = false;
        ok = o_epilogue(owe_orow, owe_gl) && warp_all(mbar_wait(bar(kBarOFree), owe_orow & 1u));
      }
      for (int it = 0; it < n && ok; ++it) {
        const uint32_t gb = g + it;
        const bool more = it + kStages < n;
        switch (gb % kStages) {
          case 0: block(gb, it == 0, more, S0{}); break;
          case 1: block(gb, it == 0, more, S1{}); break;
          default: block(gb, it == 0, more, S2{}); break;
        }
        // Before this row's last PV: if the next row is published and its Q
        // has landed, issue its first two S products now (their buffers held
        // P of this row's blocks n-3 and n-2, whose PVs are issued), so they
        // are ready when the softmax warps finish this row.  Checks only: if
        // either is not there yet they follow the last PV as usual.
        if (it == n - 2 && ok) {
          const int k1 = k + 1;
          if (warp_all(mbar_try_wait(bar(kBarRowFull + (k1 & 1)), (uint32_t)(k1 >> 1) & 1u))) {
            const RowDesc* d1 = rdesc + (k1 & 1);
            const int r1 = d1->r, n1 = d1->n;
            if (r1 >= 0 && n1 > 0 && warp_all(mbar_try_wait(bar(kBarQ), qrows & 1u))) {
              ++qrows;
              ahead = n1 >= 2 ? 2 : 1;
              tc_fence_after();
              for (int a = 0; a < ahead && ok; ++a) issue_s_any(g + n + a);
            }
          }
        }
      }
      owe = true;
      owe_orow = this_orow;
      owe_gl = g + n - 1;
      g += n;
    }
    if (ok && owe) ok = o_epilogue(owe_orow, owe_gl);
    if (!ok && leader) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int rbase = 32 * (warp & 3) + 16 * (warp >> 2);  // first of the warp's 16 rows
    const int t0 = lane & 3;
    const int ra = rbase + (lane >> 2), rb = ra + 8;         // this thread's two rows
    const uint32_t lane_off = (uint32_t)rbase << 16;
    bool failed = false;
    uint32_t g = 0;      // blocks of the rows so far
    uint32_t orows = 0;  // rows with blocks so far
    for (int k = 0; !failed; ++k) {
      if (!warp_all(row_wait(k))) {
        failed = true;
        break;
      }
      const RowDesc* d = rdesc + (k & 1);
      const int r = d->r;
      if (r < 0) break;
      const int s0 = d->s0, n = d->n;
      const int bh = r / nB, q0 = (r - bh * nB) * BM;
      const int qlen = min(BM, N - q0);
      float mref_a = -INFINITY, mref_b = -INFINITY;  // reference maxima (log2 units)
      float l_a = 0.f, l_b = 0.f;                    // this thread's share of the row sums
      // Warps 4-7 start each row half a block behind warps 0-3 (they begin
      // once S(1) is ready, one S MMA later than S(0)), so the two softmax
      // warps of each SM sub-partition tend to be out of phase: one is in
      // its exp2 stretch (MUFU-bound) while the other loads, reduces and
      // stores.  (S(g + 4) cannot complete before these warps have produced
      // P(g + 1), so the wait below sees the right phase of buffer g + 1.)
#if DSA_SOFTMAX_LAG
      if ((warp >> 2) == 1 && n > 1) {
        const uint32_t g1 = g + 1;
        if (!warp_all(mbar_wait(bar(kBarSFull + g1 % kSBufs), (g1 / kSBufs) & 1u))) {
          failed = true;
          break;
        }
      }
#endif
      for (int it = 0; it < n; ++it) {
        const uint32_t gb = g + it;
        const uint32_t b = gb % kSBufs;
        const uint32_t tS = tmem + lane_off + 128u * b;
        if (!warp_all(mbar_wait(bar(kBarSFull + b), (gb / kSBufs) & 1u))) {
          failed = true;
          break;
        }
        tc_fence_after();
        // sv[4k + u]: row ra, key 8k + 2*t0 + u; sv[4k + 2 + u]: row rb, same key
        uint32_t sv[64];
        tmem_ld16x256b_x16(tS, sv);
        tmem_wait_ld_regs64(sv);
        const bool rag = it < 1024 ? ((d->ragged[it >> 5] >> (it & 31)) & 1u)
                                   : (kv_last < BN && col_idx[s0 + it] == nB - 1);
        if (rag) {
#pragma unroll
          for (int kc = 0; kc < 16; ++kc)
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (8 * kc + 2 * t0 + u >= kv_last) {
                sv[4 * kc + u] = __float_as_uint(-INFINITY);
                sv[4 * kc + 2 + u] = __float_as_uint(-INFINITY);
              }
        }
        // The exps run against the reference; the row maxima are computed
        // only for the first block, or when a thread's partial row sums show
        // the reference has fallen far below this block's maxima.
        const uint64_t sc2 = pack_f32x2(scale_log2, scale_log2);
        uint32_t pk[32];
        float rs_a = 0.f, rs_b = 0.f;
        auto exps = [&]() {
          const uint64_t na2 = pack_f32x2(-mref_a, -mref_a), nb2 = pack_f32x2(-mref_b, -mref_b);
          uint64_t rsa2[2] = {0ull, 0ull}, rsb2[2] = {0ull, 0ull};
#pragma unroll
          for (int kc = 0; kc < 16; ++kc) {
            float a0, a1, b0, b1;
            const uint64_t xa = fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * kc]), __uint_as_float(sv[4 * kc + 1])), sc2, na2);
            const uint64_t xb = fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * kc + 2]), __uint_as_float(sv[4 * kc + 3])), sc2, nb2);
            if (poly_chunk(kc, kPoly)) {
              unpack_f32x2(exp2_poly_x2(xa), a0, a1);
              unpack_f32x2(exp2_poly_x2(xb), b0, b1);
            } else {
              unpack_f32x2(xa, a0, a1);
              unpack_f32x2(xb, b0, b1);
              a0 = exp2_mufu(a0);
              a1 = exp2_mufu(a1);
              b0 = exp2_mufu(b0);
              b1 = exp2_mufu(b1);
            }
            rsa2[kc & 1] = add_f32x2(rsa2[kc & 1], pack_f32x2(a0, a1));
            rsb2[kc & 1] = add_f32x2(rsb2[kc & 1], pack_f32x2(b0, b1));
            const __nv_bfloat162 ha = __floats2bfloat162_rn(a0, a1);
            const __nv_bfloat162 hb = __floats2bfloat162_rn(b0, b1);
            pk[2 * kc] = *reinterpret_cast<const uint32_t*>(&ha);
            pk[2 * kc + 1] = *reinterpret_cast<const uint32_t*>(&hb);
          }
          float u0, u1, u2, u3;
          unpack_f32x2(add_f32x2(rsa2[0], rsa2[1]), u0, u1);
          unpack_f32x2(add_f32x2(rsb2[0], rsb2[1]), u2, u3);
          rs_a = u0 + u1;
          rs_b = u2 + u3;
        };
        float alpha_a = 1.0f, alpha_b = 1.0f;
        bool warp_need = false;
        auto new_reference = [&]() {
          float ma4[4], mb4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ma4[u] = fmaxf(__uint_as_float(sv[4 * u]), __uint_as_float(sv[4 * u + 1]));
            mb4[u] = fmaxf(__uint_as_float(sv[4 * u + 2]), __uint_as_float(sv[4 * u + 3]));
          }
#pragma unroll
          for (int kc = 4; kc < 16; ++kc) {
            ma4[kc & 3] = max3f(ma4[kc & 3], __uint_as_float(sv[4 * kc]), __uint_as_float(sv[4 * kc + 1]));
            mb4[kc & 3] = max3f(mb4[kc & 3], __uint_as_float(sv[4 * kc + 2]), __uint_as_float(sv[4 * kc + 3]));
          }
          float ma = max3f(ma4[0], ma4[1], fmaxf(ma4[2], ma4[3]));
          float mb = max3f(mb4[0], mb4[1], fmaxf(mb4[2], mb4[3]));
          ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
          ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
          const float xa = ma * scale_log2, xb = mb * scale_log2;
          const bool need_a = xa > mref_a, need_b = xb > mref_b;
          warp_need = __any_sync(0xffffffffu, need_a || need_b);
          if (need_a) {
            alpha_a = exp2f(mref_a - xa);  // 0 on the first block
            l_a *= alpha_a;
            mref_a = xa;
          }
          if (need_b) {
            alpha_b = exp2f(mref_b - xb);
            l_b *= alpha_b;
            mref_b = xb;
          }
        };
        if (it == 0) new_reference();
        exps();
        if (it > 0 && __any_sync(0xffffffffu, !(rs_a < kPMax) || !(rs_b < kPMax))) {
          new_reference();
          exps();
        }
        tmem_st16x128b_x16(tS, pk);
        if (warp_need && it > 0) {
          // O holds the sum through block it-1; wait for PV(it-1), then move
          // O to the new reference before PV(it) accumulates onto it
          const uint32_t gp = gb - 1;
          if (!warp_all(mbar_wait(bar(kBarPVDone + gp % kStages), (gp / kStages) & 1u))) {
            failed = true;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_off + kTmemO + 64 * c;
            tmem_ld16x256b_x8(ta, o);
            tmem_wait_ld_regs(o);
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
              o[4 * kc] = __float_as_uint(__uint_as_float(o[4 * kc]) * alpha_a);
              o[4 * kc + 1] = __float_as_uint(__uint_as_float(o[4 * kc + 1]) * alpha_a);
              o[4 * kc + 2] = __float_as_uint(__uint_as_float(o[4 * kc + 2]) * alpha_b);
              o[4 * kc + 3] = __float_as_uint(__uint_as_float(o[4 * kc + 3]) * alpha_b);
            }
            tmem_st16x256b_x8(ta, o);
          }
        }
        l_a += rs_a;
        l_b += rs_b;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull + b));
        if (blk_lse != nullptr) {
          // the block's share of each row's denominator: sum over the quad
          float ta = rs_a + __shfl_xor_sync(0xffffffffu, rs_a, 1);
          float tb = rs_b + __shfl_xor_sync(0xffffffffu, rs_b, 1);
          ta += __shfl_xor_sync(0xffffffffu, ta, 2);
          tb += __shfl_xor_sync(0xffffffffu, tb, 2);
          if (t0 == 0) {
            if (ra < qlen) blk_lse[(size_t)(s0 + it) * BN + ra] = (mref_a + lg2_mufu(ta)) * kLn2;
            if (rb < qlen) blk_lse[(size_t)(s0 + it) * BN + rb] = (mref_b + lg2_mufu(tb)) * kLn2;
          }
        }
      }
      if (failed) break;

      if (n > 0) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        // lse, and 1/l for the warps that write O out (warps 8-11, once the
        // last PV is done); this warp goes on to the next row at once
        if (t0 == 0) {
          if (lse != nullptr) {
            if (ra < qlen) lse[(size_t)bh * N + q0 + ra] = (mref_a + log2f(l_a)) * kLn2;
            if (rb < qlen) lse[(size_t)bh * N + q0 + rb] = (mref_b + log2f(l_b)) * kLn2;
          }
          inv_l[(orows & 1u) * BM + ra] = 1.0f / l_a;
          inv_l[(orows & 1u) * BM + rb] = 1.0f / l_b;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarLReady + (orows & 1u)));  // release: 1/l is visible
        ++orows;
      } else {
        __nv_bfloat16* ra_out = out + ((size_t)bh * N + q0 + ra) * D;
        __nv_bfloat16* rb_out = out + ((size_t)bh * N + q0 + rb) * D;
#pragma unroll
        for (int h = 0; h < D / 32; ++h) {
          if (ra < qlen) *reinterpret_cast<uint4*>(ra_out + 8 * (4 * h + t0)) = make_uint4(0u, 0u, 0u, 0u);
          if (rb < qlen) *reinterpret_cast<uint4*>(rb_out + 8 * (4 * h + t0)) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (t0 == 0 && lse != nullptr) {
          if (ra < qlen) lse[(size_t)bh * N + q0 + ra] = -INFINITY;
          if (rb < qlen) lse[(size_t)bh * N + q0 + rb] = -INFINITY;
        }
      }
      // done with this row's descriptor (its ragged marks)
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarRowFree + (k & 1)));
      g += n;
    }
    if (failed) {
      *abort_flag = 1;
      if (lane == 0) flag_error(err, kErrTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A role gave up: copies and MMAs may still be in flight.  Let every one
    // of them finish (bounded) before shared and tensor memory are released.
    if (warp == kMmaWarp && had_rows) {
      if (lane == 0) {
        mma_commit(bar(kBarDrain));  // arrives once all MMAs issued so far are done
        mbar_wait(bar(kBarDrain), 0u);
      }
      __syncwarp();
    } else if (warp == kKLoadWarp && lane == 0) {
      for (uint32_t b = k_issued > kStages ? k_issued - kStages : 0; b < k_issued; ++b)
        mbar_wait(bar(kBarKFull + b % kStages), (b / kStages) & 1u);
      if (q_issued > 0) mbar_wait(bar(kBarQ), (q_issued - 1) & 1u);
    } else if (warp == kVLoadWarp && lane == 0) {
      for (uint32_t b = v_issued > kStages ? v_issued - kStages : 0; b < v_issued; ++b)
        mbar_wait(bar(kBarVFull + b % kStages), (b / kStages) & 1u);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // The last CTA to finish resets the launch's ticket counter for the next
  // launch that uses it (every CTA has drawn its last ticket by now).
  if (tid == 0 && atomicAdd(&tickets[1], 1u) == gridDim.x - 1) {
    atomicExch(&tickets[0], 0u);
    atomicExch(&tickets[1], 0u);
  }
}


// cuTensorMapEncodeTiled, looked up once through the runtime (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

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

// [B*H, N, D] bf16 viewed as a 3-D tensor {D, N, B*H}; boxes of 64 x 128 x 1.
bool make_tile_map(CUtensorMap* map, const void* ptr, int BH, int N, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mo, int BH, int N, float scale, const int32_t* row_ptr, const int32_t* col_idx,
                     const int32_t* row_order, void* out, float* lse, float* blk_lse, unsigned* tickets, int num_sms,
                     unsigned* err, cudaStream_t s) {
  const int nB = ceil_div(N, BN);
  const int rows = BH * nB;
  if (rows == 0) return cudaSuccess;
  const int smem = SmemLayout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  // one CTA per SM (384 threads at up to 168 registers fill an SM's register
  // file, so no second CTA fits beside one)
  const int grid = rows < num_sms ? rows : num_sms;
  attn_fwd_sm100_kernel<D><<<grid, kThreads, smem, s>>>(
      mq, mk, mv, mo, N, nB, rows, scale_log2, row_ptr, col_idx, row_order, static_cast<__nv_bfloat16*>(out),
      lse, blk_lse, tickets, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, int BH, int N,
                              int D, float scale, const int32_t* row_ptr,
                              const int32_t* col_idx, const int32_t* row_order, void* out,
                              float* lse, float* blk_lse, unsigned* tickets, int num_sms,
                              unsigned* err, cudaStream_t s, const char** why) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map(&mq, q, BH, N, D) || !make_tile_map(&mk, k, BH, N, D) ||
      !make_tile_map(&mv, v, BH, N, D) || !make_tile_map(&mo, out, BH, N, D)) {
    if (why) *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  if (D == 64)
    return launch_d<64>(mq, mk, mv, mo, BH, N, scale, row_ptr, col_idx, row_order, out, lse,
                        blk_lse, tickets, num_sms, err, s);
  return launch_d<128>(mq, mk, mv, mo, BH, N, scale, row_ptr, col_idx, row_order, out, lse,
                       blk_lse, tickets, num_sms, err, s);
}

}  // namespace dsa
