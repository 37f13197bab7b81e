// Block-sparse attention forward on Blackwell tensor cores (sm_100a):
// TMA loads of the indexed K/V blocks, tcgen05 MMAs with fp32 accumulators
// in tensor memory, online softmax on CUDA cores, warp-specialised.
//
// GSRS (arXiv 2610.21129), abstract: exact attention over the selected
// blocks inside a FlashAttention-style pass that also yields the exact
// per-block attention weights.  DSV (arXiv 2502.07590), abstract: the work
// per query block is skewed, so every query block is its own work item.
//
// One CTA per CSR row (one query block of 128 rows).  320 threads:
//   warps 0-7  softmax: warp w owns the 16 query rows (TMEM lanes)
//              32*(w%4) + 16*(w/4) .. +15; thread t of it owns two rows
//              (t/4 and t/4 + 8 of those) and, in every 8-key chunk, keys
//              2*(t%4) and 2*(t%4)+1 (the tcgen05.ld 16x256b layout), so the
//              four threads of a quad share two rows and a row reduction is
//              two quad shuffles; no warp waits for another
//   warp  8    MMA issuer (one thread) and TMEM allocation (whole warp)
//   warp  9    TMA loader (one thread)
// Tensor memory (512 columns): three S buffers at columns 0, 128, 256 (S of
// block it in buffer it % 3; P, packed bf16 pairs, overwrites the first 64
// columns of its buffer) and O at column 384.
// Shared memory: Q, a 3-deep K ring and a 3-deep V ring of [128 x D] tiles.
//
// Pipeline.  The MMA thread issues S(0), S(1), S(2), then for every block
//   PV(it) [after P(it) is ready], S(it+3)
// so two S tiles are computed ahead of the softmax, and the softmax warps
// go from block to block without waiting for the tensor cores.  tcgen05 MMAs
// from one thread execute in order: S(it+3) overwrites buffer it % 3 only
// after PV(it) has read P(it) from it.
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
// sets the device error word and the CTA winds down.
#include <type_traits>

#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int BM = 128;         // query rows per CTA (one query block)
constexpr int BN = 128;         // keys per key block
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kMmaWarp = 8, kLoadWarp = 9;
constexpr int kStages = 3;      // depth of the K ring and of the V ring
constexpr int kSBufs = 3;       // S/P buffers in tensor memory
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 384;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kPMax = 0x1p64f;  // partial row sums at or above this redo the block

// mbarrier slots, one per ring stage (block it uses stage it % 3 of the K
// and V rings and S buffer it % 3, so one barrier per event serves both the
// ring and the buffer).  Each tcgen05.commit and each fence costs the tensor
// pipe a few dozen cycles, so a block signals only two events:
//   SFull:  S(it) is done -- S is ready for the softmax and K slot is free
//   PVDone: PV(it) is done -- V slot is free, O holds blocks 0..it
static_assert(kStages == kSBufs, "ring stages and S buffers share barriers");
enum : int {
  kBarQ = 0,
  kBarKFull = 1,                        // + stage: K tile landed
  kBarVFull = kBarKFull + kStages,      // + stage: V tile landed
  kBarSFull = kBarVFull + kStages,      // + stage: S(it) done
  kBarPFull = kBarSFull + kStages,      // + stage: P(it) written (one arrival per softmax warp)
  kBarPVDone = kBarPFull + kStages,     // + stage: PV(it) done
  kBarDrain = kBarPVDone + kStages,     // teardown after an abort: every MMA issued is done
  kNumBars = kBarDrain + 1
};

template <int D>
struct SmemLayout {
  static constexpr int kTile = BM * D * 2;                // one [128 x D] bf16 tile
  static constexpr int kSub = BM * 64 * 2;                // one 128B-swizzled [128 x 64] sub-tile
  static constexpr int kQ = 0;
  static constexpr int kK = kTile;                        // K ring
  static constexpr int kV = kK + kStages * kTile;         // V ring
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kRagged = kBar + 8 * kNumBars;     // uint32 [32]: list positions of the ragged block
  static constexpr int kSlot = kRagged + 32 * 4;          // TMEM base, abort flag
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

// 2^x for a pair of fp32 values on the FMA pipe.  Range reduction in the
// manner of Cody and Waite for base 2: x = j + r with j = round(x), taken by
// adding the shifter 1.5 * 2^23 (the sum keeps j in its low mantissa bits)
// and r = x - j in [-0.5, 0.5]; 2^r by the degree-4 polynomial of least
// maximum relative error on [-0.5, 0.5] (Remez exchange, error 2.6e-6, 2.7e-6
// when evaluated in fp32); 2^j by adding j to the exponent field of 2^r.  x is
// clamped to [-126, 127] first, so the exponent stays in range: results
// below 2^-126 come out as about 2^-126 instead of 0, and anything that
// would overflow comes out at or above 2^126.5.
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99999928474426270f, c1 = 0.69312179088592529f,
                  c2 = 0.24024743318367004f, c3 = 0.055917859077453613f,
                  c4 = 0.0095701022073626518f;
  float x0, x1;
  unpack_f32x2(x2, x0, x1);
  x0 = fminf(fmaxf(x0, -126.0f), 127.0f);
  x1 = fminf(fmaxf(x1, -126.0f), 127.0f);
  const uint64_t xc = pack_f32x2(x0, x1);
  const uint64_t t = add_f32x2(xc, pack_f32x2(kShift, kShift));     // shifter + j
  const uint64_t j = add_f32x2(t, pack_f32x2(-kShift, -kShift));    // j, exactly
  const uint64_t r = fma_f32x2(j, pack_f32x2(-1.0f, -1.0f), xc);    // x - j, exactly
  uint64_t p = fma_f32x2(pack_f32x2(c4, c4), r, pack_f32x2(c3, c3));
  p = fma_f32x2(p, r, pack_f32x2(c2, c2));
  p = fma_f32x2(p, r, pack_f32x2(c1, c1));
  p = fma_f32x2(p, r, pack_f32x2(c0, c0));
  float t0, t1, p0, p1;
  unpack_f32x2(t, t0, t1);
  unpack_f32x2(p, p0, p1);
  // (shifter + j) << 23 leaves j << 23 (the shifter's bits shift out)
  const uint32_t e0 = __float_as_uint(p0) + (__float_as_uint(t0) << 23);
  const uint32_t e1 = __float_as_uint(p1) + (__float_as_uint(t1) << 23);
  return pack_f32x2(__uint_as_float(e0), __uint_as_float(e1));
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
                      const __grid_constant__ CUtensorMap tmO, int N, int nB,
                      float scale_log2, const int32_t* __restrict__ row_ptr,
                      const int32_t* __restrict__ col_idx, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse, float* __restrict__ blk_lse, unsigned* err) {
  using L = SmemLayout<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, true);
  constexpr uint32_t kTileBytes = L::kTile;
  constexpr int kHalfD = D / 2;   // O columns owned by each half of a row
  constexpr int kPoly = poly_chunks<D>();
  constexpr bool kTmaStoreO = D == 128;  // O leaves through shared memory and one TMA store

  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) flag_error(err, kErrAlign);
    return;
  }
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  const uint32_t bars = base + L::kBar;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* ragged_bits = reinterpret_cast<uint32_t*>(smem + L::kRagged);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;
  const int bh = r / nB, qi = r - bh * nB;
  const int q0 = qi * BM;
  const int qlen = min(BM, N - q0);
  const int kv_last = N - (nB - 1) * BN;  // keys in the last (possibly ragged) block

  if (tid < 32) ragged_bits[tid] = 0u;
  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int i = 0; i < kNumBars; ++i)
        mbar_init(bar(i), (i >= kBarPFull && i < kBarPFull + kStages) ? kSoftmaxThreads / 32 : 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    prefetch_tensormap(&tmO);
  }
  __syncthreads();

  // validate the row and mark where the ragged last key block sits in it
  int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  bool bad = s0 < 0 || s1 < s0;
  if (!bad)
    for (int e = s0 + tid; e < s1; e += kThreads) {
      const int j = col_idx[e];
      bad |= (j < 0 || j >= nB);
      if (j == nB - 1 && kv_last < BN && e - s0 < 1024)
        atomicOr(&ragged_bits[(e - s0) >> 5], 1u << ((e - s0) & 31));
    }
  tc_fence_before();
  const bool any_bad = __syncthreads_or(bad);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (any_bad) {
    if (tid == 0) flag_error(err, kErrCsrIndex | kErrRowPtr);
    s1 = s0;
  }
  const int n = s1 - s0;
  int k_issued = 0, v_issued = 0;  // loader: blocks whose K / V loads were issued

  if (warp == kLoadWarp) {
    // ---------------------------------------------------------------- loader
    if (lane == 0 && n > 0) {
      // K runs kKLead blocks ahead of V: S(it) needs K(it) a block earlier
      // than PV(it) needs V(it), and K(it + 3)'s slot frees as soon as S(it)
      // is done, so K gets about three block periods to arrive from L2.
      constexpr int kKLead = 2;
      bool ok = true;
      mbar_expect_tx(bar(kBarQ), kTileBytes);
      tma_tile<D>(sQ, &tmQ, q0, bh, bar(kBarQ));
      for (int step = 0; step < n + kKLead && ok; ++step) {
        if (step < n) {
          const int it = step, s = it % kStages;
          const int j = col_idx[s0 + it];
          // K slot s is free once S(it - 3) is done
          ok = mbar_wait_idle(bar(kBarSFull + s), ((uint32_t)(it / kStages) & 1u) ^ 1u, kIdleSleepNs) && !*abort_flag;
          if (!ok) break;
          mbar_expect_tx(bar(kBarKFull + s), kTileBytes);
          tma_tile<D>(sK + s * kTileBytes, &tmK, j * BN, bh, bar(kBarKFull + s));
          k_issued = it + 1;
        }
        if (step >= kKLead) {
          const int it = step - kKLead, s = it % kStages;
          const int j = col_idx[s0 + it];
          // V slot s is free once PV(it - 3) is done
          ok = mbar_wait_idle(bar(kBarPVDone + s), ((uint32_t)(it / kStages) & 1u) ^ 1u, kIdleSleepNs) && !*abort_flag;
          if (!ok) break;
          mbar_expect_tx(bar(kBarVFull + s), kTileBytes);
          tma_tile<D>(sV + s * kTileBytes, &tmV, j * BN, bh, bar(kBarVFull + s));
          v_issued = it + 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so the waits, descriptors and addresses
    // stay warp-uniform; lane 0 issues each MMA and commit.  The issuing warp
    // shares its SM sub-partition with two busy softmax warps, so every
    // instruction it saves shortens the tensor pipe's gaps.  The block loop
    // is unrolled by the ring depth, which makes every stage index and
    // descriptor offset a compile-time constant.
    if (n > 0) {
      const bool leader = lane == 0;
      // three base descriptors; every other one differs only in its start
      // address field (address >> 4, 14 bits, no carry below 256 KB)
      const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sV, L::kSub, 1024);
      auto kdesc = [](int kk) -> uint64_t {  // K step kk of a K-major tile
        return (uint64_t)(((kk >> 2) * L::kSub + (kk & 3) * 32) >> 4);
      };
      bool ok = warp_all(mbar_wait(bar(kBarQ), 0u));
      // S(it) = Q K^T into buffer it % 3.  The TMA load and the MMA both act
      // in the async proxy and are ordered by the mbarrier alone.
      auto issue_s = [&](int it, auto stage) {
        constexpr int s = decltype(stage)::value;
        if (!(ok = ok && warp_all(mbar_wait_idle(bar(kBarKFull + s), (uint32_t)(it / kStages) & 1u, kIdleSleepNs))))
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
      // O += P(it) V(it), P from tensor memory; then S(it + 3) into the same buffer
      auto block = [&](int it, auto stage) {
        constexpr int s = decltype(stage)::value;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!(ok = ok && warp_all(mbar_wait_idle(bar(kBarPFull + s), ph, kIdleSleepNs)) &&
                   warp_all(mbar_wait_idle(bar(kBarVFull + s), ph, kIdleSleepNs))))
          return;
        tc_fence_after();
        if (leader) {
          const uint32_t p = tmem + 128u * s;
          const uint64_t v0 = dv0 + (uint64_t)((s * kTileBytes) >> 4);
          if (it == 0)
            mma_ts(tmem + kTmemO, p, v0, kIdescO, 0u);
          else
            mma_ts_acc(tmem + kTmemO, p, v0, kIdescO);
#pragma unroll
          for (int kk = 1; kk < BN / 16; ++kk)
            mma_ts_acc(tmem + kTmemO, p + kk * 8, v0 + (uint64_t)((kk * 2048) >> 4), kIdescO);
          mma_commit(bar(kBarPVDone + s));
        }
        __syncwarp();
        if (it + kStages < n) issue_s(it + kStages, stage);
      };
      using S0 = std::integral_constant<int, 0>;
      using S1 = std::integral_constant<int, 1>;
      using S2 = std::integral_constant<int, 2>;
      issue_s(0, S0{});
      if (n > 1) issue_s(1, S1{});
      if (n > 2) issue_s(2, S2{});
      for (int it = 0; it < n && ok; it += kStages) {
        block(it, S0{});
        if (it + 1 < n) block(it + 1, S1{});
        if (it + 2 < n) block(it + 2, S2{});
      }
      if (!ok && leader) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int rbase = 32 * (warp & 3) + 16 * (warp >> 2);  // first of the warp's 16 rows
    const int t0 = lane & 3;
    const int ra = rbase + (lane >> 2), rb = ra + 8;         // this thread's two rows
    const uint32_t lane_off = (uint32_t)rbase << 16;
    float mref_a = -INFINITY, mref_b = -INFINITY;  // reference maxima (log2 units)
    float l_a = 0.f, l_b = 0.f;                    // this thread's share of the row sums
    bool failed = false;
    // Warps 4-7 start half a block behind warps 0-3 (they begin once S(1) is
    // ready, one S MMA later than S(0)), so the two softmax warps of each SM
    // sub-partition are out of phase: one is in its exp2 stretch (MUFU-bound)
    // while the other loads, reduces and stores.  The lag is stable: S is
    // triple-buffered and the leading warps never wait for the trailing ones
    // except through PV(it) -> S(it + 3).  (S(4) cannot complete before these
    // warps have produced P(1), so the wait below sees the first phase of
    // buffer 1.)
#if DSA_SOFTMAX_LAG
    if ((warp >> 2) == 1 && n > 1) {
      if (!warp_all(mbar_wait(bar(kBarSFull + 1), 0u))) failed = true;
    }
#endif
    for (int it = 0; it < n && !failed; ++it) {
      const int b = it % kSBufs;
      const uint32_t tS = tmem + lane_off + 128u * (uint32_t)b;
      if (!warp_all(mbar_wait(bar(kBarSFull + b), (uint32_t)(it / kSBufs) & 1u))) {
        failed = true;
        break;
      }
      tc_fence_after();
      // sv[4k + u]: row ra, key 8k + 2*t0 + u; sv[4k + 2 + u]: row rb, same key
      uint32_t sv[64];
      tmem_ld16x256b_x16(tS, sv);
      tmem_wait_ld_regs64(sv);
      const bool rag = it < 1024 ? ((ragged_bits[it >> 5] >> (it & 31)) & 1u)
                                 : (kv_last < BN && col_idx[s0 + it] == nB - 1);
      if (rag) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (8 * k + 2 * t0 + u >= kv_last) {
              sv[4 * k + u] = __float_as_uint(-INFINITY);
              sv[4 * k + 2 + u] = __float_as_uint(-INFINITY);
            }
      }
      // The exps run against the reference; the row maxima are computed only
      // for the first block, or when a thread's partial row sums show the
      // reference has fallen far below this block's maxima.
      const uint64_t sc2 = pack_f32x2(scale_log2, scale_log2);
      uint32_t pk[32];
      float rs_a = 0.f, rs_b = 0.f;
      auto exps = [&]() {
        const uint64_t na2 = pack_f32x2(-mref_a, -mref_a), nb2 = pack_f32x2(-mref_b, -mref_b);
        uint64_t rsa2[2] = {0ull, 0ull}, rsb2[2] = {0ull, 0ull};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float a0, a1, b0, b1;
          const uint64_t xa = fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * k]), __uint_as_float(sv[4 * k + 1])), sc2, na2);
          const uint64_t xb = fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * k + 2]), __uint_as_float(sv[4 * k + 3])), sc2, nb2);
          if (poly_chunk(k, kPoly)) {
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
          rsa2[k & 1] = add_f32x2(rsa2[k & 1], pack_f32x2(a0, a1));
          rsb2[k & 1] = add_f32x2(rsb2[k & 1], pack_f32x2(b0, b1));
          const __nv_bfloat162 ha = __floats2bfloat162_rn(a0, a1);
          const __nv_bfloat162 hb = __floats2bfloat162_rn(b0, b1);
          pk[2 * k] = *reinterpret_cast<const uint32_t*>(&ha);
          pk[2 * k + 1] = *reinterpret_cast<const uint32_t*>(&hb);
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
        for (int k = 4; k < 16; ++k) {
          ma4[k & 3] = max3f(ma4[k & 3], __uint_as_float(sv[4 * k]), __uint_as_float(sv[4 * k + 1]));
          mb4[k & 3] = max3f(mb4[k & 3], __uint_as_float(sv[4 * k + 2]), __uint_as_float(sv[4 * k + 3]));
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
        // O holds the sum through block it-1; wait for PV(it-1), then move O to
        // the new reference before PV(it) accumulates onto it
        const int pb = (it - 1) % kStages;
        if (!warp_all(mbar_wait(bar(kBarPVDone + pb), (uint32_t)((it - 1) / kStages) & 1u))) {
          *abort_flag = 1;
        } else {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_off + kTmemO + 64 * c;
            tmem_ld16x256b_x8(ta, o);
            tmem_wait_ld_regs(o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[4 * k] = __float_as_uint(__uint_as_float(o[4 * k]) * alpha_a);
              o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * alpha_a);
              o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * alpha_b);
              o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * alpha_b);
            }
            tmem_st16x256b_x8(ta, o);
          }
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

    bool o_ok = false;  // this warp's rows of O are in shared memory
    if (failed) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
    } else if (n > 0) {
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      if (!warp_all(mbar_wait(bar(kBarPVDone + (n - 1) % kStages), (uint32_t)((n - 1) / kStages) & 1u))) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      } else {
        tc_fence_after();
        const float inv_a = 1.0f / l_a, inv_b = 1.0f / l_b;
        // D = 128: O / l as bf16 into the Q tile's shared memory (every MMA,
        // and so every read of Q, is done), in the 128-byte-swizzled layout
        // of the tensor map (16-byte chunk k of row r sits at chunk
        // k ^ (r % 8)), for one TMA store below.  D = 64: straight to global
        // memory (measured faster there).
        uint8_t* sa = smem + L::kQ + ra * 128 + 4 * t0;
        uint8_t* sb = smem + L::kQ + rb * 128 + 4 * t0;
        __nv_bfloat16* ga = out + ((size_t)bh * N + q0 + ra) * D + 2 * t0;
        __nv_bfloat16* gb = out + ((size_t)bh * N + q0 + rb) * D + 2 * t0;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[32];
          tmem_ld16x256b_x8(tmem + lane_off + kTmemO + 64 * c, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const __nv_bfloat162 ha = __floats2bfloat162_rn(__uint_as_float(o[4 * k]) * inv_a,
                                                            __uint_as_float(o[4 * k + 1]) * inv_a);
            const __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(o[4 * k + 2]) * inv_b,
                                                            __uint_as_float(o[4 * k + 3]) * inv_b);
            if (kTmaStoreO) {
              *reinterpret_cast<__nv_bfloat162*>(sa + c * L::kSub + ((k ^ (ra & 7)) << 4)) = ha;
              *reinterpret_cast<__nv_bfloat162*>(sb + c * L::kSub + ((k ^ (rb & 7)) << 4)) = hb;
            } else {
              if (ra < qlen) *reinterpret_cast<__nv_bfloat162*>(ga + 64 * c + 8 * k) = ha;
              if (rb < qlen) *reinterpret_cast<__nv_bfloat162*>(gb + 64 * c + 8 * k) = hb;
            }
          }
        }
        if (kTmaStoreO) fence_proxy_async_smem();
        o_ok = true;
        if (t0 == 0 && lse != nullptr) {
          if (ra < qlen) lse[(size_t)bh * N + q0 + ra] = (mref_a + log2f(l_a)) * kLn2;
          if (rb < qlen) lse[(size_t)bh * N + q0 + rb] = (mref_b + log2f(l_b)) * kLn2;
        }
      }
    } else {
      const __nv_bfloat162 z = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < D / 8; ++k) {
        if (ra < qlen) *reinterpret_cast<__nv_bfloat162*>(out + ((size_t)bh * N + q0 + ra) * D + 8 * k + 2 * t0) = z;
        if (rb < qlen) *reinterpret_cast<__nv_bfloat162*>(out + ((size_t)bh * N + q0 + rb) * D + 8 * k + 2 * t0) = z;
      }
      if (t0 == 0 && lse != nullptr) {
        if (ra < qlen) lse[(size_t)bh * N + q0 + ra] = -INFINITY;
        if (rb < qlen) lse[(size_t)bh * N + q0 + rb] = -INFINITY;
      }
    }
    if (kTmaStoreO && n > 0) {
      // Every softmax warp arrives here, the ones that gave up too, so none
      // waits alone; then one thread stores the O tile with TMA (rows past N
      // fall outside the tensor and are not written) and waits until the
      // copy has read shared memory.
      const bool any_fail = named_bar_or(1, kSoftmaxThreads, !o_ok);
      if (!any_fail && tid == 0) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_store_3d(&tmO, sQ + c * L::kSub, c * 64, q0, bh);
        tma_store_commit();
        tma_store_wait_read();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A role gave up: copies and MMAs may still be in flight.  Let every one
    // of them finish (bounded) before shared and tensor memory are released.
    if (warp == kMmaWarp && n > 0) {
      if (lane == 0) {
        mma_commit(bar(kBarDrain));  // arrives once all MMAs issued so far are done
        mbar_wait(bar(kBarDrain), 0u);
      }
      __syncwarp();
    } else if (warp == kLoadWarp && lane == 0 && n > 0) {
      for (int b = k_issued - kStages > 0 ? k_issued - kStages : 0; b < k_issued; ++b)
        mbar_wait(bar(kBarKFull + b % kStages), (uint32_t)(b / kStages) & 1u);
      for (int b = v_issued - kStages > 0 ? v_issued - kStages : 0; b < v_issued; ++b)
        mbar_wait(bar(kBarVFull + b % kStages), (uint32_t)(b / kStages) & 1u);
      mbar_wait(bar(kBarQ), 0u);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
                     const CUtensorMap& mo, int BH,
                     int N, float scale, const int32_t* row_ptr, const int32_t* col_idx,
                     void* out, float* lse, float* blk_lse, unsigned* err, cudaStream_t s) {
  const int nB = ceil_div(N, BN);
  const int rows = BH * nB;
  const int smem = SmemLayout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  attn_fwd_sm100_kernel<D><<<rows, kThreads, smem, s>>>(
      mq, mk, mv, mo, N, nB, scale_log2, row_ptr, col_idx, static_cast<__nv_bfloat16*>(out), lse,
      blk_lse, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, int BH, int N,
                              int D, float scale, const int32_t* row_ptr,
                              const int32_t* col_idx, void* out, float* lse, float* blk_lse,
                              unsigned* err, cudaStream_t s, const char** why) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map(&mq, q, BH, N, D) || !make_tile_map(&mk, k, BH, N, D) ||
      !make_tile_map(&mv, v, BH, N, D) || !make_tile_map(&mo, out, BH, N, D)) {
    if (why) *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  if (D == 64) return launch_d<64>(mq, mk, mv, mo, BH, N, scale, row_ptr, col_idx, out, lse, blk_lse, err, s);
  return launch_d<128>(mq, mk, mv, mo, BH, N, scale, row_ptr, col_idx, out, lse, blk_lse, err, s);
}

}  // namespace dsa
