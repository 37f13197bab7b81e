// Backward pass of the block-sparse attention on Blackwell tensor cores
// (sm_100a), bf16 inputs, blocks of 128 rows, D = 64 or 128.
//
// DSV (arXiv 2502.07590), abstract: video DiTs are trained with the dynamic
// sparse attention, so its gradients run over the selected blocks.  For a
// fixed mask, with P the softmax over each query's selected keys (taken from
// the forward's lse) and delta = rowsum(dO * O):
//   dS = P * (dP - delta),  dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
//
// Two kernels, each one CTA per CSR row of its side:
//   dq    one query block i against its selected key blocks j (the mask);
//         S = Q K^T and dP = dO V^T into tensor memory, dS on CUDA cores,
//         then dQ += dS K.
//   dkdv  one key block j against the query blocks i that selected it (the
//         transposed mask, ascending i); S^T = K Q^T and dP^T = V dO^T, then
//         dV += P^T dO and dK += dS^T Q.
// The S-type products read the tiles K-major, the gradient products read the
// same tiles MN-major (as the forward reads V), so each tile is loaded once.
//
// P and dS go to the gradient products as two bf16 terms each, hi =
// bf16(x) and lo = bf16(x - hi), accumulated by two MMAs: dS sums to zero
// along a row, so dQ = sum dS K cancels heavily and a single bf16 dS would
// lose about 1 % of it; with the split the products are accurate to about
// 2^-17 of each term.  Each 32-column chunk of S (or S^T) and dP (dP^T) is
// read from tensor memory and its packed outputs are written back into the
// 32 columns it just vacated: in dq, dS hi at chunk columns 0-15 and dS lo at
// 16-31 of the S chunk; in dkdv, P hi / lo in the S^T chunk and dS hi / lo in
// the dP^T chunk.  An MMA K-step of 16 elements reads 8 packed columns, so
// step kk takes its A operand at column 32 (kk / 2) + 8 (kk % 2) (+16 for lo).
//
// Each block's S-type products run as two halves of 64 columns with their own
// barriers: the element-wise warps start on the first half while the second
// is computed, and the MMA warp issues the first half's gradient product and
// the next block's first half while they work on the second, so the tensor
// pipe and the element-wise pass overlap within the one S/dP buffer that
// tensor memory leaves room for.
//
// Warps 0-3: element-wise (thread = tensor-memory lane = row of the block);
// warp 4: MMA issuer (one thread) and tensor-memory allocation; warp 5: TMA
// loader (one thread).  Tensor memory: S 0-127, dP 128-255, then the fp32
// gradient accumulators (dQ; or dV and dK).  Shared memory: the two fixed
// tiles of the CTA and a 2-deep ring of the two streamed tiles.  Every
// mbarrier wait is bounded; a timeout sets the device error word and the
// CTA winds down.
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int BB = 128;            // rows of a block (queries and keys)
constexpr int kBwdThreads = 192;
constexpr int kMmaWarp = 4, kLoadWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 128, kColG = 256;
constexpr float kLog2e = 1.4426950408889634f;

// barriers (8 bytes each)
// (kBarS, kBarP: one per half of the block's columns)
// (kBarDrain: teardown after an abort, every MMA issued is done)
enum : int { kBarFixed = 0, kBarRing = 1, kBarFree = 3, kBarS = 5, kBarP = 7, kBarDrain = 9,
             kNumBars = 10 };

template <int D>
struct BwdSmem {
  static constexpr int kTile = BB * D * 2;   // one [128 x D] bf16 tile
  static constexpr int kSub = BB * 64 * 2;   // one 128B-swizzled [128 x 64] sub-tile
  static constexpr int kFixA = 0;            // two fixed tiles
  static constexpr int kFixB = kTile;
  static constexpr int kRingA = 2 * kTile;   // ring of the first streamed tile, 2 stages
  static constexpr int kRingB = 4 * kTile;   // ring of the second streamed tile
  static constexpr int kVec = 6 * kTile;     // float [2][2][128]: -lse2, -delta of the current query block (dkdv)
  static constexpr int kBar = kVec + 2 * 2 * BB * 4;
  static constexpr int kSlot = kBar + 8 * kNumBars;
  static constexpr int kBytes = kSlot + 16;
};

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

template <int D>
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int row, int bh,
                                         uint32_t bar) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_3d(dst + c * BwdSmem<D>::kSub, map, c * 64, row, bh, bar);
}

// K step kk (16 elements along D) of a K-major tile, as a descriptor offset
template <int D>
__device__ __forceinline__ uint64_t kstep(int kk) {
  return (uint64_t)(((kk >> 2) * BwdSmem<D>::kSub + (kk & 3) * 32) >> 4);
}

// bf16 pair (lo element first) as one 32-bit word
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi), for a pair of values
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16(a - __low2float(h), b - __high2float(h));
}

// S-type product for half h of the block's columns: D[tmem, 64 columns] =
// A B_h^T, A a [128 x D] tile and B_h rows 64h .. 64h + 63 of another, both
// K-major (64 rows of 128 bytes per 64-column sub-tile: 8192 bytes on).
template <int D>
__device__ __forceinline__ void mma_rows_half(uint32_t d, uint64_t a0, uint64_t b0, int h) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(BB, BB / 2, false);
  const uint64_t bh = b0 + (uint64_t)((h * (BB / 2) * 128) >> 4);
  mma_ss(d, a0 + kstep<D>(0), bh + kstep<D>(0), kIdesc, 0u);
#pragma unroll
  for (int kk = 1; kk < D / 16; ++kk) mma_ss_acc(d, a0 + kstep<D>(kk), bh + kstep<D>(kk), kIdesc);
}

// gradient product over half h of the K dimension: D[tmem] (+)= (hi + lo)
// [tmem, rows x K steps 4h .. 4h + 3, packed as above] B, B a [128 x D] tile
// read MN-major (its rows are the K dimension)
template <int D>
__device__ __forceinline__ void mma_grad_half(uint32_t d, uint32_t a, uint64_t b0, int h,
                                              bool accumulate) {
  constexpr uint32_t kIdesc = idesc_bf16_f32(BB, D, true);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int kk = 4 * h + q;
    const uint32_t ah = a + 32u * (uint32_t)(kk >> 1) + 8u * (uint32_t)(kk & 1);
    const uint64_t b = b0 + (uint64_t)((kk * 2048) >> 4);
    if (q == 0 && !accumulate)
      mma_ts(d, ah, b, kIdesc, 0u);
    else
      mma_ts_acc(d, ah, b, kIdesc);
    mma_ts_acc(d, ah + 16u, b, kIdesc);
  }
}

// After a role gave up, copies and MMAs may still be in flight: the MMA
// issuer commits once more and waits (bounded) until every MMA it issued is
// done, the loader waits for the fixed tiles and its last ring loads, then
// the whole CTA meets before shared and tensor memory are released.  Called
// by every thread of the CTA.
template <typename Bar>
__device__ __forceinline__ void drain_after_abort(int warp, int lane, int n, int issued, Bar bar) {
  if (warp == kMmaWarp && n > 0) {
    if (lane == 0) {
      mma_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0u);
    }
    __syncwarp();
  } else if (warp == kLoadWarp && lane == 0 && n > 0) {
    for (int b = issued - 2 > 0 ? issued - 2 : 0; b < issued; ++b)
      mbar_wait(bar(kBarRing + (b & 1)), (uint32_t)(b >> 1) & 1u);
    mbar_wait(bar(kBarFixed), 0u);
  }
  tc_fence_before();
  __syncthreads();
}

// Stores 32 fp32 accumulator columns of this thread's row, times `mul`, as bf16.
__device__ __forceinline__ void store_row_chunk(__nv_bfloat16* dst, const uint32_t (&g)[32], float mul) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint4 o;
    o.x = pack_bf16(__uint_as_float(g[8 * w + 0]) * mul, __uint_as_float(g[8 * w + 1]) * mul);
    o.y = pack_bf16(__uint_as_float(g[8 * w + 2]) * mul, __uint_as_float(g[8 * w + 3]) * mul);
    o.z = pack_bf16(__uint_as_float(g[8 * w + 4]) * mul, __uint_as_float(g[8 * w + 5]) * mul);
    o.w = pack_bf16(__uint_as_float(g[8 * w + 6]) * mul, __uint_as_float(g[8 * w + 7]) * mul);
    d4[w] = o;
  }
}

// One CTA per query block: dQ over the block's selected key blocks.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    int N, int nB, float scale, float scale_log2, const float* __restrict__ lse,
                    const float* __restrict__ delta, const int32_t* __restrict__ row_ptr,
                    const int32_t* __restrict__ col_idx, __nv_bfloat16* __restrict__ dq,
                    unsigned* err) {
  using L = BwdSmem<D>;
  constexpr uint32_t kTileBytes = L::kTile;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) flag_error(err, kErrAlign);
    return;
  }
  const uint32_t sQ = base + L::kFixA, sO = base + L::kFixB;   // Q, dO of the query block
  const uint32_t sK = base + L::kRingA, sV = base + L::kRingB;  // K, V of the key blocks
  const uint32_t bars = base + L::kBar;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;
  const int bh = r / nB, q0 = (r - bh * nB) * BB;
  const int qlen = min(BB, N - q0);
  const int kv_last = N - (nB - 1) * BB;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == kBarP || i == kBarP + 1) ? 4u : 1u);
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
  int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  bool bad = s0 < 0 || s1 < s0;
  if (!bad)
    for (int e = s0 + tid; e < s1; e += kBwdThreads) {
      const int j = col_idx[e];
      bad |= (j < 0 || j >= nB);
    }
  tc_fence_before();
  if (__syncthreads_or(bad)) s1 = s0;  // the mask kernel flags the error
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = s1 - s0;
  int issued = 0;  // loader: blocks whose ring loads were issued

  if (warp == kLoadWarp) {
    if (lane == 0 && n > 0) {
      bool ok = true;
      mbar_expect_tx(bar(kBarFixed), 2 * kTileBytes);
      tma_tile<D>(sQ, &tmQ, q0, bh, bar(kBarFixed));
      tma_tile<D>(sO, &tmO, q0, bh, bar(kBarFixed));
      for (int it = 0; it < n; ++it) {
        const int s = it & 1;
        const int j = col_idx[s0 + it];
        // slot s is free once dQ of block it - 2 is done
        ok = mbar_wait(bar(kBarFree + s), ((uint32_t)(it >> 1) & 1u) ^ 1u) && !*abort_flag;
        if (!ok) break;
        mbar_expect_tx(bar(kBarRing + s), 2 * kTileBytes);
        tma_tile<D>(sK + s * kTileBytes, &tmK, j * BB, bh, bar(kBarRing + s));
        tma_tile<D>(sV + s * kTileBytes, &tmV, j * BB, bh, bar(kBarRing + s));
        issued = it + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else if (warp == kMmaWarp) {
    if (n > 0) {
      const bool leader = lane == 0;
      const uint64_t dQk = smem_desc_sw128(sQ, 16, 1024), dOk = smem_desc_sw128(sO, 16, 1024);
      const uint64_t dKk = smem_desc_sw128(sK, 16, 1024), dVk = smem_desc_sw128(sV, 16, 1024);
      const uint64_t dKm = smem_desc_sw128(sK, L::kSub, 1024);
      bool ok = warp_all(mbar_wait(bar(kBarFixed), 0u));
      // S and dP of half h (keys 64h .. 64h + 63) of block it
      auto issue_half = [&](int it, int h) {
        const int s = it & 1;
        if (h == 0 && !(ok = ok && warp_all(mbar_wait(bar(kBarRing + s), (uint32_t)(it >> 1) & 1u))))
          return;
        tc_fence_after();
        if (leader) {
          const uint64_t off = (uint64_t)((s * kTileBytes) >> 4);
          mma_rows_half<D>(tmem + kColS + 64 * h, dQk, dKk + off, h);
          mma_rows_half<D>(tmem + kColP + 64 * h, dOk, dVk + off, h);
          mma_commit(bar(kBarS + h));
        }
        __syncwarp();
      };
      issue_half(0, 0);
      if (ok) issue_half(0, 1);
      for (int it = 0; it < n && ok; ++it) {
        const int s = it & 1;
        for (int h = 0; h < 2 && ok; ++h) {
          if (!(ok = warp_all(mbar_wait(bar(kBarP + h), (uint32_t)it & 1u)))) break;
          tc_fence_after();
          if (leader) {
            mma_grad_half<D>(tmem + kColG, tmem + kColS, dKm + (uint64_t)((s * kTileBytes) >> 4), h,
                             it > 0 || h > 0);
            if (h == 1) mma_commit(bar(kBarFree + s));
          }
          __syncwarp();
          // half h of block it + 1 overwrites half h's dS columns only after
          // dQ has read them (the MMAs of one thread run in order), while the
          // element-wise warps work on the other half
          if (it + 1 < n) issue_half(it + 1, h);
        }
      }
      if (!ok && leader) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------- element-wise
    const int row = 32 * warp + lane;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const bool valid = row < qlen;
    const size_t tok = (size_t)bh * N + q0 + row;
    // -lse (base 2) and -delta of the row, as packed pairs; rows past N get
    // -inf, so their P is 0
    const float nl = valid ? -lse[tok] * kLog2e : -INFINITY;
    const float nd = valid ? -delta[tok] : 0.f;
    const uint64_t sc2 = pack_f32x2(scale_log2, scale_log2);
    const uint64_t nl2 = pack_f32x2(nl, nl), nd2 = pack_f32x2(nd, nd);
    bool failed = false;
    for (int it = 0; it < n && !failed; ++it) {
      // the ragged last key block: keys past N get S = -inf, so P = 0
      const bool rag = kv_last < BB && col_idx[s0 + it] == nB - 1;
      for (int h = 0; h < 2; ++h) {
        if (!warp_all(mbar_wait(bar(kBarS + h), (uint32_t)it & 1u))) {
          failed = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * h + cc;
          uint32_t sv[32], pv[32];
          tmem_ld32(tmem + lane_off + kColS + 32 * c, sv);
          tmem_ld32(tmem + lane_off + kColP + 32 * c, pv);
          tmem_wait_ld_regs(sv);
          tmem_wait_ld_regs(pv);
          if (rag) {
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (32 * c + u >= kv_last) sv[u] = __float_as_uint(-INFINITY);
          }
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            float t0, t1, g0, g1;
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * m]), __uint_as_float(sv[2 * m + 1])),
                                   sc2, nl2), t0, t1);
            const uint64_t p2 = pack_f32x2(exp2_approx(t0), exp2_approx(t1));
            const uint64_t d2 = add_f32x2(pack_f32x2(__uint_as_float(pv[2 * m]), __uint_as_float(pv[2 * m + 1])), nd2);
            unpack_f32x2(mul_f32x2(p2, d2), g0, g1);
            split_pair(g0, g1, hi[m], lo[m]);
          }
          tmem_st16(tmem + lane_off + kColS + 32 * c, hi);
          tmem_st16(tmem + lane_off + kColS + 32 * c + 16, lo);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarP + h));
      }
    }
    __nv_bfloat16* drow = dq + tok * D;
    if (failed) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
    } else if (n > 0) {
      if (!warp_all(mbar_wait(bar(kBarFree + ((n - 1) & 1)), (uint32_t)((n - 1) >> 1) & 1u))) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      } else {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t g[32];
          tmem_ld32(tmem + lane_off + kColG + 32 * c, g);
          tmem_wait_ld_regs(g);
          if (valid) store_row_chunk(drow + 32 * c, g, scale);
        }
      }
    } else if (valid) {
      uint4* d4 = reinterpret_cast<uint4*>(drow);
#pragma unroll
      for (int w = 0; w < D / 8; ++w) d4[w] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) drain_after_abort(warp, lane, n, issued, bar);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One CTA per key block: dK and dV over the query blocks that selected it.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      int N, int nB, float scale, float scale_log2, const float* __restrict__ lse,
                      const float* __restrict__ delta, const int32_t* __restrict__ t_row_ptr,
                      const int32_t* __restrict__ t_col, __nv_bfloat16* __restrict__ dk,
                      __nv_bfloat16* __restrict__ dv, unsigned* err) {
  using L = BwdSmem<D>;
  constexpr uint32_t kTileBytes = L::kTile;
  constexpr uint32_t kColV = kColG, kColK = kColG + D;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) flag_error(err, kErrAlign);
    return;
  }
  const uint32_t sK = base + L::kFixA, sV = base + L::kFixB;    // K, V of the key block
  const uint32_t sQ = base + L::kRingA, sO = base + L::kRingB;  // Q, dO of the query blocks
  float* vec = reinterpret_cast<float*>(smem + L::kVec);        // [buf][-lse2 | -delta][128]
  const uint32_t bars = base + L::kBar;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;
  const int bh = r / nB, k0 = (r - bh * nB) * BB;
  const int klen = min(BB, N - k0);

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == kBarP || i == kBarP + 1) ? 4u : 1u);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int t0 = t_row_ptr[r];
  const int n = t_row_ptr[r + 1] - t0;  // built by the mask transpose: ascending, in range
  int issued = 0;  // loader: blocks whose ring loads were issued

  if (warp == kLoadWarp) {
    if (lane == 0 && n > 0) {
      bool ok = true;
      mbar_expect_tx(bar(kBarFixed), 2 * kTileBytes);
      tma_tile<D>(sK, &tmK, k0, bh, bar(kBarFixed));
      tma_tile<D>(sV, &tmV, k0, bh, bar(kBarFixed));
      for (int it = 0; it < n; ++it) {
        const int s = it & 1;
        const int i = t_col[t0 + it];
        ok = mbar_wait(bar(kBarFree + s), ((uint32_t)(it >> 1) & 1u) ^ 1u) && !*abort_flag;
        if (!ok) break;
        mbar_expect_tx(bar(kBarRing + s), 2 * kTileBytes);
        tma_tile<D>(sQ + s * kTileBytes, &tmQ, i * BB, bh, bar(kBarRing + s));
        tma_tile<D>(sO + s * kTileBytes, &tmO, i * BB, bh, bar(kBarRing + s));
        issued = it + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else if (warp == kMmaWarp) {
    if (n > 0) {
      const bool leader = lane == 0;
      const uint64_t dKk = smem_desc_sw128(sK, 16, 1024), dVk = smem_desc_sw128(sV, 16, 1024);
      const uint64_t dQk = smem_desc_sw128(sQ, 16, 1024), dOk = smem_desc_sw128(sO, 16, 1024);
      const uint64_t dQm = smem_desc_sw128(sQ, L::kSub, 1024), dOm = smem_desc_sw128(sO, L::kSub, 1024);
      bool ok = warp_all(mbar_wait(bar(kBarFixed), 0u));
      // S^T and dP^T of half h (queries 64h .. 64h + 63) of block it
      auto issue_half = [&](int it, int h) {
        const int s = it & 1;
        if (h == 0 && !(ok = ok && warp_all(mbar_wait(bar(kBarRing + s), (uint32_t)(it >> 1) & 1u))))
          return;
        tc_fence_after();
        if (leader) {
          const uint64_t off = (uint64_t)((s * kTileBytes) >> 4);
          mma_rows_half<D>(tmem + kColS + 64 * h, dKk, dQk + off, h);  // S^T = K Q^T
          mma_rows_half<D>(tmem + kColP + 64 * h, dVk, dOk + off, h);  // dP^T = V dO^T
          mma_commit(bar(kBarS + h));
        }
        __syncwarp();
      };
      issue_half(0, 0);
      if (ok) issue_half(0, 1);
      for (int it = 0; it < n && ok; ++it) {
        const int s = it & 1;
        const uint64_t off = (uint64_t)((s * kTileBytes) >> 4);
        for (int h = 0; h < 2 && ok; ++h) {
          if (!(ok = warp_all(mbar_wait(bar(kBarP + h), (uint32_t)it & 1u)))) break;
          tc_fence_after();
          if (leader) {
            mma_grad_half<D>(tmem + kColV, tmem + kColS, dOm + off, h, it > 0 || h > 0);  // dV += P^T dO
            mma_grad_half<D>(tmem + kColK, tmem + kColP, dQm + off, h, it > 0 || h > 0);  // dK += dS^T Q
            if (h == 1) mma_commit(bar(kBarFree + s));
          }
          __syncwarp();
          if (it + 1 < n) issue_half(it + 1, h);
        }
      }
      if (!ok && leader) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------- element-wise
    // thread = key row of the block; columns = the query block's queries
    const int row = 32 * warp + lane;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const uint64_t sc2 = pack_f32x2(scale_log2, scale_log2);
    bool failed = false;
    for (int it = 0; it < n; ++it) {
      const int i = t_col[t0 + it];
      const int q0 = i * BB, qlen = min(BB, N - q0);
      float* nl = vec + (it & 1) * 2 * BB;
      float* nd = nl + BB;
      // this query block's -lse (base 2) and -delta; queries past N get
      // -inf, so their P is 0
      const size_t tok = (size_t)bh * N + q0 + row;
      nl[row] = row < qlen ? -lse[tok] * kLog2e : -INFINITY;
      nd[row] = row < qlen ? -delta[tok] : 0.f;
      // A barrier of the four warps at each half serves two ends: it makes a
      // timed-out wait a decision of all four warps, so none is left alone at
      // a later barrier, and the first one publishes the vectors just written
      // (the other buffer was last read before it).
      for (int h = 0; h < 2; ++h) {
        const bool late = !warp_all(mbar_wait(bar(kBarS + h), (uint32_t)it & 1u));
        if (named_bar_or(1, 128, late)) {
          failed = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * h + cc;
          uint32_t sv[32], pv[32];
          tmem_ld32(tmem + lane_off + kColS + 32 * c, sv);
          tmem_ld32(tmem + lane_off + kColP + 32 * c, pv);
          tmem_wait_ld_regs(sv);
          tmem_wait_ld_regs(pv);
          uint32_t ph[16], pl[16], dh[16], dl[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const int qq = 32 * c + 2 * m;  // even: the pairs are 8-byte aligned
            float t0, t1, g0, g1;
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * m]), __uint_as_float(sv[2 * m + 1])),
                                   sc2, *reinterpret_cast<const uint64_t*>(nl + qq)), t0, t1);
            const float p0 = exp2_approx(t0), p1 = exp2_approx(t1);
            split_pair(p0, p1, ph[m], pl[m]);
            const uint64_t d2 = add_f32x2(pack_f32x2(__uint_as_float(pv[2 * m]), __uint_as_float(pv[2 * m + 1])),
                                          *reinterpret_cast<const uint64_t*>(nd + qq));
            unpack_f32x2(mul_f32x2(pack_f32x2(p0, p1), d2), g0, g1);
            split_pair(g0, g1, dh[m], dl[m]);
          }
          tmem_st16(tmem + lane_off + kColS + 32 * c, ph);
          tmem_st16(tmem + lane_off + kColS + 32 * c + 16, pl);
          tmem_st16(tmem + lane_off + kColP + 32 * c, dh);
          tmem_st16(tmem + lane_off + kColP + 32 * c + 16, dl);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarP + h));
      }
      if (failed) break;
    }
    const bool valid = row < klen;
    const size_t ktok = (size_t)bh * N + k0 + row;
    if (failed) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
    } else if (n > 0) {
      if (!warp_all(mbar_wait(bar(kBarFree + ((n - 1) & 1)), (uint32_t)((n - 1) >> 1) & 1u))) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      } else {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t g[32];
          tmem_ld32(tmem + lane_off + kColV + 32 * c, g);
          tmem_wait_ld_regs(g);
          if (valid) store_row_chunk(dv + ktok * D + 32 * c, g, 1.0f);
          tmem_ld32(tmem + lane_off + kColK + 32 * c, g);
          tmem_wait_ld_regs(g);
          if (valid) store_row_chunk(dk + ktok * D + 32 * c, g, scale);
        }
      }
    } else if (valid) {
      uint4* a = reinterpret_cast<uint4*>(dk + ktok * D);
      uint4* b = reinterpret_cast<uint4*>(dv + ktok * D);
#pragma unroll
      for (int w = 0; w < D / 8; ++w) a[w] = b[w] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) drain_after_abort(warp, lane, n, issued, bar);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda)
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                             CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                             CUtensorMapFloatOOBfill);

// [BH, N, D] bf16 as the 3-D tensor {D, N, BH}, boxes of 64 x 128 x 1,
// 128-byte swizzle; rows past N read as zeros.
bool bwd_tile_map(CUtensorMap* map, const void* ptr, int BH, int N, int D) {
  static EncodeFn fn = []() -> EncodeFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeFn>(p);
  }();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_bwd_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, int BH, int N, float scale, const float* lse,
                         const float* delta, const int32_t* row_ptr, const int32_t* col_idx,
                         const int32_t* t_row_ptr, const int32_t* t_col, void* dq, void* dk,
                         void* dv, unsigned* err, cudaStream_t s) {
  const int nB = ceil_div(N, BB);
  const int rows = BH * nB;
  const int smem = BwdSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * kLog2e;
  bwd_dq_sm100_kernel<D><<<rows, kBwdThreads, smem, s>>>(mq, mk, mv, mo, N, nB, scale, scale_log2, lse,
                                                         delta, row_ptr, col_idx,
                                                         static_cast<__nv_bfloat16*>(dq), err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkdv_sm100_kernel<D><<<rows, kBwdThreads, smem, s>>>(mq, mk, mv, mo, N, nB, scale, scale_log2,
                                                           lse, delta, t_row_ptr, t_col,
                                                           static_cast<__nv_bfloat16*>(dk),
                                                           static_cast<__nv_bfloat16*>(dv), err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_sm100(const void* q, const void* k, const void* v, const void* dout,
                                  const float* lse, const float* delta, int BH, int N, int D,
                                  float scale, const int32_t* row_ptr, const int32_t* col_idx,
                                  const int32_t* t_row_ptr, const int32_t* t_col, void* dq, void* dk,
                                  void* dv, unsigned* err, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mo;
  if (!bwd_tile_map(&mq, q, BH, N, D) || !bwd_tile_map(&mk, k, BH, N, D) ||
      !bwd_tile_map(&mv, v, BH, N, D) || !bwd_tile_map(&mo, dout, BH, N, D))
    return cudaErrorInvalidValue;
  if (D == 64)
    return launch_bwd_d<64>(mq, mk, mv, mo, BH, N, scale, lse, delta, row_ptr, col_idx, t_row_ptr, t_col,
                            dq, dk, dv, err, s);
  return launch_bwd_d<128>(mq, mk, mv, mo, BH, N, scale, lse, delta, row_ptr, col_idx, t_row_ptr, t_col,
                           dq, dk, dv, err, s);
}

}  // namespace dsa
