// Block-sparse attention forward on Blackwell tensor cores (sm_100a):
// TMA loads of the indexed K/V blocks, tcgen05 MMAs with fp32 accumulators
// in tensor memory, online softmax on CUDA cores, warp-specialised.
//
// GSRS (arXiv 2610.21129), abstract: exact attention over the selected
// blocks inside a FlashAttention-style pass that also yields the exact
// per-block attention weights.  DSV (arXiv 2502.07590), abstract: the work
// per query block is skewed, so rows are small independent work items.
//
// One CTA per pair of CSR rows (two query blocks, "tiles" 0 and 1, each with
// its own list of key blocks).  320 threads in four roles:
//   warps 0-3  softmax of tile 0     (thread t <-> query row t <-> TMEM lane t)
//   warps 4-7  softmax of tile 1
//   warp  8    MMA issuer (one thread) and TMEM allocation (whole warp)
//   warp  9    TMA loader (one thread)
// Ten warps put three on some SM sub-partitions, whose 16K registers then
// cap every thread at 168; the softmax keeps its 128 S values in registers
// within that budget.
// Tensor memory (512 columns): S_t at 256t .. 256t+127 (P_t, packed bf16
// pairs, overwrites its first 64 columns), O_t at 256t+128 .. +D-1.
//
// MMA issue order (each MMA in the same order as its operands are loaded):
//   S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) PV1(1) S1(2) | ...
// so the tensor cores work on one tile while the other tile's softmax runs.
// tcgen05 MMAs issued by one thread execute in order, so S_t(j+1) reuses the
// columns of P_t(j) only after PV_t(j) has read them, and the completion of
// S_t(j+1) implies that of PV_t(j): when a softmax warp sees S_t(j+1) it may
// rescale O_t in place.  K and V stream through separate two-stage rings.
//
// Online softmax with a lazy reference: the running max m_ref moves only when
// a block's max exceeds it by more than 8 (log2 units); otherwise P is
// formed against the stale m_ref (values up to 2^8, exact in fp32 and
// representable in bf16), which skips most O rescales.  The final O / l and
// lse use the same reference, so the result is exact.
//
// Each selected block's log-sum (for the exact block mass) is
// m_ref + log2(sum of that block's P row), written per query row.
//
// K/V tile of block j: one 3-D TMA box {64 cols, 128 rows, 1 head} per 64
// columns of D over the tensor {D, N, B*H}: rows past N are zero-filled and
// masked to -inf.  No multicast.  Every mbarrier wait is bounded; a timeout
// sets the device error word and the CTA winds down.
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int BM = 128;        // query rows per tile (one query block)
constexpr int BN = 128;        // keys per key block
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8, kLoadWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// mbarrier slots
enum : int {
  kBarQ = 0,
  kBarKFull = 1,   // +stage (2)
  kBarKEmpty = 3,  // +stage
  kBarVFull = 5,   // +stage
  kBarVEmpty = 7,  // +stage
  kBarSFull = 9,   // +tile
  kBarPFull = 11,  // +tile (128 arrivals)
  kBarOFull = 13,  // +tile
  kNumBars = 15
};

template <int D>
struct SmemLayout {
  static constexpr int kTile = BM * D * 2;  // bytes of one [128 x D] bf16 tile
  static constexpr int kSub = BM * 64 * 2;  // one 128B-swizzled [128 x 64] sub-tile
  static constexpr int kQ = 0;              // Q of tiles 0, 1
  static constexpr int kK = 2 * kTile;      // K ring, 2 stages
  static constexpr int kV = 4 * kTile;      // V ring, 2 stages
  static constexpr int kBar = 6 * kTile;
  static constexpr int kSlot = kBar + 8 * kNumBars;  // TMEM base, abort flag
  static constexpr int kBytes = kSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;       // room to align tiles to 1024 B
};

struct Tile {
  int bh, q0, qlen, s0, n;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

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
                      const __grid_constant__ CUtensorMap tmV, int N, int nB, int rows,
                      float scale_log2, const int32_t* __restrict__ row_ptr,
                      const int32_t* __restrict__ col_idx, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse, float* __restrict__ blk_lse, unsigned* err) {
  using L = SmemLayout<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, true);
  constexpr uint32_t kTileBytes = L::kTile;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  const uint32_t bars = base + L::kBar;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kSlot + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- the two rows of this CTA --------------------------------------------
  Tile tl[2];
  bool bad[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r = 2 * blockIdx.x + t;
    tl[t].bh = 0; tl[t].q0 = 0; tl[t].qlen = 0; tl[t].s0 = 0; tl[t].n = 0;
    bad[t] = false;
    if (r < rows) {
      const int bh = r / nB, i = r - bh * nB;
      tl[t].bh = bh;
      tl[t].q0 = i * BM;
      tl[t].qlen = min(BM, N - i * BM);
      const int s0 = row_ptr[r], s1 = row_ptr[r + 1];
      tl[t].s0 = s0;
      tl[t].n = s1 - s0;
      bad[t] = s0 < 0 || s1 < s0;
      if (!bad[t])
        for (int e = s0 + tid; e < s1; e += kThreads) {
          const int j = col_idx[e];
          bad[t] |= (j < 0 || j >= nB);
        }
    }
  }

  if (warp == kMmaWarp) {
    if (lane == 0) {
      mbar_init(bar(kBarQ), 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(kBarKFull + s), 1);
        mbar_init(bar(kBarKEmpty + s), 1);
        mbar_init(bar(kBarVFull + s), 1);
        mbar_init(bar(kBarVEmpty + s), 1);
        mbar_init(bar(kBarSFull + s), 1);
        mbar_init(bar(kBarPFull + s), 128);
        mbar_init(bar(kBarOFull + s), 1);
      }
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
  }
  tc_fence_before();
  const bool bad0 = __syncthreads_or(bad[0]);
  const bool bad1 = __syncthreads_or(bad[1]);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (bad0) {
    if (tid == 0) flag_error(err, kErrCsrIndex | kErrRowPtr);
    tl[0].n = 0;
  }
  if (bad1) {
    if (tid == 0) flag_error(err, kErrCsrIndex | kErrRowPtr);
    tl[1].n = 0;
  }
  const int n0 = tl[0].n, n1 = tl[1].n;
  const int nmax = n0 > n1 ? n0 : n1;

  if (warp == kLoadWarp) {
    // ---------------------------------------------------------------- loader
    if (lane == 0 && nmax > 0) {
      bool ok = true;
      uint32_t kc = 0, vc = 0;           // loads issued into each ring
      uint32_t k_used = 0, v_used = 0;   // bit s: stage s has received a load
      uint32_t k_last_ph = 0, v_last_ph = 0;  // bit s: parity of its last load
      mbar_expect_tx(bar(kBarQ), (n0 > 0 ? kTileBytes : 0) + (n1 > 0 ? kTileBytes : 0));
      if (n0 > 0) tma_tile<D>(sQ, &tmQ, tl[0].q0, tl[0].bh, bar(kBarQ));
      if (n1 > 0) tma_tile<D>(sQ + kTileBytes, &tmQ, tl[1].q0, tl[1].bh, bar(kBarQ));
      auto load_k = [&](int t, int it) {
        const uint32_t s = kc & 1u, ph = ((kc >> 1) & 1u) ^ 1u;
        if (!(ok = ok && mbar_wait(bar(kBarKEmpty + s), ph))) return;
        const int j = col_idx[tl[t].s0 + it];
        mbar_expect_tx(bar(kBarKFull + s), kTileBytes);
        tma_tile<D>(sK + s * kTileBytes, &tmK, j * BN, tl[t].bh, bar(kBarKFull + s));
        k_used |= 1u << s;
        k_last_ph = (k_last_ph & ~(1u << s)) | (((kc >> 1) & 1u) << s);
        ++kc;
      };
      auto load_v = [&](int t, int it) {
        const uint32_t s = vc & 1u, ph = ((vc >> 1) & 1u) ^ 1u;
        if (!(ok = ok && mbar_wait(bar(kBarVEmpty + s), ph))) return;
        const int j = col_idx[tl[t].s0 + it];
        mbar_expect_tx(bar(kBarVFull + s), kTileBytes);
        tma_tile<D>(sV + s * kTileBytes, &tmV, j * BN, tl[t].bh, bar(kBarVFull + s));
        v_used |= 1u << s;
        v_last_ph = (v_last_ph & ~(1u << s)) | (((vc >> 1) & 1u) << s);
        ++vc;
      };
      if (n0 > 0) load_k(0, 0);
      if (n1 > 0 && ok) load_k(1, 0);
      for (int it = 0; it < nmax && ok && !*abort_flag; ++it) {
        if (it < n0) {
          load_v(0, it);
          if (it + 1 < n0 && ok) load_k(0, it + 1);
        }
        if (it < n1 && ok) {
          load_v(1, it);
          if (it + 1 < n1 && ok) load_k(1, it + 1);
        }
      }
      if (!ok || *abort_flag) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
        // let the loads still in flight land before shared memory is released
        for (int s = 0; s < 2; ++s) {
          if ((k_used >> s) & 1u) mbar_wait(bar(kBarKFull + s), (k_last_ph >> s) & 1u);
          if ((v_used >> s) & 1u) mbar_wait(bar(kBarVFull + s), (v_last_ph >> s) & 1u);
        }
        mbar_wait(bar(kBarQ), 0);
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && nmax > 0) {
      bool ok = mbar_wait(bar(kBarQ), 0);
      uint32_t kc = 0, vc = 0;
      auto issue_s = [&](int t) {
        const uint32_t s = kc & 1u, ph = (kc >> 1) & 1u;
        if (!(ok = ok && mbar_wait(bar(kBarKFull + s), ph))) return;
        tc_fence_after();
        const uint32_t q = sQ + t * kTileBytes, k = sK + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kSub + (kk & 3) * 32;
          mma_ss(tmem + 256u * t, smem_desc_sw128(q + off, 16, 1024),
                 smem_desc_sw128(k + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarKEmpty + s));
        mma_commit(bar(kBarSFull + t));
        ++kc;
      };
      auto issue_pv = [&](int t, int it, int n) {
        if (!(ok = ok && mbar_wait(bar(kBarPFull + t), (uint32_t)it & 1u))) return;
        const uint32_t s = vc & 1u, ph = (vc >> 1) & 1u;
        if (!(ok = ok && mbar_wait(bar(kBarVFull + s), ph))) return;
        tc_fence_after();
        const uint32_t v = sV + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + 256u * t + 128u, tmem + 256u * t + kk * 8,
                 smem_desc_sw128(v + kk * 2048, L::kSub, 1024), kIdescO,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(kBarVEmpty + s));
        if (it == n - 1) mma_commit(bar(kBarOFull + t));
        ++vc;
      };
      if (n0 > 0 && ok) issue_s(0);
      if (n1 > 0 && ok) issue_s(1);
      for (int it = 0; it < nmax && ok && !*abort_flag; ++it) {
        if (it < n0) {
          issue_pv(0, it, n0);
          if (it + 1 < n0 && ok) issue_s(0);
        }
        if (it < n1 && ok) {
          issue_pv(1, it, n1);
          if (it + 1 < n1 && ok) issue_s(1);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;
    const Tile T = t ? tl[1] : tl[0];
    const int row = tid - 128 * t;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 256u * t + lane_off;
    const uint32_t tO = tS + 128u;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < T.n; ++it) {
      ok = warp_all(mbar_wait(bar(kBarSFull + t), (uint32_t)it & 1u)) && !warp_all(*abort_flag != 0);
      if (!ok) break;
      tc_fence_after();
      const int j = col_idx[T.s0 + it];
      uint32_t sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_wait_ld_regs(*reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
      const int kv_len = min(BN, N - j * BN);
      if (kv_len < BN) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= kv_len) sv[e] = __float_as_uint(-INFINITY);
      }
      float mx = __uint_as_float(sv[0]);
#pragma unroll
      for (int e = 1; e < 128; ++e) mx = fmaxf(mx, __uint_as_float(sv[e]));
      const float mb = mx * scale_log2;
      const bool need = mb > m_ref + kRescaleThreshold;
      const bool warp_need = __any_sync(0xffffffffu, need);
      float alpha = 1.0f;
      if (need) {
        alpha = exp2f(m_ref - mb);  // 0 on the first block
        l *= alpha;
        m_ref = mb;
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = exp2f(fmaf(__uint_as_float(sv[32 * c + 2 * e]), scale_log2, -m_ref));
          const float p1 = exp2f(fmaf(__uint_as_float(sv[32 * c + 2 * e + 1]), scale_log2, -m_ref));
          rs += p0 + p1;
          const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);  // .x = p0, low half
          pk[e] = *reinterpret_cast<const uint32_t*>(&h);
        }
        tmem_st16(tS + c * 16, pk);
      }
      // O_t holds the sum up to block it-1 (its PV completed before S_t(it));
      // move it to the new reference before PV_t(it) accumulates onto it
      if (warp_need && it > 0) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + t));
      if (blk_lse != nullptr && row < T.qlen)
        blk_lse[(size_t)(T.s0 + it) * BN + row] = (m_ref + log2f(rs)) * kLn2;
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
    } else if (T.n > 0) {
      ok = warp_all(mbar_wait(bar(kBarOFull + t), 0u));
      if (!ok) {
        *abort_flag = 1;
        flag_error(err, kErrTimeout);
      } else {
        tc_fence_after();
        __nv_bfloat16* orow = out + ((size_t)T.bh * N + T.q0 + row) * D;
        const float inv_l = 1.0f / l;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld_regs(o);
          if (row < T.qlen) {
            uint4 pkt[4];
            uint32_t* w = reinterpret_cast<uint32_t*>(pkt);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv_l,
                                                             __uint_as_float(o[2 * e + 1]) * inv_l);
              w[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) dst[u] = pkt[u];
          }
        }
        if (lse != nullptr && row < T.qlen) lse[(size_t)T.bh * N + T.q0 + row] = (m_ref + log2f(l)) * kLn2;
      }
    } else if (row < T.qlen) {
      uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)T.bh * N + T.q0 + row) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
      if (lse != nullptr) lse[(size_t)T.bh * N + T.q0 + row] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
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
cudaError_t launch_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, int BH,
                     int N, float scale, const int32_t* row_ptr, const int32_t* col_idx,
                     void* out, float* lse, float* blk_lse, unsigned* err, cudaStream_t s) {
  const int nB = ceil_div(N, BN);
  const int rows = BH * nB;
  const int smem = SmemLayout<D>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  attn_fwd_sm100_kernel<D><<<ceil_div(rows, 2), kThreads, smem, s>>>(
      mq, mk, mv, N, nB, rows, scale_log2, row_ptr, col_idx, static_cast<__nv_bfloat16*>(out),
      lse, blk_lse, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, int BH, int N,
                              int D, float scale, const int32_t* row_ptr,
                              const int32_t* col_idx, void* out, float* lse, float* blk_lse,
                              unsigned* err, cudaStream_t s, const char** why) {
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, q, BH, N, D) || !make_tile_map(&mk, k, BH, N, D) ||
      !make_tile_map(&mv, v, BH, N, D)) {
    if (why) *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  if (D == 64) return launch_d<64>(mq, mk, mv, BH, N, scale, row_ptr, col_idx, out, lse, blk_lse, err, s);
  return launch_d<128>(mq, mk, mv, BH, N, scale, row_ptr, col_idx, out, lse, blk_lse, err, s);
}

}  // namespace dsa
