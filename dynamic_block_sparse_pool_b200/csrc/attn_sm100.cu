// Block-sparse attention forward on Blackwell tensor cores (sm_100a):
// TMA loads of the indexed K/V blocks, tcgen05 MMAs with fp32 accumulators
// in tensor memory, online softmax on CUDA cores.
//
// GSRS (arXiv 2610.21129), abstract: exact attention over the selected
// blocks inside a FlashAttention-style pass that also yields the exact
// per-block attention weights.  DSV (arXiv 2502.07590), abstract: the
// workload is skewed across heads and blocks, so every (head, query block)
// is its own CTA and the hardware scheduler balances them.
//
// One CTA (4 warps, 128 threads) per (batch*head, query block i); thread t
// owns query row t, which is TMEM lane t.  For each selected key block j:
//   S = Q K_j^T            tcgen05.mma, A = Q and B = K_j from shared memory
//                          (K-major, 128B swizzle), D = S in TMEM (128 cols)
//   softmax                tcgen05.ld of S, running max / sum in registers,
//                          P = exp2(S*scale*log2e - m) packed to bf16 and
//                          stored back into TMEM over S
//   O += P V_j             tcgen05.mma with A = P from TMEM and B = V_j from
//                          shared memory (MN-major), D = O in TMEM
// O is rescaled in TMEM when the running max grows.  K_{j+1} streams in
// during the softmax and PV of block j; V_{j+1} during S and softmax of
// block j+1.  Two CTAs share an SM (about 97 KB of shared memory and 256
// TMEM columns each), so one CTA's tensor-core work overlaps the other's
// softmax.
//
// The K/V tile of block j is one 3-D TMA box {64 cols, 128 rows, 1 head}
// per 64 columns of D over the tensor {D, N, B*H}: rows past N (the ragged
// last block, or another head's rows) are filled with zeros by the TMA unit
// and masked to -inf before the softmax.  No multicast is used.
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int BM = 128;        // query rows per CTA (one query block)
constexpr int BN = 128;        // keys per key block
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct SmemLayout {
  static constexpr int kTile = BM * D * 2;      // bytes of one [128 x D] bf16 tile
  static constexpr int kSub = BM * 64 * 2;      // one 128B-swizzled [128 x 64] sub-tile
  static constexpr int kQ = 0;
  static constexpr int kK = kTile;
  static constexpr int kV = 2 * kTile;
  static constexpr int kBar = 3 * kTile;        // 5 mbarriers, 8 B each
  static constexpr int kSlot = kBar + 64;       // TMEM base address
  static constexpr int kBytes = kSlot + 16;
  // The extra 1 KB lets the kernel align the tiles to 1024 B.  D = 64 pads
  // to 100 KB so that at most two CTAs (2 x 256 TMEM columns) share an SM.
  static constexpr int kAlloc = (kBytes + 1024) > 100 * 1024 ? (kBytes + 1024) : 100 * 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, int N, int nB, float scale_log2,
                      const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                      float* __restrict__ blk_lse, unsigned* err) {
  using L = SmemLayout<D>;
  constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, true);
  constexpr uint32_t kTileBytes = L::kTile;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  const uint32_t bar_q = base + L::kBar;
  const uint32_t bar_k = bar_q + 8, bar_v = bar_q + 16, bar_s = bar_q + 24, bar_o = bar_q + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kSlot);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = blockIdx.x;
  const int bh = r / nB, i = r - bh * nB;
  const int q0 = i * BM;
  const int qlen = min(BM, N - q0);

  int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  bool bad = s0 < 0 || s1 < s0;
  if (!bad)
    for (int e = s0 + tid; e < s1; e += kThreads) {
      const int j = col_idx[e];
      bad |= (j < 0 || j >= nB);
    }

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  const bool any_bad = __syncthreads_or(bad);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (any_bad) {
    if (tid == 0) flag_error(err, (s0 < 0 || s1 < s0) ? kErrRowPtr : kErrCsrIndex);
    s1 = s0;
  }
  const int n = s1 - s0;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tmem;         // S (fp32, 128 cols); P (bf16 pairs) over cols 0..63
  const uint32_t tO = tmem + 128;   // O (fp32, D cols)
  const int row = tid;

  float m = -INFINITY, l = 0.f;
  bool ok = true;                   // every wait of this thread succeeded
  bool stop = false;                // some thread of the CTA timed out
  bool k_pending = false, v_pending = false;  // TMA loads in flight (thread 0)
  uint32_t k_par = 0, v_par = 0;              // completion parity of those loads

  if (n > 0) {
    if (tid == 0) {
      const int j0 = col_idx[s0];
      mbar_expect_tx(bar_q, kTileBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_3d(sQ + c * L::kSub, &tmQ, c * 64, q0, bh, bar_q);
      mbar_expect_tx(bar_k, kTileBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sK + c * L::kSub, &tmK, c * 64, j0 * BN, bh, bar_k);
      mbar_expect_tx(bar_v, kTileBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sV + c * L::kSub, &tmV, c * 64, j0 * BN, bh, bar_v);
      k_pending = v_pending = true;
    }

    for (int it = 0; it < n; ++it) {
      const uint32_t ph = (uint32_t)it & 1u;
      const int j = col_idx[s0 + it];

      // ---- S = Q K_j^T ------------------------------------------------------
      if (tid == 0) {
        ok = (it > 0 || mbar_wait(bar_q, 0)) && mbar_wait(bar_k, ph);
        if (ok) {
          k_pending = false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kSub + (kk & 3) * 32;
            mma_ss(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK + off, 16, 1024),
                   kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_s);
        }
      }
      ok = mbar_wait(bar_s, ph) && ok;
      tc_fence_after();
      if (tid == 0 && ok && it + 1 < n) {  // K_j has been read: fetch K_{j+1}
        const int jn = col_idx[s0 + it + 1];
        mbar_expect_tx(bar_k, kTileBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sK + c * L::kSub, &tmK, c * 64, jn * BN, bh, bar_k);
        k_pending = true;
        k_par = (uint32_t)(it + 1) & 1u;
      }

      // ---- online softmax on row `row` ---------------------------------------
      uint32_t sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tS + lane_off + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
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
      const float m_new = fmaxf(m, mx * scale_log2);
      const float alpha = exp2f(m - m_new);
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float p0 = exp2f(fmaf(__uint_as_float(sv[2 * e]), scale_log2, -m_new));
        const float p1 = exp2f(fmaf(__uint_as_float(sv[2 * e + 1]), scale_log2, -m_new));
        rs += p0 + p1;
        const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);  // .x = p0 in the low half
        pk[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      l = l * alpha + rs;
      m = m_new;
      if (blk_lse != nullptr && row < qlen)
        blk_lse[(size_t)(s0 + it) * BN + row] = (m_new + log2f(rs)) * kLn2;

      // rescale O (the previous PV product is complete) when the max grew
      if (it > 0 && __any_sync(0xffffffffu, alpha < 1.0f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + lane_off + c * 32, o);
        }
      }
      {
        uint32_t p_lo[32], p_hi[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          p_lo[e] = pk[e];
          p_hi[e] = pk[32 + e];
        }
        tmem_st32(tS + lane_off + 0, p_lo);
        tmem_st32(tS + lane_off + 32, p_hi);
      }
      tmem_wait_st();
      tc_fence_before();
      stop = __syncthreads_or(!ok);
      if (stop) break;
      tc_fence_after();

      // ---- O += P V_j -----------------------------------------------------------
      if (tid == 0) {
        ok = mbar_wait(bar_v, ph);
        if (ok) {
          v_pending = false;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(tO, tS + kk * 8, smem_desc_sw128(sV + kk * 2048, L::kSub, 1024), kIdescO,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_o);
        }
      }
      ok = mbar_wait(bar_o, ph) && ok;
      tc_fence_after();
      if (tid == 0 && ok && it + 1 < n) {  // V_j has been read: fetch V_{j+1}
        const int jn = col_idx[s0 + it + 1];
        mbar_expect_tx(bar_v, kTileBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sV + c * L::kSub, &tmV, c * 64, jn * BN, bh, bar_v);
        v_pending = true;
        v_par = (uint32_t)(it + 1) & 1u;
      }
    }
    if (!stop) stop = __syncthreads_or(!ok);
  }

  if (stop) {
    if (tid == 0) {
      flag_error(err, kErrTimeout);
      // let loads still in flight land before the shared memory is released
      if (k_pending) mbar_wait(bar_k, k_par);
      if (v_pending) mbar_wait(bar_v, v_par);
    }
  } else if (n > 0) {
    // every thread takes part in the warp-collective TMEM loads; rows past
    // N only skip the stores
    __nv_bfloat16* orow = out + ((size_t)bh * N + q0 + row) * D;
    const float inv_l = 1.0f / l;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + lane_off + c * 32, o);
      tmem_wait_ld_regs(o);
      if (row < qlen) {
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
    if (lse != nullptr && row < qlen) lse[(size_t)bh * N + q0 + row] = (m + log2f(l)) * kLn2;
  } else if (row < qlen) {
    uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)bh * N + q0 + row) * D);
#pragma unroll
    for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
    if (lse != nullptr) lse[(size_t)bh * N + q0 + row] = -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
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
  const int smem = SmemLayout<D>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  attn_fwd_sm100_kernel<D><<<BH * nB, kThreads, smem, s>>>(
      mq, mk, mv, N, nB, scale_log2, row_ptr, col_idx, static_cast<__nv_bfloat16*>(out), lse,
      blk_lse, err);
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
