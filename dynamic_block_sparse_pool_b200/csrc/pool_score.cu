// Pooled block scores: block means of Q and K, then the row softmax of
// scale * qbar_i . kbar_j over all key blocks or over a candidate set.
//
// GSRS (arXiv 2610.21129), abstract and Figure 4: Top-p selection runs on a
// block-level estimate of the attention map; reduced search evaluates only
// the blocks inside an earlier candidate mask.  The estimate used here is
// the softmax of mean-pooled query/key block scores.
//
// Kernel 1 (pool_means): one CTA per (block, head, Q-or-K); 16-byte loads,
//   fp32 accumulation, mean over the block's actual rows.  HBM-bound: reads
//   Q and K once.
// Kernel 2 (block_scores): one CTA per (32 query-block rows, head): a
//   register-tiled fp32 product of the 32 pooled queries with tiles of 64
//   pooled keys; the 32 x nB raw scores stay in shared memory for the row
//   softmax, which writes P once, coalesced.
#include "common.cuh"

namespace dsa {
namespace {

template <typename T, int D>
__global__ void __launch_bounds__(256)
pool_means_kernel(const T* __restrict__ q, const T* __restrict__ k, int N, int nB,
                  int block, float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int C = D / VEC;           // 16-byte chunks per row
  constexpr int R = 256 / C;           // rows in flight per pass
  __shared__ float part[R * D];

  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const bool is_k = blockIdx.z != 0;
  const T* src = (is_k ? k : q) + ((size_t)bh * N + (size_t)i * block) * D;
  float* dst = (is_k ? kbar : qbar) + ((size_t)bh * nB + i) * D;
  const int len = min(block, N - i * block);

  const int c = threadIdx.x % C;
  const int r0 = threadIdx.x / C;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  for (int r = r0; r < len; r += R) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * D + c * VEC));
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] += Elem<T>::to_f(e[u]);
  }
#pragma unroll
  for (int u = 0; u < VEC; ++u) part[r0 * D + c * VEC + u] = acc[u];
  __syncthreads();
  const float inv_len = 1.0f / (float)len;
  for (int d = threadIdx.x; d < D; d += 256) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) s += part[r * D + d];
    dst[d] = s * inv_len;
  }
}

constexpr int kRows = 32;   // query-block rows per CTA
constexpr int kCols = 64;   // key blocks per score tile
constexpr int kDc = 32;     // head-dim slice staged in shared memory at a time

__host__ __device__ constexpr int scores_pad(int nB) { return ceil_div(nB, kCols) * kCols; }

__host__ __device__ constexpr size_t scores_smem_bytes(int nB) {
  return sizeof(float) * ((size_t)kDc * (kRows + 1) + (size_t)kDc * (kCols + 1) +
                          (size_t)kRows * scores_pad(nB)) +
         sizeof(uint32_t) * kRows * 32;
}

// Scores of 32 pooled queries against all pooled keys of a head, then the row
// softmax.  The 32 x 64 score tile is a register-tiled fp32 product: thread
// (ty, tx) of a 16 x 16 grid computes rows 2*ty, 2*ty+1 and columns
// tx + 16*c (c < 4): 6 shared-memory loads per 8 FMAs, from transposed
// slices of 32 head dimensions padded to odd strides (conflict-free both when
// staged and when read).
template <int D>
__global__ void __launch_bounds__(256)
block_scores_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                    int nB, float scale, const int32_t* __restrict__ cand_row_ptr,
                    const int32_t* __restrict__ cand_col, float* __restrict__ probs,
                    unsigned* err) {
  extern __shared__ float sm[];
  constexpr int QS = kRows + 1, KS = kCols + 1;    // padded strides
  float* qs = sm;                                  // [kDc][QS]   (transposed)
  float* ks = qs + kDc * QS;                       // [kDc][KS]   (transposed)
  float* sc = ks + kDc * KS;                       // [kRows][pad]
  const int pad = scores_pad(nB);
  uint32_t* cbits = reinterpret_cast<uint32_t*>(sc + kRows * pad);  // [kRows][32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * kRows;
  const int nrows = min(kRows, nB - i0);
  const bool reduced = cand_row_ptr != nullptr;

  if (reduced) {
    for (int idx = tid; idx < kRows * 32; idx += 256) cbits[idx] = 0u;
    __syncthreads();
    for (int rr = warp; rr < nrows; rr += 8) {
      const size_t row = (size_t)bh * nB + i0 + rr;
      const int cs = cand_row_ptr[row], ce = cand_row_ptr[row + 1];
      if (cs < 0 || ce < cs) {
        if (lane == 0) flag_error(err, kErrRowPtr);
        continue;
      }
      for (int e = cs + lane; e < ce; e += 32) {
        const int j = cand_col[e];
        if (j < 0 || j >= nB) {
          flag_error(err, kErrCsrIndex);
          continue;
        }
        atomicOr(&cbits[rr * 32 + (j >> 5)], 1u << (j & 31));
      }
    }
  }
  __syncthreads();

  const int ty = tid >> 4, tx = tid & 15;
  const float* qhead = qbar + ((size_t)bh * nB + i0) * D;
  for (int t0 = 0; t0 < nB; t0 += kCols) {
    if (reduced) {
      // skip a tile that holds no candidate of any of this CTA's rows
      bool any = false;
      if (tid < 64) {
        const int w = (t0 >> 5) + (tid >> 5);
        any = w < 32 && cbits[(tid & 31) * 32 + w] != 0u;
      }
      if (!__syncthreads_or(any)) continue;
    }
    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    const float* khead = kbar + ((size_t)bh * nB + t0) * D;
    for (int d0 = 0; d0 < D; d0 += kDc) {
      __syncthreads();  // previous slice consumed
      for (int idx = tid; idx < kRows * kDc; idx += 256) {
        const int rr = idx / kDc, d = idx - rr * kDc;
        qs[d * QS + rr] = rr < nrows ? qhead[(size_t)rr * D + d0 + d] : 0.f;
      }
      for (int idx = tid; idx < kCols * kDc; idx += 256) {
        const int cc = idx / kDc, d = idx - cc * kDc;
        ks[d * KS + cc] = t0 + cc < nB ? khead[(size_t)cc * D + d0 + d] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int d = 0; d < kDc; ++d) {
        const float q0v = qs[d * QS + 2 * ty], q1v = qs[d * QS + 2 * ty + 1];
        float kv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) kv[c] = ks[d * KS + tx + 16 * c];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[0][c] = fmaf(q0v, kv[c], acc[0][c]);
          acc[1][c] = fmaf(q1v, kv[c], acc[1][c]);
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) sc[(2 * ty + a) * pad + t0 + tx + 16 * c] = acc[a][c] * scale;
  }
  __syncthreads();

  // row softmax: one warp per row
  for (int r = warp; r < nrows; r += 8) {
    const uint32_t* bits = cbits + r * 32;
    float* srow = sc + r * pad;
    float mx = -INFINITY;
    for (int j = lane; j < nB; j += 32) {
      const bool cand = !reduced || ((bits[j >> 5] >> (j & 31)) & 1u);
      if (cand) mx = fmaxf(mx, srow[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int j = lane; j < nB; j += 32) {
      const bool cand = !reduced || ((bits[j >> 5] >> (j & 31)) & 1u);
      const float e = cand ? expf(srow[j] - mx) : 0.f;
      srow[j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    float* prow = probs + ((size_t)bh * nB + i0 + r) * nB;
    const bool empty = !(mx > -INFINITY);
    for (int j = lane; j < nB; j += 32) prow[j] = empty ? 0.f : srow[j] / sum;
  }
}

}  // namespace

cudaError_t launch_pool_means(const void* q, const void* k, bool bf16, int BH, int N,
                              int D, int block, float* qbar, float* kbar,
                              cudaStream_t s) {
  const int nB = ceil_div(N, block);
  const dim3 grid(nB, BH, 2);
  if (bf16) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    if (D == 64) pool_means_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(qq, kk, N, nB, block, qbar, kbar);
    else pool_means_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(qq, kk, N, nB, block, qbar, kbar);
  } else {
    auto* qq = static_cast<const float*>(q);
    auto* kk = static_cast<const float*>(k);
    if (D == 64) pool_means_kernel<float, 64><<<grid, 256, 0, s>>>(qq, kk, N, nB, block, qbar, kbar);
    else pool_means_kernel<float, 128><<<grid, 256, 0, s>>>(qq, kk, N, nB, block, qbar, kbar);
  }
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_scores_d(const float* qbar, const float* kbar, int BH, int nB,
                                   float scale, const int32_t* crp, const int32_t* cc,
                                   float* probs, unsigned* err, cudaStream_t s) {
  const size_t smem = scores_smem_bytes(nB);
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  block_scores_kernel<D><<<dim3(ceil_div(nB, kRows), BH), 256, smem, s>>>(
      qbar, kbar, nB, scale, crp, cc, probs, err);
  return cudaGetLastError();
}

cudaError_t launch_block_scores(const float* qbar, const float* kbar, int BH, int nB,
                                int D, float scale, const int32_t* cand_row_ptr,
                                const int32_t* cand_col, float* probs, unsigned* err,
                                cudaStream_t s) {
  if (D == 64)
    return launch_scores_d<64>(qbar, kbar, BH, nB, scale, cand_row_ptr, cand_col, probs, err, s);
  return launch_scores_d<128>(qbar, kbar, BH, nB, scale, cand_row_ptr, cand_col, probs, err, s);
}

}  // namespace dsa
