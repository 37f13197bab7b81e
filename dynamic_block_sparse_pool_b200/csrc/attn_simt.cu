// Block-sparse attention forward on CUDA cores, exact fp32 arithmetic.
//
// Serves fp32 inputs (where a tf32 tensor-core product would miss a 1e-4
// error budget) and block size 64.  Same contract as the tensor-core path:
// for every query of block i, online softmax over the keys of the blocks in
// CSR row i, plus per-block log-sums for the exact block mass (GSRS, arXiv
// 2610.21129, abstract: exact attention weights inside the FlashAttention
// computation).
//
// One CTA (256 threads) per (head, query block).  TPR = 256 / block threads
// share a query row: each owns D / TPR output columns and KT / TPR scores of
// every 32-key tile.  Q stays in shared memory as fp32; K and V tiles of 32
// keys stream through shared memory.
#include "common.cuh"

namespace dsa {
namespace {

constexpr int KT = 32;

template <int D, int BS>
__host__ __device__ constexpr size_t simt_smem_floats() {
  return (size_t)BS * (D + 1) + (size_t)KT * (D + 1) + (size_t)KT * D + (size_t)BS * (KT + 1);
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(256)
attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 int N, int nB, float scale, const int32_t* __restrict__ row_ptr,
                 const int32_t* __restrict__ col_idx, T* __restrict__ out,
                 float* __restrict__ lse, float* __restrict__ blk_lse, unsigned* err) {
  constexpr int TPR = 256 / BS;
  constexpr int SPT = KT / TPR;
  constexpr int OPT = D / TPR;
  extern __shared__ float sm[];
  float* Qs = sm;                    // [BS][D+1]
  float* Ks = Qs + BS * (D + 1);     // [KT][D+1]
  float* Vs = Ks + KT * (D + 1);     // [KT][D]
  float* Ps = Vs + KT * D;           // [BS][KT+1]

  const int tid = threadIdx.x;
  const int row = tid / TPR, part = tid % TPR;
  const int r = blockIdx.x;
  const int bh = r / nB, i = r - bh * nB;
  const int q0 = i * BS;
  const int qlen = min(BS, N - q0);
  const size_t head = (size_t)bh * N;

  int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  bool bad = s0 < 0 || s1 < s0;
  if (!bad)
    for (int e = s0 + tid; e < s1; e += 256) {
      const int j = col_idx[e];
      bad |= (j < 0 || j >= nB);
    }
  if (__syncthreads_or(bad)) {
    if (tid == 0) flag_error(err, (s0 < 0 || s1 < s0) ? kErrRowPtr : kErrCsrIndex);
    s1 = s0;  // treat the row as empty
  }

  for (int idx = tid; idx < BS * D; idx += 256) {
    const int rr = idx / D, d = idx - rr * D;
    Qs[rr * (D + 1) + d] = rr < qlen ? Elem<T>::to_f(q[(head + q0 + rr) * D + d]) : 0.f;
  }

  float o[OPT];
#pragma unroll
  for (int c = 0; c < OPT; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int slot = s0; slot < s1; ++slot) {
    const int j = col_idx[slot];
    const int k0 = j * BS;
    const int klen = min(BS, N - k0);
    float b = 0.f;  // this block's share of the denominator, relative to m
    for (int kt = 0; kt < klen; kt += KT) {
      __syncthreads();  // previous tile fully consumed (and Qs written)
      for (int idx = tid; idx < KT * D; idx += 256) {
        const int u = idx / D, d = idx - u * D;
        const bool ok = kt + u < klen;
        const size_t g = (head + k0 + kt + u) * D + d;
        Ks[u * (D + 1) + d] = ok ? Elem<T>::to_f(k[g]) : 0.f;
        Vs[u * D + d] = ok ? Elem<T>::to_f(v[g]) : 0.f;
      }
      __syncthreads();

      float sv[SPT];
#pragma unroll
      for (int c = 0; c < SPT; ++c) sv[c] = 0.f;
      for (int d = 0; d < D; ++d) {
        const float qv = Qs[row * (D + 1) + d];
#pragma unroll
        for (int c = 0; c < SPT; ++c) sv[c] = fmaf(qv, Ks[(part + TPR * c) * (D + 1) + d], sv[c]);
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < SPT; ++c) {
        sv[c] = (kt + part + TPR * c < klen) ? sv[c] * scale : -INFINITY;
        tmax = fmaxf(tmax, sv[c]);
      }
#pragma unroll
      for (int off = 1; off < TPR; off <<= 1)
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float m_new = fmaxf(m, tmax);
      const float alpha = expf(m - m_new);
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < SPT; ++c) {
        const float p = expf(sv[c] - m_new);
        Ps[row * (KT + 1) + part + TPR * c] = p;
        psum += p;
      }
#pragma unroll
      for (int off = 1; off < TPR; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      l = l * alpha + psum;
      b = b * alpha + psum;
      m = m_new;
#pragma unroll
      for (int c = 0; c < OPT; ++c) o[c] *= alpha;
      __syncwarp();
#pragma unroll 4
      for (int u = 0; u < KT; ++u) {
        const float pu = Ps[row * (KT + 1) + u];
#pragma unroll
        for (int c = 0; c < OPT; ++c) o[c] = fmaf(pu, Vs[u * D + part + TPR * c], o[c]);
      }
    }
    if (blk_lse && part == 0 && row < qlen) blk_lse[(size_t)slot * BS + row] = m + logf(b);
  }

  if (row < qlen) {
    const bool empty = s1 == s0;
    const float inv = empty ? 0.f : 1.0f / l;
    T* orow = out + (head + q0 + row) * D;
#pragma unroll
    for (int c = 0; c < OPT; ++c) orow[part + TPR * c] = Elem<T>::from_f(o[c] * inv);
    if (lse && part == 0) lse[head + q0 + row] = empty ? -INFINITY : m + logf(l);
  }
}

template <typename T, int D, int BS>
cudaError_t launch_simt_t(const void* q, const void* k, const void* v, int BH, int N,
                          float scale, const int32_t* row_ptr, const int32_t* col_idx,
                          void* out, float* lse, float* blk_lse, unsigned* err,
                          cudaStream_t s) {
  const int nB = ceil_div(N, BS);
  const size_t smem = simt_smem_floats<D, BS>() * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D, BS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_simt_kernel<T, D, BS><<<BH * nB, 256, smem, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), N, nB,
      scale, row_ptr, col_idx, static_cast<T*>(out), lse, blk_lse, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, bool bf16,
                             int BH, int N, int D, int block, float scale,
                             const int32_t* row_ptr, const int32_t* col_idx, void* out,
                             float* lse, float* blk_lse, unsigned* err, cudaStream_t s) {
#define DSA_SIMT(T, DD, BB)                                                              \
  if (D == DD && block == BB)                                                            \
    return launch_simt_t<T, DD, BB>(q, k, v, BH, N, scale, row_ptr, col_idx, out, lse,   \
                                    blk_lse, err, s);
  if (bf16) {
    DSA_SIMT(__nv_bfloat16, 64, 64)
    DSA_SIMT(__nv_bfloat16, 64, 128)
    DSA_SIMT(__nv_bfloat16, 128, 64)
    DSA_SIMT(__nv_bfloat16, 128, 128)
  } else {
    DSA_SIMT(float, 64, 64)
    DSA_SIMT(float, 64, 128)
    DSA_SIMT(float, 128, 64)
    DSA_SIMT(float, 128, 128)
  }
#undef DSA_SIMT
  return cudaErrorInvalidValue;
}

}  // namespace dsa
