// Backward pass of the block-sparse attention (exact fp32 on CUDA cores).
//
// DSV (arXiv 2502.07590), abstract: DiTs are trained with the same dynamic
// sparsity, so the attention needs gradients over the selected blocks.  For
// a fixed CSR mask, with P = softmax over each query's selected keys (the
// forward's lse), dP = dO V^T and delta = rowsum(dO * O):
//
//   dS = P * (dP - delta),  dQ = scale * dS K,  dK = scale * dS^T Q,
//   dV = P^T dO.
//
// Kernels:
//   mask_bitmap    one bit per selected (row, column)
//   mask_transpose for every key block, the query blocks that selected it,
//                  ascending (count pass, scan, fill pass), so dK and dV are
//                  summed in a fixed order without atomics
//   delta          rowsum(dO * O) per token
//   dq             one CTA per query block over its selected key blocks
//   dkdv           one CTA per key block over the query blocks that chose it
// Tiles are staged as fp32 in shared memory with rows padded to D + 1 floats
// (a thread's own row reads fall in distinct banks, shared ones broadcast);
// the accumulators stay in registers.
#include "common.cuh"

namespace dsa {
namespace {

constexpr int kChunk = 32;  // keys (dq) or queries (dkdv) per staged chunk

__global__ void __launch_bounds__(256)
mask_bitmap_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                   int rows, int nB, uint32_t* __restrict__ bitmap, unsigned* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= rows) return;
  uint32_t* w = bitmap + (size_t)r * 32;
  w[lane] = 0u;
  __syncwarp();
  const int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  if (s0 < 0 || s1 < s0) {
    if (lane == 0) flag_error(err, kErrRowPtr);
    return;
  }
  for (int s = s0 + lane; s < s1; s += 32) {
    const int j = col_idx[s];
    if (j < 0 || j >= nB) {
      flag_error(err, kErrCsrIndex);
      continue;
    }
    atomicOr(&w[j >> 5], 1u << (j & 31));
  }
}

// One warp per (head, key block j): walks the head's query blocks in order.
// t_row_ptr == nullptr: count pass (writes counts); else fill pass.
__global__ void __launch_bounds__(256)
mask_transpose_kernel(const uint32_t* __restrict__ bitmap, int BH, int nB,
                      const int32_t* __restrict__ t_row_ptr, int32_t* __restrict__ counts,
                      int32_t* __restrict__ t_col) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int idx = blockIdx.x * 8 + warp;
  if (idx >= BH * nB) return;
  const int bh = idx / nB, j = idx - bh * nB;
  const uint32_t* head = bitmap + (size_t)bh * nB * 32;
  const int base = t_row_ptr ? t_row_ptr[idx] : 0;
  int cnt = 0;
  for (int i0 = 0; i0 < nB; i0 += 32) {
    const int i = i0 + lane;
    const bool hit = i < nB && ((head[(size_t)i * 32 + (j >> 5)] >> (j & 31)) & 1u);
    const unsigned b = __ballot_sync(0xffffffffu, hit);
    if (t_row_ptr && hit) t_col[base + cnt + __popc(b & ((1u << lane) - 1u))] = i;
    cnt += __popc(b);
  }
  if (!t_row_ptr && lane == 0) counts[idx] = cnt;
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
delta_kernel(const T* __restrict__ out, const T* __restrict__ dout, long long rows,
             float* __restrict__ delta) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * 8 + warp;
  if (r >= rows) return;
  float acc = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32)
    acc = fmaf(Elem<T>::to_f(out[r * D + d]), Elem<T>::to_f(dout[r * D + d]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) delta[r] = acc;
}

template <int D, int BS>
struct DqSmem {
  static constexpr int SD = D + 1;
  static constexpr size_t kFloats = 2 * BS * SD + 2 * kChunk * SD + BS * (kChunk + 1) + 2 * BS;
  static constexpr size_t kBytes = kFloats * sizeof(float);
};

template <int D, int BS>
struct DkvSmem {
  static constexpr int SD = D + 1;
  static constexpr size_t kFloats = 2 * BS * SD + 2 * kChunk * SD + 2 * kChunk * (BS + 1) + 2 * kChunk;
  static constexpr size_t kBytes = kFloats * sizeof(float);
};

// dQ of query block (bh, i): for every chunk of 32 keys of its selected
// blocks, thread (qr, grp) first forms S and dP for query qr and keys
// grp*KPT .. +KPT-1 of the chunk, then adds dS * K into columns
// grp*DPT .. +DPT-1 of its dQ row.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256, 1)
dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
          const T* __restrict__ dout, const float* __restrict__ lse,
          const float* __restrict__ delta, int N, int nB, float scale,
          const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
          T* __restrict__ dq) {
  constexpr int SD = D + 1;
  constexpr int KG = 256 / BS, KPT = kChunk / KG, DPT = D / KG;
  extern __shared__ float sm[];
  float* Qs = sm;                        // [BS][SD]
  float* Os = Qs + BS * SD;              // dO [BS][SD]
  float* Ks = Os + BS * SD;              // [kChunk][SD]
  float* Vs = Ks + kChunk * SD;          // [kChunk][SD]
  float* dSs = Vs + kChunk * SD;         // [BS][kChunk + 1]
  float* lse_s = dSs + BS * (kChunk + 1);
  float* dl_s = lse_s + BS;

  const int tid = threadIdx.x;
  const int r = blockIdx.x;
  const int bh = r / nB, i = r - bh * nB;
  const int q0 = i * BS, qlen = min(BS, N - q0);
  const size_t head = (size_t)bh * N;
  for (int idx = tid; idx < BS * D; idx += 256) {
    const int rr = idx / D, d = idx - rr * D;
    const bool ok = rr < qlen;
    Qs[rr * SD + d] = ok ? Elem<T>::to_f(q[(head + q0 + rr) * D + d]) : 0.f;
    Os[rr * SD + d] = ok ? Elem<T>::to_f(dout[(head + q0 + rr) * D + d]) : 0.f;
  }
  for (int rr = tid; rr < BS; rr += 256) {
    lse_s[rr] = rr < qlen ? lse[head + q0 + rr] : 0.f;
    dl_s[rr] = rr < qlen ? delta[head + q0 + rr] : 0.f;
  }
  const int qr = tid % BS, grp = tid / BS;
  float acc[DPT];
#pragma unroll
  for (int c = 0; c < DPT; ++c) acc[c] = 0.f;

  const int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  for (int s = s0; s < s1; ++s) {
    const int j = col_idx[s];
    if (j < 0 || j >= nB) continue;  // flagged by mask_bitmap
    const int k0 = j * BS, klen = min(BS, N - k0);
    for (int c0 = 0; c0 < klen; c0 += kChunk) {
      __syncthreads();  // the previous chunk is consumed (and Q, dO staged)
      for (int idx = tid; idx < kChunk * D; idx += 256) {
        const int kk = idx / D, d = idx - kk * D;
        const bool ok = c0 + kk < klen;
        Ks[kk * SD + d] = ok ? Elem<T>::to_f(k[(head + k0 + c0 + kk) * D + d]) : 0.f;
        Vs[kk * SD + d] = ok ? Elem<T>::to_f(v[(head + k0 + c0 + kk) * D + d]) : 0.f;
      }
      __syncthreads();
      float sv[KPT], dp[KPT];
#pragma unroll
      for (int u = 0; u < KPT; ++u) sv[u] = dp[u] = 0.f;
#pragma unroll 4
      for (int d = 0; d < D; ++d) {
        const float qv = Qs[qr * SD + d], ov = Os[qr * SD + d];
#pragma unroll
        for (int u = 0; u < KPT; ++u) {
          const int kk = grp * KPT + u;
          sv[u] = fmaf(qv, Ks[kk * SD + d], sv[u]);
          dp[u] = fmaf(ov, Vs[kk * SD + d], dp[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        const int kk = grp * KPT + u;
        const bool ok = qr < qlen && c0 + kk < klen;
        const float p = ok ? expf(scale * sv[u] - lse_s[qr]) : 0.f;
        dSs[qr * (kChunk + 1) + kk] = p * (dp[u] - dl_s[qr]);
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kChunk; ++kk) {
        const float ds = dSs[qr * (kChunk + 1) + kk];
#pragma unroll
        for (int c = 0; c < DPT; ++c) acc[c] = fmaf(ds, Ks[kk * SD + grp * DPT + c], acc[c]);
      }
    }
  }
  if (qr < qlen) {
#pragma unroll
    for (int c = 0; c < DPT; ++c)
      dq[(head + q0 + qr) * D + grp * DPT + c] = Elem<T>::from_f(scale * acc[c]);
  }
}

// dK and dV of key block (bh, j): for every chunk of 32 queries of the query
// blocks that selected it, thread (kc, grp) forms P and dS for key kc and
// queries grp*QPT .. +QPT-1, then thread (kr, grp) adds P^T dO and dS^T Q
// into columns grp*DPT .. +DPT-1 of rows kr of dV and dK.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256, 1)
dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            const T* __restrict__ dout, const float* __restrict__ lse,
            const float* __restrict__ delta, int N, int nB, float scale,
            const int32_t* __restrict__ t_row_ptr, const int32_t* __restrict__ t_col,
            T* __restrict__ dk, T* __restrict__ dv) {
  constexpr int SD = D + 1;
  constexpr int KG = 256 / BS, QPT = kChunk / KG, DPT = D / KG;
  extern __shared__ float sm[];
  float* Ks = sm;                        // [BS][SD]
  float* Vs = Ks + BS * SD;              // [BS][SD]
  float* Qc = Vs + BS * SD;              // [kChunk][SD]
  float* Oc = Qc + kChunk * SD;          // dO [kChunk][SD]
  float* Ps = Oc + kChunk * SD;          // [kChunk][BS + 1]
  float* dSs = Ps + kChunk * (BS + 1);   // [kChunk][BS + 1]
  float* lse_c = dSs + kChunk * (BS + 1);
  float* dl_c = lse_c + kChunk;

  const int tid = threadIdx.x;
  const int idx_kb = blockIdx.x;
  const int bh = idx_kb / nB, j = idx_kb - bh * nB;
  const int k0 = j * BS, klen = min(BS, N - k0);
  const size_t head = (size_t)bh * N;
  for (int idx = tid; idx < BS * D; idx += 256) {
    const int rr = idx / D, d = idx - rr * D;
    const bool ok = rr < klen;
    Ks[rr * SD + d] = ok ? Elem<T>::to_f(k[(head + k0 + rr) * D + d]) : 0.f;
    Vs[rr * SD + d] = ok ? Elem<T>::to_f(v[(head + k0 + rr) * D + d]) : 0.f;
  }
  const int kc = tid % BS, grp = tid / BS;
  float ak[DPT], av[DPT];
#pragma unroll
  for (int c = 0; c < DPT; ++c) ak[c] = av[c] = 0.f;

  const int t0 = t_row_ptr[idx_kb], t1 = t_row_ptr[idx_kb + 1];
  for (int t = t0; t < t1; ++t) {
    const int i = t_col[t];
    const int q0 = i * BS, qlen = min(BS, N - q0);
    for (int c0 = 0; c0 < qlen; c0 += kChunk) {
      __syncthreads();  // the previous chunk is consumed (and K, V staged)
      for (int idx = tid; idx < kChunk * D; idx += 256) {
        const int qq = idx / D, d = idx - qq * D;
        const bool ok = c0 + qq < qlen;
        Qc[qq * SD + d] = ok ? Elem<T>::to_f(q[(head + q0 + c0 + qq) * D + d]) : 0.f;
        Oc[qq * SD + d] = ok ? Elem<T>::to_f(dout[(head + q0 + c0 + qq) * D + d]) : 0.f;
      }
      for (int qq = tid; qq < kChunk; qq += 256) {
        const bool ok = c0 + qq < qlen;
        lse_c[qq] = ok ? lse[head + q0 + c0 + qq] : 0.f;
        dl_c[qq] = ok ? delta[head + q0 + c0 + qq] : 0.f;
      }
      __syncthreads();
      float sv[QPT], dp[QPT];
#pragma unroll
      for (int u = 0; u < QPT; ++u) sv[u] = dp[u] = 0.f;
#pragma unroll 4
      for (int d = 0; d < D; ++d) {
        const float kv = Ks[kc * SD + d], vv = Vs[kc * SD + d];
#pragma unroll
        for (int u = 0; u < QPT; ++u) {
          const int qq = grp * QPT + u;
          sv[u] = fmaf(Qc[qq * SD + d], kv, sv[u]);
          dp[u] = fmaf(Oc[qq * SD + d], vv, dp[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < QPT; ++u) {
        const int qq = grp * QPT + u;
        const bool ok = c0 + qq < qlen && kc < klen;
        const float p = ok ? expf(scale * sv[u] - lse_c[qq]) : 0.f;
        Ps[qq * (BS + 1) + kc] = p;
        dSs[qq * (BS + 1) + kc] = p * (dp[u] - dl_c[qq]);
      }
      __syncthreads();
#pragma unroll 4
      for (int qq = 0; qq < kChunk; ++qq) {
        const float p = Ps[qq * (BS + 1) + kc], ds = dSs[qq * (BS + 1) + kc];
#pragma unroll
        for (int c = 0; c < DPT; ++c) {
          av[c] = fmaf(p, Oc[qq * SD + grp * DPT + c], av[c]);
          ak[c] = fmaf(ds, Qc[qq * SD + grp * DPT + c], ak[c]);
        }
      }
    }
  }
  if (kc < klen) {
#pragma unroll
    for (int c = 0; c < DPT; ++c) {
      dk[(head + k0 + kc) * D + grp * DPT + c] = Elem<T>::from_f(scale * ak[c]);
      dv[(head + k0 + kc) * D + grp * DPT + c] = Elem<T>::from_f(av[c]);
    }
  }
}

template <typename T, int D, int BS>
cudaError_t launch_grads(const void* q, const void* k, const void* v, const void* dout,
                         const float* lse, const float* delta, int BH, int N, int nB,
                         float scale, const int32_t* row_ptr, const int32_t* col_idx,
                         const int32_t* t_row_ptr, const int32_t* t_col, void* dq, void* dk,
                         void* dv, cudaStream_t s) {
  const size_t sq = DqSmem<D, BS>::kBytes, skv = DkvSmem<D, BS>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(dq_kernel<T, D, BS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(dkdv_kernel<T, D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)skv);
  if (e != cudaSuccess) return e;
  const int rows = BH * nB;
  dq_kernel<T, D, BS><<<rows, 256, sq, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dout), lse, delta, N, nB, scale, row_ptr, col_idx,
      static_cast<T*>(dq));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dkdv_kernel<T, D, BS><<<rows, 256, skv, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dout), lse, delta, N, nB, scale, t_row_ptr, t_col,
      static_cast<T*>(dk), static_cast<T*>(dv));
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_grads_t(int D, int block, const void* q, const void* k, const void* v,
                           const void* dout, const float* lse, const float* delta, int BH,
                           int N, int nB, float scale, const int32_t* row_ptr,
                           const int32_t* col_idx, const int32_t* t_row_ptr,
                           const int32_t* t_col, void* dq, void* dk, void* dv, cudaStream_t s) {
#define DSA_GRADS(DD, BB)                                                                    \
  if (D == DD && block == BB)                                                                \
    return launch_grads<T, DD, BB>(q, k, v, dout, lse, delta, BH, N, nB, scale, row_ptr,   \
                                   col_idx, t_row_ptr, t_col, dq, dk, dv, s);
  DSA_GRADS(64, 64) DSA_GRADS(64, 128) DSA_GRADS(128, 64) DSA_GRADS(128, 128)
#undef DSA_GRADS
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, bool bf16, int BH, int N, int D,
                            int block, float scale, const int32_t* row_ptr,
                            const int32_t* col_idx, void* dq, void* dk, void* dv,
                            uint32_t* bitmap, int32_t* counts, int32_t* t_row_ptr,
                            int32_t* t_col, float* delta, unsigned* err, cudaStream_t s) {
  const int nB = ceil_div(N, block);
  const int rows = BH * nB;
  mask_bitmap_kernel<<<ceil_div(rows, 8), 256, 0, s>>>(row_ptr, col_idx, rows, nB, bitmap, err);
  mask_transpose_kernel<<<ceil_div(rows, 8), 256, 0, s>>>(bitmap, BH, nB, nullptr, counts,
                                                          nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if ((e = launch_csr_scan(counts, rows, t_row_ptr, s)) != cudaSuccess) return e;
  mask_transpose_kernel<<<ceil_div(rows, 8), 256, 0, s>>>(bitmap, BH, nB, t_row_ptr, counts,
                                                          t_col);
  const long long tok = (long long)BH * N;
  const int dgrid = (int)((tok + 7) / 8);
  if (bf16) {
    if (D == 64)
      delta_kernel<__nv_bfloat16, 64><<<dgrid, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), tok, delta);
    else
      delta_kernel<__nv_bfloat16, 128><<<dgrid, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), tok, delta);
  } else {
    if (D == 64)
      delta_kernel<float, 64><<<dgrid, 256, 0, s>>>(static_cast<const float*>(out),
                                                     static_cast<const float*>(dout), tok, delta);
    else
      delta_kernel<float, 128><<<dgrid, 256, 0, s>>>(static_cast<const float*>(out),
                                                      static_cast<const float*>(dout), tok, delta);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // bf16 with blocks of 128: the tensor-core kernels; otherwise exact fp32 on CUDA cores
  if (bf16 && block == 128)
    return launch_attn_bwd_sm100(q, k, v, dout, lse, delta, BH, N, D, scale, row_ptr, col_idx,
                                 t_row_ptr, t_col, dq, dk, dv, err, s);
  if (bf16)
    return launch_grads_t<__nv_bfloat16>(D, block, q, k, v, dout, lse, delta, BH, N, nB, scale,
                                         row_ptr, col_idx, t_row_ptr, t_col, dq, dk, dv, s);
  return launch_grads_t<float>(D, block, q, k, v, dout, lse, delta, BH, N, nB, scale, row_ptr,
                               col_idx, t_row_ptr, t_col, dq, dk, dv, s);
}

}  // namespace dsa
