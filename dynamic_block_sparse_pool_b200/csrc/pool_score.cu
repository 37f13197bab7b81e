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
// Two-level estimate (DFSAttn abstract: hierarchical block scoring): the
//   two kernels above at sub-block granularity, then aggregate_probs folds
//   the fine row softmax back into block rows (token-weighted over query
//   sub-blocks, summed over key sub-blocks).
// Kernel 2 (block_scores): one CTA per (64 query-block rows, head): a
//   register-tiled fp32 product of the 64 pooled queries with tiles of 64
//   pooled keys (cp.async; one tile buffer and three CTAs per SM), scaled
//   scores written to P with a running max and sum per row, then P
//   normalised in place from L2.
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

constexpr int kTile = 64;  // query-block rows per CTA and key blocks per score tile
// Key tiles in shared memory: with one (76 KB per CTA, 80 registers) three
// CTAs fit on an SM, and the other two hide each one's tile loads; with two
// (double buffering, 110 KB) only two fit, and a launch over 40 heads (400
// CTAs) takes two waves of 296 slots.
#ifndef DSA_SCORE_KBUFS
#define DSA_SCORE_KBUFS 1
#endif
constexpr int kKBufs = DSA_SCORE_KBUFS;
constexpr int kScoreCtasPerSm = kKBufs == 1 ? 3 : 2;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Shared memory of the score kernel: the CTA's 64 pooled queries, a double
// buffer of 64 pooled keys (rows padded to D + 4 floats: 16-byte aligned, and
// each quarter-warp's float4 reads fall in distinct banks), the candidate
// bitmaps and the per-row softmax statistics.
template <int D>
struct ScoreSmem {
  static constexpr int kStride = D + 4;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile * kStride;          // floats
  static constexpr int kBits = kK + kKBufs * kTile * kStride;  // floats -> uint32 [64][32]
  static constexpr int kStat = kBits + kTile * 32;         // float2 [64]
  static constexpr size_t kBytes = sizeof(float) * (size_t)(kStat + 2 * kTile);
};

// Copies `count` rows (count >= 1) of D floats starting at row `first` into a
// 64-row tile; rows past `count` repeat the last row (their scores are never
// used).
template <int D>
__device__ __forceinline__ void stage_rows(float* dst, const float* src, int first, int count,
                                           int tid) {
  constexpr int C = D / 4;  // 16-byte chunks per row
#pragma unroll 2
  for (int c = tid; c < kTile * C; c += 256) {
    const int r = c / C, q4 = c - r * C;
    const int rr = min(r, count - 1);
    cp_async16(dst + r * ScoreSmem<D>::kStride + q4 * 4, src + (size_t)(first + rr) * D + q4 * 4);
  }
}

// Softmax over the key blocks of scale * qbar_i . kbar_j for 64 query blocks
// of one head (all key blocks, or the candidate set of each row).
//   Pass 1: 64 x 64 score tiles, thread (ty, tx) of a 16 x 16 grid holding
//     rows 4ty .. 4ty+3 and columns tx + 16c (c < 4), fp32 FMAs over the
//     head dimension.  The scaled scores go to P as they are; each thread
//     keeps a running (max, sum of exp) per row, merged across the 16
//     threads of a row at the end.
//   Pass 2: one warp per row rewrites P as exp(s - max) / sum (reads hit L2:
//     the CTA wrote them just before).  Non-candidates and empty rows get 0.
template <int D>
__global__ void __launch_bounds__(256, kScoreCtasPerSm)
block_scores_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                    int nB, float scale, const int32_t* __restrict__ cand_row_ptr,
                    const int32_t* __restrict__ cand_col, float* __restrict__ probs,
                    unsigned* err) {
  using L = ScoreSmem<D>;
  constexpr int S = L::kStride;
  extern __shared__ __align__(16) float sm[];
  float* qs = sm + L::kQ;
  float* ks = sm + L::kK;
  uint32_t* cbits = reinterpret_cast<uint32_t*>(sm + L::kBits);  // [64][32]
  float2* stat = reinterpret_cast<float2*>(sm + L::kStat);       // [64]
  __shared__ uint32_t live_tiles;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ty = tid >> 4, tx = tid & 15;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * kTile;
  const int nrows = min(kTile, nB - i0);
  const int n_tiles = ceil_div(nB, kTile);
  const bool reduced = cand_row_ptr != nullptr;
  const float* khead = kbar + (size_t)bh * nB * D;

  stage_rows<D>(qs, qbar + (size_t)bh * nB * D, i0, nrows, tid);
  cp_async_commit();

  if (tid == 0) live_tiles = reduced ? 0u : (n_tiles >= 32 ? 0xFFFFFFFFu : (1u << n_tiles) - 1u);
  if (reduced) {
    for (int idx = tid; idx < kTile * 32; idx += 256) cbits[idx] = 0u;
    __syncthreads();
    for (int rr = warp; rr < nrows; rr += 8) {
      const size_t row = (size_t)bh * nB + i0 + rr;
      const int cs = cand_row_ptr[row], ce = cand_row_ptr[row + 1];
      if (cs < 0 || ce < cs) {
        if (lane == 0) flag_error(err, kErrRowPtr);
        continue;
      }
      // four independent index loads per lane in flight, then the marks
      constexpr int kU = 4;
      for (int e0 = cs + lane; e0 < ce; e0 += 32 * kU) {
        int jj[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int e = e0 + 32 * u;
          jj[u] = e < ce ? cand_col[e] : 0;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (e0 + 32 * u >= ce) continue;  // past the row's end
          const int j = jj[u];
          if (j < 0 || j >= nB) {
            flag_error(err, kErrCsrIndex);
            continue;
          }
          atomicOr(&cbits[rr * 32 + (j >> 5)], 1u << (j & 31));
        }
      }
    }
    __syncthreads();
    // tiles holding a candidate of any of the CTA's rows (word w covers tile w / 2)
    uint32_t mine = 0u;
    for (int rr = warp; rr < nrows; rr += 8)
      if (cbits[rr * 32 + lane]) mine |= 1u << (lane >> 1);
    mine = __reduce_or_sync(0xffffffffu, mine);
    if (lane == 0 && mine) atomicOr(&live_tiles, mine);
  }
  __syncthreads();
  uint32_t live = live_tiles;

  float run_m[4], run_s[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    run_m[a] = -INFINITY;
    run_s[a] = 0.f;
  }
  float* prow_base = probs + ((size_t)bh * nB + i0) * nB;

  int t = live ? __ffs(live) - 1 : n_tiles;
  if (t < n_tiles) stage_rows<D>(ks, khead, t * kTile, min(kTile, nB - t * kTile), tid);
  cp_async_commit();
  for (int buf = 0; t < n_tiles; buf = kKBufs == 2 ? buf ^ 1 : 0) {
    live &= ~(1u << t);
    const int tn = live ? __ffs(live) - 1 : n_tiles;
    if (kKBufs == 2) {
      if (tn < n_tiles)
        stage_rows<D>(ks + (buf ^ 1) * kTile * S, khead, tn * kTile, min(kTile, nB - tn * kTile), tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const float* kt = ks + buf * kTile * S;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 2
    for (int d = 0; d < D; d += 4) {
      float4 qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = *reinterpret_cast<const float4*>(qs + (4 * ty + a) * S + d);
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = *reinterpret_cast<const float4*>(kt + (tx + 16 * c) * S + d);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[a][c] = fmaf(qv[a].x, kv[c].x, acc[a][c]);
          acc[a][c] = fmaf(qv[a].y, kv[c].y, acc[a][c]);
          acc[a][c] = fmaf(qv[a].z, kv[c].z, acc[a][c]);
          acc[a][c] = fmaf(qv[a].w, kv[c].w, acc[a][c]);
        }
    }

#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = 4 * ty + a;
      float x[4];
      bool ok[4];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = t * kTile + tx + 16 * c;
        x[c] = acc[a][c] * scale;
        ok[c] = r < nrows && j < nB && (!reduced || ((cbits[r * 32 + (j >> 5)] >> (j & 31)) & 1u));
        if (ok[c]) {
          prow_base[(size_t)r * nB + j] = x[c];
          mx = fmaxf(mx, x[c]);
        }
      }
      if (mx > run_m[a]) {
        run_s[a] = run_m[a] == -INFINITY ? 0.f : run_s[a] * expf(run_m[a] - mx);
        run_m[a] = mx;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (ok[c]) run_s[a] += expf(x[c] - run_m[a]);
    }
    __syncthreads();  // every read of this buffer is done; it is refilled next
    if (kKBufs == 1) {
      if (tn < n_tiles) stage_rows<D>(ks, khead, tn * kTile, min(kTile, nB - tn * kTile), tid);
      cp_async_commit();
    }
    t = tn;
  }
  cp_async_wait<0>();

  // merge the 16 partial (max, sum) of each row: lanes tx of one half-warp
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    float m = run_m[a], s = run_s[a];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m, o);
      const float so = __shfl_xor_sync(0xffffffffu, s, o);
      const float M = fmaxf(m, mo);
      s = (m == -INFINITY ? 0.f : s * expf(m - M)) + (mo == -INFINITY ? 0.f : so * expf(mo - M));
      m = M;
    }
    if (tx == 0) stat[4 * ty + a] = make_float2(m, s);
  }
  __syncthreads();  // also orders pass 1's global writes before pass 2's reads

  // 16 independent loads per lane in flight (the reads come from L2)
  constexpr int kU = 16;
  for (int r = warp; r < nrows; r += 8) {
    const float2 ms = stat[r];
    const bool empty = !(ms.x > -INFINITY);
    const uint32_t* bits = cbits + r * 32;
    float* prow = prow_base + (size_t)r * nB;
    for (int j0 = lane; j0 < nB; j0 += 32 * kU) {
      float x[kU];
      bool cand[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + 32 * u;
        cand[u] = j < nB && !empty && (!reduced || ((bits[j >> 5] >> (j & 31)) & 1u));
        x[u] = cand[u] ? prow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + 32 * u;
        if (j < nB) prow[j] = cand[u] ? expf(x[u] - ms.x) / ms.y : 0.f;
      }
    }
  }
}

// Block rows of the two-level estimate from the fine (sub-block) row softmax
// pf [BH, nBf, nBf]: P[i, j] = sum over the query sub-blocks a of block i of
// (|a| / |B_i|) * (sum of pf[a, b] over the key sub-blocks b of block j).
// One warp per block row, lanes over block columns; each fine value is read
// once.
__global__ void __launch_bounds__(256)
aggregate_probs_kernel(const float* __restrict__ pf, int N, int block, int sub, int nB, int nBf,
                       float* __restrict__ probs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (i >= nB) return;
  const int bf = block / sub;
  const int i0 = i * block;
  const float inv_len = 1.0f / (float)min(block, N - i0);
  const float* fhead = pf + (size_t)bh * nBf * nBf;
  float* prow = probs + ((size_t)bh * nB + i) * nB;
  for (int j = lane; j < nB; j += 32) {
    float acc = 0.f;
    for (int a = i * sub; a < min((i + 1) * sub, nBf); ++a) {
      const float w = (float)min(bf, N - a * bf) * inv_len;
      const float* frow = fhead + (size_t)a * nBf;
      float part = 0.f;
      for (int b = j * sub; b < min((j + 1) * sub, nBf); ++b) part += frow[b];
      acc = fmaf(w, part, acc);
    }
    prow[j] = acc;
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
  const size_t smem = ScoreSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  block_scores_kernel<D><<<dim3(ceil_div(nB, kTile), BH), 256, smem, s>>>(
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

namespace dsa {

cudaError_t launch_aggregate_probs(const float* pf, int BH, int N, int block, int sub, int nB,
                                   int nBf, float* probs, cudaStream_t s) {
  aggregate_probs_kernel<<<dim3(ceil_div(nB, 8), BH), 256, 0, s>>>(pf, N, block, sub, nB, nBf, probs);
  return cudaGetLastError();
}

}  // namespace dsa
