// Exact softmax mass of every selected key block.
//
// GSRS (arXiv 2610.21129), abstract: the exact attention weight of each
// block comes out of the FlashAttention pass at negligible overhead; Figure
// 2 measures the recall of a block mask with the same quantity.
//
// mass[s] = mean over the queries t of block i of exp(blk_lse[s, t] - lse_t),
// where blk_lse[s, t] is the log of the block's share of the softmax
// denominator and lse_t the log of the whole denominator (both written by
// the attention kernel).  One CTA per CSR row; each of its 8 warps keeps the
// row's lse values in registers and reduces every 8th slot, two at a time,
// reading each slot's block-size run of blk_lse once, coalesced.
//
// mass_to_probs scatters those masses back into dense rows, so that a Top-p
// selection can run on exact attention weights (GSRS abstract: Top-p
// selection supported by exact attention weights from the FlashAttention
// pass; Figure 4: later searches evaluate only the candidate mask).
#include "common.cuh"

namespace dsa {
namespace {

template <int BS>
__global__ void __launch_bounds__(256)
block_mass_kernel(const float* __restrict__ lse, const float* __restrict__ blk, int N,
                  int nB, const int32_t* __restrict__ row_ptr, float* __restrict__ mass) {
  constexpr int PER = BS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x;
  const int bh = r / nB, i = r - bh * nB;
  const int q0 = i * BS;
  const int qlen = min(BS, N - q0);
  // the row's lse values load together with its row_ptr entries (they
  // depend on the row index only)
  float lv[PER];
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    const int t = lane + 32 * m;
    lv[m] = t < qlen ? lse[(size_t)bh * N + q0 + t] : 0.f;
  }
  const int s0 = row_ptr[r], s1 = row_ptr[r + 1];
  if (s1 <= s0) return;
  const float inv = 1.0f / (float)qlen;
  // the row's slots are spread over the CTA's 8 warps, two slots per step
  // (2 * PER loads per lane in flight)
  for (int s = s0 + warp; s < s1; s += 16) {
    const bool two = s + 8 < s1;
    const float* b0 = blk + (size_t)s * BS;
    const float* b1 = blk + (size_t)(two ? s + 8 : s) * BS;
    float x0[PER], x1[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int t = lane + 32 * m;
      x0[m] = t < qlen ? b0[t] : 0.f;
      x1[m] = t < qlen ? b1[t] : 0.f;
    }
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int t = lane + 32 * m;
      if (t < qlen) {
        acc0 += expf(x0[m] - lv[m]);
        acc1 += expf(x1[m] - lv[m]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
      acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
    }
    if (lane == 0) {
      mass[s] = acc0 * inv;
      if (two) mass[s + 8] = acc1 * inv;
    }
  }
}

// Dense probability rows from the exact masses of a CSR mask: row r of
// probs gets mass[s] at column col_idx[s] for each of its slots s and 0
// elsewhere.  One warp per row: it zeroes the row (coalesced), then writes
// its slots; __syncwarp orders the two.
__global__ void __launch_bounds__(256)
mass_to_probs_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                     const float* __restrict__ mass, int rows, int nB, float* __restrict__ probs,
                     unsigned* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= rows) return;  // whole warp leaves together
  float* prow = probs + (size_t)r * nB;
  for (int j = lane; j < nB; j += 32) prow[j] = 0.f;
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
    prow[j] = mass[s];
  }
}

}  // namespace

cudaError_t launch_mass_to_probs(const int32_t* row_ptr, const int32_t* col_idx,
                                 const float* mass, int rows, int nB, float* probs,
                                 unsigned* err, cudaStream_t s) {
  if (rows > 0)
    mass_to_probs_kernel<<<ceil_div(rows, 8), 256, 0, s>>>(row_ptr, col_idx, mass, rows, nB,
                                                           probs, err);
  return cudaGetLastError();
}

cudaError_t launch_block_mass(const float* lse, const float* blk_lse, int BH, int N,
                              int block, const int32_t* row_ptr, float* mass,
                              cudaStream_t s) {
  const int nB = ceil_div(N, block);
  const int rows = BH * nB;
  if (block == 64)
    block_mass_kernel<64><<<rows, 256, 0, s>>>(lse, blk_lse, N, nB, row_ptr, mass);
  else
    block_mass_kernel<128><<<rows, 256, 0, s>>>(lse, blk_lse, N, nB, row_ptr, mass);
  return cudaGetLastError();
}

}  // namespace dsa
