// Token reordering along a 3-D Hilbert curve.
//
// GSRS (arXiv 2610.21129), Figure 6: with curve ordering a block holds the
// tokens of a compact spatio-temporal region instead of a flat slab of the
// row-major order; Figures 1 and 3 reorder tokens along Hilbert curves.
// DFSAttn (abstract): Hilbert-curve token reordering keeps fine-grained
// sparsity while the kernels still work on contiguous blocks.
//
// Host: dsa_hilbert_order places every grid cell (t, y, x) by its index
// along the 3-D Hilbert curve of the enclosing cube of side 2^bits, computed
// with Skilling's axes-to-transpose method ("Programming the Hilbert curve",
// AIP Conf. Proc. 707, 2004); cells outside the grid are skipped and the
// text prefix keeps its leading positions.
// Device: permute_tokens copies whole token rows, dst[i] = src[perm[i]]
// (gather) or dst[perm[i]] = src[i] (scatter), in 16-byte pieces.
#include <algorithm>
#include <utility>
#include <vector>

#include "common.cuh"

namespace dsa {

// Index of (t, y, x) along the Hilbert curve of side 2^bits (t most
// significant in each 3-bit digit).
uint64_t hilbert_key3(uint32_t t, uint32_t y, uint32_t x, int bits) {
  uint32_t c[3] = {t, y, x};
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (c[i] & q) {
        c[0] ^= low;
      } else {
        const uint32_t sw = (c[0] ^ c[i]) & low;
        c[0] ^= sw;
        c[i] ^= sw;
      }
    }
  }
  c[1] ^= c[0];
  c[2] ^= c[1];
  uint32_t flip = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (c[2] & q) flip ^= q - 1;
  for (int i = 0; i < 3; ++i) c[i] ^= flip;
  uint64_t key = 0;
  for (int b = bits - 1; b >= 0; --b)
    for (int i = 0; i < 3; ++i) key = (key << 1) | ((c[i] >> b) & 1u);
  return key;
}

namespace {

template <int CHUNK>
__global__ void __launch_bounds__(256)
permute_tokens_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int N,
                      int chunks_per_row, const int32_t* __restrict__ perm, bool inverse,
                      long long total, unsigned* err) {
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long row = idx / chunks_per_row;
    const int c = (int)(idx - row * chunks_per_row);
    const long long bh = row / N;
    const int i = (int)(row - bh * N);
    const int j = perm[i];
    if (j < 0 || j >= N) {
      if (c == 0) flag_error(err, kErrPerm);
      continue;
    }
    const long long from = inverse ? row : bh * N + j;
    const long long to = inverse ? bh * N + j : row;
    dst[to * chunks_per_row + c] = src[from * chunks_per_row + c];
  }
}

}  // namespace

cudaError_t launch_permute_tokens(const void* src, void* dst, int elem_bytes, int BH, int N,
                                  int D, const int32_t* perm, bool inverse, unsigned* err,
                                  cudaStream_t s) {
  const int chunks = D * elem_bytes / 16;
  const long long total = (long long)BH * N * chunks;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (total + 255) / 256;
  const int grid = (int)std::min<long long>(want, (long long)sms * 8);
  permute_tokens_kernel<16><<<grid, 256, 0, s>>>(static_cast<const uint4*>(src),
                                                 static_cast<uint4*>(dst), N, chunks, perm,
                                                 inverse, total, err);
  return cudaGetLastError();
}

}  // namespace dsa
