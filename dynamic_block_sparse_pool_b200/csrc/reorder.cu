// Token reordering along a 3-D Hilbert curve (of the enclosing power-of-two
// cube, or generalised to the grid's own box).
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

// ------------------------------------------------ generalised Hilbert walk --
// GSRS Figure 6 walks blocks along a Gilbert curve: a Hilbert curve that
// fills a box of any size, so consecutive tokens stay grid neighbours even
// when the grid is not a power-of-two cube.  The construction here is
// Hilbert's recursion on the box itself.  A "walk" of an a x b x c box
// starts at a corner and ends at the corner a - 1 cells away along its
// first edge (the travel edge), visiting every cell with unit steps.  By a
// two-colouring of the cells it exists iff the box is a single cell or
// a >= 2 and not (a odd and b*c even).  A box is split near the middle of
// its longest edge (ties: travel edge first, then the second, then the
// third), taking the first split point, nearest the middle, whose parts all
// have walks:
//   - along the travel edge: two boxes walked one after the other;
//   - a U-turn along another edge X: the part u < h, x < m walked along +X,
//     the part x >= m walked along the travel edge, the part u >= h, x < m
//     walked back along -X; when the travel edge is 2 long, the two
//     one-cell slabs u = 0 and u = 1 walked along +X and back along -X.
namespace {

struct Edge {
  int axis, dir, len;  // axis 0 = t, 1 = y, 2 = x; dir +-1; len cells
};

bool walkable(long a, long b, long c) {
  if (a * b * c == 1) return true;
  return a >= 2 && !((a & 1) && ((b * c) & 1) == 0);
}

// The integers of [lo, hi], nearest to n first (the smaller on a tie).
void nearest_first(int n, int lo, int hi, std::vector<int>& out) {
  out.clear();
  if (n >= lo && n <= hi) out.push_back(n);
  for (int d = 1; d <= hi - lo + 1; ++d) {
    if (n - d >= lo && n - d <= hi) out.push_back(n - d);
    if (n + d >= lo && n + d <= hi) out.push_back(n + d);
  }
}

struct Cell {
  int c[3];
  Cell step(const Edge& e, int d) const {
    Cell r = *this;
    r.c[e.axis] += e.dir * d;
    return r;
  }
};

class GeneralisedHilbert {
 public:
  explicit GeneralisedHilbert(std::vector<Cell>* out) : out_(out) {}

  bool walk(const Cell& entry, const Edge& U, const Edge& V, const Edge& W) {
    const int a = U.len, b = V.len, c = W.len;
    if (b == 1 && c == 1) {
      for (int i = 0; i < a; ++i) out_->push_back(entry.step(U, i));
      return true;
    }
    // edges by length, longest first (ties keep the order U, V, W)
    const Edge* by_len[3] = {&U, &V, &W};
    std::stable_sort(by_len, by_len + 3, [](const Edge* p, const Edge* q) { return p->len > q->len; });
    std::vector<int> split_u, split_x;
    for (const Edge* e : by_len) {
      if (e == &U) {
        nearest_first(a / 2, 1, a - 1, split_u);
        for (int a1 : split_u)
          if (walkable(a1, b, c) && walkable(a - a1, b, c)) {
            const Edge u1{U.axis, U.dir, a1}, u2{U.axis, U.dir, a - a1};
            return walk(entry, u1, V, W) && walk(entry.step(U, a1), u2, V, W);
          }
        continue;
      }
      const Edge& X = *e;
      const Edge& Y = (e == &V) ? W : V;
      const int x = X.len;
      if (a < 2 || x < 2) continue;
      if (a == 2 && walkable(x, 1, Y.len)) {
        const Edge slab{U.axis, U.dir, 1}, back{X.axis, -X.dir, x};
        return walk(entry, X, slab, Y) && walk(entry.step(U, 1).step(X, x - 1), back, slab, Y);
      }
      nearest_first(x / 2, 1, x - 1, split_x);
      nearest_first(a / 2, 1, a - 1, split_u);
      for (int m : split_x)
        for (int h : split_u) {
          if (!(walkable(m, h, Y.len) && walkable(a, x - m, Y.len) && walkable(m, a - h, Y.len)))
            continue;
          const Edge up{X.axis, X.dir, m}, near_u{U.axis, U.dir, h};
          const Edge far_x{X.axis, X.dir, x - m};
          const Edge down{X.axis, -X.dir, m}, far_u{U.axis, -U.dir, a - h};
          return walk(entry, up, near_u, Y) && walk(entry.step(X, m), U, far_x, Y) &&
                 walk(entry.step(U, a - 1).step(X, m - 1), down, far_u, Y);
        }
    }
    return false;  // no split works (not reached for walkable boxes)
  }

 private:
  std::vector<Cell>* out_;
};

}  // namespace

bool generalised_hilbert_cells(int T, int H, int W, std::vector<int32_t>& grid_order) {
  const int dims[3] = {T, H, W};
  int order[3] = {0, 1, 2};
  std::stable_sort(order, order + 3, [&](int i, int j) { return dims[i] > dims[j]; });
  int axis = -1, r0 = -1, r1 = -1;
  for (int k = 0; k < 3 && axis < 0; ++k) {
    const int ax = order[k];
    const int o0 = ax == 0 ? 1 : 0, o1 = ax == 2 ? 1 : 2;
    if (walkable(dims[ax], dims[o0], dims[o1])) {
      axis = ax;
      r0 = o0;
      r1 = o1;
    }
  }
  if (axis < 0) return false;
  std::vector<Cell> cells;
  cells.reserve((size_t)T * H * W);
  GeneralisedHilbert g(&cells);
  if (!g.walk(Cell{{0, 0, 0}}, Edge{axis, 1, dims[axis]}, Edge{r0, 1, dims[r0]},
              Edge{r1, 1, dims[r1]}))
    return false;
  grid_order.resize(cells.size());
  for (size_t i = 0; i < cells.size(); ++i)
    grid_order[i] = (int32_t)(((long long)cells[i].c[0] * H + cells[i].c[1]) * W + cells[i].c[2]);
  return true;
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
