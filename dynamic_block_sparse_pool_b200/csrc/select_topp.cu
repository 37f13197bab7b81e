// Per-row Top-p block selection -> CSR block-index lists.
//
// GSRS (arXiv 2610.21129), abstract: Top-p selection for adaptive sparsity;
// Figure 4: progressively tighter Top-p keeps fewer blocks, and reduced
// search evaluates only blocks of an earlier candidate mask.
//
// Selection rule: order the row's candidate blocks by (probability desc,
// block index asc) and keep the shortest prefix whose mass reaches p.  The
// running mass is kept as an exact integer: an fp32 value in [0, 1] is
// mant * 2^(e-150) with a 24-bit mant, i.e. an integer multiple of 2^-149
// below 2^150, so sums of up to 1024 of them fit in 192 bits and every
// summation order gives the same cut.
//
// Kernel 1 (select): one warp per row.  Keys (prob bits, inverted index) for
//   up to 32 * R blocks sit in registers (R per lane) and are sorted by a
//   bitonic network (in-register and shuffle compare-exchange); a warp scan
//   of 192-bit lane sums finds the cut; the kept set becomes a 1024-bit mask
//   plus a count.
// Kernel 2 (scan): exclusive scan of the counts into row_ptr (one CTA).
// Kernel 3 (compact): one warp per row writes the kept indices ascending.
#include <cstring>

#include "common.cuh"

namespace dsa {
namespace {

struct U192 {
  uint64_t w0, w1, w2;  // w0 least significant
};

__device__ __forceinline__ void add192(U192& a, const U192& b) {
  const uint64_t s0 = a.w0 + b.w0;
  const uint64_t c0 = s0 < a.w0;
  const uint64_t t1 = a.w1 + b.w1;
  uint64_t c1 = t1 < a.w1;
  const uint64_t s1 = t1 + c0;
  c1 += s1 < t1;
  a.w2 = a.w2 + b.w2 + c1;
  a.w1 = s1;
  a.w0 = s0;
}

__device__ __forceinline__ bool ge192(const U192& a, const U192& b) {
  if (a.w2 != b.w2) return a.w2 > b.w2;
  if (a.w1 != b.w1) return a.w1 > b.w1;
  return a.w0 >= b.w0;
}

// The fp32 value with bit pattern `bits` (sign clear, <= 1.0f) times 2^149.
__host__ __device__ __forceinline__ U192 fixed_of_bits(uint32_t bits) {
  const uint32_t E = bits >> 23, M = bits & 0x7FFFFFu;
  const uint64_t mant = E ? (uint64_t)(M | 0x800000u) : (uint64_t)M;
  const int sh = E ? (int)E - 1 : 0;
  const int limb = sh >> 6, off = sh & 63;
  const uint64_t lo = mant << off;
  const uint64_t hi = off ? (mant >> (64 - off)) : 0ull;
  U192 r{0ull, 0ull, 0ull};
  if (limb == 0) {
    r.w0 = lo;
    r.w1 = hi;
  } else if (limb == 1) {
    r.w1 = lo;
    r.w2 = hi;
  } else {
    r.w2 = lo;
  }
  return r;
}

constexpr unsigned FULL = 0xffffffffu;

// Compare-exchange of the in-register pairs (r, r | J) of a bitonic stage;
// positions are lane * R + r, and block size k decides the direction.
template <int J, int R>
__device__ __forceinline__ void bitonic_in_lane(uint64_t (&key)[R], int lane, int k) {
  if constexpr (J < R) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if ((r & J) == 0) {
        const int pr = r | J;
        const bool desc = ((lane * R + r) & k) == 0;
        const uint64_t a = key[r], b = key[pr];
        const bool sw = desc ? (a < b) : (a > b);
        key[r] = sw ? b : a;
        key[pr] = sw ? a : b;
      }
    }
  }
}

// Bitonic sort of 32 * R keys held R per lane, descending; afterwards lane L
// holds sorted positions L*R .. L*R + R - 1.  The (k, j) stages are runtime
// loops so the code stays small (a fully unrolled 1024-key network does not
// fit the instruction cache); register indices stay compile-time constants.
template <int R>
__device__ __forceinline__ void bitonic_sort_desc(uint64_t (&key)[R], int lane) {
#pragma unroll 1
  for (int k = 2; k <= 32 * R; k <<= 1) {
#pragma unroll 1
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= R) {
        const int lm = j / R;
        const bool lower = (lane & lm) == 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint64_t o = __shfl_xor_sync(FULL, key[r], lm);
          const bool desc = ((lane * R + r) & k) == 0;
          const bool take_max = lower == desc;
          key[r] = take_max ? (key[r] > o ? key[r] : o) : (key[r] < o ? key[r] : o);
        }
      } else {
        switch (j) {
          case 16: bitonic_in_lane<16>(key, lane, k); break;
          case 8: bitonic_in_lane<8>(key, lane, k); break;
          case 4: bitonic_in_lane<4>(key, lane, k); break;
          case 2: bitonic_in_lane<2>(key, lane, k); break;
          default: bitonic_in_lane<1>(key, lane, k); break;
        }
      }
    }
  }
}

// Level of a probability for the threshold search: its exponent and the top
// three mantissa bits (values within 12.5 % share a level).  Probabilities
// are in [0, 1], so levels run from 0 to 1016.
__device__ __forceinline__ int level_of(uint32_t bits) { return (int)(bits >> 20); }
constexpr int kLevels = 1017;

__device__ __forceinline__ U192 warp_sum192(U192 v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    U192 o;
    o.w0 = __shfl_xor_sync(FULL, v.w0, off);
    o.w1 = __shfl_xor_sync(FULL, v.w1, off);
    o.w2 = __shfl_xor_sync(FULL, v.w2, off);
    add192(v, o);
  }
  return v;
}

template <int R>
__device__ __forceinline__ double level_sum_f64(const uint32_t (&bits)[R], uint32_t valid, int lv) {
  double s = 0.0;
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (((valid >> r) & 1u) && level_of(bits[r]) >= lv) s += (double)__uint_as_float(bits[r]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
  return s;
}

// Sorts the n boundary keys of a warp (in shared memory) descending and
// returns how many of them, taken in order, first bring the running exact
// sum `base` to `target` (n if none does).  R = keys per lane.
template <int R>
__device__ __noinline__ int boundary_cut(uint64_t* keys, int n, U192 base, const U192 target,
                                         int lane) {
  uint64_t key[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int i = lane * R + r;
    key[r] = i < n ? keys[i] : 0ull;
  }
  bitonic_sort_desc<R>(key, lane);
  U192 own{0ull, 0ull, 0ull};
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (key[r]) add192(own, fixed_of_bits((uint32_t)(key[r] >> 32) - 1u));
  U192 incl = own;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    U192 o;
    o.w0 = __shfl_up_sync(FULL, incl.w0, off);
    o.w1 = __shfl_up_sync(FULL, incl.w1, off);
    o.w2 = __shfl_up_sync(FULL, incl.w2, off);
    if (lane >= off) add192(incl, o);
  }
  U192 excl;
  excl.w0 = __shfl_up_sync(FULL, incl.w0, 1);
  excl.w1 = __shfl_up_sync(FULL, incl.w1, 1);
  excl.w2 = __shfl_up_sync(FULL, incl.w2, 1);
  if (lane == 0) excl = U192{0ull, 0ull, 0ull};
  U192 ti = incl;
  add192(ti, base);
  const unsigned ball = __ballot_sync(FULL, ge192(ti, target));
  int cut = n;
  if (ball) {
    const int L = __ffs(ball) - 1;
    int kk = 0;
    if (lane == L) {
      U192 acc = excl;
      add192(acc, base);
      bool done = false;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (!done && key[r]) {
          add192(acc, fixed_of_bits((uint32_t)(key[r] >> 32) - 1u));
          if (ge192(acc, target)) {
            kk = L * R + r + 1;
            done = true;
          }
        }
      }
    }
    cut = __shfl_sync(FULL, kk, L);
  }
  // write the sorted order back so the caller can mark the first `cut`
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int i = lane * R + r;
    if (i < n) keys[i] = key[r];
  }
  __syncwarp();
  return cut;
}

// One warp per row: values of up to 32 * R candidate blocks, R per lane
// (element e = r * 32 + lane).
//   1. A binary search over levels, with fp64 sums (exact to ~1e-13), finds
//      the level t where the mass of everything at or above t first reaches p.
//   2. An exact 192-bit pass verifies mass(level > t) < p <= mass(level >= t)
//      and moves t by one level if rounding misled the search.
//   3. Everything above level t is kept.  The few blocks on level t are
//      sorted by (probability desc, index asc) and kept until the exact sum
//      reaches p.
template <int R>
__global__ void __launch_bounds__(128)
select_kernel(const float* __restrict__ probs, int rows, int nB, int p_one,
              uint64_t t0, uint64_t t1, uint64_t t2,
              const int32_t* __restrict__ cand_row_ptr, const int32_t* __restrict__ cand_col,
              uint32_t* __restrict__ bitmaps, int32_t* __restrict__ counts, unsigned* err) {
  __shared__ uint32_t cbits_all[4][32];
  __shared__ uint32_t sel_all[4][32];
  __shared__ uint64_t bkeys_all[4][32 * R];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= rows) return;  // whole warp leaves together
  uint32_t* cbits = cbits_all[warp];
  uint32_t* sel = sel_all[warp];
  uint64_t* bkeys = bkeys_all[warp];
  const bool reduced = cand_row_ptr != nullptr;
  const U192 target{t0, t1, t2};

  sel[lane] = 0u;
  if (reduced) {
    cbits[lane] = 0u;
    __syncwarp();
    const int cs = cand_row_ptr[row], ce = cand_row_ptr[row + 1];
    if (cs < 0 || ce < cs) {
      if (lane == 0) flag_error(err, kErrRowPtr);
    } else {
      for (int e = cs + lane; e < ce; e += 32) {
        const int j = cand_col[e];
        if (j < 0 || j >= nB) {
          flag_error(err, kErrCsrIndex);
          continue;
        }
        atomicOr(&cbits[j >> 5], 1u << (j & 31));
      }
    }
  }
  __syncwarp();

  const float* prow = probs + (size_t)row * nB;
  uint32_t bits[R];
  uint32_t valid = 0u;  // bit r: element r * 32 + lane is a candidate
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = r * 32 + lane;
    bits[r] = 0u;
    if (e < nB && (!reduced || ((cbits[e >> 5] >> (e & 31)) & 1u))) {
      float f = prow[e];
      if (!(f >= 0.f && f <= 1.f)) {
        flag_error(err, kErrProb);
        f = 0.f;
      }
      bits[r] = __float_as_uint(f) & 0x7FFFFFFFu;
      valid |= 1u << r;
    }
  }

  int kstar_extra = 0;  // boundary blocks kept (only when cut inside a level)
  int t_level = -1;     // keep everything with level > t_level (-1: keep all)
  int n_bnd = 0;
  if (!p_one) {
    // 1. threshold level from fp64 sums: largest t with mass(level >= t) >= p
    const double tgt = ldexp((double)t0, -149) + ldexp((double)t1, -85) + ldexp((double)t2, -21);
    int lo = -1, hi = kLevels;  // invariant: mass(>= lo) >= p (lo = -1: all), mass(>= hi) < p
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (level_sum_f64<R>(bits, valid, mid) >= tgt) lo = mid;
      else hi = mid;
    }
    // 2. exact check of mass(level > t) < p <= mass(level >= t); fix by a level
    int t = lo;
    // each correction moves t one level towards the exact answer, so the loop
    // ends; fp64 sums of at most 1024 non-negative terms are off by ~1e-13,
    // which moves t by at most one level in practice
    for (int guard = 0; guard <= kLevels + 1; ++guard) {
      U192 above{0ull, 0ull, 0ull}, at_or_above{0ull, 0ull, 0ull};
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if ((valid >> r) & 1u) {
          const int lv = level_of(bits[r]);
          if (lv >= t) {
            const U192 x = fixed_of_bits(bits[r]);
            add192(at_or_above, x);
            if (lv > t) add192(above, x);
          }
        }
      }
      above = warp_sum192(above);
      at_or_above = warp_sum192(at_or_above);
      if (t >= 0 && !ge192(at_or_above, target)) {
        --t;  // the fp64 search stopped one level too high
        continue;
      }
      if (ge192(above, target)) {
        ++t;  // one level too low
        continue;
      }
      // 3. blocks on level t, compacted in index order, then sorted and cut
      if (t >= 0) {
        int mine = 0;
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (((valid >> r) & 1u) && level_of(bits[r]) == t) ++mine;
        int incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int o = __shfl_up_sync(FULL, incl, off);
          if (lane >= off) incl += o;
        }
        n_bnd = __shfl_sync(FULL, incl, 31);
        int pos = incl - mine;
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (((valid >> r) & 1u) && level_of(bits[r]) == t)
            bkeys[pos++] = ((uint64_t)(bits[r] + 1u) << 32) |
                           (uint64_t)(0xFFFFFFFFu - (uint32_t)(r * 32 + lane));
        __syncwarp();
        const int rb = (n_bnd + 31) / 32;
        if (rb <= 1) kstar_extra = boundary_cut<1>(bkeys, n_bnd, above, target, lane);
        else if (rb <= 2) kstar_extra = boundary_cut<2 <= R ? 2 : R>(bkeys, n_bnd, above, target, lane);
        else if (rb <= 4) kstar_extra = boundary_cut<4 <= R ? 4 : R>(bkeys, n_bnd, above, target, lane);
        else if (rb <= 8) kstar_extra = boundary_cut<8 <= R ? 8 : R>(bkeys, n_bnd, above, target, lane);
        else if (rb <= 16) kstar_extra = boundary_cut<16 <= R ? 16 : R>(bkeys, n_bnd, above, target, lane);
        else kstar_extra = boundary_cut<R>(bkeys, n_bnd, above, target, lane);
      }
      t_level = t;
      break;
    }
  }

  // keep: level > t_level, plus the first kstar_extra sorted boundary blocks
  int kept = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (((valid >> r) & 1u) && level_of(bits[r]) > t_level) {
      const int e = r * 32 + lane;
      atomicOr(&sel[e >> 5], 1u << (e & 31));
      ++kept;
    }
  }
  for (int i = lane; i < kstar_extra; i += 32) {
    const uint32_t e = 0xFFFFFFFFu - (uint32_t)bkeys[i];
    atomicOr(&sel[e >> 5], 1u << (e & 31));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(FULL, kept, o);
  __syncwarp();
  bitmaps[(size_t)row * 32 + lane] = sel[lane];
  if (lane == 0) counts[row] = kept + kstar_extra;
}

__global__ void __launch_bounds__(1024)
csr_scan_kernel(const int32_t* __restrict__ counts, int rows, int32_t* __restrict__ row_ptr) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    carry = 0;
    row_ptr[0] = 0;
  }
  __syncthreads();
  constexpr int PER = 4;
  for (int base = 0; base < rows; base += 1024 * PER) {
    int v[PER];
    int tsum = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int idx = base + tid * PER + u;
      v[u] = idx < rows ? counts[idx] : 0;
      tsum += v[u];
    }
    int incl = tsum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(FULL, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
      int wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(FULL, wi, off);
        if (lane >= off) wi += o;
      }
      warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int run = carry + warp_tot[warp] + incl - tsum;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int idx = base + tid * PER + u;
      run += v[u];
      if (idx < rows) row_ptr[idx + 1] = run;
    }
    __syncthreads();
    if (tid == 1023) carry = run;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256)
compact_kernel(const uint32_t* __restrict__ bitmaps, int rows,
               const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  uint32_t word = bitmaps[(size_t)row * 32 + lane];
  const int c = __popc(word);
  int incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(FULL, incl, off);
    if (lane >= off) incl += o;
  }
  int pos = row_ptr[row] + incl - c;
  while (word) {
    const int b = __ffs(word) - 1;
    col_idx[pos++] = lane * 32 + b;
    word &= word - 1u;
  }
}

}  // namespace

cudaError_t launch_select(const float* probs, int rows, int nB, float p,
                          const int32_t* cand_row_ptr, const int32_t* cand_col,
                          int32_t* row_ptr, int32_t* col_idx, uint32_t* bitmaps,
                          int32_t* counts, unsigned* err, cudaStream_t s) {
  uint32_t pbits;
  memcpy(&pbits, &p, sizeof(pbits));
  const int p_one = p >= 1.0f ? 1 : 0;
  const U192 t = fixed_of_bits(p_one ? 0x3F800000u : pbits);
  const int grid = ceil_div(rows, 8);
  const int R = nB <= 32 ? 1 : nB <= 64 ? 2 : nB <= 128 ? 4 : nB <= 256 ? 8 : nB <= 512 ? 16 : 32;
  switch (R) {
#define DSA_SEL(RR)                                                                            \
  case RR:                                                                                     \
    select_kernel<RR><<<ceil_div(rows, 4), 128, 0, s>>>(probs, rows, nB, p_one, t.w0, t.w1,   \
                                                        t.w2, cand_row_ptr, cand_col, bitmaps, \
                                                        counts, err);                          \
    break;
    DSA_SEL(1) DSA_SEL(2) DSA_SEL(4) DSA_SEL(8) DSA_SEL(16) DSA_SEL(32)
#undef DSA_SEL
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  csr_scan_kernel<<<1, 1024, 0, s>>>(counts, rows, row_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  compact_kernel<<<grid, 256, 0, s>>>(bitmaps, rows, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace dsa
