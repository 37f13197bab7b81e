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
// Kernel 1 (select): one warp per row, no sort.  The kept set is every block
//   above a threshold value tau plus, at tau itself, the first few ties in
//   index order; tau comes from a bisection over the fp32 bit patterns with
//   fp32 sums, accepted when an fp64 check with its error bound decides the
//   cut and otherwise settled with exact 192-bit sums.  The kept set becomes a
//   1024-bit mask (one ballot per register) plus a count.
// Kernel 2 (scan): exclusive scan of the counts into row_ptr (one CTA).
// Kernel 3 (compact): one warp per row writes the kept indices ascending.
// Kernel 4 (row order, its own call): each head's rows by descending block
//   count, the order in which the persistent attention kernel takes them.
#include <cstring>

#include "common.cuh"
#include "dsa.h"

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

// a * m for a small multiplier m (the result stays below 2^192 for the
// values used here: a <= 2^149, m <= 1024).
__device__ __forceinline__ U192 mul192(const U192& a, uint32_t m) {
  const uint64_t p0 = a.w0 * m, c0 = __umul64hi(a.w0, m);
  const uint64_t p1 = a.w1 * m, c1 = __umul64hi(a.w1, m);
  U192 r;
  r.w0 = p0;
  r.w1 = p1 + c0;
  r.w2 = a.w2 * m + c1 + (r.w1 < p1);
  return r;
}

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

// Butterfly sum: every lane ends with the same value (fp addition is
// commutative), so decisions taken on it are warp-uniform.
__device__ __forceinline__ double warp_sum_f64(double s) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
  return s;
}

// Candidate c * 32 + lane of a row, read from memory: its key (bit pattern
// of the probability, sanitised like the main load) or false if it is not a
// candidate.
__device__ __forceinline__ bool load_key(const float* __restrict__ prow, const uint32_t* cbits,
                                         int nB, int c, int lane, uint32_t& key) {
  const int e = c * 32 + lane;
  if (e >= nB || (cbits != nullptr && !((cbits[c] >> lane) & 1u))) return false;
  const float f = prow[e];
  key = (f >= 0.f && f <= 1.f) ? (__float_as_uint(f) & 0x7FFFFFFFu) : 0u;
  return true;
}

// Exact selection of one row with 192-bit sums, re-reading the row from
// memory (used only when the fp64 search cannot decide: a prefix mass within
// the fp64 error of p, or several blocks tied at the threshold).
//   tau: starting guess for the threshold key (-1: keep everything).  Each
//   correction moves it to the neighbouring key present in the row, so the
//   loop ends.  Then: keys > tau are kept, and the tie of rank k (0-based,
//   index order) at tau is kept iff mass(key > tau) + k * tau < p.
// Returns the number kept; lane L receives word L of the row bitmap.
__device__ __noinline__ int select_row_exact(const float* __restrict__ prow, const uint32_t* cbits,
                                             int nB, U192 target, int tau, int lane,
                                             uint32_t& myword) {
  const int nC = (nB + 31) >> 5;
  U192 above{0ull, 0ull, 0ull};
  for (int guard = 0; guard <= 32 * nC + 1; ++guard) {
    U192 a{0ull, 0ull, 0ull};
    int ties = 0;
    for (int c = 0; c < nC; ++c) {
      uint32_t k;
      if (load_key(prow, cbits, nB, c, lane, k)) {
        if ((int)k > tau) add192(a, fixed_of_bits(k));
        else if ((int)k == tau) ++ties;
      }
    }
    above = warp_sum192(a);
    if (ge192(above, target)) {  // tau too low: next larger key present
      uint32_t nxt = 0xFFFFFFFFu;
      for (int c = 0; c < nC; ++c) {
        uint32_t k;
        if (load_key(prow, cbits, nB, c, lane, k) && (int)k > tau) nxt = min(nxt, k);
      }
      tau = (int)__reduce_min_sync(FULL, nxt);
      continue;
    }
    if (tau >= 0) {
      ties = (int)__reduce_add_sync(FULL, (unsigned)ties);
      U192 all = mul192(fixed_of_bits((uint32_t)tau), (uint32_t)ties);
      add192(all, above);
      if (!ge192(all, target)) {  // tau too high: next smaller key, or keep all
        int prv = -1;
        for (int c = 0; c < nC; ++c) {
          uint32_t k;
          if (load_key(prow, cbits, nB, c, lane, k) && (int)k < tau) prv = max(prv, (int)k);
        }
        tau = __reduce_max_sync(FULL, prv);
        continue;
      }
    }
    break;
  }
  const U192 unit = tau >= 0 ? fixed_of_bits((uint32_t)tau) : U192{0ull, 0ull, 0ull};
  int kept = 0, run = 0;
  myword = 0u;
  for (int c = 0; c < nC; ++c) {
    uint32_t k = 0u;
    const bool v = load_key(prow, cbits, nB, c, lane, k);
    const bool tie = v && tau >= 0 && (int)k == tau;
    const unsigned tb = __ballot_sync(FULL, tie);
    bool keep = v && (tau < 0 || (int)k > tau);
    if (tie) {
      U192 pre = mul192(unit, (uint32_t)(run + __popc(tb & ((1u << lane) - 1u))));
      add192(pre, above);
      keep = !ge192(pre, target);
    }
    run += __popc(tb);
    const unsigned w = __ballot_sync(FULL, keep);
    kept += __popc(w);
    if (lane == c) myword = w;
  }
  return kept;
}

__device__ __forceinline__ float warp_sum_f32(float s) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
  return s;
}

// One warp per row; element e = r * 32 + lane is held by lane `lane` in
// register r (R = ceil(nB / 32) registers).
//
// With the blocks ordered by (probability desc, index asc), the kept prefix
// is {prob > tau} followed by the first m blocks (in index order) whose
// probability equals tau, where tau is the largest probability with
// mass(prob >= tau) >= p.  Non-negative fp32 values order like their bit
// patterns (keys), so comparisons run on the integer keys.
//   1. Bisection over keys with fp32 sums.  Each pass sums the blocks at or
//      above the midpoint and also finds the smallest of them and the
//      largest block below it, so the lower end always sits on a present
//      value and the search stops once no present value lies strictly
//      between the two ends (about 10 passes on attention-map rows, against
//      ~27 for a plain bisection of the key range).
//   2. One fp64 pass: mass(>= tau), mass(> tau), the number of blocks at
//      tau and the row total T.  Sums of at most n terms in [0, 1] are
//      within n * 2^-53 * T of exact; when mass(>= tau) - p and
//      p - mass(> tau) both exceed twice that and tau is held by one block,
//      the cut is decided: keep prob >= tau.  Otherwise (an fp32 search that
//      went astray, a prefix mass within rounding of p, or ties at tau) the
//      row is decided exactly with 192-bit sums.
// If the whole row's mass is below p, every candidate is kept.
template <int R>
__global__ void __launch_bounds__(128, 8)
select_kernel(const float* __restrict__ probs, int rows, int nB, float p,
              uint64_t t0, uint64_t t1, uint64_t t2,
              const int32_t* __restrict__ cand_row_ptr, const int32_t* __restrict__ cand_col,
              uint32_t* __restrict__ bitmaps, int32_t* __restrict__ counts, unsigned* err) {
  __shared__ uint32_t cbits_all[4][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= rows) return;  // whole warp leaves together
  uint32_t* cbits = cbits_all[warp];
  const bool reduced = cand_row_ptr != nullptr;

  if (reduced) {
    cbits[lane] = 0u;
    __syncwarp();
    const int cs = cand_row_ptr[row], ce = cand_row_ptr[row + 1];
    if (cs < 0 || ce < cs) {
      if (lane == 0) flag_error(err, kErrRowPtr);
    } else {
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
          atomicOr(&cbits[j >> 5], 1u << (j & 31));
        }
      }
    }
    __syncwarp();
  }

  const float* prow = probs + (size_t)row * nB;
  uint32_t kv[R];       // keys of the candidates (0 for non-candidates)
  uint32_t valid = 0u;  // bit r: element r * 32 + lane is a candidate
#pragma unroll
  for (int r = 0; r < R; ++r) {
    kv[r] = 0u;
    const int e = r * 32 + lane;
    if (e < nB && (!reduced || ((cbits[r] >> lane) & 1u))) {
      float f = prow[e];
      if (!(f >= 0.f && f <= 1.f)) {
        flag_error(err, kErrProb);
        f = 0.f;
      }
      kv[r] = __float_as_uint(f) & 0x7FFFFFFFu;  // -0 -> +0
      valid |= 1u << r;
    }
  }

  int mode = 0;  // 0: keep every candidate, 1: keep key >= tau, 2: exact path
  int tau = -1;
  if (p < 1.f) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) s += __uint_as_float(kv[r]);
    if (warp_sum_f32(s) >= p) {
      uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if ((valid >> r) & 1u) {
          kmin = min(kmin, kv[r]);
          kmax = max(kmax, kv[r]);
        }
      }
      // invariants: lo is a present key with G(lo) >= p; G(hi) < p;
      // below_hi = the largest present key below hi
      uint32_t lo = __reduce_min_sync(FULL, kmin);
      uint32_t below_hi = __reduce_max_sync(FULL, kmax);
      uint32_t hi = below_hi + 1u;
      while (below_hi != lo) {
        const uint32_t mid = (lo + hi) >> 1;  // lo < mid < hi
        float s0 = 0.f, s1 = 0.f;
        uint32_t up = 0xFFFFFFFFu, dn = 0u;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool ge = kv[r] >= mid;
          if (r & 1) s1 += ge ? __uint_as_float(kv[r]) : 0.f;
          else s0 += ge ? __uint_as_float(kv[r]) : 0.f;
          up = min(up, ge ? kv[r] : 0xFFFFFFFFu);
          dn = max(dn, ge ? 0u : kv[r]);
        }
        const float g = warp_sum_f32(s0 + s1);
        up = __reduce_min_sync(FULL, up);
        dn = __reduce_max_sync(FULL, dn);
        if (g >= p) {
          lo = up;
        } else {
          hi = mid;
          below_hi = dn;
        }
      }
      tau = (int)lo;
    }
    // 2. fp64 check of the cut
    double g_ge = 0.0, g_gt = 0.0, tot = 0.0;
    int ties = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const double d = (double)__uint_as_float(kv[r]);
      tot += d;
      if ((int)kv[r] >= tau) g_ge += d;
      if ((int)kv[r] > tau) g_gt += d;
      ties += (((valid >> r) & 1u) && (int)kv[r] == tau) ? 1 : 0;
    }
    tot = warp_sum_f64(tot);
    g_ge = warp_sum_f64(g_ge);
    g_gt = warp_sum_f64(g_gt);
    ties = (int)__reduce_add_sync(FULL, (unsigned)ties);
    const int nv = (int)__reduce_add_sync(FULL, (unsigned)__popc(valid));
    const double pd = (double)p;
    const double eps = (double)(nv + 1) * tot * 0x1p-52;  // twice the fp64 error bound
    if (tau < 0) mode = tot + eps < pd ? 0 : 2;
    else mode = (g_ge - eps >= pd && g_gt + eps < pd && ties == 1) ? 1 : 2;
  }

  uint32_t myword = 0u;
  int kept = 0;
  if (mode == 2) {
    kept = select_row_exact(prow, reduced ? cbits : nullptr, nB, U192{t0, t1, t2}, tau, lane,
                            myword);
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const bool keep = ((valid >> r) & 1u) && (mode == 0 || (int)kv[r] >= tau);
      const unsigned w = __ballot_sync(FULL, keep);
      kept += __popc(w);
      if (lane == r) myword = w;
    }
  }
  bitmaps[(size_t)row * 32 + lane] = myword;
  if (lane == 0) counts[row] = kept;
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

// Stable rank of every row of head blockIdx.x by descending block count.
// Row j's key is (len_j << 11) | (2047 - j), len_j clamped to [0, 2^20): the
// keys of a head are distinct, and key_j > key_i exactly when row j has more
// blocks than row i, or as many and a lower index, so
//   rank(i) = #{j : key_j > key_i}
// maps the head's rows one to one onto 0 .. nB-1 whatever row_ptr holds (a
// malformed row_ptr only changes the lengths).  Every CTA of the head loads
// all nB keys into shared memory (padded with -1 to a multiple of 4; at
// least 256 threads, so the loads take a few rounds) and ranks its own
// slice of the rows, one row per thread, reading the keys four at a time
// (broadcast loads).
__global__ void __launch_bounds__(1024)
row_order_kernel(const int32_t* __restrict__ row_ptr, int nB, int per_cta,
                 int32_t* __restrict__ order) {
  __shared__ __align__(16) int key[DSA_MAX_BLOCKS];
  const int bh = blockIdx.x;
  const int32_t* rp = row_ptr + (size_t)bh * nB;
  const int nB4 = (nB + 3) & ~3;
  for (int j = threadIdx.x; j < nB4; j += blockDim.x) {
    int k = -1;
    if (j < nB) {
      long long len = (long long)rp[j + 1] - rp[j];
      len = len < 0 ? 0 : (len > (1 << 20) - 1 ? (1 << 20) - 1 : len);
      k = (int)(len << 11) | (2047 - j);
    }
    key[j] = k;
  }
  __syncthreads();
  const int i = blockIdx.y * per_cta + threadIdx.x;
  if (threadIdx.x >= per_cta || i >= nB) return;
  const int ki = key[i];
  const int4* k4 = reinterpret_cast<const int4*>(key);
  int rank = 0;
#pragma unroll 4
  for (int j = 0; j < nB4 / 4; ++j) {
    const int4 k = k4[j];
    rank += (k.x > ki) + (k.y > ki) + (k.z > ki) + (k.w > ki);
  }
  order[(size_t)bh * nB + rank] = bh * nB + i;
}

}  // namespace

cudaError_t launch_row_order(const int32_t* row_ptr, int BH, int nB, int num_sms, int32_t* order,
                             cudaStream_t s) {
  if (nB < 1 || nB > DSA_MAX_BLOCKS || BH < 1) return cudaErrorInvalidValue;
  // enough CTAs for about two per SM, at least 64 rows each
  int split = ceil_div(2 * (num_sms > 0 ? num_sms : 1), BH);
  const int most = ceil_div(nB, 64);
  split = split < 1 ? 1 : (split > most ? most : split);
  const int per = ceil_div(nB, split);
  const int threads = per > 256 ? ceil_div(per, 32) * 32 : 256;  // <= 1024
  row_order_kernel<<<dim3(BH, ceil_div(nB, per)), threads, 0, s>>>(row_ptr, nB, per, order);
  return cudaGetLastError();
}

cudaError_t launch_csr_scan(const int32_t* counts, int rows, int32_t* row_ptr, cudaStream_t s) {
  csr_scan_kernel<<<1, 1024, 0, s>>>(counts, rows, row_ptr);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* probs, int rows, int nB, float p,
                          const int32_t* cand_row_ptr, const int32_t* cand_col,
                          int32_t* row_ptr, int32_t* col_idx, uint32_t* bitmaps,
                          int32_t* counts, unsigned* err, cudaStream_t s) {
  uint32_t pbits;
  memcpy(&pbits, &p, sizeof(pbits));
  const U192 t = fixed_of_bits(p >= 1.0f ? 0x3F800000u : pbits);
  const int grid = ceil_div(rows, 8);
  const int R = ceil_div(nB, 32);  // registers per lane, 1 .. 32
  switch (R) {
#define DSA_SEL(RR)                                                                            \
  case RR:                                                                                     \
    select_kernel<RR><<<ceil_div(rows, 4), 128, 0, s>>>(probs, rows, nB, p, t.w0, t.w1, t.w2,  \
                                                        cand_row_ptr, cand_col, bitmaps,       \
                                                        counts, err);                          \
    break;
    DSA_SEL(1) DSA_SEL(2) DSA_SEL(3) DSA_SEL(4) DSA_SEL(5) DSA_SEL(6) DSA_SEL(7) DSA_SEL(8)
    DSA_SEL(9) DSA_SEL(10) DSA_SEL(11) DSA_SEL(12) DSA_SEL(13) DSA_SEL(14) DSA_SEL(15)
    DSA_SEL(16) DSA_SEL(17) DSA_SEL(18) DSA_SEL(19) DSA_SEL(20) DSA_SEL(21) DSA_SEL(22)
    DSA_SEL(23) DSA_SEL(24) DSA_SEL(25) DSA_SEL(26) DSA_SEL(27) DSA_SEL(28) DSA_SEL(29)
    DSA_SEL(30) DSA_SEL(31) DSA_SEL(32)
#undef DSA_SEL
    default:
      return cudaErrorInvalidValue;
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
