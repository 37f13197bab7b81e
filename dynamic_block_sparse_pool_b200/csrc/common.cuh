// Shared definitions for the libdsa kernels (device side and launchers).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace dsa {

// Bits of the device-side error word (see dsa_device_status).
enum : unsigned {
  kErrCsrIndex = 1u,     // a CSR column index outside [0, nB)
  kErrRowPtr = 2u,       // a row_ptr entry that is negative or decreasing
  kErrProb = 4u,         // a probability outside [0, 1] or NaN
  kErrTimeout = 8u,      // a bounded wait on an mbarrier ran out
  kErrAlign = 16u,       // dynamic shared memory not 1024-byte aligned
  kErrPerm = 32u,        // a token permutation entry outside [0, N)
  kErrRowOrder = 64u,    // an attention row-order entry outside [0, rows)
};

// Upper bound for one mbarrier wait before a kernel gives up (nanoseconds).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ void flag_error(unsigned* err, unsigned bits) {
  if (err) atomicOr(err, bits);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Launchers (one per kernel family); all return the launch error.
cudaError_t launch_pool_means(const void* q, const void* k, bool bf16, int BH, int N,
                              int D, int block, float* qbar, float* kbar,
                              cudaStream_t s);
cudaError_t launch_block_scores(const float* qbar, const float* kbar, int BH, int nB,
                                int D, float scale, const int32_t* cand_row_ptr,
                                const int32_t* cand_col, float* probs, unsigned* err,
                                cudaStream_t s);
cudaError_t launch_select(const float* probs, int rows, int nB, float p,
                          const int32_t* cand_row_ptr, const int32_t* cand_col,
                          int32_t* row_ptr, int32_t* col_idx, uint32_t* bitmaps,
                          int32_t* counts, unsigned* err, cudaStream_t s);
cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, bool bf16,
                             int BH, int N, int D, int block, float scale,
                             const int32_t* row_ptr, const int32_t* col_idx, void* out,
                             float* lse, float* blk_lse, unsigned* err, cudaStream_t s);
// Each head's rows of a CSR mask by descending block count (ties by row
// index), as global row indices: order[bh*nB .. (bh+1)*nB) holds head bh's.
cudaError_t launch_row_order(const int32_t* row_ptr, int BH, int nB, int num_sms, int32_t* order,
                             cudaStream_t s);
// tickets: two zeroed words of device memory that no concurrent launch uses
// (the kernel leaves them zeroed); num_sms: the device's SM count; row_order:
// the order in which the CTAs take the rows (NULL: index order).
cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, int BH,
                              int N, int D, float scale, const int32_t* row_ptr,
                              const int32_t* col_idx, const int32_t* row_order, void* out, float* lse,
                              float* blk_lse, unsigned* tickets, int num_sms,
                              unsigned* err, cudaStream_t s, const char** why);
cudaError_t launch_mass_to_probs(const int32_t* row_ptr, const int32_t* col_idx,
                                 const float* mass, int rows, int nB, float* probs,
                                 unsigned* err, cudaStream_t s);
// Index of grid cell (t, y, x) along the 3-D Hilbert curve of side 2^bits (host).
uint64_t hilbert_key3(uint32_t t, uint32_t y, uint32_t x, int bits);
cudaError_t launch_permute_tokens(const void* src, void* dst, int elem_bytes, int BH, int N,
                                  int D, const int32_t* perm, bool inverse, unsigned* err,
                                  cudaStream_t s);
cudaError_t launch_aggregate_probs(const float* pf, int BH, int N, int block, int sub, int nB,
                                   int nBf, float* probs, cudaStream_t s);
// Exclusive scan of `rows` counts into row_ptr[0 .. rows] (one CTA).
cudaError_t launch_csr_scan(const int32_t* counts, int rows, int32_t* row_ptr, cudaStream_t s);
cudaError_t launch_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, bool bf16, int BH, int N, int D,
                            int block, float scale, const int32_t* row_ptr,
                            const int32_t* col_idx, void* dq, void* dk, void* dv,
                            uint32_t* bitmap, int32_t* counts, int32_t* t_row_ptr,
                            int32_t* t_col, float* delta, unsigned* err, cudaStream_t s);
// dQ, dK, dV on tcgen05 (bf16, blocks of 128): after the mask transpose and
// the row term delta of launch_attn_bwd.
cudaError_t launch_attn_bwd_sm100(const void* q, const void* k, const void* v, const void* dout,
                                  const float* lse, const float* delta, int BH, int N, int D,
                                  float scale, const int32_t* row_ptr, const int32_t* col_idx,
                                  const int32_t* t_row_ptr, const int32_t* t_col, void* dq, void* dk,
                                  void* dv, unsigned* err, cudaStream_t s);
// One CTA that waits on an mbarrier nobody arrives at, with the given limit.
cudaError_t launch_wait_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t s);
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s);
cudaError_t launch_block_mass(const float* lse, const float* blk_lse, int BH, int N,
                              int block, const int32_t* row_ptr, float* mass,
                              cudaStream_t s);

}  // namespace dsa
