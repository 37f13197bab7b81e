// dsa_select_topp_static: Top-p block selection that needs no scratch
// memory from the caller and allocates none.
//
// Some callers cannot allocate device memory when they call in: a host that
// hands a plugin only its input and output buffers and offers no workspace
// hook, a service that keeps every byte of device memory inside its own
// pre-sized pool, or a latency-critical loop where cudaMalloc / cudaFree
// (which may synchronise the device) are not allowed.  This entry point
// serves them: its scratch (per-row selection bitmaps and counts) lives in
// the file-scope array below, which every GPU that loads the library keeps
// for the life of the process (DSA_STATIC_MAX_ROWS * 33 words, 4.3 MB).
//
// The selection itself is dsa_select_topp's: same kernels, same results.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "dsa.h"

namespace dsa {
dsa_status api_checked_device(unsigned** err_word);
void api_set_last_error(const char* msg);
}  // namespace dsa

namespace {

constexpr size_t kScratchWords = (size_t)DSA_STATIC_MAX_ROWS * 33;

// Scratch shared by every call on a device: rows*32 bitmap words, then rows
// counts.  Each call writes every word it later reads, so nothing has to be
// cleared between calls.
static __device__ __align__(256) uint32_t g_select_scratch[kScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
uint32_t* g_scratch_ptr[kMaxDevices] = {};

dsa_status fail(dsa_status st, const char* msg) {
  dsa::api_set_last_error(msg);
  return st;
}

// Device address of the scratch array on the current device.  The first call
// on each device looks it up (the array's name in host code is only a
// host-side handle and must not be passed to a kernel).
dsa_status scratch_for_current_device(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device id out of range");
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) {
      char buf[256];
      snprintf(buf, sizeof(buf), "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      return fail(DSA_ERR_CUDA, buf);
    }
    g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_select_topp_static(const float* probs, int rows, int nB, float p,
                                             const int32_t* cand_row_ptr,
                                             const int32_t* cand_col, int32_t* row_ptr,
                                             int32_t* col_idx, void* stream) {
  dsa::api_set_last_error("");
  if (!probs || !row_ptr || !col_idx) return fail(DSA_ERR_INVALID_ARG, "null probs, row_ptr or col_idx");
  if (rows < 1) return fail(DSA_ERR_INVALID_ARG, "rows must be >= 1");
  if (rows > DSA_STATIC_MAX_ROWS) {
    char buf[160];
    snprintf(buf, sizeof(buf),
             "rows = %d exceeds DSA_STATIC_MAX_ROWS = %d of the built-in scratch; "
             "use dsa_select_topp with a workspace", rows, DSA_STATIC_MAX_ROWS);
    return fail(DSA_ERR_INVALID_ARG, buf);
  }
  if (nB < 1 || nB > DSA_MAX_BLOCKS) return fail(DSA_ERR_INVALID_ARG, "nB outside 1..DSA_MAX_BLOCKS");
  if (!(p > 0.f && p <= 1.f)) return fail(DSA_ERR_INVALID_ARG, "p must be in (0, 1]");
  if ((cand_row_ptr == nullptr) != (cand_col == nullptr))
    return fail(DSA_ERR_INVALID_ARG, "cand_row_ptr and cand_col must both be set or both be NULL");
  if ((reinterpret_cast<uintptr_t>(probs) | reinterpret_cast<uintptr_t>(row_ptr) |
       reinterpret_cast<uintptr_t>(col_idx)) % 4 != 0)
    return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  unsigned* err_word = nullptr;
  dsa_status st = dsa::api_checked_device(&err_word);
  if (st != DSA_OK) return st;
  uint32_t* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != DSA_OK) return st;
  uint32_t* bitmaps = scratch;
  int32_t* counts = reinterpret_cast<int32_t*>(scratch + (size_t)rows * 32);
  const cudaError_t e = dsa::launch_select(probs, rows, nB, p, cand_row_ptr, cand_col, row_ptr,
                                           col_idx, bitmaps, counts, err_word,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, cudaGetErrorString(e));
  return DSA_OK;
}
