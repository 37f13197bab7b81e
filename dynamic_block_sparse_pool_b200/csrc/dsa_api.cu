// C ABI of libdsa (declared in include/dsa.h): argument checks, error
// reporting and dispatch to the kernel launchers.  No call allocates device
// memory or synchronises the host, except dsa_device_status.
#include <algorithm>
#include <utility>
#include <vector>
#include <climits>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include "common.cuh"
#include "dsa.h"

namespace dsa {
// Grid cells of a T x H x W grid in generalised Hilbert walk order, as
// row-major indices (t*H + y)*W + x (reorder.cu).
bool generalised_hilbert_cells(int T, int H, int W, std::vector<int32_t>& grid_order);
}  // namespace dsa

namespace {

thread_local std::string g_last_error;

// Device-side error word shared by all kernels of the library.
__device__ unsigned g_device_error;

// Ticket counters of the tensor-core attention kernel, which hands its rows
// to persistent CTAs dynamically: each launch takes one pair (next row,
// finished CTAs), in rotation, and its last CTA zeroes the pair again.
// Launches that overlap in time use different pairs while fewer than
// kTicketPairs launches lie between them.
constexpr unsigned kTicketPairs = 4096;
__device__ unsigned g_attn_tickets[2 * kTicketPairs];

constexpr int kMaxDevices = 64;

dsa_status fail(dsa_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
dsa_status fail(dsa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dsa_status cuda_fail(cudaError_t e, const char* where) {
  return fail(DSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  unsigned* err_word = nullptr;
  unsigned* tickets = nullptr;    // g_attn_tickets on this device
  int num_sms = 0;
  std::atomic<unsigned> next_pair{0};
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

// Per-device set-up: architecture check and the error word's address.
dsa_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device id %d", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    d.sm100 = (major == 10 && minor == 0);
    if (d.sm100) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_device_error);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
      d.err_word = static_cast<unsigned*>(p);
      e = cudaGetSymbolAddress(&p, g_attn_tickets);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
      d.tickets = static_cast<unsigned*>(p);
      e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    }
    d.init = true;
  }
  if (!d.sm100)
    return fail(DSA_ERR_UNSUPPORTED, "libdsa is built for sm_100a (B200); device %d is not", dev);
  *out = &d;
  return DSA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by the tensor-level calls.
dsa_status check_shape(int B, int H, int N, int D, int block) {
  if (B < 1 || H < 1 || N < 1) return fail(DSA_ERR_INVALID_ARG, "B, H, N must be >= 1 (got %d, %d, %d)", B, H, N);
  if ((long long)B * H > 65535) return fail(DSA_ERR_INVALID_ARG, "B*H = %lld exceeds 65535", (long long)B * H);
  if (D != 64 && D != 128) return fail(DSA_ERR_INVALID_ARG, "head_dim D must be 64 or 128 (got %d)", D);
  if (block != 64 && block != 128) return fail(DSA_ERR_INVALID_ARG, "block must be 64 or 128 (got %d)", block);
  const long long nB = (N + (long long)block - 1) / block;
  if ((long long)B * H * nB >= INT_MAX) return fail(DSA_ERR_INVALID_ARG, "too many block rows");
  return DSA_OK;
}

dsa_status check_blocks_limit(long long rows, int nB) {
  if (nB < 1 || nB > DSA_MAX_BLOCKS)
    return fail(DSA_ERR_INVALID_ARG, "nB = %d blocks per row; supported 1..%d", nB, DSA_MAX_BLOCKS);
  if (rows * nB >= INT_MAX) return fail(DSA_ERR_INVALID_ARG, "rows * nB exceeds the int32 CSR range");
  return DSA_OK;
}

bool cand_ok(const int32_t* rp, const int32_t* col) { return (rp == nullptr) == (col == nullptr); }

size_t pool_ws_bytes(long long BH, long long nB, int D) { return (size_t)(2 * BH * nB * D) * sizeof(float); }
size_t select_ws_bytes(long long rows) { return (size_t)(rows * 33) * sizeof(uint32_t); }

// ---- host-buffer pipeline (dsa_sparse_attention_host) ----

// Byte offsets of one chunk's device buffers inside a pipeline slot, each
// 256-byte aligned; `bytes` is the slot's size.
struct HostSlot {
  size_t q, k, v, out, lse, probs, ws_pool, ws_sel, row_ptr, col_idx, order, blk_lse, mass, bytes;
  size_t pool_bytes, sel_bytes;
};

HostSlot host_slot(long long c, long long N, long long D, long long block, size_t elem) {
  const long long nB = (N + block - 1) / block, rows = c * nB;
  auto take = [](size_t& off, size_t n) {
    const size_t at = off;
    off += (n + 255) & ~(size_t)255;
    return at;
  };
  HostSlot s{};
  size_t off = 0;
  s.q = take(off, (size_t)(c * N * D) * elem);
  s.k = take(off, (size_t)(c * N * D) * elem);
  s.v = take(off, (size_t)(c * N * D) * elem);
  s.out = take(off, (size_t)(c * N * D) * elem);
  s.lse = take(off, (size_t)(c * N) * sizeof(float));
  s.probs = take(off, (size_t)(rows * nB) * sizeof(float));
  s.pool_bytes = pool_ws_bytes(c, nB, (int)D);
  s.ws_pool = take(off, s.pool_bytes);
  s.sel_bytes = select_ws_bytes(rows);
  s.ws_sel = take(off, s.sel_bytes);
  s.row_ptr = take(off, (size_t)(rows + 1) * sizeof(int32_t));
  s.col_idx = take(off, (size_t)(rows * nB) * sizeof(int32_t));
  s.order = take(off, (size_t)rows * sizeof(int32_t));
  s.blk_lse = take(off, (size_t)(rows * nB * block) * sizeof(float));
  s.mass = take(off, (size_t)(rows * nB) * sizeof(float));
  s.bytes = off;
  return s;
}

int host_chunk(long long BH, int chunk_heads) {
  long long c = chunk_heads > 0 ? chunk_heads : BH / 8;
  if (c < 1) c = 1;
  if (c > BH) c = BH;
  return (int)c;
}

// The three streams and the events of the host-buffer pipeline, per device,
// created on first use.  One call at a time enqueues on them (the mutex), so
// a wait always refers to the event record of its own call.
struct HostStreams {
  bool init = false;
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> ev;
  std::mutex mu;
};
HostStreams g_host[kMaxDevices];

cudaError_t host_events(HostStreams& h, size_t n) {
  while (h.ev.size() < n) {
    cudaEvent_t e;
    cudaError_t r = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
    if (r != cudaSuccess) return r;
    h.ev.push_back(e);
  }
  return cudaSuccess;
}
// fine means (2 * BH * nBf * D floats) and the fine row softmax (BH * nBf^2 floats)
size_t hier_ws_bytes(long long BH, long long nBf, int D) {
  return (size_t)(2 * BH * nBf * D + BH * nBf * nBf) * sizeof(float);
}
constexpr int kMaxFineBlocks = 2048;
// mask bitmap (32 words per row), counts, transposed row_ptr and column
// capacity (rows * nB), delta (B*H*N floats)
size_t bwd_ws_bytes(long long BH, long long nB, long long N) {
  const long long rows = BH * nB;
  return (size_t)(rows * 32 + rows + (rows + 1) + rows * nB + BH * N) * 4;
}  // the score kernel's tile mask covers 32 tiles of 64

}  // namespace

extern "C" {

int dsa_version(void) { return 101; }

const char* dsa_last_error(void) { return g_last_error.c_str(); }

size_t dsa_workspace_size(int op, int B, int H, int N, int D, int block) {
  if (check_shape(B, H, N, D, block) != DSA_OK) return 0;
  const long long nB = (N + (long long)block - 1) / block;
  const long long BH = (long long)B * H;
  if (op == DSA_OP_POOL_SCORE) return pool_ws_bytes(BH, nB, D);
  if (op == DSA_OP_SELECT_TOPP) return select_ws_bytes(BH * nB);
  if (op == DSA_OP_ATTN_BWD) return bwd_ws_bytes(BH, nB, N);
  if (op == DSA_OP_POOL_SCORE_HIER2 || op == DSA_OP_POOL_SCORE_HIER4) {
    const int sub = op == DSA_OP_POOL_SCORE_HIER2 ? 2 : 4;
    const long long bf = block / sub;
    return hier_ws_bytes(BH, (N + bf - 1) / bf, D);
  }
  return 0;
}

dsa_status dsa_pool_score(const void* q, const void* k, dsa_dtype dt, int B, int H, int N,
                          int D, int block, float scale, const int32_t* cand_row_ptr,
                          const int32_t* cand_col, float* probs, void* workspace,
                          size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k || !probs || !workspace) return fail(DSA_ERR_INVALID_ARG, "null q, k, probs or workspace");
  if (dt != DSA_F32 && dt != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  dsa_status st = check_shape(B, H, N, D, block);
  if (st != DSA_OK) return st;
  const int nB = (N + block - 1) / block;
  const long long BH = (long long)B * H;
  if ((st = check_blocks_limit(BH * nB, nB)) != DSA_OK) return st;
  if (!cand_ok(cand_row_ptr, cand_col)) return fail(DSA_ERR_INVALID_ARG, "cand_row_ptr and cand_col must both be set or both be NULL");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(workspace, 16) || !aligned(probs, 4))
    return fail(DSA_ERR_INVALID_ARG, "q, k and workspace must be 16-byte aligned, probs 4-byte aligned");
  if (ws_bytes < pool_ws_bytes(BH, nB, D))
    return fail(DSA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes, pool_ws_bytes(BH, nB, D));
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* qbar = static_cast<float*>(workspace);
  float* kbar = qbar + BH * nB * D;
  cudaError_t e = dsa::launch_pool_means(q, k, dt == DSA_BF16, (int)BH, N, D, block, qbar, kbar, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool_means launch");
  e = dsa::launch_block_scores(qbar, kbar, (int)BH, nB, D, scale, cand_row_ptr, cand_col, probs,
                               dev->err_word, s);
  if (e != cudaSuccess) return cuda_fail(e, "block_scores launch");
  return DSA_OK;
}

dsa_status dsa_pool_score_hier(const void* q, const void* k, dsa_dtype dt, int B, int H, int N,
                               int D, int block, int sub, float scale, float* probs,
                               void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k || !probs || !workspace) return fail(DSA_ERR_INVALID_ARG, "null q, k, probs or workspace");
  if (dt != DSA_F32 && dt != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  dsa_status st = check_shape(B, H, N, D, block);
  if (st != DSA_OK) return st;
  if (sub != 1 && sub != 2 && sub != 4) return fail(DSA_ERR_INVALID_ARG, "sub must be 1, 2 or 4 (got %d)", sub);
  const int nB = (N + block - 1) / block;
  const int bf = block / sub;
  const int nBf = (N + bf - 1) / bf;
  const long long BH = (long long)B * H;
  if ((st = check_blocks_limit(BH * nB, nB)) != DSA_OK) return st;
  if (nBf > kMaxFineBlocks)
    return fail(DSA_ERR_INVALID_ARG, "%d sub-blocks per row; at most %d supported", nBf, kMaxFineBlocks);
  if (BH * nBf * nBf >= INT_MAX) return fail(DSA_ERR_INVALID_ARG, "fine score matrix too large");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(workspace, 16) || !aligned(probs, 4))
    return fail(DSA_ERR_INVALID_ARG, "q, k and workspace must be 16-byte aligned, probs 4-byte aligned");
  if (ws_bytes < hier_ws_bytes(BH, nBf, D))
    return fail(DSA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes, hier_ws_bytes(BH, nBf, D));
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* qbar = static_cast<float*>(workspace);
  float* kbar = qbar + BH * nBf * D;
  float* pf = kbar + BH * nBf * D;
  cudaError_t e = dsa::launch_pool_means(q, k, dt == DSA_BF16, (int)BH, N, D, bf, qbar, kbar, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool_means launch");
  e = dsa::launch_block_scores(qbar, kbar, (int)BH, nBf, D, scale, nullptr, nullptr, pf,
                               dev->err_word, s);
  if (e != cudaSuccess) return cuda_fail(e, "block_scores launch");
  e = dsa::launch_aggregate_probs(pf, (int)BH, N, block, sub, nB, nBf, probs, s);
  if (e != cudaSuccess) return cuda_fail(e, "aggregate_probs launch");
  return DSA_OK;
}

dsa_status dsa_select_topp(const float* probs, int rows, int nB, float p,
                           const int32_t* cand_row_ptr, const int32_t* cand_col,
                           int32_t* row_ptr, int32_t* col_idx, void* workspace,
                           size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (!probs || !row_ptr || !col_idx || !workspace)
    return fail(DSA_ERR_INVALID_ARG, "null probs, row_ptr, col_idx or workspace");
  if (rows < 1) return fail(DSA_ERR_INVALID_ARG, "rows must be >= 1 (got %d)", rows);
  dsa_status st = check_blocks_limit(rows, nB);
  if (st != DSA_OK) return st;
  if (!(p > 0.f && p <= 1.f)) return fail(DSA_ERR_INVALID_ARG, "p must be in (0, 1] (got %g)", (double)p);
  if (!cand_ok(cand_row_ptr, cand_col)) return fail(DSA_ERR_INVALID_ARG, "cand_row_ptr and cand_col must both be set or both be NULL");
  if (!aligned(probs, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(workspace, 16))
    return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  if (ws_bytes < select_ws_bytes(rows))
    return fail(DSA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes, select_ws_bytes(rows));
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  uint32_t* bitmaps = static_cast<uint32_t*>(workspace);
  int32_t* counts = reinterpret_cast<int32_t*>(bitmaps + (size_t)rows * 32);
  cudaError_t e = dsa::launch_select(probs, rows, nB, p, cand_row_ptr, cand_col, row_ptr, col_idx,
                                     bitmaps, counts, dev->err_word, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select_topp launch");
  return DSA_OK;
}

dsa_status dsa_row_order(const int32_t* row_ptr, int B, int H, int nB, int32_t* order,
                         void* stream) {
  g_last_error.clear();
  if (!row_ptr || !order) return fail(DSA_ERR_INVALID_ARG, "null row_ptr or order");
  if (B < 1 || H < 1) return fail(DSA_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", B, H);
  if (nB < 1 || nB > DSA_MAX_BLOCKS) return fail(DSA_ERR_INVALID_ARG, "nB outside 1..DSA_MAX_BLOCKS");
  if ((long long)B * H * nB >= INT_MAX) return fail(DSA_ERR_INVALID_ARG, "too many block rows");
  if (!aligned(row_ptr, 4) || !aligned(order, 4)) return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  DeviceInfo* dev = nullptr;
  dsa_status st = device_info(&dev);
  if (st != DSA_OK) return st;
  cudaError_t e = dsa::launch_row_order(row_ptr, B * H, nB, dev->num_sms, order,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "row_order launch");
  return DSA_OK;
}

dsa_status dsa_attn_fwd(const void* q, const void* k, const void* v, dsa_dtype dt, int B, int H,
                        int N, int D, int block, float scale, const int32_t* row_ptr,
                        const int32_t* col_idx, void* out, float* lse, float* blk_lse,
                        void* stream) {
  return dsa_attn_fwd_ordered(q, k, v, dt, B, H, N, D, block, scale, row_ptr, col_idx, nullptr,
                              out, lse, blk_lse, stream);
}

dsa_status dsa_attn_fwd_ordered(const void* q, const void* k, const void* v, dsa_dtype dt, int B,
                                int H, int N, int D, int block, float scale,
                                const int32_t* row_ptr, const int32_t* col_idx,
                                const int32_t* row_order, void* out, float* lse, float* blk_lse,
                                void* stream) {
  g_last_error.clear();
  if (!q || !k || !v || !out || !row_ptr || !col_idx)
    return fail(DSA_ERR_INVALID_ARG, "null q, k, v, out, row_ptr or col_idx");
  if (dt != DSA_F32 && dt != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  dsa_status st = check_shape(B, H, N, D, block);
  if (st != DSA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(row_order, 4) || !aligned(lse, 4) ||
      !aligned(blk_lse, 4))
    return fail(DSA_ERR_INVALID_ARG, "q, k, v, out must be 16-byte aligned; index and float arrays 4-byte aligned");
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  cudaError_t e;
  if (dt == DSA_BF16 && block == 128 && N >= 128) {
    const char* why = nullptr;
    const unsigned pair = dev->next_pair.fetch_add(1u) % kTicketPairs;
    e = dsa::launch_attn_sm100(q, k, v, BH, N, D, scale, row_ptr, col_idx, row_order, out, lse,
                               blk_lse, dev->tickets + 2 * pair, dev->num_sms, dev->err_word, s,
                               &why);
    if (e != cudaSuccess && why) return fail(DSA_ERR_CUDA, "attn_fwd: %s", why);
  } else {
    e = dsa::launch_attn_simt(q, k, v, dt == DSA_BF16, BH, N, D, block, scale, row_ptr, col_idx,
                              out, lse, blk_lse, dev->err_word, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd launch");
  return DSA_OK;
}

dsa_status dsa_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, dsa_dtype dt, int B, int H, int N,
                        int D, int block, float scale, const int32_t* row_ptr,
                        const int32_t* col_idx, void* dq, void* dk, void* dv, void* workspace,
                        size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k || !v || !out || !dout || !lse || !row_ptr || !col_idx || !dq || !dk || !dv || !workspace)
    return fail(DSA_ERR_INVALID_ARG, "null pointer argument");
  if (dt != DSA_F32 && dt != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  dsa_status st = check_shape(B, H, N, D, block);
  if (st != DSA_OK) return st;
  const int nB = (N + block - 1) / block;
  const long long BH = (long long)B * H;
  if ((st = check_blocks_limit(BH * nB, nB)) != DSA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(out, 4) || !aligned(dout, 4) ||
      !aligned(dq, 4) || !aligned(dk, 4) || !aligned(dv, 4) || !aligned(lse, 4) ||
      !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(workspace, 16))
    return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  if (ws_bytes < bwd_ws_bytes(BH, nB, N))
    return fail(DSA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes, bwd_ws_bytes(BH, nB, N));
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  const long long rows = BH * nB;
  uint32_t* bitmap = static_cast<uint32_t*>(workspace);
  int32_t* counts = reinterpret_cast<int32_t*>(bitmap + rows * 32);
  int32_t* t_row_ptr = counts + rows;
  int32_t* t_col = t_row_ptr + rows + 1;
  float* delta = reinterpret_cast<float*>(t_col + rows * nB);
  cudaError_t e = dsa::launch_attn_bwd(q, k, v, out, dout, lse, dt == DSA_BF16, (int)BH, N, D, block,
                                       scale, row_ptr, col_idx, dq, dk, dv, bitmap, counts, t_row_ptr,
                                       t_col, delta, dev->err_word, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_bwd launch");
  return DSA_OK;
}

dsa_status dsa_block_mass(const float* lse, const float* blk_lse, int B, int H, int N, int block,
                          const int32_t* row_ptr, float* mass, void* stream) {
  g_last_error.clear();
  if (!lse || !blk_lse || !row_ptr || !mass)
    return fail(DSA_ERR_INVALID_ARG, "null lse, blk_lse, row_ptr or mass");
  dsa_status st = check_shape(B, H, N, 64, block);
  if (st != DSA_OK) return st;
  if (!aligned(lse, 4) || !aligned(blk_lse, 4) || !aligned(row_ptr, 4) || !aligned(mass, 4))
    return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaError_t e = dsa::launch_block_mass(lse, blk_lse, B * H, N, block, row_ptr, mass,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block_mass launch");
  return DSA_OK;
}

dsa_status dsa_mass_to_probs(const int32_t* row_ptr, const int32_t* col_idx, const float* mass,
                             int rows, int nB, float* probs, void* stream) {
  g_last_error.clear();
  if (!row_ptr || !col_idx || !mass || !probs)
    return fail(DSA_ERR_INVALID_ARG, "null row_ptr, col_idx, mass or probs");
  if (rows < 1) return fail(DSA_ERR_INVALID_ARG, "rows must be >= 1 (got %d)", rows);
  dsa_status st = check_blocks_limit(rows, nB);
  if (st != DSA_OK) return st;
  if (!aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(mass, 4) || !aligned(probs, 4))
    return fail(DSA_ERR_INVALID_ARG, "misaligned pointer");
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaError_t e = dsa::launch_mass_to_probs(row_ptr, col_idx, mass, rows, nB, probs, dev->err_word,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mass_to_probs launch");
  return DSA_OK;
}

dsa_status dsa_hilbert_order(int T, int H, int W, int n_prefix, int32_t* perm) {
  g_last_error.clear();
  if (!perm) return fail(DSA_ERR_INVALID_ARG, "null perm");
  if (T < 1 || H < 1 || W < 1 || n_prefix < 0)
    return fail(DSA_ERR_INVALID_ARG, "need T, H, W >= 1 and n_prefix >= 0");
  const int side = std::max(T, std::max(H, W));
  if (side > (1 << 20)) return fail(DSA_ERR_INVALID_ARG, "grid side above 2^20");
  const long long cells = (long long)T * H * W;
  if (cells + n_prefix > 0x7fffffffLL) return fail(DSA_ERR_INVALID_ARG, "too many tokens");
  int bits = 1;
  while ((1 << bits) < side) ++bits;
  std::vector<std::pair<uint64_t, int32_t>> keys;
  keys.reserve((size_t)cells);
  for (int t = 0; t < T; ++t)
    for (int y = 0; y < H; ++y)
      for (int x = 0; x < W; ++x)
        keys.emplace_back(dsa::hilbert_key3((uint32_t)t, (uint32_t)y, (uint32_t)x, bits),
                          (int32_t)(n_prefix + ((long long)t * H + y) * W + x));
  std::sort(keys.begin(), keys.end());
  for (int i = 0; i < n_prefix; ++i) perm[i] = i;
  for (size_t i = 0; i < keys.size(); ++i) perm[n_prefix + i] = keys[i].second;
  return DSA_OK;
}

dsa_status dsa_gilbert_order(int T, int H, int W, int n_prefix, int32_t* perm) {
  g_last_error.clear();
  if (!perm) return fail(DSA_ERR_INVALID_ARG, "null perm");
  if (T < 1 || H < 1 || W < 1 || n_prefix < 0)
    return fail(DSA_ERR_INVALID_ARG, "need T, H, W >= 1 and n_prefix >= 0");
  if (std::max(T, std::max(H, W)) > (1 << 20)) return fail(DSA_ERR_INVALID_ARG, "grid side above 2^20");
  const long long cells = (long long)T * H * W;
  if (cells + n_prefix > 0x7fffffffLL) return fail(DSA_ERR_INVALID_ARG, "too many tokens");
  std::vector<int32_t> grid;
  if (!dsa::generalised_hilbert_cells(T, H, W, grid) || (long long)grid.size() != cells)
    return fail(DSA_ERR_INVALID_ARG, "no walk for a %d x %d x %d grid", T, H, W);
  for (int i = 0; i < n_prefix; ++i) perm[i] = i;
  for (size_t i = 0; i < grid.size(); ++i) perm[n_prefix + i] = n_prefix + grid[i];
  return DSA_OK;
}

dsa_status dsa_permute_tokens(const void* src, void* dst, dsa_dtype dt, int B, int H, int N, int D,
                              const int32_t* perm, int inverse, void* stream) {
  g_last_error.clear();
  if (!src || !dst || !perm) return fail(DSA_ERR_INVALID_ARG, "null src, dst or perm");
  if (src == dst) return fail(DSA_ERR_INVALID_ARG, "src and dst must differ");
  if (dt != DSA_F32 && dt != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (B < 1 || H < 1 || N < 1) return fail(DSA_ERR_INVALID_ARG, "need B, H, N >= 1");
  if (D != 64 && D != 128) return fail(DSA_ERR_INVALID_ARG, "D must be 64 or 128 (got %d)", D);
  if (inverse != 0 && inverse != 1) return fail(DSA_ERR_INVALID_ARG, "inverse must be 0 or 1");
  if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(perm, 4))
    return fail(DSA_ERR_INVALID_ARG, "src and dst must be 16-byte aligned, perm 4-byte aligned");
  DeviceInfo* dev = nullptr;
  dsa_status st = device_info(&dev);
  if (st != DSA_OK) return st;
  cudaError_t e = dsa::launch_permute_tokens(src, dst, dt == DSA_BF16 ? 2 : 4, B * H, N, D, perm,
                                             inverse != 0, dev->err_word,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "permute_tokens launch");
  return DSA_OK;
}

size_t dsa_host_pipeline_workspace_size(dsa_dtype dt, int B, int H, int N, int D, int block,
                                        int chunk_heads) {
  if (dt != DSA_BF16 && dt != DSA_F32) return 0;
  if (check_shape(B, H, N, D, block) != DSA_OK) return 0;
  const int c = host_chunk((long long)B * H, chunk_heads);
  return 2 * host_slot(c, N, D, block, dt == DSA_BF16 ? 2 : 4).bytes;
}

dsa_status dsa_sparse_attention_host(const void* q, const void* k, const void* v, dsa_dtype dt,
                                     int B, int H, int N, int D, int block, float scale, float p,
                                     int chunk_heads, void* out, void* workspace,
                                     size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (dt != DSA_BF16 && dt != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "dt must be DSA_BF16 or DSA_F32");
  dsa_status st = check_shape(B, H, N, D, block);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !out || !workspace) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.f && p <= 1.f)) return fail(DSA_ERR_INVALID_ARG, "p must be in (0, 1] (got %g)", (double)p);
  if (!aligned(workspace, 256)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const long long BH = (long long)B * H;
  const int c = host_chunk(BH, chunk_heads);
  const size_t elem = dt == DSA_BF16 ? 2 : 4;
  const HostSlot L = host_slot(c, N, D, block, elem);
  if (ws_bytes < 2 * L.bytes)
    return fail(DSA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, 2 * L.bytes);
  const long long nB = (N + (long long)block - 1) / block;
  if ((st = check_blocks_limit(c * nB, (int)nB)) != DSA_OK) return st;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  int id = 0;
  cudaError_t e = cudaGetDevice(&id);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  HostStreams& h = g_host[id];
  std::lock_guard<std::mutex> lock(h.mu);
  if (!h.init) {
    e = cudaStreamCreateWithFlags(&h.s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h.s_comp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h.s_out, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
    h.init = true;
  }
  const long long n_chunks = (BH + c - 1) / c;
  // events: [0] start, [1] end, then in / comp / out done per chunk
  if ((e = host_events(h, (size_t)(2 + 3 * n_chunks))) != cudaSuccess)
    return cuda_fail(e, "cudaEventCreateWithFlags");
  cudaEvent_t* ev = h.ev.data();
  auto in_done = [&](long long i) { return ev[2 + 3 * i]; };
  auto comp_done = [&](long long i) { return ev[3 + 3 * i]; };
  auto out_done = [&](long long i) { return ev[4 + 3 * i]; };
  cudaStream_t caller = static_cast<cudaStream_t>(stream);
  auto ok = [&](cudaError_t r) { return (e = r) == cudaSuccess; };
  if (!ok(cudaEventRecord(ev[0], caller)) || !ok(cudaStreamWaitEvent(h.s_in, ev[0], 0)))
    return cuda_fail(e, "host pipeline start");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t head_bytes = (size_t)N * D * elem;
  for (long long ci = 0; ci < n_chunks; ++ci) {
    const long long h0 = ci * c, n = (h0 + c <= BH ? c : BH - h0);
    uint8_t* slot = ws + (size_t)(ci & 1) * L.bytes;
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)n * head_bytes;
    // copy-in: the slot's inputs are free once chunk ci - 2 has computed
    if (ci >= 2 && !ok(cudaStreamWaitEvent(h.s_in, comp_done(ci - 2), 0))) break;
    if (!ok(cudaMemcpyAsync(slot + L.q, static_cast<const uint8_t*>(q) + off, bytes,
                            cudaMemcpyHostToDevice, h.s_in)) ||
        !ok(cudaMemcpyAsync(slot + L.k, static_cast<const uint8_t*>(k) + off, bytes,
                            cudaMemcpyHostToDevice, h.s_in)) ||
        !ok(cudaMemcpyAsync(slot + L.v, static_cast<const uint8_t*>(v) + off, bytes,
                            cudaMemcpyHostToDevice, h.s_in)) ||
        !ok(cudaEventRecord(in_done(ci), h.s_in)))
      break;
    // compute: after the copy-in, and once the slot's O of chunk ci - 2 is out
    if (!ok(cudaStreamWaitEvent(h.s_comp, in_done(ci), 0))) break;
    if (ci >= 2 && !ok(cudaStreamWaitEvent(h.s_comp, out_done(ci - 2), 0))) break;
    const int hn = (int)n;
    const int rows = (int)(n * nB);
    float* probs = reinterpret_cast<float*>(slot + L.probs);
    int32_t* rp = reinterpret_cast<int32_t*>(slot + L.row_ptr);
    int32_t* ci_idx = reinterpret_cast<int32_t*>(slot + L.col_idx);
    int32_t* order = reinterpret_cast<int32_t*>(slot + L.order);
    float* lse = reinterpret_cast<float*>(slot + L.lse);
    float* bl = reinterpret_cast<float*>(slot + L.blk_lse);
    if ((st = dsa_pool_score(slot + L.q, slot + L.k, dt, 1, hn, N, D, block, scale, nullptr,
                             nullptr, probs, slot + L.ws_pool, L.pool_bytes, h.s_comp)) != DSA_OK ||
        (st = dsa_select_topp(probs, rows, (int)nB, p, nullptr, nullptr, rp, ci_idx,
                              slot + L.ws_sel, L.sel_bytes, h.s_comp)) != DSA_OK ||
        (st = dsa_row_order(rp, 1, hn, (int)nB, order, h.s_comp)) != DSA_OK ||
        (st = dsa_attn_fwd_ordered(slot + L.q, slot + L.k, slot + L.v, dt, 1, hn, N, D, block,
                                   scale, rp, ci_idx, order, slot + L.out, lse, bl,
                                   h.s_comp)) != DSA_OK ||
        (st = dsa_block_mass(lse, bl, 1, hn, N, block, rp, reinterpret_cast<float*>(slot + L.mass),
                             h.s_comp)) != DSA_OK)
      return st;  // the inner call set the message
    if (!ok(cudaEventRecord(comp_done(ci), h.s_comp))) break;
    // copy-out
    if (!ok(cudaStreamWaitEvent(h.s_out, comp_done(ci), 0)) ||
        !ok(cudaMemcpyAsync(static_cast<uint8_t*>(out) + off, slot + L.out, bytes,
                            cudaMemcpyDeviceToHost, h.s_out)) ||
        !ok(cudaEventRecord(out_done(ci), h.s_out)))
      break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline enqueue");
  if (!ok(cudaEventRecord(ev[1], h.s_out)) || !ok(cudaStreamWaitEvent(caller, ev[1], 0)))
    return cuda_fail(e, "host pipeline end");
  return DSA_OK;
}

dsa_status dsa_selftest_wait_timeout(unsigned long long limit_ns, void* stream) {
  g_last_error.clear();
  if (limit_ns < 1000ull || limit_ns > dsa::kWaitLimitNs)
    return fail(DSA_ERR_INVALID_ARG, "limit_ns must be in [1000, %llu] (got %llu)",
                dsa::kWaitLimitNs, limit_ns);
  DeviceInfo* dev = nullptr;
  dsa_status st = device_info(&dev);
  if (st != DSA_OK) return st;
  cudaError_t e = dsa::launch_wait_timeout(limit_ns, dev->err_word, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait_timeout launch");
  return DSA_OK;
}

dsa_status dsa_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  g_last_error.clear();
  if (n < 0) return fail(DSA_ERR_INVALID_ARG, "n must be >= 0 (got %d)", n);
  if (n > 0 && (x == nullptr || y == nullptr)) return fail(DSA_ERR_INVALID_ARG, "x and y must not be null");
  if (!aligned(x, 4) || !aligned(y, 4)) return fail(DSA_ERR_INVALID_ARG, "x and y must be 4-byte aligned");
  DeviceInfo* dev = nullptr;
  dsa_status st = device_info(&dev);
  if (st != DSA_OK) return st;
  if (n == 0) return DSA_OK;
  cudaError_t e = dsa::launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "exp2_poly launch");
  return DSA_OK;
}

dsa_status dsa_device_status(void* stream) {
  g_last_error.clear();
  DeviceInfo* dev = nullptr;
  dsa_status st = device_info(&dev);
  if (st != DSA_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word == 0) return DSA_OK;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  return fail(DSA_ERR_DEVICE, "device error word 0x%x:%s%s%s%s%s%s%s", word,
              (word & dsa::kErrCsrIndex) ? " csr-index-out-of-range" : "",
              (word & dsa::kErrRowPtr) ? " bad-row-ptr" : "",
              (word & dsa::kErrProb) ? " probability-outside-[0,1]" : "",
              (word & dsa::kErrTimeout) ? " wait-timeout" : "",
              (word & dsa::kErrAlign) ? " shared-memory-misaligned" : "",
              (word & dsa::kErrPerm) ? " permutation-index-out-of-range" : "",
              (word & dsa::kErrRowOrder) ? " row-order-index-out-of-range" : "");
}

}  // extern "C"

namespace dsa {

// For the library's other entry points: the current device's set-up
// (architecture check, error word) and the per-thread error text.
dsa_status api_checked_device(unsigned** err_word) {
  DeviceInfo* d = nullptr;
  const dsa_status st = device_info(&d);
  if (st == DSA_OK) *err_word = d->err_word;
  return st;
}

void api_set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

}  // namespace dsa
