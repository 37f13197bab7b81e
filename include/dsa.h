/*
 * dsa.h -- C ABI of libdsa: dynamic block-sparse self-attention for video
 * diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * The pipeline, per (batch b, head h), over N tokens cut into nB = ceil(N /
 * block) blocks B_i = [i*block, min(N, (i+1)*block)):
 *
 *   dsa_pool_score   qbar_i, kbar_j = means of the rows of Q, K in each block;
 *                    P_ij = softmax_j(scale * qbar_i . kbar_j), over all key
 *                    blocks or over a candidate set C_i (reduced search).
 *   dsa_select_topp  per row i: the shortest prefix of the candidates ordered
 *                    by (P desc, block index asc) whose mass is >= p, as CSR.
 *   dsa_row_order    the order in which the attention takes a mask's rows
 *                    (each head's longest first), for dsa_attn_fwd_ordered.
 *   dsa_attn_fwd     exact softmax attention of every query in B_i over the
 *                    keys of the selected blocks, with per-block log-sums
 *                    (dsa_attn_fwd_ordered: the same, rows in a given order).
 *   dsa_block_mass   the exact softmax mass each selected block receives.
 *   dsa_attn_bwd     gradients of the attention for a fixed mask.
 *   dsa_mass_to_probs  those masses as dense rows, for a Top-p selection on
 *                    exact attention weights (the next mask of a schedule).
 *   dsa_sparse_attention_host  the four calls above on host-resident Q, K, V
 *                    (chunks of heads, copies overlapped with compute).
 *   dsa_selftest_wait_timeout, dsa_selftest_exp2_poly  self-tests.
 *   dsa_hilbert_order, dsa_gilbert_order, dsa_permute_tokens  token
 *                    reordering along a 3-D Hilbert curve (the enclosing
 *                    cube's, or one generalised to the grid's own box) before
 *                    the pipeline, and back after it.
 *
 * Sources: "Sparse Attention for Video Generation Acceleration via Growing
 * Sparsity and Reduced Search" (GSRS, arXiv 2610.21129): abstract (Top-p
 * selection; exact attention weights inside the FlashAttention pass; reduced
 * search over an early candidate set), Figure 3 (block-level attention maps)
 * and Figure 4 (growing Top-p, reduced search, mask reuse).  "DSV" (arXiv
 * 2502.07590) abstract: kernels that identify critical key blocks and then
 * compute the sparse attention.  The mean-pooled block score is the method's
 * cheap estimator of the block-level map; the papers do not spell it out.
 *
 * Conventions shared by every call:
 *  - Q, K, V, O are contiguous [B, H, N, D] tensors (row-major, D fastest),
 *    in DSA_BF16 or DSA_F32.  D is 64 or 128; block is 64 or 128.
 *  - Every pointer argument is a DEVICE pointer owned by the caller unless
 *    stated otherwise; the library keeps no reference after a call returns
 *    and allocates no device memory at call time.  Scratch memory is passed
 *    in as `workspace` (size from dsa_workspace_size).  What the library
 *    itself holds per device, for the life of the process: the device
 *    error word and the attention's ticket counters (module data, 32 KB),
 *    the static selection scratch of dsa_select_topp_static, and, once
 *    dsa_sparse_attention_host has run, three streams and a pool of events.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and never synchronises the host, except
 *    dsa_device_status.
 *  - Q/K/V/O pointers must be 16-byte aligned; float and int32 arrays 4-byte
 *    aligned.
 *  - Errors: every call returns a dsa_status and never aborts or traps.
 *    DSA_ERR_INVALID_ARG  a null required pointer, an unsupported size
 *                         (see each call), p outside (0, 1], bad alignment.
 *    DSA_ERR_UNSUPPORTED  dtype/size combination not built, or a device
 *                         that is not sm_100.
 *    DSA_ERR_CUDA         a CUDA runtime error at launch; the text is
 *                         available from dsa_last_error().
 *    DSA_ERR_DEVICE       reported by dsa_device_status when a kernel saw
 *                         malformed input (a CSR index out of range, a
 *                         probability outside [0, 1]) or a bounded wait ran
 *                         out; the kernel skipped the affected work.
 *    On an error nothing is launched.  dsa_last_error() is per host thread.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,
  DSA_ERR_UNSUPPORTED = 2,
  DSA_ERR_CUDA = 3,
  DSA_ERR_DEVICE = 4
} dsa_status;

typedef enum dsa_dtype { DSA_F32 = 0, DSA_BF16 = 1 } dsa_dtype;

/* Operation ids for dsa_workspace_size. */
enum { DSA_OP_POOL_SCORE = 0, DSA_OP_SELECT_TOPP = 1, DSA_OP_POOL_SCORE_HIER2 = 2,
       DSA_OP_POOL_SCORE_HIER4 = 3, DSA_OP_ATTN_BWD = 4 };

/* Largest number of blocks per row that dsa_pool_score / dsa_select_topp
 * accept (one warp sorts a row of up to 1024 blocks in registers). */
#define DSA_MAX_BLOCKS 1024

/*
 * Bytes of scratch memory `op` needs for the given sizes (B, H, N, D,
 * block as in the calls below).  Returns 0 for invalid sizes.
 *   DSA_OP_POOL_SCORE : 2 * B*H*nB*D floats (pooled means).
 *   DSA_OP_SELECT_TOPP: B*H*nB * 33 words (selection bitmaps and counts).
 *   DSA_OP_POOL_SCORE_HIER2 / _HIER4: dsa_pool_score_hier with sub = 2 / 4:
 *     2 * B*H*nBf*D floats (sub-block means) + B*H*nBf^2 floats (their row
 *     softmax), nBf = ceil(N / (block / sub)).
 *   DSA_OP_ATTN_BWD: 4-byte words: B*H*nB*32 (mask bitmap) + B*H*nB (counts)
 *     + B*H*nB + 1 (transposed row_ptr) + B*H*nB*nB (transposed columns)
 *     + B*H*N (rowsum(dO * O)).
 */
size_t dsa_workspace_size(int op, int B, int H, int N, int D, int block);

/*
 * Pooled block scores and their row softmax (GSRS abstract: the cheap block
 * importance estimate that Top-p selection consumes; Figure 4: reduced
 * search evaluates only blocks inside the candidate mask).
 *
 *   q, k      [B, H, N, D] in dtype dt.
 *   scale     score scale, > 0 (normally 1/sqrt(D)).
 *   cand_row_ptr, cand_col
 *             optional candidate CSR over the B*H*nB block rows (row r =
 *             (b*H + h)*nB + i): cand_row_ptr [B*H*nB + 1] int32 ascending,
 *             cand_col int32 in [0, nB).  Both NULL = full search.
 *   probs     out, fp32 [B*H, nB, nB]: P_ij, exactly 0 outside C_i; a row
 *             with no candidates is all 0.
 *   workspace >= dsa_workspace_size(DSA_OP_POOL_SCORE, ...) bytes, 16-byte
 *             aligned, contents ignored and overwritten.
 * Limits: nB <= DSA_MAX_BLOCKS.
 */
dsa_status dsa_pool_score(const void* q, const void* k, dsa_dtype dt,
                          int B, int H, int N, int D, int block, float scale,
                          const int32_t* cand_row_ptr, const int32_t* cand_col,
                          float* probs, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * Two-level block estimate (DFSAttn abstract: hierarchical block scoring for
 * block importance; the pages give no construction, so this is the plain
 * two-level pooling): the block means and row softmax of dsa_pool_score,
 * taken over sub-blocks of block/sub rows, then folded back into block rows.
 *
 *   Pf[a, b] = softmax_b(scale * qbar_a . kbar_b) over the sub-blocks,
 *   probs[i, j] = sum over the query sub-blocks a of block i of
 *                 (|a| / |B_i|) * sum over the key sub-blocks b of block j of Pf[a, b].
 *
 * sub = 1 gives dsa_pool_score's P.  Full search only (no candidate set).
 *   sub       1, 2 or 4 (block / sub rows per sub-block).
 *   workspace >= dsa_workspace_size(DSA_OP_POOL_SCORE_HIER2 or _HIER4, ...)
 *             bytes (sub = 1 needs the _HIER2 size or more), 16-byte aligned.
 *   probs     device out, fp32 [B*H, nB, nB]; rows sum to 1.
 * Limits: nB <= DSA_MAX_BLOCKS and at most 2048 sub-blocks per head.
 */
dsa_status dsa_pool_score_hier(const void* q, const void* k, dsa_dtype dt, int B, int H, int N,
                               int D, int block, int sub, float scale, float* probs,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * Per-row Top-p block selection (GSRS abstract: Top-p selection for
 * adaptive sparsity; Figure 4: tighter thresholds keep fewer blocks).
 *
 * For each of the `rows` rows of `probs` ([rows, nB] fp32 in [0, 1]): order
 * the candidate blocks by (probability desc, block index asc) and keep the
 * shortest prefix whose exact sum (integer arithmetic on the fp32 values,
 * independent of summation order) is >= p.  p >= 1 keeps every candidate;
 * if no prefix reaches p every candidate is kept.
 *
 *   p          threshold in (0, 1], used as the fp32 value given.
 *   cand_*     optional candidate CSR as in dsa_pool_score (row r of probs
 *              uses candidates cand_col[cand_row_ptr[r] .. cand_row_ptr[r+1])).
 *   row_ptr    out, int32 [rows + 1]: row_ptr[0] = 0, row_ptr[rows] = nnz.
 *   col_idx    out, int32 [nnz], ascending within each row; the caller
 *              provides capacity for rows * nB entries.
 *   workspace  >= dsa_workspace_size(DSA_OP_SELECT_TOPP, ...) bytes with
 *              B*H*nB = rows.
 * Limits: nB <= DSA_MAX_BLOCKS.  The caller reads nnz from row_ptr[rows].
 */
dsa_status dsa_select_topp(const float* probs, int rows, int nB, float p,
                           const int32_t* cand_row_ptr, const int32_t* cand_col,
                           int32_t* row_ptr, int32_t* col_idx,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * The order in which the attention's persistent CTAs take a mask's rows (DSV
 * abstract: the work per query block is skewed, and handed out
 * dynamically).  The CTAs draw rows one at a time, each as soon as it is
 * free; the launch ends when the last CTA finishes, so the rows drawn last
 * should be short.  This call lists each head's rows longest first:
 *
 *   order[bh*nB + j] = bh*nB + i,  i the row of head bh with the j-th most
 *   blocks (row_ptr[r+1] - row_ptr[r]), ties by ascending i.
 *
 * Heads stay in index order, so the rows in flight still read the K and V
 * of one or two heads (which stay in L2).
 *
 *   row_ptr   device, int32 [B*H*nB + 1]: a CSR mask (dsa_select_topp's).
 *   order     device out, int32 [B*H*nB]: a permutation of 0 .. B*H*nB-1
 *             whatever row_ptr holds (a malformed row_ptr only makes the
 *             order arbitrary).
 * One launch of a few CTAs per head (about two per SM in all), nB^2
 * comparisons per head (40 heads of nB = 591: under 10 microseconds).
 * Limits: nB <= DSA_MAX_BLOCKS.
 */
dsa_status dsa_row_order(const int32_t* row_ptr, int B, int H, int nB, int32_t* order,
                         void* stream);

/*
 * Exact block-sparse attention forward (GSRS abstract: exact attention over
 * the selected blocks, computed FlashAttention-style with the exact weights
 * as a by-product).
 *
 * For query t in block i of (b, h): o_t = sum_u softmax_u(scale q_t.k_u) v_u
 * over the keys u < N of the blocks col_idx[row_ptr[r] .. row_ptr[r+1]),
 * r = (b*H + h)*nB + i.
 *
 *   q, k, v   [B, H, N, D] in dt.   out: [B, H, N, D] in dt.
 *   row_ptr, col_idx   CSR block mask over the B*H*nB rows (any column order).
 *   lse       optional out, fp32 [B, H, N]: natural-log sum of exp(scale q.k)
 *             over the attended keys; -inf for a row with no blocks.
 *   blk_lse   optional out, fp32 [nnz, block]: blk_lse[s*block + t'] =
 *             log sum over the keys of block col_idx[s] of exp(scale q.k)
 *             for the t'-th query of the row's block (entries past a ragged
 *             last block are not written).
 * A row with no blocks gives O = 0.  bf16 runs on tcgen05 tensor cores with
 * fp32 accumulation; fp32 (and block 64) runs on an exact-fp32 CUDA-core
 * path.
 * Scheduling (bf16, block 128): one persistent CTA per SM takes rows from a
 * ticket counter in device memory that the library keeps per device (4,096
 * counters used in rotation, one per launch; the launch's last CTA zeroes its
 * counter again), so rows of skewed length are balanced dynamically (DSV
 * abstract); this call takes them in index order, dsa_attn_fwd_ordered in a
 * given one.  Launches that run at the same time, on any streams, use
 * different counters while fewer than 4,096 launches lie between them; a
 * captured CUDA graph replays its launch with the counter of its capture.
 * Errors: a malformed row (column index outside [0, nB), decreasing row_ptr)
 * sets the device error word and is written as an empty row; a device wait
 * that runs out (1 s) sets the error word and leaves the rows that the
 * affected CTA had not finished unwritten.  dsa_device_status reports both.
 */
dsa_status dsa_attn_fwd(const void* q, const void* k, const void* v, dsa_dtype dt,
                        int B, int H, int N, int D, int block, float scale,
                        const int32_t* row_ptr, const int32_t* col_idx,
                        void* out, float* lse, float* blk_lse, void* stream);

/*
 * dsa_attn_fwd with the rows taken in a given order (DSV abstract: skewed
 * work per query block).  The persistent CTAs draw tickets 0, 1, 2, ...;
 * ticket t is row row_order[t].  With each head's rows longest first
 * (dsa_row_order) the short rows come at the end of the launch, where they
 * fill the gaps that the last long rows leave.
 *
 *   row_order optional, device, int32 [B*H*nB]: a permutation of the row
 *             indices; NULL takes them in index order (= dsa_attn_fwd).
 *   the other arguments as for dsa_attn_fwd.
 * The order changes only which CTA computes a row and when: every output is
 * the same with any order.  The fp32 / block-64 path ignores it.
 * Errors as for dsa_attn_fwd, and: a row_order entry outside [0, B*H*nB)
 * sets the device error word and is passed over (a row that a
 * non-permutation leaves out is not written; one it names twice is written
 * twice, with the same values).
 */
dsa_status dsa_attn_fwd_ordered(const void* q, const void* k, const void* v, dsa_dtype dt,
                                int B, int H, int N, int D, int block, float scale,
                                const int32_t* row_ptr, const int32_t* col_idx,
                                const int32_t* row_order, void* out, float* lse,
                                float* blk_lse, void* stream);

/*
 * Gradients of dsa_attn_fwd's O for a fixed mask (DSV abstract: DiTs are
 * trained with the same dynamic sparsity).  With P the softmax of each
 * query over the keys of its row's selected blocks (from the forward's
 * lse), dP = dO V^T and delta = rowsum(dO * O):
 *
 *   dS = P * (dP - delta),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
 *
 *   q, k, v, out, dout  device, [B, H, N, D] in dt (out: dsa_attn_fwd's O).
 *   lse        device, fp32 [B, H, N]: dsa_attn_fwd's lse.
 *   row_ptr, col_idx   the forward's CSR mask (no repeated column in a row).
 *   dq, dk, dv device out, [B, H, N, D] in dt; key blocks that no row
 *              selected get dK = dV = 0, queries of empty rows dQ = 0.
 *   workspace  >= dsa_workspace_size(DSA_OP_ATTN_BWD, ...) bytes, 16-byte
 *              aligned.
 * Arithmetic: bf16 with block 128 runs on tcgen05 tensor cores with fp32
 * accumulation, and P and dS enter the gradient products as two bf16 terms
 * each (hi = bf16(x), lo = bf16(x - hi)), about 2^-17 of each term; fp32,
 * and block 64, run in exact fp32 on CUDA cores.  Every key block's
 * contributions are summed in ascending query-block order, so the result is
 * the same from run to run.  Errors as for dsa_attn_fwd; a malformed mask
 * sets the device error word.
 */
dsa_status dsa_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, dsa_dtype dt, int B, int H, int N,
                        int D, int block, float scale, const int32_t* row_ptr,
                        const int32_t* col_idx, void* dq, void* dk, void* dv, void* workspace,
                        size_t ws_bytes, void* stream);

/*
 * Exact softmax mass of each selected block (GSRS abstract: exact attention
 * weights at negligible overhead; Figure 2: the recall of a block mask).
 *
 *   mass[s] = mean over the queries t of block i of exp(blk_lse[s, t] - lse_t)
 * for every slot s of row r = (b*H + h)*nB + i.  Inputs are dsa_attn_fwd's
 * lse [B, H, N] and blk_lse [nnz, block]; mass is fp32 [nnz], aligned with
 * col_idx.  Over a row the masses sum to 1.
 */
dsa_status dsa_block_mass(const float* lse, const float* blk_lse,
                          int B, int H, int N, int block, const int32_t* row_ptr,
                          float* mass, void* stream);

/*
 * The whole pipeline (dsa_pool_score, dsa_select_topp, dsa_row_order,
 * dsa_attn_fwd_ordered with that order, dsa_block_mass; full search, Top-p
 * threshold p) on HOST-resident Q, K,
 * V, with O written back to host memory.  Every (b, h) is an independent
 * problem (DSV abstract: each head is its own work item), so the B*H axis is
 * cut into chunks of `chunk_heads` heads that run on three streams the
 * library keeps per device: the copy-in of chunk c+1 (host -> device) and
 * the copy-out of chunk c-1 overlap the compute of chunk c.  Two device
 * slots in `workspace` alternate; events keep a slot from being refilled
 * before its compute, or its O before its copy-out, has finished.
 *
 *   q, k, v     host, [B, H, N, D] in dt, contiguous; page-locked (pinned)
 *               for the copies to overlap (pageable memory works, with
 *               copies that do not overlap).
 *   out         host, [B, H, N, D] in dt, same rules.
 *   p, scale    as in dsa_select_topp and dsa_pool_score / dsa_attn_fwd.
 *   chunk_heads heads per chunk, 1 .. B*H; <= 0 picks max(1, B*H / 8).
 *   workspace   device, >= dsa_host_pipeline_workspace_size(...) bytes with
 *               the same shape and chunk_heads, 256-byte aligned.
 * Asynchronous: the copy-in waits for the work already on `stream`, and
 * `stream` waits for the last copy-out, so synchronising `stream` (or the
 * device) makes O visible in `out`.  Calls on one device are serialised on
 * its three pipeline streams.  Errors: those of the five calls (shape,
 * limits), DSA_ERR_INVALID_ARG for null pointers, a small or misaligned
 * workspace or p outside (0, 1]; device-side flags as for those calls
 * (dsa_device_status).
 */
dsa_status dsa_sparse_attention_host(const void* q, const void* k, const void* v, dsa_dtype dt,
                                     int B, int H, int N, int D, int block, float scale, float p,
                                     int chunk_heads, void* out, void* workspace,
                                     size_t ws_bytes, void* stream);

/* Device workspace bytes for dsa_sparse_attention_host (two slots of one
 * chunk's device buffers: Q, K, V, O, lse, P, the CSR at full capacity,
 * per-block log-sums and masses, and the score and selection workspaces);
 * 0 for an invalid shape. */
size_t dsa_host_pipeline_workspace_size(dsa_dtype dt, int B, int H, int N, int D, int block,
                                        int chunk_heads);

/*
 * Dense probability rows from the exact block masses of a CSR mask, so that
 * dsa_select_topp can select on exact attention weights (GSRS abstract:
 * Top-p selection supported by exact attention weights computed within the
 * FlashAttention pass; Figure 4: later searches evaluate only the blocks of
 * the candidate mask).
 *
 *   probs[r, j] = mass[s]  for every slot s of row r with col_idx[s] = j,
 *   probs[r, j] = 0        for every other column j < nB.
 *
 *   row_ptr, col_idx   device, int32: the CSR mask over `rows` rows (any
 *                      column order, no repeated column within a row).
 *   mass      device, fp32 [nnz], aligned with col_idx (dsa_block_mass's
 *             output; over a row the masses sum to 1).
 *   rows, nB  rows >= 1, 1 <= nB <= DSA_MAX_BLOCKS.
 *   probs     device out, fp32 [rows, nB].
 * Passing probs with the same CSR as candidates to dsa_select_topp keeps
 * the shortest prefix of each row's blocks, by exact mass, reaching p.
 * Errors: DSA_ERR_INVALID_ARG for null or misaligned pointers and bad
 * sizes; a column index outside [0, nB) or a decreasing row_ptr sets the
 * device error word (dsa_device_status) and that slot or row is skipped.
 */
dsa_status dsa_mass_to_probs(const int32_t* row_ptr, const int32_t* col_idx, const float* mass,
                             int rows, int nB, float* probs, void* stream);

/*
 * Token order along a 3-D Hilbert curve (GSRS Figure 6: a block then holds
 * the tokens of a compact spatio-temporal region instead of a flat slab;
 * Figures 1 and 3 and the DFSAttn abstract reorder tokens along Hilbert
 * curves).  Host function, no device work.
 *
 *   perm[i] = the original index of the token placed at position i.
 *   The text prefix keeps positions 0 .. n_prefix-1; grid token (t, y, x),
 *   original index n_prefix + (t*H + y)*W + x, is placed by its index along
 *   the Hilbert curve of the enclosing cube of side 2^bits (Skilling's
 *   axes-to-transpose method, t the most significant axis); cells outside
 *   the grid are skipped.
 *
 *   perm   host out, int32 [n_prefix + T*H*W].
 * Errors: DSA_ERR_INVALID_ARG for a null perm, T, H or W < 1, n_prefix < 0,
 * a side above 2^20 or more than 2^31 - 1 tokens.
 */
dsa_status dsa_hilbert_order(int T, int H, int W, int n_prefix, int32_t* perm);

/*
 * Token order along a generalised Hilbert curve of the T x H x W grid itself
 * (GSRS Figure 6: blocks along a Gilbert curve, the Hilbert curve extended
 * to boxes of any size).  Host function, no device work.  Same perm
 * convention and prefix rule as dsa_hilbert_order, but every two
 * consecutive grid tokens are grid neighbours (one step in t, y or x), also
 * on grids that are not power-of-two cubes.
 *
 * Construction (the pages give none): Hilbert's recursion on the box.  A
 * walk of an a x b x c box runs from a corner to the corner a - 1 cells
 * away along its first edge; it exists iff the box is one cell or a >= 2
 * and not (a odd and b*c even).  The longest edge is split near its middle
 * -- two boxes in a row along the travel edge, or a U-turn along another
 * edge (two one-cell slabs when the travel edge is 2 long) -- at the first
 * point, nearest the middle, whose parts all have walks.  The whole grid
 * is walked from (0, 0, 0) along its longest edge that admits a walk.
 *
 *   perm       host, int32 [n_prefix + T*H*W].
 * Errors: DSA_ERR_INVALID_ARG for null perm, non-positive sizes, a side
 * above 2^20 or more than 2^31 - 1 tokens.
 */
dsa_status dsa_gilbert_order(int T, int H, int W, int n_prefix, int32_t* perm);

/*
 * Reorders whole token rows of a [B, H, N, D] tensor by a permutation of N:
 *   inverse = 0 (gather):  dst[b, h, i, :] = src[b, h, perm[i], :]
 *   inverse = 1 (scatter): dst[b, h, perm[i], :] = src[b, h, i, :]
 * so gathering Q, K, V with dsa_hilbert_order's perm, running the pipeline
 * and scattering O gives the attention of the original token order with
 * blocks drawn along the curve.
 *
 *   src, dst   device, contiguous [B, H, N, D], distinct, 16-byte aligned.
 *   perm       device, int32 [N], a permutation of 0 .. N-1.
 * Errors: DSA_ERR_INVALID_ARG for null, aliased or misaligned pointers, an
 * unknown dtype, D not in {64, 128} or B, H, N < 1; an entry of perm
 * outside [0, N) sets the device error word (dsa_device_status) and that
 * row is not copied.
 */
dsa_status dsa_permute_tokens(const void* src, void* dst, dsa_dtype dt, int B, int H, int N, int D,
                              const int32_t* perm, int inverse, void* stream);

/* Largest `rows` that dsa_select_topp_static accepts. */
#define DSA_STATIC_MAX_ROWS 32768

/*
 * dsa_select_topp without a workspace argument.  (No counterpart in the
 * papers: this is a calling convention of this library.)
 *
 * For callers that cannot allocate device memory when they call in -- a
 * host that gives a plugin only its input and output buffers, a service
 * whose device memory all lives in its own pre-sized pool, a loop that must
 * not call cudaMalloc or cudaFree because they can synchronise the device.
 * Same arguments and results as dsa_select_topp, minus the workspace: the
 * scratch (selection bitmaps and counts) is a fixed array inside the
 * library, DSA_STATIC_MAX_ROWS * 33 words (about 4.3 MB), which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * nothing.
 *
 *  - rows > DSA_STATIC_MAX_ROWS returns DSA_ERR_INVALID_ARG (use
 *    dsa_select_topp with a workspace instead).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls on a device share the one array.  Calls that may overlap on
 *    the GPU (different streams, or several host threads) race on it and can
 *    return wrong lists; order them on one stream or serialise them.  Each
 *    call overwrites every scratch word it later reads, so nothing needs
 *    clearing between calls.
 */
dsa_status dsa_select_topp_static(const float* probs, int rows, int nB, float p,
                                  const int32_t* cand_row_ptr, const int32_t* cand_col,
                                  int32_t* row_ptr, int32_t* col_idx, void* stream);

/*
 * Failure-detection self-test.  (No counterpart in the papers: it checks
 * that this library's kernels report a stall instead of hanging.)
 * Launches one CTA on `stream` that waits, with a limit of `limit_ns`
 * nanoseconds, on a shared-memory mbarrier that nothing ever arrives at --
 * the same bounded wait every tensor-core kernel of the library uses -- so
 * the wait runs out, the kernel records a wait timeout in the device error
 * word and returns.  It copies nothing, issues no MMA and
 * holds no tensor memory.  After it, dsa_device_status returns
 * DSA_ERR_DEVICE with "wait-timeout" in dsa_last_error, and the device
 * stays usable.
 *
 *   limit_ns   1000 .. 1e9 (the library's own limit for one wait).
 * Errors: DSA_ERR_INVALID_ARG for a limit outside that range.
 */
dsa_status dsa_selftest_wait_timeout(unsigned long long limit_ns, void* stream);

/*
 * Self-test of the attention softmax's FMA-pipe exponential (a build-time
 * option, off by default: exponentials then all run on the MUFU).
 * (No counterpart in the papers: GSRS's abstract computes the exact softmax
 * weights; this checks the arithmetic that may produce them.)
 * y[i] = 2^x[i] by the same device function the attention kernel uses:
 * Cody-Waite reduction x = j + r, j = round(x), |r| <= 1/2; 2^r by a
 * degree-4 polynomial of least maximum relative error on [-1/2, 1/2]
 * (Remez exchange); 2^j added to the exponent field.  x is first clamped to
 * [-126, 127].  Relative error below 3e-6 over that range (about 25 units in
 * the last place of fp32, far below the 2^-9 of the bf16 P it feeds).
 *
 *   x, y   device, fp32 [n], 4-byte aligned; y is written, x is not.
 *   n      >= 0.
 * Asynchronous on `stream`.  Errors: DSA_ERR_INVALID_ARG for n < 0 or a null
 * or misaligned pointer with n > 0.
 */
dsa_status dsa_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * Synchronises `stream`, then reads and clears the library's device-side
 * error word.  Returns DSA_OK, DSA_ERR_DEVICE (details in dsa_last_error)
 * or DSA_ERR_CUDA.
 */
dsa_status dsa_device_status(void* stream);

/* Text of the last error on this host thread ("" if none). */
const char* dsa_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
