/*
 * calibatt.h -- C ABI of libcalibatt, the B200 (sm_100a) hot path of
 * CalibAtt (Calibrated Sparse Attention).
 *
 * Method: "Accelerating Text-to-Video Generation with Calibrated Sparse
 * Attention" (Yehezkel et al., arXiv 2603.05503). Passages are cited by the
 * zhichai.net explainer page of that paper ("explainer") and its sections:
 *   §二  observations (B x B blocks with B = 128; repetition across rows),
 *   §三  method: offline calibration (block energy, greedy eps selection,
 *        rho aggregation, eps(t) schedule) and online inference (skip list
 *        for non-repeated heads, k = 5 anchor rows for repeated heads),
 *   §六  spatial repetition (row-major tokens within an H x W frame).
 *
 * Conventions (all entry points):
 *  - Return value: CALIBATT_OK (0) or a negative calibatt_status code. Argument
 *    errors are detected on the host before anything is enqueued; nothing is
 *    launched when a call returns an error.
 *  - Device pointers are caller-owned device memory; host pointers are marked
 *    "host". The library never frees what it is given and keeps no pointer
 *    after a call returns.
 *  - Work is enqueued on the caller's stream (a cudaStream_t; NULL = legacy
 *    default stream). No entry point synchronises except calibatt_get_status.
 *  - Faults detected inside a kernel (a malformed skip list, a bounded wait
 *    that ran out) are recorded in a device status word; read and clear it
 *    with calibatt_get_status. Kernels never trap.
 *  - Tensors are contiguous, row-major: q, k, v, o are bf16 [heads][n][128]
 *    (d = 128 is the only supported head size), lse is fp32 [heads][n].
 *    Device pointers to bf16 tensors must be 16-byte aligned.
 *  - Blocks are B = 128 tokens of the flattened sequence (explainer §二):
 *    nb = ceil(n / 128); a ragged last block is padded and masked.
 *  - Token order: t = f*H*W + r*W + c (explainer §六).
 */
#ifndef CALIBATT_H_
#define CALIBATT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t calibatt_bf16;          /* bf16 bit pattern */
typedef struct CUstream_st* calibatt_stream_t; /* same handle as cudaStream_t */

typedef enum calibatt_status {
  CALIBATT_OK = 0,
  CALIBATT_ERR_ARG = -1,         /* null pointer, bad size or count, short workspace */
  CALIBATT_ERR_CSR = -2,         /* malformed skip list (row_ptr / col_idx) */
  CALIBATT_ERR_ALIGN = -3,       /* device pointer not 16-byte aligned */
  CALIBATT_ERR_UNSUPPORTED = -4, /* d != 128, or nb > 1024 for calibration */
  CALIBATT_ERR_CUDA = -5,        /* a CUDA runtime/driver call failed */
  CALIBATT_ERR_TIMEOUT = -6,     /* a bounded in-kernel wait ran out (device status) */
  CALIBATT_ERR_CAPACITY = -7     /* nnz exceeds the caller's col_idx capacity */
} calibatt_status;

#define CALIBATT_BLOCK 128
#define CALIBATT_HEAD_DIM 128
#define CALIBATT_MAX_CALIB_NB 1024

/* Text for a status code (static string, never NULL). */
const char* calibatt_strerror(int code);

/* Library ABI version (major*100 + minor). */
int calibatt_version(void);

/* Synchronises `stream`, then returns and clears the status word of the
 * current device (CALIBATT_OK if no kernel recorded a fault since the last
 * call). There is one word per device, not per stream: a fault recorded by a
 * kernel on any stream of the device is reported (and cleared) here, and when
 * several kernels fault only the first code is kept. Callers that need to
 * tell streams apart serialise their status checks. */
int calibatt_get_status(calibatt_stream_t stream);

/* Limit, in seconds, of every bounded in-kernel wait of the launches made
 * later on the current device (default 2 s; seconds <= 0 restores it; at most
 * 60). A pipeline wait that runs out makes the kernel wind down without
 * touching its outputs further and record CALIBATT_ERR_TIMEOUT for
 * calibatt_get_status; the GPU context stays usable. Waits that only drain
 * copies and tensor-core work already issued keep the default limit, so no
 * kernel exits with work in flight. A short limit is a test knob: it makes the
 * first wait that is not already satisfied run out.
 * Returns CALIBATT_ERR_ARG for NaN or > 60 s. */
int calibatt_set_wait_limit(double seconds);

/* ---------------------------------------------------------------- host helpers */

/* eps(t) = A + (C - A) * exp(-k t / T): the energy threshold schedule,
 * C at the early high-noise step, relaxing towards A (explainer §三). */
double calibatt_eps_schedule(double A, double C, double k, double t, double T);

/* Checks a host copy of a skip list: row_ptr [heads*nb + 1] non-decreasing
 * from 0 to nnz, every col_idx in [0, nb) and strictly ascending within a
 * row. Returns CALIBATT_OK or CALIBATT_ERR_CSR (CALIBATT_ERR_ARG on bad sizes). */
int calibatt_validate_csr(const int32_t* row_ptr, const int32_t* col_idx, int heads, int nb, int64_t nnz);

/* Tile-scheduler plan (host): the work units (h*nb + r) of the heads marked
 * active (all heads if head_active is NULL), head by head in index order and,
 * within a head, by kept-block count descending, ties by block index. Units
 * that run at the same time then mostly belong to one head and share its K/V
 * tiles in L2 (measured 6 % faster on the Wan-720p workload than one
 * longest-first order over all heads); the longest-first order inside a head
 * keeps the end of the launch short. Units with no kept block are included
 * (their rows get O = 0, LSE = -inf).
 * row_ptr: host [heads*nb + 1]; head_active: host [heads] or NULL;
 * work_list: host output with room for heads*nb entries; *n_work: count. */
int calibatt_build_plan(const int32_t* row_ptr, int heads, int nb, const uint8_t* head_active,
                        int32_t* work_list, int32_t* n_work);

/* Anchor rows of a repeated head: the centres of k equal bands of the H rows
 * of a frame, a_j = floor((2j + 1) H / (2k)), j = 0..k-1 (explainer §三,
 * "k = 5 anchor rows"; the pages do not fix the spacing, this is the plainest
 * even one). anchors: host [k]. Requires 1 <= k <= H. */
int calibatt_anchor_rows(int H, int k_anchor, int32_t* anchors);

/* Integer form of "mean mask >= rho" for n inputs: the smallest count c in
 * [0, n] with (double)c / n >= rho, or n + 1 if none (explainer §三). */
int calibatt_rho_threshold(int n_inputs, double rho, int32_t* threshold);

/* ---------------------------------------------------------------- inference */

/* Block-sparse attention over a calibrated skip list (explainer §三, online
 * inference for non-repeated heads; blocks of explainer §二).
 * For each work unit u = h*nb + r in work_list[0..n_work): query rows
 * [128r, min(128r+128, n)) of head h attend to the keys of the blocks
 * col_idx[row_ptr[u] .. row_ptr[u+1]) (keys >= n masked):
 *   O = softmax(scale * Q K^T) V,  lse = ln sum exp(scale * Q K^T).
 * A unit with no kept block gets O = 0 and lse = -inf. Rows of heads that no
 * unit names are not written.
 *   q, k, v : device bf16 [heads][n][128];  o : device bf16 [heads][n][128]
 *   row_ptr : device int32 [heads*nb + 1], global offsets into col_idx
 *   col_idx : device int32 [nnz], ascending within a row, values in [0, nb)
 *   work_list: device int32 [n_work] (from calibatt_build_plan)
 *   lse     : device fp32 [heads][n] or NULL
 * A malformed list is clamped in the kernel and reported as CALIBATT_ERR_CSR
 * through calibatt_get_status; validate host copies with calibatt_validate_csr. */
int calibatt_sparse_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v,
                             int heads, int n, int d, float scale, const int32_t* row_ptr,
                             const int32_t* col_idx, int64_t nnz, const int32_t* work_list, int32_t n_work,
                             calibatt_bf16* o, float* lse, calibatt_stream_t stream);

/* Workspace bytes needed by calibatt_repeat_attn_fwd (the packed anchor
 * queries): n_rep * frames * k_anchor * W * 128 * 2, rounded up to 256. */
size_t calibatt_repeat_workspace_size(int n_rep, int frames, int H, int W, int k_anchor);

/* Spatially repeated heads (explainer §三 online inference for repeated heads,
 * §六): for each head rep_heads[i], only the k anchor rows of every frame
 * (calibatt_anchor_rows) are computed, as dense attention of those queries
 * over all n = frames*H*W keys; every row r of a frame then receives, column
 * by column, the output (and lse) of its nearest anchor row (ties -> lower
 * anchor).
 *   rep_heads: device int32 [n_rep], head indices in [0, heads)
 *   ws       : device scratch of at least calibatt_repeat_workspace_size bytes
 * Other heads' rows are not written. */
int calibatt_repeat_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v,
                             int heads, int frames, int H, int W, int d, int k_anchor, float scale,
                             const int32_t* rep_heads, int32_t n_rep, calibatt_bf16* o, float* lse, void* ws,
                             size_t ws_bytes, calibatt_stream_t stream);

/* Lays a work list out (in place, host) for the persistent attention
 * kernel's static schedule so that its worker slots finish together. The
 * kernel runs G = 2 * min(n_slots / 2, ceil(n_work / 2)) slots and slot g
 * takes, in round t, entry t*G + g (t even) or t*G + G-1-g (t odd). Each
 * round's G entries stay in that round (so units that run together keep the
 * list's order: one head at a time), but are matched to the slots: the
 * costliest unit to the slot with the least work so far. Cost of a unit: its
 * kept blocks + 2 (a unit code >= heads*nb, an anchor-query unit of a
 * repeated head: nb + 2). Measured on B200 against the unbalanced lists of
 * calibatt_build_mixed_plan: Wan-480p 14.8 % faster, Mochi 6.9 %, Wan-720p
 * 2.1 %; the output is bit for bit the same (each unit is computed alone).
 *   work_list   : host int32 [n_work], reordered in place
 *   row_ptr     : host int32 [heads*nb + 1] (the skip list of the plan)
 *   n_slots     : worker slots, two per SM; <= 0: two per SM of the current
 *                 device (CALIBATT_ERR_CUDA if there is none)
 * A permutation of the list: any order gives the same results. */
int calibatt_balance_plan(int32_t* work_list, int32_t n_work, const int32_t* row_ptr, int heads, int nb,
                          int n_slots);

/* calibatt_balance_plan for a work list of calibatt_mixed_masked_attn_fwd:
 * the cost of an anchor-query unit is its kept blocks in the anchor skip list
 * row_ptr_b (host int32 [n_rep * ceil(frames*k_anchor*W / 128) + 1]) instead
 * of every key block; row_ptr_b may be NULL when n_rep = 0. Same layout rule
 * and result guarantees as calibatt_balance_plan. */
int calibatt_balance_mixed_plan(int32_t* work_list, int32_t n_work, const int32_t* row_ptr, int heads, int nb,
                                const int32_t* row_ptr_b, int n_rep, int frames, int W, int k_anchor, int n_slots);

/* Work list for calibatt_mixed_attn_fwd: first the anchor-query units of the
 * repeated heads, ceil(frames*k_anchor*W / 128) per head rep_heads[i] (codes
 * heads*nb + i*ceil(..) + b, each taking every key block), then head by head
 * as in calibatt_build_plan the block-sparse units h*nb + r of every other
 * head with head_active[h] != 0 (every other head if NULL), longest first
 * within a head (row_ptr: host int32 [heads*nb + 1]). Measured on the
 * Wan-720p workload: as fast as the two separate calls, while placing the
 * repeated heads among the others in head order was 8 % slower.
 *   rep_heads: host int32 [n_rep], distinct, in [0, heads)
 *   work_list: host int32 with room for heads*nb + n_rep*ceil(..) entries */
int calibatt_build_mixed_plan(const int32_t* row_ptr, int heads, int nb, const uint8_t* head_active, int n_rep,
                              const int32_t* rep_heads, int frames, int H, int W, int k_anchor, int32_t* work_list,
                              int32_t* n_work);

/* One attention call with both kinds of heads (explainer §三 online
 * inference): block-sparse heads over their skip lists as in
 * calibatt_sparse_attn_fwd and the n_rep repeated heads rep_heads as in
 * calibatt_repeat_attn_fwd, in one persistent launch that follows work_list
 * (calibatt_build_mixed_plan), after the gather of the anchor queries into ws.
 * The repeated heads' skip-list rows are not read; only heads named in the
 * work list are written. Arguments as in the two calls above;
 * ws: calibatt_repeat_workspace_size(n_rep, ...) bytes (unused if n_rep = 0). */
int calibatt_mixed_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v, int heads,
                            int frames, int H, int W, int d, int k_anchor, float scale, const int32_t* row_ptr,
                            const int32_t* col_idx, int64_t nnz, const int32_t* rep_heads, int32_t n_rep,
                            const int32_t* work_list, int32_t n_work, calibatt_bf16* o, float* lse, void* ws,
                            size_t ws_bytes, calibatt_stream_t stream);

/* calibatt_mixed_attn_fwd with a block mask on the repeated heads' anchor
 * rows (explainer §三 makes both run-time decisions per (t, l, h): a head's
 * skip list and its spatial repetition; the pages do not combine them, and
 * this call applies both): the anchor queries of repeated head rep_heads[i],
 * taken frame by frame (packed row f*k*W + j*W + c is token
 * f*H*W + a_j*W + c) and grouped into blocks of 128, attend only to the key
 * blocks of their block's row in the anchor skip list; every row still takes
 * its nearest anchor row's output. An anchor block with no kept block gives
 * O = 0 and lse = -inf to every row it feeds.
 *   row_ptr_b : device int32 [n_rep * ceil(frames*k_anchor*W / 128) + 1],
 *               global offsets into col_idx_b (rows of repeated head i start
 *               at i * ceil(frames*k_anchor*W / 128))
 *   col_idx_b : device int32 [nnz_b], ascending within a row, in [0, nb)
 * Calibrate it with calibatt_anchor_block_energy and
 * calibatt_aggregate_mask_rows. Other arguments as in
 * calibatt_mixed_attn_fwd (work list from calibatt_build_mixed_plan, laid out
 * by calibatt_balance_mixed_plan); a malformed anchor list is clamped and
 * reported as CALIBATT_ERR_CSR through calibatt_get_status. */
int calibatt_mixed_masked_attn_fwd(const calibatt_bf16* q, const calibatt_bf16* k, const calibatt_bf16* v,
                                   int heads, int frames, int H, int W, int d, int k_anchor, float scale,
                                   const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz,
                                   const int32_t* rep_heads, int32_t n_rep, const int32_t* row_ptr_b,
                                   const int32_t* col_idx_b, int64_t nnz_b, const int32_t* work_list, int32_t n_work,
                                   calibatt_bf16* o, float* lse, void* ws, size_t ws_bytes,
                                   calibatt_stream_t stream);

/* Head sharding of one attention call over n_ranks GPUs (host). A head's
 * output depends only on its own q, k, v, so ranks need no exchange; the
 * work is balanced by kept tiles (a block-sparse head: its kept blocks; a
 * repeated head: ceil(frames*k_anchor*W / 128) anchor blocks x nb): heads in
 * descending cost (ties: lower head first), each to the least-loaded rank
 * (ties: lower rank). Each rank then builds its work list with
 * calibatt_build_mixed_plan, head_active[h] = (owner[h] == rank), and its
 * own repeated heads.
 *   row_ptr_host : host int32 [heads*nb + 1]; rep_heads_host: host int32 [n_rep]
 *   owner        : host int32 [heads] (output: rank of each head)
 *   load         : host int64 [n_ranks] (output: kept tiles per rank) or NULL */
int calibatt_shard_heads(const int32_t* row_ptr_host, int heads, int nb, const int32_t* rep_heads_host, int n_rep,
                         int frames, int W, int k_anchor, int n_ranks, int32_t* owner, int64_t* load);

/* Device workspace bytes of calibatt_mixed_attn_fwd_host (anchor queries of
 * one chunk plus every chunk's work list); heads_per_chunk <= 0 means 2. */
size_t calibatt_mixed_host_workspace_size(int heads, int frames, int H, int W, int k_anchor, int n_rep,
                                          int heads_per_chunk);

/* calibatt_mixed_attn_fwd on host buffers, pipelined over chunks of
 * heads_per_chunk heads (<= 0: 2; on the Wan-720p workload 2 heads per chunk
 * measured best of 2, 3, 4, 5, 8 and 20): while the attention of chunk c runs on
 * `stream`, q, k, v of chunk c+1 are copied in on a second stream and o (and
 * lse) of chunk c-1 copied out on a third, so copies and compute overlap. The
 * first chunk holds ceil(heads_per_chunk / 2) heads, so that the copy-in
 * that nothing overlaps is short. Odd chunks run their attention on a fourth
 * stream (with their own anchor buffer), so that a chunk's launch can start
 * on the SMs that the previous chunk's last units leave idle.
 * Returns once everything is enqueued; the results are in o_host (lse_host)
 * when `stream` completes. Use page-locked host memory, else the copies do not
 * overlap. The skip list, work lists and repeated heads are those of
 * calibatt_mixed_attn_fwd; the work list of each chunk is built here from
 * row_ptr_host (calibatt_build_mixed_plan, then calibatt_balance_plan). Of a repeated head's q only the anchor pixel rows are copied
 * (its other rows of q_dev are neither read nor written): the in-copy per step
 * is 3*heads*n*256 bytes less n_rep*frames*(H - k_anchor)*W*256.
 *   q_host, k_host, v_host : host bf16 [heads][n][128]; o_host: host bf16 (output)
 *   lse_host  : host fp32 [heads][n] or NULL (then lse_dev may be NULL)
 *   row_ptr_host : host int32 [heads*nb + 1]; row_ptr, col_idx: the same list on the device
 *   rep_heads_host : host int32 [n_rep]
 *   q_dev, k_dev, v_dev, o_dev, lse_dev : device buffers of the full tensors
 *   ws : device scratch of calibatt_mixed_host_workspace_size bytes
 * Calls for one device are serialised on a host lock while they enqueue. */
int calibatt_mixed_attn_fwd_host(const calibatt_bf16* q_host, const calibatt_bf16* k_host,
                                 const calibatt_bf16* v_host, calibatt_bf16* o_host, float* lse_host, int heads,
                                 int frames, int H, int W, int d, int k_anchor, float scale,
                                 const int32_t* row_ptr_host, const int32_t* row_ptr, const int32_t* col_idx,
                                 int64_t nnz, const int32_t* rep_heads_host, int32_t n_rep, int heads_per_chunk,
                                 calibatt_bf16* q_dev, calibatt_bf16* k_dev, calibatt_bf16* v_dev,
                                 calibatt_bf16* o_dev, float* lse_dev, void* ws, size_t ws_bytes,
                                 calibatt_stream_t stream);

/* ---------------------------------------------------------------- calibration */

/* Block energy of one calibration input (explainer §三 offline calibration,
 * steps 1-2): with P = softmax(scale * Q K^T) over all n keys,
 *   E[h][r][c] = (1 / |I_r|) * sum_{i in block r, j in block c} P_ij,
 * |I_r| the query rows present in block r (128 except a ragged last block,
 * which keeps every row sum at 1). P is never stored: a first pass writes the
 * row log-sum-exp to lse_ws, a second recomputes S and reduces exp(S - lse)
 * tile by tile.
 * When fuse_select != 0 the same kernel applies the greedy selection of
 * calibatt_select_mask at `eps` to each finished energy row and writes mask
 * and/or kept and/or tie and/or adds the mask into counts.
 *   lse_ws : device fp32 scratch [heads][nb*128]
 *   energy : device fp32 [heads][nb][nb] or NULL
 *   mask   : device uint8 [heads][nb][nb] or NULL; kept: device int32 [heads][nb] or NULL
 *   counts : device uint16 [heads][nb][nb] or NULL (counts += mask)
 *   tie, tie_window : as in calibatt_select_mask
 * Requires nb <= CALIBATT_MAX_CALIB_NB. */
int calibatt_block_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int n, int d, float scale,
                          float* lse_ws, float* energy, int fuse_select, double eps, uint8_t* mask,
                          int32_t* kept, uint16_t* counts, uint8_t* tie, double tie_window,
                          calibatt_stream_t stream);

/* Workspace bytes of calibatt_block_energy_1pass for heads x n tokens on the
 * current device (it depends on the number of SMs; 0 on bad sizes). */
size_t calibatt_energy_workspace_size(int heads, int n);

/* calibatt_block_energy in one pass over the keys instead of two: each query
 * row keeps its exact running max m and running sum, and stores its key
 * blocks' sums of 2^(scale' s - m) in ws, eight key blocks at a time, all
 * relative to the m reached at the eighth (36 bytes per row and eight key
 * blocks); once the row's log-sum-exp is known the stored sums are rescaled
 * and reduced into the same energies
 * (and fused selection) as calibatt_block_energy, which computes S twice.
 * With pix_energy != NULL it also writes the profiles of
 * calibatt_pixel_row_energy for pixel rows of pix_W consecutive queries
 * (pix_energy: device fp32 [heads][n / pix_W][nb], cleared first; pix_W must
 * divide n).
 *   ws : device scratch of calibatt_energy_workspace_size(heads, n) bytes,
 *        16-byte aligned (no lse_ws is needed)
 * Other arguments and outputs as in calibatt_block_energy. */
int calibatt_block_energy_1pass(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int n, int d,
                                float scale, void* ws, size_t ws_bytes, float* energy, int fuse_select, double eps,
                                uint8_t* mask, int32_t* kept, uint16_t* counts, uint8_t* tie, double tie_window,
                                float* pix_energy, int pix_W, calibatt_stream_t stream);

/* Device workspace bytes of calibatt_anchor_block_energy (0 on bad sizes). */
size_t calibatt_anchor_energy_workspace_size(int heads, int n_rep, int frames, int H, int W, int k_anchor);

/* Block energies of the repeated heads' anchor queries (the calibration of
 * the anchor-row masks of calibatt_mixed_masked_attn_fwd; explainer §三 step
 * 2, taken over anchor queries): the anchor queries of head rep_heads[i],
 * packed frame by frame as in calibatt_mixed_masked_attn_fwd and grouped into
 * nbq = ceil(frames*k_anchor*W / 128) blocks, against every key block of the
 * head, in one pass over the keys:
 *   E[i][r][c] = (1 / |I_r|) * sum_{a in packed block r, j in block c} P_aj,
 * P = softmax(scale * Q K^T) over all n keys. With fuse_select, the greedy
 * selection of calibatt_select_mask at eps runs on every finished row.
 *   rep_heads : device int32 [n_rep], in [0, heads)
 *   ws        : device scratch of calibatt_anchor_energy_workspace_size bytes,
 *               16-byte aligned (the packed queries, then the pass's sums)
 *   energy    : device fp32 [n_rep][nbq][nb] or NULL
 *   mask, kept, counts, tie : as in calibatt_block_energy, with n_rep*nbq rows
 * Requires nb <= CALIBATT_MAX_CALIB_NB. */
int calibatt_anchor_block_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int frames, int H, int W,
                                 int d, int k_anchor, float scale, const int32_t* rep_heads, int32_t n_rep, void* ws,
                                 size_t ws_bytes, float* energy, int fuse_select, double eps, uint8_t* mask,
                                 int32_t* kept, uint16_t* counts, uint8_t* tie, double tie_window,
                                 calibatt_stream_t stream);

/* Greedy eps selection (explainer §三, step 3) on rows of block energies:
 * order the row's blocks by energy descending (equal energies: lower column
 * first) and keep the shortest prefix whose running sum reaches eps. The sum
 * is exact: each fp32 energy is taken in fixed point with 50 fraction bits
 * (truncated), so the result does not depend on summation order. If no prefix
 * reaches eps, every block with nonzero energy is kept; at least one block is
 * always kept. Energies are clamped to [0, 4] (NaN -> 0).
 *   energy : device fp32 [rows][nb], rows = heads*nb
 *   mask   : device uint8 [rows][nb] or NULL; kept: device int32 [rows] or NULL
 *   counts : device uint16 [rows][nb] or NULL (counts += mask)
 *   tie    : device uint8 [rows] or NULL: 1 where the row's decision is
 *            tie-affected at tie_window: the running sum with or without the
 *            last kept block (in greedy order) lies within tie_window of eps,
 *            or the last kept block's energy exceeds the next block's by less
 *            than tie_window (the next block in greedy order; none when every
 *            block is kept). Such decisions can flip under a perturbation of
 *            the energies of that size; the benchmark counts them at 1e-6.
 *   tie_window : >= 0 (0: no row is flagged); ignored when tie is NULL
 * Requires nb <= CALIBATT_MAX_CALIB_NB. */
int calibatt_select_mask(const float* energy, int heads, int nb, double eps, uint8_t* mask, int32_t* kept,
                         uint16_t* counts, uint8_t* tie, double tie_window, calibatt_stream_t stream);

/* counts[i] += mask[i] (saturating at 65535) for `cells` entries: folds one
 * calibration input's mask into the running sum over inputs (explainer §三). */
int calibatt_accumulate_masks(const uint8_t* mask, int64_t cells, uint16_t* counts, calibatt_stream_t stream);

/* Workspace bytes needed by calibatt_aggregate_masks. */
size_t calibatt_aggregate_workspace_size(int heads, int nb);

/* Aggregation and skip-list build (explainer §三): keep block (h, r, c) where
 * counts / n_inputs >= rho (in integers: counts >= calibatt_rho_threshold),
 * write the binary mask and its CSR skip list with global offsets, columns
 * ascending.
 *   counts  : device uint16 [heads][nb][nb]
 *   mask    : device uint8 [heads][nb][nb] (output)
 *   row_ptr : device int32 [heads*nb + 1] (output)
 *   col_idx : device int32 [nnz_cap] (output)
 *   nnz     : device int64 [1] (output: total kept blocks)
 *   ws      : device scratch of calibatt_aggregate_workspace_size bytes
 * If the kept total exceeds nnz_cap, col_idx holds the first nnz_cap entries
 * and calibatt_get_status reports CALIBATT_ERR_CAPACITY. */
int calibatt_aggregate_masks(const uint16_t* counts, int n_inputs, int heads, int nb, double rho, uint8_t* mask,
                             int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap, int64_t* nnz, void* ws,
                             size_t ws_bytes, calibatt_stream_t stream);

/* Workspace bytes needed by calibatt_aggregate_mask_rows for `rows` rows. */
size_t calibatt_aggregate_rows_workspace_size(int64_t rows);

/* calibatt_aggregate_masks for any number of mask rows of `cols` columns
 * (for example the n_rep * nbq anchor rows of calibatt_anchor_block_energy):
 * keep cell (r, c) where counts[r][c] / n_inputs >= rho, and build the CSR
 * skip list of the rows (row_ptr [rows + 1], global offsets, columns
 * ascending). Outputs, capacity and errors as in calibatt_aggregate_masks. */
int calibatt_aggregate_mask_rows(const uint16_t* counts, int n_inputs, int64_t rows, int cols, double rho,
                                 uint8_t* mask, int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap, int64_t* nnz,
                                 void* ws, size_t ws_bytes, calibatt_stream_t stream);

/* ---------------------------------------------------------------- spatial repetition */

/* Largest frame height H accepted by calibatt_spatial_score. */
#define CALIBATT_MAX_FRAME_ROWS 512

/* Block-energy profiles of pixel rows (explainer §二 observation 4 and §六:
 * the pixel rows of a frame attend alike; §三: the spatial similarity score
 * is computed per head at calibration). Tokens are frame-major, row-major
 * inside a frame (token = f*H*W + r*W + c, n = frames*H*W); pixel row
 * R = f*H + r holds W queries. With P = softmax(scale * Q K^T) over all n keys,
 *   pix_energy[h][R][c] = (1 / W) * sum_{i in pixel row R, j in key block c} P_ij.
 * Two passes as in calibatt_block_energy: the first writes the row
 * log-sum-exp to lse_ws, the second recomputes S; when `energy` is not NULL
 * that pass also writes the block energies of calibatt_block_energy (no
 * selection). pix_energy is cleared first and then accumulated with fp32
 * atomics, so its last bits may differ between runs.
 *   lse_ws     : device fp32 scratch [heads][nb*128]
 *   energy     : device fp32 [heads][nb][nb] or NULL
 *   pix_energy : device fp32 [heads][frames*H][nb] (output)
 * Requires nb <= CALIBATT_MAX_CALIB_NB. */
int calibatt_pixel_row_energy(const calibatt_bf16* q, const calibatt_bf16* k, int heads, int frames, int H,
                              int W, int d, float scale, float* lse_ws, float* energy, float* pix_energy,
                              calibatt_stream_t stream);

/* Spatial similarity score of each head (explainer §三: a head is marked
 * spatially repeated when its score exceeds gamma = 0.87; the pages give no
 * formula). Reading used: the mean, over every frame and every pixel row r
 * that is not an anchor row, of the cosine similarity between the profile of
 * row r and the profile of its nearest anchor row (calibatt_anchor_rows; ties
 * -> lower anchor), i.e. the row whose output a repeated head copies to r.
 * A cosine with an all-zero profile counts as 0; with k_anchor = H the score
 * is 1.
 *   pix_energy : device fp32 [heads][frames*H][nb] (calibatt_pixel_row_energy)
 *   score      : device fp32 [heads] (output)
 *   flag       : device uint8 [heads] or NULL (output: score > gamma)
 * Requires 1 <= k_anchor <= H <= CALIBATT_MAX_FRAME_ROWS. */
int calibatt_spatial_score(const float* pix_energy, int heads, int frames, int H, int nb, int k_anchor,
                           float gamma, float* score, uint8_t* flag, calibatt_stream_t stream);

/* ---------------------------------------------------------------- calibration bank */

/* Keep-rate histogram of calibrated blocks (explainer §二 observation 3: over
 * the calibration inputs most blocks are kept by almost all of them or by
 * almost none, a bimodal histogram of count / n): for each head,
 * hist[h][c] = number of blocks kept by exactly c of the n_inputs inputs.
 *   counts : device uint16 [heads][cells] (calibatt_accumulate_masks or the
 *            fused selection of calibatt_block_energy)
 *   hist   : device int64 [heads][n_inputs + 1] (output; cleared first)
 * Counts above n_inputs go to the last bin and are reported through
 * calibatt_get_status as CALIBATT_ERR_ARG. Requires n_inputs <= 4096. */
int calibatt_keep_histogram(const uint16_t* counts, int heads, int64_t cells, int n_inputs, int64_t* hist,
                            calibatt_stream_t stream);

/* The (t, l) mask bank read by online inference (explainer §三: calibration
 * runs once offline; online, each step looks up the skip list or the repeat
 * marks of its (t, l, h) with no decision at run time). A bank is a host-side
 * index over device memory the caller owns: calibatt_bank_put copies one
 * entry (skip list, work list, repeated heads) into a caller buffer of
 * calibatt_bank_entry_bytes and records where it is; calibatt_bank_get hands
 * the device pointers back for calibatt_mixed_attn_fwd. Keep each entry's
 * buffer alive while the bank is used. */
typedef struct calibatt_bank calibatt_bank;

typedef struct calibatt_bank_entry {
  const int32_t* row_ptr;   /* device int32 [heads*nb + 1] */
  const int32_t* col_idx;   /* device int32 [nnz] */
  int64_t nnz;
  const int32_t* work_list; /* device int32 [n_work] (calibatt_build_mixed_plan order) */
  int32_t n_work;
  const int32_t* rep_heads; /* device int32 [n_rep] */
  int32_t n_rep;
  double eps;               /* energy threshold of the calibration, eps(t) */
} calibatt_bank_entry;

/* A bank of timesteps x layers entries for heads heads of frames x H x W
 * tokens and k_anchor anchor rows; NULL on bad sizes or no host memory. */
calibatt_bank* calibatt_bank_create(int timesteps, int layers, int heads, int frames, int H, int W, int k_anchor);
void calibatt_bank_destroy(calibatt_bank* bank);

/* Device bytes of one entry with nnz kept blocks and n_rep repeated heads
 * (0 on bad arguments). */
size_t calibatt_bank_entry_bytes(const calibatt_bank* bank, int64_t nnz, int n_rep);

/* Stores entry (t, l), calibrated at eps, replacing any earlier one: copies
 * row_ptr (host int32 [heads*nb + 1]), col_idx (device int32 [nnz]) and
 * rep_heads (host int32 [n_rep]) into dst, with the work list that
 * calibatt_build_mixed_plan makes of them, laid out by calibatt_balance_plan
 * for the current device, on `stream`.
 *   dst: device buffer of at least calibatt_bank_entry_bytes, 256-byte aligned
 * Returns CALIBATT_ERR_CSR if row_ptr does not run from 0 to nnz. */
int calibatt_bank_put(calibatt_bank* bank, int t, int l, double eps, const int32_t* row_ptr_host,
                      const int32_t* col_idx, int64_t nnz, const int32_t* rep_heads_host, int n_rep, void* dst,
                      size_t dst_bytes, calibatt_stream_t stream);

/* Entry (t, l) (host only; CALIBATT_ERR_ARG if it was never stored). */
int calibatt_bank_get(const calibatt_bank* bank, int t, int l, calibatt_bank_entry* out);

/* ---------------------------------------------------------------- no-allocation variant */

/* Largest heads * nb accepted by calibatt_aggregate_masks_noalloc. */
#define CALIBATT_NOALLOC_MAX_ROWS (1 << 18)

/* calibatt_aggregate_masks without a workspace argument. The method has no
 * counterpart for this: it exists for callers that cannot allocate device
 * memory when they build a skip list -- for example a plugin that only
 * receives pointers from a host engine whose allocator owns the GPU's memory,
 * or a serving loop under a fixed memory budget where an allocation could fail
 * or stall. Same arguments, outputs and errors as calibatt_aggregate_masks
 * (the caller still passes counts, mask, row_ptr, col_idx and nnz); the
 * aggregation's kept totals (one per span of the flat mask, at most one per
 * row) live in a static device array of CALIBATT_NOALLOC_MAX_ROWS int32
 * (1 MiB), held by every GPU that loads the library until exit.
 *  - Returns CALIBATT_ERR_ARG when heads * nb > CALIBATT_NOALLOC_MAX_ROWS.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture.
 *  - All calls share the array: calls whose kernels overlap on the GPU (for
 *    example on two streams at once) race and corrupt each other's results.
 *    Every total in it is rewritten by each call before it is read, so
 *    nothing needs clearing. */
int calibatt_aggregate_masks_noalloc(const uint16_t* counts, int n_inputs, int heads, int nb, double rho,
                                     uint8_t* mask, int32_t* row_ptr, int32_t* col_idx, int64_t nnz_cap,
                                     int64_t* nnz, calibatt_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CALIBATT_H_ */
