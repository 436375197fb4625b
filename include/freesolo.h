/*
 * freesolo.h - C ABI of the FreeSolo sparse-attention forward pass for NVIDIA B200 (sm_100a).
 *
 * The method ("FreeSolo" technical summary, section "Methodology") gives every attention
 * head two branches and adds them (§3.1, eq. (2)):
 *
 *     o_i = o_i^sr + alpha_h * o_i^lr
 *
 *   o_i^sr  (§3.2, eqs. (3)-(4)): softmax attention of the RoPE-rotated query over the keys
 *           j in L_i = [max(0, i-w), i] (look-back radius w), logits q.k/sqrt(d).
 *   o_i^lr  (§3.3, eqs. (5), (7)-(9)): the keys are cut into cells of s consecutive tokens;
 *           each cell c has a mean key kbar_c and a max key norm a_c (eq. (5)).  The
 *           candidates C_i are the cells lying wholly before the window, (c+1)s <= i-w.
 *           FS-L pruning (eq. (8)) keeps A_i = the W most recent candidates plus the P
 *           candidates of largest a_c.  Each cell of A_i is scored (eq. (7))
 *               r_ic = q_i.kbar_c/sqrt(d) + lambda_h a_c erf((i - p_c)/(2 sigma_h)),
 *           p_c = (c + 1/2)s, the K best form S_i, and o_i^lr = RMSNorm(u_i) where u_i is
 *           softmax attention of the unrotated query over every token of S_i (eq. (9)).
 *
 * Readings where the summary is silent: RoPE pairs are interleaved (2m, 2m+1) with
 * theta_m = base^(-2m/d); RMSNorm has no gain, u/sqrt(mean(u^2)+eps); ties in TopP and in
 * the top-K go to the lower cell index; |A_i| < K selects all of A_i; an empty S_i gives
 * o^lr = 0; W < 0 and P < 0 together mean no pruning (base FS, A_i = C_i).
 *
 * Layout: Q is [B, H, Nq, d]; K, V are [B, H, Nk, d]; O is [B, H, Nq, d]; all contiguous,
 * row-major, of type `dtype`.  Query row r has position Nk - Nq + r among the keys, so
 * Nq = Nk is a prefill and Nq < Nk appends Nq new tokens to an archive of Nk - Nq.
 * Cell summaries: kbar [B, H, C, d] and amax [B, H, C], float32, C = floor(Nk / s).
 * Selected cells: idx [B, H, Nq, K] int32, ascending, padded with -1.
 *
 * Ownership and errors: the caller owns every buffer; the library allocates nothing and
 * enqueues its kernels on `stream` (a cudaStream_t; NULL is the legacy default stream).
 * Pointers named d* / Q, K, V, O, kbar, amax, idx, ws are device pointers; the per-head
 * arrays alpha / lambda / sigma are HOST pointers read during the call.  Device arrays
 * start on a 16-byte boundary (as cudaMalloc and torch allocations do): the kernels read
 * and write them in 16-byte vectors and describe them to the tensor-memory-access unit.
 * Argument errors are returned before anything is enqueued.  No exception crosses the ABI.
 *
 * Supported: d = 64, s = 32, w a multiple of s, 0 <= K <= 64, W + P <= 2048,
 * 1 <= H <= 256; dtype bf16 or f32.  Anything else returns FS_ERR_UNSUPPORTED.
 */
#ifndef FREESOLO_H
#define FREESOLO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FS_OK = 0,
    FS_ERR_INVALID_ARG = 1,   /* NULL pointer, negative size, Nq > Nk, ... */
    FS_ERR_UNSUPPORTED = 2,   /* a size or option outside the supported set above */
    FS_ERR_WORKSPACE = 3,     /* workspace missing or smaller than fs_workspace_size() */
    FS_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed */
    FS_ERR_TIMEOUT = 5,       /* a kernel gave up a bounded wait (device error flag) */
    FS_ERR_KERNEL_CHECK = 6   /* a kernel's internal consistency check failed (device flag) */
} fs_status;

typedef enum { FS_BF16 = 0, FS_F32 = 1 } fs_dtype;

#define FS_MAX_HEADS 256

typedef struct {
    int B, H, Nq, Nk, d;   /* batch, heads, query rows, key rows, head dim */
    int w;                 /* look-back radius of the local branch (eq. (3)); L_i = [i-w, i] */
    int s;                 /* cell size in tokens (eq. (5)) */
    int K;                 /* cells kept per query (top-K of eq. (7)) */
    int W, P;              /* FS-L recent and norm budgets (eq. (8)); W < 0 && P < 0: off */
    float rope_base;       /* RoPE base, e.g. 10000 */
    const float *alpha;    /* host [H]: per-head weight of the long-range branch (eq. (2)) */
    const float *lambda;   /* host [H] or NULL (prior off): lambda_h >= 0 (eq. (7)) */
    const float *sigma;    /* host [H] or NULL: sigma_h > 0 (eq. (7)) */
    float rms_eps;         /* RMSNorm epsilon (eq. (9)), e.g. 1e-6 */
    fs_dtype dtype;        /* type of Q, K, V and O; summaries are always float32 */
} fs_params;

/* Bytes of device workspace the calls below need for these parameters (> 0).
 * The workspace's first bytes hold the device error flag read by fs_sync_status. */
fs_status fs_workspace_size(const fs_params *p, size_t *bytes);

/* Cell summaries, eq. (5): kbar [B,H,C,d] = mean key of each s-token cell, amax [B,H,C] =
 * the largest key norm in the cell.  Only whole cells (C = floor(Nk/s)) are summarised.
 * K is a device pointer of type p->dtype; kbar and amax are device float32 outputs. */
fs_status fs_cell_summaries(const fs_params *p, const void *K, float *kbar, float *amax,
                            void *stream);

/* Long-range selection, eqs. (7)-(8): for every query row, the K best cells of A_i by
 * r_ic, written to idx [B,H,Nq,K] (ascending, -1 padded).  kbar/amax are the summaries
 * of fs_cell_summaries (or the caller's own, same layout).  ws/ws_bytes: workspace. */
fs_status fs_select_topk(const fs_params *p, const void *Q, const float *kbar,
                         const float *amax, int32_t *idx, void *ws, size_t ws_bytes,
                         void *stream);

/* Token-level rerank of the selection ("FreeSolo" summary §3.4, eq. (12)): each cell of a
 * shortlist of A_i is rescored by
 *     rt_ic = log sum_{j in I_c} exp(q_i.k_j/sqrt(d)) + lambda_h a_c erf((i - p_c)/(2 sigma_h))
 * over its tokens' raw (unrotated) keys, and the K best form S_i, written to idx
 * [B,H,Nq,K] (ascending, -1 padded; ties go to the lower cell).  The shortlist is the
 * `shortlist` best cells of A_i by eq. (7), or all of A_i when shortlist = 0 (the summary
 * gives no size; with shortlist = K the set equals fs_select_topk's).  K is the keys array
 * [B,H,Nk,d] of type p->dtype; kbar/amax as for fs_select_topk.  The readout on these cells
 * is fs_forward with idx.  Requires |A_i| <= 128 (W + P <= 128, or without pruning
 * floor(Nk/s) <= 128), else FS_ERR_UNSUPPORTED; shortlist < 0 is FS_ERR_INVALID_ARG. */
fs_status fs_select_topk_rerank(const fs_params *p, const void *Q, const void *K, const float *kbar,
                                const float *amax, int shortlist, int32_t *idx, void *ws,
                                size_t ws_bytes, void *stream);

/* The forward pass with the eq. (12) rerank as its selection: fs_select_topk_rerank's
 * cells (shortlist as there), then the readout on them and the window, O = o^sr + alpha_h
 * o^lr.  kbar/amax may be NULL (computed here); idx, if not NULL, receives the selected
 * cells [B,H,Nq,K].  bf16 runs the fused tensor-core readout + window on the reranked
 * cells; f32 runs the CUDA-core readout.  Requirements as for fs_select_topk_rerank. */
fs_status fs_forward_rerank(const fs_params *p, const void *Q, const void *K, const void *V,
                            const float *kbar, const float *amax, int shortlist, int32_t *idx,
                            void *O, void *ws, size_t ws_bytes, void *stream);

/* The whole forward pass, eq. (2): O = o^sr + alpha_h o^lr.
 * kbar/amax may be NULL (then computed here into the workspace) or caller-given summaries
 * (e.g. an archive summarised once for decoding).  idx may be NULL (then selected here)
 * or caller-given cells, which skips eqs. (7)-(8) and runs the readout on them. */
fs_status fs_forward(const fs_params *p, const void *Q, const void *K, const void *V,
                     const float *kbar, const float *amax, const int32_t *idx, void *O,
                     void *ws, size_t ws_bytes, void *stream);

/* Bytes of device scratch fs_forward_host needs: device copies of Q, K, V, O plus the
 * workspace. */
fs_status fs_host_scratch_size(const fs_params *p, size_t *bytes);

/* fs_forward on HOST buffers hQ, hK, hV -> hO (pinned memory makes the copies async).
 * Copies in, computes and copies out using the caller's device scratch
 * (fs_host_scratch_size bytes), pipelined over chunks of heads: a chunk's inputs copy in
 * on an internal stream while the previous chunk computes on `stream` and the one before
 * copies out on another internal stream; `stream` waits for the last copy out.  Returns
 * after enqueueing; synchronize `stream` (or call fs_sync_status) before reading hO. */
fs_status fs_forward_host(const fs_params *p, const void *hQ, const void *hK, const void *hV,
                          void *hO, void *dscratch, size_t scratch_bytes, void *stream);

/* Synchronizes `stream`, then reads and clears the device error flag in `ws`.
 * Returns FS_ERR_TIMEOUT if a kernel gave up a bounded wait since the last check,
 * FS_ERR_KERNEL_CHECK if a kernel found its inputs inconsistent (e.g. more distinct
 * selected cells in a 128-row tile than the bound derived from W and P),
 * FS_ERR_CUDA if the stream reports an error, else FS_OK.
 * ws == NULL: the flag read and cleared is the status word of fs_select_topk_noalloc on
 * the current device (FS_OK without touching the GPU if that call never ran there). */
fs_status fs_sync_status(void *ws, void *stream);

/* Static description of a status code. */
const char *fs_status_string(fs_status s);

/* ---- selection without any device allocation (no counterpart in the method) ----
 * fs_select_topk_noalloc computes exactly what fs_select_topk computes, for callers that
 * cannot allocate device memory or hand the library a workspace: programs running inside
 * a fixed device-memory budget planned in advance, plugins whose host framework owns all
 * device allocations, and latency-critical loops where cudaMalloc/cudaFree would stall on
 * a device-wide synchronization.  Its one scratch buffer, the TopP exit table, is a
 * fixed array of FS_NOALLOC_MAX_CELLS ints (4 MiB) compiled into the library, beside a
 * one-int status word; every GPU that loads the library holds them until the process
 * exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 *   - With pruning on (W, P >= 0), B * H * floor(Nk / s) must not exceed
 *     FS_NOALLOC_MAX_CELLS, else FS_ERR_UNSUPPORTED is returned before anything runs.
 *   - Set-up: with the device current, the call looks up the array's device address (a
 *     host-side query).  It does so on every call made outside stream capture, so a device
 *     reset (cudaDeviceReset, which reloads the library's module) leaves nothing stale;
 *     inside a capture it reuses the address an earlier call on that device found.  So make
 *     the first call on a device, and the first call after a device reset, before any
 *     stream capture begins.
 *   - All calls on a device share the one array, which keeps the last call's contents
 *     (nothing in it has to start at zero: each call writes every entry it reads).  Calls
 *     that overlap on the GPU (different streams, or threads, without ordering between
 *     them) race on it; order them, e.g. by issuing them on one stream.
 *   - Device-side failures (a bounded wait that ran out, a failed consistency check:
 *     idx may then be partly unwritten) are recorded in the status word, which stays set
 *     until fs_sync_status(NULL, stream) reads and clears it (FS_ERR_TIMEOUT or
 *     FS_ERR_KERNEL_CHECK).
 * Arguments, layouts and the argument errors are those of fs_select_topk. */
#define FS_NOALLOC_MAX_CELLS (1 << 20)
fs_status fs_select_topk_noalloc(const fs_params *p, const void *Q, const float *kbar,
                                 const float *amax, int32_t *idx, void *stream);

/* ---- backward pass of eq. (2) ----
 * Gradients of O = o^sr + alpha_h RMSNorm(u) (eqs. (2)-(4), (9)) with respect to Q, K, V
 * and alpha, for an upstream gradient dO, with the selection held fixed: the cells idx
 * [B,H,Nq,K] the forward pass read (from fs_select_topk, or fs_forward_rerank's idx).  The
 * top-K is piecewise constant in Q and K, and the summaries only feed it, so neither
 * carries a gradient (reading; the summary gives no backward pass).
 *   window:  dv_j += p_j dO, dl_j = p_j (dO.v_j - dO.o^sr), through the RoPE rotations
 *   readout: du = r (dy - y (dy.y)/d) with y = u r, r = (mean(u^2)+eps)^(-1/2),
 *            dy = alpha_h dO; then the same softmax rule on NoPE logits
 *   dalpha_h = sum_i dO_i . y_i
 * Q, K, V, dO are device arrays of type p->dtype ([B,H,Nq,d] / [B,H,Nk,d]); dQ [B,H,Nq,d],
 * dK, dV [B,H,Nk,d] and dalpha [H] (or NULL) are device float32 outputs, overwritten.
 * idx entries outside [0, Nk/s) (the -1 padding) are skipped; a row with no cell has y = 0.
 * bws/bws_bytes: device scratch of fs_backward_workspace_size bytes (rotated keys and
 * queries, per-row softmax terms, the readout's du, the cell-to-rows lists, tile records).
 * Its first bytes hold a device error flag that must be zero before the first call (as a
 * forward workspace's); fs_sync_status(bws, stream) reads and clears it.  Enqueued on
 * `stream`; FS_ERR_INVALID_ARG / FS_ERR_UNSUPPORTED as for fs_forward.
 * The window's part runs on CUDA cores.  With bf16 and at most 128 distinct cells per
 * 128-row tile (W + P + 10 <= 128 with pruning, floor(Nk/s) <= 128 without; true of any
 * selection from A_i), the readout's part runs on the tensor cores (dK, dV added with
 * float32 atomics, so their last bits depend on the order); a tile whose rows select more
 * than 128 cells then sets the flag (FS_ERR_KERNEL_CHECK from fs_sync_status) and its
 * extra cells are left out.  Otherwise, and for float32, it runs on CUDA cores. */
fs_status fs_backward_workspace_size(const fs_params *p, size_t *bytes);
fs_status fs_backward(const fs_params *p, const void *Q, const void *K, const void *V, const int32_t *idx,
                      const void *dO, float *dQ, float *dK, float *dV, float *dalpha, void *bws,
                      size_t bws_bytes, void *stream);

/* ---- FS-L streaming cache ("FreeSolo" summary, "Practical Implications" 3: the per-head
 * memory of a stream is bounded by O((P+W)s + w + B + s)·d, whatever its length) ----
 * Tokens arrive in blocks of at most max_block (the B of that bound); after each block,
 * attention can be computed for any of its most recent positions from the cache alone.
 * The cache keeps, per (batch, head):
 *   - a ring of the last max_block + w + 2s tokens (raw keys, RoPE-rotated keys, values):
 *     the window of every query still to come plus the cells not yet candidates;
 *   - the candidate cells some upcoming query may still admit under eq. (8): the W most
 *     recent candidates and the TopP by max key norm, at most W + P + 2*ceil(max_block/s)
 *     + 4 cells, each with its keys, values, mean key and max norm (eq. (5)).
 * A cell leaves when no prefix still in reach admits it.  This is exact, not an
 * approximation: as the prefix grows a cell's rank by norm never improves, so a cell out
 * of TopP never re-enters it, and one older than the W most recent never becomes recent
 * again.  Base FS (no pruning) has no bounded state: W < 0 or P < 0 is FS_ERR_UNSUPPORTED.
 *
 * `cache` is a caller-owned device buffer of fs_cache_bytes bytes; every call on one cache
 * must pass the same p (B, H, d, w, s, K, W, P, dtype, rope_base, alpha, lambda, sigma,
 * rms_eps; Nq and Nk are ignored) and the same max_block (1 <= max_block <= 65536).
 * Calls enqueue on `stream` and must be ordered (one stream).  Errors found on the device
 * (e.g. attending more positions than have been appended) set the cache's error flag,
 * read by fs_cache_status. */
fs_status fs_cache_bytes(const fs_params *p, int max_block, size_t *bytes);

/* Empties the cache (no tokens). */
fs_status fs_cache_reset(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                         void *stream);

/* Appends n_new tokens (0 <= n_new <= max_block): K_new, V_new are device [B,H,n_new,d]
 * of type p->dtype, at positions t .. t+n_new-1 where t counts the tokens appended so far. */
fs_status fs_cache_append(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                          const void *K_new, const void *V_new, int n_new, void *stream);

/* O = o^sr + alpha_h o^lr (eq. (2)) for the n_q most recent positions t-n_q .. t-1
 * (1 <= n_q <= max_block, n_q <= t): Q_new and O are device [B,H,n_q,d] of type p->dtype.
 * idx, if not NULL, receives the selected cells [B,H,n_q,K] (ascending, -1 padded). */
fs_status fs_cache_attend(const fs_params *p, int max_block, void *cache, size_t cache_bytes,
                          const void *Q_new, int n_q, int32_t *idx, void *O, void *stream);

/* Synchronizes `stream`, then reads and clears the cache's error flag: FS_ERR_KERNEL_CHECK
 * if a call found its inputs inconsistent (n_q > t, or a state invariant broken),
 * FS_ERR_CUDA if the stream reports an error, else FS_OK. */
fs_status fs_cache_status(void *cache, void *stream);

/* ---- FS-B: balanced-tree search ("FreeSolo" summary §3.4, eqs. (10)-(11)) ----
 * Two causal forests per (batch, head): forest 0 over every cell in time order (admitted
 * set A^0_i = C_i), forest tau over the cells with a_c >= tau_h in time order (A^tau_i),
 * eq. (10).  Over a forest's sequence there is one balanced binary tree per aligned block
 * of 2^k entries, every k; the query at position i searches the trees covering its
 * candidate prefix (the set bits of its length).  A tree's leaves are its cells sorted by a
 * 16-bit code, the signs of kbar_c's first 16 coordinates (coordinate 0 most significant),
 * ties by time; node v stores mu_v = mean kbar_c, rho_v = max ||kbar_c - mu_v||, A_v =
 * max a_c and p_v^min = min p_c over its leaves and is ranked by eq. (11):
 *   U_v = (q_i.mu_v + c ||q_i|| rho_v) / sqrt(d) + lambda_h A_v erf((i - p_v^min) / (2 sigma_h)).
 * Beam search of width `beam` on each forest (from the prefix's roots; every internal node
 * of the beam replaced by its two children, the `beam` best kept by U_v, ties to the lower
 * p_v^min, until only leaves remain); S_i = the K best cells by eq. (7) among the leaves
 * both beams end on.  W and P are not used (FS-B does not prune).  With c >= 1 and
 * lambda_h >= 0, U_v bounds eq. (7) over the leaves below v; a beam that holds every leaf
 * gives base FS's selection. */
#define FS_TREE_MAX_BEAM 64

/* Bytes of the forest buffer for p (B, H, Nk, s): O(B H (Nk/s) log2(Nk/s) d) floats.
 * A forest buffer is laid out for its capacity: the largest cell count whose forest fits
 * in its bytes (so a buffer sized for a longer archive serves every shorter one).  Pass
 * the same forest_bytes to every call on one buffer. */
fs_status fs_forest_bytes(const fs_params *p, size_t *bytes);

/* Builds both forests for the C = Nk/s cells of p from the cell summaries
 * (fs_cell_summaries' kbar [B,H,C,d], amax [B,H,C], device f32) into the caller's device
 * buffer `forest`.  tau: HOST [H] thresholds of eq. (10), or NULL for forest 0 alone. */
fs_status fs_forest_build(const fs_params *p, const float *kbar, const float *amax, const float *tau,
                          void *forest, size_t forest_bytes, void *stream);

/* The archive grew ("FreeSolo" summary §3.4: balanced trees over an archive that keeps
 * growing): brings a forest built for at least prev_cells cells to the C = Nk/s cells of p
 * by rebuilding only the trees whose blocks end after cell prev_cells, as a binary counter
 * carries (amortised O(log C) trees per appended cell; a block of 2^k completes once every
 * 2^k cells).  kbar, amax: summaries of all C cells; those of the first prev_cells cells,
 * B, H, the capacity and tau (same values, or NULL as before) must be those of the earlier
 * build.  prev_cells below the cells built rebuilds from there (the later cells were
 * rewritten).  A forest that does not match (other sizes, fewer than prev_cells cells
 * built) is marked in its header, and the next search reports FS_ERR_KERNEL_CHECK through
 * fs_sync_status.  0 <= prev_cells <= C; prev_cells = 0 is fs_forest_build. */
fs_status fs_forest_append(const fs_params *p, int prev_cells, const float *kbar, const float *amax,
                           const float *tau, void *forest, size_t forest_bytes, void *stream);

/* FS-B selection: idx [B,H,Nq,K] (ascending, -1 padded) for the device queries Q, from a
 * forest built (or appended to) for the same B, H and C = Nk/s.  1 <= beam <= FS_TREE_MAX_BEAM; c_explore is eq. (11)'s
 * c.  ws (fs_workspace_size bytes) carries the device error flag: a forest not built for
 * these sizes is reported by fs_sync_status as FS_ERR_KERNEL_CHECK. */
fs_status fs_select_topk_tree(const fs_params *p, const void *Q, const void *forest, size_t forest_bytes,
                              int beam, float c_explore, int32_t *idx, void *ws, size_t ws_bytes,
                              void *stream);

/* The forward pass with the FS-B selection: summaries, forest build, search, then the
 * per-row readout (eq. (9)) on the selected cells and the window + combine (eqs. (2)-(4)).
 * idx, if not NULL, receives the selection. */
fs_status fs_forward_tree(const fs_params *p, const void *Q, const void *K, const void *V, const float *tau,
                          int beam, float c_explore, int32_t *idx, void *O, void *ws, size_t ws_bytes,
                          void *forest, size_t forest_bytes, void *stream);

/* ---- diagnostics (no counterpart in the method: measurement support) ----
 * fs_launch_count: kernels this library has launched since load (all calls, streams).
 * fs_timing_enable(1): from now on every kernel launch is bracketed by two CUDA events
 *   recorded on its own stream.  fs_kernel_times waits for the recorded events, writes per
 *   kernel id (0 <= id < max_ids) the launches and summed device milliseconds since the
 *   previous read, clears them, and returns the number of kernel ids.
 * fs_kernel_name: the name of a kernel id, or NULL past the last one.
 * fs_selftest_timeout: enqueues one small kernel that waits on a shared-memory barrier
 *   nothing arrives at, with the bounded wait every tensor-core kernel of this library
 *   uses (about 2 s); the wait runs out and the kernel records the timeout in the device
 *   error flag at the start of ws (a workspace of any of the calls above) and returns.
 *   fs_sync_status(ws, stream) then returns FS_ERR_TIMEOUT and clears the flag; the
 *   context stays usable.  It checks the failure-reporting path without a fault. */
long long fs_launch_count(void);
fs_status fs_timing_enable(int on);
int fs_kernel_times(int max_ids, long long *launches, double *ms);
const char *fs_kernel_name(int id);
fs_status fs_selftest_timeout(void *ws, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FREESOLO_H */
