/*
 * asa.h -- C ABI of the B200 (sm_100a) Adaptive Block-Sparse Attention library
 * (libasa.so).
 *
 * The method is ASA from "Video-BLADE: Block-Sparse Attention Meets Step
 * Distillation for Efficient Video Generation" (arXiv 2508.10774), section
 * "Adaptive Block-Sparse Attention":
 *   Preprocessing  -- Gilbert rearrangement of the (T, H, W) token grid, then
 *                     blocks of b = 128 consecutive permuted tokens;
 *   Step 1         -- block importance P_imp from k = 16 sampled tokens per block;
 *   Step 2.1       -- per query block, the fewest key blocks whose cumulative share
 *                     of P_imp reaches tau;
 *   Step 2.2       -- attention over the kept (query block, key block) tiles only:
 *                     standard ASA, or ASA_G with mean-pooled global tokens whose
 *                     logits carry a fixed additive ln(n);
 *   the same mask restricts the backward pass (end of Step 2.1).
 *
 * Conventions for every entry point:
 *   - Tensors are bf16 unless stated; "device" pointers are CUDA device memory
 *     owned by the caller, "host" pointers are host memory owned by the caller.
 *     The library never frees caller memory.
 *   - Layouts: the model layout is raster [B, N, H, d] (token n = (t*Hg + y)*W + x);
 *     the permuted layout is [B, H, N, d] (head-major, tokens in Gilbert order).
 *     Rows are dense; every pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream; none synchronises the host except
 *     the first call for a new (T, Hg, W) shape, which builds and uploads the
 *     permutation table once (the library owns that table until asa_shutdown).
 *   - Supported: head dim d in {64, 128}, block b = 128, samples k = 16,
 *     N = number of tokens in [1, ASA_MAX_TOKENS].
 *   - Return 0 (ASA_OK) or a negative ASA_ERR_* code; asa_last_error_string()
 *     then describes the failure of the calling thread's last failing call.
 *     Argument checks run on the host before anything is launched, so a
 *     rejected call touches no device memory.
 */
#ifndef ASA_H_
#define ASA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ASA_OK 0
#define ASA_ERR_INVALID_ARG (-1) /* null/misaligned pointer, bad shape, N != T*Hg*W, tau <= 0 */
#define ASA_ERR_UNSUPPORTED (-2) /* d not in {64,128}, block != 128, samples != 16, too large */
#define ASA_ERR_WORKSPACE (-3)   /* workspace missing or smaller than the *_workspace_size() */
#define ASA_ERR_CUDA (-4)        /* a CUDA call or kernel launch failed */
#define ASA_ERR_TIMEOUT (-5)     /* a device-side bounded wait expired (see asa_check_device_status) */

#define ASA_MAX_TOKENS 262144   /* N limit: at most 2048 blocks of 128 */
#define ASA_BLOCK 128
#define ASA_MAX_RANKS 64       /* sequence-parallel ranks of the asa_seqpar_* calls */
#define ASA_SAMPLES 16

/* Library version as 10000*major + 100*minor + patch. */
int asa_version(void);

/* Message of the calling thread's last failing call ("" if none). Never NULL. */
const char* asa_last_error_string(void);

/*
 * Gilbert order (Preprocessing paragraph): perm_host[i] = raster index of the token
 * at curve position i, for the T x Hg x W grid.  perm_host: host, N = T*Hg*W int32.
 * Pure host computation.  The curve is a generalised Hilbert curve whose
 * consecutive cells are grid neighbours and which reduces to the Hilbert curve on
 * 2^m x 2^m frames.
 */
int asa_gilbert_index(int T, int Hg, int W, int32_t* perm_host);

/*
 * Gather to Gilbert order (Preprocessing paragraph):
 *   xp[b, h, i, :] = x[b, perm[i], h, :]
 * x: device bf16 [B, N, H, d] raster; xp: device bf16 [B, H, N, d]; N = T*Hg*W.
 * x and xp must not overlap.
 */
int asa_gilbert_permute(const void* x, void* xp, int B, int T, int Hg, int W, int H, int d,
                        void* stream);

/* Same gather applied to three tensors in one launch (Q, K and V of one call). */
int asa_gilbert_permute3(const void* x0, const void* x1, const void* x2, void* xp0, void* xp1,
                         void* xp2, int B, int T, int Hg, int W, int H, int d, void* stream);

/*
 * Inverse scatter back to raster order: x[b, perm[i], h, :] = xp[b, h, i, :].
 * xp: device bf16 [B, H, N, d]; x: device bf16 [B, N, H, d].
 */
int asa_unpermute(const void* xp, void* x, int B, int T, int Hg, int W, int H, int d, void* stream);

/*
 * Workspace bytes needed by asa_estimate / asa_build_mask / asa_estimate_mask for
 * this shape (device memory, any content on entry, 256-byte aligned).
 */
size_t asa_estimate_mask_workspace_size(int B, int H, int N);

/*
 * Step 1, block importance (P_imp) only.
 * Block I holds permuted positions [128 I, min(128 I + 128, N)) of L_I tokens; its
 * k_I = min(16, L_I) samples are offsets floor(j L_I / k_I).  With Q_s, K_s the
 * sampled rows of qp, kp (M rows in block order),
 *   P_approx = rowsoftmax(Q_s K_s^T / sqrt(d)),
 *   P_imp[b, h, I, J] = max over the k_I x k_J tile (I, J) of P_approx.
 * qp, kp: device bf16 [B, H, N, d]; p_imp: device fp32 [B, H, nb, nb], nb = ceil(N/128).
 */
int asa_estimate(const void* qp, const void* kp, int B, int H, int N, int d, int block,
                 int samples, void* workspace, size_t ws_bytes, float* p_imp, void* stream);

/*
 * Step 2.1 from a given P_imp: per row (b, h, I), with shares R = P_imp / rowsum,
 * keep the fewest key blocks whose cumulative share (shares in descending order,
 * ties by lower J) reaches tau (tau >= 1 keeps all).  Emits the kept blocks as CSR:
 *   row_ptr  device int32 [B*H*nb + 1], rows in (b, h, I) order;
 *   col_idx  device int32, capacity B*H*nb*nb (upper bound), J ascending per row;
 *   nnz_out  device int32 [1] = row_ptr[B*H*nb];
 *   col_ptr_t, row_idx_t (both NULL or both set): the transposed CSR, for each
 *            (b, h, J) the q-blocks I keeping J, ascending (same capacities);
 *            the backward pass walks it.
 * p_imp: device fp32 [B, H, nb, nb].  tau must be > 0.
 */
int asa_build_mask(const float* p_imp, int B, int H, int N, float tau, void* workspace,
                   size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                   int32_t* col_ptr_t, int32_t* row_idx_t, void* stream);

/*
 * asa_estimate without any allocation and without a caller workspace, for callers
 * that cannot allocate device memory (a host engine that owns all GPU memory in a
 * fixed pool and forbids third-party allocations, or a latency-critical loop that
 * must not risk the synchronisation cudaMalloc may cause).  The paper has no
 * counterpart: this is a library convenience.  Same arguments, layouts and result
 * as asa_estimate minus the workspace.
 *   - Scratch: one file-scope device array of ASA_NOALLOC_SCRATCH_BYTES.  Under CUDA's
 *     lazy module loading (the default) it is reserved on a device when the library's
 *     module is first loaded there, which the first call on that device does, and it
 *     is held until the process exits.  That first call may therefore reserve the
 *     32 MiB and synchronise: make it during set-up, before any stream capture.
 *     Shapes needing more (about 6.2 MB per head at N = 32,760 and d = 128, i.e. at
 *     most 5 heads per call at that shape) are rejected with ASA_ERR_WORKSPACE before
 *     anything is launched.
 *   - Every call looks up the array's device address in the current context (the
 *     address is not cached, so it stays valid across a context re-creation).
 *   - Every call shares the array and overwrites what it reads (nothing in it needs to
 *     start at zero).  Calls whose kernels overlap on the GPU (different streams, or
 *     several host threads) race on the array: serialise them.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define ASA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int asa_estimate_noalloc(const void* qp, const void* kp, int B, int H, int N, int d, int block,
                         int samples, float* p_imp, void* stream);

/*
 * Statistical-threshold mask, a second mask mode with the same inputs and outputs as
 * asa_build_mask: BSA's adaptive key-block selection (the BSA page, design point 2:
 * p = mean(S_b) + std(S_b) * U(1 - k/n), U the normal quantile function, n the number
 * of blocks, k the target candidate count).  Reading
 * taken: per query block, S_b are the row's shares R_J = P_imp[I, J] / sum_J P_imp[I, J];
 * p = mean(R) + std(R) * Phi^-1(1 - k_target/nb) (population std); every key block with
 * R_J >= p is kept (about k_target of nb blocks when the shares are normal); a row that
 * keeps none keeps its largest share (lowest J on ties).  k_target >= nb keeps every
 * block.  Sums in fp64.  p_imp: device fp32 [B, H, nb, nb]; the workspace and the CSR
 * outputs are those of asa_build_mask.
 */
int asa_build_mask_stat(const float* p_imp, int B, int H, int N, int k_target, void* workspace,
                        size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                        int32_t* col_ptr_t, int32_t* row_idx_t, void* stream);

/* Steps 1 + 2.1 in one call (P_imp stays in the workspace). Arguments as above. */
int asa_estimate_mask(const void* qp, const void* kp, int B, int H, int N, int d, int block,
                      int samples, float tau, void* workspace, size_t ws_bytes, int32_t* row_ptr,
                      int32_t* col_idx, int32_t* nnz_out, int32_t* col_ptr_t, int32_t* row_idx_t,
                      void* stream);

/*
 * ASA_G global tokens (Step 2.2, variant 2): xg[b, h, g, :] = bf16(mean of
 * xp[b, h, i, :] over permuted positions i in [n g, min(n g + n, N))), g < ceil(N/n).
 * xp: device bf16 [B, H, N, d]; xg: device bf16 [B, H, ceil(N/n), d]; n >= 1.
 */
int asa_global_pool(const void* xp, void* xg, int B, int H, int N, int d, int n, void* stream);

/* asa_global_pool of K (into kg) and V (into vg) in one launch, as the ASA_G forward and
 * backward build their global tokens.  Same layouts and errors as asa_global_pool. */
int asa_global_pool_kv(const void* kp, const void* vp, void* kg, void* vg, int B, int H, int N,
                       int d, int n, void* stream);

/* Workspace bytes of asa_sparse_attn_fwd: the launch order of the query blocks
 * (longest kept list first), plus the global tokens for ASA_G. */
size_t asa_fwd_workspace_size(int B, int H, int N, int d, int global_window);

/*
 * Step 2.2, forward over the kept tiles only.  For a query i of block I:
 *   O_i = softmax_j(q_i . k_j / sqrt(d)) V over the tokens j of the kept blocks
 *   of row (b, h, I)  [standard ASA, global_window = 0];
 * with global_window = n > 0 (ASA_G) the softmax also spans all ceil(N/n) global
 * tokens (asa_global_pool of K and V, built in the workspace) with logits
 * q_i . kg / sqrt(d) + ln(n).
 * qp, kp, vp: device bf16 [B, H, N, d]; row_ptr/col_idx: the CSR of asa_build_mask;
 * o: device bf16 [B, H, N, d]; lse: device fp32 [B, H, N], natural-log
 * log-sum-exp of each row's logits (kept for the backward).
 */
int asa_sparse_attn_fwd(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                        const int32_t* col_idx, int B, int H, int N, int d, int block,
                        int global_window, void* workspace, size_t ws_bytes, void* o, float* lse,
                        void* stream);

/*
 * asa_sparse_attn_fwd followed by the inverse Gilbert permutation (Preprocessing: the
 * output returns to the original token order), fused: each output row is stored
 * straight to its raster position, o[b, perm[i], h, :] = O[b, h, i, :], so no permuted
 * O is written.  N = T*Hg*W; qp, kp, vp, the CSR, workspace (asa_fwd_workspace_size)
 * and lse (device fp32 [B, H, N], Gilbert order) as in asa_sparse_attn_fwd;
 * o: device bf16 [B, N, H, d] (raster layout, as asa_unpermute writes), not aliasing
 * an input.  The result is bit-identical to asa_sparse_attn_fwd then asa_unpermute.
 * Errors as asa_sparse_attn_fwd, plus ASA_ERR_INVALID_ARG for a bad grid.
 */
int asa_sparse_attn_fwd_raster(const void* qp, const void* kp, const void* vp,
                               const int32_t* row_ptr, const int32_t* col_idx, int B, int T,
                               int Hg, int W, int H, int d, int block, int global_window,
                               void* workspace, size_t ws_bytes, void* o, float* lse,
                               void* stream);

/*
 * Workspace bytes of asa_sparse_attn_fwd_train (0 for invalid sizes): those of
 * asa_sparse_attn_fwd plus an fp16 copy of V (B*H*N*d * 2 bytes) and, with
 * global_window = n > 0, an fp16 copy of the G global V tokens (B*H*G*d * 2 bytes).
 */
size_t asa_fwd_train_workspace_size(int B, int H, int N, int d, int global_window);

/*
 * The forward of asa_sparse_attn_fwd (same computation, arguments, layouts and errors)
 * for training: it also writes o32, the output in fp32 before its bf16 rounding, from
 * which asa_sparse_attn_bwd_train takes D = rowsum(dO * O) ("Step 2.1": the mask of
 * the forward restricts the backward too; D is the row term of the softmax gradient).
 * For that D to be accurate, the P V product takes P in fp16 (11 significant bits, the
 * inference forward's bf16 has 8) against an fp16 copy of V made in the workspace; V
 * magnitudes must therefore stay at or below 65504 (a larger value is reported by the
 * next asa_check_device_status as ASA_ERR_INVALID_ARG).  o: device bf16 [B, H, N, d];
 * lse: device fp32 [B, H, N]; o32: device fp32 [B, H, N, d], 16-byte aligned.
 */
int asa_sparse_attn_fwd_train(const void* qp, const void* kp, const void* vp,
                              const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N,
                              int d, int block, int global_window, void* workspace,
                              size_t ws_bytes, void* o, float* lse, float* o32, void* stream);

/*
 * Workspace bytes of asa_sparse_attn_bwd (0 for invalid sizes): per-row lse*log2(e)
 * and D (fp32, rows padded to whole blocks), fp16 copies of Q and K
 * (2 * B*H*N*d * 2 bytes), and the launch orders of query and key blocks; with
 * global_window = n > 0 also the G = ceil(N/n) global tokens (bf16 K, V and fp16 K,
 * B*H*G*d each) and their fp32 gradients (2 * B*H*G*d * 4 bytes).
 */
size_t asa_bwd_workspace_size(int B, int H, int N, int d, int global_window);

/*
 * Backward of ASA under the fixed mask (Video-BLADE, "Step 2.1": the same block mask
 * applies in training as at inference; it is not differentiated):
 *   P = exp(S - LSE), dP = dO V^T, D = rowsum(P * dP), dS = P * (dP - D),
 *   dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d), dV = P^T dO, all over kept tiles only.
 * global_window = n > 0: the backward of ASA_G ("Step 2.2", variant 2, the forward
 * with the same n): the softmax also spans the G = ceil(N/n) global tokens (mean of
 * K and V over each window of n permuted rows, logits + ln(n)); dQ gains their term,
 * and the gradient of each global token reaches the rows of its window divided by
 * the window's row count (its bf16 rounding passes gradients unchanged).
 * D equals rowsum(dO * O) in exact arithmetic; it is recomputed in fp32 from the kept
 * tiles because the bf16-rounded O would cost ~4e-3 relative L2 on dQ.  `o` is
 * validated but not read (asa_sparse_attn_bwd_d_from_o reads it instead of the exact
 * D pass).  dS enters the dQ and dK products in fp16 (so do Q and K,
 * as fp16 copies in the workspace): Q and K magnitudes must stay at or below 65504;
 * a larger value is reported by the next asa_check_device_status as
 * ASA_ERR_INVALID_ARG (the gradients of that call are then meaningless).
 * Deterministic: every output row is written by one CTA, without atomics.
 * qp, kp, vp, o, dout: device bf16 [B, H, N, d]; lse: device fp32 [B, H, N] from the
 * forward; row_ptr/col_idx and col_ptr_t/row_idx_t: both CSRs of asa_build_mask;
 * dq, dk, dv: device bf16 [B, H, N, d] (fully written; no accumulation into them).
 */
int asa_sparse_attn_bwd(const void* qp, const void* kp, const void* vp, const void* o,
                        const void* dout, const float* lse, const int32_t* row_ptr,
                        const int32_t* col_idx, const int32_t* col_ptr_t,
                        const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                        int global_window, void* workspace, size_t ws_bytes, void* dq, void* dk,
                        void* dv, void* stream);

/*
 * asa_sparse_attn_bwd with D taken as rowsum(dO * O) from the forward's bf16 O (read
 * here) instead of the exact pass over the kept tiles: one GEMM pair per kept tile
 * less, about a fifth of the backward's time.  The rounding of O to bf16 then enters
 * dS: on the parity cases it adds about 3e-3 relative L2 to dQ and dK (dV does not
 * depend on D and is bit-identical to asa_sparse_attn_bwd's).  Same arguments,
 * workspace and errors as asa_sparse_attn_bwd; opt in where that accuracy suffices.
 */
int asa_sparse_attn_bwd_d_from_o(const void* qp, const void* kp, const void* vp, const void* o,
                                 const void* dout, const float* lse, const int32_t* row_ptr,
                                 const int32_t* col_idx, const int32_t* col_ptr_t,
                                 const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                                 int global_window, void* workspace, size_t ws_bytes, void* dq,
                                 void* dk, void* dv, void* stream);

/*
 * asa_sparse_attn_bwd for a forward run by asa_sparse_attn_fwd_train: D is taken as
 * rowsum(dO * O) from that forward's fp32 output o32 (device fp32 [B, H, N, d]) in one
 * pass over dO and o32, instead of the exact pass over the kept tiles (two GEMMs per
 * kept tile).  The gradients meet the same tolerances as asa_sparse_attn_bwd's (the
 * fp16 P of that forward leaves O within ~2^-12 relative of its exact value); dV does
 * not depend on D and is bit-identical to asa_sparse_attn_bwd's.  Same workspace
 * (asa_bwd_workspace_size), arguments and errors as asa_sparse_attn_bwd, with o32 in
 * place of o; lse must come from the same training forward.  Deterministic.
 */
int asa_sparse_attn_bwd_train(const void* qp, const void* kp, const void* vp, const float* o32,
                              const void* dout, const float* lse, const int32_t* row_ptr,
                              const int32_t* col_idx, const int32_t* col_ptr_t,
                              const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                              int global_window, void* workspace, size_t ws_bytes, void* dq,
                              void* dk, void* dv, void* stream);

/* ------------------------------------------------------------------------------
 * Query pruning with token filling ("Bidirectional Sparse Attention for Faster
 * Video Diffusion Training", section "Key designs", item 1), layered on ASA's
 * blocks of 128 permuted tokens.
 *
 * A block of L tokens is cut into windows of `window` consecutive permuted tokens
 * from the block start (the last one ragged); the centre of a window of length l
 * starting at s is token s + l/2.  The block keeps K = max(ceil(r L), windows)
 * queries: every centre, then the other tokens with the largest 1 - cos(q_centre,
 * q_i) to their own window's centre (ties to the lower position; a norm below 1e-8
 * counts as 1e-8; ceil(r L) is taken in double on the float r).  Attention is
 * computed for kept queries only; a pruned token takes its centre's output row and
 * LSE.  In the backward a pruned token's output gradient is added to its centre's
 * and it gets no gradient of its own.
 *
 * Kept queries live in a compact buffer q_s [B, H, Ns, d] of 128-row tiles: tile t
 * holds blocks t*pack .. t*pack+pack-1, block I in rows (I % pack) * 128/pack + j of
 * its tile (its j-th kept query in position order; unused rows zero).  One tile runs
 * over the union of its blocks' kept key blocks (asa_prune_mask); a union entry is
 * seen only by the 32-row lane quarters of the blocks that keep it.
 * ---------------------------------------------------------------------------- */

/* Largest pack in {1, 2, 4} whose slots (128/pack rows) hold every block's kept
 * queries for this r and window; ASA_ERR_INVALID_ARG for r outside [0, 1] or window
 * outside [1, 128]. */
int asa_prune_pack(float r, int window);

/* Ns = ceil(ceil(N/128) / pack) * 128 (rows per head of q_s), or a negative code. */
int asa_prune_rows(int N, int pack);

/*
 * Selects the kept queries and packs them.  qp: device bf16 [B, H, N, d] (permuted
 * layout); q_s: device bf16 [B, H, Ns, d], fully written (zeros in unused rows);
 * src_pos: device int32 [B, H, N], the permuted position whose output token i
 * takes (i if kept, else its window centre); src_row: device int32 [B, H, N], the
 * row of q_s (and of the pruned forward's compact output) holding it.  pack must be
 * in {1, 2, 4} and at most asa_prune_pack(r, window).
 */
int asa_prune_queries(const void* qp, int B, int H, int N, int d, int block, float r, int window,
                      int pack, void* q_s, int32_t* src_pos, int32_t* src_row, void* stream);

/* Workspace bytes of asa_prune_mask (a count per tile), 0 for invalid sizes. */
size_t asa_prune_mask_workspace_size(int B, int H, int N, int pack);

/*
 * Tile CSR of the packed queries from a block mask (row_ptr/col_idx of
 * asa_build_mask or asa_build_mask_stat): tile_ptr [B*H*ntile + 1] (ntile =
 * ceil(ceil(N/128)/pack)), tile_col [capacity nnz of the input] ascending key
 * blocks of the union, tile_quarters [same] with bit q set when lane quarter q
 * (rows 32q .. 32q+31 of the tile) belongs to a block that keeps that key block;
 * nnz_out: device int32, the union's entry count.  An input column outside
 * [0, ceil(N/128)) is skipped and reported by asa_check_device_status as
 * ASA_ERR_INVALID_ARG.
 */
int asa_prune_mask(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N, int pack,
                   void* workspace, size_t ws_bytes, int32_t* tile_ptr, int32_t* tile_col,
                   uint8_t* tile_quarters, int32_t* nnz_out, void* stream);

/* Workspace bytes of asa_sparse_attn_fwd_pruned: the tile launch order, the compact
 * output (bf16 [B, H, Ns, d]) and LSE (fp32 [B, H, Ns]), the ASA_G global tokens. */
size_t asa_fwd_pruned_workspace_size(int B, int H, int N, int d, int pack, int global_window);

/*
 * Step 2.2 (ASA, or ASA_G with global_window = n > 0) for the kept queries only,
 * then token filling: o [B, H, N, d] bf16 and lse [B, H, N] fp32 take, for every
 * token i, the compact row src_row[i].  q_s, src_row: from asa_prune_queries; kp,
 * vp: the full permuted keys and values; tile_*: from asa_prune_mask.  A src_row
 * outside [0, Ns) writes a zero row, lse -inf, and is reported as
 * ASA_ERR_INVALID_ARG by asa_check_device_status.
 */
int asa_sparse_attn_fwd_pruned(const void* q_s, const void* kp, const void* vp,
                               const int32_t* tile_ptr, const int32_t* tile_col,
                               const uint8_t* tile_quarters, const int32_t* src_row, int B, int H,
                               int N, int d, int block, int pack, int global_window,
                               void* workspace, size_t ws_bytes, void* o, float* lse,
                               void* stream);

/* Workspace bytes of asa_sparse_attn_bwd_pruned: the backward's pieces with the query
 * side in the compact layout (lse2, D, fp16 queries: B*H*Ns rows), the compact output
 * gradient and dQ (bf16 [B, H, Ns, d] each), and the transposed tile CSR (a dense
 * [B*H][Ns/128][ceil(N/128)] byte matrix, its counts, pointers, tile indices and
 * quarter bits).  0 for invalid sizes. */
size_t asa_bwd_pruned_workspace_size(int B, int H, int N, int d, int pack, int global_window);

/*
 * Backward with query pruning under the fixed mask, on the packed tiles of the pruned
 * forward.  A pruned token's output is its centre's row, so with dO'[c] = the sum of
 * dO[i] over the tokens i with src_pos[i] = c (stored in bf16) it computes
 * asa_sparse_attn_bwd's gradients of the kept rows only, and pruned rows get dQ = 0.
 * The query side runs over q_s's compact rows (a (tile, key block) entry restricted to
 * the lane quarters of tile_quarters); the key side walks the transposed tile CSR,
 * built in the workspace.  Inputs: q_s, src_pos, src_row from asa_prune_queries
 * (each token must map to a kept token of its own block; other rows are skipped and
 * reported as ASA_ERR_INVALID_ARG), tile_* from asa_prune_mask, lse from
 * asa_sparse_attn_fwd_pruned, dout bf16 [B, H, N, d] (permuted layout), kp, vp as in
 * the forward.  Outputs dq, dk, dv bf16 [B, H, N, d].  Deterministic.
 */
int asa_sparse_attn_bwd_pruned(const void* q_s, const void* kp, const void* vp, const void* dout,
                               const float* lse, const int32_t* src_pos, const int32_t* src_row,
                               const int32_t* tile_ptr, const int32_t* tile_col,
                               const uint8_t* tile_quarters, int B, int H, int N, int d, int block,
                               int pack, int global_window, void* workspace, size_t ws_bytes,
                               void* dq, void* dk, void* dv, void* stream);

/* ------------------------------------------------------------------------------
 * One ASA (or ASA_G) self-attention call on HOST buffers: raster q, k, v in, raster O
 * out, with the copies pipelined against the compute.
 * ---------------------------------------------------------------------------- */

/* Workspace bytes of asa_attention_host: two pipeline slots, each holding the device
 * copies of head_chunk heads (raster and permuted Q, K, V; raster O), the
 * estimator and mask workspace and CSR, the forward workspace and the LSE of those
 * heads.  head_chunk = 0 takes the default below.  0 for invalid sizes. */
size_t asa_attention_host_workspace_size(int B, int T, int Hg, int W, int H, int d,
                                         int global_window, int head_chunk);

/*
 * The whole call of asa_gilbert_permute3 -> asa_estimate_mask ->
 * asa_sparse_attn_fwd_raster (Preprocessing, Steps 1, 2.1, 2.2; the forward stores O
 * straight to raster order) for host buffers q, k, v, o
 * (bf16 [B, T*Hg*W, H, d], raster order), in chunks of head_chunk heads (0: the default,
 * max(ceil(256/d), ceil(H/24)) heads, capped at H: host rows of at least 512 bytes in
 * the strided copies, which narrower rows slow down, and at most 24 chunks; the last
 * of two or more default chunks is split in two, shortening the pipeline's tail).
 * Chunk c's strided host-to-device copies, chunk c-1's kernels and chunk c-2's
 * device-to-host copy run at once on three streams the library owns (one set per
 * device, released by asa_shutdown); two workspace slots alternate.  The call is
 * ordered on `stream`: the pipeline starts after the work already queued there and
 * the stream waits for its end, so an event recorded on `stream` after the call marks
 * the output's arrival in `o` (synchronise the stream before reading it).  Copies
 * overlap only when the host buffers are page-locked (pinned); pageable buffers give
 * the same results, copied synchronously.  The outputs equal asa_attention's per
 * head: each head's mask and rows do not depend on the other heads.  Returns as the
 * composed calls do (their argument checks apply per chunk).
 */
int asa_attention_host(const void* q, const void* k, const void* v, int B, int T, int Hg, int W,
                       int H, int d, float tau, int global_window, int head_chunk,
                       void* workspace, size_t ws_bytes, void* o, void* stream);

/* ------------------------------------------------------------------------------
 * Sequence parallelism (a sequence-sharded DiT): P ranks, rank r holding the raster
 * tokens [tok_off[r], tok_off[r+1]) of every head, x_r [B, N_r, H, d].  Attention
 * needs every token of a head, so before it an all-to-all (NCCL, into local buffers)
 * gives rank r every token of its heads [head_off[r], head_off[r+1]), H_r of them;
 * the inverse all-to-all follows.  These calls are the local steps around the two
 * exchanges; the Gilbert gather reads the receive buffer's per-rank chunks directly
 * and the inverse writes straight into the send buffer's chunks.  Offsets are host
 * arrays of P + 1 ints from 0 to N (tokens) or H (heads), non-decreasing;
 * 1 <= P <= ASA_MAX_RANKS.  Device buffers bf16, 16-byte aligned.
 * ---------------------------------------------------------------------------- */

/* Send buffer of the first exchange: send = chunks s = 0..P-1 back to back, chunk s =
 * x[:, :, head_off[s]:head_off[s+1], :] as [B, Nr, H_s, d] (for rank s).  x: [B, Nr, H, d]. */
int asa_seqpar_pack(const void* x, void* send, int B, int Nr, int H, int d, const int* head_off,
                    int P, void* stream);

/* Inverse of asa_seqpar_pack, applied to the receive buffer of the second exchange:
 * chunk s (from rank s, its heads) back into x [B, Nr, H, d]. */
int asa_seqpar_unpack(const void* recv, void* x, int B, int Nr, int H, int d, const int* head_off,
                      int P, void* stream);

/*
 * Preprocessing on the receive buffers of the first exchange: r = chunks s = 0..P-1
 * back to back, chunk s = rank s's tokens of this rank's Hl heads as [B, N_s, Hl, d];
 * xp[b, h, i, :] = the row of token perm[i] (Gilbert order of the T x Hg x W grid)
 * taken from its rank's chunk.  xp: [B, Hl, N, d]; three tensors (Q, K, V) at once.
 * With P = 1 it is asa_gilbert_permute3.
 */
int asa_seqpar_permute3(const void* r0, const void* r1, const void* r2, void* xp0, void* xp1,
                        void* xp2, int B, int T, int Hg, int W, int Hl, int d, const int* tok_off,
                        int P, void* stream);

/* Inverse of asa_seqpar_permute3 for one tensor: op [B, Hl, N, d] (permuted) into the
 * send buffer of the second exchange, chunk s = rank s's tokens [B, N_s, Hl, d]. */
int asa_seqpar_unpermute(const void* op, void* send, int B, int T, int Hg, int W, int Hl, int d,
                         const int* tok_off, int P, void* stream);

/*
 * Synchronises `stream`, then reads and clears the library's device error word of
 * the current device.  Returns ASA_OK, ASA_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last check, ASA_ERR_INVALID_ARG if a backward call met Q or
 * K values beyond fp16 range, or ASA_ERR_CUDA on a CUDA error.
 */
int asa_check_device_status(void* stream);

/*
 * Test hook for failure detection (no counterpart on the pages): launches one CTA whose
 * bounded mbarrier wait (the primitive every kernel uses) waits on a barrier that
 * nothing ever arrives at, so it gives up after `limit_cycles` SM clock cycles (1 to
 * 2^31, about 1 s at most), records the expiry in the device error word and returns.
 * The next asa_check_device_status then returns ASA_ERR_TIMEOUT and clears the word;
 * the context stays usable.  Asynchronous on `stream`; nothing else calls it.
 */
int asa_selftest_wait_timeout(long long limit_cycles, void* stream);

/* Frees the cached permutation tables of every device.  Safe to call twice. */
void asa_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* ASA_H_ */
