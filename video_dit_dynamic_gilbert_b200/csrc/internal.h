// Launchers shared between the kernel files and the C ABI (api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace asa {

constexpr int kSamplesHost = 16;  // k: sampled tokens per block
constexpr int kMaxBlocksHost = 2048;  // 262,144 tokens in blocks of 128

// Device error word bit set when a caller-provided index (a CSR column, a pruning
// source row or position) is out of range; the access is skipped.
constexpr unsigned int kErrBadIndex = 32u;

bool gilbert_order_host(int T, int Hg, int W, int32_t* out);

// Sequence parallelism: P ranks, rank s owning the items [off[s], off[s+1]) (tokens or
// heads); passed to kernels by value.
constexpr int kMaxRanks = 64;
struct Segs {
  int P;
  int off[kMaxRanks + 1];
};

// Records the calling thread's error message for asa_last_error_string(); returns code.
int record_error(int code, const char* fmt, ...);

cudaError_t launch_permute(const void* const* src, void* const* dst, int ntensors, bool to_permuted,
                           const int32_t* perm_dev, int B, int N, int H, int d, int num_sms,
                           cudaStream_t stream);

// Estimator scratch (floats, 256-byte aligned base): G, lse2, per-chunk sums, Q_s, K_s.
size_t est_scratch_floats(int BH, int nb);
cudaError_t launch_estimate(const void* qp, const void* kp, int BH, int N, int d, float* scratch,
                            float* p_imp, unsigned int* err_word, int num_sms,
                            cudaStream_t stream);

// Device address of the library's error word on the current device (bounded waits
// that expire set bits in it: 1 = attention forward, 2 = estimator).
cudaError_t device_error_word(unsigned int** out);

cudaError_t launch_build_mask(const float* p_imp, int BH, int nb, float tau, uint8_t* bitmap,
                              int32_t* counts, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                              int32_t* counts_t, int32_t* col_ptr_t, int32_t* row_idx_t, int num_sms,
                              cudaStream_t stream);

// Statistical-threshold mask: z = Phi^-1(1 - k/n); keep_all when k >= n.
cudaError_t launch_build_mask_stat(const float* p_imp, int BH, int nb, double z, bool keep_all,
                                   uint8_t* bitmap, int32_t* counts, int32_t* row_ptr,
                                   int32_t* col_idx, int32_t* nnz_out, int32_t* counts_t,
                                   int32_t* col_ptr_t, int32_t* row_idx_t, int num_sms,
                                   cudaStream_t stream);

cudaError_t launch_global_pool(const void* xp, void* xg, int BH, int N, int d, int n, int num_sms,
                               cudaStream_t stream, const void* xp2 = nullptr,
                               void* xg2 = nullptr);

// perm_out != nullptr: O goes straight to raster layout [B, N, H, d], permuted row i of
// head h to token perm_out[i] (BH = B * H); otherwise O is [BH][N][d] in Gilbert order
cudaError_t launch_fwd_tc(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                          const int32_t* col_idx, const void* kg, const void* vg, int32_t* order,
                          int BH, int N, int d, int global_window, void* o, float* lse,
                          unsigned int* err_word, cudaStream_t stream,
                          const int32_t* perm_out = nullptr, int H = 1);

// Training forward: PV with fp16 P and the fp16 copies vp16, vg16 of V and of the
// global V tokens; writes O (bf16), LSE and the fp32 O.
cudaError_t launch_fwd_tc_train(const void* qp, const void* kp, const void* vp16,
                                const int32_t* row_ptr, const int32_t* col_idx, const void* kg,
                                const void* vg16, int32_t* order, int BH, int N, int d,
                                int global_window, void* o, float* lse, float* o32,
                                unsigned int* err_word, cudaStream_t stream);

// Launch order of the rows of a CSR (ptr[BH * nrows + 1], global offsets): heads in
// order, inside each head the rows with the most entries first; maxc bounds a row's
// entry count (the number of key blocks).
cudaError_t launch_lpt_order(const int32_t* ptr, int BH, int nrows, int maxc, int32_t* order,
                             cudaStream_t stream);

// Backward workspace (bytes, 256-aligned pieces): lse2 and D [BH][nb*128] f32,
// fp16 copies of Q and K [BH][N][d], launch orders of query and key blocks [BH*nb];
// with ASA_G the global tokens and their fp32 gradients.
size_t bwd_tc_workspace_bytes(int BH, int N, int d, int global_window);
cudaError_t launch_bwd_tc(const void* qp, const void* kp, const void* vp, const void* dout,
                          const float* lse, const int32_t* row_ptr, const int32_t* col_idx,
                          const int32_t* col_ptr_t, const int32_t* row_idx_t, int BH, int N,
                          int d, int global_window, void* workspace, void* dq, void* dk,
                          void* dv, unsigned int* err_word, int num_sms, cudaStream_t stream,
                          const void* o_for_d = nullptr, bool o_f32 = false);

// fp16 copy of n bf16 elements (n a multiple of 8); a value beyond fp16 range ORs 8
// into the device error word
cudaError_t launch_f16_copy(const void* src, void* dst, int64_t n, unsigned int* err_word,
                            int num_sms, cudaStream_t stream);

// Gilbert gather from / scatter into per-rank token chunks: chunk s holds the rows
// [B][tok.off[s+1] - tok.off[s]][H][d] of rank s's tokens, chunks back to back (the
// layout of an all-to-all receive or send buffer).
cudaError_t launch_permute_chunks(const void* const* src, void* const* dst, int ntensors,
                                  bool to_permuted, const int32_t* perm_dev, int B, int N, int H,
                                  int d, const Segs& tok, int num_sms, cudaStream_t stream);
// Head groups: x [B][Nr][H][d] <-> chunks [P][B][Nr][heads of group s][d].
cudaError_t launch_head_groups(const void* src, void* dst, bool pack, int B, int Nr, int H, int d,
                               const Segs& heads, int num_sms, cudaStream_t stream);

// Exclusive scan of n int32 counts on one CTA: out[i] = sum_{k<i} in[k], out[n] and
// *total (if non-null) = the sum.
cudaError_t launch_scan(const int32_t* in, int n, int32_t* out, int32_t* total,
                        cudaStream_t stream);

// Query pruning with token filling (BSA).  q_s: [BH][Ns][d] bf16 compact queries,
// `pack` blocks per 128-row tile; src_pos / src_row: [BH][N] int32.
cudaError_t launch_prune(const void* qp, int BH, int N, int d, float r, int w, int pack, void* q_s,
                         int Ns, int32_t* src_pos, int32_t* src_row, cudaStream_t stream);
// Tile CSR (union of the tile's blocks' kept key blocks) with a quarter bit mask per
// entry; counts: [BH * ntile] scratch.
cudaError_t launch_prune_mask(const int32_t* row_ptr, const int32_t* col_idx, int BH, int nb,
                              int pack, int32_t* counts, int32_t* tile_ptr, int32_t* tile_col,
                              uint8_t* tile_quarters, int32_t* nnz_out, unsigned int* err_word,
                              int num_sms, cudaStream_t stream);
cudaError_t launch_fill_out(const void* o_s, const float* lse_s, const int32_t* src_row, int BH,
                            int N, int Ns, int d, void* o, float* lse, unsigned int* err_word,
                            int num_sms, cudaStream_t stream);
// Pruned backward inputs in the compact layout (dO' sums and lse2 of the kept rows).
cudaError_t launch_dout_compact(const void* dout, const float* lse, const int32_t* src_pos,
                                const int32_t* src_row, int BH, int N, int Ns, int d,
                                void* dout_s, float* lse2_s, unsigned int* err_word, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_dq_scatter(const void* dq_s, const int32_t* src_pos, const int32_t* src_row,
                              int BH, int N, int Ns, int d, void* dq, unsigned int* err_word,
                              int num_sms, cudaStream_t stream);
// Transposed tile CSR (per key block, the tiles holding it) through a dense
// [BH][ntile][nbk] quarter matrix qmat; counts: [BH * nbk] scratch.
cudaError_t launch_tile_transpose(const int32_t* tile_ptr, const int32_t* tile_col,
                                  const uint8_t* tile_quarters, int BH, int ntile, int nbk,
                                  uint8_t* qmat, int32_t* counts, int32_t* tcol_ptr,
                                  int32_t* trow_idx, uint8_t* tquarters, unsigned int* err_word,
                                  int num_sms, cudaStream_t stream);
// Forward over a packed tile CSR: q_s has Ns rows per head; quarters[e] says which
// 32-row lane quarters of the tile see entry e; o_s, lse_s: [BH][Ns].
cudaError_t launch_fwd_tc_pruned(const void* q_s, const void* kp, const void* vp,
                                 const int32_t* tile_ptr, const int32_t* tile_col,
                                 const uint8_t* quarters, const void* kg, const void* vg,
                                 int32_t* order, int BH, int N, int Ns, int d, int global_window,
                                 void* o_s, float* lse_s, unsigned int* err_word,
                                 cudaStream_t stream);

// Backward with query pruning on packed tiles (workspace: bwd_tc_pruned_workspace_bytes).
size_t bwd_tc_pruned_workspace_bytes(int BH, int N, int Ns, int d, int global_window);
cudaError_t launch_bwd_tc_pruned(const void* q_s, const void* kp, const void* vp, const void* dout,
                                 const float* lse, const int32_t* src_pos, const int32_t* src_row,
                                 const int32_t* tile_ptr, const int32_t* tile_col,
                                 const uint8_t* tile_quarters, int BH, int N, int Ns, int d,
                                 int global_window, void* workspace, void* dq, void* dk, void* dv,
                                 unsigned int* err_word, int num_sms, cudaStream_t stream);

// Failure-detection test hook: one bounded wait on a barrier nothing arrives at.
cudaError_t launch_wait_timeout(unsigned int* err_word, long long limit, cudaStream_t stream);

}  // namespace asa
