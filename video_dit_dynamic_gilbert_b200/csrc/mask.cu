// Threshold mask (Video-BLADE, "Step 2.1: Sparse mask construction") and its CSR.
//
// Per row (b, h, I) of P_imp: shares R_J = P_imp[I, J] / sum_J P_imp[I, J]; order
// the key blocks by (R descending, J ascending); keep the first c* blocks, c* the
// least count whose cumulative share reaches tau (tau >= 1 keeps every block).
//
// The kept set is found without a sort.  With f(v) = sum of the P_imp values >= v,
// the smallest kept value v* is the largest v with f(v) >= tau * total: a bisection
// over the (monotone) bit patterns of non-negative floats, 31 warp-wide passes over
// the row.  Blocks above v* are kept, and blocks equal to v* are added in J order
// until the cumulative sum reaches the target.  Sums are taken in fp64.
//
// Statistical threshold (the BSA mode; "Video-BLADE" names BSA's adaptive selection as
// related work): shares R as above, p = mean(R) + std(R) z with z = Phi^-1(1 - k/n)
// (computed on the host), keep every block with R >= p; a row that keeps none keeps its
// largest share (lowest J on ties).  Sums in fp64.
//
// Kernels: mask_rows / stat_rows (one warp per row) -> bitmap [rows][nb] + counts; scan ->
// row_ptr (+ nnz); fill -> col_idx (J ascending); and for the transposed CSR
// (per key block the query blocks that keep it): tcount -> scan -> tfill.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kMaskWarps = 4;

__global__ void __launch_bounds__(kMaskWarps * 32)
    mask_rows_kernel(const float* __restrict__ p_imp, int rows, int nb, float tau,
                     uint8_t* __restrict__ bitmap, int32_t* __restrict__ counts) {
  extern __shared__ float srow_all[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* srow = srow_all + warp * nb;
  for (int row = blockIdx.x * kMaskWarps + warp; row < rows; row += gridDim.x * kMaskWarps) {
    const float* src = p_imp + static_cast<int64_t>(row) * nb;
    double part = 0.0;
    for (int J = lane; J < nb; J += 32) {
      const float v = fmaxf(src[J], 0.f);
      srow[J] = v;
      part += v;
    }
    const double total = warp_sum_d(part);
    __syncwarp();
    uint8_t* brow = bitmap + static_cast<int64_t>(row) * nb;
    if (tau >= 1.f || !(total > 0.0)) {
      for (int J = lane; J < nb; J += 32) brow[J] = 1;
      if (lane == 0) counts[row] = nb;
      continue;
    }
    const double target = static_cast<double>(tau) * total;
    // largest bit pattern u with sum_{bits(v) >= u} v >= target
    uint32_t lo = 0u, hi = 0x7f800000u;
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      double s = 0.0;
      for (int J = lane; J < nb; J += 32) {
        const float v = srow[J];
        if (__float_as_uint(v) >= mid) s += v;
      }
      s = warp_sum_d(s);
      if (s >= target) lo = mid; else hi = mid;
    }
    const float vstar = __uint_as_float(lo);
    double above = 0.0;
    for (int J = lane; J < nb; J += 32) {
      const float v = srow[J];
      if (v > vstar) above += v;
    }
    above = warp_sum_d(above);
    // blocks equal to v* are taken in J order until the target is reached
    int ntie = 0;
    for (int J0 = 0; J0 < nb; J0 += 32) {
      const int J = J0 + lane;
      ntie += __popc(__ballot_sync(0xffffffffu, J < nb && srow[J] == vstar));
    }
    int need = 0;
    for (double c = above; need < ntie && c < target; ++need) c += static_cast<double>(vstar);
    int kept = 0, ties_seen = 0;
    for (int J0 = 0; J0 < nb; J0 += 32) {
      const int J = J0 + lane;
      const float v = J < nb ? srow[J] : -1.f;
      const unsigned tmask = __ballot_sync(0xffffffffu, J < nb && v == vstar);
      const int rank = ties_seen + __popc(tmask & ((1u << lane) - 1u));
      const bool keep = J < nb && (v > vstar || (v == vstar && rank < need));
      if (J < nb) brow[J] = keep ? 1 : 0;
      kept += __popc(__ballot_sync(0xffffffffu, keep));
      ties_seen += __popc(tmask);
    }
    if (lane == 0) counts[row] = kept;
  }
}

// Statistical threshold, one warp per row; keep_all: k >= nb (every block)
__global__ void __launch_bounds__(kMaskWarps * 32)
    stat_rows_kernel(const float* __restrict__ p_imp, int rows, int nb, double z, int keep_all,
                     uint8_t* __restrict__ bitmap, int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int row = blockIdx.x * kMaskWarps + warp; row < rows; row += gridDim.x * kMaskWarps) {
    const float* src = p_imp + static_cast<int64_t>(row) * nb;
    uint8_t* brow = bitmap + static_cast<int64_t>(row) * nb;
    double part = 0.0;
    for (int J = lane; J < nb; J += 32) part += fmaxf(src[J], 0.f);
    const double total = warp_sum_d(part);
    if (keep_all || !(total > 0.0)) {
      for (int J = lane; J < nb; J += 32) brow[J] = 1;
      if (lane == 0) counts[row] = nb;
      continue;
    }
    double sr = 0.0;
    for (int J = lane; J < nb; J += 32) sr += fmaxf(src[J], 0.f) / total;
    const double mean = warp_sum_d(sr) / nb;
    double sq = 0.0;
    for (int J = lane; J < nb; J += 32) {
      const double dv = fmaxf(src[J], 0.f) / total - mean;
      sq += dv * dv;
    }
    const double thr = mean + sqrt(warp_sum_d(sq) / nb) * z;
    int kept = 0;
    float best = -1.f;
    int best_j = nb;
    for (int J0 = 0; J0 < nb; J0 += 32) {
      const int J = J0 + lane;
      const float v = J < nb ? fmaxf(src[J], 0.f) : -1.f;
      const bool keep = J < nb && static_cast<double>(v) / total >= thr;
      if (J < nb) brow[J] = keep ? 1 : 0;
      kept += __popc(__ballot_sync(0xffffffffu, keep));
      if (v > best) {  // lane-local first maximum
        best = v;
        best_j = J;
      }
    }
    if (kept == 0) {
      // the row's largest share, lowest J on ties
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oj = __shfl_xor_sync(0xffffffffu, best_j, o);
        if (ob > best || (ob == best && oj < best_j)) {
          best = ob;
          best_j = oj;
        }
      }
      if (lane == 0) brow[best_j] = 1;
      kept = 1;
    }
    if (lane == 0) counts[row] = kept;
  }
}

// Exclusive scan of n int32 counts by one CTA: out[i] = sum_{k<i} in[k], out[n] = total.
__global__ void __launch_bounds__(1024)
    scan_kernel(const int32_t* __restrict__ in, int n, int32_t* __restrict__ out,
                int32_t* __restrict__ total_out) {
  __shared__ int32_t warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  int32_t s = 0;
  for (int i = beg; i < end; ++i) s += in[i];
  int32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < (blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int32_t run = incl - s + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int i = beg; i < end; ++i) {
    out[i] = run;
    run += in[i];
  }
  if (tid == blockDim.x - 1) {
    out[n] = run;
    if (total_out) *total_out = run;
  }
}

// col_idx of each row, J ascending, from the bitmap (one warp per row)
__global__ void fill_kernel(const uint8_t* __restrict__ bitmap, const int32_t* __restrict__ row_ptr,
                            int rows, int nb, int32_t* __restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int row = blockIdx.x * wpb + (threadIdx.x >> 5); row < rows; row += gridDim.x * wpb) {
    const uint8_t* brow = bitmap + static_cast<int64_t>(row) * nb;
    int pos = row_ptr[row];
    for (int J0 = 0; J0 < nb; J0 += 32) {
      const int J = J0 + lane;
      const bool on = J < nb && brow[J];
      const unsigned m = __ballot_sync(0xffffffffu, on);
      if (on) col_idx[pos + __popc(m & ((1u << lane) - 1u))] = J;
      pos += __popc(m);
    }
  }
}

// counts_t[bh, J] = number of q-blocks I with bitmap[bh, I, J]
__global__ void tcount_kernel(const uint8_t* __restrict__ bitmap, int BH, int nb,
                              int32_t* __restrict__ counts_t) {
  const int64_t total = static_cast<int64_t>(BH) * nb;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int J = static_cast<int>(idx % nb);
    const int64_t bh = idx / nb;
    const uint8_t* base = bitmap + bh * nb * nb + J;
    int c = 0;
    for (int I = 0; I < nb; ++I) c += base[static_cast<int64_t>(I) * nb];
    counts_t[idx] = c;
  }
}

__global__ void tfill_kernel(const uint8_t* __restrict__ bitmap, const int32_t* __restrict__ col_ptr_t,
                             int BH, int nb, int32_t* __restrict__ row_idx_t) {
  const int64_t total = static_cast<int64_t>(BH) * nb;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int J = static_cast<int>(idx % nb);
    const int64_t bh = idx / nb;
    const uint8_t* base = bitmap + bh * nb * nb + J;
    int pos = col_ptr_t[idx];
    for (int I = 0; I < nb; ++I)
      if (base[static_cast<int64_t>(I) * nb]) row_idx_t[pos++] = I;
  }
}

inline unsigned grid_for(int64_t work, int per_block, int num_sms, int max_per_sm) {
  int64_t b = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * max_per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

}  // namespace

namespace {

// row_ptr / col_idx (and the transposed CSR when requested) from the bitmap and counts
cudaError_t csr_from_bitmap(const uint8_t* bitmap, int32_t* counts, int BH, int nb,
                            int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                            int32_t* counts_t, int32_t* col_ptr_t, int32_t* row_idx_t,
                            int num_sms, cudaStream_t stream) {
  const int rows = BH * nb;
  scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr, nnz_out);
  fill_kernel<<<grid_for(rows, 8, num_sms, 16), 256, 0, stream>>>(bitmap, row_ptr, rows, nb, col_idx);
  if (col_ptr_t != nullptr && row_idx_t != nullptr) {
    tcount_kernel<<<grid_for(rows, 256, num_sms, 8), 256, 0, stream>>>(bitmap, BH, nb, counts_t);
    scan_kernel<<<1, 1024, 0, stream>>>(counts_t, rows, col_ptr_t, nullptr);
    tfill_kernel<<<grid_for(rows, 256, num_sms, 8), 256, 0, stream>>>(bitmap, col_ptr_t, BH, nb,
                                                                     row_idx_t);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan(const int32_t* in, int n, int32_t* out, int32_t* total,
                        cudaStream_t stream) {
  scan_kernel<<<1, 1024, 0, stream>>>(in, n, out, total);
  return cudaGetLastError();
}

cudaError_t launch_build_mask(const float* p_imp, int BH, int nb, float tau, uint8_t* bitmap,
                              int32_t* counts, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                              int32_t* counts_t, int32_t* col_ptr_t, int32_t* row_idx_t, int num_sms,
                              cudaStream_t stream) {
  const int rows = BH * nb;
  const size_t smem = static_cast<size_t>(kMaskWarps) * nb * sizeof(float);
  cudaFuncSetAttribute(mask_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  mask_rows_kernel<<<grid_for(rows, kMaskWarps, num_sms, 16), kMaskWarps * 32, smem, stream>>>(
      p_imp, rows, nb, tau, bitmap, counts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return csr_from_bitmap(bitmap, counts, BH, nb, row_ptr, col_idx, nnz_out, counts_t, col_ptr_t,
                         row_idx_t, num_sms, stream);
}

cudaError_t launch_build_mask_stat(const float* p_imp, int BH, int nb, double z, bool keep_all,
                                   uint8_t* bitmap, int32_t* counts, int32_t* row_ptr,
                                   int32_t* col_idx, int32_t* nnz_out, int32_t* counts_t,
                                   int32_t* col_ptr_t, int32_t* row_idx_t, int num_sms,
                                   cudaStream_t stream) {
  const int rows = BH * nb;
  stat_rows_kernel<<<grid_for(rows, kMaskWarps, num_sms, 16), kMaskWarps * 32, 0, stream>>>(
      p_imp, rows, nb, z, keep_all ? 1 : 0, bitmap, counts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return csr_from_bitmap(bitmap, counts, BH, nb, row_ptr, col_idx, nnz_out, counts_t, col_ptr_t,
                         row_idx_t, num_sms, stream);
}

}  // namespace asa
