// Gilbert gather / scatter between the model layout and the permuted layout.
//
// Video-BLADE, "Preprocessing": tokens are reordered along the Gilbert curve before
// blocking; the inverse runs on the attention output.
//   permute:   xp[b, h, i, :] = x[b, perm[i], h, :]   x [B,N,H,d] -> xp [B,H,N,d]
//   unpermute: x[b, perm[i], h, :] = xp[b, h, i, :]
// Pure data movement, bound by HBM: each token moves H*d*2 bytes in and out.  One
// warp moves one token: the raster side is one contiguous H*d*2-byte row, the
// permuted side is H rows of d*2 contiguous bytes, so both sides are read and
// written in whole 32-byte sectors with 16-byte vector accesses.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kWarps = 8;
constexpr int kInflight = 8;  // 16-byte vectors per lane in flight

template <bool kToPermuted>
__global__ void __launch_bounds__(kWarps * 32)
    permute_kernel(const uint4* __restrict__ src0, const uint4* __restrict__ src1,
                   const uint4* __restrict__ src2, uint4* __restrict__ dst0, uint4* __restrict__ dst1,
                   uint4* __restrict__ dst2, const int32_t* __restrict__ perm, int B, int N, int H,
                   int vec_per_head) {
  const uint4* src = blockIdx.y == 0 ? src0 : (blockIdx.y == 1 ? src1 : src2);
  uint4* dst = blockIdx.y == 0 ? dst0 : (blockIdx.y == 1 ? dst1 : dst2);
  const int lane = threadIdx.x & 31;
  const int vec_per_tok = H * vec_per_head;
  const int64_t total = static_cast<int64_t>(B) * N;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t t = warp0; t < total; t += nwarps) {
    const int b = static_cast<int>(t / N);
    const int i = static_cast<int>(t - static_cast<int64_t>(b) * N);
    const int64_t raster_row = (static_cast<int64_t>(b) * N + __ldg(perm + i)) * vec_per_tok;
    for (int v0 = 0; v0 < vec_per_tok; v0 += 32 * kInflight) {
      uint4 buf[kInflight];
#pragma unroll
      for (int u = 0; u < kInflight; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vec_per_tok) {
          const int h = v / vec_per_head;
          const int c = v - h * vec_per_head;
          const int64_t head_row =
              ((static_cast<int64_t>(b) * H + h) * N + i) * vec_per_head + c;
          buf[u] = kToPermuted ? __ldcs(src + raster_row + v) : __ldcs(src + head_row);
        }
      }
#pragma unroll
      for (int u = 0; u < kInflight; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vec_per_tok) {
          const int h = v / vec_per_head;
          const int c = v - h * vec_per_head;
          const int64_t head_row =
              ((static_cast<int64_t>(b) * H + h) * N + i) * vec_per_head + c;
          if (kToPermuted)
            dst[head_row] = buf[u];
          else
            dst[raster_row + v] = buf[u];
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute(const void* const* src, void* const* dst, int ntensors, bool to_permuted,
                           const int32_t* perm_dev, int B, int N, int H, int d, int num_sms,
                           cudaStream_t stream) {
  const int vec_per_head = d / 8;
  const int64_t tokens = static_cast<int64_t>(B) * N;
  int64_t blocks = (tokens + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  dim3 grid(static_cast<unsigned>(blocks), ntensors);
  auto s = [&](int k) { return static_cast<const uint4*>(src[k < ntensors ? k : 0]); };
  auto t = [&](int k) { return static_cast<uint4*>(dst[k < ntensors ? k : 0]); };
  if (to_permuted)
    permute_kernel<true><<<grid, kWarps * 32, 0, stream>>>(s(0), s(1), s(2), t(0), t(1), t(2),
                                                           perm_dev, B, N, H, vec_per_head);
  else
    permute_kernel<false><<<grid, kWarps * 32, 0, stream>>>(s(0), s(1), s(2), t(0), t(1), t(2),
                                                            perm_dev, B, N, H, vec_per_head);
  return cudaGetLastError();
}

}  // namespace asa
