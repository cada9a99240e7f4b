// Gilbert gather / scatter between the model layout and the permuted layout.
//
// Video-BLADE, "Preprocessing": tokens are reordered along the Gilbert curve before
// blocking; the inverse runs on the attention output.
//   permute:   xp[b, h, i, :] = x[b, perm[i], h, :]   x [B,N,H,d] -> xp [B,H,N,d]
//   unpermute: x[b, perm[i], h, :] = xp[b, h, i, :]
// With sequence parallelism the raster side may be the per-rank token chunks of an
// all-to-all buffer instead of one [B,N,H,d] tensor (same kernel, chunked row index).
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

// Row of token t of batch b in the raster side.  kChunks: per-rank token chunks back to
// back (chunk s: [B][N_s] rows of rank s's tokens, so it starts at row B * off[s]);
// otherwise the plain [B][N] raster.
template <bool kChunks>
__device__ __forceinline__ int64_t raster_row_of(int b, int t, int N, int B, const Segs& tok) {
  if constexpr (!kChunks) {
    return static_cast<int64_t>(b) * N + t;
  } else {
    int s = 0;
    while (s + 1 < tok.P && t >= tok.off[s + 1]) ++s;
    const int ns = tok.off[s + 1] - tok.off[s];
    return static_cast<int64_t>(B) * tok.off[s] + static_cast<int64_t>(b) * ns + (t - tok.off[s]);
  }
}

template <bool kToPermuted, bool kChunks>
__global__ void __launch_bounds__(kWarps * 32)
    permute_kernel(const uint4* __restrict__ src0, const uint4* __restrict__ src1,
                   const uint4* __restrict__ src2, uint4* __restrict__ dst0, uint4* __restrict__ dst1,
                   uint4* __restrict__ dst2, const int32_t* __restrict__ perm, int B, int N, int H,
                   int vec_per_head, const __grid_constant__ Segs tok) {
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
    const int64_t raster_row = raster_row_of<kChunks>(b, __ldg(perm + i), N, B, tok) * vec_per_tok;
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
  Segs none{};
  if (to_permuted)
    permute_kernel<true, false><<<grid, kWarps * 32, 0, stream>>>(
        s(0), s(1), s(2), t(0), t(1), t(2), perm_dev, B, N, H, vec_per_head, none);
  else
    permute_kernel<false, false><<<grid, kWarps * 32, 0, stream>>>(
        s(0), s(1), s(2), t(0), t(1), t(2), perm_dev, B, N, H, vec_per_head, none);
  return cudaGetLastError();
}

cudaError_t launch_permute_chunks(const void* const* src, void* const* dst, int ntensors,
                                  bool to_permuted, const int32_t* perm_dev, int B, int N, int H,
                                  int d, const Segs& tok, int num_sms, cudaStream_t stream) {
  const int vec_per_head = d / 8;
  const int64_t tokens = static_cast<int64_t>(B) * N;
  int64_t blocks = (tokens + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  dim3 grid(static_cast<unsigned>(blocks), ntensors);
  auto s = [&](int k) { return static_cast<const uint4*>(src[k < ntensors ? k : 0]); };
  auto t = [&](int k) { return static_cast<uint4*>(dst[k < ntensors ? k : 0]); };
  if (to_permuted)
    permute_kernel<true, true><<<grid, kWarps * 32, 0, stream>>>(
        s(0), s(1), s(2), t(0), t(1), t(2), perm_dev, B, N, H, vec_per_head, tok);
  else
    permute_kernel<false, true><<<grid, kWarps * 32, 0, stream>>>(
        s(0), s(1), s(2), t(0), t(1), t(2), perm_dev, B, N, H, vec_per_head, tok);
  return cudaGetLastError();
}

namespace {

// x [B][Nr][H][d] <-> head-group chunks: chunk s = [B][Nr][Hs][d] with the heads
// [heads.off[s], heads.off[s+1]), chunks back to back (chunk s starts at element
// B * Nr * heads.off[s] * d).  One warp per token row, 16-byte pieces.
template <bool kPack>
__global__ void __launch_bounds__(kWarps * 32)
    head_groups_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int B, int Nr,
                       int H, int vec_per_head, const __grid_constant__ Segs heads) {
  const int lane = threadIdx.x & 31;
  const int vec_per_tok = H * vec_per_head;
  const int64_t rows = static_cast<int64_t>(B) * Nr;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t row = warp0; row < rows; row += nwarps) {
    for (int v = lane; v < vec_per_tok; v += 32) {
      const int h = v / vec_per_head, c = v - h * vec_per_head;
      int s = 0;
      while (s + 1 < heads.P && h >= heads.off[s + 1]) ++s;
      const int hs = heads.off[s + 1] - heads.off[s];
      const int64_t chunk = rows * heads.off[s] * vec_per_head +
                            (row * hs + (h - heads.off[s])) * vec_per_head + c;
      const int64_t flat = row * vec_per_tok + v;
      if (kPack)
        dst[chunk] = __ldcs(src + flat);
      else
        dst[flat] = __ldcs(src + chunk);
    }
  }
}

}  // namespace

cudaError_t launch_head_groups(const void* src, void* dst, bool pack, int B, int Nr, int H, int d,
                               const Segs& heads, int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(B) * Nr;
  int64_t blocks = (rows + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const auto* s = static_cast<const uint4*>(src);
  auto* t = static_cast<uint4*>(dst);
  if (pack)
    head_groups_kernel<true><<<static_cast<unsigned>(blocks), kWarps * 32, 0, stream>>>(
        s, t, B, Nr, H, d / 8, heads);
  else
    head_groups_kernel<false><<<static_cast<unsigned>(blocks), kWarps * 32, 0, stream>>>(
        s, t, B, Nr, H, d / 8, heads);
  return cudaGetLastError();
}

}  // namespace asa
