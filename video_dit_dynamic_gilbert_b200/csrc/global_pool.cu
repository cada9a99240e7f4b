// Global tokens of ASA_G (Video-BLADE, "Step 2.2: Computation"): the keys and values
// are mean-pooled over windows of n consecutive permuted tokens, giving ceil(N/n)
// global tokens per head that every query attends to with a + ln(n) logit bias.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 8;

// xg[bh, g, :] = bf16(mean of xp[bh, i, :], i in [n g, min(n g + n, N))).  One CTA per
// window: its rows are one contiguous run of (rows x D) bf16, read as 16-byte chunks,
// up to eight independent loads per thread in flight (chunk c = tid + 128 k; its column
// chunk c % (D/8) = tid % (D/8), since 128 is a multiple of D/8).  Column sums are then
// added across the lanes of a warp that share a column chunk (xor shuffles over the
// lane bits above log2(D/8)) and across the four warps in shared memory.
// Blocks [0, BH G) pool xp into xg; with a second tensor (xp2 non-null), blocks
// [BH G, 2 BH G) pool xp2 into xg2 in the same launch.
__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const __nv_bfloat16* __restrict__ xp, __nv_bfloat16* __restrict__ xg,
                const __nv_bfloat16* __restrict__ xp2, __nv_bfloat16* __restrict__ xg2, int BH,
                int N, int D, int n, int G) {
  __shared__ float red[kPoolThreads / 32][16][8];
  const int CH = D / 8;
  int64_t blk = blockIdx.x;
  if (blk >= static_cast<int64_t>(BH) * G) {
    blk -= static_cast<int64_t>(BH) * G;
    xp = xp2;
    xg = xg2;
  }
  const int gi = static_cast<int>(blk % G);
  const int64_t bh = blk / G;
  const int beg = gi * n, end = min(N, beg + n);
  const int nchunk = (end - beg) * CH;
  const uint4* src = reinterpret_cast<const uint4*>(xp + (bh * N + beg) * D);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto add = [&](const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  };
  int c = tid;
  for (; c + (kPoolUnroll - 1) * kPoolThreads < nchunk; c += kPoolUnroll * kPoolThreads) {
    uint4 v[kPoolUnroll];
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) v[u] = __ldg(src + c + u * kPoolThreads);
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) add(v[u]);
  }
  for (; c < nchunk; c += kPoolThreads) add(__ldg(src + c));
  for (int o = CH; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  }
  if (lane < CH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane][e] = acc[e];
  }
  __syncthreads();
  if (tid < CH) {
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = red[0][tid][e];
#pragma unroll
    for (int w = 1; w < kPoolThreads / 32; ++w) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sum[e] += red[w][tid][e];
    }
    const float cnt = static_cast<float>(end - beg);
    uint4 out;
    uint32_t* po = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) po[e] = pack_bf16(sum[2 * e] / cnt, sum[2 * e + 1] / cnt);
    *reinterpret_cast<uint4*>(xg + (bh * G + gi) * D + tid * 8) = out;
  }
}

}  // namespace

cudaError_t launch_global_pool(const void* xp, void* xg, int BH, int N, int d, int n, int num_sms,
                               cudaStream_t stream, const void* xp2, void* xg2) {
  (void)num_sms;
  const int G = (N + n - 1) / n;
  const int64_t blocks = static_cast<int64_t>(BH) * G * (xp2 != nullptr ? 2 : 1);  // one per window
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  pool_kernel<<<static_cast<unsigned>(blocks), kPoolThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(xp), static_cast<__nv_bfloat16*>(xg),
      static_cast<const __nv_bfloat16*>(xp2), static_cast<__nv_bfloat16*>(xg2), BH, N, d, n, G);
  return cudaGetLastError();
}

}  // namespace asa
