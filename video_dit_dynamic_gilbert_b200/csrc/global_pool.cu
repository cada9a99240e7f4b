// Global tokens of ASA_G (Video-BLADE, "Step 2.2: Computation"): the keys and values
// are mean-pooled over windows of n consecutive permuted tokens, giving ceil(N/n)
// global tokens per head that every query attends to with a + ln(n) logit bias.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

// xg[bh, gidx, :] = bf16(mean of xp[bh, i, :], i in [n gidx, min(n gidx + n, N)))
__global__ void pool_kernel(const __nv_bfloat16* __restrict__ xp, __nv_bfloat16* __restrict__ xg,
                            int BH, int N, int D, int n, int G) {
  const int CH = D / 8;
  const int64_t total = static_cast<int64_t>(BH) * G * CH;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int ch = static_cast<int>(idx % CH);
    const int64_t r = idx / CH;
    const int gi = static_cast<int>(r % G);
    const int64_t bh = r / G;
    const int beg = gi * n, end = min(N, beg + n);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = beg; i < end; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xp + (bh * N + i) * D + ch * 8));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    const float cnt = static_cast<float>(end - beg);
    uint4 out;
    uint32_t* po = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) po[e] = pack_bf16(acc[2 * e] / cnt, acc[2 * e + 1] / cnt);
    *reinterpret_cast<uint4*>(xg + (bh * G + gi) * D + ch * 8) = out;
  }
}

}  // namespace

cudaError_t launch_global_pool(const void* xp, void* xg, int BH, int N, int d, int n, int num_sms,
                               cudaStream_t stream) {
  const int G = (N + n - 1) / n;
  const int64_t work = static_cast<int64_t>(BH) * G * (d / 8);
  int64_t blocks = (work + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
  if (blocks < 1) blocks = 1;
  pool_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(xp), static_cast<__nv_bfloat16*>(xg), BH, N, d, n, G);
  return cudaGetLastError();
}

}  // namespace asa
