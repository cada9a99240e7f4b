// Block-importance estimation (Video-BLADE, "Step 1: Efficient block importance
// estimation").
//
// For one head: Q_s, K_s = the k_I = min(16, L_I) evenly strided sample tokens of
// every block (offsets floor(j L_I / k_I)); P_approx = rowsoftmax(Q_s K_s^T/sqrt d);
// P_imp[I, J] = max over the k_I x k_J tile.  Softmax is monotone, so the tile max of
// P_approx is exp2(max logit of the tile - lse2 of the row), maximised over the rows
// of block I.  Two kernels:
//   est_logits: one pass of Q_s K_s^T on tensor cores; per sample row it keeps an
//     online (max, sum) in the log2 domain and writes, per key block J, the row's
//     max logit G[bh, J, r]; at the end lse2[bh, r] = m + log2(l).
//   est_pool:   P_imp[bh, I, J] = max_{r in I} exp2(G[bh, J, r] - lse2[bh, r]).
// G (16 * nb floats per key block and head) lives in the caller's workspace.
#include <mutex>

#include "../../include/asa.h"
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kEstWarps = 4;             // one warp per query block: 16 sample rows
constexpr int kEstRows = kEstWarps * 16;  // sample rows per CTA
constexpr int kEstCols = 64;              // sample columns (4 key blocks) per chunk

__device__ __forceinline__ int sample_token(int I, int j, int N, bool& valid) {
  const int L = min(kBlock, N - kBlock * I);
  const int kI = min(kSamples, L);
  valid = j < kI;
  return kBlock * I + (valid ? (j * L) / kI : 0);
}

template <int D>
__global__ void __launch_bounds__(kEstWarps * 32)
    est_logits_kernel(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
                      float* __restrict__ G, float* __restrict__ lse2, int N, int nb, float c2) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sK = sQ + kEstRows * D;  // [2][kEstCols][D]

  const int bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Mpad = kSamples * nb;
  const int Msamp = kSamples * (nb - 1) + min(kSamples, N - kBlock * (nb - 1));
  const __nv_bfloat16* qh = qp + static_cast<int64_t>(bh) * N * D;
  const __nv_bfloat16* kh = kp + static_cast<int64_t>(bh) * N * D;

  // gather this CTA's 64 sample rows of Q
  for (int idx = tid; idx < kEstRows * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    const int I = blockIdx.x * kEstWarps + row / 16;
    bool valid = false;
    int tok = 0;
    if (I < nb) tok = sample_token(I, row & 15, N, valid);
    cp_async16(smem_u32(sQ) + swz<CH>(row, ch), qh + static_cast<int64_t>(tok) * D + ch * 8, valid);
  }
  cp_async_commit();

  auto load_k_chunk = [&](int c, int stage) {
    __nv_bfloat16* dst = sK + stage * kEstCols * D;
    for (int idx = tid; idx < kEstCols * CH; idx += blockDim.x) {
      const int row = idx / CH, ch = idx - row * CH;
      const int J = c * 4 + row / 16;
      bool valid = false;
      int tok = 0;
      if (J < nb) tok = sample_token(J, row & 15, N, valid);
      cp_async16(smem_u32(dst) + swz<CH>(row, ch), kh + static_cast<int64_t>(tok) * D + ch * 8,
                 valid);
    }
    cp_async_commit();
  };

  const int nch = (nb + 3) / 4;
  load_k_chunk(0, 0);
  cp_async_wait<1>();
  __syncthreads();

  // Q fragments of this warp's 16 rows
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int row = warp * 16 + (lane & 15);
    const int ch = 2 * ks + (lane >> 4);
    ldsm_x4(smem_u32(sQ) + swz<CH>(row, ch), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }

  const int I = blockIdx.x * kEstWarps + warp;
  const int g = lane >> 2, t = lane & 3;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};

  for (int c = 0; c < nch; ++c) {
    if (c + 1 < nch) {
      load_k_chunk(c + 1, (c + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t kbase = smem_u32(sK + (c & 1) * kEstCols * D);
    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(kbase + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(acc[2 * np], qf[ks], b0, b1);
        mma_bf16(acc[2 * np + 1], qf[ks], b2, b3);
      }
    }
    // log2-domain logits; columns past the last sample are -inf
    float gmax[2][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = c * kEstCols + n * 8 + 2 * t + (e & 1);
        acc[n][e] = col < Msamp ? acc[n][e] * c2 : -INFINITY;
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v = fmaxf(fmaxf(acc[2 * jj][2 * h], acc[2 * jj][2 * h + 1]),
                        fmaxf(acc[2 * jj + 1][2 * h], acc[2 * jj + 1][2 * h + 1]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
        gmax[h][jj] = v;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float cm = fmaxf(fmaxf(gmax[h][0], gmax[h][1]), fmaxf(gmax[h][2], gmax[h][3]));
      const float mn = fmaxf(m[h], cm);  // finite: every chunk has a valid column
      float s = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) s += fast_exp2(acc[n][2 * h] - mn) + fast_exp2(acc[n][2 * h + 1] - mn);
      l[h] = l[h] * fast_exp2(m[h] - mn) + s;
      m[h] = mn;
    }
    // lane t of each quad writes key block 4c + t for the quad's two rows
    if (I < nb) {
      const int J = c * 4 + t;
      const int kI = min(kSamples, N - kBlock * I);
      if (J < nb) {
        float* gdst = G + (static_cast<int64_t>(bh) * nb + J) * Mpad + kSamples * I;
        const float v0 = t == 0 ? gmax[0][0] : t == 1 ? gmax[0][1] : t == 2 ? gmax[0][2] : gmax[0][3];
        const float v1 = t == 0 ? gmax[1][0] : t == 1 ? gmax[1][1] : t == 2 ? gmax[1][2] : gmax[1][3];
        if (g < kI) gdst[g] = v0;
        if (g + 8 < kI) gdst[g + 8] = v1;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
  }
  if (I < nb && t == 0) {
    const int kI = min(kSamples, N - kBlock * I);
    float* ldst = lse2 + static_cast<int64_t>(bh) * Mpad + kSamples * I;
    if (g < kI) ldst[g] = m[0] + __log2f(l[0]);
    if (g + 8 < kI) ldst[g + 8] = m[1] + __log2f(l[1]);
  }
}

__global__ void est_pool_kernel(const float* __restrict__ G, const float* __restrict__ lse2,
                                float* __restrict__ p_imp, int BH, int N, int nb) {
  const int64_t total = static_cast<int64_t>(BH) * nb * nb;
  const int Mpad = kSamples * nb;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int J = static_cast<int>(idx % nb);
    const int64_t rowi = idx / nb;
    const int I = static_cast<int>(rowi % nb);
    const int bh = static_cast<int>(rowi / nb);
    const int kI = min(kSamples, N - kBlock * I);
    const float4* gsrc =
        reinterpret_cast<const float4*>(G + (static_cast<int64_t>(bh) * nb + J) * Mpad + kSamples * I);
    const float4* lsrc = reinterpret_cast<const float4*>(lse2 + static_cast<int64_t>(bh) * Mpad + kSamples * I);
    float best = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 gv = __ldg(gsrc + q);
      const float4 lv = __ldg(lsrc + q);
      const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
      const float ll[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (4 * q + e < kI) best = fmaxf(best, exp2f(gg[e] - ll[e]));
    }
    p_imp[idx] = best;
  }
}

}  // namespace

size_t est_scratch_floats(int BH, int nb) {
  // G [BH][nb][16 nb] + lse2 [BH][16 nb]
  return static_cast<size_t>(BH) * nb * kSamples * nb + static_cast<size_t>(BH) * kSamples * nb;
}

cudaError_t launch_estimate(const void* qp, const void* kp, int BH, int N, int d, float* G,
                            float* lse2, float* p_imp, int num_sms, cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  const float c2 = kLog2e / sqrtf(static_cast<float>(d));
  dim3 grid((nb + kEstWarps - 1) / kEstWarps, BH);
  const size_t smem = static_cast<size_t>(kEstRows + 2 * kEstCols) * d * 2;
  if (d == 128) {
    cudaFuncSetAttribute(est_logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    est_logits_kernel<128><<<grid, kEstWarps * 32, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp), G, lse2, N, nb, c2);
  } else {
    cudaFuncSetAttribute(est_logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    est_logits_kernel<64><<<grid, kEstWarps * 32, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp), G, lse2, N, nb, c2);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = static_cast<int64_t>(BH) * nb * nb;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
  est_pool_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(G, lse2, p_imp, BH, N, nb);
  return cudaGetLastError();
}

}  // namespace asa

// ---------------------------------------------------------------------------------
// Allocation-free variant of asa_estimate.
//
// Some callers cannot allocate device memory at all: code embedded in a host
// application or inference engine that owns every byte of the GPU through its own
// fixed, pre-reserved pool and forbids third-party allocations, or a latency-critical
// loop that must not risk the device-wide synchronisation cudaMalloc / cudaFree can
// cause.  For them the estimator's scratch (per sample row, the max logit of every key
// block, and the row's log2-sum-exp) lives in one file-scope device array of fixed
// size, reserved when the library is loaded on a device and held until the process
// exits.  The caller still passes the inputs and the P_imp output.
namespace {

constexpr size_t kNoallocScratchFloats = ASA_NOALLOC_SCRATCH_BYTES / sizeof(float);
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

std::mutex g_noalloc_mu;
float* g_noalloc_addr[64] = {nullptr};

// Device address of the scratch array on the current device, looked up once per
// device (the host-side name of the array is not a device address).
int noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return asa::record_error(ASA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return asa::record_error(ASA_ERR_UNSUPPORTED, "device %d >= 64", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return asa::record_error(ASA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s",
                               cudaGetErrorString(e));
    g_noalloc_addr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_addr[dev];
  return ASA_OK;
}

}  // namespace

extern "C" int asa_estimate_noalloc(const void* qp, const void* kp, int B, int H, int N, int d,
                                    int block, int samples, float* p_imp, void* stream) {
  if (B < 1 || H < 1 || N < 1)
    return asa::record_error(ASA_ERR_INVALID_ARG, "B=%d, H=%d, N=%d must be >= 1", B, H, N);
  if (static_cast<int64_t>(B) * H > 65535 || N > ASA_MAX_TOKENS)
    return asa::record_error(ASA_ERR_UNSUPPORTED, "B*H=%lld or N=%d too large",
                             static_cast<long long>(B) * H, N);
  if (d != 64 && d != 128)
    return asa::record_error(ASA_ERR_UNSUPPORTED, "head dim d=%d not in {64,128}", d);
  if (block != ASA_BLOCK || samples != ASA_SAMPLES)
    return asa::record_error(ASA_ERR_UNSUPPORTED, "block=%d, samples=%d (only 128, 16)", block,
                             samples);
  if (qp == nullptr || kp == nullptr || p_imp == nullptr)
    return asa::record_error(ASA_ERR_INVALID_ARG, "qp, kp and p_imp must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(qp) & 15u) || (reinterpret_cast<uintptr_t>(kp) & 15u) ||
      (reinterpret_cast<uintptr_t>(p_imp) & 3u))
    return asa::record_error(ASA_ERR_INVALID_ARG, "qp/kp need 16-byte, p_imp 4-byte alignment");
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  const size_t need = asa::est_scratch_floats(B * H, nb);
  if (need > kNoallocScratchFloats)
    return asa::record_error(ASA_ERR_WORKSPACE,
                             "shape needs %zu bytes of scratch, above the fixed %zu bytes of "
                             "asa_estimate_noalloc",
                             need * sizeof(float), static_cast<size_t>(ASA_NOALLOC_SCRATCH_BYTES));
  float* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != ASA_OK) return rc;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  float* G = scratch;
  float* lse2 = scratch + static_cast<size_t>(B) * H * nb * asa::kSamplesHost * nb;
  cudaError_t e = asa::launch_estimate(qp, kp, B * H, N, d, G, lse2, p_imp, sms,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return asa::record_error(ASA_ERR_CUDA, "estimate launch: %s", cudaGetErrorString(e));
  return ASA_OK;
}
