// Allocation-free variant of asa_estimate (the estimator itself is in estimate_tc.cu).
#include "../../include/asa.h"
#include "common.cuh"
#include "internal.h"

// ---------------------------------------------------------------------------------
// Allocation-free variant of asa_estimate.
//
// Some callers cannot allocate device memory at all: code embedded in a host
// application or inference engine that owns every byte of the GPU through its own
// fixed, pre-reserved pool and forbids third-party allocations, or a latency-critical
// loop that must not risk the device-wide synchronisation cudaMalloc / cudaFree can
// cause.  For them the estimator's scratch (the compact sample rows, per sample row the
// max logit of every key block and the row's log2-sum-exp) lives in one file-scope
// device array of fixed
// size.  With CUDA's lazy module loading (the default) the array is reserved on a
// device when this file's module is first loaded there, i.e. at the first call on that
// device, and held until the process exits; that first call may synchronise, so make
// it during set-up.  The caller still passes the inputs and the P_imp output.
namespace {

constexpr size_t kNoallocScratchFloats = ASA_NOALLOC_SCRATCH_BYTES / sizeof(float);
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

// Device address of the scratch array in the current context, looked up on every call
// (the host-side name of the array is not a device address).  Nothing is cached: a
// cached address would go stale when the context is torn down and re-created
// (cudaDeviceReset), and the lookup itself allocates nothing.
int noalloc_scratch(float** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return asa::record_error(ASA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s",
                             cudaGetErrorString(e));
  *out = static_cast<float*>(p);
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
  unsigned int* err_word = nullptr;
  cudaError_t e = asa::device_error_word(&err_word);
  if (e != cudaSuccess)
    return asa::record_error(ASA_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  e = asa::launch_estimate(qp, kp, B * H, N, d, scratch, p_imp, err_word, sms,
                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return asa::record_error(ASA_ERR_CUDA, "estimate launch: %s", cudaGetErrorString(e));
  return ASA_OK;
}
