// C ABI of libasa.so (declarations and contracts in include/asa.h).
//
// Every entry point validates its arguments on the host before it launches
// anything, carves the caller's workspace, and launches the kernels of its step on
// the caller's stream.  The library owns only the per-shape Gilbert permutation table
// (built on the host once per (device, T, Hg, W) and uploaded) and, per device, the
// three streams and the events of the pipelined host-buffer call.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/asa.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(ASA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int num_sms_current() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

std::mutex g_perm_mu;
std::map<std::tuple<int, int, int, int>, int32_t*> g_perm_cache;

// Device copy of the Gilbert table for the current device (built once per shape).
int get_perm(int T, int Hg, int W, const int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_perm_mu);
  auto key = std::make_tuple(dev, T, Hg, W);
  auto it = g_perm_cache.find(key);
  if (it != g_perm_cache.end()) {
    *out = it->second;
    return ASA_OK;
  }
  const size_t N = static_cast<size_t>(T) * Hg * W;
  std::vector<int32_t> host(N);
  if (!asa::gilbert_order_host(T, Hg, W, host.data()))
    return fail(ASA_ERR_INVALID_ARG, "gilbert order failed for %dx%dx%d", T, Hg, W);
  int32_t* d = nullptr;
  e = cudaMalloc(&d, N * sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(permutation table)");
  e = cudaMemcpy(d, host.data(), N * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(d);
    return cuda_fail(e, "cudaMemcpy(permutation table)");
  }
  g_perm_cache[key] = d;
  *out = d;
  return ASA_OK;
}

int check_common(int B, int H, int N, int d) {
  if (B < 1 || H < 1) return fail(ASA_ERR_INVALID_ARG, "B=%d and H=%d must be >= 1", B, H);
  if (static_cast<int64_t>(B) * H > 65535)
    return fail(ASA_ERR_UNSUPPORTED, "B*H=%lld exceeds 65535", static_cast<long long>(B) * H);
  if (N < 1) return fail(ASA_ERR_INVALID_ARG, "N=%d must be >= 1", N);
  if (N > ASA_MAX_TOKENS) return fail(ASA_ERR_UNSUPPORTED, "N=%d exceeds %d", N, ASA_MAX_TOKENS);
  if (d != 64 && d != 128) return fail(ASA_ERR_UNSUPPORTED, "head dim d=%d not in {64,128}", d);
  return ASA_OK;
}

int check_grid(int T, int Hg, int W, int64_t* N) {
  if (T < 1 || Hg < 1 || W < 1)
    return fail(ASA_ERR_INVALID_ARG, "grid %dx%dx%d: sides must be >= 1", T, Hg, W);
  const int64_t n = static_cast<int64_t>(T) * Hg * W;
  if (n > ASA_MAX_TOKENS)
    return fail(ASA_ERR_UNSUPPORTED, "grid %dx%dx%d has %lld > %d tokens", T, Hg, W,
                static_cast<long long>(n), ASA_MAX_TOKENS);
  *N = n;
  return ASA_OK;
}

int check_ptr(const void* p, const char* name, bool need16 = true) {
  if (p == nullptr) return fail(ASA_ERR_INVALID_ARG, "%s is NULL", name);
  if (need16 && !aligned16(p)) return fail(ASA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  if (!need16 && (reinterpret_cast<uintptr_t>(p) & 3u))
    return fail(ASA_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);
  return ASA_OK;
}

#define ASA_TRY(x)          \
  do {                      \
    const int rc__ = (x);   \
    if (rc__ != ASA_OK) return rc__; \
  } while (0)

struct MaskWs {
  float* est;  // estimator scratch
  float* p_imp;
  uint8_t* bitmap;
  int32_t* counts;
  int32_t* counts_t;
  size_t bytes;
};

MaskWs carve_mask_ws(void* base, int BH, int nb) {
  MaskWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += align256(n);
    return o;
  };
  const size_t o_g = take(asa::est_scratch_floats(BH, nb) * sizeof(float) + 256);
  const size_t o_p = take(static_cast<size_t>(BH) * nb * nb * sizeof(float));
  const size_t o_b = take(static_cast<size_t>(BH) * nb * nb);
  const size_t o_c = take(static_cast<size_t>(BH) * nb * sizeof(int32_t));
  const size_t o_t = take(static_cast<size_t>(BH) * nb * sizeof(int32_t));
  w.bytes = off;
  if (base) {
    char* b = static_cast<char*>(base);
    w.est = reinterpret_cast<float*>(b + o_g);
    w.p_imp = reinterpret_cast<float*>(b + o_p);
    w.bitmap = reinterpret_cast<uint8_t*>(b + o_b);
    w.counts = reinterpret_cast<int32_t*>(b + o_c);
    w.counts_t = reinterpret_cast<int32_t*>(b + o_t);
  }
  return w;
}

int check_ws(const void* ws, size_t have, size_t need) {
  if (need == 0) return ASA_OK;
  if (ws == nullptr) return fail(ASA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(ASA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (have < need) return fail(ASA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
  return ASA_OK;
}

int check_block(int block, int samples) {
  if (block != ASA_BLOCK) return fail(ASA_ERR_UNSUPPORTED, "block=%d (only 128)", block);
  if (samples != ASA_SAMPLES) return fail(ASA_ERR_UNSUPPORTED, "samples=%d (only 16)", samples);
  return ASA_OK;
}

}  // namespace

__device__ unsigned int g_device_error = 0;

namespace asa {
int record_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}
}  // namespace asa

namespace asa {
// Device address of g_device_error for the current device (kernels set bits in it
// when a bounded wait expires).
cudaError_t device_error_word(unsigned int** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
  *out = static_cast<unsigned int*>(p);
  return e;
}
}  // namespace asa
using asa::device_error_word;

extern "C" {

int asa_version(void) { return 100; }

const char* asa_last_error_string(void) { return g_last_error.c_str(); }

int asa_gilbert_index(int T, int Hg, int W, int32_t* perm_host) {
  int64_t N = 0;
  ASA_TRY(check_grid(T, Hg, W, &N));
  ASA_TRY(check_ptr(perm_host, "perm_host", false));
  if (!asa::gilbert_order_host(T, Hg, W, perm_host))
    return fail(ASA_ERR_INVALID_ARG, "gilbert order failed for %dx%dx%d", T, Hg, W);
  return ASA_OK;
}

static int permute_impl(const void* const* src, void* const* dst, int nt, bool to_perm, int B,
                        int T, int Hg, int W, int H, int d, void* stream) {
  int64_t N = 0;
  ASA_TRY(check_grid(T, Hg, W, &N));
  ASA_TRY(check_common(B, H, static_cast<int>(N), d));
  for (int k = 0; k < nt; ++k) {
    ASA_TRY(check_ptr(src[k], "input"));
    ASA_TRY(check_ptr(dst[k], "output"));
    if (src[k] == dst[k]) return fail(ASA_ERR_INVALID_ARG, "input and output alias");
  }
  const int32_t* perm = nullptr;
  ASA_TRY(get_perm(T, Hg, W, &perm));
  cudaError_t e = asa::launch_permute(src, dst, nt, to_perm, perm, B, static_cast<int>(N), H, d,
                                      num_sms_current(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, to_perm ? "permute launch" : "unpermute launch");
  return ASA_OK;
}

int asa_gilbert_permute(const void* x, void* xp, int B, int T, int Hg, int W, int H, int d,
                        void* stream) {
  const void* s[1] = {x};
  void* t[1] = {xp};
  return permute_impl(s, t, 1, true, B, T, Hg, W, H, d, stream);
}

int asa_gilbert_permute3(const void* x0, const void* x1, const void* x2, void* xp0, void* xp1,
                         void* xp2, int B, int T, int Hg, int W, int H, int d, void* stream) {
  const void* s[3] = {x0, x1, x2};
  void* t[3] = {xp0, xp1, xp2};
  return permute_impl(s, t, 3, true, B, T, Hg, W, H, d, stream);
}

int asa_unpermute(const void* xp, void* x, int B, int T, int Hg, int W, int H, int d, void* stream) {
  const void* s[1] = {xp};
  void* t[1] = {x};
  return permute_impl(s, t, 1, false, B, T, Hg, W, H, d, stream);
}

size_t asa_estimate_mask_workspace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1 || N > ASA_MAX_TOKENS) return 0;
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  return carve_mask_ws(nullptr, B * H, nb).bytes;
}

int asa_estimate(const void* qp, const void* kp, int B, int H, int N, int d, int block, int samples,
                 void* workspace, size_t ws_bytes, float* p_imp, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, samples));
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(p_imp, "p_imp", false));
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  MaskWs w = carve_mask_ws(workspace, B * H, nb);
  ASA_TRY(check_ws(workspace, ws_bytes, w.bytes));
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_estimate(qp, kp, B * H, N, d, w.est, p_imp, err_word, num_sms_current(),
                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "estimate launch");
  return ASA_OK;
}

static int build_mask_impl(const float* p_imp, int B, int H, int N, float tau, const MaskWs& w,
                           int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                           int32_t* col_ptr_t, int32_t* row_idx_t, void* stream) {
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  cudaError_t e = asa::launch_build_mask(p_imp, B * H, nb, tau, w.bitmap, w.counts, row_ptr, col_idx,
                                         nnz_out, w.counts_t, col_ptr_t, row_idx_t,
                                         num_sms_current(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mask launch");
  return ASA_OK;
}

static int check_mask_args(float tau, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                           int32_t* col_ptr_t, int32_t* row_idx_t) {
  if (!(tau > 0.f)) return fail(ASA_ERR_INVALID_ARG, "tau=%g must be > 0", static_cast<double>(tau));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(nnz_out, "nnz_out", false));
  if ((col_ptr_t == nullptr) != (row_idx_t == nullptr))
    return fail(ASA_ERR_INVALID_ARG, "col_ptr_t and row_idx_t must both be set or both NULL");
  if (col_ptr_t) {
    ASA_TRY(check_ptr(col_ptr_t, "col_ptr_t", false));
    ASA_TRY(check_ptr(row_idx_t, "row_idx_t", false));
  }
  return ASA_OK;
}

int asa_build_mask(const float* p_imp, int B, int H, int N, float tau, void* workspace,
                   size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                   int32_t* col_ptr_t, int32_t* row_idx_t, void* stream) {
  ASA_TRY(check_common(B, H, N, 64));
  ASA_TRY(check_ptr(p_imp, "p_imp", false));
  ASA_TRY(check_mask_args(tau, row_ptr, col_idx, nnz_out, col_ptr_t, row_idx_t));
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  MaskWs w = carve_mask_ws(workspace, B * H, nb);
  ASA_TRY(check_ws(workspace, ws_bytes, w.bytes));
  return build_mask_impl(p_imp, B, H, N, tau, w, row_ptr, col_idx, nnz_out, col_ptr_t, row_idx_t,
                         stream);
}

// Phi^-1(p) for 0 < p < 1: bisection on the standard normal CDF 0.5 erfc(-x / sqrt 2),
// to the resolution of double
static double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200 && hi - lo > 1e-15 * (1.0 + std::fabs(lo)); ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

int asa_build_mask_stat(const float* p_imp, int B, int H, int N, int k_target, void* workspace,
                        size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                        int32_t* col_ptr_t, int32_t* row_idx_t, void* stream) {
  ASA_TRY(check_common(B, H, N, 64));
  ASA_TRY(check_ptr(p_imp, "p_imp", false));
  if (k_target < 1) return fail(ASA_ERR_INVALID_ARG, "k_target=%d must be >= 1", k_target);
  ASA_TRY(check_mask_args(1.f, row_ptr, col_idx, nnz_out, col_ptr_t, row_idx_t));
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  MaskWs w = carve_mask_ws(workspace, B * H, nb);
  ASA_TRY(check_ws(workspace, ws_bytes, w.bytes));
  const bool keep_all = k_target >= nb;
  const double z = keep_all ? 0.0 : normal_quantile(1.0 - static_cast<double>(k_target) / nb);
  cudaError_t e = asa::launch_build_mask_stat(p_imp, B * H, nb, z, keep_all, w.bitmap, w.counts,
                                              row_ptr, col_idx, nnz_out, w.counts_t, col_ptr_t,
                                              row_idx_t, num_sms_current(),
                                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mask launch");
  return ASA_OK;
}

int asa_estimate_mask(const void* qp, const void* kp, int B, int H, int N, int d, int block,
                      int samples, float tau, void* workspace, size_t ws_bytes, int32_t* row_ptr,
                      int32_t* col_idx, int32_t* nnz_out, int32_t* col_ptr_t, int32_t* row_idx_t,
                      void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, samples));
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_mask_args(tau, row_ptr, col_idx, nnz_out, col_ptr_t, row_idx_t));
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  MaskWs w = carve_mask_ws(workspace, B * H, nb);
  ASA_TRY(check_ws(workspace, ws_bytes, w.bytes));
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_estimate(qp, kp, B * H, N, d, w.est, w.p_imp, err_word, num_sms_current(),
                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "estimate launch");
  return build_mask_impl(w.p_imp, B, H, N, tau, w, row_ptr, col_idx, nnz_out, col_ptr_t, row_idx_t,
                         stream);
}

int asa_global_pool_kv(const void* kp, const void* vp, void* kg, void* vg, int B, int H, int N,
                       int d, int n, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(vp, "vp"));
  ASA_TRY(check_ptr(kg, "kg"));
  ASA_TRY(check_ptr(vg, "vg"));
  if (n < 1) return fail(ASA_ERR_INVALID_ARG, "global window n=%d must be >= 1", n);
  cudaError_t e = asa::launch_global_pool(kp, kg, B * H, N, d, n, num_sms_current(),
                                          static_cast<cudaStream_t>(stream), vp, vg);
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  return ASA_OK;
}

int asa_global_pool(const void* xp, void* xg, int B, int H, int N, int d, int n, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_ptr(xp, "xp"));
  ASA_TRY(check_ptr(xg, "xg"));
  if (n < 1) return fail(ASA_ERR_INVALID_ARG, "global window n=%d must be >= 1", n);
  cudaError_t e = asa::launch_global_pool(xp, xg, B * H, N, d, n, num_sms_current(),
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  return ASA_OK;
}

size_t asa_fwd_workspace_size(int B, int H, int N, int d, int global_window) {
  if (B < 1 || H < 1 || N < 1 || global_window < 0) return 0;
  const size_t nb = (static_cast<size_t>(N) + ASA_BLOCK - 1) / ASA_BLOCK;
  size_t bytes = align256(static_cast<size_t>(B) * H * nb * sizeof(int32_t));  // launch order
  if (global_window > 0) {
    const size_t G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    bytes += 2 * align256(static_cast<size_t>(B) * H * G * d * 2);
  }
  return bytes;
}

// perm_out != nullptr: O in raster layout [B, N, H, d] (token perm_out[i] for row i)
static int fwd_impl(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                    const int32_t* col_idx, int B, int H, int N, int d, int block,
                    int global_window, void* workspace, size_t ws_bytes, void* o, float* lse,
                    const int32_t* perm_out, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(vp, "vp"));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(o, "o"));
  ASA_TRY(check_ptr(lse, "lse", false));
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  const size_t need = asa_fwd_workspace_size(B, H, N, d, global_window);
  ASA_TRY(check_ws(workspace, ws_bytes, need));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* kg = nullptr;
  const void* vg = nullptr;
  const size_t nb = (static_cast<size_t>(N) + ASA_BLOCK - 1) / ASA_BLOCK;
  int32_t* order = static_cast<int32_t*>(workspace);
  if (global_window > 0) {
    const size_t G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    char* base = static_cast<char*>(workspace) + align256(static_cast<size_t>(B) * H * nb * sizeof(int32_t));
    void* kgw = base;
    void* vgw = base + align256(static_cast<size_t>(B) * H * G * d * 2);
    cudaError_t e = asa::launch_global_pool(kp, kgw, B * H, N, d, global_window, num_sms_current(),
                                            s, vp, vgw);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    kg = kgw;
    vg = vgw;
  }
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_fwd_tc(qp, kp, vp, row_ptr, col_idx, kg, vg, order, B * H, N, d, global_window, o,
                         lse, err_word, s, perm_out, H);
  if (e != cudaSuccess) return cuda_fail(e, "forward launch");
  return ASA_OK;
}

int asa_sparse_attn_fwd(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                        const int32_t* col_idx, int B, int H, int N, int d, int block,
                        int global_window, void* workspace, size_t ws_bytes, void* o, float* lse,
                        void* stream) {
  return fwd_impl(qp, kp, vp, row_ptr, col_idx, B, H, N, d, block, global_window, workspace,
                  ws_bytes, o, lse, nullptr, stream);
}

int asa_sparse_attn_fwd_raster(const void* qp, const void* kp, const void* vp,
                               const int32_t* row_ptr, const int32_t* col_idx, int B, int T,
                               int Hg, int W, int H, int d, int block, int global_window,
                               void* workspace, size_t ws_bytes, void* o, float* lse,
                               void* stream) {
  int64_t N = 0;
  ASA_TRY(check_grid(T, Hg, W, &N));
  ASA_TRY(check_common(B, H, static_cast<int>(N), d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(vp, "vp"));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(o, "o"));
  ASA_TRY(check_ptr(lse, "lse", false));
  if (o == qp || o == kp || o == vp) return fail(ASA_ERR_INVALID_ARG, "o aliases an input");
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  // every host-side check before the permutation table is looked up on the device
  ASA_TRY(check_ws(workspace, ws_bytes,
                   asa_fwd_workspace_size(B, H, static_cast<int>(N), d, global_window)));
  const int32_t* perm = nullptr;
  ASA_TRY(get_perm(T, Hg, W, &perm));
  return fwd_impl(qp, kp, vp, row_ptr, col_idx, B, H, static_cast<int>(N), d, block,
                  global_window, workspace, ws_bytes, o, lse, perm, stream);
}

size_t asa_fwd_train_workspace_size(int B, int H, int N, int d, int global_window) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128) || global_window < 0) return 0;
  size_t bytes = asa_fwd_workspace_size(B, H, N, d, global_window);
  bytes += align256(static_cast<size_t>(B) * H * N * d * 2);  // fp16 V
  if (global_window > 0) {
    const size_t G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    bytes += align256(static_cast<size_t>(B) * H * G * d * 2);  // fp16 global V tokens
  }
  return bytes;
}

int asa_sparse_attn_fwd_train(const void* qp, const void* kp, const void* vp,
                              const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N,
                              int d, int block, int global_window, void* workspace,
                              size_t ws_bytes, void* o, float* lse, float* o32, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(vp, "vp"));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(o, "o"));
  ASA_TRY(check_ptr(lse, "lse", false));
  ASA_TRY(check_ptr(o32, "o32"));
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  const size_t need = asa_fwd_train_workspace_size(B, H, N, d, global_window);
  ASA_TRY(check_ws(workspace, ws_bytes, need));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current();
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  // workspace: launch order, [global K and V tokens,] fp16 V, [fp16 global V tokens]
  char* base = static_cast<char*>(workspace);
  const size_t nb = (static_cast<size_t>(N) + ASA_BLOCK - 1) / ASA_BLOCK;
  int32_t* order = reinterpret_cast<int32_t*>(base);
  size_t off = align256(static_cast<size_t>(B) * H * nb * sizeof(int32_t));
  const void* kg = nullptr;
  void* vg = nullptr;
  size_t G = 0;
  if (global_window > 0) {
    G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    void* kgw = base + off;
    off += align256(static_cast<size_t>(B) * H * G * d * 2);
    vg = base + off;
    off += align256(static_cast<size_t>(B) * H * G * d * 2);
    e = asa::launch_global_pool(kp, kgw, B * H, N, d, global_window, sms, s, vp, vg);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    kg = kgw;
  }
  void* v16 = base + off;
  off += align256(static_cast<size_t>(B) * H * N * d * 2);
  e = asa::launch_f16_copy(vp, v16, static_cast<int64_t>(B) * H * N * d, err_word, sms, s);
  void* vg16 = nullptr;
  if (e == cudaSuccess && global_window > 0) {
    vg16 = base + off;
    e = asa::launch_f16_copy(vg, vg16, static_cast<int64_t>(B) * H * G * d, err_word, sms, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "fp16 copy launch");
  e = asa::launch_fwd_tc_train(qp, kp, v16, row_ptr, col_idx, kg, vg16, order, B * H, N, d,
                               global_window, o, lse, o32, err_word, s);
  if (e != cudaSuccess) return cuda_fail(e, "forward launch");
  return ASA_OK;
}

size_t asa_bwd_workspace_size(int B, int H, int N, int d, int global_window) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128) || global_window < 0) return 0;
  return asa::bwd_tc_workspace_bytes(B * H, N, d, global_window);
}

static int bwd_impl(const void* qp, const void* kp, const void* vp, const void* o,
                    const void* dout, const float* lse, const int32_t* row_ptr,
                    const int32_t* col_idx, const int32_t* col_ptr_t, const int32_t* row_idx_t,
                    int B, int H, int N, int d, int block, int global_window, void* workspace,
                    size_t ws_bytes, void* dq, void* dk, void* dv, void* stream, bool d_from_o,
                    bool o_f32 = false) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  const void* bf[] = {qp, kp, vp, o, dout, dq, dk, dv};
  const char* names[] = {"qp", "kp", "vp", o_f32 ? "o32" : "o", "dout", "dq", "dk", "dv"};
  for (int k = 0; k < 8; ++k) ASA_TRY(check_ptr(bf[k], names[k]));
  ASA_TRY(check_ptr(lse, "lse", false));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(col_ptr_t, "col_ptr_t", false));
  ASA_TRY(check_ptr(row_idx_t, "row_idx_t", false));
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  const size_t need = asa_bwd_workspace_size(B, H, N, d, global_window);
  ASA_TRY(check_ws(workspace, ws_bytes, need));
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_bwd_tc(qp, kp, vp, dout, lse, row_ptr, col_idx, col_ptr_t, row_idx_t, B * H, N,
                         d, global_window, workspace, dq, dk, dv, err_word, num_sms_current(),
                         static_cast<cudaStream_t>(stream), d_from_o ? o : nullptr, o_f32);
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return ASA_OK;
}

int asa_sparse_attn_bwd(const void* qp, const void* kp, const void* vp, const void* o,
                        const void* dout, const float* lse, const int32_t* row_ptr,
                        const int32_t* col_idx, const int32_t* col_ptr_t,
                        const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                        int global_window, void* workspace, size_t ws_bytes, void* dq, void* dk,
                        void* dv, void* stream) {
  return bwd_impl(qp, kp, vp, o, dout, lse, row_ptr, col_idx, col_ptr_t, row_idx_t, B, H, N, d,
                  block, global_window, workspace, ws_bytes, dq, dk, dv, stream, false);
}

int asa_sparse_attn_bwd_d_from_o(const void* qp, const void* kp, const void* vp, const void* o,
                                 const void* dout, const float* lse, const int32_t* row_ptr,
                                 const int32_t* col_idx, const int32_t* col_ptr_t,
                                 const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                                 int global_window, void* workspace, size_t ws_bytes, void* dq,
                                 void* dk, void* dv, void* stream) {
  return bwd_impl(qp, kp, vp, o, dout, lse, row_ptr, col_idx, col_ptr_t, row_idx_t, B, H, N, d,
                  block, global_window, workspace, ws_bytes, dq, dk, dv, stream, true);
}

int asa_sparse_attn_bwd_train(const void* qp, const void* kp, const void* vp, const float* o32,
                              const void* dout, const float* lse, const int32_t* row_ptr,
                              const int32_t* col_idx, const int32_t* col_ptr_t,
                              const int32_t* row_idx_t, int B, int H, int N, int d, int block,
                              int global_window, void* workspace, size_t ws_bytes, void* dq,
                              void* dk, void* dv, void* stream) {
  return bwd_impl(qp, kp, vp, o32, dout, lse, row_ptr, col_idx, col_ptr_t, row_idx_t, B, H, N, d,
                  block, global_window, workspace, ws_bytes, dq, dk, dv, stream, true, true);
}

// ---------------------------------------------------------------- query pruning (BSA)

namespace {

int prune_kept_max(float r, int window) {
  return std::max(static_cast<int>(std::ceil(static_cast<double>(r) * ASA_BLOCK)),
                  (ASA_BLOCK + window - 1) / window);
}

int check_prune(float r, int window) {
  if (!(r >= 0.f && r <= 1.f)) return fail(ASA_ERR_INVALID_ARG, "keep ratio r=%g not in [0, 1]", r);
  if (window < 1 || window > ASA_BLOCK)
    return fail(ASA_ERR_INVALID_ARG, "window=%d not in [1, %d]", window, ASA_BLOCK);
  return ASA_OK;
}

int check_pack(int pack) {
  if (pack != 1 && pack != 2 && pack != 4)
    return fail(ASA_ERR_INVALID_ARG, "pack=%d not in {1, 2, 4}", pack);
  return ASA_OK;
}

size_t prune_tiles(int B, int H, int N, int pack) {
  const size_t nb = (static_cast<size_t>(N) + ASA_BLOCK - 1) / ASA_BLOCK;
  return static_cast<size_t>(B) * H * ((nb + pack - 1) / pack);
}

}  // namespace

int asa_prune_pack(float r, int window) {
  ASA_TRY(check_prune(r, window));
  const int k = prune_kept_max(r, window);
  return k <= ASA_BLOCK / 4 ? 4 : (k <= ASA_BLOCK / 2 ? 2 : 1);
}

int asa_prune_rows(int N, int pack) {
  if (N < 1 || N > ASA_MAX_TOKENS) return fail(ASA_ERR_INVALID_ARG, "N=%d not in [1, %d]", N, ASA_MAX_TOKENS);
  ASA_TRY(check_pack(pack));
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  return (nb + pack - 1) / pack * ASA_BLOCK;
}

int asa_prune_queries(const void* qp, int B, int H, int N, int d, int block, float r, int window,
                      int pack, void* q_s, int32_t* src_pos, int32_t* src_row, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_prune(r, window));
  ASA_TRY(check_pack(pack));
  if (pack > asa_prune_pack(r, window))
    return fail(ASA_ERR_INVALID_ARG, "pack=%d: a block keeps up to %d queries, more than 128/%d",
                pack, prune_kept_max(r, window), pack);
  ASA_TRY(check_ptr(qp, "qp"));
  ASA_TRY(check_ptr(q_s, "q_s"));
  ASA_TRY(check_ptr(src_pos, "src_pos", false));
  ASA_TRY(check_ptr(src_row, "src_row", false));
  const int Ns = asa_prune_rows(N, pack);
  cudaError_t e = asa::launch_prune(qp, B * H, N, d, r, window, pack, q_s, Ns, src_pos, src_row,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prune launch");
  return ASA_OK;
}

size_t asa_prune_mask_workspace_size(int B, int H, int N, int pack) {
  if (B < 1 || H < 1 || N < 1 || N > ASA_MAX_TOKENS || (pack != 1 && pack != 2 && pack != 4))
    return 0;
  return align256(prune_tiles(B, H, N, pack) * sizeof(int32_t));
}

int asa_prune_mask(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N, int pack,
                   void* workspace, size_t ws_bytes, int32_t* tile_ptr, int32_t* tile_col,
                   uint8_t* tile_quarters, int32_t* nnz_out, void* stream) {
  ASA_TRY(check_common(B, H, N, 64));
  ASA_TRY(check_pack(pack));
  ASA_TRY(check_ptr(row_ptr, "row_ptr", false));
  ASA_TRY(check_ptr(col_idx, "col_idx", false));
  ASA_TRY(check_ptr(tile_ptr, "tile_ptr", false));
  ASA_TRY(check_ptr(tile_col, "tile_col", false));
  if (tile_quarters == nullptr) return fail(ASA_ERR_INVALID_ARG, "tile_quarters is NULL");
  ASA_TRY(check_ptr(nnz_out, "nnz_out", false));
  ASA_TRY(check_ws(workspace, ws_bytes, asa_prune_mask_workspace_size(B, H, N, pack)));
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  const int nb = (N + ASA_BLOCK - 1) / ASA_BLOCK;
  e = asa::launch_prune_mask(row_ptr, col_idx, B * H, nb, pack, static_cast<int32_t*>(workspace),
                             tile_ptr, tile_col, tile_quarters, nnz_out, err_word,
                             num_sms_current(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prune mask launch");
  return ASA_OK;
}

size_t asa_fwd_pruned_workspace_size(int B, int H, int N, int d, int pack, int global_window) {
  if (B < 1 || H < 1 || N < 1 || N > ASA_MAX_TOKENS || (d != 64 && d != 128) ||
      (pack != 1 && pack != 2 && pack != 4) || global_window < 0)
    return 0;
  const size_t tiles = prune_tiles(B, H, N, pack);
  const size_t rows = tiles * ASA_BLOCK;  // B*H*Ns
  size_t bytes = align256(tiles * sizeof(int32_t)) + align256(rows * d * 2) +
                 align256(rows * sizeof(float));
  if (global_window > 0) {
    const size_t G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    bytes += 2 * align256(static_cast<size_t>(B) * H * G * d * 2);
  }
  return bytes;
}

int asa_sparse_attn_fwd_pruned(const void* q_s, const void* kp, const void* vp,
                               const int32_t* tile_ptr, const int32_t* tile_col,
                               const uint8_t* tile_quarters, const int32_t* src_row, int B, int H,
                               int N, int d, int block, int pack, int global_window,
                               void* workspace, size_t ws_bytes, void* o, float* lse,
                               void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_pack(pack));
  ASA_TRY(check_ptr(q_s, "q_s"));
  ASA_TRY(check_ptr(kp, "kp"));
  ASA_TRY(check_ptr(vp, "vp"));
  ASA_TRY(check_ptr(tile_ptr, "tile_ptr", false));
  ASA_TRY(check_ptr(tile_col, "tile_col", false));
  if (tile_quarters == nullptr) return fail(ASA_ERR_INVALID_ARG, "tile_quarters is NULL");
  ASA_TRY(check_ptr(src_row, "src_row", false));
  ASA_TRY(check_ptr(o, "o"));
  ASA_TRY(check_ptr(lse, "lse", false));
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  ASA_TRY(check_ws(workspace, ws_bytes, asa_fwd_pruned_workspace_size(B, H, N, d, pack, global_window)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const int Ns = asa_prune_rows(N, pack);
  const size_t tiles = prune_tiles(B, H, N, pack);
  char* p = static_cast<char*>(workspace);
  int32_t* order = reinterpret_cast<int32_t*>(p);
  p += align256(tiles * sizeof(int32_t));
  void* o_s = p;
  p += align256(tiles * ASA_BLOCK * d * 2);
  float* lse_s = reinterpret_cast<float*>(p);
  p += align256(tiles * ASA_BLOCK * sizeof(float));
  const void* kg = nullptr;
  const void* vg = nullptr;
  cudaError_t e = cudaSuccess;
  if (global_window > 0) {
    const size_t G = (static_cast<size_t>(N) + global_window - 1) / global_window;
    void* kgw = p;
    void* vgw = p + align256(static_cast<size_t>(BH) * G * d * 2);
    e = asa::launch_global_pool(kp, kgw, BH, N, d, global_window, num_sms_current(), s, vp, vgw);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    kg = kgw;
    vg = vgw;
  }
  unsigned int* err_word = nullptr;
  e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_fwd_tc_pruned(q_s, kp, vp, tile_ptr, tile_col, tile_quarters, kg, vg, order, BH,
                                N, Ns, d, global_window, o_s, lse_s, err_word, s);
  if (e != cudaSuccess) return cuda_fail(e, "pruned forward launch");
  e = asa::launch_fill_out(o_s, lse_s, src_row, BH, N, Ns, d, o, lse, err_word, num_sms_current(), s);
  if (e != cudaSuccess) return cuda_fail(e, "fill launch");
  return ASA_OK;
}

size_t asa_bwd_pruned_workspace_size(int B, int H, int N, int d, int pack, int global_window) {
  if (B < 1 || H < 1 || N < 1 || N > ASA_MAX_TOKENS || (d != 64 && d != 128) ||
      (pack != 1 && pack != 2 && pack != 4) || global_window < 0)
    return 0;
  const int Ns = asa_prune_rows(N, pack);
  return asa::bwd_tc_pruned_workspace_bytes(B * H, N, Ns, d, global_window);
}

int asa_sparse_attn_bwd_pruned(const void* q_s, const void* kp, const void* vp, const void* dout,
                               const float* lse, const int32_t* src_pos, const int32_t* src_row,
                               const int32_t* tile_ptr, const int32_t* tile_col,
                               const uint8_t* tile_quarters, int B, int H, int N, int d, int block,
                               int pack, int global_window, void* workspace, size_t ws_bytes,
                               void* dq, void* dk, void* dv, void* stream) {
  ASA_TRY(check_common(B, H, N, d));
  ASA_TRY(check_block(block, ASA_SAMPLES));
  ASA_TRY(check_pack(pack));
  const void* bf[] = {q_s, kp, vp, dout, dq, dk, dv};
  const char* names[] = {"q_s", "kp", "vp", "dout", "dq", "dk", "dv"};
  for (int k = 0; k < 7; ++k) ASA_TRY(check_ptr(bf[k], names[k]));
  ASA_TRY(check_ptr(lse, "lse", false));
  ASA_TRY(check_ptr(src_pos, "src_pos", false));
  ASA_TRY(check_ptr(src_row, "src_row", false));
  ASA_TRY(check_ptr(tile_ptr, "tile_ptr", false));
  ASA_TRY(check_ptr(tile_col, "tile_col", false));
  if (tile_quarters == nullptr) return fail(ASA_ERR_INVALID_ARG, "tile_quarters is NULL");
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  ASA_TRY(check_ws(workspace, ws_bytes,
                   asa_bwd_pruned_workspace_size(B, H, N, d, pack, global_window)));
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  const int Ns = asa_prune_rows(N, pack);
  e = asa::launch_bwd_tc_pruned(q_s, kp, vp, dout, lse, src_pos, src_row, tile_ptr, tile_col,
                                tile_quarters, B * H, N, Ns, d, global_window, workspace, dq, dk,
                                dv, err_word, num_sms_current(), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pruned backward launch");
  return ASA_OK;
}

// ---------------------------------------------------------------- host-buffer call

namespace {

// Streams (copy in, compute, copy out) and events of the host-buffer call, one set per
// device, created on first use and released by asa_shutdown.
struct HostPipe {
  cudaStream_t h2d = nullptr, cmp = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> ev;
};
std::mutex g_pipe_mu;
std::map<int, HostPipe> g_pipes;

// Default heads per chunk: at least 512 contiguous bytes per host row of a chunk's
// strided copies (narrower rows copy markedly slower over PCIe), and at most 24
// chunks (each chunk's copy and compute ends add fill and drain to the pipeline).
int host_chunk(int H, int d, int head_chunk) {
  if (head_chunk > 0) return std::min(head_chunk, H);
  return std::min(H, std::max((256 + d - 1) / d, (H + 23) / 24));
}

// One slot of the pipeline: raster inputs, permuted inputs, permuted and raster
// output, estimator + mask workspace and CSR, forward workspace and LSE, for hc heads.
struct HostSlot {
  char* x[3];
  char* xp[3];
  char* out;
  char* est_ws;
  size_t est_bytes;
  int32_t *row_ptr, *col_idx, *nnz;
  char* fwd_ws;
  size_t fwd_bytes;
  float* lse;
  size_t bytes;
};

HostSlot carve_host_slot(char* base, int B, int hc, int N, int d, int global_window) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base == nullptr ? nullptr : base + off;
    off += align256(bytes);
    return p;
  };
  HostSlot r{};
  const size_t t = static_cast<size_t>(B) * hc * N * d * 2;
  const size_t nb = (static_cast<size_t>(N) + ASA_BLOCK - 1) / ASA_BLOCK;
  const size_t rows = static_cast<size_t>(B) * hc * nb;
  for (int i = 0; i < 3; ++i) r.x[i] = take(t);
  for (int i = 0; i < 3; ++i) r.xp[i] = take(t);
  r.out = take(t);
  r.est_bytes = asa_estimate_mask_workspace_size(B, hc, N);
  r.est_ws = take(r.est_bytes);
  r.row_ptr = reinterpret_cast<int32_t*>(take((rows + 1) * 4));
  r.col_idx = reinterpret_cast<int32_t*>(take(rows * nb * 4));
  r.nnz = reinterpret_cast<int32_t*>(take(4));
  r.fwd_bytes = asa_fwd_workspace_size(B, hc, N, d, global_window);
  r.fwd_ws = take(r.fwd_bytes);
  r.lse = reinterpret_cast<float*>(take(static_cast<size_t>(B) * hc * N * 4));
  r.bytes = off;
  return r;
}

}  // namespace

size_t asa_attention_host_workspace_size(int B, int T, int Hg, int W, int H, int d,
                                         int global_window, int head_chunk) {
  const int64_t N = static_cast<int64_t>(T) * Hg * W;
  if (B < 1 || H < 1 || T < 1 || Hg < 1 || W < 1 || N > ASA_MAX_TOKENS || (d != 64 && d != 128) ||
      global_window < 0 || head_chunk < 0)
    return 0;
  const int hc = host_chunk(H, d, head_chunk);
  return 2 * carve_host_slot(nullptr, B, hc, static_cast<int>(N), d, global_window).bytes;
}

int asa_attention_host(const void* q, const void* k, const void* v, int B, int T, int Hg, int W,
                       int H, int d, float tau, int global_window, int head_chunk,
                       void* workspace, size_t ws_bytes, void* o, void* stream) {
  int64_t N64 = 0;
  ASA_TRY(check_grid(T, Hg, W, &N64));
  const int N = static_cast<int>(N64);
  ASA_TRY(check_common(B, H, N, d));
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
    return fail(ASA_ERR_INVALID_ARG, "a host buffer (q, k, v or o) is NULL");
  if (head_chunk < 0) return fail(ASA_ERR_INVALID_ARG, "head_chunk=%d < 0", head_chunk);
  if (global_window < 0) return fail(ASA_ERR_INVALID_ARG, "global_window=%d < 0", global_window);
  if (!(tau > 0.f)) return fail(ASA_ERR_INVALID_ARG, "tau=%g must be > 0", tau);
  ASA_TRY(check_ws(workspace, ws_bytes,
                   asa_attention_host_workspace_size(B, T, Hg, W, H, d, global_window, head_chunk)));
  const int hc = host_chunk(H, d, head_chunk);
  // chunk c covers heads [ch0[c], ch0[c + 1]); with the default chunk size the last
  // chunk is split in two, which halves the compute and copy-out that remain after
  // the last copy-in
  std::vector<int> ch0;
  for (int h = 0; h < H; h += hc) ch0.push_back(h);
  ch0.push_back(H);
  if (head_chunk == 0 && ch0.size() > 2) {
    const int a = ch0[ch0.size() - 2], last = H - a;
    if (last >= 2) ch0.insert(ch0.end() - 1, a + (last + 1) / 2);
  }
  const int nch = static_cast<int>(ch0.size()) - 1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& P = g_pipes[dev];
  if (P.h2d == nullptr) {
    if ((e = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&P.cmp, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "stream creation");
  }
  const size_t need_ev = 4 + 3 * static_cast<size_t>(nch);
  while (P.ev.size() < need_ev) {
    cudaEvent_t ev;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "event creation");
    P.ev.push_back(ev);
  }
  cudaStream_t caller = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev_start = P.ev[0];
  auto h2d_done = [&](int c) { return P.ev[4 + 3 * c]; };
  auto cmp_done = [&](int c) { return P.ev[5 + 3 * c]; };
  auto d2h_done = [&](int c) { return P.ev[6 + 3 * c]; };
  // on any failure after work was enqueued: the caller's stream still waits for it
  auto finish = [&](int rc) {
    cudaEventRecord(P.ev[1], P.h2d);
    cudaEventRecord(P.ev[2], P.cmp);
    cudaEventRecord(P.ev[3], P.d2h);
    for (int i = 1; i <= 3; ++i) cudaStreamWaitEvent(caller, P.ev[i], 0);
    return rc;
  };
  if ((e = cudaEventRecord(ev_start, caller)) != cudaSuccess) return cuda_fail(e, "event record");
  for (cudaStream_t s : {P.h2d, P.cmp, P.d2h}) cudaStreamWaitEvent(s, ev_start, 0);

  const size_t slot_bytes = carve_host_slot(nullptr, B, hc, N, d, global_window).bytes;
  const size_t pitch = static_cast<size_t>(H) * d * 2;
  const void* src[3] = {q, k, v};
  for (int c = 0; c < nch; ++c) {
    const HostSlot S = carve_host_slot(static_cast<char*>(workspace) + (c & 1) * slot_bytes, B, hc,
                                       N, d, global_window);
    const int h0 = ch0[c], hcur = ch0[c + 1] - ch0[c];
    const size_t width = static_cast<size_t>(hcur) * d * 2;
    // copy in: the slot's inputs are free once chunk c - 2 has been computed
    if (c >= 2) cudaStreamWaitEvent(P.h2d, cmp_done(c - 2), 0);
    for (int i = 0; i < 3; ++i) {
      e = cudaMemcpy2DAsync(S.x[i], width, static_cast<const char*>(src[i]) + h0 * d * 2, pitch,
                            width, static_cast<size_t>(B) * N, cudaMemcpyHostToDevice, P.h2d);
      if (e != cudaSuccess) return finish(cuda_fail(e, "host-to-device copy"));
    }
    cudaEventRecord(h2d_done(c), P.h2d);
    // compute: the slot's output is free once chunk c - 2 has been copied out
    cudaStreamWaitEvent(P.cmp, h2d_done(c), 0);
    if (c >= 2) cudaStreamWaitEvent(P.cmp, d2h_done(c - 2), 0);
    int rc = asa_gilbert_permute3(S.x[0], S.x[1], S.x[2], S.xp[0], S.xp[1], S.xp[2], B, T, Hg, W,
                                  hcur, d, P.cmp);
    if (rc == ASA_OK)
      rc = asa_estimate_mask(S.xp[0], S.xp[1], B, hcur, N, d, ASA_BLOCK, ASA_SAMPLES, tau, S.est_ws,
                             S.est_bytes, S.row_ptr, S.col_idx, S.nnz, nullptr, nullptr, P.cmp);
    if (rc == ASA_OK)
      rc = asa_sparse_attn_fwd_raster(S.xp[0], S.xp[1], S.xp[2], S.row_ptr, S.col_idx, B, T, Hg,
                                      W, hcur, d, ASA_BLOCK, global_window, S.fwd_ws, S.fwd_bytes,
                                      S.out, S.lse, P.cmp);
    if (rc != ASA_OK) return finish(rc);
    cudaEventRecord(cmp_done(c), P.cmp);
    // copy out
    cudaStreamWaitEvent(P.d2h, cmp_done(c), 0);
    e = cudaMemcpy2DAsync(static_cast<char*>(o) + h0 * d * 2, pitch, S.out, width, width,
                          static_cast<size_t>(B) * N, cudaMemcpyDeviceToHost, P.d2h);
    if (e != cudaSuccess) return finish(cuda_fail(e, "device-to-host copy"));
    cudaEventRecord(d2h_done(c), P.d2h);
  }
  if ((e = cudaStreamWaitEvent(caller, d2h_done(nch - 1), 0)) != cudaSuccess)
    return finish(cuda_fail(e, "stream wait"));
  return ASA_OK;
}

// ---------------------------------------------------------------- sequence parallelism

namespace {

// P + 1 offsets from 0 to total, non-decreasing, P in [1, ASA_MAX_RANKS]
int check_segs(const int* off, int P, int total, const char* what, asa::Segs* out) {
  if (off == nullptr) return fail(ASA_ERR_INVALID_ARG, "%s offsets are NULL", what);
  if (P < 1 || P > ASA_MAX_RANKS)
    return fail(ASA_ERR_INVALID_ARG, "P=%d ranks not in [1, %d]", P, ASA_MAX_RANKS);
  if (off[0] != 0 || off[P] != total)
    return fail(ASA_ERR_INVALID_ARG, "%s offsets must run from 0 to %d", what, total);
  out->P = P;
  for (int s = 0; s <= P; ++s) {
    if (s > 0 && off[s] < off[s - 1])
      return fail(ASA_ERR_INVALID_ARG, "%s offsets decrease at rank %d", what, s);
    out->off[s] = off[s];
  }
  return ASA_OK;
}

}  // namespace

int asa_seqpar_pack(const void* x, void* send, int B, int Nr, int H, int d, const int* head_off,
                    int P, void* stream) {
  ASA_TRY(check_common(B, H, std::max(Nr, 1), d));
  if (Nr < 0) return fail(ASA_ERR_INVALID_ARG, "Nr=%d < 0", Nr);
  ASA_TRY(check_ptr(x, "x"));
  ASA_TRY(check_ptr(send, "send"));
  asa::Segs heads{};
  ASA_TRY(check_segs(head_off, P, H, "head", &heads));
  if (Nr == 0) return ASA_OK;
  cudaError_t e = asa::launch_head_groups(x, send, true, B, Nr, H, d, heads, num_sms_current(),
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ASA_OK : cuda_fail(e, "pack launch");
}

int asa_seqpar_unpack(const void* recv, void* x, int B, int Nr, int H, int d, const int* head_off,
                      int P, void* stream) {
  ASA_TRY(check_common(B, H, std::max(Nr, 1), d));
  if (Nr < 0) return fail(ASA_ERR_INVALID_ARG, "Nr=%d < 0", Nr);
  ASA_TRY(check_ptr(recv, "recv"));
  ASA_TRY(check_ptr(x, "x"));
  asa::Segs heads{};
  ASA_TRY(check_segs(head_off, P, H, "head", &heads));
  if (Nr == 0) return ASA_OK;
  cudaError_t e = asa::launch_head_groups(recv, x, false, B, Nr, H, d, heads, num_sms_current(),
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ASA_OK : cuda_fail(e, "unpack launch");
}

static int seqpar_permute_impl(const void* const* src, void* const* dst, int nt, bool to_perm,
                               int B, int T, int Hg, int W, int Hl, int d, const int* tok_off,
                               int P, void* stream) {
  int64_t N = 0;
  ASA_TRY(check_grid(T, Hg, W, &N));
  ASA_TRY(check_common(B, Hl, static_cast<int>(N), d));
  for (int k = 0; k < nt; ++k) {
    ASA_TRY(check_ptr(src[k], "src"));
    ASA_TRY(check_ptr(dst[k], "dst"));
  }
  asa::Segs tok{};
  ASA_TRY(check_segs(tok_off, P, static_cast<int>(N), "token", &tok));
  const int32_t* perm = nullptr;
  ASA_TRY(get_perm(T, Hg, W, &perm));
  cudaError_t e = asa::launch_permute_chunks(src, dst, nt, to_perm, perm, B, static_cast<int>(N),
                                             Hl, d, tok, num_sms_current(),
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ASA_OK : cuda_fail(e, "chunk permute launch");
}

int asa_seqpar_permute3(const void* r0, const void* r1, const void* r2, void* xp0, void* xp1,
                        void* xp2, int B, int T, int Hg, int W, int Hl, int d, const int* tok_off,
                        int P, void* stream) {
  const void* s[3] = {r0, r1, r2};
  void* t[3] = {xp0, xp1, xp2};
  return seqpar_permute_impl(s, t, 3, true, B, T, Hg, W, Hl, d, tok_off, P, stream);
}

int asa_seqpar_unpermute(const void* op, void* send, int B, int T, int Hg, int W, int Hl, int d,
                         const int* tok_off, int P, void* stream) {
  const void* s[1] = {op};
  void* t[1] = {send};
  return seqpar_permute_impl(s, t, 1, false, B, T, Hg, W, Hl, d, tok_off, P, stream);
}

int asa_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > (1ll << 31))
    return fail(ASA_ERR_INVALID_ARG, "limit_cycles=%lld outside [1, 2^31]", limit_cycles);
  unsigned int* err_word = nullptr;
  cudaError_t e = device_error_word(&err_word);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  e = asa::launch_wait_timeout(err_word, limit_cycles, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ASA_OK;
}

int asa_check_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (word & 8u)
      return fail(ASA_ERR_INVALID_ARG,
                  "a Q or K value (backward) or V value (training forward) is out of fp16 range "
                  "(|x| > 65504) (word 0x%x)", word);
    if (word & 32u)
      return fail(ASA_ERR_INVALID_ARG,
                  "an index argument (CSR column, src_pos or src_row) is out of range (word 0x%x)",
                  word);
    return fail(ASA_ERR_TIMEOUT, "a device-side bounded wait expired (word 0x%x)", word);
  }
  return ASA_OK;
}

void asa_shutdown(void) {
  {
    std::lock_guard<std::mutex> plock(g_pipe_mu);
    int cur = 0;
    const bool have = cudaGetDevice(&cur) == cudaSuccess;
    for (auto& kv : g_pipes) {
      if (have) cudaSetDevice(kv.first);
      for (cudaStream_t s : {kv.second.h2d, kv.second.cmp, kv.second.d2h})
        if (s != nullptr) {
          cudaStreamSynchronize(s);
          cudaStreamDestroy(s);
        }
      for (cudaEvent_t ev : kv.second.ev) cudaEventDestroy(ev);
    }
    if (have) cudaSetDevice(cur);
    g_pipes.clear();
  }
  std::lock_guard<std::mutex> lock(g_perm_mu);
  int cur = 0;
  const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
  for (auto& kv : g_perm_cache) {
    if (have_dev) cudaSetDevice(std::get<0>(kv.first));
    cudaFree(kv.second);
  }
  if (have_dev) cudaSetDevice(cur);
  g_perm_cache.clear();
}

}  // extern "C"
