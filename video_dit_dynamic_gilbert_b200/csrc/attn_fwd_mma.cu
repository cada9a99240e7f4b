// Block-sparse attention forward over the kept tiles (Video-BLADE, "Step 2.2:
// Computation": standard ASA and ASA_G), register-tiled tensor-core version.
//
// One CTA per (b, h, query block I): 8 warps x 16 query rows.  The CTA walks the
// CSR row of I (kept key blocks, each as two 64-row halves), then for ASA_G the
// ceil(N/n) global tokens in 64-row tiles whose logits carry + log2(n) (ln(n) in the
// natural domain).  K/V tiles are double-buffered through shared memory with
// cp.async; S = Q K^T and O += P V run on mma.sync m16n8k16 with fp32 accumulation;
// the softmax is the online (running max, running sum) form in the log2 domain.
// Rows past N (ragged last block) are zero-filled on load, masked to -inf as keys
// and never stored as queries.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kFwdWarps = 8;
constexpr int kTileN = 64;

template <int D>
struct FwdSmem {
  static constexpr int kQBytes = kBlock * D * 2;
  static constexpr int kKVBytes = kTileN * D * 2;
  static constexpr int kTotal = kQBytes + 4 * kKVBytes;  // Q + 2 x (K, V)
};

template <int D>
__global__ void __launch_bounds__(kFwdWarps * 32)
    fwd_mma_kernel(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
                   const __nv_bfloat16* __restrict__ vp, const int32_t* __restrict__ row_ptr,
                   const int32_t* __restrict__ col_idx, const __nv_bfloat16* __restrict__ kg,
                   const __nv_bfloat16* __restrict__ vg, int N, int nb, int G, float gbias2,
                   float c2, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sKV = reinterpret_cast<__nv_bfloat16*>(smem + FwdSmem<D>::kQBytes);

  const int I = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t head = static_cast<int64_t>(bh) * N * D;
  const int q0 = I * kBlock;

  const int rbeg = row_ptr[bh * nb + I], rend = row_ptr[bh * nb + I + 1];
  const int n_fine = 2 * (rend - rbeg);
  const int n_glob = G > 0 ? (G + kTileN - 1) / kTileN : 0;
  const int n_tiles = n_fine + n_glob;

  // tile -> (source K, source V, first row, valid rows, bias)
  auto tile_info = [&](int tt, const __nv_bfloat16*& ks, const __nv_bfloat16*& vs, int& r0,
                       int& nvalid, float& bias) {
    if (tt < n_fine) {
      const int J = col_idx[rbeg + (tt >> 1)];
      r0 = J * kBlock + (tt & 1) * kTileN;
      nvalid = min(kTileN, N - r0);
      ks = kp + head;
      vs = vp + head;
      bias = 0.f;
    } else {
      r0 = (tt - n_fine) * kTileN;
      nvalid = min(kTileN, G - r0);
      ks = kg + static_cast<int64_t>(bh) * G * D;
      vs = vg + static_cast<int64_t>(bh) * G * D;
      bias = gbias2;
    }
  };

  auto load_tile = [&](int tt, int stage) {
    const __nv_bfloat16 *ks, *vs;
    int r0, nvalid;
    float bias;
    tile_info(tt, ks, vs, r0, nvalid, bias);
    __nv_bfloat16* dK = sKV + stage * 2 * kTileN * D;
    __nv_bfloat16* dV = dK + kTileN * D;
    for (int idx = tid; idx < kTileN * CH; idx += blockDim.x) {
      const int row = idx / CH, ch = idx - row * CH;
      const bool ok = row < nvalid;
      const int64_t off = static_cast<int64_t>(ok ? r0 + row : 0) * D + ch * 8;
      cp_async16(smem_u32(dK) + swz<CH>(row, ch), ks + off, ok);
      cp_async16(smem_u32(dV) + swz<CH>(row, ch), vs + off, ok);
    }
    cp_async_commit();
  };

  // Q tile
  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    const bool ok = q0 + row < N;
    cp_async16(smem_u32(sQ) + swz<CH>(row, ch),
               qp + head + static_cast<int64_t>(ok ? q0 + row : 0) * D + ch * 8, ok);
  }
  cp_async_commit();
  if (n_tiles > 0) load_tile(0, 0);
  cp_async_wait<0>();
  __syncthreads();

  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int row = warp * 16 + (lane & 15);
    ldsm_x4(smem_u32(sQ) + swz<CH>(row, 2 * ks + (lane >> 4)), qf[ks][0], qf[ks][1], qf[ks][2],
            qf[ks][3]);
  }

  float oacc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};

  for (int tt = 0; tt < n_tiles; ++tt) {
    if (tt + 1 < n_tiles) {
      load_tile(tt + 1, (tt + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16 *ks_, *vs_;
    int r0, nvalid;
    float bias;
    tile_info(tt, ks_, vs_, r0, nvalid, bias);
    const uint32_t kbase = smem_u32(sKV + (tt & 1) * 2 * kTileN * D);
    const uint32_t vbase = kbase + kTileN * D * 2;

    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldsm_x4(kbase + swz<CH>(row, 2 * ks + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
    }
    float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n * 8 + 2 * t + (e & 1);
        s[n][e] = col < nvalid ? fmaf(s[n][e], c2, bias) : -INFINITY;
        rmax[e >> 1] = fmaxf(rmax[e >> 1], s[n][e]);
      }
    }
    float alpha[2], ref[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      rmax[h] = fmaxf(rmax[h], __shfl_xor_sync(0xffffffffu, rmax[h], 1));
      rmax[h] = fmaxf(rmax[h], __shfl_xor_sync(0xffffffffu, rmax[h], 2));
      const float mn = fmaxf(m[h], rmax[h]);
      ref[h] = mn == -INFINITY ? 0.f : mn;
      alpha[h] = fast_exp2(m[h] - ref[h]);
      m[h] = mn;
    }
    float rsum[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[n][e] = fast_exp2(s[n][e] - ref[e >> 1]);
        rsum[e >> 1] += s[n][e];
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) l[h] = l[h] * alpha[h] + rsum[h];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      oacc[n][0] *= alpha[0];
      oacc[n][1] *= alpha[0];
      oacc[n][2] *= alpha[1];
      oacc[n][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int row = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldsm_x4_t(vbase + swz<CH>(row, 2 * dp + (lane >> 4)), b0, b1, b2, b3);
        mma_bf16(oacc[2 * dp], a, b0, b1);
        mma_bf16(oacc[2 * dp + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

  // epilogue: normalise, stage the bf16 tile in shared memory, store 16-byte rows
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
  }
  const float inv0 = l[0] > 0.f ? 1.f / l[0] : 0.f;
  const float inv1 = l[1] > 0.f ? 1.f / l[1] : 0.f;
  __syncthreads();
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int r_lo = warp * 16 + g, col = n * 8 + 2 * t;
    uint32_t* p0 = reinterpret_cast<uint32_t*>(smem + swz<CH>(r_lo, col / 8) + (col % 8) * 2);
    uint32_t* p1 = reinterpret_cast<uint32_t*>(smem + swz<CH>(r_lo + 8, col / 8) + (col % 8) * 2);
    *p0 = pack_bf16(oacc[n][0] * inv0, oacc[n][1] * inv0);
    *p1 = pack_bf16(oacc[n][2] * inv1, oacc[n][3] * inv1);
  }
  if (t == 0) {
    const int r_lo = q0 + warp * 16 + g;
    if (r_lo < N) lse[static_cast<int64_t>(bh) * N + r_lo] = l[0] > 0.f ? (m[0] + __log2f(l[0])) * kLn2 : -INFINITY;
    if (r_lo + 8 < N)
      lse[static_cast<int64_t>(bh) * N + r_lo + 8] = l[1] > 0.f ? (m[1] + __log2f(l[1])) * kLn2 : -INFINITY;
  }
  __syncthreads();
  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    if (q0 + row < N)
      *reinterpret_cast<uint4*>(o + head + static_cast<int64_t>(q0 + row) * D + ch * 8) =
          *reinterpret_cast<const uint4*>(smem + swz<CH>(row, ch));
  }
}

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

cudaError_t launch_fwd_mma(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                           const int32_t* col_idx, const void* kg, const void* vg, int BH, int N,
                           int d, int global_window, void* o, float* lse, cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  const int G = global_window > 0 ? (N + global_window - 1) / global_window : 0;
  const float gbias2 = global_window > 0 ? log2f(static_cast<float>(global_window)) : 0.f;
  const float c2 = kLog2e / sqrtf(static_cast<float>(d));
  dim3 grid(nb, BH);
#define ASA_LAUNCH_FWD(DD)                                                                      \
  do {                                                                                          \
    const int smem = FwdSmem<DD>::kTotal;                                                       \
    cudaFuncSetAttribute(fwd_mma_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); \
    fwd_mma_kernel<DD><<<grid, kFwdWarps * 32, smem, stream>>>(                                 \
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp),          \
        static_cast<const __nv_bfloat16*>(vp), row_ptr, col_idx,                                \
        static_cast<const __nv_bfloat16*>(kg), static_cast<const __nv_bfloat16*>(vg), N, nb, G, \
        gbias2, c2, static_cast<__nv_bfloat16*>(o), lse);                                       \
  } while (0)
  if (d == 128)
    ASA_LAUNCH_FWD(128);
  else
    ASA_LAUNCH_FWD(64);
#undef ASA_LAUNCH_FWD
  return cudaGetLastError();
}

}  // namespace asa
