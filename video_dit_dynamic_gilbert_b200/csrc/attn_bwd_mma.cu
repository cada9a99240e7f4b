// Backward of standard ASA under the fixed mask (Video-BLADE: the binary mask
// restricts attention "during both training and inference"; the mask itself is not
// differentiated).  Register-tiled tensor-core version.
//
//   P = exp2(S c2 - lse2), S = Q K^T, c2 = log2(e)/sqrt(d)
//   D_i = sum_j P_ij dP_ij = dO_i . O_i           (bwd_dq<pass 0>, exact in fp32:
//                                                  the bf16-rounded O would cost
//                                                  ~4e-3 relative L2 on dQ)
//   dV_J = sum_{I keeps J} P^T dO_I,  dP = dO V^T,  dS = P (dP - D)
//   dK_J = sum_{I keeps J} dS^T Q_I / sqrt(d)     (bwd_dkv: one CTA per key block,
//                                                  walking the transposed CSR)
//   dQ_I = sum_{J kept by I} dS K_J / sqrt(d)     (bwd_dq: one CTA per query block,
//                                                  walking the CSR)
// Each output row is written once by one CTA: no atomics, deterministic.
// dS enters the dQ and dK products in fp16 (Q and K converted from bf16, exact for
// magnitudes below 65504): rounding dS to bf16 would put ~3.5e-3 relative L2 error
// on dQ and dK by itself.
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr int kBwdWarps = 8;
constexpr int kTile = 64;

// ---------------------------------------------------------------- dK, dV

template <int D>
struct DkvSmem {
  static constexpr int kKV = kBlock * D * 2;   // K or V block
  static constexpr int kT = kTile * D * 2;     // Q or dO tile
  static constexpr int kTotal = 2 * kKV + 4 * kT + 4 * kTile * 4;
};

template <int D>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dkv_kernel(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
                   const __nv_bfloat16* __restrict__ vp, const __nv_bfloat16* __restrict__ dout,
                   const float* __restrict__ lse2, const float* __restrict__ Dvec,
                   const int32_t* __restrict__ col_ptr_t, const int32_t* __restrict__ row_idx_t,
                   int N, int nb, float c2, float scale, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv) {
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sK = smem;
  unsigned char* sV = sK + DkvSmem<D>::kKV;
  unsigned char* sT = sV + DkvSmem<D>::kKV;  // [2 stages][Q tile, dO tile]
  float* sL = reinterpret_cast<float*>(sT + 4 * DkvSmem<D>::kT);  // [2][lse2 64, D 64]

  const int J = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t head = static_cast<int64_t>(bh) * N * D;
  const int k0 = J * kBlock;

  const int cbeg = col_ptr_t[bh * nb + J], cend = col_ptr_t[bh * nb + J + 1];
  const int n_tiles = 2 * (cend - cbeg);

  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    const bool ok = k0 + row < N;
    const int64_t off = head + static_cast<int64_t>(ok ? k0 + row : 0) * D + ch * 8;
    cp_async16(smem_u32(sK) + swz<CH>(row, ch), kp + off, ok);
    cp_async16(smem_u32(sV) + swz<CH>(row, ch), vp + off, ok);
  }
  cp_async_commit();

  auto load_tile = [&](int tt, int stage) {
    const int I = row_idx_t[cbeg + (tt >> 1)];
    const int r0 = I * kBlock + (tt & 1) * kTile;
    const int nvalid = min(kTile, N - r0);
    unsigned char* dQ = sT + stage * 2 * DkvSmem<D>::kT;
    unsigned char* dO = dQ + DkvSmem<D>::kT;
    for (int idx = tid; idx < kTile * CH; idx += blockDim.x) {
      const int row = idx / CH, ch = idx - row * CH;
      const bool ok = row < nvalid;
      const int64_t off = head + static_cast<int64_t>(ok ? r0 + row : 0) * D + ch * 8;
      cp_async16(smem_u32(dQ) + swz<CH>(row, ch), qp + off, ok);
      cp_async16(smem_u32(dO) + swz<CH>(row, ch), dout + off, ok);
    }
    if (tid < kTile) {
      float* l2 = sL + stage * 2 * kTile;
      const bool ok = tid < nvalid;
      l2[tid] = ok ? lse2[static_cast<int64_t>(bh) * N + r0 + tid] : INFINITY;  // P = 0
      l2[kTile + tid] = ok ? Dvec[static_cast<int64_t>(bh) * N + r0 + tid] : 0.f;
    }
    cp_async_commit();
  };

  if (n_tiles > 0) load_tile(0, 0);

  float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dka[n][e] = dva[n][e] = 0.f;

  for (int tt = 0; tt < n_tiles; ++tt) {
    if (tt + 1 < n_tiles) {
      load_tile(tt + 1, (tt + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int stage = tt & 1;
    const uint32_t qb = smem_u32(sT + stage * 2 * DkvSmem<D>::kT);
    const uint32_t ob = qb + DkvSmem<D>::kT;
    const float* l2 = sL + stage * 2 * kTile;
    const float* dd = l2 + kTile;

    // S^T = K_w Q^T and dP^T = V_w dO^T  (16 key rows x 64 query columns)
    float st[8][4], dpt[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t ka[4], va[4];
      const int arow = warp * 16 + (lane & 15);
      ldsm_x4(smem_u32(sK) + swz<CH>(arow, 2 * ks + (lane >> 4)), ka[0], ka[1], ka[2], ka[3]);
      ldsm_x4(smem_u32(sV) + swz<CH>(arow, 2 * ks + (lane >> 4)), va[0], va[1], va[2], va[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(qb + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(st[2 * np], ka, b0, b1);
        mma_bf16(st[2 * np + 1], ka, b2, b3);
        ldsm_x4(ob + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(dpt[2 * np], va, b0, b1);
        mma_bf16(dpt[2 * np + 1], va, b2, b3);
      }
    }
    // P^T and dS^T
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n * 8 + 2 * t + (e & 1);
        const float p = fast_exp2(st[n][e] * c2 - l2[col]);
        st[n][e] = p;
        dpt[n][e] = p * (dpt[n][e] - dd[col]);
      }
    }
    // dV += P^T dO ; dK += dS^T Q   (k = the 64 query rows)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4], sa[4];
      pa[0] = pack_bf16(st[2 * kk][0], st[2 * kk][1]);
      pa[1] = pack_bf16(st[2 * kk][2], st[2 * kk][3]);
      pa[2] = pack_bf16(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      pa[3] = pack_bf16(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      sa[0] = pack_f16(dpt[2 * kk][0], dpt[2 * kk][1]);
      sa[1] = pack_f16(dpt[2 * kk][2], dpt[2 * kk][3]);
      sa[2] = pack_f16(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
      sa[3] = pack_f16(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int row = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = 2 * dp + (lane >> 4);
        ldsm_x4_t(ob + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(dva[2 * dp], pa, b0, b1);
        mma_bf16(dva[2 * dp + 1], pa, b2, b3);
        ldsm_x4_t(qb + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_f16(dka[2 * dp], sa, bf16x2_to_f16x2(b0), bf16x2_to_f16x2(b1));
        mma_f16(dka[2 * dp + 1], sa, bf16x2_to_f16x2(b2), bf16x2_to_f16x2(b3));
      }
    }
    __syncthreads();
  }

  // stage dK in sK and dV in sV (bf16), then store full rows
  __syncthreads();
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int r_lo = warp * 16 + g, col = n * 8 + 2 * t;
    const uint32_t off_lo = swz<CH>(r_lo, col / 8) + (col % 8) * 2;
    const uint32_t off_hi = swz<CH>(r_lo + 8, col / 8) + (col % 8) * 2;
    *reinterpret_cast<uint32_t*>(sK + off_lo) = pack_bf16(dka[n][0] * scale, dka[n][1] * scale);
    *reinterpret_cast<uint32_t*>(sK + off_hi) = pack_bf16(dka[n][2] * scale, dka[n][3] * scale);
    *reinterpret_cast<uint32_t*>(sV + off_lo) = pack_bf16(dva[n][0], dva[n][1]);
    *reinterpret_cast<uint32_t*>(sV + off_hi) = pack_bf16(dva[n][2], dva[n][3]);
  }
  __syncthreads();
  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    if (k0 + row < N) {
      const int64_t off = head + static_cast<int64_t>(k0 + row) * D + ch * 8;
      *reinterpret_cast<uint4*>(dk + off) = *reinterpret_cast<const uint4*>(sK + swz<CH>(row, ch));
      *reinterpret_cast<uint4*>(dv + off) = *reinterpret_cast<const uint4*>(sV + swz<CH>(row, ch));
    }
  }
}

// ---------------------------------------------------------------- dQ

template <int D>
struct DqSmem {
  static constexpr int kQ = kBlock * D * 2;
  static constexpr int kT = kTile * D * 2;
  static constexpr int kTotal = 2 * kQ + 4 * kT;
};

// kDPass: walk the tiles once to produce D and lse2 (no dQ); otherwise dQ.
template <int D, bool kDPass>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dq_kernel(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
                  const __nv_bfloat16* __restrict__ vp, const __nv_bfloat16* __restrict__ dout,
                  const float* __restrict__ lse, float* __restrict__ lse2,
                  float* __restrict__ Dvec, const int32_t* __restrict__ row_ptr,
                  const int32_t* __restrict__ col_idx, int N, int nb, float c2, float scale,
                  __nv_bfloat16* __restrict__ dq) {
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sQ = smem;
  unsigned char* sO = sQ + DqSmem<D>::kQ;  // dO block
  unsigned char* sT = sO + DqSmem<D>::kQ;  // [2 stages][K tile, V tile]

  const int I = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t head = static_cast<int64_t>(bh) * N * D;
  const int q0 = I * kBlock;
  const int rbeg = row_ptr[bh * nb + I], rend = row_ptr[bh * nb + I + 1];
  const int n_tiles = 2 * (rend - rbeg);

  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    const bool ok = q0 + row < N;
    const int64_t off = head + static_cast<int64_t>(ok ? q0 + row : 0) * D + ch * 8;
    cp_async16(smem_u32(sQ) + swz<CH>(row, ch), qp + off, ok);
    cp_async16(smem_u32(sO) + swz<CH>(row, ch), dout + off, ok);
  }
  cp_async_commit();

  auto load_tile = [&](int tt, int stage) {
    const int J = col_idx[rbeg + (tt >> 1)];
    const int r0 = J * kBlock + (tt & 1) * kTile;
    const int nvalid = min(kTile, N - r0);
    unsigned char* dK = sT + stage * 2 * DqSmem<D>::kT;
    unsigned char* dV = dK + DqSmem<D>::kT;
    for (int idx = tid; idx < kTile * CH; idx += blockDim.x) {
      const int row = idx / CH, ch = idx - row * CH;
      const bool ok = row < nvalid;
      const int64_t off = head + static_cast<int64_t>(ok ? r0 + row : 0) * D + ch * 8;
      cp_async16(smem_u32(dK) + swz<CH>(row, ch), kp + off, ok);
      cp_async16(smem_u32(dV) + swz<CH>(row, ch), vp + off, ok);
    }
    cp_async_commit();
  };
  if (n_tiles > 0) load_tile(0, 0);

  const int r_lo = q0 + warp * 16 + g;
  const int64_t rowb = static_cast<int64_t>(bh) * N;
  const float l2r[2] = {r_lo < N ? lse[rowb + r_lo] * kLog2e : 0.f,
                        r_lo + 8 < N ? lse[rowb + r_lo + 8] * kLog2e : 0.f};
  float ddr[2] = {0.f, 0.f};
  if (!kDPass) {
    ddr[0] = r_lo < N ? Dvec[rowb + r_lo] : 0.f;
    ddr[1] = r_lo + 8 < N ? Dvec[rowb + r_lo + 8] : 0.f;
  }
  float dsum[2] = {0.f, 0.f};

  float dqa[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) dqa[n][0] = dqa[n][1] = dqa[n][2] = dqa[n][3] = 0.f;

  for (int tt = 0; tt < n_tiles; ++tt) {
    if (tt + 1 < n_tiles) {
      load_tile(tt + 1, (tt + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int J = col_idx[rbeg + (tt >> 1)];
    const int nvalid = min(kTile, N - (J * kBlock + (tt & 1) * kTile));
    const uint32_t kb = smem_u32(sT + (tt & 1) * 2 * DqSmem<D>::kT);
    const uint32_t vb = kb + DqSmem<D>::kT;

    float s[8][4], dp[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qa[4], oa[4];
      const int arow = warp * 16 + (lane & 15);
      ldsm_x4(smem_u32(sQ) + swz<CH>(arow, 2 * ks + (lane >> 4)), qa[0], qa[1], qa[2], qa[3]);
      ldsm_x4(smem_u32(sO) + swz<CH>(arow, 2 * ks + (lane >> 4)), oa[0], oa[1], oa[2], oa[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(kb + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa, b0, b1);
        mma_bf16(s[2 * np + 1], qa, b2, b3);
        ldsm_x4(vb + swz<CH>(row, ch), b0, b1, b2, b3);
        mma_bf16(dp[2 * np], oa, b0, b1);
        mma_bf16(dp[2 * np + 1], oa, b2, b3);
      }
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n * 8 + 2 * t + (e & 1);
        const int h = e >> 1;
        const float p = col < nvalid ? fast_exp2(s[n][e] * c2 - l2r[h]) : 0.f;
        if (kDPass)
          dsum[h] = fmaf(p, dp[n][e], dsum[h]);
        else
          s[n][e] = p * (dp[n][e] - ddr[h]);  // dS
      }
    }
    if (kDPass) {
      __syncthreads();
      continue;
    }
    // dQ += dS K
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dpi = 0; dpi < D / 16; ++dpi) {
        uint32_t b0, b1, b2, b3;
        const int row = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldsm_x4_t(kb + swz<CH>(row, 2 * dpi + (lane >> 4)), b0, b1, b2, b3);
        mma_f16(dqa[2 * dpi], a, bf16x2_to_f16x2(b0), bf16x2_to_f16x2(b1));
        mma_f16(dqa[2 * dpi + 1], a, bf16x2_to_f16x2(b2), bf16x2_to_f16x2(b3));
      }
    }
    __syncthreads();
  }

  if (kDPass) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      dsum[h] += __shfl_xor_sync(0xffffffffu, dsum[h], 1);
      dsum[h] += __shfl_xor_sync(0xffffffffu, dsum[h], 2);
    }
    if (t == 0) {
      if (r_lo < N) {
        Dvec[rowb + r_lo] = dsum[0];
        lse2[rowb + r_lo] = l2r[0];
      }
      if (r_lo + 8 < N) {
        Dvec[rowb + r_lo + 8] = dsum[1];
        lse2[rowb + r_lo + 8] = l2r[1];
      }
    }
    return;
  }
  __syncthreads();
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int rl = warp * 16 + g, col = n * 8 + 2 * t;
    *reinterpret_cast<uint32_t*>(sQ + swz<CH>(rl, col / 8) + (col % 8) * 2) =
        pack_bf16(dqa[n][0] * scale, dqa[n][1] * scale);
    *reinterpret_cast<uint32_t*>(sQ + swz<CH>(rl + 8, col / 8) + (col % 8) * 2) =
        pack_bf16(dqa[n][2] * scale, dqa[n][3] * scale);
  }
  __syncthreads();
  for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
    const int row = idx / CH, ch = idx - row * CH;
    if (q0 + row < N)
      *reinterpret_cast<uint4*>(dq + head + static_cast<int64_t>(q0 + row) * D + ch * 8) =
          *reinterpret_cast<const uint4*>(sQ + swz<CH>(row, ch));
  }
}

}  // namespace

cudaError_t launch_bwd_mma(const void* qp, const void* kp, const void* vp, const void* o,
                           const void* dout, const float* lse, const int32_t* row_ptr,
                           const int32_t* col_idx, const int32_t* col_ptr_t,
                           const int32_t* row_idx_t, int BH, int N, int d, float* Dvec,
                           float* lse2, void* dq, void* dk, void* dv, int num_sms,
                           cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  (void)o;
  (void)num_sms;
  const float c2 = kLog2e / sqrtf(static_cast<float>(d));
  const float scale = 1.f / sqrtf(static_cast<float>(d));
  dim3 grid(nb, BH);
#define ASA_LAUNCH_BWD(DD)                                                                         \
  do {                                                                                             \
    cudaFuncSetAttribute(bwd_dq_kernel<DD, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,     \
                         DqSmem<DD>::kTotal);                                                      \
    bwd_dq_kernel<DD, true><<<grid, kBwdWarps * 32, DqSmem<DD>::kTotal, stream>>>(                 \
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp),             \
        static_cast<const __nv_bfloat16*>(vp), static_cast<const __nv_bfloat16*>(dout), lse, lse2, \
        Dvec, row_ptr, col_idx, N, nb, c2, scale, static_cast<__nv_bfloat16*>(dq));                \
    cudaFuncSetAttribute(bwd_dkv_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,          \
                         DkvSmem<DD>::kTotal);                                                     \
    bwd_dkv_kernel<DD><<<grid, kBwdWarps * 32, DkvSmem<DD>::kTotal, stream>>>(                     \
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp),             \
        static_cast<const __nv_bfloat16*>(vp), static_cast<const __nv_bfloat16*>(dout), lse2, Dvec, \
        col_ptr_t, row_idx_t, N, nb, c2, scale, static_cast<__nv_bfloat16*>(dk),                   \
        static_cast<__nv_bfloat16*>(dv));                                                          \
    cudaFuncSetAttribute(bwd_dq_kernel<DD, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                         DqSmem<DD>::kTotal);                                                      \
    bwd_dq_kernel<DD, false><<<grid, kBwdWarps * 32, DqSmem<DD>::kTotal, stream>>>(                \
        static_cast<const __nv_bfloat16*>(qp), static_cast<const __nv_bfloat16*>(kp),             \
        static_cast<const __nv_bfloat16*>(vp), static_cast<const __nv_bfloat16*>(dout), lse, lse2, \
        Dvec, row_ptr, col_idx, N, nb, c2, scale, static_cast<__nv_bfloat16*>(dq));                \
  } while (0)
  if (d == 128)
    ASA_LAUNCH_BWD(128);
  else
    ASA_LAUNCH_BWD(64);
#undef ASA_LAUNCH_BWD
  return cudaGetLastError();
}

}  // namespace asa
