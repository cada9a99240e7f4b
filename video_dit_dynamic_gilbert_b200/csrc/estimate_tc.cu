// Block-importance estimation on tcgen05 tensor cores (Video-BLADE, "Step 1: Efficient
// block importance estimation").
//
// For one head: Q_s, K_s = the k_I = min(16, L_I) evenly strided sample tokens of every
// block (offsets floor(j L_I / k_I)); P_approx = rowsoftmax(Q_s K_s^T / sqrt d);
// P_imp[I, J] = max over the k_I x k_J tile.  Softmax is monotone, so the tile max of
// P_approx is exp2(max scaled logit of the tile - lse2 of the row), maximised over the
// rows of block I.  Kernels:
//   est_gather   compact Q_s, K_s [BH][Mp][d] (row 16 I + j = sample j of block I;
//                rows past a short last block and past 16 nb are zero);
//   est_tc       one CTA per (head, 128 sample rows, chunk of 128-column tiles):
//                S = Q_s K_s^T tiles on tcgen05 into a double-buffered TMEM S; two
//                softmax warpgroups split every tile's columns (warpgroup w takes
//                [64 w, 64 w + 64); thread = sample row): each writes its 16-column
//                groups' max logit G[bh, J, r] and keeps the row's online (max, sum)
//                over its half of the chunk;
//   est_combine  lse2[bh, r] from the (max, sum) of every chunk half;
//   est_pool     P_imp[bh, I, J] = max_{r in I} exp2(G[bh, J, r] - lse2[bh, r]).
// 10 warps and 256 TMEM columns per CTA, two CTAs per SM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "softmax_math.cuh"
#include "tc.cuh"

namespace asa {

bool make_map_rows(CUtensorMap* m, const void* ptr, int BH, int rows, int D);

namespace {

constexpr int kEstThreads = 320;      // producer, MMA, two softmax warpgroups
constexpr int kEstHalves = 2;         // softmax warpgroups, each a partial (max, sum) per row
constexpr uint32_t kEstTmemCols = 256;  // two 128-column S buffers
constexpr int kEstStages = 2;
constexpr int kTilesPerChunk = 8;     // 128-column tiles per CTA

__host__ __device__ constexpr int round_up128(int x) { return (x + 127) / 128 * 128; }

template <int D>
struct EstLayout {
  static constexpr uint32_t kTile = 128u * D * 2u;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kTile;
  static constexpr uint32_t kBars = kK + kEstStages * kTile;
  // q_full, k_full[S], k_empty[S], s_full[2], s_empty[2], drain
  static constexpr uint32_t kNumBars = 1 + 2 * kEstStages + 2 + 2 + 1;
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kSmem = kTmemSlot + 16 + 1024;
};

// qs[bh, 16 I + j] = qp[bh, 128 I + floor(j L_I / k_I)] (j < k_I), zero otherwise
__global__ void est_gather_kernel(const uint4* __restrict__ qp, const uint4* __restrict__ kp,
                                  uint4* __restrict__ qs, uint4* __restrict__ ks, int BH, int N,
                                  int nb, int Mp, int vec_per_row) {
  const int64_t total = static_cast<int64_t>(BH) * Mp * vec_per_row;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % vec_per_row);
    const int64_t rr = idx / vec_per_row;
    const int r = static_cast<int>(rr % Mp);
    const int64_t bh = rr / Mp;
    const int I = r >> 4, j = r & 15;
    uint4 vq = make_uint4(0, 0, 0, 0), vk = vq;
    if (I < nb) {
      const int L = min(kBlock, N - kBlock * I);
      const int kI = min(kSamples, L);
      if (j < kI) {
        const int64_t src = (bh * N + kBlock * I + (j * L) / kI) * vec_per_row + c;
        vq = __ldg(qp + src);
        vk = __ldg(kp + src);
      }
    }
    qs[idx] = vq;
    ks[idx] = vk;
  }
}

template <int D>
__global__ void __launch_bounds__(kEstThreads, 2)
    est_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  float* __restrict__ G, float2* __restrict__ part, int N, int nb, int Mp,
                  int nchunk, float c2, unsigned int* __restrict__ err_word, long long wait_limit) {
  using L = EstLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int ntn = Mp / 128;  // column tiles of the head
  const int chunk = blockIdx.x % nchunk;
  const int mt = (blockIdx.x / nchunk) % ntn;
  const int bh = blockIdx.x / (nchunk * ntn);
  const int t0 = chunk * kTilesPerChunk;
  const int ntile = min(kTilesPerChunk, ntn - t0);
  const int M = kSamples * (nb - 1) + min(kSamples, N - kBlock * (nb - 1));  // valid samples
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = base + L::kBars;
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (1 + kEstStages + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 2 * kEstStages + b); };
  auto s_empty = [&](int b) { return bar0 + 8u * (3 + 2 * kEstStages + b); };
  const uint32_t drain = bar0 + 8u * (5 + 2 * kEstStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kTmemSlot);

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kEstStages; ++s) {
      tc::mbar_init(k_full(s), 1);
      tc::mbar_init(k_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full(b), 1);
      tc::mbar_init(s_empty(b), 128 * kEstHalves);
    }
    tc::mbar_init(drain, 1);
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kEstTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::mbar_expect_tx(q_full, L::kTile);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tc::tma_load_3d(base + L::kQ + h * 16384u, &tmQ, 64 * h, 128 * mt, bh, q_full);
      int issued = 0;
      for (int j = 0; j < ntile; ++j) {
        const int st = j % kEstStages, n = j / kEstStages;
        if (n > 0 && !tc::mbar_wait(k_empty(st), (n - 1) & 1, wait_limit)) {
          failed = true;
          break;
        }
        tc::mbar_expect_tx(k_full(st), L::kTile);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(base + L::kK + st * L::kTile + h * 16384u, &tmK, 64 * h,
                          128 * (t0 + j), bh, k_full(st));
        issued = j + 1;
      }
      tc::mbar_wait(q_full, 0, wait_limit);
      for (int j = (issued > kEstStages ? issued - kEstStages : 0); j < issued; ++j) {
        tc::mbar_wait(k_full(j % kEstStages), (j / kEstStages) & 1, wait_limit);
        tc::mbar_wait(k_empty(j % kEstStages), (j / kEstStages) & 1, wait_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      const uint64_t dQ = tc::sdesc_sw128(base + L::kQ, 16, 1024);
      const uint64_t dK = tc::sdesc_sw128(base + L::kK, 16, 1024);
      bool ok = tc::mbar_wait(q_full, 0, wait_limit);
      int issued_any = 0;
      for (int j = 0; ok && j < ntile; ++j) {
        const int st = j % kEstStages, b = j & 1;
        if (!(ok = tc::mbar_wait(k_full(st), (j / kEstStages) & 1, wait_limit))) break;
        if (j >= 2 && !(ok = tc::mbar_wait(s_empty(b), ((j >> 1) - 1) & 1, wait_limit))) break;
        tc::fence_after();
        const uint32_t dS = tmem + 128u * b;
        const uint64_t kst = dK + ((st * L::kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;
          tc::umma_ss(dS, dQ + off, kst + off, idS, kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(s_full(b));
        tc::umma_commit(k_empty(st));
        issued_any = 1;
      }
      failed = !ok;
      if (issued_any) {
        tc::umma_commit(drain);
        tc::mbar_wait(drain, 0, wait_limit);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int w = (warp - 2) >> 2;  // warps 2-5: columns [0, 64); warps 6-9: [64, 128)
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int r = 128 * mt + row;  // sample row of the head
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 64u * w;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < ntile; ++j) {
      const int b = j & 1;
      const bool ok = tc::mbar_wait(s_full(b), (j >> 1) & 1, wait_limit);
      if (__all_sync(0xffffffffu, ok) == 0) {
        failed = true;
        break;
      }
      tc::fence_after();
      uint32_t s[64];
      tc::tmem_ld32(trow + 128u * b, s);
      tc::tmem_ld32(trow + 128u * b + 32u, s + 32);
      tc::tmem_wait_ld_dep32(s);
      tc::tmem_wait_ld_dep32(s + 32);
      // the buffer is free for the tile after next as soon as both halves are in registers
      tc::fence_before();
      tc::mbar_arrive(s_empty(b));
      const int nt = t0 + j;                   // column tile
      const int nvalid = M - 128 * nt - 64 * w;  // valid sample columns in this half
      if (nvalid < 64) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k >= nvalid) s[k] = __float_as_uint(-INFINITY);
      }
      // block maxima (raw scores; c2 > 0 keeps the order) and the row max
      float gm[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float a = max3f(__uint_as_float(s[16 * g]), __uint_as_float(s[16 * g + 1]),
                        __uint_as_float(s[16 * g + 2]));
        float bq = max3f(__uint_as_float(s[16 * g + 3]), __uint_as_float(s[16 * g + 4]),
                         __uint_as_float(s[16 * g + 5]));
#pragma unroll
        for (int k = 6; k < 14; k += 4) {
          a = max3f(a, __uint_as_float(s[16 * g + k]), __uint_as_float(s[16 * g + k + 1]));
          bq = max3f(bq, __uint_as_float(s[16 * g + k + 2]), __uint_as_float(s[16 * g + k + 3]));
        }
        gm[g] = max3f(a, bq, fmaxf(__uint_as_float(s[16 * g + 14]), __uint_as_float(s[16 * g + 15])));
      }
      const float mraw = fmaxf(max3f(gm[0], gm[1], gm[2]), gm[3]);
      if (r < M) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int J = 8 * nt + 4 * w + g;
          if (J < nb) G[(static_cast<int64_t>(bh) * nb + J) * (kSamples * nb) + r] = gm[g] * c2;
        }
      }
      // a half with no valid column (the last tile's) keeps its running (max, sum)
      if (mraw == -INFINITY) continue;
      const float m_new = fmaxf(m, mraw * c2);
      const uint64_t c2x2 = f2_pack(c2, c2), offx2 = f2_pack(-m_new, -m_new);
      uint64_t rs = f2_pack(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const uint64_t x2 =
            f2_fma(f2_pack(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2x2, offx2);
        float a, bq;
        if ((k & 3) == 0) {
          exp2_fma2(x2, a, bq);
          // exp2_fma clamps at -125: keep masked columns at zero
          if (nvalid < 64) {
            a = 2 * k < nvalid ? a : 0.f;
            bq = 2 * k + 1 < nvalid ? bq : 0.f;
          }
        } else {
          float xa, xb;
          f2_unpack(x2, xa, xb);
          a = fast_exp2(xa);
          bq = fast_exp2(xb);
        }
        rs = f2_add(rs, f2_pack(a, bq));
      }
      float ra, rb;
      f2_unpack(rs, ra, rb);
      l = l * fast_exp2(m - m_new) + (ra + rb);
      m = m_new;
    }
    if (r < Mp)
      part[(static_cast<int64_t>(bh) * nchunk * kEstHalves + kEstHalves * chunk + w) * Mp + r] =
          make_float2(m, l);
  }

  if (failed) atomicOr(err_word, 2u);
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after();
    tc::tmem_dealloc(tmem, kEstTmemCols);
  }
}

// lse2[bh, r] = log2 sum_c l_c 2^(m_c) over the column chunks of row r
__global__ void est_combine_kernel(const float2* __restrict__ part, float* __restrict__ lse2,
                                   int BH, int Mp, int Mpad16, int nchunk) {
  const int64_t total = static_cast<int64_t>(BH) * Mpad16;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(idx % Mpad16);
    const int64_t bh = idx / Mpad16;
    float m = -INFINITY;
    for (int c = 0; c < nchunk; ++c) m = fmaxf(m, part[(bh * nchunk + c) * Mp + r].x);
    float l = 0.f;
    for (int c = 0; c < nchunk; ++c) {
      const float2 v = part[(bh * nchunk + c) * Mp + r];
      if (v.y > 0.f) l += v.y * exp2f(v.x - m);
    }
    lse2[idx] = m + __log2f(l);
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

inline unsigned grid_cap(int64_t work, int per_block, int num_sms, int per_sm) {
  int64_t b = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

template <int D>
cudaError_t launch_est_tc(const void* qs, const void* ks, int BH, int N, int nb, int Mp,
                          float* G, float2* part, float* lse2, float* p_imp,
                          unsigned int* err_word, int num_sms, cudaStream_t stream) {
  using L = EstLayout<D>;
  CUtensorMap mq, mk;
  if (!make_map_rows(&mq, qs, BH, Mp, D) || !make_map_rows(&mk, ks, BH, Mp, D))
    return cudaErrorInvalidValue;
  const int ntn = Mp / 128;
  const int nchunk = (ntn + kTilesPerChunk - 1) / kTilesPerChunk;
  const float c2 = kLog2e / sqrtf(static_cast<float>(D));
  cudaError_t e = cudaFuncSetAttribute(est_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kSmem);
  if (e != cudaSuccess) return e;
  est_tc_kernel<D><<<BH * ntn * nchunk, kEstThreads, L::kSmem, stream>>>(
      mq, mk, G, part, N, nb, Mp, nchunk, c2, err_word, 1ll << 31);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int Mpad16 = kSamples * nb;
  est_combine_kernel<<<grid_cap(static_cast<int64_t>(BH) * Mpad16, 256, num_sms, 16), 256, 0,
                       stream>>>(part, lse2, BH, Mp, Mpad16, nchunk * kEstHalves);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  est_pool_kernel<<<grid_cap(static_cast<int64_t>(BH) * nb * nb, 256, num_sms, 16), 256, 0,
                    stream>>>(G, lse2, p_imp, BH, N, nb);
  return cudaGetLastError();
}

}  // namespace

size_t est_scratch_floats(int BH, int nb) {
  const size_t Mp = static_cast<size_t>(round_up128(kSamples * nb));
  const size_t ntn = Mp / 128;
  const size_t nchunk = (ntn + kTilesPerChunk - 1) / kTilesPerChunk;
  return static_cast<size_t>(BH) * nb * kSamples * nb   // G
         + static_cast<size_t>(BH) * kSamples * nb      // lse2
         + static_cast<size_t>(BH) * nchunk * kEstHalves * Mp * 2  // per chunk half (max, sum)
         + 2 * static_cast<size_t>(BH) * Mp * 128 / 2   // Q_s, K_s (bf16, d <= 128)
         + 64;                                          // alignment of Q_s
}

cudaError_t launch_estimate(const void* qp, const void* kp, int BH, int N, int d, float* scratch,
                            float* p_imp, unsigned int* err_word, int num_sms,
                            cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  const int Mp = round_up128(kSamples * nb);
  const int ntn = Mp / 128;
  const int nchunk = (ntn + kTilesPerChunk - 1) / kTilesPerChunk;
  float* G = scratch;
  float* lse2 = G + static_cast<size_t>(BH) * nb * kSamples * nb;
  float2* part = reinterpret_cast<float2*>(lse2 + static_cast<size_t>(BH) * kSamples * nb);
  // Q_s, K_s at a 16-byte boundary after the partial sums
  uintptr_t qa =
      reinterpret_cast<uintptr_t>(part + static_cast<size_t>(BH) * nchunk * kEstHalves * Mp);
  qa = (qa + 255) & ~static_cast<uintptr_t>(255);
  uint4* qs = reinterpret_cast<uint4*>(qa);
  uint4* ks = qs + static_cast<size_t>(BH) * Mp * d / 8;
  const int vpr = d / 8;
  est_gather_kernel<<<grid_cap(static_cast<int64_t>(BH) * Mp * vpr, 256, num_sms, 16), 256, 0,
                      stream>>>(static_cast<const uint4*>(qp), static_cast<const uint4*>(kp), qs,
                                ks, BH, N, nb, Mp, vpr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (d == 128)
    return launch_est_tc<128>(qs, ks, BH, N, nb, Mp, G, part, lse2, p_imp, err_word, num_sms, stream);
  return launch_est_tc<64>(qs, ks, BH, N, nb, Mp, G, part, lse2, p_imp, err_word, num_sms, stream);
}

}  // namespace asa
