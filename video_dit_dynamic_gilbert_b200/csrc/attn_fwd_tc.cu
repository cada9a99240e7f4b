// Block-sparse attention forward on tcgen05 tensor cores (Video-BLADE, "Step 2.2:
// Computation": standard ASA over the kept tiles of M, and ASA_G with global tokens).
//
// One CTA per (b, h, query block I of 128 rows), 6 warps, warp-specialised:
//   warp 0      TMA producer: Q once, then for every kept key block J (the CSR row
//               of I) its 128-row K and V tiles into an NST-stage ring; for ASA_G
//               then the ceil(N/n) global tokens in 128-row tiles.  Tiles past N
//               (ragged last block) are zero-filled by TMA.
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_j = Q K_j^T   (SS MMA, M=128 N=128, into TMEM S buffer j%2)
//                 O  += P_j V_j   (TS MMA: P read from TMEM, V from shared memory)
//               S_{j+1} is issued before PV_j so it overlaps the softmax of tile j.
//   warps 2..5  softmax warpgroup: thread = query row = TMEM lane.  Reads S_j,
//               masks columns past the tile's valid rows, keeps the running max /
//               sum in the log2 domain, computes P_j = exp2(.) into registers while
//               PV_{j-1} still runs, then waits for PV_{j-1}, rescales O in TMEM only
//               when the running max grew by more than 2^8 (until then P is taken
//               against the stale max; exact after the final division), and writes
//               P_j as bf16 over S_j.  Epilogue: O / l -> bf16 rows, LSE (natural log).
// TMEM: S buffers at columns [0,128) and [128,256), O at [256, 256+D).
// Every wait is bounded: on expiry the kernel sets the device error word, drains its
// own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace asa {

namespace {

constexpr int kFwdTcThreads = 320;  // producer, MMA, 2 softmax warpgroups
constexpr uint32_t kTmemCols = 512;

template <int D, int NST>
struct FwdTcLayout {
  static constexpr uint32_t kTile = 128u * D * 2u;  // one 128-row bf16 tile of Q, K or V
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kV = kK + NST * kTile;
  static constexpr uint32_t kBars = kV + NST * kTile;
  // barriers: q_full, k_full[NST], v_full[NST], kv_empty[NST], s_full[2], p_full[2],
  //           o_done, drain; then the TMEM base address slot
  static constexpr uint32_t kNumBars = 1 + 3 * NST + 2 + 2 + 1 + 1;
  static constexpr uint32_t kRed = kBars + 8 * kNumBars;    // [2 warpgroups][128 rows] fp32
  static constexpr uint32_t kTmemSlot = kRed + 2 * 128 * 4;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;  // + alignment slack
};

// exp2 on the FMA pipe: 2^x = 2^n 2^f, n = round(x) (via the 1.5*2^23 rounding
// constant), f in [-1/2, 1/2], 2^f by a degree-3 minimax polynomial (relative error
// 7.5e-5; coefficients from csrc/gen_exp2_poly.py).  x is clamped at -125 so that the
// exponent add stays in the normal range.  Used for a share of the softmax
// exponentials so that MUFU and the FMA pipe split the work.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.f);
  const float j = x + 12582912.f;
  const float f = x - (j - 12582912.f);
  const float p = fmaf(fmaf(fmaf(5.517166853e-02f, f, 2.426111251e-01f), f, 6.932609677e-01f), f,
                       9.999280572e-01f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// One in kPolyEvery P pairs takes exp2_fma (0: all on MUFU).  The forward is issue-
// bound in the softmax, where a MUFU exp2 costs one instruction and exp2_fma nine.
constexpr int kPolyEvery = 0;

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// barrier over `nthreads` threads that also returns the AND of every thread's `v`
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}

struct TileSrc {
  int row0, nvalid;
  bool global;
};

__device__ __forceinline__ TileSrc tile_src(int j, int nfine, const int32_t* cols, int N, int G) {
  TileSrc t;
  if (j < nfine) {
    t.row0 = cols[j] * kBlock;
    t.nvalid = min(kBlock, N - t.row0);
    t.global = false;
  } else {
    t.row0 = (j - nfine) * kBlock;
    t.nvalid = min(kBlock, G - t.row0);
    t.global = true;
  }
  return t;
}

template <int D, int NST>
__global__ void __launch_bounds__(kFwdTcThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKg,
                  const __grid_constant__ CUtensorMap tmVg, const int32_t* __restrict__ row_ptr,
                  const int32_t* __restrict__ col_idx, int N, int nb, int G, float gbias2,
                  float c2, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                  unsigned int* __restrict__ err_word, long long wait_limit) {
  using L = FwdTcLayout<D, NST>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int I = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = I * kBlock;
  const int rbeg = row_ptr[bh * nb + I];
  const int nfine = row_ptr[bh * nb + I + 1] - rbeg;
  const int nglob = G > 0 ? (G + kBlock - 1) / kBlock : 0;
  const int ntile = nfine + nglob;
  const int32_t* cols = col_idx + rbeg;

  const uint32_t bar0 = base + L::kBars;
  auto q_full = [&]() { return bar0; };
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (1 + NST + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NST + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 3 * NST + b); };
  auto p_full = [&](int b) { return bar0 + 8u * (3 + 3 * NST + b); };
  const uint32_t o_done = bar0 + 8u * (5 + 3 * NST);
  const uint32_t drain = bar0 + 8u * (6 + 3 * NST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kTmemSlot);

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full(), 1);
    for (int s = 0; s < NST; ++s) {
      tc::mbar_init(k_full(s), 1);
      tc::mbar_init(v_full(s), 1);
      tc::mbar_init(kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full(b), 1);
      tc::mbar_init(p_full(b), 256);
    }
    tc::mbar_init(o_done, 1);
    tc::mbar_init(drain, 1);
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
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
      tc::tma_prefetch(&tmQ);
      tc::tma_prefetch(&tmK);
      tc::tma_prefetch(&tmV);
      tc::mbar_expect_tx(q_full(), L::kTile);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tc::tma_load_3d(base + L::kQ + h * 16384u, &tmQ, 64 * h, q0, bh, q_full());
      int issued = 0;
      for (int j = 0; j < ntile; ++j) {
        const int st = j % NST, n = j / NST;
        if (n > 0 && !tc::mbar_wait(kv_empty(st), (n - 1) & 1, wait_limit)) {
          failed = true;
          break;
        }
        const TileSrc t = tile_src(j, nfine, cols, N, G);
        const CUtensorMap* mk = t.global ? &tmKg : &tmK;
        const CUtensorMap* mv = t.global ? &tmVg : &tmV;
        tc::mbar_expect_tx(k_full(st), L::kTile);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(base + L::kK + st * L::kTile + h * 16384u, mk, 64 * h, t.row0, bh,
                          k_full(st));
        tc::mbar_expect_tx(v_full(st), L::kTile);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(base + L::kV + st * L::kTile + h * 16384u, mv, 64 * h, t.row0, bh,
                          v_full(st));
        issued = j + 1;
      }
      // drain: every issued copy has landed, and the MMAs have released the last
      // stages (their commits arrive before the CTA exits)
      tc::mbar_wait(q_full(), 0, wait_limit);
      for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j) {
        tc::mbar_wait(k_full(j % NST), (j / NST) & 1, wait_limit);
        tc::mbar_wait(v_full(j % NST), (j / NST) & 1, wait_limit);
        tc::mbar_wait(kv_empty(j % NST), (j / NST) & 1, wait_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idPV = tc::idesc_bf16(128, D, false, true);
      const uint32_t tO = tmem + 256u;
      auto issue_s = [&](int j) {
        const int st = j % NST;
        const uint32_t dS = tmem + 128u * (j & 1);
        const uint32_t kb = base + L::kK + st * L::kTile;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;
          tc::umma_ss(dS, tc::sdesc_sw128(base + L::kQ + off, 16, 1024),
                      tc::sdesc_sw128(kb + off, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
      };
      bool ok = tc::mbar_wait(q_full(), 0, wait_limit);
      int issued_any = 0;
      if (ok && ntile > 0) {
        ok = tc::mbar_wait(k_full(0), 0, wait_limit);
        if (ok) {
          tc::fence_after();
          issue_s(0);
          tc::umma_commit(s_full(0));
          issued_any = 1;
        }
      }
      for (int j = 0; ok && j < ntile; ++j) {
        if (j + 1 < ntile) {
          const int st1 = (j + 1) % NST;
          if (!(ok = tc::mbar_wait(k_full(st1), ((j + 1) / NST) & 1, wait_limit))) break;
          tc::fence_after();
          issue_s(j + 1);
          tc::umma_commit(s_full((j + 1) & 1));
        }
        if (!(ok = tc::mbar_wait(p_full(j & 1), (j >> 1) & 1, wait_limit))) break;
        if (!(ok = tc::mbar_wait(v_full(j % NST), (j / NST) & 1, wait_limit))) break;
        tc::fence_after();
        const uint32_t tP = tmem + 128u * (j & 1);
        const uint32_t vb = base + L::kV + (j % NST) * L::kTile;
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          tc::umma_ts(tO, tP + 8u * ks, tc::sdesc_sw128(vb + ks * 2048u, 16384, 1024), idPV,
                      (j > 0 || ks > 0) ? 1u : 0u);
        tc::umma_commit(kv_empty(j % NST));
        tc::umma_commit(o_done);
      }
      failed = !ok;
      if (issued_any) {
        // drain: all MMAs of this CTA complete before TMEM is released
        tc::umma_commit(drain);
        tc::mbar_wait(drain, 0, wait_limit);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    // Two warpgroups share each row: warpgroup wg owns columns [64 wg, 64 wg + 64) of
    // every S tile, of P and of O; the row max is combined through shared memory.
    // tcgen05.ld/st are warp-collective and the named barriers span both warpgroups:
    // every wait result is AND-reduced over all 256 softmax threads, so that every
    // branch (including a timeout) is taken by all of them together.
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int col0 = 64 * wg;
    float* red = reinterpret_cast<float*>(sbase + L::kRed);
    // bounded wait, result identical in all 256 softmax threads (barrier `id`)
    auto wait_all = [&](uint32_t bar, uint32_t parity, int id) {
      const bool ok = tc::mbar_wait(bar, parity, wait_limit);
      __syncwarp();
      return named_bar_and(id, 256, ok);
    };
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < ntile; ++j) {
      const int b = j & 1;
      // (barrier 2 also orders this tile's exchange after the partner's last read)
      if (!wait_all(s_full(b), (j >> 1) & 1, 2)) {
        failed = true;
        break;
      }
      tc::fence_after();
      const TileSrc t = tile_src(j, nfine, cols, N, G);
      const float bias = t.global ? gbias2 : 0.f;
      const int nv = t.nvalid - col0;  // valid columns in this half (may be <= 0 or >= 64)
      uint32_t s[64];
      tc::tmem_ld32(trow + 128u * b + col0, s);
      tc::tmem_ld32(trow + 128u * b + col0 + 32u, s + 32);
      tc::tmem_wait_ld_dep32(s);
      tc::tmem_wait_ld_dep32(s + 32);
      // full tiles skip every per-column validity test
      if (nv < 64) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k >= nv) s[k] = __float_as_uint(-INFINITY);
      }
      // row max on the raw scores (c2 > 0 keeps the order), combined across halves
      float m0 = max3f(__uint_as_float(s[0]), __uint_as_float(s[1]), __uint_as_float(s[2]));
      float m1 = max3f(__uint_as_float(s[3]), __uint_as_float(s[4]), __uint_as_float(s[5]));
#pragma unroll
      for (int k = 6; k < 62; k += 4) {
        m0 = max3f(m0, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
        m1 = max3f(m1, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]));
      }
      float mraw = max3f(m0, m1, fmaxf(__uint_as_float(s[62]), __uint_as_float(s[63])));
      red[wg * 128 + row] = mraw;
      named_bar_sync(1, 256);
      mraw = fmaxf(mraw, red[(1 - wg) * 128 + row]);
      const float mx = fmaf(mraw, c2, bias);
      const float m_new = fmaxf(m_ref, mx);
      const bool need = m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + 8.f);
      const bool any_need = __any_sync(0xffffffffu, need) != 0;
      const float alpha = need ? (m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - m_new)) : 1.f;
      if (need) m_ref = m_new;
      // P = exp2(s c2 + bias - m) packed to bf16 pairs (masked columns give exp2(-inf) = 0)
      const float off = bias - (m_ref == -INFINITY ? 0.f : m_ref);
      uint32_t p[32];
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float xa = fmaf(__uint_as_float(s[2 * k]), c2, off);
        const float xb = fmaf(__uint_as_float(s[2 * k + 1]), c2, off);
        float a, bb;
        if (kPolyEvery > 0 && (k % (kPolyEvery > 0 ? kPolyEvery : 1)) == 0) {
          a = exp2_fma(xa);
          bb = exp2_fma(xb);
        } else {
          a = fast_exp2(xa);
          bb = fast_exp2(xb);
        }
        rs0 += a;
        rs1 += bb;
        p[k] = pack_bf16(a, bb);
      }
      const float rs = rs0 + rs1;
      l = l * alpha + rs;
      if (j > 0) {
        // PV_{j-1} done: O may be rescaled, and P_j may overwrite nothing in use
        if (!wait_all(o_done, (j - 1) & 1, 3)) {
          failed = true;
          break;
        }
        tc::fence_after();
        if (any_need) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            const uint32_t oc = trow + 256u + (D / 2) * wg + 32u * c;
            uint32_t ov[32];
            tc::tmem_ld32_sync(oc, ov);
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tc::tmem_st16(oc, ov);
            tc::tmem_st16(oc + 16u, ov + 16);
            tc::tmem_wait_st();
          }
        }
      }
      tc::tmem_st16(trow + 128u * b + 32u * wg, p);
      tc::tmem_st16(trow + 128u * b + 32u * wg + 16u, p + 16);
      tc::tmem_wait_st();
      tc::fence_before();
      tc::mbar_arrive(p_full(b));
    }
    bool have_o = false;
    if (!failed && ntile > 0) {
      if (wait_all(o_done, (ntile - 1) & 1, 3)) {
        tc::fence_after();
        have_o = true;
      } else {
        failed = true;
      }
    }
    // row sum across the two halves
    named_bar_sync(2, 256);
    red[wg * 128 + row] = l;
    named_bar_sync(1, 256);
    const float l_row = l + red[(1 - wg) * 128 + row];
    // epilogue: this thread's query row, columns [D/2 wg, D/2 wg + D/2)
    const int q = q0 + row;
    __nv_bfloat16* orow = o + (static_cast<int64_t>(bh) * N + (q < N ? q : 0)) * D + (D / 2) * wg;
    const float inv = (have_o && l_row > 0.f) ? 1.f / l_row : 0.f;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t ov[32];
      if (have_o) {
        tc::tmem_ld32_sync(trow + 256u + (D / 2) * wg + 32u * c, ov);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = 0u;
      }
      if (q < N) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 pk;
          pk.x = pack_bf16(__uint_as_float(ov[8 * v + 0]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
          pk.y = pack_bf16(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
          pk.z = pack_bf16(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
          pk.w = pack_bf16(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + 32 * c + 8 * v) = pk;
        }
      }
    }
    if (q < N && wg == 0)
      lse[static_cast<int64_t>(bh) * N + q] =
          (have_o && l_row > 0.f) ? (m_ref + __log2f(l_row)) * kLn2 : -INFINITY;
  }

  if (failed) atomicOr(err_word, 1u);
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [BH][rows][D] bf16, boxes of 64 columns x 128 rows, 128-byte swizzle, zero fill
bool make_map(CUtensorMap* m, const void* ptr, int BH, int rows, int D) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(rows) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NST>
cudaError_t launch_tc(const CUtensorMap* maps, const int32_t* row_ptr, const int32_t* col_idx,
                      int BH, int N, int G, float gbias2, void* o, float* lse,
                      unsigned int* err_word, cudaStream_t stream) {
  using L = FwdTcLayout<D, NST>;
  const int nb = (N + kBlock - 1) / kBlock;
  const float c2 = kLog2e / sqrtf(static_cast<float>(D));
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D, NST>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  const long long limit = 1ll << 31;  // ~1 s of SM clock per wait
  fwd_tc_kernel<D, NST><<<dim3(nb, BH), kFwdTcThreads, L::kSmem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], row_ptr, col_idx, N, nb, G, gbias2, c2,
      static_cast<__nv_bfloat16*>(o), lse, err_word, limit);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                          const int32_t* col_idx, const void* kg, const void* vg, int BH, int N,
                          int d, int global_window, void* o, float* lse, unsigned int* err_word,
                          cudaStream_t stream) {
  const int G = global_window > 0 ? (N + global_window - 1) / global_window : 0;
  const float gbias2 = global_window > 0 ? log2f(static_cast<float>(global_window)) : 0.f;
  CUtensorMap maps[5];
  if (!make_map(&maps[0], qp, BH, N, d) || !make_map(&maps[1], kp, BH, N, d) ||
      !make_map(&maps[2], vp, BH, N, d))
    return cudaErrorInvalidValue;
  if (G > 0) {
    if (!make_map(&maps[3], kg, BH, G, d) || !make_map(&maps[4], vg, BH, G, d))
      return cudaErrorInvalidValue;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  if (d == 128) return launch_tc<128, 3>(maps, row_ptr, col_idx, BH, N, G, gbias2, o, lse, err_word, stream);
  return launch_tc<64, 6>(maps, row_ptr, col_idx, BH, N, G, gbias2, o, lse, err_word, stream);
}

}  // namespace asa
