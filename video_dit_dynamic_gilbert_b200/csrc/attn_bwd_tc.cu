// Backward of standard ASA under the fixed mask on tcgen05 tensor cores (Video-BLADE,
// "Step 2.2: Computation": the binary mask restricts attention in training as in
// inference; the mask itself is not differentiated).
//
//   S = Q K^T,  c2 = log2(e)/sqrt(d),  P = exp2(S c2 - lse2),  lse2 = lse log2(e)
//   dP = dO V^T,  D_i = sum_j P_ij dP_ij,  dS = P o (dP - D)
//   dV_J = sum_{I keeps J} P_IJ^T dO_I
//   dK_J = sum_{I keeps J} dS_IJ^T Q_I / sqrt(d)
//   dQ_I = sum_{J kept by I} dS_IJ K_J / sqrt(d)
//
// Kernels, in launch order (one CTA per 128-row block; heads in order, inside a head
// the blocks with the most partners first):
//   bwd_prep        fp16 copies of Q and K, lse2 (rows past N: +inf, so P = 0 there),
//                   D cleared.  fp16 holds every bf16 value of magnitude in
//                   [2^-17, 65504] exactly; a value that overflows ORs 8 into the
//                   device error word.
//   bwd_row<D pass> per query block I, walking its CSR row: S and dP into TMEM,
//                   D_I = rowsum(P o dP) exactly in fp32.  (D from the bf16-rounded O
//                   would put ~3.5e-3 relative L2 error on dQ by itself.)
//   bwd_col         per key block J, walking the transposed CSR: S^T = K Q^T and
//                   dP^T = V dO^T into TMEM; P^T (bf16) and dS^T (fp16) written back
//                   over them; dV += P^T dO and dK += dS^T Q with the TMEM operand.
//   bwd_row<dQ>     per query block again: dS (fp16) written over S, dQ += dS K.
// Each output row is written by one CTA: no atomics, deterministic.  dS enters the dK
// and dQ products in fp16 (in bf16 it would cost ~3.5e-3 relative L2 on its own); a
// kind::f16 MMA takes A and B of one type, hence the fp16 copies of Q and K, which
// also serve S (exact products, fp32 accumulation: the same S as in bf16).
//
// Warp roles (12 warps, as in the forward): warp 0 lane 0 loads the two stationary
// tiles and ring A by TMA, lane 1 ring B; warp 1 owns TMEM and issues the MMAs; warps
// 2-3 idle (they complete warpgroup 0 for the register split); warps 4-11 are two
// elementwise warpgroups, warpgroup w taking columns [64 w, 64 w + 64) of every
// 128 x 128 tile, thread = TMEM lane = the stationary block's row.
//
//            stationary      ring A (3 stages)    ring B (2 stages)
//   row      Q16, dO         K16 (S, dQ)          V (dP)
//   col      K16, V          Q16 (S^T, dK)        dO (dP^T, dV)
//
// TMEM (512 columns):
//   row   S buffers [0,128) and [128,256) (tile t in buffer t % 2; dS_t over S_t),
//         dP [256,384), dQ [384,384+D)
//   col   S^T [0,128) (P^T over it), dP^T [128,256) (dS^T over it), dV [256,256+D),
//         dK [384,384+D)
// Each elementwise warpgroup writes its 64 packed results (32 columns) over the first
// half of its own 64 loaded columns, so no warp overwrites columns another warp may not
// have read yet; the MMA reading them takes K-steps 0-3 from [0,32) and 4-7 from
// [64,96) of the buffer.  A buffer is rewritten by the next MMA only after the MMA that
// reads the packed operand, in issue order.  Every wait is bounded: on expiry the
// kernel ORs 4 into the device error word, drains its copies and MMAs, frees TMEM
// and returns.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "softmax_math.cuh"
#include "tc.cuh"

namespace asa {

bool make_map_rows(CUtensorMap* m, const void* ptr, int BH, int rows, int D);
bool make_map_rows_f16(CUtensorMap* m, const void* ptr, int BH, int rows, int D);

namespace {

constexpr int kBwdThreads = 384;
// 384 threads x 168 registers at launch; 128 x 72 + 256 x 216 = 64,512 (the forward's
// split).  The launcher checks the compiled count: a split above the launch allocation
// would wait forever.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kRegsLow = 72, kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh == kBwdThreads * kLaunchRegs,
              "register split must equal the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr int kNA = 3, kNB = 2;  // ring stages
constexpr int kElemWarps = 8;
constexpr int kPolyEvery = 4;    // one exp2 pair in 4 on the FMA pipe
constexpr unsigned int kErrWait = 4u, kErrRange = 8u;

template <int D>
struct BwdLayout {
  static constexpr uint32_t kTile = 128u * D * 2u;
  static constexpr uint32_t kStat0 = 0;
  static constexpr uint32_t kStat1 = kTile;
  static constexpr uint32_t kA = 2 * kTile;
  static constexpr uint32_t kB = kA + kNA * kTile;
  static constexpr uint32_t kBars = kB + kNB * kTile;
  static constexpr uint32_t kNumBars = 20;
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;  // + alignment slack
};
static_assert(BwdLayout<128>::kSmem <= 232448, "backward tiles exceed shared memory");

// stat_full, a_full[3], a_empty[3], b_full[2], b_empty[2], s_full[2], dp_full, dp_free,
// p_full, ds_full[2], acc_done, drain
struct Bars {
  uint32_t b0;
  __device__ uint32_t stat_full() const { return b0; }
  __device__ uint32_t a_full(int s) const { return b0 + 8u * (1 + s); }
  __device__ uint32_t a_empty(int s) const { return b0 + 8u * (1 + kNA + s); }
  __device__ uint32_t b_full(int s) const { return b0 + 8u * (1 + 2 * kNA + s); }
  __device__ uint32_t b_empty(int s) const { return b0 + 8u * (1 + 2 * kNA + kNB + s); }
  __device__ uint32_t s_full(int b) const { return b0 + 8u * (1 + 2 * kNA + 2 * kNB + b); }
  __device__ uint32_t dp_full() const { return b0 + 8u * (3 + 2 * kNA + 2 * kNB); }
  __device__ uint32_t dp_free() const { return b0 + 8u * (4 + 2 * kNA + 2 * kNB); }
  __device__ uint32_t p_full() const { return b0 + 8u * (5 + 2 * kNA + 2 * kNB); }
  __device__ uint32_t ds_full(int b) const { return b0 + 8u * (6 + 2 * kNA + 2 * kNB + b); }
  __device__ uint32_t acc_done() const { return b0 + 8u * (8 + 2 * kNA + 2 * kNB); }
  __device__ uint32_t drain() const { return b0 + 8u * (9 + 2 * kNA + 2 * kNB); }
  __device__ void init() const {
    tc::mbar_init(stat_full(), 1);
    for (int s = 0; s < kNA; ++s) {
      tc::mbar_init(a_full(s), 1);
      tc::mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < kNB; ++s) {
      tc::mbar_init(b_full(s), 1);
      tc::mbar_init(b_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full(b), 1);
      tc::mbar_init(ds_full(b), kElemWarps);
    }
    tc::mbar_init(dp_full(), 1);
    tc::mbar_init(dp_free(), kElemWarps);
    tc::mbar_init(p_full(), kElemWarps);
    tc::mbar_init(acc_done(), 1);
    tc::mbar_init(drain(), 1);
    tc::fence_barrier_init();
  }
};
static_assert(10 + 2 * kNA + 2 * kNB == BwdLayout<128>::kNumBars, "barrier count");

// the warp's tcgen05 loads/stores are complete: one arrive per warp
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
  tc::fence_before();
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(bar);
}

// K-step ks (16 elements of K) of a K-major SW128 tile: the 64-column halves are 16 KB
// apart, the 16-element steps inside a half 32 bytes apart (descriptor units: >> 4)
__device__ __forceinline__ uint32_t kmajor_step(int ks) {
  return ((ks >> 2) * 16384u + (ks & 3) * 32u) >> 4;
}

// TMA side, warp 0: lane 0 the stationary tiles and ring A, lane 1 ring B.  Ring tile
// t < nfirst is the 128-row block idx[t] (t itself when idx is null) of mA / mB; tile
// t >= nfirst is the 128-row tile t - nfirst of mA2 / mB2 (the ASA_G global tokens).
// Stage s of ring A is refilled after the a_empty(s) commit of its previous tile,
// likewise for B.
template <int D>
__device__ bool produce(const Bars& br, uint32_t base, int lane, const CUtensorMap* m0,
                        const CUtensorMap* m1, int row_stat, const CUtensorMap* mA,
                        const CUtensorMap* mB, const int32_t* idx, int nfirst,
                        const CUtensorMap* mA2, const CUtensorMap* mB2, int n, int bh,
                        long long limit) {
  using L = BwdLayout<D>;
  const bool isA = lane == 0;
  if (isA) {
    tc::tma_prefetch(m0);
    tc::tma_prefetch(m1);
    tc::tma_prefetch(mA);
    tc::mbar_expect_tx(br.stat_full(), 2 * L::kTile);
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      tc::tma_load_3d(base + L::kStat0 + h * 16384u, m0, 64 * h, row_stat, bh, br.stat_full());
      tc::tma_load_3d(base + L::kStat1 + h * 16384u, m1, 64 * h, row_stat, bh, br.stat_full());
    }
  } else {
    tc::tma_prefetch(mB);
  }
  const int NS = isA ? kNA : kNB;
  const uint32_t ring = base + (isA ? L::kA : L::kB);
  bool ok = true;
  int issued = 0;
  for (int t = 0; t < n; ++t) {
    const int st = t % NS, k = t / NS;
    if (k > 0 && !tc::mbar_wait(isA ? br.a_empty(st) : br.b_empty(st), (k - 1) & 1, limit)) {
      ok = false;
      break;
    }
    const bool second = t >= nfirst;
    const int row = second ? (t - nfirst) * kBlock : (idx != nullptr ? idx[t] : t) * kBlock;
    const CUtensorMap* m = isA ? (second ? mA2 : mA) : (second ? mB2 : mB);
    const uint32_t full = isA ? br.a_full(st) : br.b_full(st);
    tc::mbar_expect_tx(full, L::kTile);
#pragma unroll
    for (int h = 0; h < D / 64; ++h)
      tc::tma_load_3d(ring + st * L::kTile + h * 16384u, m, 64 * h, row, bh, full);
    issued = t + 1;
  }
  // every issued copy has landed and its stage has been released before the CTA exits
  if (isA) tc::mbar_wait(br.stat_full(), 0, limit);
  for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t) {
    const int st = t % NS;
    tc::mbar_wait(isA ? br.a_full(st) : br.b_full(st), (t / NS) & 1, limit);
    tc::mbar_wait(isA ? br.a_empty(st) : br.b_empty(st), (t / NS) & 1, limit);
  }
  return ok;
}

// P for 64 columns: p[k] = exp2(s[k] c2 + off(k)), one pair in kPolyEvery on the FMA pipe
template <typename Off>
__device__ __forceinline__ void exp2_64(const uint32_t* s, float c2, Off off, float* p) {
  const uint64_t c2x2 = f2_pack(c2, c2);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])),
                               c2x2, f2_pack(off(2 * k), off(2 * k + 1)));
    if (k % kPolyEvery == 0) {
      exp2_fma2(x2, p[2 * k], p[2 * k + 1]);
    } else {
      float xa, xb;
      f2_unpack(x2, xa, xb);
      p[2 * k] = fast_exp2(xa);
      p[2 * k + 1] = fast_exp2(xb);
    }
  }
}

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t* a, float f) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 pk;
    pk.x = pack_bf16(__uint_as_float(a[8 * v + 0]) * f, __uint_as_float(a[8 * v + 1]) * f);
    pk.y = pack_bf16(__uint_as_float(a[8 * v + 2]) * f, __uint_as_float(a[8 * v + 3]) * f);
    pk.z = pack_bf16(__uint_as_float(a[8 * v + 4]) * f, __uint_as_float(a[8 * v + 5]) * f);
    pk.w = pack_bf16(__uint_as_float(a[8 * v + 6]) * f, __uint_as_float(a[8 * v + 7]) * f);
    *reinterpret_cast<uint4*>(dst + 8 * v) = pk;
  }
}

// ------------------------------------------------------------------ query-block kernel

// kPruned: packed query tiles of the pruned forward; entry t is seen only by the lane
// quarters whose bit is set in quarters[rbeg + t] (the others give it probability 0).
template <int D, bool kDPass, bool kPruned>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_row_kernel(const __grid_constant__ CUtensorMap tmQ16,
                   const __grid_constant__ CUtensorMap tmdO,
                   const __grid_constant__ CUtensorMap tmK16,
                   const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmKg16,
                   const __grid_constant__ CUtensorMap tmVg, const int32_t* __restrict__ row_ptr,
                   const int32_t* __restrict__ col_idx, const uint8_t* __restrict__ quarters,
                   const int32_t* __restrict__ order, int N, int Nq, int nb, int Np, int G,
                   float gbias2, float c2, float scale, const float* __restrict__ lse2,
                   float* __restrict__ Dvec, __nv_bfloat16* __restrict__ dq,
                   unsigned int* __restrict__ err_word, long long wait_limit) {
  using L = BwdLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int rowid = order[blockIdx.x];
  const int I = rowid % nb, bh = rowid / nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = I * kBlock;
  const int rbeg = row_ptr[bh * nb + I];
  const int nfine = row_ptr[bh * nb + I + 1] - rbeg;
  const int n = nfine + (G > 0 ? (G + kBlock - 1) / kBlock : 0);  // + ASA_G global tiles
  const int32_t* cols = col_idx + rbeg;

  const Bars br{base + L::kBars};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kTmemSlot);
  if (threadIdx.x == 0) br.init();
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      if (lane < 2)
        failed = !produce<D>(br, base, lane, &tmQ16, &tmdO, q0, &tmK16, &tmV, cols, nfine, &tmKg16,
                             &tmVg, n, bh,
                             wait_limit);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = tc::idesc_f16(128, 128, false, false);
      constexpr uint32_t idP = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idQ = tc::idesc_f16(128, D, false, true);
      const uint64_t dQ16 = tc::sdesc_sw128(base + L::kStat0, 16, 1024);
      const uint64_t dDO = tc::sdesc_sw128(base + L::kStat1, 16, 1024);
      const uint64_t dKk = tc::sdesc_sw128(base + L::kA, 16, 1024);      // K16 as B, K-major
      const uint64_t dKm = tc::sdesc_sw128(base + L::kA, 16384, 1024);   // K16 as B, MN-major
      const uint64_t dVk = tc::sdesc_sw128(base + L::kB, 16, 1024);
      auto issue_S = [&](int t) {  // S_t = Q K_t^T into S buffer t % 2
        const uint64_t kst = dKk + (((t % kNA) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::umma_ss(tmem + 128u * (t & 1), dQ16 + kmajor_step(ks), kst + kmajor_step(ks), idS,
                      ks > 0 ? 1u : 0u);
      };
      auto issue_dP = [&](int t) {  // dP_t = dO V_t^T
        const uint64_t vst = dVk + (((t % kNB) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::umma_ss(tmem + 256u, dDO + kmajor_step(ks), vst + kmajor_step(ks), idP,
                      ks > 0 ? 1u : 0u);
      };
      auto issue_dQ = [&](int t) {  // dQ += dS_t K_t, dS_t packed fp16 in S buffer t % 2
        const uint64_t kst = dKm + (((t % kNA) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          tc::umma_ts(tmem + 384u, tmem + 128u * (t & 1) + tc::packed_half_step(ks),
                      kst + ((ks * 2048u) >> 4), idQ, (t > 0 || ks > 0) ? 1u : 0u);
      };
      bool ok = tc::mbar_wait(br.stat_full(), 0, wait_limit);
      bool any = false;
      for (int t = 0; ok && t < 2 && t < n; ++t) {
        if (!(ok = tc::mbar_wait(br.a_full(t % kNA), (t / kNA) & 1, wait_limit))) break;
        tc::fence_after();
        issue_S(t);
        tc::umma_commit(br.s_full(t & 1));
        if (kDPass) tc::umma_commit(br.a_empty(t % kNA));
        any = true;
      }
      if (ok && n > 0 && (ok = tc::mbar_wait(br.b_full(0), 0, wait_limit))) {
        tc::fence_after();
        issue_dP(0);
        tc::umma_commit(br.dp_full());
        tc::umma_commit(br.b_empty(0));
      }
      for (int t = 0; ok && t < n; ++t) {
        // dP_t has been read: the next dP may overwrite it
        if (!(ok = tc::mbar_wait(br.dp_free(), t & 1, wait_limit))) break;
        if (t + 1 < n) {
          if (!(ok = tc::mbar_wait(br.b_full((t + 1) % kNB), ((t + 1) / kNB) & 1, wait_limit)))
            break;
          tc::fence_after();
          issue_dP(t + 1);
          tc::umma_commit(br.dp_full());
          tc::umma_commit(br.b_empty((t + 1) % kNB));
        }
        // D pass: S_t has been read; dQ pass: dS_t is in TMEM
        if (!(ok = tc::mbar_wait(br.ds_full(t & 1), (t >> 1) & 1, wait_limit))) break;
        tc::fence_after();
        if (!kDPass) {
          issue_dQ(t);
          tc::umma_commit(br.a_empty(t % kNA));
        }
        if (t + 2 < n) {
          if (!(ok = tc::mbar_wait(br.a_full((t + 2) % kNA), ((t + 2) / kNA) & 1, wait_limit)))
            break;
          tc::fence_after();
          issue_S(t + 2);
          tc::umma_commit(br.s_full(t & 1));
          if (kDPass) tc::umma_commit(br.a_empty((t + 2) % kNA));
        }
      }
      if (ok && !kDPass && n > 0) tc::umma_commit(br.acc_done());
      failed = !ok;
      if (any) {
        tc::umma_commit(br.drain());
        tc::mbar_wait(br.drain(), 0, wait_limit);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // ------------------------------------------------------------------ elementwise
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int q = q0 + row;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t vrow = static_cast<int64_t>(bh) * Np + q0 + row;
    const float nl2 = -lse2[vrow];  // rows past N: -inf, so P = 0
    const uint8_t* qbits = kPruned ? quarters + rbeg : nullptr;
    const float dd = kDPass ? 0.f : Dvec[vrow];
    auto wait_warp = [&](uint32_t bar, uint32_t parity) {
      const bool ok = tc::mbar_wait(bar, parity, wait_limit);
      return __all_sync(0xffffffffu, ok) != 0;
    };
    uint64_t dsum2 = f2_pack(0.f, 0.f);
    for (int t = 0; t < n; ++t) {
      const uint32_t tS = trow + 128u * (t & 1) + 64u * w;
      // global tokens carry + ln(n) (log2(n) in these units); with query pruning a
      // warp whose rows do not keep key block cols[t] gives it probability 0.  Key
      // columns past N (the ragged last block) or past G get no weight.  The CSR reads
      // come before the wait for S, so their latency is not added after it.
      const bool glob = t >= nfine;
      const bool mine = !kPruned || glob || ((qbits[t] >> quarter) & 1u);
      const float off = mine ? nl2 + (glob ? gbias2 : 0.f) : -INFINITY;
      const int nvalid = (glob ? min(kBlock, G - (t - nfine) * kBlock)
                               : min(kBlock, N - cols[t] * kBlock)) - 64 * w;
      if (!wait_warp(br.s_full(t & 1), (t >> 1) & 1)) {
        failed = true;
        break;
      }
      tc::fence_after();
      uint32_t s[64];
      tc::tmem_ld32(tS, s);
      tc::tmem_ld32(tS + 32u, s + 32);
      tc::tmem_wait_ld_dep32(s);
      tc::tmem_wait_ld_dep32(s + 32);
      if (kDPass) warp_arrive(br.ds_full(t & 1), lane);
      float p[64];
      exp2_64(s, c2, [&](int) { return off; }, p);
      if (nvalid < 64) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k >= nvalid) p[k] = 0.f;
      }
      if (!wait_warp(br.dp_full(), t & 1)) {
        failed = true;
        break;
      }
      tc::fence_after();
      uint32_t dp[64];
      tc::tmem_ld32(trow + 256u + 64u * w, dp);
      tc::tmem_ld32(trow + 256u + 64u * w + 32u, dp + 32);
      tc::tmem_wait_ld_dep32(dp);
      tc::tmem_wait_ld_dep32(dp + 32);
      warp_arrive(br.dp_free(), lane);
      if (kDPass) {
#pragma unroll
        for (int k = 0; k < 32; ++k)
          dsum2 = f2_fma(f2_pack(p[2 * k], p[2 * k + 1]),
                         f2_pack(__uint_as_float(dp[2 * k]), __uint_as_float(dp[2 * k + 1])), dsum2);
      } else {
        uint32_t ds[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          ds[k] = pack_f16(p[2 * k] * (__uint_as_float(dp[2 * k]) - dd),
                           p[2 * k + 1] * (__uint_as_float(dp[2 * k + 1]) - dd));
        tc::tmem_st16(tS, ds);
        tc::tmem_st16(tS + 16u, ds + 16);
        tc::tmem_wait_st();
        warp_arrive(br.ds_full(t & 1), lane);
      }
    }
    if (kDPass) {
      // D = the two warpgroups' partial sums; the exchange goes through Q16's tile, which
      // no MMA reads once both warpgroups have taken every S
      float da, db;
      f2_unpack(dsum2, da, db);
      const float part = da + db;
      float* red = reinterpret_cast<float*>(sbase + L::kStat0);
      tc::named_bar_sync(1, 256);
      if (w == 1) red[row] = part;
      tc::named_bar_sync(1, 256);
      if (w == 0 && q < Nq) Dvec[vrow] = part + red[row];
    } else {
      bool have = n > 0 && !failed;
      if (have) {
        if (wait_warp(br.acc_done(), 0)) {
          tc::fence_after();
        } else {
          failed = true;
          have = false;
        }
      }
      // warpgroup w writes columns [D/2 w, D/2 w + D/2) of its rows
      __nv_bfloat16* drow = dq + (static_cast<int64_t>(bh) * Nq + (q < Nq ? q : 0)) * D + (D / 2) * w;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t a[32];
        if (have) {
          tc::tmem_ld32_sync(trow + 384u + (D / 2) * w + 32u * c, a);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = 0u;
        }
        if (q < Nq) store_row_bf16(drow + 32 * c, a, scale);
      }
    }
  }

  if (failed) atomicOr(err_word, kErrWait);
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ key-block kernel

// kGlobal = false: one CTA per fine key block J, walking the query blocks that keep J
// (transposed CSR); with ASA_G (gw > 0) the epilogue adds each row's share of its
// window's global-token gradient, dKg[g] / count_g and dVg[g] / count_g, before the
// single bf16 rounding.
// kGlobal = true (ASA_G): one CTA per 128 global tokens, walking every query block
// (every query attends to every global token, logits + ln(n)); writes dKg (with the
// 1/sqrt(d)) and dVg in fp32.
template <int D, bool kGlobal>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_col_kernel(const __grid_constant__ CUtensorMap tmK16,
                   const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ16,
                   const __grid_constant__ CUtensorMap tmdO, const int32_t* __restrict__ col_ptr_t,
                   const int32_t* __restrict__ row_idx_t, const uint8_t* __restrict__ tquarters,
                   const int32_t* __restrict__ order, int N, int nbk, int nbq, int Np, int G,
                   int gw, float gbias2, float c2, float scale,
                   const float* __restrict__ lse2, const float* __restrict__ Dvec,
                   __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                   float* __restrict__ dKg32, float* __restrict__ dVg32,
                   unsigned int* __restrict__ err_word, long long wait_limit) {
  using L = BwdLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, k0, n;
  const int32_t* rows;
  const uint8_t* tq = nullptr;        // quarter bits of the query tiles (query pruning)
  if constexpr (kGlobal) {
    const int ng = (G + kBlock - 1) / kBlock;
    bh = blockIdx.x / ng;
    k0 = (blockIdx.x % ng) * kBlock;  // first global token of the tile
    n = nbq;
    rows = nullptr;                   // query block t at step t
  } else {
    const int colid = order[blockIdx.x];
    const int J = colid % nbk;
    bh = colid / nbk;
    k0 = J * kBlock;
    const int cbeg = col_ptr_t[bh * nbk + J];
    n = col_ptr_t[bh * nbk + J + 1] - cbeg;
    rows = row_idx_t + cbeg;
    if (tquarters != nullptr) tq = tquarters + cbeg;
  }

  const Bars br{base + L::kBars};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kTmemSlot);
  if (threadIdx.x == 0) br.init();
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      if (lane < 2)
        failed = !produce<D>(br, base, lane, &tmK16, &tmV, k0, &tmQ16, &tmdO, rows, n, &tmQ16,
                             &tmdO, n, bh,
                             wait_limit);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = tc::idesc_f16(128, 128, false, false);
      constexpr uint32_t idP = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idV = tc::idesc_bf16(128, D, false, true);
      constexpr uint32_t idK = tc::idesc_f16(128, D, false, true);
      const uint64_t dK16 = tc::sdesc_sw128(base + L::kStat0, 16, 1024);
      const uint64_t dVa = tc::sdesc_sw128(base + L::kStat1, 16, 1024);
      const uint64_t dQk = tc::sdesc_sw128(base + L::kA, 16, 1024);      // Q16 as B, K-major
      const uint64_t dQm = tc::sdesc_sw128(base + L::kA, 16384, 1024);   // Q16 as B, MN-major
      const uint64_t dOk = tc::sdesc_sw128(base + L::kB, 16, 1024);
      const uint64_t dOm = tc::sdesc_sw128(base + L::kB, 16384, 1024);
      auto issue_S = [&](int t) {  // S^T_t = K Q_t^T
        const uint64_t qst = dQk + (((t % kNA) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::umma_ss(tmem, dK16 + kmajor_step(ks), qst + kmajor_step(ks), idS, ks > 0 ? 1u : 0u);
      };
      auto issue_dP = [&](int t) {  // dP^T_t = V dO_t^T
        const uint64_t ost = dOk + (((t % kNB) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          tc::umma_ss(tmem + 128u, dVa + kmajor_step(ks), ost + kmajor_step(ks), idP,
                      ks > 0 ? 1u : 0u);
      };
      auto issue_dV = [&](int t) {  // dV += P^T_t dO_t
        const uint64_t ost = dOm + (((t % kNB) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          tc::umma_ts(tmem + 256u, tmem + tc::packed_half_step(ks), ost + ((ks * 2048u) >> 4), idV,
                      (t > 0 || ks > 0) ? 1u : 0u);
      };
      auto issue_dK = [&](int t) {  // dK += dS^T_t Q_t (the 1/sqrt(d) comes in the epilogue)
        const uint64_t qst = dQm + (((t % kNA) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          tc::umma_ts(tmem + 384u, tmem + 128u + tc::packed_half_step(ks), qst + ((ks * 2048u) >> 4), idK,
                      (t > 0 || ks > 0) ? 1u : 0u);
      };
      bool ok = tc::mbar_wait(br.stat_full(), 0, wait_limit);
      bool any = false;
      if (ok && n > 0) {
        if ((ok = tc::mbar_wait(br.a_full(0), 0, wait_limit))) {
          tc::fence_after();
          issue_S(0);
          tc::umma_commit(br.s_full(0));
          any = true;
          if ((ok = tc::mbar_wait(br.b_full(0), 0, wait_limit))) {
            tc::fence_after();
            issue_dP(0);
            tc::umma_commit(br.dp_full());
          }
        }
      }
      for (int t = 0; ok && t < n; ++t) {
        if (!(ok = tc::mbar_wait(br.p_full(), t & 1, wait_limit))) break;
        tc::fence_after();
        issue_dV(t);
        tc::umma_commit(br.b_empty(t % kNB));
        if (t + 1 < n) {  // S^T_{t+1} over P^T_t, after the MMA that reads it
          if (!(ok = tc::mbar_wait(br.a_full((t + 1) % kNA), ((t + 1) / kNA) & 1, wait_limit)))
            break;
          tc::fence_after();
          issue_S(t + 1);
          tc::umma_commit(br.s_full(0));
        }
        if (!(ok = tc::mbar_wait(br.ds_full(0), t & 1, wait_limit))) break;
        tc::fence_after();
        issue_dK(t);
        tc::umma_commit(br.a_empty(t % kNA));
        if (t + 1 < n) {
          if (!(ok = tc::mbar_wait(br.b_full((t + 1) % kNB), ((t + 1) / kNB) & 1, wait_limit)))
            break;
          tc::fence_after();
          issue_dP(t + 1);
          tc::umma_commit(br.dp_full());
        }
      }
      if (ok && n > 0) tc::umma_commit(br.acc_done());
      failed = !ok;
      if (any) {
        tc::umma_commit(br.drain());
        tc::mbar_wait(br.drain(), 0, wait_limit);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // ------------------------------------------------------------------ elementwise
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int kr = k0 + row;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float* l2h = lse2 + static_cast<int64_t>(bh) * Np + 64 * w;
    const float* ddh = Dvec + static_cast<int64_t>(bh) * Np + 64 * w;
    auto wait_warp = [&](uint32_t bar, uint32_t parity) {
      const bool ok = tc::mbar_wait(bar, parity, wait_limit);
      return __all_sync(0xffffffffu, ok) != 0;
    };
    const float bias = kGlobal ? gbias2 : 0.f;  // global tokens: + ln(n) in log2 units
    for (int t = 0; t < n; ++t) {
      // the query tile's lse2 and D (same addresses across the warp: broadcast loads)
      const int qb = kGlobal ? t : rows[t];
      const float4* lv = reinterpret_cast<const float4*>(l2h + qb * kBlock);
      const float4* dvv = reinterpret_cast<const float4*>(ddh + qb * kBlock);
      float off[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = __ldg(lv + c);
        off[4 * c] = bias - v.x;
        off[4 * c + 1] = bias - v.y;
        off[4 * c + 2] = bias - v.z;
        off[4 * c + 3] = bias - v.w;
      }
      if (tq != nullptr) {
        // query pruning: the 32-row quarters of the tile that do not keep this key
        // block give it probability 0 (columns 32 h .. 32 h + 31 of this warpgroup)
        const uint32_t bits = tq[t];
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (((bits >> (2 * w + h)) & 1u) == 0u) {
#pragma unroll
            for (int k = 0; k < 32; ++k) off[32 * h + k] = -INFINITY;
          }
      }
      if (!wait_warp(br.s_full(0), t & 1)) {
        failed = true;
        break;
      }
      tc::fence_after();
      uint32_t s[64];
      tc::tmem_ld32(trow + 64u * w, s);
      tc::tmem_ld32(trow + 64u * w + 32u, s + 32);
      tc::tmem_wait_ld_dep32(s);
      tc::tmem_wait_ld_dep32(s + 32);
      float p[64];
      exp2_64(s, c2, [&](int k) { return off[k]; }, p);  // query rows past N: lse2 = +inf, P = 0
      float4 dq4[16];  // the query tile's D, loaded while P^T is stored and dP^T awaited
#pragma unroll
      for (int c = 0; c < 16; ++c) dq4[c] = __ldg(dvv + c);
      uint32_t pk[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) pk[k] = pack_bf16(p[2 * k], p[2 * k + 1]);
      tc::tmem_st16(trow + 64u * w, pk);
      tc::tmem_st16(trow + 64u * w + 16u, pk + 16);
      tc::tmem_wait_st();
      warp_arrive(br.p_full(), lane);
      if (!wait_warp(br.dp_full(), t & 1)) {
        failed = true;
        break;
      }
      tc::fence_after();
      uint32_t dp[64];
      tc::tmem_ld32(trow + 128u + 64u * w, dp);
      tc::tmem_ld32(trow + 128u + 64u * w + 32u, dp + 32);
      tc::tmem_wait_ld_dep32(dp);
      tc::tmem_wait_ld_dep32(dp + 32);
      uint32_t ds[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = dq4[c];
        ds[2 * c] = pack_f16(p[4 * c] * (__uint_as_float(dp[4 * c]) - v.x),
                             p[4 * c + 1] * (__uint_as_float(dp[4 * c + 1]) - v.y));
        ds[2 * c + 1] = pack_f16(p[4 * c + 2] * (__uint_as_float(dp[4 * c + 2]) - v.z),
                                 p[4 * c + 3] * (__uint_as_float(dp[4 * c + 3]) - v.w));
      }
      tc::tmem_st16(trow + 128u + 64u * w, ds);
      tc::tmem_st16(trow + 128u + 64u * w + 16u, ds + 16);
      tc::tmem_wait_st();
      warp_arrive(br.ds_full(0), lane);
    }
    bool have = n > 0 && !failed;
    if (have) {
      if (wait_warp(br.acc_done(), 0)) {
        tc::fence_after();
      } else {
        failed = true;
        have = false;
      }
    }
    // warpgroup 0 writes dV, warpgroup 1 dK (scaled by 1/sqrt(d)); a key block that no
    // query block keeps gets zeros (plus, with ASA_G, its global share)
    const float f = w == 0 ? 1.f : scale;
    if constexpr (kGlobal) {
      float* grow = (w == 0 ? dVg32 : dKg32) + (static_cast<int64_t>(bh) * G + (kr < G ? kr : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[32];
        if (have) {
          tc::tmem_ld32_sync(trow + 256u + 128u * w + 32u * c, a);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = 0u;
        }
        if (kr < G) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<float4*>(grow + 32 * c + 4 * v) =
                make_float4(__uint_as_float(a[4 * v]) * f, __uint_as_float(a[4 * v + 1]) * f,
                            __uint_as_float(a[4 * v + 2]) * f, __uint_as_float(a[4 * v + 3]) * f);
        }
      }
    } else {
      __nv_bfloat16* drow =
          (w == 0 ? dv : dk) + (static_cast<int64_t>(bh) * N + (kr < N ? kr : 0)) * D;
      // the row's window in the global tokens (ASA_G): its gradient / the window's rows
      const float* gsrc = nullptr;
      float ginv = 0.f;
      if (gw > 0 && kr < N) {
        const int g = kr / gw;
        gsrc = (w == 0 ? dVg32 : dKg32) + (static_cast<int64_t>(bh) * G + g) * D;
        ginv = 1.f / static_cast<float>(min(gw, N - g * gw));
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[32];
        if (have) {
          tc::tmem_ld32_sync(trow + 256u + 128u * w + 32u * c, a);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = 0u;
        }
        if (kr < N) {
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = __float_as_uint(__uint_as_float(a[k]) * f);
          if (gsrc != nullptr) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 gv = *reinterpret_cast<const float4*>(gsrc + 32 * c + 4 * v);
              a[4 * v] = __float_as_uint(fmaf(gv.x, ginv, __uint_as_float(a[4 * v])));
              a[4 * v + 1] = __float_as_uint(fmaf(gv.y, ginv, __uint_as_float(a[4 * v + 1])));
              a[4 * v + 2] = __float_as_uint(fmaf(gv.z, ginv, __uint_as_float(a[4 * v + 2])));
              a[4 * v + 3] = __float_as_uint(fmaf(gv.w, ginv, __uint_as_float(a[4 * v + 3])));
            }
          }
          store_row_bf16(drow + 32 * c, a, 1.f);
        }
      }
    }
  }

  if (failed) atomicOr(err_word, kErrWait);
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ preparation

// fp16 copies of Q and K (8 elements per step; n8q and n8k pieces), lse2 padded to
// whole blocks (all +inf when lse is null: the pruned backward scatters the kept
// rows' values afterwards), D cleared
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const uint4* __restrict__ q, uint4* __restrict__ q16, int64_t n8q,
                    const uint4* __restrict__ k, uint4* __restrict__ k16, int64_t n8k,
                    const float* __restrict__ lse, float* __restrict__ lse2,
                    float* __restrict__ Dvec, int BH, int N, int Np,
                    unsigned int* __restrict__ err_word) {
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t bad = 0;
  auto cvt = [&](uint32_t v) {
    const uint32_t h = bf16x2_to_f16x2(v);
    bad |= ((h & 0x7c00u) == 0x7c00u) | ((h & 0x7c000000u) == 0x7c000000u);
    return h;
  };
  for (int64_t j = i0; j < n8q; j += stride) {
    const uint4 a = q[j];
    q16[j] = make_uint4(cvt(a.x), cvt(a.y), cvt(a.z), cvt(a.w));
  }
  for (int64_t j = i0; j < n8k; j += stride) {
    const uint4 b = k[j];
    k16[j] = make_uint4(cvt(b.x), cvt(b.y), cvt(b.z), cvt(b.w));
  }
  const int64_t nv = static_cast<int64_t>(BH) * Np;
  for (int64_t j = i0; j < nv; j += stride) {
    const int64_t h = j / Np;
    const int r = static_cast<int>(j - h * Np);
    lse2[j] = (lse != nullptr && r < N) ? lse[h * N + r] * kLog2e : INFINITY;
    Dvec[j] = 0.f;
  }
  if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0) atomicOr(err_word, kErrRange);
}

// fp16 copy of a bf16 tensor (8 elements per step; overflow ORs kErrRange)
__global__ void __launch_bounds__(256)
    f16_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n8,
                    unsigned int* __restrict__ err_word) {
  uint32_t bad = 0;
  auto cvt = [&](uint32_t v) {
    const uint32_t h = bf16x2_to_f16x2(v);
    bad |= ((h & 0x7c00u) == 0x7c00u) | ((h & 0x7c000000u) == 0x7c000000u);
    return h;
  };
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n8;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 a = src[j];
    dst[j] = make_uint4(cvt(a.x), cvt(a.y), cvt(a.z), cvt(a.w));
  }
  if (__any_sync(0xffffffffu, bad != 0) && (threadIdx.x & 31) == 0) atomicOr(err_word, kErrRange);
}

size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// D = rowsum(dO * O) from a stored O: the bf16 O of the inference forward (the opt-in
// approximate D) or the fp32 O of the training forward.  One warp per row, fp32
// accumulation; rows past N keep the 0 of bwd_prep.
template <int D, bool kF32>
__global__ void __launch_bounds__(256)
    d_from_o_kernel(const __nv_bfloat16* __restrict__ dout, const void* __restrict__ o,
                    int64_t rows, int N, int Np, float* __restrict__ Dvec) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps) {
    const __nv_bfloat16* a = dout + row * D + lane * E;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t ua = *reinterpret_cast<const uint32_t*>(a + e);
      float b0, b1;
      if constexpr (kF32) {
        const float2 v = *reinterpret_cast<const float2*>(static_cast<const float*>(o) + row * D +
                                                          lane * E + e);
        b0 = v.x;
        b1 = v.y;
      } else {
        const uint32_t ub = *reinterpret_cast<const uint32_t*>(
            static_cast<const __nv_bfloat16*>(o) + row * D + lane * E + e);
        b0 = __uint_as_float(ub << 16);
        b1 = __uint_as_float(ub & 0xffff0000u);
      }
      acc = fmaf(__uint_as_float(ua << 16), b0, acc);
      acc = fmaf(__uint_as_float(ua & 0xffff0000u), b1, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const int64_t bh = row / N;
      Dvec[bh * Np + (row - bh * N)] = acc;
    }
  }
}

// Workspace pieces (256-byte aligned, in this order): lse2, D [BH][nbq*128] f32; Q16
// [BH][Nq][d] f16, K16 [BH][N][d] f16; launch orders of query and key blocks
// [BH*nbq], [BH*nbk] i32; with ASA_G (G global tokens): Kg, Vg [BH][G][d] bf16, Kg16
// [BH][G][d] f16, dKg, dVg [BH][G][d] f32.  Without pruning Nq = N; with it Nq = Ns,
// the compact query rows, and the pruned pieces follow (carve_pruned).
struct BwdWs {
  float *lse2, *Dvec;
  void *q16, *k16;
  int32_t *ord_r, *ord_c;
  void *kg, *vg, *kg16;
  float *dkg, *dvg;
  size_t bytes;
};

BwdWs carve_bwd(void* base, int BH, int Nq, int N, int d, int G) {
  const size_t nbq = (static_cast<size_t>(Nq) + kBlock - 1) / kBlock;
  const size_t nbk = (static_cast<size_t>(N) + kBlock - 1) / kBlock;
  char* w = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = w == nullptr ? nullptr : w + off;
    off += a256(bytes);
    return p;
  };
  BwdWs r{};
  r.lse2 = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * nbq * kBlock * 4));
  r.Dvec = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * nbq * kBlock * 4));
  r.q16 = take(static_cast<size_t>(BH) * Nq * d * 2);
  r.k16 = take(static_cast<size_t>(BH) * N * d * 2);
  r.ord_r = reinterpret_cast<int32_t*>(take(static_cast<size_t>(BH) * nbq * 4));
  r.ord_c = reinterpret_cast<int32_t*>(take(static_cast<size_t>(BH) * nbk * 4));
  if (G > 0) {
    const size_t gd = static_cast<size_t>(BH) * G * d;
    r.kg = take(gd * 2);
    r.vg = take(gd * 2);
    r.kg16 = take(gd * 2);
    r.dkg = reinterpret_cast<float*>(take(gd * 4));
    r.dvg = reinterpret_cast<float*>(take(gd * 4));
  }
  r.bytes = off;
  return r;
}

// Query side: Nq rows in nbq blocks (CSR row_ptr/col_idx over them, quarter bits
// `quarters` with query pruning); key side: N rows in nbk blocks (transposed CSR
// col_ptr_t/row_idx_t, quarter bits `tquarters`).
template <int D, bool kPruned>
cudaError_t launch_kernels(const CUtensorMap* maps, const int32_t* row_ptr,
                           const int32_t* col_idx, const uint8_t* quarters,
                           const int32_t* col_ptr_t, const int32_t* row_idx_t,
                           const uint8_t* tquarters, const BwdWs& ws, int BH, int N, int Nq,
                           int G, int gw, void* dq, void* dk, void* dv, unsigned int* err_word,
                           cudaStream_t stream, bool d_pass = true) {
  using L = BwdLayout<D>;
  const int nbq = (Nq + kBlock - 1) / kBlock;
  const int nbk = (N + kBlock - 1) / kBlock;
  const int Np = nbq * kBlock;
  const float c2 = kLog2e / sqrtf(static_cast<float>(D));
  const float scale = 1.f / sqrtf(static_cast<float>(D));
  const float gbias2 = gw > 0 ? log2f(static_cast<float>(gw)) : 0.f;
  const long long limit = 1ll << 31;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwd_row_kernel<D, true, kPruned>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem)) ||
      (e = cudaFuncSetAttribute(bwd_row_kernel<D, false, kPruned>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem)) ||
      (e = cudaFuncSetAttribute(bwd_col_kernel<D, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem)) ||
      (e = cudaFuncSetAttribute(bwd_col_kernel<D, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem)))
    return e;
  static int regs_checked = 0;
  if (regs_checked == 0) {
    const void* fns[4] = {reinterpret_cast<const void*>(bwd_row_kernel<D, true, kPruned>),
                          reinterpret_cast<const void*>(bwd_row_kernel<D, false, kPruned>),
                          reinterpret_cast<const void*>(bwd_col_kernel<D, false>),
                          reinterpret_cast<const void*>(bwd_col_kernel<D, true>)};
    regs_checked = 1;
    for (const void* fn : fns) {
      cudaFuncAttributes fa{};
      if ((e = cudaFuncGetAttributes(&fa, fn))) return e;
      if (fa.numRegs != kLaunchRegs) regs_checked = -1;
    }
  }
  if (regs_checked < 0) return cudaErrorInvalidConfiguration;
  const int grid_q = BH * nbq, grid_k = BH * nbk;
  // maps: Q16, dO, K16, V, Kg16, Vg (the last two stand in for K16, V without ASA_G)
  if (d_pass) {  // otherwise D is already in ws.Dvec (rowsum(dO * O) from the stored O)
    bwd_row_kernel<D, true, kPruned><<<grid_q, kBwdThreads, L::kSmem, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], row_ptr, col_idx, quarters,
        ws.ord_r, N, Nq, nbq, Np, G, gbias2, c2, scale, ws.lse2, ws.Dvec, nullptr, err_word, limit);
    if ((e = cudaGetLastError())) return e;
  }
  if (G > 0) {
    const int gtiles = BH * ((G + kBlock - 1) / kBlock);
    bwd_col_kernel<D, true><<<gtiles, kBwdThreads, L::kSmem, stream>>>(
        maps[4], maps[5], maps[0], maps[1], col_ptr_t, row_idx_t, nullptr, ws.ord_c, N, nbk, nbq,
        Np, G, gw, gbias2, c2, scale, ws.lse2, ws.Dvec, nullptr, nullptr, ws.dkg, ws.dvg,
        err_word, limit);
    if ((e = cudaGetLastError())) return e;
  }
  bwd_col_kernel<D, false><<<grid_k, kBwdThreads, L::kSmem, stream>>>(
      maps[2], maps[3], maps[0], maps[1], col_ptr_t, row_idx_t, tquarters, ws.ord_c, N, nbk, nbq,
      Np, G, gw, gbias2, c2, scale, ws.lse2, ws.Dvec, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), ws.dkg, ws.dvg, err_word, limit);
  if ((e = cudaGetLastError())) return e;
  bwd_row_kernel<D, false, kPruned><<<grid_q, kBwdThreads, L::kSmem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], row_ptr, col_idx, quarters, ws.ord_r,
      N, Nq, nbq, Np, G, gbias2, c2, scale, ws.lse2, ws.Dvec, static_cast<__nv_bfloat16*>(dq),
      err_word, limit);
  return cudaGetLastError();
}

// Tensor maps of the backward: Q16 (Nq rows), dO (Nq rows), K16, V (N rows) and the
// ASA_G global tokens (or K16, V again).
bool make_bwd_maps(CUtensorMap* maps, const BwdWs& ws, const void* dout, const void* vp, int BH,
                   int Nq, int N, int G, int d) {
  if (!make_map_rows_f16(&maps[0], ws.q16, BH, Nq, d) || !make_map_rows(&maps[1], dout, BH, Nq, d) ||
      !make_map_rows_f16(&maps[2], ws.k16, BH, N, d) || !make_map_rows(&maps[3], vp, BH, N, d))
    return false;
  if (G > 0)
    return make_map_rows_f16(&maps[4], ws.kg16, BH, G, d) && make_map_rows(&maps[5], ws.vg, BH, G, d);
  maps[4] = maps[2];
  maps[5] = maps[3];
  return true;
}

// the forward's global tokens, recomputed: mean-pooled K and V, Kg also in fp16
cudaError_t global_tokens(const void* kp, const void* vp, const BwdWs& ws, int BH, int N, int d,
                          int gw, int G, unsigned int* err_word, int num_sms, cudaStream_t stream) {
  cudaError_t e = launch_global_pool(kp, ws.kg, BH, N, d, gw, num_sms, stream, vp, ws.vg);
  if (e != cudaSuccess) return e;
  f16_copy_kernel<<<num_sms * 8, 256, 0, stream>>>(static_cast<const uint4*>(ws.kg),
                                                   static_cast<uint4*>(ws.kg16),
                                                   static_cast<int64_t>(BH) * G * d / 8, err_word);
  return cudaGetLastError();
}

// The pruned backward's own pieces, after carve_bwd's: dO' and dQ in the compact
// layout [BH][Ns][d] bf16; the dense quarter matrix [BH][ntile][nbk] u8; the
// transposed tile CSR (counts [BH*nbk], col_ptr [BH*nbk + 1], tile index and quarter
// bits with room for every (tile, key block) pair).
struct PrunedWs {
  void *dout_s, *dq_s;
  uint8_t* qmat;
  int32_t *counts, *tcol_ptr, *trow_idx;
  uint8_t* tquarters;
  size_t bytes;
};

PrunedWs carve_pruned(void* base, size_t start, int BH, int N, int Ns, int d) {
  const size_t ntile = static_cast<size_t>(Ns) / kBlock;
  const size_t nbk = (static_cast<size_t>(N) + kBlock - 1) / kBlock;
  char* w = static_cast<char*>(base);
  size_t off = start;
  auto take = [&](size_t bytes) {
    char* p = w == nullptr ? nullptr : w + off;
    off += a256(bytes);
    return p;
  };
  PrunedWs r{};
  const size_t pairs = static_cast<size_t>(BH) * ntile * nbk;
  r.dout_s = take(static_cast<size_t>(BH) * Ns * d * 2);
  r.dq_s = take(static_cast<size_t>(BH) * Ns * d * 2);
  r.qmat = reinterpret_cast<uint8_t*>(take(pairs));
  r.counts = reinterpret_cast<int32_t*>(take(static_cast<size_t>(BH) * nbk * 4));
  r.tcol_ptr = reinterpret_cast<int32_t*>(take((static_cast<size_t>(BH) * nbk + 1) * 4));
  r.trow_idx = reinterpret_cast<int32_t*>(take(pairs * 4));
  r.tquarters = reinterpret_cast<uint8_t*>(take(pairs));
  r.bytes = off;
  return r;
}

}  // namespace

cudaError_t launch_f16_copy(const void* src, void* dst, int64_t n, unsigned int* err_word,
                            int num_sms, cudaStream_t stream) {
  f16_copy_kernel<<<num_sms * 8, 256, 0, stream>>>(static_cast<const uint4*>(src),
                                                   static_cast<uint4*>(dst), n / 8, err_word);
  return cudaGetLastError();
}

size_t bwd_tc_workspace_bytes(int BH, int N, int d, int global_window) {
  if (BH < 1 || N < 1 || global_window < 0) return 0;
  const int G = global_window > 0 ? (N + global_window - 1) / global_window : 0;
  return carve_bwd(nullptr, BH, N, N, d, G).bytes;
}

size_t bwd_tc_pruned_workspace_bytes(int BH, int N, int Ns, int d, int global_window) {
  if (BH < 1 || N < 1 || Ns < kBlock || Ns % kBlock != 0 || global_window < 0) return 0;
  const int G = global_window > 0 ? (N + global_window - 1) / global_window : 0;
  const size_t base = carve_bwd(nullptr, BH, Ns, N, d, G).bytes;
  return carve_pruned(nullptr, base, BH, N, Ns, d).bytes;
}

cudaError_t launch_bwd_tc(const void* qp, const void* kp, const void* vp, const void* dout,
                          const float* lse, const int32_t* row_ptr, const int32_t* col_idx,
                          const int32_t* col_ptr_t, const int32_t* row_idx_t, int BH, int N,
                          int d, int global_window, void* workspace, void* dq, void* dk, void* dv,
                          unsigned int* err_word, int num_sms, cudaStream_t stream,
                          const void* o_for_d, bool o_f32) {
  const int nb = (N + kBlock - 1) / kBlock;
  const int Np = nb * kBlock;
  const int gw = global_window;
  const int G = gw > 0 ? (N + gw - 1) / gw : 0;
  const BwdWs ws = carve_bwd(workspace, BH, N, N, d, G);
  CUtensorMap maps[6];
  if (!make_bwd_maps(maps, ws, dout, vp, BH, N, N, G, d)) return cudaErrorInvalidValue;
  const int64_t n8 = static_cast<int64_t>(BH) * N * d / 8;
  bwd_prep_kernel<<<num_sms * 8, 256, 0, stream>>>(
      static_cast<const uint4*>(qp), static_cast<uint4*>(ws.q16), n8,
      static_cast<const uint4*>(kp), static_cast<uint4*>(ws.k16), n8, lse, ws.lse2, ws.Dvec, BH,
      N, Np, err_word);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && G > 0) e = global_tokens(kp, vp, ws, BH, N, d, gw, G, err_word, num_sms, stream);
  if (e == cudaSuccess) e = launch_lpt_order(row_ptr, BH, nb, nb, ws.ord_r, stream);
  if (e == cudaSuccess) e = launch_lpt_order(col_ptr_t, BH, nb, nb, ws.ord_c, stream);
  if (e == cudaSuccess && o_for_d != nullptr) {
    const int64_t rows = static_cast<int64_t>(BH) * N;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>((rows + 7) / 8, num_sms * 16));
    const auto* a = static_cast<const __nv_bfloat16*>(dout);
    if (o_f32 && d == 128)
      d_from_o_kernel<128, true><<<grid, 256, 0, stream>>>(a, o_for_d, rows, N, Np, ws.Dvec);
    else if (o_f32)
      d_from_o_kernel<64, true><<<grid, 256, 0, stream>>>(a, o_for_d, rows, N, Np, ws.Dvec);
    else if (d == 128)
      d_from_o_kernel<128, false><<<grid, 256, 0, stream>>>(a, o_for_d, rows, N, Np, ws.Dvec);
    else
      d_from_o_kernel<64, false><<<grid, 256, 0, stream>>>(a, o_for_d, rows, N, Np, ws.Dvec);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  const bool d_pass = o_for_d == nullptr;
  if (d == 128)
    return launch_kernels<128, false>(maps, row_ptr, col_idx, nullptr, col_ptr_t, row_idx_t,
                                      nullptr, ws, BH, N, N, G, gw, dq, dk, dv, err_word, stream,
                                      d_pass);
  return launch_kernels<64, false>(maps, row_ptr, col_idx, nullptr, col_ptr_t, row_idx_t, nullptr,
                                   ws, BH, N, N, G, gw, dq, dk, dv, err_word, stream, d_pass);
}

// Backward with query pruning on the packed tiles of the pruned forward: the query
// side runs over the compact rows (Ns per head: ntile tiles), each (tile, key block)
// entry restricted to the lane quarters whose block keeps it; the key side walks the
// transposed tile CSR.  Work is proportional to the packed forward's.
cudaError_t launch_bwd_tc_pruned(const void* q_s, const void* kp, const void* vp, const void* dout,
                                 const float* lse, const int32_t* src_pos, const int32_t* src_row,
                                 const int32_t* tile_ptr, const int32_t* tile_col,
                                 const uint8_t* tile_quarters, int BH, int N, int Ns, int d,
                                 int global_window, void* workspace, void* dq, void* dk, void* dv,
                                 unsigned int* err_word, int num_sms, cudaStream_t stream) {
  const int ntile = Ns / kBlock;
  const int nbk = (N + kBlock - 1) / kBlock;
  const int gw = global_window;
  const int G = gw > 0 ? (N + gw - 1) / gw : 0;
  const BwdWs ws = carve_bwd(workspace, BH, Ns, N, d, G);
  const PrunedWs pw = carve_pruned(workspace, ws.bytes, BH, N, Ns, d);
  CUtensorMap maps[6];
  if (!make_bwd_maps(maps, ws, pw.dout_s, vp, BH, Ns, N, G, d)) return cudaErrorInvalidValue;
  // compact dO' (unused rows zero) and lse2 (unused rows +inf: probability 0)
  cudaError_t e = cudaMemsetAsync(pw.dout_s, 0, static_cast<size_t>(BH) * Ns * d * 2, stream);
  if (e != cudaSuccess) return e;
  bwd_prep_kernel<<<num_sms * 8, 256, 0, stream>>>(
      static_cast<const uint4*>(q_s), static_cast<uint4*>(ws.q16),
      static_cast<int64_t>(BH) * Ns * d / 8, static_cast<const uint4*>(kp),
      static_cast<uint4*>(ws.k16), static_cast<int64_t>(BH) * N * d / 8, nullptr, ws.lse2, ws.Dvec,
      BH, Ns, Ns, err_word);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_dout_compact(dout, lse, src_pos, src_row, BH, N, Ns, d, pw.dout_s, ws.lse2, err_word,
                          num_sms, stream);
  if (e == cudaSuccess && G > 0) e = global_tokens(kp, vp, ws, BH, N, d, gw, G, err_word, num_sms, stream);
  if (e == cudaSuccess)
    e = launch_tile_transpose(tile_ptr, tile_col, tile_quarters, BH, ntile, nbk, pw.qmat, pw.counts,
                              pw.tcol_ptr, pw.trow_idx, pw.tquarters, err_word, num_sms, stream);
  if (e == cudaSuccess) e = launch_lpt_order(tile_ptr, BH, ntile, nbk, ws.ord_r, stream);
  if (e == cudaSuccess) e = launch_lpt_order(pw.tcol_ptr, BH, nbk, ntile, ws.ord_c, stream);
  if (e != cudaSuccess) return e;
  if (d == 128)
    e = launch_kernels<128, true>(maps, tile_ptr, tile_col, tile_quarters, pw.tcol_ptr,
                                  pw.trow_idx, pw.tquarters, ws, BH, N, Ns, G, gw, pw.dq_s, dk, dv,
                                  err_word, stream);
  else
    e = launch_kernels<64, true>(maps, tile_ptr, tile_col, tile_quarters, pw.tcol_ptr, pw.trow_idx,
                                 pw.tquarters, ws, BH, N, Ns, G, gw, pw.dq_s, dk, dv, err_word,
                                 stream);
  if (e != cudaSuccess) return e;
  return launch_dq_scatter(pw.dq_s, src_pos, src_row, BH, N, Ns, d, dq, err_word, num_sms, stream);
}

}  // namespace asa
