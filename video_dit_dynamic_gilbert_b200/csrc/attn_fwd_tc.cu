// Block-sparse attention forward on tcgen05 tensor cores (Video-BLADE, "Step 2.2:
// Computation": standard ASA over the kept tiles of M, and ASA_G with global tokens).
//
// One CTA per (b, h, query block I of 128 rows), 12 warps, warp-specialised:
//   warp 0      TMA producer: Q once, then for every kept key block J (the CSR row
//               of I) its 128-row K and V tiles into an NST-stage ring; for ASA_G
//               then the ceil(N/n) global tokens in 128-row tiles.  Rows past N
//               (ragged last block) are zero-filled by TMA.
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_j = Q K_j^T   (SS MMA, M=128 N=128) into TMEM S buffer j%2,
//                 O_{j%2} += P_j V_j   (TS MMA: P read from TMEM, V from shared memory).
//   warps 2, 3  idle (they complete warpgroup 0 for the register split)
//   warps 4..11 two softmax warpgroups.  Warpgroup w takes the tiles j = w, w+2, ...:
//               an independent online softmax (running max / sum in the log2 domain)
//               with its own S buffer and its own O accumulator, so that one
//               warpgroup's loads, reductions and stores overlap the other's exp2 work
//               and the tensor pipe always has a tile to run.  Thread = query row =
//               TMEM lane.  P_j is written as bf16 over S_j; O is rescaled in TMEM only
//               when the running max grows by more than 2^8 (until then P is taken
//               against the stale max; exact after the final division).  Epilogue:
//               the two partial results are merged (max, scaled sums) and O / l is
//               written as bf16 rows with the natural-log LSE.
// TMEM: S buffers at columns [0,128) and [128,256), O_0 at [256,256+D), O_1 at
// [384,384+D).
// Training variant (kTrain): P is packed as fp16 and multiplies an fp16 copy of V (a
// kind::f16 MMA takes A and B of one type), and the merged fp32 O is also written out.
// P <= 2^8 by the rescale rule, so fp16 holds it; its 11 significant bits put ~8x less
// rounding error on O than bf16's 8, which is what lets the backward take
// D = rowsum(dO o O) from that fp32 O instead of a pass of its own.  Every wait is bounded: on expiry the kernel sets the device error word,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "softmax_math.cuh"
#include "tc.cuh"

namespace asa {

namespace {

constexpr int kFwdTcThreads = 384;  // warpgroup 0: producer, MMA; 1, 2: softmax streams
// Register split (launch: 384 threads x 168 = 64,512 registers): warpgroup 0 gives
// back to 72 per thread, the softmax warpgroups grow to 216.  128 x 72 + 256 x 216 =
// 64,512; per sub-partition one warp of each warpgroup: 32 x (72 + 2 x 216) <= 16,384.
// The launcher checks the compiled count: a split above the launch allocation would
// wait forever.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kRegsLow = 72, kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh == kFwdTcThreads * kLaunchRegs,
              "register split must equal the launch allocation");
constexpr uint32_t kTmemCols = 512;

template <int D, int NST>
struct FwdTcLayout {
  static constexpr uint32_t kTile = 128u * D * 2u;  // one 128-row bf16 tile of Q, K or V
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kV = kK + NST * kTile;
  static constexpr uint32_t kBars = kV + NST * kTile;
  // barriers: q_full, k_full[NST], v_full[NST], k_empty[NST], v_empty[NST], s_full[2],
  //           p_full[2], o_done[2], drain; then the TMEM base address slot
  static constexpr uint32_t kNumBars = 1 + 4 * NST + 2 + 2 + 2 + 1;
  static constexpr uint32_t kTmemSlot = kBars + 8 * kNumBars;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;  // + alignment slack
};

// One in kPolyEvery(D) P pairs takes exp2_fma (0: all on MUFU).  A single softmax warp
// reaches only part of MUFU's 4 exp2/clk per sub-partition; measured best: one pair in
// 4 at d=64 (the tile is exponential-bound), one in 8 at d=128.
template <int D>
constexpr int poly_every() { return D == 128 ? 8 : 4; }

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

// kPruned: the query tiles are packed tiles of pruned queries (Nq rows per head).
// Entry e of the tile's CSR row is seen only by the 32-row lane quarters q with bit q
// of quarters[e] set; the other quarters' rows give that key tile probability 0.
template <int D, int NST, bool kPruned, bool kTrain>
__global__ void __launch_bounds__(kFwdTcThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKg,
                  const __grid_constant__ CUtensorMap tmVg, const int32_t* __restrict__ row_ptr,
                  const int32_t* __restrict__ col_idx, const uint8_t* __restrict__ quarters,
                  const int32_t* __restrict__ order, int N, int Nq, int nb, int G, float gbias2,
                  float c2, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                  float* __restrict__ o32, const int32_t* __restrict__ perm_out, int H,
                  unsigned int* __restrict__ err_word, long long wait_limit) {
  using L = FwdTcLayout<D, NST>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);

  // CTAs take the heads in order and, inside a head, the longest query blocks first
  const int rowid = order[blockIdx.x];
  const int I = rowid % nb, bh = rowid / nb;
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
  auto k_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NST + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (1 + 3 * NST + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 4 * NST + b); };
  auto p_full = [&](int b) { return bar0 + 8u * (3 + 4 * NST + b); };
  auto o_done = [&](int b) { return bar0 + 8u * (5 + 4 * NST + b); };
  const uint32_t drain = bar0 + 8u * (7 + 4 * NST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kTmemSlot);

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full(), 1);
    for (int s = 0; s < NST; ++s) {
      tc::mbar_init(k_full(s), 1);
      tc::mbar_init(v_full(s), 1);
      tc::mbar_init(k_empty(s), 1);
      tc::mbar_init(v_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full(b), 1);
      tc::mbar_init(p_full(b), 128);
      tc::mbar_init(o_done(b), 1);
    }
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

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers
    // lane 0 streams Q and the K tiles, lane 1 the V tiles: a K stage is released as
    // soon as its S MMA completes, a V stage only after its PV MMA.
    if (lane < 2) {
      const bool isK = lane == 0;
      if (isK) {
        tc::tma_prefetch(&tmQ);
        tc::tma_prefetch(&tmK);
        tc::mbar_expect_tx(q_full(), L::kTile);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(base + L::kQ + h * 16384u, &tmQ, 64 * h, q0, bh, q_full());
      } else {
        tc::tma_prefetch(&tmV);
      }
      const uint32_t ring = base + (isK ? L::kK : L::kV);
      int issued = 0;
      for (int j = 0; j < ntile; ++j) {
        const int st = j % NST, n = j / NST;
        if (n > 0 && !tc::mbar_wait(isK ? k_empty(st) : v_empty(st), (n - 1) & 1, wait_limit)) {
          failed = true;
          break;
        }
        const TileSrc t = tile_src(j, nfine, cols, N, G);
        const CUtensorMap* m = t.global ? (isK ? &tmKg : &tmVg) : (isK ? &tmK : &tmV);
        const uint32_t full = isK ? k_full(st) : v_full(st);
        tc::mbar_expect_tx(full, L::kTile);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tc::tma_load_3d(ring + st * L::kTile + h * 16384u, m, 64 * h, t.row0, bh, full);
        issued = j + 1;
      }
      // drain: every issued copy has landed, and the MMAs have released the last
      // stages (their commits arrive before the CTA exits)
      if (isK) tc::mbar_wait(q_full(), 0, wait_limit);
      for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j) {
        tc::mbar_wait(isK ? k_full(j % NST) : v_full(j % NST), (j / NST) & 1, wait_limit);
        tc::mbar_wait(isK ? k_empty(j % NST) : v_empty(j % NST), (j / NST) & 1, wait_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idPV =
          kTrain ? tc::idesc_f16(128, D, false, true) : tc::idesc_bf16(128, D, false, true);
      // Descriptors are built once; an offset of `o` bytes into a tile adds o >> 4 to
      // the start-address field (all tiles lie below 256 KB, so it never carries).
      const uint64_t dQ = tc::sdesc_sw128(base + L::kQ, 16, 1024);
      const uint64_t dK = tc::sdesc_sw128(base + L::kK, 16, 1024);
      const uint64_t dV = tc::sdesc_sw128(base + L::kV, 16384, 1024);
      // S_j = Q K_j^T into S buffer j % 2
      auto issue_s = [&](int j) {
        const uint32_t dS = tmem + 128u * (j & 1);
        const uint64_t kst = dK + (((j % NST) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * 16384u + (ks & 3) * 32u) >> 4;
          tc::umma_ss(dS, dQ + off, kst + off, idS, ks > 0 ? 1u : 0u);
        }
      };
      bool ok = tc::mbar_wait(q_full(), 0, wait_limit);
      int issued_any = 0;
      // the first tile of each stream
      for (int j = 0; ok && j < 2 && j < ntile; ++j) {
        if (!(ok = tc::mbar_wait(k_full(j % NST), (j / NST) & 1, wait_limit))) break;
        tc::fence_after();
        issue_s(j);
        tc::umma_commit(s_full(j & 1));
        tc::umma_commit(k_empty(j % NST));
        issued_any = 1;
      }
      for (int j = 0; ok && j < ntile; ++j) {
        const int b = j & 1;
        // operands first, P last: once P_j lands, PV_j and S_{j+2} issue at once
        if (!(ok = tc::mbar_wait(v_full(j % NST), (j / NST) & 1, wait_limit))) break;
        if (j + 2 < ntile &&
            !(ok = tc::mbar_wait(k_full((j + 2) % NST), ((j + 2) / NST) & 1, wait_limit)))
          break;
        if (!(ok = tc::mbar_wait(p_full(b), (j >> 1) & 1, wait_limit))) break;
        tc::fence_after();
        // O_b += P_j V_j; the first tile of a stream initialises its O
        const uint32_t tP = tmem + 128u * b;
        const uint32_t tO = tmem + 256u + 128u * b;
        const uint64_t vst = dV + (((j % NST) * L::kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < kBlock / 16; ++ks)
          tc::umma_ts(tO, tP + 8u * ks, vst + ((ks * 2048u) >> 4), idPV,
                      (j >= 2 || ks > 0) ? 1u : 0u);
        // the stream's next S goes into the buffer P_j just left (in issue order); the
        // commits follow both MMA groups (each costs the issuing thread, and a commit
        // tracks every MMA issued before it).  MMAs of one thread complete in order, so
        // the S_{j+2} that the stream waits for next also tells it that PV_j is done;
        // o_done is committed only after a stream's last PV, for the epilogue.
        if (j + 2 < ntile) issue_s(j + 2);
        tc::umma_commit(v_empty(j % NST));
        if (j + 2 < ntile) {
          tc::umma_commit(s_full(b));
          tc::umma_commit(k_empty((j + 2) % NST));
        } else {
          tc::umma_commit(o_done(b));
        }
      }
      failed = !ok;
      if (issued_any) {
        // drain: all MMAs of this CTA complete before TMEM is released
        tc::umma_commit(drain);
        tc::mbar_wait(drain, 0, wait_limit);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // ------------------------------------------------------------ softmax warpgroups
    // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform
    // (wait results are AND-reduced over the warp).
    const int w = (warp - 4) >> 2;  // stream: tiles w, w + 2, ...
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t tS = trow + 128u * w;
    const uint32_t tO = trow + 256u + 128u * w;
    auto wait_warp = [&](uint32_t bar, uint32_t parity) {
      const bool ok = tc::mbar_wait(bar, parity, wait_limit);
      return __all_sync(0xffffffffu, ok) != 0;
    };
    float m_ref = -INFINITY, l = 0.f;
    int it = 0;  // tiles of this stream done
    for (int j = w; j < ntile; j += 2, ++it) {
      // the tile's key block (and, with pruning, its lane-quarter bits) are read before
      // the wait for S, so that their load latency is not added after it
      const TileSrc t = tile_src(j, nfine, cols, N, G);
      const bool skip = kPruned && !t.global && ((quarters[rbeg + j] >> quarter) & 1u) == 0u;
      if (!wait_warp(s_full(w), it & 1)) {
        failed = true;
        break;
      }
      tc::fence_after();
      if constexpr (kPruned) {
        if (skip) {
          // these rows do not keep key block cols[j]: P = 0, running max and sum unchanged
          uint32_t z[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) z[k] = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) tc::tmem_st16(tS + 16u * c, z);
          tc::tmem_wait_st();
          tc::fence_before();
          tc::mbar_arrive(p_full(w));
          continue;
        }
      }
      const float bias = t.global ? gbias2 : 0.f;
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(tS + 32u * c, s + 32 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_wait_ld_dep32(s + 32 * c);
      // full tiles skip every per-column validity test
      if (t.nvalid < kBlock) {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= t.nvalid) s[k] = __float_as_uint(-INFINITY);
      }
      // row max on the raw scores (c2 > 0 keeps the order)
      float m0 = max3f(__uint_as_float(s[0]), __uint_as_float(s[1]), __uint_as_float(s[2]));
      float m1 = max3f(__uint_as_float(s[3]), __uint_as_float(s[4]), __uint_as_float(s[5]));
#pragma unroll
      for (int k = 6; k < 126; k += 4) {
        m0 = max3f(m0, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
        m1 = max3f(m1, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]));
      }
      const float mraw = max3f(m0, m1, fmaxf(__uint_as_float(s[126]), __uint_as_float(s[127])));
      const float mx = fmaf(mraw, c2, bias);
      const float m_new = fmaxf(m_ref, mx);
      const bool need = m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + 8.f);
      const bool any_need = __any_sync(0xffffffffu, need) != 0;
      const float alpha = need ? (m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - m_new)) : 1.f;
      if (need) m_ref = m_new;
      // P = exp2(s c2 + bias - m) packed to bf16 pairs, fp16 in training (masked columns
      // give exp2(-inf) = 0)
      const float off = bias - (m_ref == -INFINITY ? 0.f : m_ref);
      uint32_t p[64];
      const uint64_t c2x2 = f2_pack(c2, c2), offx2 = f2_pack(off, off);
      uint64_t rs = f2_pack(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const uint64_t x2 =
            f2_fma(f2_pack(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2x2, offx2);
        float a, bb;
        constexpr int kPolyEvery = poly_every<D>();
        if (kPolyEvery > 0 && (k % (kPolyEvery > 0 ? kPolyEvery : 1)) == 0) {
          exp2_fma2(x2, a, bb);
        } else {
          float xa, xb;
          f2_unpack(x2, xa, xb);
          a = fast_exp2(xa);
          bb = fast_exp2(xb);
        }
        rs = f2_add(rs, f2_pack(a, bb));
        p[k] = kTrain ? pack_f16(a, bb) : pack_bf16(a, bb);
      }
      float rsa, rsb;
      f2_unpack(rs, rsa, rsb);
      l = l * alpha + (rsa + rsb);
      if (it > 0) {
        // this stream's previous PV is done (it was issued before this tile's S, which
        // has completed): O may be rescaled
        if (any_need) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tc::tmem_ld32_sync(tO + 32u * c, ov);
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tc::tmem_st16(tO + 32u * c, ov);
            tc::tmem_st16(tO + 32u * c + 16u, ov + 16);
            tc::tmem_wait_st();
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_st16(tS + 16u * c, p + 16 * c);
      tc::tmem_wait_st();
      tc::fence_before();
      tc::mbar_arrive(p_full(w));
    }
    // this stream's last PV (o_done is committed once per stream)
    const bool had = !failed && it > 0;
    bool have_o = false;
    if (had) {
      if (wait_warp(o_done(w), 0)) {
        tc::fence_after();
        have_o = true;
      } else {
        failed = true;
      }
    }
    // merge the two streams: (m, l) through shared memory, over Q's bytes (every MMA
    // that reads Q is complete once both warpgroups hold their last PV)
    float* red = reinterpret_cast<float*>(sbase + L::kQ);  // [2][2][128]: m, l per stream
    // with pruning a stream may hold no tile these rows see (O stays 0, m = -inf)
    const bool live = kPruned ? (have_o && m_ref != -INFINITY) : have_o;
    tc::named_bar_sync(1, 256);
    red[(2 * w) * 128 + row] = live ? m_ref : -INFINITY;
    red[(2 * w + 1) * 128 + row] = live ? l : 0.f;
    red[(4 + w) * 128 + row] = live ? 1.f : 0.f;
    tc::named_bar_sync(1, 256);
    const float m_0 = red[0 * 128 + row], l_0 = red[1 * 128 + row];
    const float m_1 = red[2 * 128 + row], l_1 = red[3 * 128 + row];
    const bool has_0 = red[4 * 128 + row] != 0.f, has_1 = red[5 * 128 + row] != 0.f;
    const float m = fmaxf(m_0, m_1);
    const float s_0 = has_0 ? fast_exp2(m_0 - m) : 0.f;
    const float s_1 = has_1 ? fast_exp2(m_1 - m) : 0.f;
    const float l_row = l_0 * s_0 + l_1 * s_1;
    const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
    // warpgroup w writes columns [D/2 w, D/2 w + D/2) of its rows
    const int q = q0 + row;
    int64_t orow_off;
    if (perm_out != nullptr) {
      // O straight into raster layout [B, N, H, D] (the inverse Gilbert permutation
      // fused into the store): permuted row q is token perm_out[q] of head h
      const int b = bh / H, h = bh - b * H;
      const int tok = q < Nq ? __ldg(perm_out + q) : 0;
      orow_off = ((static_cast<int64_t>(b) * Nq + tok) * H + h) * D + (D / 2) * w;
    } else {
      orow_off = (static_cast<int64_t>(bh) * Nq + (q < Nq ? q : 0)) * D + (D / 2) * w;
    }
    __nv_bfloat16* orow = o + orow_off;
    const bool h0 = __all_sync(0xffffffffu, has_0) != 0 || __any_sync(0xffffffffu, has_0) != 0;
    const bool h1 = __any_sync(0xffffffffu, has_1) != 0;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t a0[32], a1[32];
      const uint32_t col = (D / 2) * w + 32u * c;
      if (h0) {
        tc::tmem_ld32_sync(trow + 256u + col, a0);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) a0[k] = 0u;
      }
      if (h1) {
        tc::tmem_ld32_sync(trow + 384u + col, a1);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) a1[k] = 0u;
      }
      const float f0 = s_0 * inv, f1 = s_1 * inv;
      if (q < Nq) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float o0 = has_0 ? __uint_as_float(a0[8 * v + e]) * f0 : 0.f;
            const float o1 = has_1 ? __uint_as_float(a1[8 * v + e]) * f1 : 0.f;
            x[e] = o0 + o1;
          }
          uint4 pk;
          pk.x = pack_bf16(x[0], x[1]);
          pk.y = pack_bf16(x[2], x[3]);
          pk.z = pack_bf16(x[4], x[5]);
          pk.w = pack_bf16(x[6], x[7]);
          *reinterpret_cast<uint4*>(orow + 32 * c + 8 * v) = pk;
          if constexpr (kTrain) {
            float4* o32row = reinterpret_cast<float4*>(o32 + orow_off + 32 * c + 8 * v);
            o32row[0] = make_float4(x[0], x[1], x[2], x[3]);
            o32row[1] = make_float4(x[4], x[5], x[6], x[7]);
          }
        }
      }
    }
    if (q < Nq && w == 0)
      lse[static_cast<int64_t>(bh) * Nq + q] = l_row > 0.f ? (m + __log2f(l_row)) * kLn2 : -INFINITY;
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

// Launch order of the query blocks: heads in order (concurrent CTAs then share one
// head's K and V in L2), and inside each head the query blocks with the most kept
// blocks first, so that the grid ends on short CTAs.  One CTA per head: a counting
// sort of its nrows rows by entry count (bins 0..maxc; a larger count, possible only
// in a malformed CSR, is sorted as maxc).
__global__ void __launch_bounds__(1024) lpt_order_kernel(const int32_t* __restrict__ row_ptr,
                                                        int nrows, int maxc,
                                                        int32_t* __restrict__ order) {
  extern __shared__ int32_t start[];  // maxc + 1 bins
  __shared__ int32_t chunk_tot[1024];
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * nrows;
  auto count = [&](int r) { return min(max(row_ptr[r0 + r + 1] - row_ptr[r0 + r], 0), maxc); };
  for (int c = tid; c <= maxc; c += blockDim.x) start[c] = 0;
  __syncthreads();
  for (int r = tid; r < nrows; r += blockDim.x) atomicAdd(&start[count(r)], 1);
  __syncthreads();
  // exclusive scan over bins in descending count: bin c starts after all bins > c
  const int nbins = maxc + 1;
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int lo = min(nbins, tid * per), hi = min(nbins, lo + per);  // reversed bin index
  int32_t sum = 0;
  for (int k = lo; k < hi; ++k) sum += start[maxc - k];
  chunk_tot[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int32_t run = 0;
    for (int t = 0; t < static_cast<int>(blockDim.x); ++t) {
      const int32_t v = chunk_tot[t];
      chunk_tot[t] = run;
      run += v;
    }
  }
  __syncthreads();
  int32_t run = chunk_tot[tid];
  for (int k = lo; k < hi; ++k) {
    const int32_t v = start[maxc - k];
    start[maxc - k] = run;
    run += v;
  }
  __syncthreads();
  for (int r = tid; r < nrows; r += blockDim.x) order[r0 + atomicAdd(&start[count(r)], 1)] = r0 + r;
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

// [BH][rows][D] 16-bit elements, boxes of 64 columns x 128 rows, 128-byte swizzle,
// zero fill outside the tensor
bool make_map_dtype(CUtensorMap* m, const void* ptr, int BH, int rows, int D,
                    CUtensorMapDataType dtype) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(rows) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dtype, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* ptr, int BH, int rows, int D) {
  return make_map_dtype(m, ptr, BH, rows, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

}  // namespace

bool make_map_rows(CUtensorMap* m, const void* ptr, int BH, int rows, int D) {
  return make_map(m, ptr, BH, rows, D);
}

bool make_map_rows_f16(CUtensorMap* m, const void* ptr, int BH, int rows, int D) {
  return make_map_dtype(m, ptr, BH, rows, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

cudaError_t launch_lpt_order(const int32_t* ptr, int BH, int nrows, int maxc, int32_t* order,
                             cudaStream_t stream) {
  lpt_order_kernel<<<BH, 1024, (maxc + 1) * sizeof(int32_t), stream>>>(ptr, nrows, maxc, order);
  return cudaGetLastError();
}

namespace {

// Nq query rows per head in nb query tiles (N, ceil(N/128) without pruning).
template <int D, int NST, bool kPruned, bool kTrain>
cudaError_t launch_tc(const CUtensorMap* maps, const int32_t* row_ptr, const int32_t* col_idx,
                      const uint8_t* quarters, int32_t* order, int BH, int N, int Nq, int G,
                      float gbias2, void* o, float* lse, float* o32, const int32_t* perm_out,
                      int H, unsigned int* err_word, cudaStream_t stream) {
  using L = FwdTcLayout<D, NST>;
  const int nb = (Nq + kBlock - 1) / kBlock;
  const float c2 = kLog2e / sqrtf(static_cast<float>(D));
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D, NST, kPruned, kTrain>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  // the register split inside the kernel assumes exactly kLaunchRegs per thread at launch
  static int regs_checked = 0;
  if (regs_checked == 0) {
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, fwd_tc_kernel<D, NST, kPruned, kTrain>);
    if (e != cudaSuccess) return e;
    regs_checked = fa.numRegs == kLaunchRegs ? 1 : -1;
  }
  if (regs_checked < 0) return cudaErrorInvalidConfiguration;
  const long long limit = 1ll << 31;  // ~1 s of SM clock per wait
  const int rows = nb * BH;
  // a row holds at most one entry per key block
  e = launch_lpt_order(row_ptr, BH, nb, (N + kBlock - 1) / kBlock, order, stream);
  if (e != cudaSuccess) return e;
  fwd_tc_kernel<D, NST, kPruned, kTrain><<<rows, kFwdTcThreads, L::kSmem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], row_ptr, col_idx, quarters, order, N, Nq, nb,
      G, gbias2, c2, static_cast<__nv_bfloat16*>(o), lse, o32, perm_out, H, err_word, limit);
  return cudaGetLastError();
}

// kTrain: vp and vg are the fp16 copies of V and of the global V tokens.
template <bool kPruned, bool kTrain = false>
cudaError_t launch_fwd_any(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                           const int32_t* col_idx, const uint8_t* quarters, const void* kg,
                           const void* vg, int32_t* order, int BH, int N, int Nq, int d,
                           int global_window, void* o, float* lse, float* o32,
                           unsigned int* err_word, cudaStream_t stream,
                           const int32_t* perm_out = nullptr, int H = 1) {
  const int G = global_window > 0 ? (N + global_window - 1) / global_window : 0;
  const float gbias2 = global_window > 0 ? log2f(static_cast<float>(global_window)) : 0.f;
  const CUtensorMapDataType vtype =
      kTrain ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap maps[5];
  if (!make_map(&maps[0], qp, BH, Nq, d) || !make_map(&maps[1], kp, BH, N, d) ||
      !make_map_dtype(&maps[2], vp, BH, N, d, vtype))
    return cudaErrorInvalidValue;
  if (G > 0) {
    if (!make_map(&maps[3], kg, BH, G, d) || !make_map_dtype(&maps[4], vg, BH, G, d, vtype))
      return cudaErrorInvalidValue;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  if (d == 128)
    return launch_tc<128, 3, kPruned, kTrain>(maps, row_ptr, col_idx, quarters, order, BH, N, Nq,
                                              G, gbias2, o, lse, o32, perm_out, H, err_word,
                                              stream);
  return launch_tc<64, 6, kPruned, kTrain>(maps, row_ptr, col_idx, quarters, order, BH, N, Nq, G,
                                           gbias2, o, lse, o32, perm_out, H, err_word, stream);
}

}  // namespace

cudaError_t launch_fwd_tc(const void* qp, const void* kp, const void* vp, const int32_t* row_ptr,
                          const int32_t* col_idx, const void* kg, const void* vg, int32_t* order,
                          int BH, int N, int d, int global_window, void* o, float* lse,
                          unsigned int* err_word, cudaStream_t stream, const int32_t* perm_out,
                          int H) {
  return launch_fwd_any<false>(qp, kp, vp, row_ptr, col_idx, nullptr, kg, vg, order, BH, N, N, d,
                               global_window, o, lse, nullptr, err_word, stream, perm_out, H);
}

cudaError_t launch_fwd_tc_train(const void* qp, const void* kp, const void* vp16,
                                const int32_t* row_ptr, const int32_t* col_idx, const void* kg,
                                const void* vg16, int32_t* order, int BH, int N, int d,
                                int global_window, void* o, float* lse, float* o32,
                                unsigned int* err_word, cudaStream_t stream) {
  return launch_fwd_any<false, true>(qp, kp, vp16, row_ptr, col_idx, nullptr, kg, vg16, order, BH,
                                     N, N, d, global_window, o, lse, o32, err_word, stream);
}

cudaError_t launch_fwd_tc_pruned(const void* q_s, const void* kp, const void* vp,
                                 const int32_t* tile_ptr, const int32_t* tile_col,
                                 const uint8_t* quarters, const void* kg, const void* vg,
                                 int32_t* order, int BH, int N, int Ns, int d, int global_window,
                                 void* o_s, float* lse_s, unsigned int* err_word,
                                 cudaStream_t stream) {
  return launch_fwd_any<true>(q_s, kp, vp, tile_ptr, tile_col, quarters, kg, vg, order, BH, N, Ns,
                              d, global_window, o_s, lse_s, nullptr, err_word, stream);
}

}  // namespace asa
