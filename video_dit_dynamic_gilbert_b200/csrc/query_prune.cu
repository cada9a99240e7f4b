// Query pruning with token filling ("Bidirectional Sparse Attention for Faster Video
// Diffusion Training", "Key designs", item 1), on ASA's blocks of 128 permuted tokens.
//
// A block is cut into windows of w consecutive tokens; the token in the middle of
// each window (offset len/2) is its centre.  The block keeps every centre and the
// other tokens with the largest 1 - cos(q_centre, q_i), K = max(ceil(r L), windows)
// in all (ties to the lower position).  Kept queries are packed into a compact
// buffer of 128-row tiles holding `pack` blocks each (slots of 128/pack rows, a
// block's kept rows in position order, the rest of its slot zero), so that one
// tcgen05 tile computes the kept rows of `pack` blocks at once.  The attention of a
// tile runs over the union of its blocks' kept key blocks, and each key block of the
// union carries a bit per 32-row TMEM lane quarter telling which rows may see it.
// A pruned token then takes its centre's output row and LSE (token filling).
//
// Kernels: prune_kernel (selection and packing), pack_count/pack_fill (tile CSR with
// quarter bits), fill_out_kernel (token filling of O and LSE); for the packed
// backward, dout_compact_kernel (each kept row's summed output gradient and lse2 in
// the compact layout), tile_dense/tile_transpose (the tile CSR per key block) and
// dq_scatter_kernel (dQ back to every token, zero for pruned ones).
#include "common.cuh"
#include "internal.h"

namespace asa {

namespace {

constexpr float kCosEps = 1e-8f;
constexpr int kPackThreads = 256;  // 8 warps, one tile each
constexpr int kMaxWords = kMaxBlocksHost / 32;

template <int E>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float* x) {
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    x[0] = __uint_as_float(u << 16);
    x[1] = __uint_as_float(u & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kPruneThreads = 256;
constexpr int kPruneWarps = kPruneThreads / 32;

// One CTA per (b, h, block I), two threads per token.  The block's queries are staged
// in shared memory (every load in flight before the stores); 16-byte piece c of row t
// is stored at piece c ^ (t mod kVec), so that the threads of a warp, each reading its
// own row, spread over all banks.  Thread pair (2t, 2t + 1) computes token t's dot
// products over one half of d each and ranks it against one half of the block.
template <int D>
__global__ void __launch_bounds__(kPruneThreads)
    prune_kernel(const __nv_bfloat16* __restrict__ qp, int N, int nb, float r, int w, int pack,
                 __nv_bfloat16* __restrict__ q_s, int Ns, int32_t* __restrict__ src_pos,
                 int32_t* __restrict__ src_row) {
  constexpr int kVec = D / 8;  // 16-byte pieces per row
  __shared__ uint4 s_q[kBlock * kVec];
  __shared__ float s_dis[kBlock];
  __shared__ int s_slot[kBlock];
  __shared__ int s_tok[kBlock];
  __shared__ int s_wtot[kPruneWarps];
  const int bh = blockIdx.x / nb, I = blockIdx.x % nb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s0 = I * kBlock;
  const int L = min(kBlock, N - s0);
  const __nv_bfloat16* qb = qp + (static_cast<int64_t>(bh) * N + s0) * D;
  auto piece = [](int row, int c) { return row * kVec + (c ^ (row & (kVec - 1))); };
  {
    constexpr int kPer = kBlock * kVec / kPruneThreads;
    const uint4* src = reinterpret_cast<const uint4*>(qb);
    uint4 v[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kPruneThreads;
      if (i < L * kVec) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kPruneThreads;
      if (i < L * kVec) s_q[piece(i / kVec, i % kVec)] = v[u];
    }
  }
  __syncthreads();
  auto centre = [&](int t) {
    const int ws = (t / w) * w;
    return ws + min(w, L - ws) / 2;
  };

  // 1 - cos(q_centre, q_t) in fp32; centres are kept unconditionally: -inf keeps them
  // out of the ranking
  const int t = tid >> 1, half = tid & 1;
  {
    float dot = 0.f, na = 0.f, nc = 0.f;
    const int c = t < L ? centre(t) : 0;
    if (t < L && c != t) {
#pragma unroll
      for (int j = 0; j < kVec / 2; ++j) {
        const int pc = half * (kVec / 2) + j;
        const uint4 a4 = s_q[piece(t, pc)], b4 = s_q[piece(c, pc)];
        const uint32_t av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a0 = __uint_as_float(av[e] << 16), a1 = __uint_as_float(av[e] & 0xffff0000u);
          const float b0 = __uint_as_float(bv[e] << 16), b1 = __uint_as_float(bv[e] & 0xffff0000u);
          dot = fmaf(a0, b0, fmaf(a1, b1, dot));
          na = fmaf(a0, a0, fmaf(a1, a1, na));
          nc = fmaf(b0, b0, fmaf(b1, b1, nc));
        }
      }
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    na += __shfl_xor_sync(0xffffffffu, na, 1);
    nc += __shfl_xor_sync(0xffffffffu, nc, 1);
    if (t < L && half == 0) {
      const float den = fmaxf(sqrtf(na), kCosEps) * fmaxf(sqrtf(nc), kCosEps);
      s_dis[t] = c == t ? -INFINITY : 1.f - dot / den;
    }
  }
  __syncthreads();

  // rank of each non-centre: tokens more dissimilar, or as dissimilar and earlier;
  // each thread of the pair counts over one half of the block
  const int windows = (L + w - 1) / w;
  const int K = max(static_cast<int>(ceil(static_cast<double>(r) * L)), windows);
  const int extra = K - windows;
  bool kept = false;
  {
    const float dt = t < L ? s_dis[t] : -INFINITY;
    int rank = 0;
    if (t < L && dt != -INFINITY && extra > 0) {
      const int u0 = half * (kBlock / 2), u1 = min(L, u0 + kBlock / 2);
      for (int u = u0; u < u1; ++u) {
        const float du = s_dis[u];
        rank += (du > dt) | ((du == dt) & (u < t));
      }
    }
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    kept = t < L && (dt == -INFINITY || (extra > 0 && rank < extra));
  }
  // compact slots in position order (one vote per token: the even thread)
  const unsigned bal = __ballot_sync(0xffffffffu, kept && half == 0);
  if (lane == 0) s_wtot[warp] = __popc(bal);
  __syncthreads();
  int base = 0, nkept = 0;
#pragma unroll
  for (int k = 0; k < kPruneWarps; ++k) {
    base += k < warp ? s_wtot[k] : 0;
    nkept += s_wtot[k];
  }
  const int slot = base + __popc(bal & ((1u << lane) - 1u));
  if (half == 0) {
    s_slot[t] = kept ? slot : -1;
    if (kept) s_tok[slot] = t;
  }
  __syncthreads();

  const int S = kBlock / pack;
  const int tile = I / pack, sub = I % pack;
  const int row0 = tile * kBlock + sub * S;  // first compact row of this block
  if (tid < L) {
    const bool kt = s_slot[tid] >= 0;
    const int c = kt ? tid : centre(tid);
    const int64_t g = static_cast<int64_t>(bh) * N + s0 + tid;
    src_pos[g] = s0 + c;
    src_row[g] = row0 + s_slot[c];
  }
  // kept rows into their slots, zeros after them; the last block also zeroes the
  // slots of its tile that no block owns.  16-byte pieces, kVec per row.
  const int zero_end = (I == nb - 1) ? (tile + 1) * kBlock - row0 : S;
  uint4* qs = reinterpret_cast<uint4*>(q_s + (static_cast<int64_t>(bh) * Ns + row0) * D);
  for (int i = tid; i < zero_end * kVec; i += kPruneThreads) {
    const int sl = i / kVec, v = i - sl * kVec;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (sl < nkept && sl < S) x = s_q[piece(s_tok[sl], v)];
    qs[i] = x;
  }
}

// Kept key blocks of the tile's blocks as bitmaps in shared memory, one per slot.
// Returns false if a column index is out of range (it is skipped).
__device__ __forceinline__ bool tile_bitmaps(const int32_t* __restrict__ row_ptr,
                                             const int32_t* __restrict__ col_idx, int r0,
                                             int nsub, int nb, int words, uint32_t* bits,
                                             int lane) {
  for (int k = lane; k < 4 * words; k += 32) bits[k] = 0u;
  __syncwarp();
  bool ok = true;
  for (int s = 0; s < nsub; ++s) {
    const int e0 = row_ptr[r0 + s], e1 = row_ptr[r0 + s + 1];
    for (int e = e0 + lane; e < e1; e += 32) {
      const int J = col_idx[e];
      if (J < 0 || J >= nb) {
        ok = false;
        continue;
      }
      atomicOr(&bits[s * words + (J >> 5)], 1u << (J & 31));
    }
  }
  __syncwarp();
  return ok;
}

__device__ __forceinline__ uint8_t slot_quarters(int s, int pack) {
  const int q = 4 / pack;
  return static_cast<uint8_t>(((1u << q) - 1u) << (s * q));
}

// counts[bh * ntile + t] = number of key blocks kept by any block of tile t
__global__ void __launch_bounds__(kPackThreads)
    pack_count_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                      int BH, int nb, int pack, int32_t* __restrict__ counts,
                      unsigned int* __restrict__ err_word) {
  __shared__ uint32_t sbits[kPackThreads / 32][4 * kMaxWords];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int ntile = (nb + pack - 1) / pack;
  const int words = (nb + 31) / 32;
  uint32_t* bits = sbits[wib];
  for (int idx = blockIdx.x * (kPackThreads / 32) + wib; idx < BH * ntile;
       idx += gridDim.x * (kPackThreads / 32)) {
    const int bh = idx / ntile, t = idx % ntile;
    const int nsub = min(pack, nb - t * pack);
    const bool ok = tile_bitmaps(row_ptr, col_idx, bh * nb + t * pack, nsub, nb, words, bits, lane);
    if (__any_sync(0xffffffffu, !ok) && lane == 0) atomicOr(err_word, kErrBadIndex);
    int c = 0;
    for (int k = lane; k < words; k += 32) {
      uint32_t u = 0;
      for (int s = 0; s < nsub; ++s) u |= bits[s * words + k];
      c += __popc(u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) counts[idx] = c;
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kPackThreads)
    pack_fill_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                     int BH, int nb, int pack, const int32_t* __restrict__ tile_ptr,
                     int32_t* __restrict__ tile_col, uint8_t* __restrict__ tile_quarters) {
  __shared__ uint32_t sbits[kPackThreads / 32][4 * kMaxWords];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int ntile = (nb + pack - 1) / pack;
  const int words = (nb + 31) / 32;
  uint32_t* bits = sbits[wib];
  for (int idx = blockIdx.x * (kPackThreads / 32) + wib; idx < BH * ntile;
       idx += gridDim.x * (kPackThreads / 32)) {
    const int bh = idx / ntile, t = idx % ntile;
    const int nsub = min(pack, nb - t * pack);
    tile_bitmaps(row_ptr, col_idx, bh * nb + t * pack, nsub, nb, words, bits, lane);
    int pos = tile_ptr[idx];
    for (int k0 = 0; k0 < words; k0 += 32) {
      const int k = k0 + lane;
      uint32_t u = 0;
      if (k < words)
        for (int s = 0; s < nsub; ++s) u |= bits[s * words + k];
      const int c = __popc(u);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int p = pos + incl - c;
      while (u != 0u) {
        const int b = __ffs(u) - 1;
        u &= u - 1u;
        uint8_t q = 0;
        for (int s = 0; s < nsub; ++s)
          if ((bits[s * words + k] >> b) & 1u) q |= slot_quarters(s, pack);
        tile_col[p] = k * 32 + b;
        tile_quarters[p] = q;
        ++p;
      }
      pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
  }
}

// O[bh, i] = O_s[bh, src_row[i]], LSE likewise: D/8 threads per row, 16 bytes each
template <int D>
__global__ void __launch_bounds__(256)
    fill_out_kernel(const __nv_bfloat16* __restrict__ o_s, const float* __restrict__ lse_s,
                    const int32_t* __restrict__ src_row, int64_t rows, int N, int Ns,
                    __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                    unsigned int* __restrict__ err_word) {
  constexpr int kVec = D / 8;
  const int64_t total = rows * kVec;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = g / kVec;
    const int v = static_cast<int>(g - row * kVec);
    const int64_t bh = row / N;
    const int sr = src_row[row];
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    float l = -INFINITY;
    if (sr >= 0 && sr < Ns) {
      const int64_t srow = bh * Ns + sr;
      x = reinterpret_cast<const uint4*>(o_s + srow * D)[v];
      l = lse_s[srow];
    } else if (v == 0) {
      atomicOr(err_word, kErrBadIndex);
    }
    reinterpret_cast<uint4*>(o + row * D)[v] = x;
    if (v == 0) lse[row] = l;
  }
}

// Backward inputs in the compact layout: for a kept token i (src_pos[i] = i) with
// compact row r = src_row[i], dO'_s[r] = the sum of dO[j] over the tokens j of i's
// block with src_pos[j] = i (its own gradient and those of the pruned tokens it
// fills), stored in bf16, and lse2_s[r] = lse[i] log2(e).  One CTA per (b, h, block):
// the block's src_pos and dO rows are staged in shared memory (every load in flight
// before the stores; every token is checked to point at a kept token of its own
// block); each warp then takes kept tokens, finds their contributors with four
// ballots and sums their rows from shared memory.
template <int D>
__global__ void __launch_bounds__(256)
    dout_compact_kernel(const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                        const int32_t* __restrict__ src_pos, const int32_t* __restrict__ src_row,
                        int N, int nb, int Ns, __nv_bfloat16* __restrict__ dout_s,
                        float* __restrict__ lse2_s, unsigned int* __restrict__ err_word) {
  constexpr int E = D / 32;
  constexpr int kVec = D / 8;  // 16-byte pieces per row
  __shared__ __align__(16) __nv_bfloat16 s_do[kBlock * D];
  __shared__ int s_sp[kBlock];
  const int bh = blockIdx.x / nb, I = blockIdx.x % nb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s0 = I * kBlock;
  const int L = min(kBlock, N - s0);
  const int64_t g0 = static_cast<int64_t>(bh) * N + s0;  // first token of the block
  {
    constexpr int kPer = kBlock * kVec / 256;
    const uint4* src = reinterpret_cast<const uint4*>(dout + g0 * D);
    uint4* dst = reinterpret_cast<uint4*>(s_do);
    uint4 v[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * 256;
      if (i < L * kVec) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * 256;
      if (i < L * kVec) dst[i] = v[u];
    }
  }
  if (tid < L) s_sp[tid] = src_pos[g0 + tid] - s0;       // block-relative source
  __syncthreads();
  if (tid < L) {
    const int p = s_sp[tid];
    if (p < 0 || p >= L || s_sp[p] != p) atomicOr(err_word, kErrBadIndex);
  }
  for (int t = warp; t < L; t += 8) {
    if (s_sp[t] != t) continue;  // pruned: its gradient goes to its source
    const int r = src_row[g0 + t];
    if (r < 0 || r >= Ns) {
      if (lane == 0) atomicOr(err_word, kErrBadIndex);
      continue;
    }
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int j0 = 0; j0 < kBlock; j0 += 32) {
      const int j = j0 + lane;
      unsigned m = __ballot_sync(0xffffffffu, j < L && s_sp[j] == t);
      while (m != 0u) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        float x[E];
        load_bf16<E>(s_do + (j0 + b) * D + lane * E, x);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += x[e];
      }
    }
    __nv_bfloat16* dst = dout_s + (static_cast<int64_t>(bh) * Ns + r) * D + lane * E;
    if constexpr (E == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0], acc[1]);
    }
    if (lane == 0) lse2_s[static_cast<int64_t>(bh) * Ns + r] = lse[g0 + t] * kLog2e;
  }
}

// dQ[i] = dQ_s[src_row[i]] for a kept token, 0 for a pruned one (its output is a copy
// of its centre's, so its query gets no gradient).  D/8 threads per row.
template <int D>
__global__ void __launch_bounds__(256)
    dq_scatter_kernel(const __nv_bfloat16* __restrict__ dq_s, const int32_t* __restrict__ src_pos,
                      const int32_t* __restrict__ src_row, int64_t rows, int N, int Ns,
                      __nv_bfloat16* __restrict__ dq, unsigned int* __restrict__ err_word) {
  constexpr int kVec = D / 8;
  const int64_t total = rows * kVec;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = g / kVec;
    const int v = static_cast<int>(g - row * kVec);
    const int64_t bh = row / N;
    const int i = static_cast<int>(row - bh * N);
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (src_pos[row] == i) {
      const int r = src_row[row];
      if (r >= 0 && r < Ns)
        x = reinterpret_cast<const uint4*>(dq_s + (bh * Ns + r) * D)[v];
      else if (v == 0)
        atomicOr(err_word, kErrBadIndex);
    }
    reinterpret_cast<uint4*>(dq + row * D)[v] = x;
  }
}

// Dense quarter matrix [BH][ntile][nbk] (zeroed by the caller) from the tile CSR:
// one warp per tile row.
__global__ void __launch_bounds__(256)
    tile_dense_kernel(const int32_t* __restrict__ tile_ptr, const int32_t* __restrict__ tile_col,
                      const uint8_t* __restrict__ tile_quarters, int rows, int nbk,
                      uint8_t* __restrict__ qmat, unsigned int* __restrict__ err_word) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    bool bad = false;
    for (int e = tile_ptr[r] + lane; e < tile_ptr[r + 1]; e += 32) {
      const int J = tile_col[e];
      if (J < 0 || J >= nbk) {
        bad = true;
        continue;
      }
      qmat[static_cast<int64_t>(r) * nbk + J] = tile_quarters[e];
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(err_word, kErrBadIndex);
  }
}

// Transposed tile CSR from the dense matrix: for each (bh, key block J) the tiles t
// holding J, t ascending, with their quarter bits.  One warp per (bh, J), lanes over t.
template <bool kFill>
__global__ void __launch_bounds__(256)
    tile_transpose_kernel(const uint8_t* __restrict__ qmat, int BH, int ntile, int nbk,
                          int32_t* __restrict__ counts, const int32_t* __restrict__ tcol_ptr,
                          int32_t* __restrict__ trow_idx, uint8_t* __restrict__ tquarters) {
  const int lane = threadIdx.x & 31;
  const int64_t cols = static_cast<int64_t>(BH) * nbk;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       c < cols; c += warps) {
    const int64_t bh = c / nbk;
    const int J = static_cast<int>(c - bh * nbk);
    int pos = kFill ? tcol_ptr[c] : 0;
    for (int t0 = 0; t0 < ntile; t0 += 32) {
      const int t = t0 + lane;
      const uint8_t q = t < ntile ? qmat[(bh * ntile + t) * nbk + J] : 0;
      const unsigned m = __ballot_sync(0xffffffffu, q != 0);
      if (kFill && q != 0) {
        const int p = pos + __popc(m & ((1u << lane) - 1u));
        trow_idx[p] = t;
        tquarters[p] = q;
      }
      pos += __popc(m);
    }
    if (!kFill && lane == 0) counts[c] = pos;
  }
}

unsigned grid_of(int64_t work, int per_block, int num_sms, int per_sm) {
  int64_t b = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

}  // namespace

cudaError_t launch_prune(const void* qp, int BH, int N, int d, float r, int w, int pack, void* q_s,
                         int Ns, int32_t* src_pos, int32_t* src_row, cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  const auto* q = static_cast<const __nv_bfloat16*>(qp);
  auto* qs = static_cast<__nv_bfloat16*>(q_s);
  if (d == 128)
    prune_kernel<128><<<BH * nb, kPruneThreads, 0, stream>>>(q, N, nb, r, w, pack, qs, Ns, src_pos,
                                                              src_row);
  else
    prune_kernel<64><<<BH * nb, kPruneThreads, 0, stream>>>(q, N, nb, r, w, pack, qs, Ns, src_pos,
                                                             src_row);
  return cudaGetLastError();
}

cudaError_t launch_prune_mask(const int32_t* row_ptr, const int32_t* col_idx, int BH, int nb,
                              int pack, int32_t* counts, int32_t* tile_ptr, int32_t* tile_col,
                              uint8_t* tile_quarters, int32_t* nnz_out, unsigned int* err_word,
                              int num_sms, cudaStream_t stream) {
  const int ntile = (nb + pack - 1) / pack;
  const int64_t tiles = static_cast<int64_t>(BH) * ntile;
  const unsigned grid = grid_of(tiles, kPackThreads / 32, num_sms, 8);
  pack_count_kernel<<<grid, kPackThreads, 0, stream>>>(row_ptr, col_idx, BH, nb, pack, counts,
                                                        err_word);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_scan(counts, static_cast<int>(tiles), tile_ptr, nnz_out, stream);
  if (e != cudaSuccess) return e;
  pack_fill_kernel<<<grid, kPackThreads, 0, stream>>>(row_ptr, col_idx, BH, nb, pack, tile_ptr,
                                                       tile_col, tile_quarters);
  return cudaGetLastError();
}

cudaError_t launch_fill_out(const void* o_s, const float* lse_s, const int32_t* src_row, int BH,
                            int N, int Ns, int d, void* o, float* lse, unsigned int* err_word,
                            int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(BH) * N;
  const unsigned grid = grid_of(rows * (d / 8), 256, num_sms, 8);
  const auto* src = static_cast<const __nv_bfloat16*>(o_s);
  auto* dst = static_cast<__nv_bfloat16*>(o);
  if (d == 128)
    fill_out_kernel<128><<<grid, 256, 0, stream>>>(src, lse_s, src_row, rows, N, Ns, dst, lse, err_word);
  else
    fill_out_kernel<64><<<grid, 256, 0, stream>>>(src, lse_s, src_row, rows, N, Ns, dst, lse, err_word);
  return cudaGetLastError();
}

cudaError_t launch_dout_compact(const void* dout, const float* lse, const int32_t* src_pos,
                                const int32_t* src_row, int BH, int N, int Ns, int d,
                                void* dout_s, float* lse2_s, unsigned int* err_word, int num_sms,
                                cudaStream_t stream) {
  const int nb = (N + kBlock - 1) / kBlock;
  const auto* src = static_cast<const __nv_bfloat16*>(dout);
  auto* dst = static_cast<__nv_bfloat16*>(dout_s);
  if (d == 128)
    dout_compact_kernel<128><<<BH * nb, 256, 0, stream>>>(src, lse, src_pos, src_row, N, nb, Ns,
                                                          dst, lse2_s, err_word);
  else
    dout_compact_kernel<64><<<BH * nb, 256, 0, stream>>>(src, lse, src_pos, src_row, N, nb, Ns,
                                                         dst, lse2_s, err_word);
  (void)num_sms;
  return cudaGetLastError();
}

cudaError_t launch_dq_scatter(const void* dq_s, const int32_t* src_pos, const int32_t* src_row,
                              int BH, int N, int Ns, int d, void* dq, unsigned int* err_word,
                              int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(BH) * N;
  const unsigned grid = grid_of(rows * (d / 8), 256, num_sms, 8);
  const auto* src = static_cast<const __nv_bfloat16*>(dq_s);
  auto* dst = static_cast<__nv_bfloat16*>(dq);
  if (d == 128)
    dq_scatter_kernel<128><<<grid, 256, 0, stream>>>(src, src_pos, src_row, rows, N, Ns, dst, err_word);
  else
    dq_scatter_kernel<64><<<grid, 256, 0, stream>>>(src, src_pos, src_row, rows, N, Ns, dst, err_word);
  return cudaGetLastError();
}

cudaError_t launch_tile_transpose(const int32_t* tile_ptr, const int32_t* tile_col,
                                  const uint8_t* tile_quarters, int BH, int ntile, int nbk,
                                  uint8_t* qmat, int32_t* counts, int32_t* tcol_ptr,
                                  int32_t* trow_idx, uint8_t* tquarters, unsigned int* err_word,
                                  int num_sms, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(BH) * ntile;
  cudaError_t e = cudaMemsetAsync(qmat, 0, static_cast<size_t>(rows) * nbk, stream);
  if (e != cudaSuccess) return e;
  tile_dense_kernel<<<grid_of(rows, 8, num_sms, 8), 256, 0, stream>>>(
      tile_ptr, tile_col, tile_quarters, static_cast<int>(rows), nbk, qmat, err_word);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t cols = static_cast<int64_t>(BH) * nbk;
  const unsigned grid = grid_of(cols, 8, num_sms, 8);
  tile_transpose_kernel<false><<<grid, 256, 0, stream>>>(qmat, BH, ntile, nbk, counts, nullptr,
                                                         nullptr, nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_scan(counts, static_cast<int>(cols), tcol_ptr, nullptr, stream)) != cudaSuccess)
    return e;
  tile_transpose_kernel<true><<<grid, 256, 0, stream>>>(qmat, BH, ntile, nbk, nullptr, tcol_ptr,
                                                        trow_idx, tquarters);
  return cudaGetLastError();
}

}  // namespace asa
