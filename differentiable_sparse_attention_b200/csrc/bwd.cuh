// Backward alpha-entmax attention kernels for sm_100a.
//
// The backward visits only the blocks the forward's bit-packed mask marks
// active (AdaSplash-2 zh §2.3, it §2C, ja §2.3: zero blocks are skipped in the
// backward too, and local accumulators replace atomics).  With
// t = [s - tau]_+, p = t^(1/(alpha-1)) and g = p^(2-alpha) (g = t at alpha = 1.5,
// g = 1[t > 0] at alpha = 2):
//     dP = dO V^T,   delta_r = sum_c g dP / sum_c g,   dZ = g (dP - delta)
//     dQ = dZ K / sqrt(D),   dK = dZ^T Q / sqrt(D),   dV = P^T dO
//
//   tile_mask_kernel / tile_mask_t_kernel  block mask -> 128x128 tile mask and its
//                                          transpose (workspace)
//   entmax_bwd_row_kernel   one CTA per 128-row query tile: delta from dO and
//                           the forward's g-weighted means of v, then dQ in one
//                           pass over the active key tiles.
//   entmax_bwd_col_kernel   one CTA per 128-key tile: dK and dV over the active
//                           query tiles, accumulated in TMEM (no atomics).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace entmax {

// ----------------------------------------------------------------- masks
// tm[bh][i][w]: bit (j % 32) of word w = j / 32 is set iff any block of the
// (block)-granularity mask inside 128x128 tile (i, j) is set.
__global__ void tile_mask_kernel(const uint32_t* __restrict__ mask, uint32_t* __restrict__ tm,
                                 int BH, int T, int block, int mask_rows, int mask_words,
                                 uint32_t* status) {
  bounds_init(status);
  const int wt = (T + 31) / 32;
  const long long total = static_cast<long long>(BH) * T * wt;
  const long long mask_total = static_cast<long long>(BH) * mask_rows * mask_words;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(idx % wt);
    const int i = static_cast<int>((idx / wt) % T);
    const int bh = static_cast<int>(idx / (static_cast<long long>(wt) * T));
    const uint32_t* mrow = mask + static_cast<size_t>(bh) * mask_rows * mask_words;
    uint32_t out = 0u;
    if (block == kTile) {
      const size_t mi = static_cast<size_t>(i) * mask_words + w;
      if (in_bounds(w < mask_words && static_cast<long long>(bh) * mask_rows * mask_words +
                                          static_cast<long long>(mi) < mask_total))
        out = mrow[mi];
    } else {  // 64: rows 2i, 2i+1 and key blocks 2j, 2j+1
      for (int a = 0; a < 2; ++a) {
        const int r = 2 * i + a;
        if (r >= mask_rows) continue;
        for (int bit = 0; bit < 32; ++bit) {
          const int j = w * 32 + bit;
          if (j >= T) break;
          const int kb = 2 * j;
          const size_t mi = static_cast<size_t>(r) * mask_words + (kb >> 5);
          if (!in_bounds((kb >> 5) < mask_words && static_cast<long long>(bh) * mask_rows *
                                                          mask_words + static_cast<long long>(mi) <
                                                      mask_total))
            continue;
          const uint32_t two = (mrow[mi] >> (kb & 31)) & 3u;
          if (two) out |= 1u << bit;
        }
      }
    }
    if (in_bounds(idx < total)) tm[idx] = out;
  }
}

// tmt[bh][j][w]: bit (i % 32) of word i / 32 = tm[bh][i] bit j.
__global__ void tile_mask_t_kernel(const uint32_t* __restrict__ tm, uint32_t* __restrict__ tmt,
                                   int BH, int T, uint32_t* status) {
  bounds_init(status);
  const int wt = (T + 31) / 32;
  const long long total = static_cast<long long>(BH) * T * wt;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(idx % wt);
    const int j = static_cast<int>((idx / wt) % T);
    const int bh = static_cast<int>(idx / (static_cast<long long>(wt) * T));
    const uint32_t* base = tm + static_cast<size_t>(bh) * T * wt;
    uint32_t out = 0u;
    for (int bit = 0; bit < 32; ++bit) {
      const int i = w * 32 + bit;
      if (i >= T) break;
      const size_t ti = static_cast<size_t>(i) * wt + (j >> 5);
      if (in_bounds(static_cast<long long>(bh) * T * wt + static_cast<long long>(ti) < total))
        out |= ((base[ti] >> (j & 31)) & 1u) << bit;
    }
    if (in_bounds(idx < total)) tmt[idx] = out;
  }
}

// bf16 -> fp16 copy of the backward's inputs (exact for |x| in [2^-14, 65504]:
// 8 significant bits fit in fp16's 11).  The backward runs its MMAs in fp16 so
// that the rounded operands built on chip (P and dS) keep 11 significant bits
// instead of bf16's 8; |x| > 65504 raises ST_RANGE.
__global__ void to_fp16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                               size_t n8, uint32_t* status) {
  bounds_init(status);
  bool bad = false;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 in = reinterpret_cast<const uint4*>(src)[i];
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
      const float2 f = __bfloat1622float2(b);
      bad |= !(fabsf(f.x) <= 65504.0f) || !(fabsf(f.y) <= 65504.0f);
      const __half2 h = __floats2half2_rn(f.x, f.y);
      o[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(dst)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (bad) atomicOr(status, ST_RANGE);
}

struct BwdParams {
  int BH, N, T, wt;          // T = 128-tiles per side, wt = words per tile-mask row
  int hg;                    // heads per work group (work_item)
  int causal;
  float c;                   // (alpha - 1) / sqrt(D)
  float inv_sqrt_d;
  float kpow;                // k = 1 / (alpha - 1), used by the generic-alpha kernels
  const float* tau;          // [BH][N]
  const uint32_t* tm;        // tile mask rows (row kernel) or transposed rows (column kernel)
  float* delta;              // workspace [BH][N]
  const float* vbar;         // [BH][N][D] g-weighted means of v from the forward
  const __half* dout16;      // [BH][N][D] fp16 copy of dO
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint32_t* status;
  unsigned long long* counters;
};

// Loads the tile list of row `r` of a [BH][T][wt] bit matrix into smem
// (executed by one warp; find-first-set / popcount traversal).
__device__ __forceinline__ int load_tile_list(const uint32_t* rowbits, int wt, uint16_t* tiles) {
  const int lane = threadIdx.x & 31;
  int total = 0;
  for (int base = 0; base < wt; base += 32) {
    const int w = base + lane;
    uint32_t word = (w < wt) ? rowbits[w] : 0u;
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = total + incl - cnt;
    while (word) {
      const int b = __ffs(word) - 1;
      if (in_bounds(pos < kMaxTiles)) tiles[pos] = static_cast<uint16_t>(w * 32 + b);
      ++pos;
      word &= word - 1u;
    }
    total += __shfl_sync(0xffffffffu, incl, 31);
  }
  return in_bounds(total <= kMaxTiles) ? total : 0;
}

// Both backward kernels work in half-tile steps: a 128 x 128 tile is two
// 64-column steps, so the S / dP accumulators fit twice in TMEM (double
// buffering) and the MMAs of one half overlap the epilogue of the other.
// Two epilogue warpgroups (warps 2-5 and 6-9) alternate: warpgroup h owns half
// h of every tile and its TMEM / SMEM buffer.
constexpr int kBwdThreads = 384;   // warp 0 TMA, warps 1, 10 and 11 MMA, warps 2-9 epilogue
constexpr int kAccWarp = 10;       // issues the accumulating MMAs (dQ; dV and dK)
constexpr int kDpWarp = 11;        // issues dP (dP^T); warp 1 issues S (S^T)
constexpr int kHalf = 64;
constexpr int kHalfBytes = kTile * kHalf * 2;   // one [128][64] fp16 slab

__device__ __forceinline__ void bwd_epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// ============================================================ row kernel (delta, dQ)
// delta_r = sum_c g dP / sum_c g with dP = dO V^T is dO_r . vbar_r, the dot of
// the row's output gradient with the forward's g-weighted mean of v: the row
// kernel forms it in its prologue and then runs a single pass over the tiles.
template <int D, int NSK, int NSV>
struct BwdRowSmem {
  __half q[kTile * D];
  __half dout[kTile * D];
  __half k[NSK][kTile * D];
  __half v[NSV][kTile * D];
  float part_delta[2][kTile];        // half-dot products per warpgroup
  uint64_t qdo_full;
  uint64_t k_full[NSK], k_empty[NSK];
  uint64_t v_full[NSV], v_empty[NSV];
  uint64_t s_full[2], s_empty[2], ds_full[2], ds_empty[2], dq_full, drain, drain_acc, drain_dp;
  uint32_t tmem_base;
  int abort_flag;
  int ntiles;
  uint16_t tiles[kMaxTiles];
};

template <int D, int NSK, int NSV>
constexpr size_t bwd_row_smem_bytes() {
  return sizeof(BwdRowSmem<D, NSK, NSV>) + 1024;
}

template <int D, int NSK, int NSV, int AM>
__global__ void __launch_bounds__(kBwdThreads, 1)
    entmax_bwd_row_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams P) {
  static_assert(NSK >= 2, "K(t - 1) stays for its dQ step while S(t) is issued");
  constexpr bool ALPHA2 = AM == AM_2;
  constexpr bool GEN = AM == AM_GEN;
  extern __shared__ uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<BwdRowSmem<D, NSK, NSV>*>(align1024(smem_raw));
  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  constexpr uint32_t kIdescS = make_idesc(kTile, kHalf, 0, 0, 0, 0);  // [128 x D] x [64 x D]^T
  constexpr uint32_t kIdescDQ = make_idesc(kTile, D, 0, 0, 0, 1);     // dS (TMEM) x K half (MN-major)
  // TMEM: buffer b holds S at 128 b, dP at 128 b + 64; the epilogue overwrites
  // S with dS (fp16, 32-key chunk c packed into columns 128 b + 32 c .. + 15)
  constexpr uint32_t kColDQ = 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // head groups that share L2, the longest causal rows first within a group
  const WorkItem wi = work_item(static_cast<int>(blockIdx.x), P.BH, P.T, P.hg);
  const int i = P.T - 1 - wi.r;
  const int bh = wi.bh;
  bounds_init(P.status);
  // elements of a [BH][N] and a [BH][N][D] tensor (bounds-checked build)
  const size_t n_rows_all = static_cast<size_t>(P.BH) * P.N;
  const size_t n_elems_all = n_rows_all * D;

  if (threadIdx.x == 0) {
    mbar_init(&sm.qdo_full, 1);
    for (int s = 0; s < NSK; ++s) { mbar_init(&sm.k_full[s], 1); mbar_init(&sm.k_empty[s], 1); }
    for (int s = 0; s < NSV; ++s) { mbar_init(&sm.v_full[s], 1); mbar_init(&sm.v_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 2);   // the S and the dP issuer each commit once
      mbar_init(&sm.s_empty[b], 4);
      mbar_init(&sm.ds_full[b], 4);
      mbar_init(&sm.ds_empty[b], 1);
    }
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain_acc, 1);
    mbar_init(&sm.drain_dp, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    const int n = load_tile_list(P.tm + (static_cast<size_t>(bh) * P.T + i) * P.wt, P.wt, sm.tiles);
    if (lane == 0) {
      sm.ntiles = n;
      atomicAdd(&P.counters[CNT_ROW_TILES], static_cast<unsigned long long>(n));
    }
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int n = sm.ntiles;
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t kc = 0, vc = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(&sm.qdo_full, 2 * kTileBytes);
      for (int s = 0; s < kSlabs; ++s) {
        tma_load_3d(sm.q + s * kTile * 64, &tm_q, &sm.qdo_full, s * 64, i * kTile, bh);
        tma_load_3d(sm.dout + s * kTile * 64, &tm_do, &sm.qdo_full, s * 64, i * kTile, bh);
      }
      {
        for (int t = 0; t < n && ok; ++t) {
          const int j = in_bounds(sm.tiles[t] < P.T) ? sm.tiles[t] : 0;
          {
            const uint32_t slot = kc % NSK, use = kc / NSK;
            if (use > 0 && !mbar_wait(&sm.k_empty[slot], (use - 1) & 1, abort_flag, P.status)) { ok = false; break; }
            mbar_expect_tx(&sm.k_full[slot], kTileBytes);
            for (int s = 0; s < kSlabs; ++s)
              tma_load_3d(sm.k[slot] + s * kTile * 64, &tm_k, &sm.k_full[slot], s * 64, j * kTile, bh);
            ++kc;
          }
          {
            const uint32_t slot = vc % NSV, use = vc / NSV;
            if (use > 0 && !mbar_wait(&sm.v_empty[slot], (use - 1) & 1, abort_flag, P.status)) { ok = false; break; }
            mbar_expect_tx(&sm.v_full[slot], kTileBytes);
            for (int s = 0; s < kSlabs; ++s)
              tma_load_3d(sm.v[slot] + s * kTile * 64, &tm_v, &sm.v_full[slot], s * 64, j * kTile, bh);
            ++vc;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == kDpWarp) {
    // ---------------------------------------------------------------- S and dP issuers
    // Three warps issue the MMAs: warp 1 S = Q K_h^T, warp kDpWarp dP = dO V_h^T,
    // warp kAccWarp the dQ steps.  A wait in one warp then leaves the others'
    // MMAs running on the tensor pipe, and each waits only for its own operand
    // (K or V).  Every lane runs the issue loop (warp-uniform descriptors); one
    // elected lane issues each MMA and commit.
    {
      const bool is_s = warp == 1;
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.qdo_full, 0, abort_flag, P.status));
      const uint32_t a_addr = is_s ? smem_u32(sm.q) : smem_u32(sm.dout);
      const uint32_t d_col = is_s ? 0u : static_cast<uint32_t>(kHalf);
      uint32_t tcn = 0;   // tiles consumed
      // step u is half h of tile u / 2
      for (uint32_t u = 0; u < 2u * static_cast<uint32_t>(n) && ok; ++u) {
        const uint32_t h = u & 1, use = u >> 1;
        const uint32_t ks = tcn % NSK, vs = tcn % NSV;
        if (h == 0) {
          ok = is_s ? __all_sync(0xffffffffu, mbar_wait(&sm.k_full[ks], (tcn / NSK) & 1, abort_flag, P.status))
                    : __all_sync(0xffffffffu, mbar_wait(&sm.v_full[vs], (tcn / NSV) & 1, abort_flag, P.status));
          if (!ok) break;
        }
        // buffer h is free once its epilogue is done; the S columns also hold the
        // dS that the dQ MMAs of step u - 2 read
        if (use > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_empty[h], (use - 1) & 1, abort_flag, P.status));
          if (ok && is_s) ok = __all_sync(0xffffffffu, mbar_wait(&sm.ds_empty[h], (use - 1) & 1, abort_flag, P.status));
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t b_addr = (is_s ? smem_u32(sm.k[ks]) : smem_u32(sm.v[vs])) + h * (kHalf * 128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
          mma_f16_ss_warp(tmem + 128 * h + d_col, smem_desc_sw128(a_addr + off, 16, 1024),
                     smem_desc_sw128(b_addr + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(&sm.s_full[h]);
        if (h == 1) {
          if (!is_s) mma_commit_warp(&sm.v_empty[vs]);
          ++tcn;
        }
      }
    }
    __syncwarp();
  } else if (warp == kAccWarp) {
    // ---------------------------------------------------------------- dQ issuer
    // dQ += dS_h K_h for step u, once the epilogue has written dS_h (ds_full).
    // K of tile t sits in slot t % NSK: the S issuer consumed it in that order,
    // and it stays until this warp's k_empty commit after the tile's second half.
    {
      bool ok = true;
      for (uint32_t u = 0; u < 2u * static_cast<uint32_t>(n) && ok; ++u) {
        const uint32_t h = u & 1, use = u >> 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.ds_full[h], use & 1, abort_flag, P.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t ks = use % NSK;
        const uint32_t k_addr = smem_u32(sm.k[ks]) + h * (kHalf * 128);
#pragma unroll
        for (int kk = 0; kk < kHalf / 16; ++kk) {
          const uint32_t a_col = 128 * h + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_f16_ts_warp(tmem + kColDQ, tmem + a_col,
                     smem_desc_sw128(k_addr + kk * 16 * 128, kSlabBytes, 1024), kIdescDQ,
                     (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_warp(&sm.ds_empty[h]);
        if (h == 1) mma_commit_warp(&sm.k_empty[ks]);
      }
      if (ok) mma_commit_warp(&sm.dq_full);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int wg = (warp - 2) >> 2;        // warpgroup: owns half wg of every tile
    const int quad = warp & 3;
    const int rl = quad * 32 + lane;
    const int row = i * kTile + rl;
    const bool row_ok = row < P.N;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + 128 * wg, t_dp = t_s + kHalf;
    const size_t row_idx = static_cast<size_t>(bh) * P.N + row;
    const float tau_r =
        row_ok && in_bounds(row_idx < n_rows_all) ? P.tau[row_idx] : INFINITY;
    bool ok = true;
    uint32_t use = 0;   // uses of this warpgroup's S/dP buffer

    // delta of the row: warpgroup wg takes dimensions [wg D/2, (wg + 1) D/2)
    {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (row_ok && in_bounds(row_idx * D + (wg + 1) * (D / 2) <= n_elems_all)) {
        const size_t off = (static_cast<size_t>(bh) * P.N + row) * D + wg * (D / 2);
        const uint4* dsrc = reinterpret_cast<const uint4*>(P.dout16 + off);
        const float4* vsrc = reinterpret_cast<const float4*>(P.vbar + off);
#pragma unroll
        for (int u = 0; u < D / 16; ++u) {
          const uint4 hv = dsrc[u];
          const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 vb = vsrc[2 * u + h];
            const float2 d0 = __half22float2(*reinterpret_cast<const __half2*>(&hw[2 * h]));
            const float2 d1 = __half22float2(*reinterpret_cast<const __half2*>(&hw[2 * h + 1]));
            acc[2 * h] = fmaf(d0.x, vb.x, fmaf(d0.y, vb.y, acc[2 * h]));
            acc[2 * h + 1] = fmaf(d1.x, vb.z, fmaf(d1.y, vb.w, acc[2 * h + 1]));
          }
        }
      }
      sm.part_delta[wg][rl] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      bwd_epi_bar();
    }
    const float delta = sm.part_delta[0][rl] + sm.part_delta[1][rl];
    if (row_ok && wg == 0 && in_bounds(row_idx < n_rows_all)) P.delta[row_idx] = delta;

    for (int t = 0; t < n; ++t) {
      const int j = in_bounds(sm.tiles[t] < P.T) ? sm.tiles[t] : 0;
      ok = mbar_wait(&sm.s_full[wg], use & 1, abort_flag, P.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++use;
      tc_fence_after();
      const int col0 = j * kTile + wg * kHalf;
      const bool msk = (P.causal && j == i) || (col0 + kHalf > P.N);
      // dS of one 32-key chunk; MASKED (diagonal and tail tiles only) drops the
      // keys at or beyond `nv` -- a tile-uniform choice, so the common path
      // carries no per-key test
      auto chunk_ds = [&](auto masked_tag, const int ch, const uint32_t (&rs)[32],
                          const uint32_t (&rp)[32], uint32_t (&w)[16]) {
        constexpr bool MASKED = decltype(masked_tag)::value;
        int nv = 32;
        if constexpr (MASKED)
          nv = min(32, max(0, (P.causal ? min(row + 1, P.N) : P.N) - (col0 + ch * 32)));
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float g2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float tt = fmaf(__uint_as_float(rs[2 * e + u]), P.c, -tau_r);
            if constexpr (MASKED) tt = (2 * e + u < nv) ? tt : -1.0f;
            if (GEN)   // g = t^(k - 1) <= 1 (alpha <= 2: k >= 1, t <= 1)
              g2[u] = tt > 0.f ? __fdividef(pow_pos(tt, P.kpow), tt) : 0.f;
            else
              g2[u] = ALPHA2 ? (tt > 0.f ? 1.f : 0.f) : fmaxf(tt, 0.f);
          }
          const float d0 = g2[0] * (__uint_as_float(rp[2 * e]) - delta);
          const float d1 = g2[1] * (__uint_as_float(rp[2 * e + 1]) - delta);
          const __half2 h2 = __floats2half2_rn(d0, d1);
          w[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
      };
      // chunk 1's loads are in flight while chunk 0 is computed and stored
      {
        uint32_t rs[2][32], rp[2][32], w[16];
        tmem_ld32x2(t_s, rs[0], t_dp, rp[0]);
        tmem_ld32x2_async(t_s + 32, rs[1], t_dp + 32, rp[1]);
        if (msk) chunk_ds(std::true_type{}, 0, rs[0], rp[0], w);
        else chunk_ds(std::false_type{}, 0, rs[0], rp[0], w);
        tmem_st16(t_s, w);             // dS over the S chunk just read
        tmem_wait_ld_x2(rs[1], rp[1]);
        if (msk) chunk_ds(std::true_type{}, 1, rs[1], rp[1], w);
        else chunk_ds(std::false_type{}, 1, rs[1], rp[1], w);
        tmem_st16(t_s + 32, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.ds_full[wg]);
        mbar_arrive(&sm.s_empty[wg]);
      }
    }
    // dQ epilogue: warpgroup wg stores columns [wg * D/2, (wg + 1) * D/2)
    if (ok && n > 0) {
      ok = mbar_wait(&sm.dq_full, 0, abort_flag, P.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    __nv_bfloat16* dst_row = P.dq + row_idx * D;
#pragma unroll 1
    for (int ch = wg * (D / 64); ch < (wg + 1) * (D / 64); ++ch) {
      uint32_t r[32];
      if (ok && n > 0) {
        tmem_ld32(t_lane + kColDQ + ch * 32, r);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      if (row_ok && in_bounds(row_idx * D + ch * 32 + 32 <= n_elems_all)) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 h2 =
              __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * P.inv_sqrt_d,
                                    __uint_as_float(r[2 * e + 1]) * P.inv_sqrt_d);
          w[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint4* dst = reinterpret_cast<uint4*>(dst_row + ch * 32);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
          dst[qd] = make_uint4(w[4 * qd], w[4 * qd + 1], w[4 * qd + 2], w[4 * qd + 3]);
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (sm.abort_flag) {
    if (warp == 0 && lane == 0) {
      mbar_wait(&sm.qdo_full, 0, nullptr, nullptr);
      for (uint32_t s = 0; s < NSK; ++s)
        if (kc > s) mbar_wait(&sm.k_full[s], ((kc - 1 - s) / NSK) & 1, nullptr, nullptr);
      for (uint32_t s = 0; s < NSV; ++s)
        if (vc > s) mbar_wait(&sm.v_full[s], ((vc - 1 - s) / NSV) & 1, nullptr, nullptr);
    }
    if (warp == 1) {
      mma_commit_warp(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, nullptr);
    }
    if (warp == kAccWarp) {
      mma_commit_warp(&sm.drain_acc);
      mbar_wait(&sm.drain_acc, 0, nullptr, nullptr);
    }
    if (warp == kDpWarp) {
      mma_commit_warp(&sm.drain_dp);
      mbar_wait(&sm.drain_dp, 0, nullptr, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================ column kernel (dK, dV)
template <int D, int NS>
struct BwdColSmem {
  __half k[kTile * D];
  __half v[kTile * D];
  __half q[NS][kTile * D];
  __half dout[NS][kTile * D];
  float tau[NS][kTile];
  float delta[NS][kTile];
  uint64_t kv_full;
  uint64_t q_full[NS], q_empty[NS];
  uint64_t s_full[2], s_empty[2], pt_full[2], pt_empty[2], acc_full, drain, drain_acc, drain_dp;
  uint32_t tmem_base;
  int abort_flag;
  int ntiles;
  uint16_t tiles[kMaxTiles];
};

template <int D, int NS>
constexpr size_t bwd_col_smem_bytes() {
  return sizeof(BwdColSmem<D, NS>) + 1024;
}

template <int D, int NS, int AM>
__global__ void __launch_bounds__(kBwdThreads, 1)
    entmax_bwd_col_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams P) {
  constexpr bool ALPHA2 = AM == AM_2;
  constexpr bool GEN = AM == AM_GEN;
  extern __shared__ uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<BwdColSmem<D, NS>*>(align1024(smem_raw));
  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  constexpr uint32_t kIdescS = make_idesc(kTile, kHalf, 0, 0, 0, 0);   // K Q_h^T, V dO_h^T
  constexpr uint32_t kIdescAcc = make_idesc(kTile, D, 0, 0, 0, 1);    // P^T_h dO_h, dS^T_h Q_h
  // TMEM buffer b: S^T at 128 b, dP^T at 128 b + 64; the epilogue overwrites
  // them with P^T and dS^T (fp16, 32-row chunk c packed into columns 32 c .. + 15).
  // dS^T is kept as two fp16 parts, hi = fp16(dS) and lo = fp16(dS - hi), the
  // lo part in columns 32 c + 16 .. + 31 of the dP^T region: dK sums dS over
  // every row that sees the key (up to N), and one fp16 rounding per term
  // (relative 2^-11) accumulated that far exceeds the output tolerance where
  // the terms cancel; hi + lo carry about 22 bits.
  constexpr uint32_t kColDV = 256, kColDK = 256 + D;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // head groups that share L2; causal: key tile j is seen by T - j row tiles,
  // so small j first within a group
  const WorkItem wi = work_item(static_cast<int>(blockIdx.x), P.BH, P.T, P.hg);
  const int j = wi.r;
  const int bh = wi.bh;
  bounds_init(P.status);
  const size_t n_rows_all = static_cast<size_t>(P.BH) * P.N;
  const size_t n_elems_all = n_rows_all * D;

  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.q_full[s], 1 + 32);  // TMA expect_tx + 32 lanes staging tau/delta
      mbar_init(&sm.q_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 2);   // the S^T and the dP^T issuer each commit once
      mbar_init(&sm.s_empty[b], 4);
      mbar_init(&sm.pt_full[b], 4);
      mbar_init(&sm.pt_empty[b], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain_acc, 1);
    mbar_init(&sm.drain_dp, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    const int n = load_tile_list(P.tm + (static_cast<size_t>(bh) * P.T + j) * P.wt, P.wt, sm.tiles);
    if (lane == 0) {
      sm.ntiles = n;
      atomicAdd(&P.counters[CNT_COL_TILES], static_cast<unsigned long long>(n));
    }
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int n = sm.ntiles;
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t qc = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    bool ok = true;
    if (lane == 0) {
      mbar_expect_tx(&sm.kv_full, 2 * kTileBytes);
      for (int s = 0; s < kSlabs; ++s) {
        tma_load_3d(sm.k + s * kTile * 64, &tm_k, &sm.kv_full, s * 64, j * kTile, bh);
        tma_load_3d(sm.v + s * kTile * 64, &tm_v, &sm.kv_full, s * 64, j * kTile, bh);
      }
    }
    for (int t = 0; t < n && ok; ++t) {
      const int it = in_bounds(sm.tiles[t] < P.T) ? sm.tiles[t] : 0;
      const uint32_t slot = qc % NS, use = qc / NS;
      if (use > 0) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&sm.q_empty[slot], (use - 1) & 1, abort_flag, P.status);
        ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
        __syncwarp();
        if (!ok) break;
      }
      if (lane == 0) {
        mbar_expect_tx(&sm.q_full[slot], 2 * kTileBytes);
        for (int s = 0; s < kSlabs; ++s) {
          tma_load_3d(sm.q[slot] + s * kTile * 64, &tm_q, &sm.q_full[slot], s * 64, it * kTile, bh);
          tma_load_3d(sm.dout[slot] + s * kTile * 64, &tm_do, &sm.q_full[slot], s * 64, it * kTile, bh);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = lane * 4 + e;
        const int row = it * kTile + r;
        const size_t g = static_cast<size_t>(bh) * P.N + row;
        const bool g_ok = row < P.N && in_bounds(g < n_rows_all);
        sm.tau[slot][r] = g_ok ? P.tau[g] : INFINITY;
        sm.delta[slot][r] = g_ok ? P.delta[g] : 0.0f;
      }
      mbar_arrive(&sm.q_full[slot]);
      ++qc;
    }
    __syncwarp();
  } else if (warp == 1 || warp == kDpWarp) {
    // ---------------------------------------------------------------- S^T and dP^T issuers
    // Three warps issue the MMAs: warp 1 S^T = K Q_h^T, warp kDpWarp
    // dP^T = V dO_h^T, warp kAccWarp the dV / dK accumulation.  A wait in one
    // warp then leaves the others' MMAs running on the tensor pipe.  Every lane
    // runs the issue loop (warp-uniform descriptors); one elected lane issues
    // each MMA and commit.
    {
      const bool is_s = warp == 1;
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full, 0, abort_flag, P.status));
      const uint32_t a_addr = is_s ? smem_u32(sm.k) : smem_u32(sm.v);
      const uint32_t d_col = is_s ? 0u : static_cast<uint32_t>(kHalf);
      // step u = 2 t + h: half h (query rows 64 h .. 64 h + 63) of active query tile t
      for (uint32_t u = 0; u < 2u * static_cast<uint32_t>(n) && ok; ++u) {
        const uint32_t t = u >> 1, h = u & 1, slot = t % NS, use = u >> 1;
        if (h == 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full[slot], (t / NS) & 1, abort_flag, P.status));
          if (!ok) break;
        }
        // buffer h is free once its epilogue is done and dV / dK read P^T / dS^T
        if (use > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_empty[h], (use - 1) & 1, abort_flag, P.status));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sm.pt_empty[h], (use - 1) & 1, abort_flag, P.status));
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t b_addr = (is_s ? smem_u32(sm.q[slot]) : smem_u32(sm.dout[slot])) + h * (kHalf * 128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
          mma_f16_ss_warp(tmem + 128 * h + d_col, smem_desc_sw128(a_addr + off, 16, 1024),
                     smem_desc_sw128(b_addr + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(&sm.s_full[h]);
      }
    }
    __syncwarp();
  } else if (warp == kAccWarp) {
    // ---------------------------------------------------------------- dV / dK issuer
    // dV += P^T_h dO_h and dK += dS^T_h Q_h (dS^T as two fp16 parts) for step u,
    // once the epilogue has written P^T and dS^T (pt_full); the Q / dO slot of
    // tile t is released after its second half.
    {
      bool ok = true;
      for (uint32_t u = 0; u < 2u * static_cast<uint32_t>(n) && ok; ++u) {
        const uint32_t t = u >> 1, h = u & 1, slot = t % NS, use = u >> 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.pt_full[h], use & 1, abort_flag, P.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm.q[slot]) + h * (kHalf * 128);
        const uint32_t do_addr = smem_u32(sm.dout[slot]) + h * (kHalf * 128);
#pragma unroll
        for (int kk = 0; kk < kHalf / 16; ++kk) {
          const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
          const uint32_t a_col = 128 * h + (kk >> 1) * 32 + (kk & 1) * 8;
          mma_f16_ts_warp(tmem + kColDV, tmem + a_col,
                     smem_desc_sw128(do_addr + kk * 16 * 128, kSlabBytes, 1024), kIdescAcc, acc);
          const uint64_t qd = smem_desc_sw128(q_addr + kk * 16 * 128, kSlabBytes, 1024);
          mma_f16_ts_warp(tmem + kColDK, tmem + a_col + kHalf, qd, kIdescAcc, acc);        // hi
          mma_f16_ts_warp(tmem + kColDK, tmem + a_col + kHalf + 16, qd, kIdescAcc, 1u);   // lo
        }
        mma_commit_warp(&sm.pt_empty[h]);
        if (h == 1) mma_commit_warp(&sm.q_empty[slot]);
      }
      if (ok) mma_commit_warp(&sm.acc_full);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int wg = (warp - 2) >> 2;           // warpgroup: owns half wg of every tile
    const int quad = warp & 3;
    const int kl = quad * 32 + lane;          // key within the tile
    const int key = j * kTile + kl;
    const bool key_ok = key < P.N;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + 128 * wg, t_dp = t_s + kHalf;
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      const int it = in_bounds(sm.tiles[t] < P.T) ? sm.tiles[t] : 0;
      const uint32_t slot = t % NS;
      ok = mbar_wait(&sm.s_full[wg], t & 1, abort_flag, P.status) &&
           mbar_wait(&sm.q_full[slot], (t / NS) & 1, abort_flag, P.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row0 = it * kTile + wg * kHalf;
      const bool msk = (P.causal && it == j) || (row0 + kHalf > P.N) || !key_ok;
      // P^T and dS^T of one 32-row chunk; MASKED (diagonal and tail tiles only)
      // keeps rows in [lo_v, hi_v) of the chunk -- a tile-uniform choice
      auto chunk_pds = [&](auto masked_tag, const int ch, const uint32_t (&rs)[32],
                           const uint32_t (&rp)[32], uint32_t (&wp)[16], uint32_t (&wd)[16],
                           uint32_t (&wl)[16]) {
        constexpr bool MASKED = decltype(masked_tag)::value;
        int lo_v = 0, hi_v = 32;
        if constexpr (MASKED) {
          const int r0 = row0 + ch * 32;
          lo_v = P.causal ? max(0, key - r0) : 0;
          hi_v = key_ok ? min(32, max(0, P.N - r0)) : 0;
        }
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int r4 = wg * kHalf + ch * 32 + e;
          const float4 tv = *reinterpret_cast<const float4*>(&sm.tau[slot][r4]);
          const float4 dv = *reinterpret_cast<const float4*>(&sm.delta[slot][r4]);
          const float taus[4] = {tv.x, tv.y, tv.z, tv.w};
          const float dels[4] = {dv.x, dv.y, dv.z, dv.w};
          float pp[4], dd[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float tt = fmaf(__uint_as_float(rs[e + u]), P.c, -taus[u]);
            if constexpr (MASKED) tt = (e + u >= lo_v && e + u < hi_v) ? tt : -1.0f;
            const float tp = fmaxf(tt, 0.0f);
            float g;
            if (GEN) {
              pp[u] = pow_pos(tt, P.kpow);
              g = tt > 0.f ? __fdividef(pp[u], tt) : 0.f;
            } else {
              g = ALPHA2 ? (tt > 0.f ? 1.f : 0.f) : tp;
              pp[u] = ALPHA2 ? tp : tp * tp;
            }
            dd[u] = g * (__uint_as_float(rp[e + u]) - dels[u]);
          }
          __half2 a0 = __floats2half2_rn(pp[0], pp[1]);
          __half2 a1 = __floats2half2_rn(pp[2], pp[3]);
          __half2 b0 = __floats2half2_rn(dd[0], dd[1]);
          __half2 b1 = __floats2half2_rn(dd[2], dd[3]);
          const float2 f0 = __half22float2(b0), f1 = __half22float2(b1);
          __half2 c0 = __floats2half2_rn(dd[0] - f0.x, dd[1] - f0.y);
          __half2 c1 = __floats2half2_rn(dd[2] - f1.x, dd[3] - f1.y);
          wp[e / 2] = *reinterpret_cast<uint32_t*>(&a0);
          wp[e / 2 + 1] = *reinterpret_cast<uint32_t*>(&a1);
          wd[e / 2] = *reinterpret_cast<uint32_t*>(&b0);
          wd[e / 2 + 1] = *reinterpret_cast<uint32_t*>(&b1);
          wl[e / 2] = *reinterpret_cast<uint32_t*>(&c0);
          wl[e / 2 + 1] = *reinterpret_cast<uint32_t*>(&c1);
        }
      };
      // chunk 1's loads are in flight while chunk 0 is computed and stored
      {
        uint32_t rs[2][32], rp[2][32], wp[16], wd[16], wl[16];
        tmem_ld32x2(t_s, rs[0], t_dp, rp[0]);
        tmem_ld32x2_async(t_s + 32, rs[1], t_dp + 32, rp[1]);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          if (ch == 1) tmem_wait_ld_x2(rs[1], rp[1]);
          if (msk) chunk_pds(std::true_type{}, ch, rs[ch], rp[ch], wp, wd, wl);
          else chunk_pds(std::false_type{}, ch, rs[ch], rp[ch], wp, wd, wl);
          tmem_st16(t_s + ch * 32, wp);         // P^T over the S^T chunk just read
          tmem_st16(t_dp + ch * 32, wd);        // dS^T (hi) over the dP^T chunk
          tmem_st16(t_dp + ch * 32 + 16, wl);   // dS^T (lo) beside it
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.pt_full[wg]);
        mbar_arrive(&sm.s_empty[wg]);
      }
    }
    if (ok && n > 0) {
      ok = mbar_wait(&sm.acc_full, 0, abort_flag, P.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    // warpgroup 0 stores dV, warpgroup 1 stores dK
    const uint32_t col = wg == 0 ? kColDV : kColDK;
    const float scale = wg == 0 ? 1.0f : P.inv_sqrt_d;
    const size_t key_idx = static_cast<size_t>(bh) * P.N + key;
    __nv_bfloat16* dst_row = (wg == 0 ? P.dv : P.dk) + key_idx * D;
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t r[32];
      if (ok && n > 0) {
        tmem_ld32(t_lane + col + ch * 32, r);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      if (key_ok && in_bounds(key_idx * D + ch * 32 + 32 <= n_elems_all)) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * scale,
                                                          __uint_as_float(r[2 * e + 1]) * scale);
          w[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint4* dst = reinterpret_cast<uint4*>(dst_row + ch * 32);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
          dst[qd] = make_uint4(w[4 * qd], w[4 * qd + 1], w[4 * qd + 2], w[4 * qd + 3]);
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (sm.abort_flag) {
    if (warp == 0 && lane == 0) {
      mbar_wait(&sm.kv_full, 0, nullptr, nullptr);
      for (uint32_t s = 0; s < NS; ++s)
        if (qc > s) mbar_wait(&sm.q_full[s], ((qc - 1 - s) / NS) & 1, nullptr, nullptr);
    }
    if (warp == 1) {
      mma_commit_warp(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, nullptr);
    }
    if (warp == kAccWarp) {
      mma_commit_warp(&sm.drain_acc);
      mbar_wait(&sm.drain_acc, 0, nullptr, nullptr);
    }
    if (warp == kDpWarp) {
      mma_commit_warp(&sm.drain_dp);
      mbar_wait(&sm.drain_dp, 0, nullptr, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace entmax
