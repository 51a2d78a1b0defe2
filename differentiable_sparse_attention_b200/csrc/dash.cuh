// DashAttention stage-0/1 router kernels for sm_100a.
//
// The Italian summary of DashAttention (gist.science/it/paper/2605.18753, which
// the AdaSplash-2 pages carry) routes each query to whole chunks of the
// context: stage 0 summarises every complete chunk of B keys by local attention
// with a learned query qbar (zero at initialisation, where the summary is the
// chunk mean), stage 1 maps the query's logits against the summaries through
// alpha-entmax, w = alpha-entmax(gamma zbar), and under GQA the probabilities of
// the query heads sharing a KV head are averaged ("Stadio 0", "Stadio 1",
// "Gestione GQA").  Query row r routes over the complete chunks before its own,
// c < floor(r / B); zbar = q . kbar / sqrt(D).
//
//   dash_chunk_mean_kernel  kbar = mean of each complete chunk's keys (qbar = 0)
//                           as two fp16 parts, hi + lo (about 22 significant
//                           bits: the logits keep fp32 accuracy though the
//                           tensor cores take fp16), zero rows up to a whole
//                           number of 128-chunk tiles.  HBM-bound: reads k once.
//   dash_route_kernel       one CTA per (batch x KV head, 128 query rows): the
//                           G query heads' logits against all chunk summaries
//                           by tcgen05 into TMEM, the row's threshold by the
//                           same certified Halley / Newton steps as the
//                           attention forward, p / G accumulated in TMEM over
//                           the heads, then wbar, the row mask and the 128-row
//                           block mask.
#pragma once

#include "fwd.cuh"

namespace entmax {

constexpr int kDashMaxChunks = 256;       // logits and accumulator share TMEM's 512 columns
constexpr int kDashWords = kDashMaxChunks / 32;

// kbar[0][bh][c][:] + kbar[1][bh][c][:] = mean of k[bh][c * chunk .. (c + 1) *
// chunk)[:] for c < C (part 0 the fp16 rounding of the mean, part 1 that of the
// remainder), 0 for C <= c < Cp.  One thread per (bh, c, 8 dims).
__global__ void dash_chunk_mean_kernel(const __nv_bfloat16* __restrict__ k,
                                       __half* __restrict__ kbar, int BH, int N, int D,
                                       int chunk, int C, int Cp, uint32_t* status) {
  bounds_init(status);
  const size_t part = static_cast<size_t>(BH) * Cp * D;
  const size_t k_elems = static_cast<size_t>(BH) * N * D;
  const int dv = D / 8;
  const long long total = static_cast<long long>(BH) * Cp * dv;
  const float inv = 1.0f / static_cast<float>(chunk);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int d8 = static_cast<int>(idx % dv);
    const long long bc = idx / dv;
    const int c = static_cast<int>(bc % Cp);
    const int bh = static_cast<int>(bc / Cp);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const size_t src_off = (static_cast<size_t>(bh) * N + static_cast<size_t>(c) * chunk) * D + d8 * 8;
    if (c < C && in_bounds(src_off + static_cast<size_t>(chunk - 1) * D + 8 <= k_elems)) {
      const __nv_bfloat16* src = k + src_off;
      for (int i = 0; i < chunk; ++i) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(i) * D);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ww[h]));
          acc[2 * h] += f.x;
          acc[2 * h + 1] += f.y;
        }
      }
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float m0 = acc[2 * h] * inv, m1 = acc[2 * h + 1] * inv;
      const __half2 o = __floats2half2_rn(m0, m1);
      const float2 of = __half22float2(o);
      const __half2 r = __floats2half2_rn(m0 - of.x, m1 - of.y);
      hi[h] = *reinterpret_cast<const uint32_t*>(&o);
      lo[h] = *reinterpret_cast<const uint32_t*>(&r);
    }
    const size_t at = (static_cast<size_t>(bh) * Cp + c) * D + d8 * 8;
    if (!in_bounds(at + 8 <= part)) continue;
    *reinterpret_cast<uint4*>(kbar + at) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(kbar + part + at) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

struct DashParams {
  int BHkv, G, N, C, Cp, chunk, tr, max_iter;
  float c;            // (alpha - 1) * gamma / sqrt(D): s = c * (q . kbar)
  float kpow;         // 1 / (alpha - 1)
  float am1;          // alpha - 1
  float* wbar;        // [BHkv][N][C]
  uint32_t* row_mask;     // [BHkv][N][W]
  uint32_t* block_mask;   // [BHkv][tr][W]
  int W;
  uint32_t* status;
};

constexpr int kDashThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 one query row each

template <int D>
struct DashSmem {
  __half kbar[2][kDashMaxChunks / kTile][kTile * D];   // [hi, lo][chunk tile]
  __half q[2][kTile * D];
  uint64_t kv_full, q_full[2], q_empty[2], s_full, s_free, drain;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t bmask[kDashWords];
};

template <int D>
constexpr size_t dash_smem_bytes() {
  return sizeof(DashSmem<D>) + 1024;
}

template <int D, int AM>
__global__ void __launch_bounds__(kDashThreads, 1)
    dash_route_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kbar, const DashParams P) {
  constexpr bool ALPHA2 = AM == AM_2;
  constexpr bool GEN = AM == AM_GEN;
  extern __shared__ uint8_t smem_raw[];
  auto& sm = *reinterpret_cast<DashSmem<D>*>(align1024(smem_raw));
  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  constexpr uint32_t kIdesc = make_idesc(kTile, kTile, 0, 0, 0, 0);   // fp16 Q x fp16 kbar, K-major
  constexpr uint32_t kColAcc = 256;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int i = static_cast<int>(blockIdx.x) / P.BHkv;
  const int bh = static_cast<int>(blockIdx.x) % P.BHkv;
  const int nct = P.Cp / kTile;
  bounds_init(P.status);
  const size_t n_rows_all = static_cast<size_t>(P.BHkv) * P.N;   // rows of wbar / row_mask

  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 4);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kDashWords) sm.bmask[threadIdx.x] = 0u;
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kbar);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int qc = 0;   // Q tiles loaded (producer)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&sm.kv_full, 2u * static_cast<uint32_t>(nct) * kTileBytes);
      for (int part = 0; part < 2; ++part)
        for (int ct = 0; ct < nct; ++ct)
          for (int s = 0; s < kSlabs; ++s)
            tma_load_3d(sm.kbar[part][ct] + s * kTile * 64, &tm_kbar, &sm.kv_full, s * 64,
                        ct * kTile, part * P.BHkv + bh);
      for (int g = 0; g < P.G; ++g) {
        const int slot = g & 1;
        if (g >= 2 && !mbar_wait(&sm.q_empty[slot], ((g >> 1) - 1) & 1, abort_flag, P.status)) break;
        mbar_expect_tx(&sm.q_full[slot], kTileBytes);
        for (int s = 0; s < kSlabs; ++s)
          tma_load_3d(sm.q[slot] + s * kTile * 64, &tm_q, &sm.q_full[slot], s * 64, i * kTile,
                      bh * P.G + g);
        ++qc;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // every lane runs the issue loop (warp-uniform descriptors); one elected
    // lane issues each MMA and commit
    {
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full, 0, abort_flag, P.status));
      for (int g = 0; g < P.G && ok; ++g) {
        const int slot = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full[slot], (g >> 1) & 1, abort_flag, P.status));
        // the epilogue must be done with head g - 1's logits
        if (ok && g > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_free, (g - 1) & 1, abort_flag, P.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm.q[slot]);
        for (int ct = 0; ct < nct; ++ct) {
          const uint32_t hi_addr = smem_u32(sm.kbar[0][ct]), lo_addr = smem_u32(sm.kbar[1][ct]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
            const uint64_t qd = smem_desc_sw128(q_addr + off, 16, 1024);
            mma_f16_ss_warp(tmem + ct * kTile, qd, smem_desc_sw128(hi_addr + off, 16, 1024), kIdesc,
                       kk > 0 ? 1u : 0u);
            mma_f16_ss_warp(tmem + ct * kTile, qd, smem_desc_sw128(lo_addr + off, 16, 1024), kIdesc, 1u);
          }
        }
        mma_commit_warp(&sm.s_full);
        mma_commit_warp(&sm.q_empty[slot]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int rl = quad * 32 + lane;
    const int row = i * kTile + rl;
    const bool row_ok = row < P.N;
    const int nvis = row_ok ? min(row / P.chunk, P.C) : 0;     // visible chunks
    const int nch = (__reduce_max_sync(0xffffffffu, nvis) + 31) / 32;   // 32-column loads
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float inv_g = 1.0f / static_cast<float>(P.G);
    bool ok = true;

    // sums over the visible logits at tau_c (s = c * logit, t = s - tau_c)
    auto pass_sums = [&](float tau_c, double& F0, double& F1, double& F2, float& tmin,
                         float& tneg) {
      float f0 = 0.f, f1 = 0.f, f2 = 0.f;
      tmin = INFINITY;
      tneg = -INFINITY;
      for (int ch = 0; ch < nch; ++ch) {
        uint32_t r[32];
        tmem_ld32(t_lane + ch * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const bool vis = ch * 32 + e < nvis;
          const float tt = vis ? fmaf(__uint_as_float(r[e]), P.c, -tau_c) : -INFINITY;
          const bool in = tt > 0.0f;
          tmin = in ? fminf(tmin, tt) : tmin;
          tneg = (vis && !in) ? fmaxf(tneg, tt) : tneg;
          if (GEN) {
            const float pk = pow_pos(tt, P.kpow);
            const float pk1 = in ? __fdividef(pk, tt) : 0.0f;
            f0 += pk;
            f1 += pk1;
            if (P.kpow >= 2.0f) f2 += in ? __fdividef(pk1, tt) : 0.0f;
          } else if (ALPHA2) {
            f0 += in ? tt : 0.0f;
            f1 += in ? 1.0f : 0.0f;
          } else {
            const float tp = in ? tt : 0.0f;
            f0 = fmaf(tp, tp, f0);
            f1 += tp;
            f2 += in ? 1.0f : 0.0f;
          }
        }
      }
      F0 = f0;
      F1 = f1;
      F2 = f2;
    };

    const int ncp = P.Cp / 32;   // 32-column groups of the padded chunk range
    float rowsum = 0.0f;

    for (int g = 0; g < P.G; ++g) {
      ok = mbar_wait(&sm.s_full, g & 1, abort_flag, P.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // the row's maximum and the bracket [m - 1, m - n^(1 - alpha)] of tau
      float m_raw = -INFINITY;
      for (int ch = 0; ch < nch; ++ch) {
        uint32_t r[32];
        tmem_ld32(t_lane + ch * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (ch * 32 + e < nvis) m_raw = fmaxf(m_raw, __uint_as_float(r[e]));
      }
      // Halley / Newton steps from tau = m - 1 until every row of the warp is
      // done: the TMEM loads are warp-wide, so all lanes run every pass (rows
      // already done, or with nothing visible, ignore the sums)
      float tau_c = 0.0f;
      double lo = 0.0, hi = 0.0, dx1 = INFINITY, dx2 = INFINITY;
      bool done = nvis == 0;
      if (nvis > 0) {
        const double m_s = static_cast<double>(m_raw) * P.c;
        const double nb = GEN ? static_cast<double>(exp2f(-P.am1 * __log2f(static_cast<float>(nvis)))) * (1.0 - 1e-5)
                              : (ALPHA2 ? 1.0 / nvis : 1.0 / sqrt(static_cast<double>(nvis)));
        lo = m_s - 1.0 - 1e-6 * fmax(1.0, fabs(m_s));
        hi = m_s - nb + 1e-6 * fmax(1.0, fabs(m_s));
        tau_c = __double2float_rd(lo);
        lo = tau_c;
      }
      for (int it = 0; it < P.max_iter; ++it) {
        if (!__any_sync(0xffffffffu, !done)) break;
        double F0, F1, F2;
        float tmin, tneg;
        pass_sums(tau_c, F0, F1, F2, tmin, tneg);
        if (!done)
          done = GEN ? solver_step_gen(F0, F1, F2, P.kpow, tau_c, lo, hi, dx1, dx2)
                     : solver_step<ALPHA2>(F0, F1, F2, tmin, tneg, -INFINITY, tau_c, lo, hi);
      }
      // p / G into the accumulator (columns kColAcc + c); every lane runs the
      // same loads (the TMEM instructions are warp-wide)
      for (int ch = 0; ch < ncp; ++ch) {
        uint32_t r[32], acc[32];
        tmem_ld32(t_lane + ch * 32, r);
        if (g > 0) {
          tmem_ld32(t_lane + kColAcc + ch * 32, acc);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0u;
        }
        uint32_t w16a[16], w16b[16];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const bool vis = ch * 32 + e < nvis;
          const float tt = vis ? fmaf(__uint_as_float(r[e]), P.c, -tau_c) : 0.0f;
          const float tp = fmaxf(tt, 0.0f);
          const float p = GEN ? pow_pos(tt, P.kpow) : (ALPHA2 ? tp : tp * tp);
          rowsum += p;
          const uint32_t val = __float_as_uint(fmaf(p, inv_g, __uint_as_float(acc[e])));
          if (e < 16) w16a[e] = val;
          else w16b[e - 16] = val;
        }
        tmem_st16(t_lane + kColAcc + ch * 32, w16a);
        tmem_st16(t_lane + kColAcc + ch * 32 + 16, w16b);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free);
    }

    // ---- outputs: wbar, the row mask (support of wbar = union of the heads'
    // supports) and the block mask (OR over the 128 rows)
    if (ok) {
      tc_fence_after();
      const size_t row_idx = static_cast<size_t>(bh) * P.N + row;
      const bool row_in = !row_ok || in_bounds(row_idx < n_rows_all);
      float* wrow = P.wbar + row_idx * P.C;
      uint32_t* mrow = P.row_mask + row_idx * P.W;
      for (int ch = 0; ch < ncp; ++ch) {
        uint32_t acc[32];
        tmem_ld32(t_lane + kColAcc + ch * 32, acc);
        uint32_t bits = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float w = __uint_as_float(acc[e]);
          bits |= (w > 0.0f ? 1u : 0u) << e;
          if (row_ok && row_in && ch * 32 + e < P.C) wrow[ch * 32 + e] = w;
        }
        if (row_ok && row_in && ch < P.W) mrow[ch] = bits;
        const uint32_t wbits = __reduce_or_sync(0xffffffffu, row_ok ? bits : 0u);
        if (lane == 0 && wbits != 0u && in_bounds(ch < kDashWords)) atomicOr(&sm.bmask[ch], wbits);
      }
      // sum of p over the G heads is G within 1e-3 per head
      if (row_ok && nvis > 0 && !(fabsf(rowsum - static_cast<float>(P.G)) <= 1e-3f * P.G))
        atomicOr(P.status, ST_NOT_CONVERGED);
    }
    tc_fence_before();
  }

  __syncthreads();
  if (!sm.abort_flag && threadIdx.x < P.W &&
      in_bounds((static_cast<size_t>(bh) * P.tr + i) * P.W + threadIdx.x <
                static_cast<size_t>(P.BHkv) * P.tr * P.W))
    P.block_mask[(static_cast<size_t>(bh) * P.tr + i) * P.W + threadIdx.x] =
        threadIdx.x < kDashWords ? sm.bmask[threadIdx.x] : 0u;
  if (sm.abort_flag) {
    if (warp == 0 && lane == 0) {
      mbar_wait(&sm.kv_full, 0, nullptr, nullptr);
      for (int s = 0; s < 2; ++s)
        if (qc > s) mbar_wait(&sm.q_full[s], ((qc - 1 - s) >> 1) & 1, nullptr, nullptr);
    }
    if (warp == 1) {
      mma_commit_warp(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace entmax
