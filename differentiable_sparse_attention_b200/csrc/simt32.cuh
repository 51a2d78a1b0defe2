// fp32 alpha-entmax attention on the CUDA cores (FFMA), head dim 64.
//
// The fp32 path exists for precision: a single TF32 tensor-core product keeps
// ~10 bits and cannot reach a 1e-5 error on O, and the split-TF32 P tiles of
// the tensor-core design do not fit in shared memory.  The per-row algorithm is
// the one of the bf16 kernels (AdaSplash-2 zh §2.1-2.3): a streaming 8-bin
// histogram and candidate list, tau_h, the safeguarded Halley / Newton
// refinement with its exactness certificate (shared hist_threshold and
// solver_step), the bit-packed block mask, and a backward that skips the blocks
// the mask marks empty.  Key and query tiles of 32 rows are staged in shared
// memory and every dot product runs in fp32.
//
//   entmax_fwd_f32_kernel      one thread per query row, 128 rows per CTA
//   entmax_bwd_row_f32_kernel  two threads per query row (32 dims each): delta, dQ
//   entmax_bwd_col_f32_kernel  two threads per key (32 dims each): dK, dV
#pragma once

#include "fwd.cuh"

namespace entmax {

constexpr int kF32D = 64;       // supported head dim
constexpr int kF32Keys = 32;    // rows of a staged K / V / Q / dO tile
constexpr int kF32Cap = 96;     // candidate slots per query row
constexpr int kF32Pad = 68;     // padded smem row (floats): 16-byte aligned rows
constexpr size_t kF32CandBytes = kF32Cap * 128 * sizeof(float);  // dynamic smem of the forward

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  const float* dout;
  float* out;
  float* tau;                 // forward: written; backward: read
  uint32_t* mask;             // forward: written; backward: read
  float* tau_trace;
  float* delta;               // workspace [BH][N]
  float* dq;
  float* dk;
  float* dv;
  int BH, N, causal, block, mask_rows, mask_words, max_iter;
  float c, cN, slim, inv_c, inv_sqrt_d;
  uint32_t* status;
  unsigned long long* counters;
};

// Stage `rows` consecutive 64-float rows starting at row r0 of one head into
// smem (zeros past N).  128 threads, float4 loads.
__device__ __forceinline__ void f32_stage(const float* __restrict__ head, int r0, int n,
                                          float (*dst)[kF32Pad]) {
  for (int idx = threadIdx.x; idx < kF32Keys * (kF32D / 4); idx += blockDim.x) {
    const int rr = idx / (kF32D / 4);
    const int cc = (idx % (kF32D / 4)) * 4;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + rr < n) val = *reinterpret_cast<const float4*>(head + static_cast<size_t>(r0 + rr) * kF32D + cc);
    *reinterpret_cast<float4*>(&dst[rr][cc]) = val;
  }
}

// dot of a register vector with a staged smem row (all threads read the same
// row: a broadcast), 4 partial sums.
template <int LEN>
__device__ __forceinline__ float f32_dot(const float (&a)[LEN], const float* b) {
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int d = 0; d < LEN; d += 4) {
    const float4 bv = *reinterpret_cast<const float4*>(b + d);
    s[0] = fmaf(a[d], bv.x, s[0]);
    s[1] = fmaf(a[d + 1], bv.y, s[1]);
    s[2] = fmaf(a[d + 2], bv.z, s[2]);
    s[3] = fmaf(a[d + 3], bv.w, s[3]);
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// ------------------------------------------------------------------ forward
template <bool ALPHA2>
__global__ void __launch_bounds__(128) entmax_fwd_f32_kernel(const F32Params P) {
  __shared__ __align__(16) float sk[kF32Keys][kF32Pad];
  __shared__ __align__(16) float sv[kF32Keys][kF32Pad];
  extern __shared__ float cand_dyn[];   // [kF32Cap][128]: slot-major, conflict free
  auto cand = [&](int a) -> float& { return cand_dyn[a * 128 + threadIdx.x]; };
  __shared__ uint32_t maskw[2][kMaxMaskWords];
  __shared__ int any_collect, any_tile;

  const int tid = threadIdx.x;
  const int i = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y;
  const int row = i * 128 + tid;
  const bool row_ok = row < P.N;
  bounds_init(P.status);
  const size_t n_rows_all = static_cast<size_t>(P.BH) * P.N;
  const float* qh = P.q + static_cast<size_t>(bh) * P.N * kF32D;
  const float* kh = P.k + static_cast<size_t>(bh) * P.N * kF32D;
  const float* vh = P.v + static_cast<size_t>(bh) * P.N * kF32D;
  const int kend = P.causal ? min(P.N, (i + 1) * 128) : P.N;
  const int n_valid = P.causal ? min(row + 1, P.N) : P.N;

  for (int w = tid; w < 2 * kMaxMaskWords; w += 128) (&maskw[0][0])[w] = 0u;
  if (tid == 0) {
    any_collect = 0;
    any_tile = 0;
  }
  float qr[kF32D];
#pragma unroll
  for (int d = 0; d < kF32D; d += 4) {
    const float4 x = row_ok ? *reinterpret_cast<const float4*>(qh + static_cast<size_t>(row) * kF32D + d)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    qr[d] = x.x;
    qr[d + 1] = x.y;
    qr[d + 2] = x.z;
    qr[d + 3] = x.w;
  }
  auto trace_store = [&](int it, float val) {
    if (P.tau_trace != nullptr && row_ok && it <= P.max_iter &&
        in_bounds((static_cast<size_t>(it) * P.BH + bh) * P.N + row <
                  static_cast<size_t>(P.max_iter + 1) * n_rows_all))
      P.tau_trace[(static_cast<size_t>(it) * P.BH + bh) * P.N + row] = val;
  };
  // raw scores q.k of keys key0 .. key0+31 (-inf where not visible)
  auto scores = [&](int key0, float (&v)[32]) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int key = key0 + e;
      const bool ok = row_ok && key < P.N && (!P.causal || key <= row);
      v[e] = ok ? f32_dot<kF32D>(qr, &sk[e][0]) : -INFINITY;
    }
  };

  // ---------------- pass 1: running max, histogram, candidates
  float m_raw = -INFINITY;
  int gtop = 0;
  bool gtop_set = false;
  uint32_t cnt[kNB + 1];
#pragma unroll
  for (int b = 0; b <= kNB; ++b) cnt[b] = 0u;
  float vclamp = -P.slim;
  uint32_t cbase = 0u;
  int ncand = 0, prunes = 0;
  float acc_raw = -INFINITY;
  bool cand_over = false;
  for (int key0 = 0; key0 < kend; key0 += kF32Keys) {
    __syncthreads();
    f32_stage(kh, key0, P.N, sk);
    __syncthreads();
    float v[32];
    scores(key0, v);
    const float cm = max32(v);
    m_raw = fmaxf(m_raw, cm);
    if (cm > -INFINITY) {
      const int gc = static_cast<int>(
          __float_as_uint(__fmaf_rd(fmaxf(cm, -P.slim), P.cN, kMagic)) - kMagicBits);
      if (!gtop_set || gc > gtop) {
        const int delta = gtop_set ? gc - gtop : kNB + 1;
        if (delta > kNB) {
#pragma unroll
          for (int b = 0; b <= kNB; ++b) cnt[b] = 0u;
        } else {
          for (int d = 0; d < delta; ++d) {
#pragma unroll
            for (int b = 0; b < kNB; ++b) cnt[b] = cnt[b + 1];
            cnt[kNB] = 0u;
          }
        }
        gtop = gc;
        gtop_set = true;
        vclamp = (static_cast<float>(gtop - kNB) - 1.5f) / P.cN;
        cbase = 0u - 7u * (kMagicBits + static_cast<uint32_t>(gtop - kNB));
      }
      if (cm > vclamp) {   // a chunk entirely below the window adds nothing
        uint64_t pk[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float u = __fmaf_rd(fmaxf(v[e], vclamp), P.cN, kMagic);
          pk[e & 3] += shl64(1ull, __float_as_uint(u) * 7u + cbase);
        }
        const uint64_t packed = (pk[0] + pk[1]) + (pk[2] + pk[3]);
#pragma unroll
        for (int b = 0; b <= kNB; ++b) cnt[b] += static_cast<uint32_t>(packed >> (7 * b)) & 127u;
      }
      acc_raw = fmaxf(acc_raw, __fsub_rd(m_raw, P.inv_c));
      if (row_ok && !cand_over && cm > acc_raw) {
        const double th = hist_threshold<ALPHA2>(cnt, gtop);
        acc_raw = fmaxf(acc_raw, __double2float_rd((th - hist_margin(th)) / P.c));
        if (ncand + 32 > kF32Cap) {
          if (prunes < kMaxPrunes) {
            ++prunes;
            int kept = 0;
            for (int a = 0; a < ncand; ++a)
              if (cand(a) > acc_raw) cand(kept++) = cand(a);
            ncand = kept;
          }
          cand_over = ncand + 32 > kF32Cap;
        }
        if (!cand_over) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (v[e] > acc_raw) cand(ncand++) = v[e];
        }
      }
    }
  }

  // ---------------- tau_h and the bracket
  double lo = 0.0, hi = 0.0, l_drop = -INFINITY, tau_h = 0.0;
  float tau_c = 0.0f;
  bool collect = false, row_done = false;
  int iter = 0;
  if (row_ok) {
    if (fabsf(m_raw * P.cN) >= 2097152.0f) atomicOr(P.status, ST_RANGE);
    tau_h = hist_threshold<ALPHA2>(cnt, gtop);
    const double margin = hist_margin(tau_h);
    const double m_s = static_cast<double>(m_raw) * P.c;
    const double nb = ALPHA2 ? 1.0 / n_valid : 1.0 / sqrt(static_cast<double>(n_valid));
    lo = tau_h - margin;
    hi = fmin(tau_h + 1.0 / kNB + margin, m_s - nb + margin);
    l_drop = static_cast<double>(acc_raw) * P.c;
    lo = fmax(lo, l_drop);
    if (hi < lo) hi = lo;
    tau_c = __double2float_rd(lo);
    lo = tau_c;
    if (cand_over && P.max_iter > 0) {
      collect = true;
      cand_over = false;
      ncand = 0;
      l_drop = lo;
      atomicOr(&any_collect, 1);
    }
  }
  trace_store(0, static_cast<float>(tau_h));
  __syncthreads();
  if (any_collect) {
    // rebuild the overflowed lists: exactly the scores above lo
    const float thr = collect ? __double2float_rd(lo / P.c) : INFINITY;
    for (int key0 = 0; key0 < kend; key0 += kF32Keys) {
      __syncthreads();
      f32_stage(kh, key0, P.N, sk);
      __syncthreads();
      if (!collect) continue;
      float v[32];
      scores(key0, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        if (v[e] > thr) {
          if (ncand < kF32Cap) cand(ncand) = v[e];
          ++ncand;
        }
      }
    }
    if (collect && ncand > kF32Cap) {
      cand_over = true;
      atomicOr(&any_tile, 1);
    }
    if (threadIdx.x == 0) atomicAdd(&P.counters[CNT_CAND_OVERFLOW], 1ull);
  }
  // refinement over the candidate list, in registers
  if (row_ok && !cand_over) {
    for (; iter < P.max_iter && !row_done;) {
      double F0 = 0.0, F1 = 0.0, F2 = 0.0;
      float tmin = INFINITY, tneg = -INFINITY;
      for (int a = 0; a < ncand; ++a) {
        const float tt = fmaf(cand(a), P.c, -tau_c);
        const bool in = tt > 0.0f;
        const float tp = fmaxf(tt, 0.0f);
        tmin = in ? fminf(tmin, tt) : tmin;
        tneg = in ? tneg : fmaxf(tneg, tt);
        if (ALPHA2) {
          F0 += tp;
          F1 += in ? 1.0 : 0.0;
        } else {
          F0 += static_cast<double>(tp) * tp;
          F1 += tp;
          F2 += in ? 1.0 : 0.0;
        }
      }
      row_done = solver_step<ALPHA2>(F0, F1, F2, tmin, tneg, l_drop, tau_c, lo, hi);
      ++iter;
      trace_store(iter, tau_c);
    }
  }
  __syncthreads();
  if (any_tile) {
    // rows whose candidates overflow refine by streaming the keys again
    for (int pass = 0; pass < P.max_iter; ++pass) {
      double F0 = 0.0, F1 = 0.0, F2 = 0.0;
      float tmin = INFINITY, tneg = -INFINITY;
      for (int key0 = 0; key0 < kend; key0 += kF32Keys) {
        __syncthreads();
        f32_stage(kh, key0, P.N, sk);
        __syncthreads();
        if (!(row_ok && cand_over && !row_done)) continue;
        float v[32];
        scores(key0, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float tt = fmaf(v[e], P.c, -tau_c);
          const bool in = tt > 0.0f;
          const float tp = fmaxf(tt, 0.0f);
          tmin = in ? fminf(tmin, tt) : tmin;
          tneg = in ? tneg : fmaxf(tneg, tt);
          if (ALPHA2) {
            F0 += tp;
            F1 += in ? 1.0 : 0.0;
          } else {
            F0 += static_cast<double>(tp) * tp;
            F1 += tp;
            F2 += in ? 1.0 : 0.0;
          }
        }
      }
      if (row_ok && cand_over && !row_done && iter < P.max_iter) {
        row_done = solver_step<ALPHA2>(F0, F1, F2, tmin, tneg, l_drop, tau_c, lo, hi);
        ++iter;
        trace_store(iter, tau_c);
      }
    }
  }
  for (int it = iter + 1; it <= P.max_iter; ++it) trace_store(it, tau_c);

  // ---------------- P.V pass, block mask
  float o[kF32D];
#pragma unroll
  for (int d = 0; d < kF32D; ++d) o[d] = 0.0f;
  float rowsum = 0.0f;
  const int spr = 128 / P.block;
  for (int key0 = 0; key0 < kend; key0 += kF32Keys) {
    __syncthreads();
    f32_stage(kh, key0, P.N, sk);
    f32_stage(vh, key0, P.N, sv);
    __syncthreads();
    float v[32];
    scores(key0, v);
    float csum = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float t = fmaxf(fmaf(v[e], P.c, -tau_c), 0.0f);
      const float p = ALPHA2 ? t : t * t;
      if (p > 0.0f) {
        csum += p;
#pragma unroll
        for (int d = 0; d < kF32D; d += 4) {
          const float4 vv = *reinterpret_cast<const float4*>(&sv[e][d]);
          o[d] = fmaf(p, vv.x, o[d]);
          o[d + 1] = fmaf(p, vv.y, o[d + 1]);
          o[d + 2] = fmaf(p, vv.z, o[d + 2]);
          o[d + 3] = fmaf(p, vv.w, o[d + 3]);
        }
      }
    }
    rowsum += csum;
    if (row_ok && csum > 0.0f) {   // a 32-key chunk lies inside one 64- or 128-key block
      const int kb = key0 / P.block;
      const int h = (row / P.block) - i * spr;
      atomicOr(&maskw[h][kb >> 5], 1u << (kb & 31));
    }
  }
  if (row_ok && in_bounds(static_cast<size_t>(bh) * P.N + row < n_rows_all)) {
    float* orow = P.out + (static_cast<size_t>(bh) * P.N + row) * kF32D;
#pragma unroll
    for (int d = 0; d < kF32D; d += 4)
      *reinterpret_cast<float4*>(orow + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
    P.tau[static_cast<size_t>(bh) * P.N + row] = tau_c;
    if (!(fabsf(rowsum - 1.0f) <= 1e-3f)) atomicOr(P.status, ST_NOT_CONVERGED);
  }
  __syncthreads();
  for (int idx = tid; idx < spr * P.mask_words; idx += 128) {
    const int h = idx / P.mask_words;
    const int w = idx - h * P.mask_words;
    const int mrow = i * spr + h;
    if (mrow < P.mask_rows &&
        in_bounds(h < 2 && w < kMaxMaskWords &&
                  (static_cast<size_t>(bh) * P.mask_rows + mrow) * P.mask_words + w <
                      static_cast<size_t>(P.BH) * P.mask_rows * P.mask_words))
      P.mask[(static_cast<size_t>(bh) * P.mask_rows + mrow) * P.mask_words + w] = maskw[h][w];
  }
}

// Is (row block of query r0, key block of key c0) active in the forward mask?
__device__ __forceinline__ bool f32_block_active(const F32Params& P, int bh, int r0, int c0) {
  const int mr = r0 / P.block, kb = c0 / P.block;
  return (P.mask[(static_cast<size_t>(bh) * P.mask_rows + mr) * P.mask_words + (kb >> 5)] >>
          (kb & 31)) & 1u;
}

// ------------------------------------------------------------------ backward rows
// 64 query rows per CTA, two threads per row (lane pairs), 32 dims each.
template <bool ALPHA2>
__global__ void __launch_bounds__(128) entmax_bwd_row_f32_kernel(const F32Params P) {
  __shared__ __align__(16) float sk[kF32Keys][kF32Pad];
  __shared__ __align__(16) float sv[kF32Keys][kF32Pad];
  const int tid = threadIdx.x;
  const int half = tid & 1;
  const int rb = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y;
  const int row = rb * 64 + (tid >> 1);
  bounds_init(P.status);
  const bool row_ok = row < P.N && in_bounds(static_cast<size_t>(bh) * P.N + row <
                                             static_cast<size_t>(P.BH) * P.N);
  const size_t hoff = static_cast<size_t>(bh) * P.N * kF32D;
  const float* kh = P.k + hoff;
  const float* vh = P.v + hoff;
  float qh[32], dh[32], dq[32];
#pragma unroll
  for (int d = 0; d < 32; ++d) {
    qh[d] = row_ok ? P.q[hoff + static_cast<size_t>(row) * kF32D + half * 32 + d] : 0.0f;
    dh[d] = row_ok ? P.dout[hoff + static_cast<size_t>(row) * kF32D + half * 32 + d] : 0.0f;
    dq[d] = 0.0f;
  }
  const float tau_r = row_ok ? P.tau[static_cast<size_t>(bh) * P.N + row] : INFINITY;
  const int r_first = rb * 64;
  const int kend = P.causal ? min(P.N, r_first + 64) : P.N;
  float delta = 0.0f;
  for (int pass = 0; pass < 2; ++pass) {
    float gdp = 0.0f, gs = 0.0f;
    for (int key0 = 0; key0 < kend; key0 += kF32Keys) {
      if (!f32_block_active(P, bh, r_first, key0)) continue;   // CTA-uniform skip
      __syncthreads();
      f32_stage(kh, key0, P.N, sk);
      f32_stage(vh, key0, P.N, sv);
      __syncthreads();
#pragma unroll 4
      for (int e = 0; e < 32; ++e) {
        float s = f32_dot<32>(qh, &sk[e][half * 32]);
        float dp = f32_dot<32>(dh, &sv[e][half * 32]);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        dp += __shfl_xor_sync(0xffffffffu, dp, 1);
        const int key = key0 + e;
        const bool ok = row_ok && key < P.N && (!P.causal || key <= row);
        const float t = ok ? fmaxf(fmaf(s, P.c, -tau_r), 0.0f) : 0.0f;
        const float g = ALPHA2 ? (t > 0.0f ? 1.0f : 0.0f) : t;
        if (pass == 0) {
          gdp = fmaf(g, dp, gdp);
          gs += g;
        } else if (g != 0.0f) {
          const float ds = g * (dp - delta);
#pragma unroll
          for (int d = 0; d < 32; ++d) dq[d] = fmaf(ds, sk[e][half * 32 + d], dq[d]);
        }
      }
    }
    if (pass == 0) {
      delta = gs > 0.0f ? gdp / gs : 0.0f;
      if (row_ok && half == 0) P.delta[static_cast<size_t>(bh) * P.N + row] = delta;
    }
  }
  if (row_ok) {
#pragma unroll
    for (int d = 0; d < 32; ++d)
      P.dq[hoff + static_cast<size_t>(row) * kF32D + half * 32 + d] = dq[d] * P.inv_sqrt_d;
  }
}

// ------------------------------------------------------------------ backward columns
// 64 keys per CTA, two threads per key, 32 dims each; rows streamed in tiles of 32.
template <bool ALPHA2>
__global__ void __launch_bounds__(128) entmax_bwd_col_f32_kernel(const F32Params P) {
  __shared__ __align__(16) float sq[kF32Keys][kF32Pad];
  __shared__ __align__(16) float sd[kF32Keys][kF32Pad];
  __shared__ float stau[kF32Keys], sdel[kF32Keys];
  const int tid = threadIdx.x;
  const int half = tid & 1;
  const int cb = blockIdx.x;
  const int bh = blockIdx.y;
  const int key = cb * 64 + (tid >> 1);
  bounds_init(P.status);
  const bool key_ok = key < P.N && in_bounds(static_cast<size_t>(bh) * P.N + key <
                                             static_cast<size_t>(P.BH) * P.N);
  const size_t hoff = static_cast<size_t>(bh) * P.N * kF32D;
  float kh[32], vh[32], dk[32], dv[32];
#pragma unroll
  for (int d = 0; d < 32; ++d) {
    kh[d] = key_ok ? P.k[hoff + static_cast<size_t>(key) * kF32D + half * 32 + d] : 0.0f;
    vh[d] = key_ok ? P.v[hoff + static_cast<size_t>(key) * kF32D + half * 32 + d] : 0.0f;
    dk[d] = 0.0f;
    dv[d] = 0.0f;
  }
  const int c_first = cb * 64;
  const int r_begin = P.causal ? c_first : 0;
  for (int r0 = r_begin; r0 < P.N; r0 += kF32Keys) {
    if (!f32_block_active(P, bh, r0, c_first)) continue;   // CTA-uniform skip
    __syncthreads();
    f32_stage(P.q + hoff, r0, P.N, sq);
    f32_stage(P.dout + hoff, r0, P.N, sd);
    if (tid < kF32Keys) {
      const int r = r0 + tid;
      stau[tid] = r < P.N ? P.tau[static_cast<size_t>(bh) * P.N + r] : INFINITY;
      sdel[tid] = r < P.N ? P.delta[static_cast<size_t>(bh) * P.N + r] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int e = 0; e < 32; ++e) {
      float s = f32_dot<32>(kh, &sq[e][half * 32]);
      float dp = f32_dot<32>(vh, &sd[e][half * 32]);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      const int r = r0 + e;
      const bool ok = key_ok && r < P.N && (!P.causal || key <= r);
      const float t = ok ? fmaxf(fmaf(s, P.c, -stau[e]), 0.0f) : 0.0f;
      if (t > 0.0f) {
        const float p = ALPHA2 ? t : t * t;
        const float g = ALPHA2 ? 1.0f : t;
        const float ds = g * (dp - sdel[e]);
#pragma unroll
        for (int d = 0; d < 32; ++d) {
          dv[d] = fmaf(p, sd[e][half * 32 + d], dv[d]);
          dk[d] = fmaf(ds, sq[e][half * 32 + d], dk[d]);
        }
      }
    }
  }
  if (key_ok) {
#pragma unroll
    for (int d = 0; d < 32; ++d) {
      P.dk[hoff + static_cast<size_t>(key) * kF32D + half * 32 + d] = dk[d] * P.inv_sqrt_d;
      P.dv[hoff + static_cast<size_t>(key) * kF32D + half * 32 + d] = dv[d];
    }
  }
}

}  // namespace entmax
