// Forward alpha-entmax attention kernel for sm_100a (bf16 inputs, f32 accumulate).
//
// One CTA owns a 128-row query tile of one (batch, head).  Warp 0 streams K/V
// tiles with TMA, warp 1 issues tcgen05 MMAs into TMEM, and warps 2-9 run the
// epilogues as two warpgroups: warpgroup h handles key columns [64 h, 64 h + 64)
// of every 128-key tile for all 128 query rows (one thread per row), keeps
// its own half of the row's state, and the halves are merged in shared memory
// at the end of each pass.  The CTA walks a sequence of passes over key tiles,
// each driven by a tile list in shared memory:
//
//   HIST    every visible key tile: S = Q K^T, running row max, 8-bin
//           histogram of the scores in the unit window below the max
//           (AdaSplash-2 zh §2.1 / it §2A / ja §2.1 / es §2A), the rounded-up
//           per-(row, tile half) score maximum kept in the workspace, and the
//           row's candidate scores (every score above a running lower bound of
//           tau*).  The reduced histogram problem gives tau_h with
//           tau* - h <= tau_h <= tau* (Proposition 1, as the summaries state it),
//           and the safeguarded Halley (alpha = 1.5) / Newton (alpha = 2) steps
//           (zh §2.2, it §2B, ja §2.2, es §2B) then run in registers over the
//           candidates until the threshold is certified exact (other alpha:
//           powers t^k and a tolerance instead of the certificate).
//   COLLECT (only if a candidate list overflowed) rebuilds the lists above the
//           final lower bound.
//   REFINE  (only if a rebuilt list still overflows) refinement steps that
//           stream the key tiles again.
//   PV      tiles whose recorded maximum exceeds the row's lower bound:
//           p = [s - tau]_+^(1/(alpha-1)) and g = p^(2-alpha) written as fp16 over
//           the scores in TMEM, O += P V and G.V += G V on the tensor cores (A
//           read from TMEM, V an fp16 copy), the bit-packed block mask (32 blocks
//           per uint32 word, zh §2.3) of blocks holding a p > 0, and per row the
//           g-weighted mean of v, G.V / sum g, which the backward's delta needs.
#pragma once

#include <cstddef>

#include <type_traits>

#include "common.cuh"

namespace entmax {

struct FwdParams {
  int BH, N, tr, tc;         // heads x batch, sequence length, 128-tiles per row / column
  int hg;                    // heads per work group (work_item)
  int causal;
  int block;                 // mask block size, 64 or 128
  int mask_rows, mask_words; // ceil(N / block), words per mask row
  int max_iter;
  float c;                   // (alpha - 1) / sqrt(D): s = c * (q . k)
  float cN;                  // c * kNB (exact: kNB is a power of two)
  float slim;                // 2^21 / cN: scores beyond are outside the exact binning range
  __nv_bfloat16* out;
  float* tau;
  uint32_t* mask;
  float* tau_trace;          // nullable, [max_iter + 1][BH][N]
  __half* tmax;              // workspace: per-(row, key tile) maxima of s, rounded up
  float inv_c;               // 1 / c rounded up
  float inv_c_dn;            // 1 / c rounded down
  float kpow;                // k = 1 / (alpha - 1): p = t^k, g = p^(2 - alpha) = t^(k - 1)
  float am1;                 // alpha - 1
  uint32_t* status;          // workspace word 0
  unsigned long long* counters;  // workspace, CNT_* work counters
  // nullable, [BH][N][D]: g-weighted mean of v per row, sum_c g v_c / sum_c g
  // with g = p^(2 - alpha).  Non-null: V is an fp16 copy and P, G are fp16;
  // null: V is the bf16 input, P is bf16 and G is not formed.
  float* vbar;
};

// tau_h: exact root of the reduced histogram problem.  cnt[b] counts the scores
// of grid bin gtop - kNB + b (bin width 1/kNB in s-units, lower edge as the
// representative); with x_b = b / kNB the problem is
// sum_b cnt_b [x_b - tau]_+^k = 1 relative to the window base.  Candidate
// supports are scanned from the top bin down; the first closed-form root that
// does not reach the next lower bin is the root (zh §2.1: the n scores become
// a sum over the bins).  Returns tau_h in s-units.
template <bool ALPHA2, typename R = double>
__device__ __forceinline__ R hist_threshold(const uint32_t (&cnt)[kNB + 1], int gtop) {
  // Scanning from the top bin, the first support {b..kNB} whose reduced
  // function is still >= 0 at the next lower edge x_(b-1) holds the root (it
  // decreases, and at its own lower edge x_b it is already < 0):
  // C x^2 - 2 S1 x + S2 - 1 >= 0 for alpha = 1.5, S1 - C x - 1 >= 0 for
  // alpha = 2.  Only the selected support's closed-form root is evaluated.
  R C = 0, S1 = 0, S2 = 0;
  R Cs = 0, S1s = 0, S2s = 0;
  bool found = false;
#pragma unroll
  for (int b = kNB; b >= 0; --b) {
    const R cb = static_cast<R>(cnt[b]);
    const R x = static_cast<R>(b) / kNB;
    C += cb;
    S1 += cb * x;
    S2 += cb * x * x;
    if (!found && C > R(0)) {
      bool holds = true;
      if (b > 0) {
        const R xl = static_cast<R>(b - 1) / kNB;
        holds = ALPHA2 ? (S1 - C * xl - R(1)) >= R(0)
                       : (C * xl * xl - R(2) * S1 * xl + S2 - R(1)) >= R(0);
      }
      if (holds) {
        found = true;
        Cs = C;
        S1s = S1;
        S2s = S2;
      }
    }
  }
  R rel;
  if (ALPHA2) {
    rel = (S1s - R(1)) / Cs;
  } else {
    const R disc = S1s * S1s - Cs * (S2s - R(1));
    rel = (S1s - sqrt(disc > R(0) ? disc : R(0))) / Cs;
  }
  return static_cast<R>(gtop - kNB) / kNB + rel;
}

// A lower bound of tau_h in s-units, cheaper than the exact root: for every b,
// the C scores of bins b..kNB (first moment A = sum c_b' b') satisfy
// sum c [x - tau]_+^k >= C (mean - tau)^k for tau <= x_b (each term is at least
// (x - tau)^k there; Cauchy-Schwarz for k = 2, equality for k = 1), so the
// reduced function is >= 1 at min(x_b, mean - C^(-1/k)) and tau_h lies above
// it.  The maximum over b is tau_h itself at alpha = 2 and within a fraction
// of a bin of it at 1.5.  Relative margins of 2e-6 cover the fp32 rounding
// (rsqrtf is within 2 ulp).
template <bool ALPHA2>
__device__ __forceinline__ float hist_lower_bound(const uint32_t (&cnt)[kNB + 1], int gtop) {
  float best = -INFINITY;
  uint32_t cc = 0u, aa = 0u;
#pragma unroll
  for (int b = kNB; b >= 0; --b) {
    cc += cnt[b];
    aa += cnt[b] * static_cast<uint32_t>(b);
    const float rs = rsqrtf(static_cast<float>(cc));
    const float ic = rs * rs;
    const float inv_k = ALPHA2 ? ic : rs;          // C^(-1/k)
    const float mean = static_cast<float>(aa) * (1.0f / kNB) * ic;
    const float rb = fminf(static_cast<float>(b) * (1.0f / kNB), mean * 0.999998f - inv_k * 1.000002f);
    best = cc > 0u ? fmaxf(best, rb) : best;
  }
  best += static_cast<float>(gtop - kNB) * (1.0f / kNB);
  return best - 2e-6f * fmaxf(1.0f, fabsf(best));
}

// tau_h for any alpha: bisection on the reduced problem sum_b c_b [x_b - tau]_+^k
// = 1 over [x_top - 1, x_top] (x_top the highest non-empty lower edge; the
// reduced function is >= 1 at its left end and 0 at its right), 20 halvings,
// powers through pow_pos.  The left end of the final bracket, less 1e-4 for the
// rounding of the powers, is returned (s-units): a lower bound of the exact root.
__device__ __forceinline__ float hist_threshold_gen(const uint32_t (&cnt)[kNB + 1], int gtop,
                                                    float k) {
  int top = 0;
#pragma unroll
  for (int b = 0; b <= kNB; ++b) top = cnt[b] > 0u ? b : top;
  float lo = static_cast<float>(top) * (1.0f / kNB) - 1.0f;
  float hi = static_cast<float>(top) * (1.0f / kNB);
#pragma unroll 1
  for (int it = 0; it < 20; ++it) {
    const float mid = 0.5f * (lo + hi);
    float f = -1.0f;
#pragma unroll
    for (int b = 0; b <= kNB; ++b)
      f = fmaf(static_cast<float>(cnt[b]), pow_pos(static_cast<float>(b) * (1.0f / kNB) - mid, k), f);
    if (f > 0.0f) lo = mid;
    else hi = mid;
  }
  return static_cast<float>(gtop - kNB) * (1.0f / kNB) + lo - 1e-4f;
}

// hist_lower_bound for any alpha: x_b - C_b^(-1/k), and for k >= 1 (x^k convex,
// Jensen) min(x_b, mean_b - C_b^(-1/k)).  C^(-1/k) = 2^(-(alpha - 1) log2 C) is
// inflated by 1e-5 for the rounding of the special-function unit.
__device__ __forceinline__ float hist_lower_bound_gen(const uint32_t (&cnt)[kNB + 1], int gtop,
                                                      float k, float am1) {
  float best = -INFINITY;
  uint32_t cc = 0u, aa = 0u;
#pragma unroll
  for (int b = kNB; b >= 0; --b) {
    cc += cnt[b];
    aa += cnt[b] * static_cast<uint32_t>(b);
    const float cf = static_cast<float>(cc);
    const float inv_k = exp2f(-am1 * __log2f(cf)) * 1.00001f;
    const float xb = static_cast<float>(b) * (1.0f / kNB);
    const float mean = static_cast<float>(aa) * (1.0f / kNB) / cf;
    const float rb = k >= 1.0f ? fminf(xb, mean * 0.999998f - inv_k) : xb - inv_k;
    best = cc > 0u ? fmaxf(best, rb) : best;
  }
  best += static_cast<float>(gtop - kNB) * (1.0f / kNB);
  return best - 2e-6f * fmaxf(1.0f, fabsf(best));
}

// One safeguarded step for any alpha (zh §2.2, it §2B, ja §2.2, es §2B): Halley
// for alpha <= 1.5, Newton beyond.  F0 = sum t^k, F1 = sum t^(k-1), F2 =
// sum t^(k-2) over t = s - tau_c > 0; f = F0 - 1, f' = -k F1, f'' = k (k - 1) F2.
// The Newton step solves the equivalent F0^(1/k) = 1 (the same root; for a
// single support score it is linear in tau): tau + (F0^(1/k) - 1) F0 /
// (F0^(1/k) F1).  The bracket [lo, hi] follows the sign of f; a step that
// leaves it, or is longer than half the step taken two iterations earlier
// (dx2; dx1 is the last one), is replaced by bisection, so the steps shrink
// geometrically and no cycle survives.  Beyond alpha = 2 the pages take secant
// steps; on the oracle this Newton step needs fewer (about 3.2 on average at
// alpha = 3, against 5.0 for the secant, whose slowest rows had not converged
// after 12).  Returns true once f is within 1e-4 and the step below
// 1e-6 max(1, |tau|), or the bracket is that narrow -- the powers are accurate
// to about 1e-6, so there is no exactness certificate as for the closed forms.
__device__ __forceinline__ bool solver_step_gen(double F0, double F1, double F2, float k,
                                                float& tau_c, double& lo, double& hi,
                                                double& dx1, double& dx2) {
  const double f = F0 - 1.0;
  const double tc = tau_c;
  if (f > 0.0) lo = fmax(lo, tc);
  else if (f < 0.0) hi = fmin(hi, tc);
  double tn = NAN;
  if (k >= 2.0f) {
    const double fp = -static_cast<double>(k) * F1;
    const double fpp = static_cast<double>(k) * (k - 1.0f) * F2;
    tn = tc - 2.0 * f * fp / (2.0 * fp * fp - f * fpp);          // Halley
  } else if (F0 > 0.0 && F1 > 0.0) {
    const double q = exp2(log2(F0) / static_cast<double>(k));     // F0^(1/k)
    tn = tc + (q - 1.0) * F0 / (q * F1);                           // Newton on F0^(1/k)
  }
  if (!(tn > lo && tn < hi) || fabs(tn - tc) > 0.5 * fabs(dx2))
    tn = 0.5 * (lo + hi);                                          // bisection fallback
  dx2 = dx1;
  dx1 = tn - tc;
  const double tol = 1e-6 * fmax(1.0, fabs(tc));
  const bool done =
      f == 0.0 || (fabs(tn - tc) <= tol && fabs(f) <= 1e-4) || hi - lo <= 2.0 * tol;
  tau_c = static_cast<float>(f == 0.0 ? tc : tn);
  return done;
}

// Safety margin below tau_h that absorbs the rounding of s and tau (2^-20 |tau|).
__device__ __forceinline__ double hist_margin(double tau_h) {
  return 9.5367431640625e-07 * fmax(1.0, fabs(tau_h));
}

// One safeguarded refinement step from tau_c (zh §2.2, it §2B, ja §2.2, es §2B).
// F0 = sum t^k, F1 = sum t^(k-1), F2 = sum t^(k-2) over the support S = {t > 0},
// t = s - tau_c (alpha = 1.5: k = 2; alpha = 2: k = 1); tmin / tneg are the
// smallest positive and the largest non-positive t seen; every score left out
// of the sums lies at or below l_drop.  The bracket [lo, hi] is updated from
// the sign of f, then r, the root of f restricted to S (linear for alpha = 2,
// the smaller root of the quadratic F2 d^2 - 2 F1 d + f in d = tau - tau_c for
// alpha = 1.5), is tau* when no score lies between tau_c and r -- the support
// does not change on the way -- and bounds tau* otherwise: from the right it is
// a lower bound, from the left a lower bound for alpha = 2 (f is convex) and an
// upper bound for alpha = 1.5 ([x]_+^2 <= x^2).  Without that certificate the
// next point is the Newton (alpha = 2) or Halley (alpha = 1.5) step, replaced
// by bisection when it leaves the bracket.  Returns true when tau_c is exact.
template <bool ALPHA2>
__device__ __forceinline__ bool solver_step(double F0, double F1, double F2, float tmin,
                                            float tneg, double l_drop, float& tau_c, double& lo,
                                            double& hi) {
  const double f = F0 - 1.0;
  if (f > 0.0) lo = fmax(lo, static_cast<double>(tau_c));
  else if (f < 0.0) hi = fmin(hi, static_cast<double>(tau_c));
  bool exact = (f == 0.0);
  double tn = tau_c;
  double r = NAN;
  if (!exact && F1 > 0.0) {
    if (ALPHA2) {
      r = tau_c + f / F1;
    } else {
      const double disc = F1 * F1 - F2 * f;
      if (disc >= 0.0 && F2 > 0.0) r = tau_c + (F1 - sqrt(disc)) / F2;
    }
    if (!isnan(r)) {
      const double d = r - tau_c;
      exact = f > 0.0 ? d <= static_cast<double>(tmin)
                      : (d >= static_cast<double>(tneg) && r >= l_drop);
      if (exact) tn = r;
      else if (ALPHA2 || f < 0.0) lo = fmax(lo, r);
      else hi = fmin(hi, r);
    }
  }
  if (!exact) {
    if (ALPHA2) {
      tn = r;                                                    // Newton step
    } else {
      const double fp = -2.0 * F1, fpp = 2.0 * F2;
      tn = tau_c - 2.0 * f * fp / (2.0 * fp * fp - f * fpp);     // Halley step
    }
    if (!(tn >= lo && tn <= hi)) tn = 0.5 * (lo + hi);           // bisection fallback
  }
  tau_c = static_cast<float>(tn);
  if (exact) lo = fmax(lo, static_cast<double>(__double2float_rd(tn)));
  return exact;
}

constexpr int kFwdThreads = 352;   // warp 0 TMA, warp 1 S MMAs, warps 2-9 epilogue, warp 10 P.V MMAs
constexpr int kFwdEpiThreads = 256;
constexpr int kPvWarp = 10;

__device__ __forceinline__ void fwd_epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// The same barrier, returning whether v held for any of the 256 threads.
__device__ __forceinline__ bool fwd_epi_bar_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0u;
}

// Per-row state that warpgroup 1 hands to warpgroup 0 at the end of a pass.
struct FwdXrow {
  float m_raw;
  int gtop;
  int gtop_set;
  float acc;
  int ncand;
  int over;
  uint32_t cnt[kNB + 1];
  float pad;
};

template <int D, int NS>
struct FwdSmem {
  __nv_bfloat16 q[kTile * D];       // D/64 swizzled slabs
  __nv_bfloat16 k[NS][kTile * D];
  __nv_bfloat16 v[NS][kTile * D];
  // candidate storage beyond the V ring (P and G of the P.V pass live in TMEM),
  // in slots of one float per row: what the 227 KB of shared memory leave
  static constexpr int kCandXSlots = D == 64 ? 184 : 88;
  float cx[kCandXSlots * kTile];
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS];
  uint64_t v_full[NS], v_empty[NS];
  // S buffers in TMEM: three at D = 64 (3 x 128 + 2 x 64 columns), two at 128
  static constexpr int kNSB = D == 64 ? 3 : 2;
  uint64_t s_full[kNSB], s_empty[kNSB];
  uint64_t p_full[kNSB], p_empty[kNSB], o_full, drain, drain_pv;
  uint32_t tmem_base;
  int abort_flag;
  int ctl_kind, ctl_n, ctl_iter;
  int not_converged;
  int cand_overflow;
  uint32_t flags[kMaxTiles / 32];
  uint32_t maskw[2][kMaxMaskWords];
  uint16_t tiles[kMaxTiles];
  // warpgroup exchange
  FwdXrow x1[kTile];          // 1 -> 0: histogram / candidate state
  double xf[3][kTile];        // 1 -> 0: refinement partial sums
  float xtmin[kTile], xtneg[kTile], xsum[kTile];
  float xg[2][kTile];         // both: partial sums of g per warpgroup
  double xlo[kTile];          // 0 -> 1: bracket lower bound
  float xtau[kTile];          // 0 -> 1: current threshold
  int xflag[kTile];           // 0 -> 1: list rebuilt by COLLECT
  int xact[kTile];            // 0 -> 1: the row still iterates over its lists
};

// Candidate scores live in the V ring and the slots after it, which stay idle
// until the P.V pass: slot-major [cap][128 rows] floats (thread r uses column r, so
// appends and reads are free of bank conflicts); warpgroup h owns slots
// [h cap/2, (h + 1) cap/2).  A list is compacted at most kMaxPrunes times;
// after that it is rebuilt by a COLLECT pass.
constexpr int kMaxPrunes = 16;

template <int D, int NS>
__host__ __device__ constexpr int fwd_cand_cap() {
  return (NS * kTile * D * 2) / (4 * kTile) + FwdSmem<D, NS>::kCandXSlots;
}

template <int D, int NS>
constexpr size_t fwd_smem_bytes() {
  return sizeof(FwdSmem<D, NS>) + 1024;  // + slack for 1024-byte alignment
}
static_assert(fwd_smem_bytes<64, 3>() <= 232448 && fwd_smem_bytes<128, 2>() <= 232448,
              "forward shared memory above the 227 KB per block");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Counts of a histogram whose top bin is g_from, re-expressed for top bin g_to >= g_from.
__device__ __forceinline__ uint32_t hist_shifted(const uint32_t (&c)[kNB + 1], int b, int d) {
  const int src = b + d;
  uint32_t r = 0u;
#pragma unroll
  for (int s = 0; s <= kNB; ++s) r = (s == src) ? c[s] : r;
  return r;
}

template <int D, int NS, int AM>
__global__ void __launch_bounds__(kFwdThreads, 1)
    entmax_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdParams P) {
  constexpr bool ALPHA2 = AM == AM_2;
  constexpr bool GEN = AM == AM_GEN;    // any other alpha: powers t^k
  extern __shared__ uint8_t smem_raw[];
  using Smem = FwdSmem<D, NS>;
  Smem& sm = *reinterpret_cast<Smem*>(align1024(smem_raw));
  constexpr int kSlabs = D / 64;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  constexpr uint32_t kIdescS = make_idesc(kTile, kTile, 1, 1, 0, 0);  // Q (K-major) x K (K-major)
  // P / G (TMEM) x V (SMEM, MN-major): fp16 with the g-weighted means, else bf16
  const uint32_t idesc_pv = P.vbar != nullptr ? make_idesc(kTile, D, 0, 0, 0, 1)
                                              : make_idesc(kTile, D, 1, 1, 0, 1);
  const bool gv = P.vbar != nullptr;
  constexpr uint32_t kNSB = Smem::kNSB;
  constexpr uint32_t kColO = kNSB * kTile;   // TMEM: S buffers (P / G of the P.V pass), O, G.V
  constexpr uint32_t kColG = kColO + D;
  static_assert(kColG + D <= 512, "TMEM columns");
  constexpr int kCap = fwd_cand_cap<D, NS>();
  constexpr int kCapH = kCap / 2;
  static_assert(offsetof(Smem, cx) == offsetof(Smem, v) + NS * kTile * D * 2,
                "candidates need the V ring and the extra slots to be adjacent");
  static_assert(kCapH * 2 == kCap, "two equal halves");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work unit: head groups that share L2, the latest (longest causal) row tiles
  // first within a group.
  const WorkItem wi = work_item(static_cast<int>(blockIdx.x), P.BH, P.tr, P.hg);
  const int i = P.tr - 1 - wi.r;
  const int bh = wi.bh;
  bounds_init(P.status);
  // elements of the tile-maxima record, of a [BH][N] and a [BH][N][D] tensor
  // (bounds-checked build)
  const size_t tmax_elems =
      static_cast<size_t>(P.BH) *
      (P.causal ? static_cast<size_t>(P.tr) * (P.tr + 1) / 2 : static_cast<size_t>(P.tr) * P.tc) *
      (2 * kTile);
  const size_t n_rows_all = static_cast<size_t>(P.BH) * P.N;
  const size_t n_elems_all = n_rows_all * D;
  const int ntc = P.causal ? (i + 1) : P.tc;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < static_cast<int>(kNSB); ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_empty[s], 8);
      mbar_init(&sm.p_full[s], 8);
      mbar_init(&sm.p_empty[s], 1);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain_pv, 1);
    sm.abort_flag = 0;
    sm.not_converged = 0;
    sm.cand_overflow = 0;
    sm.ctl_kind = PASS_HIST;
    sm.ctl_n = ntc;
    sm.ctl_iter = 0;
    fence_mbar_init();
  }
  for (int w = threadIdx.x; w < kMaxTiles / 32; w += kFwdThreads) sm.flags[w] = 0u;
  for (int w = threadIdx.x; w < 2 * kMaxMaskWords; w += kFwdThreads) (&sm.maskw[0][0])[w] = 0u;
  for (int t = threadIdx.x; t < ntc; t += kFwdThreads) sm.tiles[t] = static_cast<uint16_t>(t);
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  // -------- role state that lives across passes
  uint32_t kc = 0, vc = 0, sc = 0, pc = 0;   // K loads, V loads, S tiles, PV tiles
  bool q_issued = false, q_waited = false;

  // epilogue: warpgroup wg, one query row per thread, key columns [hc0, hc0 + 64)
  const int wg = warp >= 2 ? (warp - 2) >> 2 : 0;
  const int hc0 = wg * 64;
  const int quad = warp & 3;
  const int rl = quad * 32 + lane;
  const int row = i * kTile + rl;
  const bool row_ok = (warp >= 2) && row < P.N;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const int n_valid = P.causal ? min(row + 1, P.N) : P.N;
  float m_raw = -INFINITY;                 // running max of q.k (raw units), this half
  int gtop = 0;                            // grid index floor(kNB * s) of the max
  bool gtop_set = false;
  uint32_t cnt[kNB + 1];
#pragma unroll
  for (int b = 0; b <= kNB; ++b) cnt[b] = 0u;
  float vclamp = -P.slim;                  // scores are clamped to >= vclamp before binning
  uint32_t cbase = 0u;
  // Candidate scores of this half of the row: every q.k above acc_raw, which
  // only grows and always stays at or below a lower bound of tau* (the running
  // max - 1/c, raised to the partial histogram's tau_h).  Scores left out are
  // never in the support.
  float* cand_base = reinterpret_cast<float*>(&sm.v[0][0]);
  float* my_cand = cand_base + (wg * kCapH) * kTile + rl;     // slot a at my_cand[a * 128]
  // slot a of this thread's list (checked against the list's capacity in the
  // bounds-checked build; an out-of-range read yields -inf, below any bound)
  auto cand_put = [&](int a, float x) {
    if (in_bounds(a >= 0 && a < kCapH)) my_cand[a * kTile] = x;
  };
  auto cand_get = [&](int a) -> float {
    return in_bounds(a >= 0 && a < kCapH) ? my_cand[a * kTile] : -INFINITY;
  };
  int ncand = 0;
  float acc_raw = -INFINITY;
  bool cand_over = false;
  int prunes = 0;
  bool collect = false;                    // list rebuilt by a COLLECT pass above lo
  int ncand1 = 0;                          // warpgroup 0: size of warpgroup 1's list
  double lo = 0.0, hi = 0.0;               // bracket of tau*
  double l_drop = -INFINITY;               // every score left out of the candidates is <= l_drop
  double dx1 = INFINITY, dx2 = INFINITY;   // last two steps of the generic-alpha solver
  float tau_c = 0.0f;                      // current evaluation point / final tau
  int iter = 0;
  bool row_done = false;                   // threshold certified exact
  float rowsum = 0.0f;
  float gsum = 0.0f;                       // sum of g = p^(2 - alpha) over this half

  auto trace_store = [&](int it, float val) {
    if (P.tau_trace != nullptr && row_ok && wg == 0 && it <= P.max_iter)
      if (in_bounds((static_cast<size_t>(it) * P.BH + bh) * P.N + row <
                    static_cast<size_t>(P.max_iter + 1) * n_rows_all))
        P.tau_trace[(static_cast<size_t>(it) * P.BH + bh) * P.N + row] = val;
  };
  auto needs_mask = [&](int j) {
    return (P.causal && j == i) || (j * kTile + hc0 + 64 > P.N);
  };
  auto apply_mask = [&](float (&v)[32], int j, int ch) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int col = j * kTile + hc0 + ch * 32 + e;
      const bool ok = col < P.N && (!P.causal || col <= row);
      v[e] = ok ? v[e] : -INFINITY;
    }
  };

  for (;;) {
    __syncthreads();
    const int kind = sm.ctl_kind;
    const int n = sm.ctl_n;
    const int aborted = sm.abort_flag;
    __syncthreads();
    if (aborted || kind == PASS_DONE) break;

    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        bool ok = true;
        if (!q_issued) {
          q_issued = true;
          mbar_expect_tx(&sm.q_full, kTileBytes);
#pragma unroll
          for (int s = 0; s < kSlabs; ++s)
            tma_load_3d(sm.q + s * kTile * 64, &tm_q, &sm.q_full, s * 64, i * kTile, bh);
        }
        for (int t = 0; t < n && ok; ++t) {
          const int j = in_bounds(sm.tiles[t] < P.tc) ? sm.tiles[t] : 0;
          {
            const uint32_t slot = kc % NS, use = kc / NS;
            if (use > 0 && !mbar_wait(&sm.k_empty[slot], (use - 1) & 1, abort_flag, P.status)) {
              ok = false;
              break;
            }
            mbar_expect_tx(&sm.k_full[slot], kTileBytes);
#pragma unroll
            for (int s = 0; s < kSlabs; ++s)
              tma_load_3d(sm.k[slot] + s * kTile * 64, &tm_k, &sm.k_full[slot], s * 64,
                          j * kTile, bh);
            ++kc;
          }
          if (kind == PASS_PV) {
            const uint32_t slot = vc % NS, use = vc / NS;
            if (use > 0 && !mbar_wait(&sm.v_empty[slot], (use - 1) & 1, abort_flag, P.status)) {
              ok = false;
              break;
            }
            mbar_expect_tx(&sm.v_full[slot], kTileBytes);
#pragma unroll
            for (int s = 0; s < kSlabs; ++s)
              tma_load_3d(sm.v[slot] + s * kTile * 64, &tm_v, &sm.v_full[slot], s * 64,
                          j * kTile, bh);
            ++vc;
          }
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ S issuer
      // S = Q K^T of every pass.  In the P.V pass warp kPvWarp issues the P.V
      // MMAs, so a wait in one warp leaves the other's MMAs running on the
      // tensor pipe.  Every lane runs the issue loop (warp-uniform
      // descriptors); one elected lane issues each MMA and commit.
      {
        bool ok = true;
        if (!q_waited) {
          q_waited = true;
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full, 0, abort_flag, P.status));
        }
        const uint32_t q_addr = smem_u32(sm.q);
        for (int t = 0; t < n && ok; ++t) {
          const uint32_t slot = kc % NS;
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.k_full[slot], (kc / NS) & 1, abort_flag, P.status));
          if (!ok) break;
          const uint32_t sb = sc % kNSB, use = sc / kNSB;
          if (use > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_empty[sb], (use - 1) & 1, abort_flag, P.status));
            if (!ok) break;
          }
          // In the P.V pass S(t) reuses the TMEM buffer of P.V tile t - kNSB:
          // wait for those MMAs too
          if (kind == PASS_PV && t >= static_cast<int>(kNSB)) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_empty[t % kNSB], ((t / kNSB) - 1) & 1,
                                                   abort_flag, P.status));
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm.k[slot]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSlabBytes + (kk & 3) * 32;
            mma_f16_ss_warp(tmem + sb * kTile, smem_desc_sw128(q_addr + off, 16, 1024),
                       smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit_warp(&sm.s_full[sb]);
          mma_commit_warp(&sm.k_empty[slot]);
          ++kc;
          ++sc;
        }
      }
      __syncwarp();
    } else if (warp == kPvWarp) {
      // ------------------------------------------------------------ P.V issuer
      // O += P V and (with the g-weighted means) G.V += G V for P.V tile t.
      // P and G sit in the S buffer of their tile: 32-key chunk c occupies
      // columns 32 c .. 32 c + 31, P packed in the first 16, G in the last 16.
      // sc follows the S issuer's count (n S tiles per pass) so that tile t's
      // buffer is (S count at the pass start + t) % kNSB.
      if (kind == PASS_PV) {
        bool ok = true;
        const uint32_t sc0 = sc;
        for (int t = 0; t < n && ok; ++t) {
          const uint32_t pb = pc % kNSB;
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_full[pb], (pc / kNSB) & 1, abort_flag, P.status));
          if (!ok) break;
          const uint32_t slot = vc % NS;
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.v_full[slot], (vc / NS) & 1, abort_flag, P.status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t t_p = tmem + ((sc0 + pc) % kNSB) * kTile;
          const uint32_t v_addr = smem_u32(sm.v[slot]);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t a_col = (kk >> 1) * 32 + (kk & 1) * 8;
            const uint64_t vd = smem_desc_sw128(v_addr + kk * 16 * 128, kSlabBytes, 1024);
            const uint32_t acc = (pc > 0 || kk > 0) ? 1u : 0u;
            mma_f16_ts_warp(tmem + kColO, t_p + a_col, vd, idesc_pv, acc);
            if (gv) mma_f16_ts_warp(tmem + kColG, t_p + a_col + 16, vd, idesc_pv, acc);
          }
          mma_commit_warp(&sm.v_empty[slot]);
          mma_commit_warp(&sm.p_empty[pb]);
          ++vc;
          ++pc;
        }
        if (ok) mma_commit_warp(&sm.o_full);
      }
      sc += static_cast<uint32_t>(n);
      __syncwarp();
    } else {
      // ------------------------------------------------------------ epilogue
      bool ok = true;
      double F0 = 0.0, F1 = 0.0, F2 = 0.0;  // refinement sums at tau_c (this half)
      float Tmin = INFINITY;                // smallest positive s - tau_c
      float Tneg = -INFINITY;               // largest non-positive s - tau_c
      if (kind == PASS_PV) {
        rowsum = 0.0f;
        gsum = 0.0f;
      }
      for (int t = 0; t < n; ++t) {
        const int j = in_bounds(sm.tiles[t] < P.tc) ? sm.tiles[t] : 0;
        const uint32_t cur = sc++;
        const uint32_t sb = cur % kNSB;
        ok = mbar_wait(&sm.s_full[sb], (cur / kNSB) & 1, abort_flag, P.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const bool msk = needs_mask(j);
        const uint32_t t_s = t_lane + sb * kTile + hc0;

        if (kind == PASS_HIST) {
          // Both 32-column chunks of this tile half are loaded under one wait,
          // and the S buffer goes back to the S issuer at once: the pass only
          // reads the scores, and the candidate appends below use the registers.
          uint32_t rr[2][32];
          tmem_ld32x2(t_s, rr[0], t_s + 32, rr[1]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_empty[sb]);
          float v[2][32];
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[ch][e] = __uint_as_float(rr[ch][e]);
            if (msk) apply_mask(v[ch], j, ch);
          }
          // maxima of the 8-score groups and of each chunk (independent trees)
          float gm[2][4], cmv[2];
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float a = fmaxf(fmaxf(v[ch][8 * g], v[ch][8 * g + 1]),
                                    fmaxf(v[ch][8 * g + 2], v[ch][8 * g + 3]));
              const float b = fmaxf(fmaxf(v[ch][8 * g + 4], v[ch][8 * g + 5]),
                                    fmaxf(v[ch][8 * g + 6], v[ch][8 * g + 7]));
              gm[ch][g] = fmaxf(a, b);
            }
            cmv[ch] = fmaxf(fmaxf(gm[ch][0], gm[ch][1]), fmaxf(gm[ch][2], gm[ch][3]));
          }
          const float tile_max = fmaxf(cmv[0], cmv[1]);
          m_raw = fmaxf(m_raw, tile_max);
          // one window update per tile half: binning both chunks against the
          // window of the new running max leaves the same counts as binning
          // chunk by chunk and shifting in between (the shift drops exactly the
          // bins below the new window)
          if (tile_max > -INFINITY) {
            const int gc = static_cast<int>(
                __float_as_uint(__fmaf_rd(fmaxf(tile_max, -P.slim), P.cN, kMagic)) - kMagicBits);
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
              // Scores below the window are clamped to grid index <= base - 1,
              // whose shift amount is "negative" and adds nothing.
              vclamp = (static_cast<float>(gtop - kNB) - 1.5f) / P.cN;
              cbase = 0u - 7u * (kMagicBits + static_cast<uint32_t>(gtop - kNB));
            }
          }
          // Only 8-score groups reaching the window add to the histogram (most
          // scores of a long row lie far below it once the running max has
          // settled).  9 bins in 7-bit lanes of 64-bit words: bin b of a score
          // is floor(kNB * s) - (gtop - kNB), exact via a round-down FMA against
          // 1.5 * 2^23; two independent words, lanes hold at most 32 counts.
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            if (cmv[ch] > vclamp) {
              uint64_t pk0 = 0, pk1 = 0;
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                if (gm[ch][g] > vclamp) {
#pragma unroll
                  for (int e = 8 * g; e < 8 * g + 8; ++e) {
                    const float u = __fmaf_rd(fmaxf(v[ch][e], vclamp), P.cN, kMagic);
                    const uint32_t sh = __float_as_uint(u) * 7u + cbase;
                    if (e & 1) pk1 += shl64(1ull, sh);
                    else pk0 += shl64(1ull, sh);
                  }
                }
              }
              const uint64_t packed = pk0 + pk1;
#pragma unroll
              for (int b = 0; b <= kNB; ++b)
                cnt[b] += static_cast<uint32_t>(packed >> (7 * b)) & 127u;
            }
          }
          // Candidates of this tile half: every score above acc_raw, raised to a
          // lower bound of the partial histogram's tau_h (scores seen so far by
          // this warpgroup, so <= tau*) whenever a chunk reaches the current bound.
          {
            acc_raw = fmaxf(acc_raw, __fsub_rd(m_raw, P.inv_c));
            if (row_ok && !cand_over && gtop_set && tile_max > acc_raw) {
              const float lb = GEN ? hist_lower_bound_gen(cnt, gtop, P.kpow, P.am1)
                                   : hist_lower_bound<ALPHA2>(cnt, gtop);   // s-units
              acc_raw = fmaxf(acc_raw, lb * (lb >= 0.0f ? P.inv_c_dn : P.inv_c));
            }
          }
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const bool want = row_ok && !cand_over && cmv[ch] > acc_raw;
            if (!want) continue;
            if (ncand + 32 > kCapH) {
              if (prunes < kMaxPrunes) {
                ++prunes;
                int kept = 0;
                for (int a = 0; a < ncand; ++a) {
                  const float xa = cand_get(a);
                  if (xa > acc_raw) cand_put(kept++, xa);
                }
                ncand = kept;
              }
              cand_over = ncand + 32 > kCapH;
            }
            if (!cand_over) {
              if constexpr (D == 128) {
                // only the 8-score groups whose maximum reaches the bound (at
                // D = 64 the longer live range of the group maxima costs more
                // than the skipped compares: 0.634 against 0.612 ms at 4K)
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                  if (gm[ch][g] > acc_raw) {
#pragma unroll
                    for (int e = 8 * g; e < 8 * g + 8; ++e) {
                      if (v[ch][e] > acc_raw) cand_put(ncand++, v[ch][e]);
                    }
                  }
                }
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  if (v[ch][e] > acc_raw) cand_put(ncand++, v[ch][e]);
                }
              }
            }
          }
          const float rec = row_ok ? tile_max * P.c : -INFINITY;
          const size_t ti = tmax_index(bh, i, j, P.tr, P.tc, P.causal) + wg * kTile + rl;
          if (in_bounds(ti < tmax_elems)) P.tmax[ti] = __float2half_ru(rec);
        } else if (kind == PASS_COLLECT) {
          // rebuild the lists of the rows that overflowed: exactly the scores above lo
          const float thr = collect ? __double2float_rd(lo / P.c) : INFINITY;
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[32];
            tmem_ld32(t_s + ch * 32, r);
            if (ch == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.s_empty[sb]);
            }
            if (!collect) continue;
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
            if (msk) apply_mask(v, j, ch);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (v[e] > thr) {
                if (ncand < kCapH) cand_put(ncand, v[e]);
                ++ncand;
              }
            }
          }
        } else if (kind == PASS_REFINE) {
          // four independent partial accumulators per quantity (ILP)
          float f0[4] = {0.f, 0.f, 0.f, 0.f}, f1[4] = {0.f, 0.f, 0.f, 0.f},
                f2[4] = {0.f, 0.f, 0.f, 0.f};
          float tmin[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
          float tneg[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[32];
            tmem_ld32(t_s + ch * 32, r);
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
            if (msk) apply_mask(v, j, ch);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int a = e & 3;
              const float tt = fmaf(v[e], P.c, -tau_c);
              const bool in = tt > 0.0f;
              const float tp = fmaxf(tt, 0.0f);
              tmin[a] = in ? fminf(tmin[a], tt) : tmin[a];
              tneg[a] = in ? tneg[a] : fmaxf(tneg[a], tt);
              if (GEN) {
                const float pk = pow_pos(tt, P.kpow);
                const float pk1 = in ? __fdividef(pk, tt) : 0.0f;     // t^(k-1)
                f0[a] += pk;
                f1[a] += pk1;
                if (P.kpow >= 2.0f) f2[a] += in ? __fdividef(pk1, tt) : 0.0f;
              } else if (ALPHA2) {
                f0[a] += tp;
                f1[a] += in ? 1.0f : 0.0f;
              } else {
                f0[a] = fmaf(tp, tp, f0[a]);
                f1[a] += tp;
                f2[a] += in ? 1.0f : 0.0f;
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_empty[sb]);
          F0 += (f0[0] + f0[1]) + (f0[2] + f0[3]);
          F1 += (f1[0] + f1[1]) + (f1[2] + f1[3]);
          F2 += (f2[0] + f2[1]) + (f2[2] + f2[3]);
          Tmin = fminf(Tmin, fminf(fminf(tmin[0], tmin[1]), fminf(tmin[2], tmin[3])));
          Tneg = fmaxf(Tneg, fmaxf(fmaxf(tneg[0], tneg[1]), fmaxf(tneg[2], tneg[3])));
        } else {  // PASS_PV
          // P (and G) replace the scores in this S buffer; the S issuer puts
          // S(t + kNSB) into it only after the P.V MMAs of this tile completed.
          const uint32_t pb = pc % kNSB;
          ++pc;
          float part = 0.f, gpart = 0.f;
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[32];
            tmem_ld32(t_s + ch * 32, r);
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
            if (msk) apply_mask(v, j, ch);
            uint32_t w[16], wgt[16];
            // p (and g) of the chunk packed for the tensor core: fp16 P and G with
            // the g-weighted means, bf16 P without -- a per-launch choice, so the
            // score loop is instantiated for each
            auto pv_chunk = [&](auto gv_tag) {
            constexpr bool GV = decltype(gv_tag)::value;
            float ps[4] = {0.f, 0.f, 0.f, 0.f}, gs[4] = {0.f, 0.f, 0.f, 0.f};
            __half2 gcount = __float2half2_rn(0.0f);   // alpha = 2: support size
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (GEN) {
                const float t0 = fmaxf(fmaf(v[2 * e], P.c, -tau_c), 0.0f);
                const float t1 = fmaxf(fmaf(v[2 * e + 1], P.c, -tau_c), 0.0f);
                // g = t^(k - 1), held below 6e4 (fp16) where alpha > 2 lets it grow
                // without bound at the edge of the support
                const float p0 = pow_pos(t0, P.kpow);
                const float p1 = pow_pos(t1, P.kpow);
                const float g0 = t0 > 0.0f ? fminf(__fdividef(p0, t0), 6.0e4f) : 0.0f;
                const float g1 = t1 > 0.0f ? fminf(__fdividef(p1, t1), 6.0e4f) : 0.0f;
                ps[e & 3] += p0 + p1;
                if constexpr (GV) {
                  gs[e & 3] += g0 + g1;
                  const __half2 h2 = __floats2half2_rn(p0, p1);
                  const __half2 g2 = __floats2half2_rn(g0, g1);
                  w[e] = *reinterpret_cast<const uint32_t*>(&h2);
                  wgt[e] = *reinterpret_cast<const uint32_t*>(&g2);
                } else {
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                  w[e] = *reinterpret_cast<const uint32_t*>(&h2);
                }
              } else {
                // p = t^k <= 1 with sum p = 1, so t lies in [0, 1] at tau*: the
                // clamp to the support is a saturating FMA
                const float t0 = fma_sat(v[2 * e], P.c, -tau_c);
                const float t1 = fma_sat(v[2 * e + 1], P.c, -tau_c);
                if constexpr (GV) {
                  const __half2 th = __floats2half2_rn(t0, t1);
                  if (ALPHA2) {
                    // p = t; g = 1 on the support, counted exactly in half2
                    const __half2 g2 = __hgt2(th, __float2half2_rn(0.0f));
                    gcount = __hadd2(gcount, g2);
                    ps[(2 * e) & 3] += t0;
                    ps[(2 * e + 1) & 3] += t1;
                    w[e] = *reinterpret_cast<const uint32_t*>(&th);
                    wgt[e] = *reinterpret_cast<const uint32_t*>(&g2);
                  } else {
                    // g = t, and p = t^2 squared from the fp16 t
                    const __half2 p2 = __hmul2(th, th);
                    ps[(2 * e) & 3] = fmaf(t0, t0, ps[(2 * e) & 3]);
                    ps[(2 * e + 1) & 3] = fmaf(t1, t1, ps[(2 * e + 1) & 3]);
                    gs[(2 * e) & 3] += t0;
                    gs[(2 * e + 1) & 3] += t1;
                    w[e] = *reinterpret_cast<const uint32_t*>(&p2);
                    wgt[e] = *reinterpret_cast<const uint32_t*>(&th);
                  }
                } else {
                  const float p0 = ALPHA2 ? t0 : t0 * t0;
                  const float p1 = ALPHA2 ? t1 : t1 * t1;
                  ps[e & 3] += p0 + p1;
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                  w[e] = *reinterpret_cast<const uint32_t*>(&h2);
                }
              }
            }
            if (ALPHA2 && GV) gs[0] = __low2float(gcount) + __high2float(gcount);
            part += (ps[0] + ps[1]) + (ps[2] + ps[3]);
            gpart += (gs[0] + gs[1]) + (gs[2] + gs[3]);
            };
            if (gv) pv_chunk(std::true_type{});
            else pv_chunk(std::false_type{});
            tmem_st16(t_s + ch * 32, w);
            if (gv) tmem_st16(t_s + ch * 32 + 16, wgt);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sm.p_full[pb]);
            mbar_arrive(&sm.s_empty[sb]);
          }
          gsum += gpart;
          rowsum += part;
          const uint32_t bits = __ballot_sync(0xffffffffu, row_ok && part > 0.f);
          if (lane == 0 && bits != 0u) {
            if (P.block == kTile) {
              if (in_bounds((j >> 5) < kMaxMaskWords))
                atomicOr(&sm.maskw[0][j >> 5], 1u << (j & 31));
            } else {  // block 64: two mask rows per tile, key block 2 j + wg
              const int h = quad >> 1;
              const int kb = 2 * j + wg;
              if (in_bounds((kb >> 5) < kMaxMaskWords))
                atomicOr(&sm.maskw[h][kb >> 5], 1u << (kb & 31));
            }
          }
        }
      }

      // ---------------- end of pass: merge the halves, solve, next tile list
      auto build_list = [&](double thr_d) {
        const float thr = row_ok ? __double2float_rd(thr_d) : INFINITY;
        // 16 tile maxima in flight per thread: the loads are latency-bound
        constexpr int kU = 16;
        for (int t = 0; t < n; t += kU) {
          float hv[kU];
          int jj[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            jj[u] = (t + u < n) ? static_cast<int>(sm.tiles[t + u]) : -1;
            const size_t ti = jj[u] >= 0 ? tmax_index(bh, i, jj[u], P.tr, P.tc, P.causal) +
                                               wg * kTile + rl
                                         : 0;
            hv[u] = jj[u] >= 0 && in_bounds(ti < tmax_elems && jj[u] < P.tc)
                        ? __half2float(P.tmax[ti])
                        : -INFINITY;
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const uint32_t b = __ballot_sync(0xffffffffu, hv[u] > thr);
            if (lane == 0 && b != 0u && jj[u] >= 0 && in_bounds((jj[u] >> 5) < kMaxTiles / 32))
              atomicOr(&sm.flags[jj[u] >> 5], 1u << (jj[u] & 31));
          }
        }
      };
      // Refinement over the row's candidate lists, in registers, once the lists
      // hold every score above lo.  Each warpgroup sums over its own list;
      // warpgroup 0 adds warpgroup 1's partial sums and takes the step.  All
      // 256 epilogue threads run the same iterations (two barriers each) while
      // any row of the tile still iterates.
      auto refine_registers = [&]() {
        bool act = false;
        if (wg == 0) {
          act = row_ok && !cand_over && !(collect && kind == PASS_HIST) && !row_done &&
                iter < P.max_iter;
          sm.xact[rl] = act ? 1 : 0;
          sm.xtau[rl] = tau_c;
          sm.xlo[rl] = lo;
        }
        bool first = true;
        for (;;) {
          if (!fwd_epi_bar_any(act)) break;
          if (wg == 1) {
            act = sm.xact[rl] != 0;
            tau_c = sm.xtau[rl];
          }
          if (first && act) {
            // keep only the candidates above lo (the others contribute nothing at
            // any tau >= lo), so the iterations run over roughly the support
            const double lo_r = wg == 0 ? lo : sm.xlo[rl];
            const float thr = __double2float_rd(lo_r / P.c);
            int kept = 0;
            for (int a = 0; a < ncand; ++a) {
              const float xa = cand_get(a);
              if (xa > thr) cand_put(kept++, xa);
            }
            ncand = kept;
            if (wg == 0) l_drop = fmax(l_drop, static_cast<double>(thr) * P.c);
          }
          first = false;
          float f0[4] = {0.f, 0.f, 0.f, 0.f}, f1[4] = {0.f, 0.f, 0.f, 0.f},
                f2[4] = {0.f, 0.f, 0.f, 0.f};
          float tmn[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
          float tng[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          const int nown = act ? ncand : 0;
          for (int e0 = 0; e0 < nown; e0 += 4) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const int e = e0 + a;
              const float tt = e < nown ? fmaf(cand_get(e), P.c, -tau_c) : -INFINITY;
              const bool in = tt > 0.0f;
              const float tp = fmaxf(tt, 0.0f);
              tmn[a] = in ? fminf(tmn[a], tt) : tmn[a];
              tng[a] = in ? tng[a] : fmaxf(tng[a], tt);
              if (GEN) {
                const float pk = pow_pos(tt, P.kpow);
                const float pk1 = in ? __fdividef(pk, tt) : 0.0f;     // t^(k-1)
                f0[a] += pk;
                f1[a] += pk1;
                if (P.kpow >= 2.0f) f2[a] += in ? __fdividef(pk1, tt) : 0.0f;
              } else if (ALPHA2) {
                f0[a] += tp;
                f1[a] += in ? 1.0f : 0.0f;
              } else {
                f0[a] = fmaf(tp, tp, f0[a]);
                f1[a] += tp;
                f2[a] += in ? 1.0f : 0.0f;
              }
            }
          }
          const float s0 = (f0[0] + f0[1]) + (f0[2] + f0[3]);
          const float s1 = (f1[0] + f1[1]) + (f1[2] + f1[3]);
          const float s2 = (f2[0] + f2[1]) + (f2[2] + f2[3]);
          const float smin = fminf(fminf(tmn[0], tmn[1]), fminf(tmn[2], tmn[3]));
          const float sneg = fmaxf(fmaxf(tng[0], tng[1]), fmaxf(tng[2], tng[3]));
          if (wg == 1) {
            sm.xf[0][rl] = s0;
            sm.xf[1][rl] = s1;
            sm.xf[2][rl] = s2;
            sm.xtmin[rl] = smin;
            sm.xtneg[rl] = sneg;
          }
          fwd_epi_bar();
          if (wg == 0 && act) {
            const double F0c = static_cast<double>(s0) + sm.xf[0][rl];
            const double F1c = static_cast<double>(s1) + sm.xf[1][rl];
            const double F2c = static_cast<double>(s2) + sm.xf[2][rl];
            const float tminc = fminf(smin, sm.xtmin[rl]);
            const float tnegc = fmaxf(sneg, sm.xtneg[rl]);
            row_done = GEN ? solver_step_gen(F0c, F1c, F2c, P.kpow, tau_c, lo, hi, dx1, dx2)
                           : solver_step<ALPHA2>(F0c, F1c, F2c, tminc, tnegc, l_drop, tau_c,
                                                 lo, hi);
            ++iter;
            trace_store(iter, tau_c);
            act = !row_done && iter < P.max_iter;
            sm.xact[rl] = act ? 1 : 0;
            sm.xtau[rl] = tau_c;
          }
        }
      };
      // warpgroup 0 -> 1: the row's threshold, lower bound and COLLECT flag
      auto publish = [&]() {
        if (wg == 0) {
          sm.xtau[rl] = tau_c;
          sm.xlo[rl] = lo;
          sm.xflag[rl] = collect ? 1 : 0;
        }
        fwd_epi_bar();
        if (wg == 1) {
          tau_c = sm.xtau[rl];
          lo = sm.xlo[rl];
          collect = sm.xflag[rl] != 0;
        }
      };
      // Publish the next pass: PV unless some row still needs its list rebuilt
      // (COLLECT) or must refine over the key tiles (REFINE).
      auto next_pass = [&](int passes_done_kind) {
        // the candidate slots are V-ring memory that TMA and the tensor core
        // use next: order these generic accesses before them
        fence_proxy_async_smem();
        build_list(lo);
        fwd_epi_bar();
        if (warp == 2) {
          const int nn = compact_tiles(sm.flags, (ntc + 31) >> 5, sm.tiles);
          if (lane == 0) {
            sm.ctl_n = nn;
            int next = PASS_PV;
            if (sm.cand_overflow == 1) next = PASS_COLLECT;
            else if (sm.cand_overflow == 2 && sm.ctl_iter < P.max_iter && sm.not_converged)
              next = PASS_REFINE;
            sm.ctl_kind = next;
            sm.not_converged = 0;
            atomicAdd(&P.counters[passes_done_kind], static_cast<unsigned long long>(n));
            if (passes_done_kind == CNT_REFINE_TILES) atomicAdd(&P.counters[CNT_REFINE_PASSES], 1ull);
          }
        }
      };

      if (kind == PASS_HIST) {
        if (wg == 1) {
          FwdXrow& x = sm.x1[rl];
          x.m_raw = m_raw;
          x.gtop = gtop;
          x.gtop_set = gtop_set ? 1 : 0;
          x.acc = acc_raw;
          x.ncand = ncand;
          x.over = cand_over ? 1 : 0;
#pragma unroll
          for (int b = 0; b <= kNB; ++b) x.cnt[b] = cnt[b];
        }
        fwd_epi_bar();
        double tau_h = 0.0;
        if (wg == 0 && row_ok) {
          // merge warpgroup 1's half of the row into this one
          const FwdXrow& x = sm.x1[rl];
          if (x.gtop_set) {
            uint32_t c1[kNB + 1];
#pragma unroll
            for (int b = 0; b <= kNB; ++b) c1[b] = x.cnt[b];
            const int g = gtop_set ? max(gtop, x.gtop) : x.gtop;
            const int d0 = gtop_set ? g - gtop : kNB + 1;
            const int d1 = g - x.gtop;
#pragma unroll
            for (int b = 0; b <= kNB; ++b) {
              const uint32_t a0 = d0 <= kNB ? hist_shifted(cnt, b, d0) : 0u;
              const uint32_t a1 = d1 <= kNB ? hist_shifted(c1, b, d1) : 0u;
              cnt[b] = a0 + a1;
            }
            gtop = g;
            gtop_set = true;
          }
          m_raw = fmaxf(m_raw, x.m_raw);
          acc_raw = fmaxf(acc_raw, x.acc);
          ncand1 = x.ncand;
          cand_over = cand_over || x.over;
          if (fabsf(m_raw * P.cN) >= 2097152.0f) atomicOr(P.status, ST_RANGE);
          tau_h = GEN ? static_cast<double>(hist_threshold_gen(cnt, gtop, P.kpow))
                      : hist_threshold<ALPHA2>(cnt, gtop);
          const double margin = hist_margin(tau_h);
          const double m_s = static_cast<double>(m_raw) * P.c;
          // n^(1 - alpha), the distance of tau* below the max at the latest
          const double nb =
              GEN ? static_cast<double>(exp2f(-P.am1 * __log2f(static_cast<float>(n_valid)))) *
                        (1.0 - 1e-5)
                  : (ALPHA2 ? 1.0 / n_valid : 1.0 / sqrt(static_cast<double>(n_valid)));
          lo = tau_h - margin;
          hi = fmin(tau_h + 1.0 / kNB + margin, m_s - nb + margin);
          l_drop = static_cast<double>(acc_raw) * P.c;   // every unlisted score is <= l_drop <= tau*
          lo = fmax(lo, l_drop);
          if (hi < lo) hi = lo;
          tau_c = __double2float_rd(lo);
          lo = tau_c;
          if (cand_over && P.max_iter > 0) {
            // a list lost scores: rebuild both halves above lo in a COLLECT pass
            collect = true;
            cand_over = false;
            l_drop = lo;
            sm.cand_overflow = 1;
          }
        }
        iter = 0;
        trace_store(0, static_cast<float>(tau_h));
        refine_registers();
        publish();
        if (collect) {
          ncand = 0;
          cand_over = false;
        }
        next_pass(CNT_HIST_TILES);
        if (warp == 2 && lane == 0 && sm.ctl_kind == PASS_COLLECT)
          atomicAdd(&P.counters[CNT_CAND_OVERFLOW], 1ull);
      } else if (kind == PASS_COLLECT) {
        if (wg == 1) sm.x1[rl].ncand = ncand;
        fwd_epi_bar();
        if (wg == 0 && row_ok && collect) {
          ncand1 = sm.x1[rl].ncand;
          cand_over = ncand > kCapH || ncand1 > kCapH;
          if (cand_over) sm.cand_overflow = 2;   // refine this tile over the key tiles
        }
        fwd_epi_bar();
        if (warp == 2 && lane == 0 && sm.cand_overflow == 1) sm.cand_overflow = 0;
        fwd_epi_bar();
        refine_registers();
        if (wg == 0 && row_ok && !row_done && iter < P.max_iter) sm.not_converged = 1;
        publish();
        next_pass(CNT_REFINE_TILES);
      } else if (kind == PASS_REFINE) {
        if (wg == 1) {
          sm.xf[0][rl] = F0;
          sm.xf[1][rl] = F1;
          sm.xf[2][rl] = F2;
          sm.xtmin[rl] = Tmin;
          sm.xtneg[rl] = Tneg;
        }
        fwd_epi_bar();
        if (wg == 0 && row_ok && !row_done && iter < P.max_iter) {
          F0 += sm.xf[0][rl];
          F1 += sm.xf[1][rl];
          F2 += sm.xf[2][rl];
          Tmin = fminf(Tmin, sm.xtmin[rl]);
          Tneg = fmaxf(Tneg, sm.xtneg[rl]);
          row_done = GEN ? solver_step_gen(F0, F1, F2, P.kpow, tau_c, lo, hi, dx1, dx2)
                         : solver_step<ALPHA2>(F0, F1, F2, Tmin, Tneg, l_drop, tau_c, lo, hi);
          ++iter;
          trace_store(iter, tau_c);
          if (!row_done && iter < P.max_iter) sm.not_converged = 1;
        }
        if (warp == 2 && lane == 0) ++sm.ctl_iter;
        publish();
        next_pass(CNT_REFINE_TILES);
      } else {  // PASS_PV: write O, tau, mask
        if (ok && n > 0) {
          ok = mbar_wait(&sm.o_full, 0, abort_flag, P.status);
          ok = __all_sync(0xffffffffu, ok);
        }
        tc_fence_after();
        if (wg == 1) sm.xsum[rl] = rowsum;
        sm.xg[wg][rl] = gsum;
        fwd_epi_bar();
        const float gtot = sm.xg[0][rl] + sm.xg[1][rl];
        const size_t row_idx = static_cast<size_t>(bh) * P.N + row;
        __nv_bfloat16* orow = P.out + row_idx * D;
        // warpgroup wg stores O columns [wg D/2, (wg + 1) D/2)
#pragma unroll 1
        for (int ch = wg * (D / 64); ch < (wg + 1) * (D / 64); ++ch) {
          uint32_t r[32];
          if (ok && n > 0) {
            tmem_ld32(t_lane + kColO + ch * 32, r);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          if (row_ok && in_bounds(row_idx * D + ch * 32 + 32 <= n_elems_all)) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 h2 =
                  __floats2bfloat162_rn(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
              w[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int qd = 0; qd < 4; ++qd)
              dst[qd] = make_uint4(w[4 * qd], w[4 * qd + 1], w[4 * qd + 2], w[4 * qd + 3]);
          }
        }
        if (gv) {
          // g-weighted means of v: G.V / sum g, columns [wg D/2, (wg + 1) D/2)
          const float inv_g = gtot > 0.0f ? 1.0f / gtot : 0.0f;
          float* vrow = P.vbar + row_idx * D;
#pragma unroll 1
          for (int ch = wg * (D / 64); ch < (wg + 1) * (D / 64); ++ch) {
            uint32_t r[32];
            if (ok && n > 0) {
              tmem_ld32(t_lane + kColG + ch * 32, r);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = 0u;
            }
            if (row_ok && in_bounds(row_idx * D + ch * 32 + 32 <= n_elems_all)) {
              float4* dst = reinterpret_cast<float4*>(vrow + ch * 32);
#pragma unroll
              for (int qd = 0; qd < 8; ++qd)
                dst[qd] = make_float4(__uint_as_float(r[4 * qd]) * inv_g,
                                      __uint_as_float(r[4 * qd + 1]) * inv_g,
                                      __uint_as_float(r[4 * qd + 2]) * inv_g,
                                      __uint_as_float(r[4 * qd + 3]) * inv_g);
            }
          }
        }
        tc_fence_before();
        if (wg == 0 && row_ok) {
          rowsum += sm.xsum[rl];
          if (in_bounds(row_idx < n_rows_all)) P.tau[row_idx] = tau_c;
          // sum p = 1 within 1e-3; for k < 1 (alpha > 2) p = t^k turns a rounding
          // eps of s or tau (2^-23 of their magnitude) into eps^k at the edge of
          // the support, so the check allows 8 such terms
          float sum_tol = 1e-3f;
          if (GEN && P.kpow < 1.0f)
            sum_tol = fmaxf(sum_tol, 8.0f * pow_pos(1.2e-7f * (fabsf(tau_c) + 2.0f), P.kpow));
          if (!(fabsf(rowsum - 1.0f) <= sum_tol)) atomicOr(P.status, ST_NOT_CONVERGED);
        }
        if (wg == 0)
          for (int it = iter + 1; it <= P.max_iter; ++it) trace_store(it, tau_c);
        const int spr = kTile / P.block;
        const int et = threadIdx.x - 64;
        for (int idx = et; idx < spr * P.mask_words; idx += kFwdEpiThreads) {
          const int h = idx / P.mask_words;
          const int w = idx - h * P.mask_words;
          const int mrow = i * spr + h;
          if (mrow < P.mask_rows &&
              in_bounds(h < 2 && w < kMaxMaskWords &&
                        (static_cast<size_t>(bh) * P.mask_rows + mrow) * P.mask_words + w <
                            static_cast<size_t>(P.BH) * P.mask_rows * P.mask_words))
            P.mask[(static_cast<size_t>(bh) * P.mask_rows + mrow) * P.mask_words + w] =
                sm.maskw[h][w];
        }
        if (warp == 2 && lane == 0) {
          sm.ctl_kind = PASS_DONE;
          atomicAdd(&P.counters[CNT_PV_TILES], static_cast<unsigned long long>(n));
        }
      }
    }
  }

  // ---------------- teardown: drain in-flight copies / MMAs after an abort,
  // then release TMEM.
  if (sm.abort_flag) {
    if (warp == 0 && lane == 0) {
      for (uint32_t s = 0; s < NS; ++s) {
        if (kc > s) mbar_wait(&sm.k_full[s], ((kc - 1 - s) / NS) & 1, nullptr, nullptr);
        if (vc > s) mbar_wait(&sm.v_full[s], ((vc - 1 - s) / NS) & 1, nullptr, nullptr);
      }
    }
    if (warp == 1) {
      mma_commit_warp(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, nullptr);
    }
    if (warp == kPvWarp) {
      mma_commit_warp(&sm.drain_pv);
      mbar_wait(&sm.drain_pv, 0, nullptr, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace entmax
