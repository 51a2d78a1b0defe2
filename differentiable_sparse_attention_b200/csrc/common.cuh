// Shared constants and small device helpers of the alpha-entmax kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100.cuh"

namespace entmax {

constexpr int kTile = 128;                   // compute tile: 128 query rows x 128 keys
constexpr int kMaxN = 262144;
constexpr int kMaxTiles = kMaxN / kTile;     // 2048 tiles per row
constexpr int kMaxMaskWords = kMaxN / 64 / 32;  // words per mask row at block 64
constexpr int kSlabBytes = kTile * 128;      // one [128 rows][128 B] swizzled slab
constexpr int kNB = 8;                       // histogram bins per unit of s
constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u; // bit pattern of kMagic

// alpha: the closed forms of 1.5 (p = t^2) and 2 (p = t), or any other alpha in
// [1.05, 3] through powers t^k, k = 1 / (alpha - 1).
enum AlphaMode : int { AM_15 = 0, AM_2 = 1, AM_GEN = 2 };

// t^e for t > 0 (0 otherwise) from the base-2 logarithm and exponential of the
// special-function unit: relative error about |e log2 t| 2^-22.
__device__ __forceinline__ float pow_pos(float t, float e) {
  return t > 0.0f ? exp2f(e * __log2f(t)) : 0.0f;
}

// Exercises the bounded wait: one thread waits on an mbarrier that no thread
// arrives at, with a limit of limit_ns.  The wait gives up, raises the abort
// flag and ST_TIMEOUT in *status exactly as in the attention kernels, and the
// kernel returns; result[0] = 1 once it has returned from the wait.
__global__ void wait_selftest_kernel(uint32_t* status, uint32_t* result, unsigned long long limit_ns) {
  bounds_init(status);
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    result[0] = 1u;
    result[1] = ok ? 1u : 0u;
    result[2] = abort_flag ? 1u : 0u;
  }
}

enum PassKind : int { PASS_HIST = 0, PASS_REFINE = 1, PASS_PV = 2, PASS_DONE = 3, PASS_COLLECT = 4 };

// Work counters kept in the workspace right after the status word (uint64 each).
enum Counter : int {
  CNT_HIST_TILES = 0,    // forward: key tiles visited by histogram passes
  CNT_REFINE_TILES = 1,  // forward: key tiles visited by refinement passes
  CNT_PV_TILES = 2,      // forward: key tiles visited by the P.V pass
  CNT_REFINE_PASSES = 3, // forward: refinement passes, summed over 128-row tiles
  CNT_ROW_TILES = 4,     // backward: key tiles per pass of the row kernel
  CNT_COL_TILES = 5,     // backward: query tiles visited by the column kernel
  CNT_CAND_OVERFLOW = 6, // forward: 128-row tiles whose candidate lists overflowed
  CNT_COUNT = 8
};


// a * b + c clamped to [0, 1] in one instruction (a NaN result becomes 0).
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 64-bit left shift with the PTX clamp rule: a shift amount >= 64 (including
// "negative" amounts seen as huge unsigned values) yields 0.
__device__ __forceinline__ uint64_t shl64(uint64_t x, uint32_t sh) {
  uint64_t r;
  asm("shl.b64 %0, %1, %2;" : "=l"(r) : "l"(x), "r"(sh));
  return r;
}

// Work order of the attention kernels.  Heads run in groups of hg, a group's
// streamed K and V (or Q and dO) small enough to stay in L2 together; within a
// group the CTAs take their tile in the order r = 0, 1, ... across the group's
// heads (r = 0 the longest causal row or column).  Ordering all heads at once
// lets the resident CTAs span every head, whose tiles then miss L2 at long N;
// one head at a time unbalances the SMs when a CTA's work is comparable to an
// SM's share (short N).
struct WorkItem {
  int bh;
  int r;
};
__device__ __forceinline__ WorkItem work_item(int block, int BH, int T, int hg) {
  const int g = block / (hg * T);
  const int gsize = min(hg, BH - g * hg);
  const int rem = block - g * hg * T;
  return {g * hg + rem % gsize, rem / gsize};
}

// Offset (in elements) of the tile-max record of (row tile i, key tile j) of
// head bh: two halves (key columns 0-63 and 64-127) of 128 rows each.  Causal
// problems store only the lower triangle j <= i.
__device__ __forceinline__ size_t tmax_index(int bh, int i, int j, int tr, int tc, int causal) {
  const size_t per = causal ? static_cast<size_t>(tr) * (tr + 1) / 2
                            : static_cast<size_t>(tr) * tc;
  const size_t idx = causal ? static_cast<size_t>(i) * (i + 1) / 2 + j
                            : static_cast<size_t>(i) * tc + j;
  return (static_cast<size_t>(bh) * per + idx) * (2 * kTile);
}

// Maximum of 32 values as a 5-level tree (a linear chain would serialise 31
// dependent max operations in the epilogue).
__device__ __forceinline__ float max32(const float (&v)[32]) {
  float m[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) m[e] = fmaxf(v[e], v[e + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int e = 0; e < w; ++e) m[e] = fmaxf(m[e], m[e + w]);
  }
  return m[0];
}

// Warp-parallel compaction of the set bits of flags[0, nwords) into a sorted
// tile list (find-first-set / popcount traversal).  Clears the flags it read.
// Executed by one full warp; returns the number of tiles.
__device__ __forceinline__ int compact_tiles(uint32_t* flags, int nwords, uint16_t* tiles) {
  const int lane = threadIdx.x & 31;
  int total = 0;
  for (int base = 0; base < nwords; base += 32) {
    const int w = base + lane;
    uint32_t word = (w < nwords) ? flags[w] : 0u;
    if (w < nwords) flags[w] = 0u;
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

}  // namespace entmax
