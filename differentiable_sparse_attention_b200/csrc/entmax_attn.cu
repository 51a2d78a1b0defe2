// Host side of the C ABI declared in include/entmax_attn.h: argument checks,
// workspace layout, TMA tensor maps and kernel launches.  No memory is
// allocated here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "entmax_attn.h"
#include "dash_route.h"
#include "dash.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "simt32.cuh"

using namespace entmax;

namespace {

// ------------------------------------------------------------ workspace layout
struct WsLayout {
  size_t status = 0;     // uint32 status word (+ padding)
  size_t tmax = 0;       // fp16 per-(row, key tile) maxima of s
  size_t tilemask = 0;   // uint32 [BH][T][ceil(T/32)] 128-granularity mask
  size_t tilemaskT = 0;  // uint32 [BH][T][ceil(T/32)] its transpose
  size_t delta = 0;      // float [BH][N]
  size_t vbar = 0;       // float [BH][N][D] g-weighted means of v (forward -> backward)
  size_t half_copies = 0;  // fp16 copies of q, k, v (made by the forward), dout
  size_t total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(int B, int H, int N, int D, int causal) {
  WsLayout L;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t t = (static_cast<size_t>(N) + kTile - 1) / kTile;
  const size_t tiles = causal ? t * (t + 1) / 2 : t * t;
  const size_t words = (t + 31) / 32;
  size_t off = 256;
  L.tmax = off;
  off = align256(off + bh * tiles * 2 * kTile * sizeof(__half));
  L.tilemask = off;
  off = align256(off + bh * t * words * sizeof(uint32_t));
  L.tilemaskT = off;
  off = align256(off + bh * t * words * sizeof(uint32_t));
  L.delta = off;
  off = align256(off + bh * static_cast<size_t>(N) * sizeof(float));
  L.vbar = off;
  off = align256(off + bh * static_cast<size_t>(N) * D * sizeof(float));
  L.half_copies = off;
  off = align256(off + 4 * bh * static_cast<size_t>(N) * D * sizeof(__half));
  L.total = off;
  return L;
}

// Heads per work group of the attention kernels (work_item): as many as keep
// the K and V (or Q and dO) tiles they stream, 2 bytes x N x D each, within
// 64 MB of the 126 MB L2.
int head_group(int BH, int N, int D) {
  const double per_head = 4.0 * static_cast<double>(N) * D;
  const int hg = static_cast<int>((64.0 * 1024 * 1024) / per_head);
  return std::max(1, std::min(BH, hg));
}

// ------------------------------------------------------------ argument checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H, int N, int D, int dtype, float alpha, int block) {
  if (B < 1 || H < 1 || N < 1 || N > kMaxN) return ENTMAX_E_SHAPE;
  if (static_cast<long long>(B) * H * ((N + kTile - 1) / kTile) > 0x7fffffffLL) return ENTMAX_E_SHAPE;
  if (D != 64 && D != 128) return ENTMAX_E_UNSUPPORTED;
  if (dtype != ENTMAX_DTYPE_BF16 && dtype != ENTMAX_DTYPE_FP32) return ENTMAX_E_UNSUPPORTED;
  if (dtype == ENTMAX_DTYPE_FP32 && D != kF32D) return ENTMAX_E_UNSUPPORTED;
  if (block != 64 && block != 128) return ENTMAX_E_UNSUPPORTED;
  // closed forms at 1.5 and 2, powers t^k for the rest of [1.05, 3]
  if (!(alpha >= 1.05f && alpha <= 3.0f)) return ENTMAX_E_ALPHA;
  if (dtype == ENTMAX_DTYPE_FP32 && !(alpha == 1.5f || alpha == 2.0f)) return ENTMAX_E_UNSUPPORTED;
  return ENTMAX_OK;
}

// ------------------------------------------------------------ TMA tensor maps
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [BH][N][D] tensor as a 3-D map {D, N, BH}; box {64 bf16 = 128 B, 128 rows, 1};
// 128-byte swizzle so tiles land in the layout the UMMA descriptors describe.
// Rows past N read as zeros.
bool make_map(CUtensorMap* m, const void* base, int BH, int N, int D,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ profiling aid
// Per calling thread: when enabled, fwd/bwd record CUDA events on their stream
// around each kernel; entmax_attn_profile_read() turns them into milliseconds.
enum : int { EV_FWD0, EV_FWD1, EV_BWD0, EV_BWD_CONV, EV_BWD_MASK, EV_BWD_ROW, EV_BWD_COL, EV_COUNT };
struct Profiler {
  bool on = false;
  bool created = false;
  cudaEvent_t ev[EV_COUNT] = {};
};
thread_local Profiler g_prof;

void prof_mark(int idx, cudaStream_t st) {
  if (g_prof.on && g_prof.created) cudaEventRecord(g_prof.ev[idx], st);
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to the (kernel, device) pair, so it is set
// once per pair: a process may drive several devices.
template <typename Kernel>
bool set_smem(Kernel k, size_t bytes) {
  static std::mutex mu;
  static const void* done_kernel[64] = {};
  static uint64_t done_devices[64][4] = {};   // one bit per device 0..255
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return false;
  const void* key = reinterpret_cast<const void*>(k);
  std::lock_guard<std::mutex> lock(mu);
  int slot = -1;
  for (int a = 0; a < 64 && slot < 0; ++a) {
    if (done_kernel[a] == key) slot = a;
    else if (done_kernel[a] == nullptr) { done_kernel[a] = key; slot = a; }
  }
  if (slot < 0) {   // more kernels than slots: set the attribute on every launch
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes)) == cudaSuccess;
  }
  const uint64_t bit = 1ull << (dev & 63);
  if (done_devices[slot][dev >> 6] & bit) return true;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  done_devices[slot][dev >> 6] |= bit;
  return true;
}

// dst = src in fp16 (exact for bf16 values within the fp16 range; others set
// ENTMAX_ST_RANGE in *status).  D is a multiple of 8, so elems is too.
void launch_to_fp16(const __nv_bfloat16* src, __half* dst, size_t elems, uint32_t* status,
                    cudaStream_t st) {
  const size_t n8 = elems / 8;
  const int grid = static_cast<int>(std::min<size_t>((n8 + 255) / 256, 148 * 8));
  to_fp16_kernel<<<grid, 256, 0, st>>>(src, dst, n8, status);
}

template <int D, int NS, int AM>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const FwdParams& p, cudaStream_t st) {
  auto kern = entmax_fwd_kernel<D, NS, AM>;
  constexpr size_t smem = fwd_smem_bytes<D, NS>();
  static_assert(smem <= 232448, "forward kernel shared memory");
  if (!set_smem(kern, smem)) return ENTMAX_E_CUDA;
  const unsigned grid = static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.tr);
  kern<<<grid, kFwdThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

template <int D, int NSK, int NSV, int AM>
int launch_bwd_row(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mdo, const BwdParams& p, cudaStream_t st) {
  auto kern = entmax_bwd_row_kernel<D, NSK, NSV, AM>;
  constexpr size_t smem = bwd_row_smem_bytes<D, NSK, NSV>();
  static_assert(smem <= 232448, "bwd row kernel shared memory");
  if (!set_smem(kern, smem)) return ENTMAX_E_CUDA;
  const unsigned grid = static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.T);
  kern<<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

template <int D, int NS, int AM>
int launch_bwd_col(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mdo, const BwdParams& p, cudaStream_t st) {
  auto kern = entmax_bwd_col_kernel<D, NS, AM>;
  constexpr size_t smem = bwd_col_smem_bytes<D, NS>();
  static_assert(smem <= 232448, "bwd column kernel shared memory");
  if (!set_smem(kern, smem)) return ENTMAX_E_CUDA;
  const unsigned grid = static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.T);
  kern<<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

int alpha_mode(float alpha) {
  return alpha == 2.0f ? AM_2 : (alpha == 1.5f ? AM_15 : AM_GEN);
}

// The forward kernel for this alpha and head dim (K/V ring depth 3 at D = 64, 2 at 128).
template <int AM>
int launch_fwd_d(int D, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const FwdParams& p, cudaStream_t st) {
  return D == 64 ? launch_fwd<64, 3, AM>(mq, mk, mv, p, st)
                 : launch_fwd<128, 2, AM>(mq, mk, mv, p, st);
}
int launch_fwd_any(float alpha, int D, const CUtensorMap& mq, const CUtensorMap& mk,
                   const CUtensorMap& mv, const FwdParams& p, cudaStream_t st) {
  switch (alpha_mode(alpha)) {
    case AM_2: return launch_fwd_d<AM_2>(D, mq, mk, mv, p, st);
    case AM_15: return launch_fwd_d<AM_15>(D, mq, mk, mv, p, st);
    default: return launch_fwd_d<AM_GEN>(D, mq, mk, mv, p, st);
  }
}

// The backward row kernel, then the column kernel, for this alpha and head dim.
template <int AM>
int launch_bwd_d(int D, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const CUtensorMap& mdo, const BwdParams& prow, const BwdParams& pcol,
                 cudaStream_t st) {
  int rc = D == 64 ? launch_bwd_row<64, 3, 2, AM>(mq, mk, mv, mdo, prow, st)
                   : launch_bwd_row<128, 2, 2, AM>(mq, mk, mv, mdo, prow, st);
  if (rc != ENTMAX_OK) return rc;
  prof_mark(EV_BWD_ROW, st);
  return D == 64 ? launch_bwd_col<64, 3, AM>(mq, mk, mv, mdo, pcol, st)
                 : launch_bwd_col<128, 2, AM>(mq, mk, mv, mdo, pcol, st);
}
int launch_bwd_any(float alpha, int D, const CUtensorMap& mq, const CUtensorMap& mk,
                   const CUtensorMap& mv, const CUtensorMap& mdo, const BwdParams& prow,
                   const BwdParams& pcol, cudaStream_t st) {
  switch (alpha_mode(alpha)) {
    case AM_2: return launch_bwd_d<AM_2>(D, mq, mk, mv, mdo, prow, pcol, st);
    case AM_15: return launch_bwd_d<AM_15>(D, mq, mk, mv, mdo, prow, pcol, st);
    default: return launch_bwd_d<AM_GEN>(D, mq, mk, mv, mdo, prow, pcol, st);
  }
}

// ------------------------------------------------------------ fixed scratch
// Scratch for entmax_attn_fwd_noalloc: status word and counters (first 256
// bytes) followed by the forward's per-(row, key tile) maxima.  It is part of
// the loaded module, so each GPU that loads this library holds these 8 MiB
// until the process exits.  Every call of entmax_attn_fwd_noalloc on a device
// reuses the same bytes.
constexpr size_t kNoAllocScratchBytes = 8u << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Unique id of the calling thread's current context (0 if none): a device's
// context changes after cudaDeviceReset, and with it every device address.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_ctx == nullptr || get_id == nullptr || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device (in host code the
// symbol itself is only a host-side handle, not a device address).  Looked up
// with cudaGetSymbolAddress on the first call per device, and again whenever
// that device's context has changed since (after a cudaDeviceReset).
void* noalloc_scratch_ptr(int device) {
  static std::mutex mu;
  static void* ptrs[256] = {};
  static unsigned long long ctx_ids[256] = {};
  if (device < 0 || device >= 256) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (ptrs[device] == nullptr || ctx == 0 || ctx != ctx_ids[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    ptrs[device] = p;
    ctx_ids[device] = current_context_id();
  }
  return ptrs[device];
}

F32Params make_f32_params(int B, int H, int N, int D, float alpha, int causal, int block,
                          int max_iter, uint8_t* ws, const WsLayout& L) {
  F32Params p{};
  p.BH = B * H;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.block = block;
  p.mask_rows = (N + block - 1) / block;
  p.mask_words = (p.mask_rows + 31) / 32;
  p.max_iter = max_iter;
  p.c = (alpha - 1.0f) / std::sqrt(static_cast<float>(D));
  p.cN = p.c * static_cast<float>(kNB);
  p.slim = 2097152.0f / p.cN;
  p.inv_c = std::nextafter(1.0f / p.c, INFINITY) * (1.0f + 1e-6f);
  p.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(D));
  p.delta = reinterpret_cast<float*>(ws + L.delta);
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.counters = reinterpret_cast<unsigned long long*>(ws + L.status + 8);
  return p;
}

template <bool A2>
int launch_fwd_f32(const F32Params& p, cudaStream_t st) {
  auto kern = entmax_fwd_f32_kernel<A2>;
  if (!set_smem(kern, kF32CandBytes)) return ENTMAX_E_CUDA;
  dim3 grid((p.N + 127) / 128, p.BH);
  kern<<<grid, 128, kF32CandBytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

template <bool A2>
int launch_bwd_f32(const F32Params& p, cudaStream_t st) {
  dim3 grid((p.N + 63) / 64, p.BH);
  entmax_bwd_row_f32_kernel<A2><<<grid, 128, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ENTMAX_E_CUDA;
  prof_mark(EV_BWD_ROW, st);
  entmax_bwd_col_f32_kernel<A2><<<grid, 128, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

}  // namespace

// ============================================================== C ABI
// ------------------------------------------------------- DashAttention router
namespace {
struct DashLayout {
  size_t status = 0, kbar = 0, q16 = 0, total = 0;
  int C = 0, Cp = 0;
};
DashLayout dash_layout(int B, int Hq, int Hkv, int N, int D, int chunk) {
  DashLayout L;
  L.C = N / chunk;
  L.Cp = (L.C + kTile - 1) / kTile * kTile;
  size_t off = 256;
  L.kbar = off;
  off = align256(off + 2 * static_cast<size_t>(B) * Hkv * L.Cp * D * sizeof(__half));
  L.q16 = off;
  off = align256(off + static_cast<size_t>(B) * Hq * N * D * sizeof(__half));
  L.total = off;
  return L;
}
int dash_check(int B, int Hq, int Hkv, int N, int D, int chunk) {
  if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || N < 1 || N > kMaxN || chunk < 1)
    return ENTMAX_E_SHAPE;
  if (N / chunk > DASH_MAX_CHUNKS) return ENTMAX_E_SHAPE;
  if (static_cast<long long>(B) * Hkv * ((N + kTile - 1) / kTile) > 0x7fffffffLL) return ENTMAX_E_SHAPE;
  if (D != 64 && D != 128) return ENTMAX_E_UNSUPPORTED;
  return ENTMAX_OK;
}
template <int D, int AM>
int launch_dash(const CUtensorMap& mq, const CUtensorMap& mkb, const DashParams& p,
                cudaStream_t st) {
  auto kern = dash_route_kernel<D, AM>;
  constexpr size_t smem = dash_smem_bytes<D>();
  static_assert(smem <= 232448, "router kernel shared memory");
  if (!set_smem(kern, smem)) return ENTMAX_E_CUDA;
  const unsigned grid = static_cast<unsigned>(p.BHkv) * static_cast<unsigned>(p.tr);
  kern<<<grid, kDashThreads, smem, st>>>(mq, mkb, p);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}
template <int AM>
int launch_dash_d(int D, const CUtensorMap& mq, const CUtensorMap& mkb, const DashParams& p,
                  cudaStream_t st) {
  return D == 64 ? launch_dash<64, AM>(mq, mkb, p, st) : launch_dash<128, AM>(mq, mkb, p, st);
}
}  // namespace

extern "C" {

int entmax_attn_mask_words(int N, int block) {
  if (N < 1 || N > kMaxN) return ENTMAX_E_SHAPE;
  if (block != 64 && block != 128) return ENTMAX_E_UNSUPPORTED;
  const int tb = (N + block - 1) / block;
  return (tb + 31) / 32;
}

size_t entmax_attn_workspace_size(int B, int H, int N, int D, int block, int causal) {
  if (B < 1 || H < 1 || N < 1 || N > kMaxN) return 0;
  if ((D != 64 && D != 128) || (block != 64 && block != 128)) return 0;
  return ws_layout(B, H, N, D, causal ? 1 : 0).total;
}

int entmax_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int D,
                    int dtype, float alpha, int causal, int block, int max_iter, void* out,
                    float* tau, uint32_t* mask, float* tau_trace, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !tau || !mask || !workspace) return ENTMAX_E_NULL;
  int rc = check_common(B, H, N, D, dtype, alpha, block);
  if (rc != ENTMAX_OK) return rc;
  if (max_iter < 0 || max_iter > ENTMAX_MAX_ITER) return ENTMAX_E_MAXITER;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(tau) ||
      !aligned16(mask) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return ENTMAX_E_ALIGN;
  const WsLayout L = ws_layout(B, H, N, D, causal ? 1 : 0);
  if (workspace_bytes < L.total) return ENTMAX_E_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // status word + work counters live in the first 256 bytes
  if (cudaMemsetAsync(ws + L.status, 0, 8 + CNT_COUNT * sizeof(unsigned long long), st) != cudaSuccess)
    return ENTMAX_E_CUDA;
  if (dtype == ENTMAX_DTYPE_FP32) {
    F32Params p = make_f32_params(B, H, N, D, alpha, causal, block, max_iter, ws, L);
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.out = static_cast<float*>(out);
    p.tau = tau;
    p.mask = mask;
    p.tau_trace = tau_trace;
    prof_mark(EV_FWD0, st);
    rc = alpha == 2.0f ? launch_fwd_f32<true>(p, st) : launch_fwd_f32<false>(p, st);
    prof_mark(EV_FWD1, st);
    return rc;
  }
  // P.V and G.V run on an exact fp16 copy of v, which the backward reuses.
  const size_t elems = static_cast<size_t>(BH) * N * D;
  __half* v16 = reinterpret_cast<__half*>(ws + L.half_copies) + 2 * elems;
  prof_mark(EV_FWD0, st);
  launch_to_fp16(static_cast<const __nv_bfloat16*>(v), v16, elems,
                 reinterpret_cast<uint32_t*>(ws + L.status), st);
  if (cudaGetLastError() != cudaSuccess) return ENTMAX_E_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mk, k, BH, N, D) ||
      !make_map(&mv, v16, BH, N, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return ENTMAX_E_CUDA;

  FwdParams p{};
  p.BH = BH;
  p.N = N;
  p.tr = (N + kTile - 1) / kTile;
  p.tc = p.tr;
  p.hg = head_group(BH, N, D);
  p.causal = causal ? 1 : 0;
  p.block = block;
  p.mask_rows = (N + block - 1) / block;
  p.mask_words = (p.mask_rows + 31) / 32;
  p.max_iter = max_iter;
  p.c = (alpha - 1.0f) / std::sqrt(static_cast<float>(D));
  p.cN = p.c * static_cast<float>(kNB);
  p.slim = 2097152.0f / p.cN;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.tau = tau;
  p.mask = mask;
  p.tau_trace = tau_trace;
  p.tmax = reinterpret_cast<__half*>(ws + L.tmax);
  p.inv_c = std::nextafter(1.0f / p.c, INFINITY) * (1.0f + 1e-6f);
  p.inv_c_dn = std::nextafter(1.0f / p.c, 0.0f) * (1.0f - 1e-6f);
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.counters = reinterpret_cast<unsigned long long*>(ws + L.status + 8);
  p.vbar = reinterpret_cast<float*>(ws + L.vbar);
  p.kpow = 1.0f / (alpha - 1.0f);
  p.am1 = alpha - 1.0f;

  rc = launch_fwd_any(alpha, D, mq, mk, mv, p, st);
  prof_mark(EV_FWD1, st);
  return rc;
}

int entmax_attn_fwd_noalloc(const void* q, const void* k, const void* v, int B, int H, int N,
                            int D, int dtype, float alpha, int causal, int block, int max_iter,
                            void* out, float* tau, uint32_t* mask, void* stream) {
  if (!q || !k || !v || !out || !tau || !mask) return ENTMAX_E_NULL;
  int rc = check_common(B, H, N, D, dtype, alpha, block);
  if (rc != ENTMAX_OK) return rc;
  // only the bf16 kernel runs from the fixed scratch; fp32 inputs take entmax_attn_fwd
  if (dtype != ENTMAX_DTYPE_BF16) return ENTMAX_E_UNSUPPORTED;
  if (max_iter < 0 || max_iter > ENTMAX_MAX_ITER) return ENTMAX_E_MAXITER;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(tau) ||
      !aligned16(mask))
    return ENTMAX_E_ALIGN;
  // Only the forward's part of the workspace layout is needed: the first 256
  // bytes and the tile maxima that follow them.
  const WsLayout L = ws_layout(B, H, N, D, causal ? 1 : 0);
  if (L.tilemask > kNoAllocScratchBytes) return ENTMAX_E_SCRATCH;

  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return ENTMAX_E_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(noalloc_scratch_ptr(device));
  if (ws == nullptr) return ENTMAX_E_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mk, k, BH, N, D) || !make_map(&mv, v, BH, N, D))
    return ENTMAX_E_CUDA;
  // status word and counters must start at zero; the tile maxima are written
  // before they are read by each CTA.
  if (cudaMemsetAsync(ws + L.status, 0, 8 + CNT_COUNT * sizeof(unsigned long long), st) != cudaSuccess)
    return ENTMAX_E_CUDA;

  FwdParams p{};
  p.BH = BH;
  p.N = N;
  p.tr = (N + kTile - 1) / kTile;
  p.tc = p.tr;
  p.hg = head_group(BH, N, D);
  p.causal = causal ? 1 : 0;
  p.block = block;
  p.mask_rows = (N + block - 1) / block;
  p.mask_words = (p.mask_rows + 31) / 32;
  p.max_iter = max_iter;
  p.c = (alpha - 1.0f) / std::sqrt(static_cast<float>(D));
  p.cN = p.c * static_cast<float>(kNB);
  p.slim = 2097152.0f / p.cN;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.tau = tau;
  p.mask = mask;
  p.tau_trace = nullptr;
  p.vbar = nullptr;   // no room for the g-weighted means: P.V in bf16 on v itself
  p.tmax = reinterpret_cast<__half*>(ws + L.tmax);
  p.inv_c = std::nextafter(1.0f / p.c, INFINITY) * (1.0f + 1e-6f);
  p.inv_c_dn = std::nextafter(1.0f / p.c, 0.0f) * (1.0f - 1e-6f);
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.counters = reinterpret_cast<unsigned long long*>(ws + L.status + 8);
  p.kpow = 1.0f / (alpha - 1.0f);
  p.am1 = alpha - 1.0f;

  return launch_fwd_any(alpha, D, mq, mk, mv, p, st);
}

int entmax_attn_noalloc_status(void* stream, uint32_t* status) {
  if (!status) return ENTMAX_E_NULL;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return ENTMAX_E_CUDA;
  const void* ws = noalloc_scratch_ptr(device);
  if (ws == nullptr) return ENTMAX_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ENTMAX_E_CUDA;
  if (cudaMemcpy(status, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ENTMAX_E_CUDA;
  return ENTMAX_OK;
}

int entmax_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* tau, const uint32_t* mask, int B, int H, int N, int D,
                    int dtype, float alpha, int causal, int block, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dout || !tau || !mask || !dq || !dk || !dv || !workspace)
    return ENTMAX_E_NULL;
  int rc = check_common(B, H, N, D, dtype, alpha, block);
  if (rc != ENTMAX_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(tau) ||
      !aligned16(mask) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return ENTMAX_E_ALIGN;
  // gradients only where g = p^(2 - alpha) is bounded (alpha <= 2): beyond, it
  // is unbounded at the edge of the support and float32 scores cannot hold dQ,
  // dK, dV to the bf16 tolerance
  if (alpha > 2.0f) return ENTMAX_E_ALPHA;
  const WsLayout L = ws_layout(B, H, N, D, causal ? 1 : 0);
  if (workspace_bytes < L.total) return ENTMAX_E_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status_word = reinterpret_cast<uint32_t*>(ws + L.status);
  unsigned long long* counters = reinterpret_cast<unsigned long long*>(ws + L.status + 8);
  if (cudaMemsetAsync(counters + CNT_ROW_TILES, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    return ENTMAX_E_CUDA;
  prof_mark(EV_BWD0, st);
  if (dtype == ENTMAX_DTYPE_FP32) {
    F32Params p = make_f32_params(B, H, N, D, alpha, causal, block, 0, ws, L);
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.dout = static_cast<const float*>(dout);
    p.tau = const_cast<float*>(tau);
    p.mask = const_cast<uint32_t*>(mask);
    p.dq = static_cast<float*>(dq);
    p.dk = static_cast<float*>(dk);
    p.dv = static_cast<float*>(dv);
    prof_mark(EV_BWD_CONV, st);
    prof_mark(EV_BWD_MASK, st);
    rc = alpha == 2.0f ? launch_bwd_f32<true>(p, st) : launch_bwd_f32<false>(p, st);
    prof_mark(EV_BWD_COL, st);
    return rc;
  }
  const size_t elems = static_cast<size_t>(BH) * N * D;
  __half* h16[4];
  const void* srcs[4] = {q, k, v, dout};
  for (int a = 0; a < 4; ++a) {
    h16[a] = reinterpret_cast<__half*>(ws + L.half_copies) + a * elems;
    // v's copy was made by the forward
    if (a != 2)
      launch_to_fp16(static_cast<const __nv_bfloat16*>(srcs[a]), h16[a], elems, status_word, st);
  }
  if (cudaGetLastError() != cudaSuccess) return ENTMAX_E_CUDA;
  prof_mark(EV_BWD_CONV, st);
  CUtensorMap mq, mk, mv, mdo;
  const auto f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_map(&mq, h16[0], BH, N, D, f16) || !make_map(&mk, h16[1], BH, N, D, f16) ||
      !make_map(&mv, h16[2], BH, N, D, f16) || !make_map(&mdo, h16[3], BH, N, D, f16))
    return ENTMAX_E_CUDA;

  const int T = (N + kTile - 1) / kTile;
  const int wt = (T + 31) / 32;
  const int mask_rows = (N + block - 1) / block;
  const int mask_words = (mask_rows + 31) / 32;
  uint32_t* tm = reinterpret_cast<uint32_t*>(ws + L.tilemask);
  uint32_t* tmt = reinterpret_cast<uint32_t*>(ws + L.tilemaskT);
  {
    const long long words = static_cast<long long>(BH) * T * wt;
    const int threads = 256;
    const int grid = static_cast<int>(std::min<long long>((words + threads - 1) / threads, 148 * 16));
    tile_mask_kernel<<<grid, threads, 0, st>>>(mask, tm, BH, T, block, mask_rows, mask_words,
                                               status_word);
    tile_mask_t_kernel<<<grid, threads, 0, st>>>(tm, tmt, BH, T, status_word);
    if (cudaGetLastError() != cudaSuccess) return ENTMAX_E_CUDA;
  }
  prof_mark(EV_BWD_MASK, st);

  BwdParams p{};
  p.BH = BH;
  p.N = N;
  p.T = T;
  p.wt = wt;
  p.hg = head_group(BH, N, D);
  p.causal = causal ? 1 : 0;
  p.c = (alpha - 1.0f) / std::sqrt(static_cast<float>(D));
  p.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(D));
  p.tau = tau;
  p.delta = reinterpret_cast<float*>(ws + L.delta);
  p.vbar = reinterpret_cast<const float*>(ws + L.vbar);
  p.dout16 = h16[3];
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.status = status_word;
  p.counters = counters;
  p.kpow = 1.0f / (alpha - 1.0f);

  BwdParams prow = p;
  prow.tm = tm;
  BwdParams pcol = p;
  pcol.tm = tmt;
  rc = launch_bwd_any(alpha, D, mq, mk, mv, mdo, prow, pcol, st);
  prof_mark(EV_BWD_COL, st);
  return rc;
}

int entmax_attn_status(const void* workspace, void* stream, uint32_t* status) {
  if (!workspace || !status) return ENTMAX_E_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ENTMAX_E_CUDA;
  if (cudaMemcpy(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ENTMAX_E_CUDA;
  return ENTMAX_OK;
}

int entmax_attn_counters(const void* workspace, void* stream, unsigned long long* counters,
                         int n) {
  if (!workspace || !counters) return ENTMAX_E_NULL;
  if (n < 1 || n > CNT_COUNT) return ENTMAX_E_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ENTMAX_E_CUDA;
  if (cudaMemcpy(counters, static_cast<const uint8_t*>(workspace) + 8,
                 n * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ENTMAX_E_CUDA;
  return ENTMAX_OK;
}

int entmax_attn_profile(int enable) {
  if (enable && !g_prof.created) {
    for (int e = 0; e < EV_COUNT; ++e)
      if (cudaEventCreate(&g_prof.ev[e]) != cudaSuccess) return ENTMAX_E_CUDA;
    g_prof.created = true;
  }
  g_prof.on = enable != 0;
  return ENTMAX_OK;
}

int entmax_attn_profile_read(float* ms, int n) {
  if (!ms) return ENTMAX_E_NULL;
  if (n < 1 || n > 5) return ENTMAX_E_SHAPE;
  if (!g_prof.created) return ENTMAX_E_CUDA;
  const int pairs[5][2] = {{EV_FWD0, EV_FWD1}, {EV_BWD0, EV_BWD_CONV}, {EV_BWD_CONV, EV_BWD_MASK},
                           {EV_BWD_MASK, EV_BWD_ROW}, {EV_BWD_ROW, EV_BWD_COL}};
  for (int a = 0; a < n; ++a) {
    if (cudaEventSynchronize(g_prof.ev[pairs[a][1]]) != cudaSuccess) return ENTMAX_E_CUDA;
    if (cudaEventElapsedTime(&ms[a], g_prof.ev[pairs[a][0]], g_prof.ev[pairs[a][1]]) != cudaSuccess)
      return ENTMAX_E_CUDA;
  }
  return ENTMAX_OK;
}


size_t dash_route_workspace_size(int B, int Hq, int Hkv, int N, int D, int chunk) {
  if (dash_check(B, Hq, Hkv, N, D, chunk) != ENTMAX_OK) return 0;
  return dash_layout(B, Hq, Hkv, N, D, chunk).total;
}

int dash_route_fwd(const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, int chunk,
                   float gamma, float alpha, int max_iter, float* wbar, uint32_t* row_mask,
                   uint32_t* block_mask, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !workspace) return ENTMAX_E_NULL;
  int rc = dash_check(B, Hq, Hkv, N, D, chunk);
  if (rc != ENTMAX_OK) return rc;
  if (N / chunk == 0) return ENTMAX_OK;   // no complete chunk: the outputs are empty
  if (!wbar || !row_mask || !block_mask) return ENTMAX_E_NULL;
  if (!(alpha >= 1.05f && alpha <= 3.0f)) return ENTMAX_E_ALPHA;
  if (!(gamma > 0.0f) || !std::isfinite(gamma)) return ENTMAX_E_SHAPE;
  if (max_iter < 0 || max_iter > ENTMAX_MAX_ITER) return ENTMAX_E_MAXITER;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(wbar) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(row_mask) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(block_mask) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return ENTMAX_E_ALIGN;
  const DashLayout L = dash_layout(B, Hq, Hkv, N, D, chunk);
  if (workspace_bytes < L.total) return ENTMAX_E_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  if (cudaMemsetAsync(ws + L.status, 0, 256, st) != cudaSuccess) return ENTMAX_E_CUDA;
  __half* q16 = reinterpret_cast<__half*>(ws + L.q16);
  __half* kbar = reinterpret_cast<__half*>(ws + L.kbar);
  launch_to_fp16(static_cast<const __nv_bfloat16*>(q), q16, static_cast<size_t>(B) * Hq * N * D,
                 status, st);
  {
    const long long total = static_cast<long long>(B) * Hkv * L.Cp * (D / 8);
    const int grid = static_cast<int>(std::min<long long>((total + 255) / 256, 148 * 8));
    dash_chunk_mean_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k), kbar, B * Hkv,
                                                 N, D, chunk, L.C, L.Cp, status);
  }
  if (cudaGetLastError() != cudaSuccess) return ENTMAX_E_CUDA;
  CUtensorMap mq, mkb;
  const auto f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_map(&mq, q16, B * Hq, N, D, f16) || !make_map(&mkb, kbar, 2 * B * Hkv, L.Cp, D, f16))
    return ENTMAX_E_CUDA;

  DashParams p{};
  p.BHkv = B * Hkv;
  p.G = Hq / Hkv;
  p.N = N;
  p.C = L.C;
  p.Cp = L.Cp;
  p.chunk = chunk;
  p.tr = (N + kTile - 1) / kTile;
  p.max_iter = max_iter;
  p.c = (alpha - 1.0f) * gamma / std::sqrt(static_cast<float>(D));
  p.kpow = 1.0f / (alpha - 1.0f);
  p.am1 = alpha - 1.0f;
  p.wbar = wbar;
  p.row_mask = row_mask;
  p.block_mask = block_mask;
  p.W = (L.C + 31) / 32;
  p.status = status;
  switch (alpha_mode(alpha)) {
    case AM_2: return launch_dash_d<AM_2>(D, mq, mkb, p, st);
    case AM_15: return launch_dash_d<AM_15>(D, mq, mkb, p, st);
    default: return launch_dash_d<AM_GEN>(D, mq, mkb, p, st);
  }
}

int entmax_attn_wait_selftest(void* workspace, uint32_t* result, unsigned long long limit_ns,
                              void* stream) {
  if (!workspace || !result) return ENTMAX_E_NULL;
  if (limit_ns < 1 || limit_ns > 1000000000ull) return ENTMAX_E_SHAPE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(result) & 3u) != 0)
    return ENTMAX_E_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) return ENTMAX_E_CUDA;
  if (cudaMemsetAsync(result, 0, 3 * sizeof(uint32_t), st) != cudaSuccess) return ENTMAX_E_CUDA;
  wait_selftest_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(workspace), result, limit_ns);
  return cudaGetLastError() == cudaSuccess ? ENTMAX_OK : ENTMAX_E_CUDA;
}

const char* entmax_attn_error_string(int code) {
  switch (code) {
    case ENTMAX_OK: return "success";
    case ENTMAX_E_NULL: return "a required pointer is NULL";
    case ENTMAX_E_ALIGN: return "a tensor pointer is not 16-byte aligned (workspace: 256-byte)";
    case ENTMAX_E_SHAPE: return "B, H or N out of range";
    case ENTMAX_E_UNSUPPORTED: return "head dim, dtype or block size not supported";
    case ENTMAX_E_ALPHA: return "alpha outside [1.05, 3] (forward) or [1.05, 2] (backward)";
    case ENTMAX_E_WORKSPACE: return "workspace smaller than entmax_attn_workspace_size()";
    case ENTMAX_E_CUDA: return "a CUDA call failed";
    case ENTMAX_E_MAXITER: return "max_iter out of range";
    case ENTMAX_E_SCRATCH:
      return "problem needs more scratch than entmax_attn_fwd_noalloc's fixed 8 MiB";
    default: return "unknown error code";
  }
}

}  // extern "C"
