/*
 * entmax_attn.h -- C ABI of the B200 (sm_100a) alpha-entmax attention library.
 *
 * What is computed.  For every (batch b, head h) and query row r:
 *     z_rc = q_r . k_c / sqrt(D)            (causal: only keys c <= r)
 *     s_rc = (alpha - 1) * z_rc
 *     p_rc = [ s_rc - tau_r ]_+ ^ (1/(alpha-1)),  tau_r chosen so sum_c p_rc = 1
 *     O_r  = sum_c p_rc v_c
 * alpha-entmax is the sparse, differentiable softmax replacement that the
 * AdaSplash-2 summaries ("AdaSplash-2: Faster Differentiable Sparse
 * Attention", zh/it/ja/es pages, section 1) build on; tau is the normaliser
 * they liken to log-sum-exp.  tau is reported in s-units (the units of s
 * above, i.e. (alpha-1) * z).
 *
 * How (zh §2.1-2.3, it §2A-2C, ja §2.1-2.3, es §2A-2C): one streaming pass
 * over the key blocks builds an on-chip histogram of the scores per query row
 * and solves the reduced problem for a lower bound tau_h of tau; one or two
 * safeguarded Halley (alpha <= 1.5) or Newton (beyond) steps refine it; a
 * bit-packed block mask (32 blocks per uint32) records the non-zero blocks and
 * P.V, dQ, dK and dV visit only those blocks.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory: scratch space is the caller's `workspace`.
 *   - q, k, v, out, dout, dq, dk, dv: contiguous [B][H][N][D], element type
 *     `dtype` (ENTMAX_DTYPE_BF16 or ENTMAX_DTYPE_FP32), 16-byte aligned.
 *   - tau: float32 [B][H][N].  mask: uint32 [B][H][Tb][W] with
 *     Tb = ceil(N / block) row blocks and W = entmax_attn_mask_words(N, block)
 *     words per row block; bit (j % 32) of word j / 32 is key block j (least
 *     significant bit = lowest block index).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; a return of ENTMAX_OK means the work
 *     was enqueued, not that it finished.
 *   - Work runs on the calling thread's current CUDA device.  Every pointer
 *     and the stream must belong to that device.  A process may drive several
 *     devices: each kernel's shared-memory limit is raised once per device,
 *     on that device's first launch of the kernel.
 *   - Arguments are validated before anything is enqueued; on an error return
 *     nothing has been launched and no output was touched.
 *   - Conditions found on the device (a row whose probabilities do not sum to
 *     1 within 1e-3, a bounded wait that timed out, an out-of-range score) are
 *     OR-ed into a status word at the start of the workspace; read it with
 *     entmax_attn_status().  Kernels never trap.
 *   - Supported: D in {64, 128}; block in {64, 128}; 1 <= N <= ENTMAX_MAX_N;
 *     alpha in [1.05, 3] for bf16 (closed forms at 1.5 and 2, powers
 *     t^(1/(alpha-1)) through the special-function unit otherwise) and
 *     {1.5, 2.0} for fp32; dtype bf16 (tcgen05 tensor-core path) or fp32
 *     (CUDA-core path for full fp32 precision, D = 64 only).
 */
#ifndef ENTMAX_ATTN_H
#define ENTMAX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define ENTMAX_OK             0
#define ENTMAX_E_NULL        -1  /* a required pointer is NULL                     */
#define ENTMAX_E_ALIGN       -2  /* a tensor pointer is not 16-byte aligned         */
#define ENTMAX_E_SHAPE       -3  /* B, H or N out of range                          */
#define ENTMAX_E_UNSUPPORTED -4  /* D, dtype or block not supported                 */
#define ENTMAX_E_ALPHA       -5  /* alpha outside [1.05, 3]                         */
#define ENTMAX_E_WORKSPACE   -6  /* workspace smaller than entmax_attn_workspace_size */
#define ENTMAX_E_CUDA        -7  /* a CUDA call failed (launch, tensor-map encode)  */
#define ENTMAX_E_MAXITER     -8  /* max_iter outside [0, ENTMAX_MAX_ITER]            */
#define ENTMAX_E_SCRATCH     -9  /* entmax_attn_fwd_noalloc: problem needs more than
                                    ENTMAX_NOALLOC_SCRATCH_BYTES of scratch          */

/* element types */
#define ENTMAX_DTYPE_BF16 0
#define ENTMAX_DTYPE_FP32 1

/* device status bits (entmax_attn_status) */
#define ENTMAX_ST_NOT_CONVERGED 1u /* some row's sum of p is off 1 by more than 1e-3 */
#define ENTMAX_ST_TIMEOUT       2u /* a bounded wait gave up; outputs are not valid   */
#define ENTMAX_ST_RANGE         4u /* |s| * 8 reached 2^21 somewhere: histogram inexact */
#define ENTMAX_ST_BOUNDS        8u /* bounds-checked build (-DENTMAX_BOUNDS_CHECK) only: an
                                      index fell outside its buffer; that access was skipped */

#define ENTMAX_MAX_N    262144
#define ENTMAX_MAX_ITER 16
#define ENTMAX_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * Number of uint32 words per row block of the block mask: ceil(ceil(N/block)/32).
 * Returns a negative error code for unsupported N or block.
 */
int entmax_attn_mask_words(int N, int block);

/*
 * Bytes of device workspace that entmax_attn_fwd and entmax_attn_bwd need for
 * this problem (the same buffer serves both, and carries data from the bf16
 * forward to its backward).  It holds the status word and work counters, the
 * per-(row, key tile) score maxima of the histogram pass (fp16, rounded up),
 * the tile-granularity mask and its transpose, the per-row delta of the
 * backward, the forward's per-row g-weighted means of v (float32, B*H*N*D)
 * and fp16 copies of q, k, v and dout (v's made by the forward).
 * Returns 0 for unsupported arguments.
 */
size_t entmax_attn_workspace_size(int B, int H, int N, int D, int block, int causal);

/*
 * Forward pass.  AdaSplash-2 zh §2.1 (histogram initialisation), §2.2 (hybrid
 * solver, one or two iterations), §2.3 (bit-packed block mask, zero-block
 * skipping); it §2A-2C; ja §2.1-2.3; es §2A-2C.
 *
 *   q, k, v      in   [B][H][N][D], dtype.
 *   alpha        in   in [1.05, 3].  1.5 and 2.0 use closed forms (p = t^2, p = t)
 *                     and certified-exact Halley / Newton steps; any other alpha
 *                     computes p = t^(1/(alpha-1)) with the special-function unit
 *                     (relative error about 1e-6) and takes Halley (alpha < 1.5)
 *                     or Newton steps, bisection-safeguarded, until f is within
 *                     1e-4 and the step below 1e-6 max(1, |tau|) (zh §2.2,
 *                     es §2B); give it a max_iter of about 12.  Beyond alpha = 3
 *                     a float32 tau cannot hold the outputs to 2e-2: p = t^k has
 *                     an unbounded slope where a score enters the support.  For
 *                     alpha > 2, g = p^(2-alpha) also grows without bound there:
 *                     the forward holds g below 6e4 in the G.V product, and
 *                     entmax_attn_bwd rejects alpha > 2.
 *   causal       in   nonzero: key c is visible to query r iff c <= r.
 *   block        in   block size of the mask (64 or 128), rows and keys alike.
 *   max_iter     in   at most this many refinement passes after the histogram
 *                     bound (0..ENTMAX_MAX_ITER).  A row stops once its threshold is
 *                     certified exact -- the step did not cross any score of
 *                     the current support, so the closed-form root on that
 *                     support is tau* -- and a 128-row tile stops once all of
 *                     its rows have; the summaries report 1, at most 2,
 *                     iterations (zh §2.2), 4 is a safe cap.
 *   out          out  [B][H][N][D], dtype.
 *   tau          out  float32 [B][H][N], s-units.
 *   mask         out  uint32 [B][H][ceil(N/block)][W], bit set iff the block
 *                     holds a non-zero probability (at the final tau).
 *   tau_trace    out  optional (NULL = off): float32 [max_iter+1][B][H][N];
 *                     entry 0 is the histogram bound tau_h, entry i the
 *                     threshold after refinement step i.
 *   workspace    in/out  device buffer of >= entmax_attn_workspace_size() bytes,
 *                     256-byte aligned; its status word is cleared here.  For
 *                     bf16 the forward also leaves there what its backward
 *                     reads: an exact fp16 copy of v (the P.V products run on
 *                     it; a v entry beyond the fp16 range raises
 *                     ENTMAX_ST_RANGE) and, per row, the g-weighted mean of v,
 *                     vbar_r = sum_c g_rc v_c / sum_c g_rc with g = p^(2-alpha),
 *                     formed by one more MMA next to P.V.
 */
int entmax_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int D,
                    int dtype, float alpha, int causal, int block, int max_iter, void* out,
                    float* tau, uint32_t* mask, float* tau_trace, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Forward pass without a workspace argument, for callers that cannot obtain
 * device memory at call time: code that runs where cudaMalloc is unavailable
 * or forbidden (inside a host callback or another library's critical section,
 * under an allocator that must not grow, or in a plain C program that owns no
 * allocator).  The paper has no counterpart to this entry point; it exists
 * only for such callers.
 *
 * It runs the bf16 kernel of entmax_attn_fwd with the same arguments and
 * outputs (no tau_trace; dtype must be ENTMAX_DTYPE_BF16, fp32 returns
 * ENTMAX_E_UNSUPPORTED): tau and the mask are the same, and O differs only in the
 * rounding of P, which is bf16 here (it multiplies v itself, as no fp16 copy
 * of v fits the scratch) instead of fp16.  It forms no g-weighted means, so
 * entmax_attn_bwd cannot follow it.  Its scratch -- status word, work counters
 * and the histogram pass's tile maxima -- lives in one fixed device array of
 * ENTMAX_NOALLOC_SCRATCH_BYTES (8 MiB) that is part of this library:
 * every GPU that loads the library holds those 8 MiB until the process exits.
 * The call allocates nothing and calls no allocating routine.
 *   - Problems whose scratch exceeds the 8 MiB return ENTMAX_E_SCRATCH and
 *     launch nothing (causal: 256 + B*H*T*(T+1)/2*512 bytes, T = ceil(N/128);
 *     e.g. B*H = 16 at N = 4096 needs 4.3 MB).
 *   - The array's device address is looked up (cudaGetSymbolAddress) on the
 *     first call made while a device is current, and looked up again when
 *     that device's context has changed since (after cudaDeviceReset).  With
 *     CUDA's lazy module loading (the default) that first lookup may also load
 *     the library's device code, which is when the driver places the 8 MiB
 *     array in device memory: a caller that must see no device allocation at
 *     all during its critical section makes one call (a tiny problem will do)
 *     during its set-up, and makes the first call on a device before any
 *     stream capture on it.
 *   - All calls on a device share the one array, which keeps the previous
 *     call's contents; the call clears the parts that must start at zero.
 *     Calls whose kernels may overlap on the GPU (other streams, other host
 *     threads) race on the array: serialise them.
 *   - The device status word (ENTMAX_ST_* bits) stays in the array;
 *     entmax_attn_noalloc_status reads it.
 */
int entmax_attn_fwd_noalloc(const void* q, const void* k, const void* v, int B, int H, int N,
                            int D, int dtype, float alpha, int causal, int block, int max_iter,
                            void* out, float* tau, uint32_t* mask, void* stream);

/*
 * Status of the last entmax_attn_fwd_noalloc on the current device (no
 * counterpart on the pages; it belongs to the no-alloc entry point above):
 * synchronises `stream`, then copies the status word of the fixed scratch
 * array (ENTMAX_ST_* bits, cleared by each entmax_attn_fwd_noalloc call) to
 * *status.  Allocates nothing.  Returns ENTMAX_E_CUDA if the stream reported
 * an error.  Only meaningful once the calls it should cover were enqueued on
 * `stream` (or have finished): a later call on the device clears the word.
 */
int entmax_attn_noalloc_status(void* stream, uint32_t* status);

/*
 * Backward pass over the forward's mask (zh §2.3 and ja §2.3: zero blocks are
 * skipped in the backward as well; ja §2.3: local accumulators instead of
 * atomics).  With g = p^(2-alpha) on the support:
 *     dP = dO V^T,  delta_r = sum_c g dP / sum_c g,  dZ = g (dP - delta)
 *     dQ = dZ K / sqrt(D),  dK = dZ^T Q / sqrt(D),  dV = P^T dO
 *
 *   q, k, v, dout  in  [B][H][N][D], dtype.
 *   tau, mask      in  exactly as written by entmax_attn_fwd for these inputs.
 *   alpha, causal, block   as given to entmax_attn_fwd; alpha in [1.05, 2]
 *                  (ENTMAX_E_ALPHA beyond: g = p^(2-alpha) is unbounded at the
 *                  edge of the support, where float32 scores cannot hold the
 *                  gradients to the bf16 tolerance -- 0.14 on dQ at alpha = 3).
 *   dq, dk, dv     out [B][H][N][D], dtype (fully overwritten).
 *   workspace      in/out  the same size rule as for the forward; status bits
 *                  are OR-ed into the existing status word.  bf16: the
 *                  workspace the forward of these same inputs wrote, unchanged
 *                  since (delta_r = dO_r . vbar_r uses its g-weighted means of
 *                  v, the MMAs its fp16 copy of v); anything else gives
 *                  undefined gradients.  fp32 computes delta in a pass of its
 *                  own and needs no forward data.
 * The backward's MMAs run on exact fp16 copies of the bf16 inputs, so that
 * the operands rounded on chip (P and dS) keep 11 significant bits; an input
 * of magnitude above 65504 (outside fp16) raises ENTMAX_ST_RANGE.
 */
int entmax_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* tau, const uint32_t* mask, int B, int H, int N, int D,
                    int dtype, float alpha, int causal, int block, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Diagnostics of the failure handling (the pages have no counterpart): runs a
 * one-thread kernel that waits on an mbarrier nothing ever arrives at, with a
 * limit of limit_ns nanoseconds (1..10^9) instead of the kernels' 2 s, so the
 * bounded wait runs out: it raises ENTMAX_ST_TIMEOUT in `workspace`'s status
 * word (cleared first) and the kernel returns.  result: device uint32[3],
 * written [1 = returned, 1 = the wait succeeded, 1 = abort flag raised].  No
 * fault, trap or unbounded loop is involved; the context stays usable.
 */
int entmax_attn_wait_selftest(void* workspace, uint32_t* result, unsigned long long limit_ns,
                              void* stream);

/*
 * Synchronises `stream` and copies the device status word (ENTMAX_ST_* bits)
 * of `workspace` to *status.  Returns ENTMAX_E_CUDA if the stream reported an
 * error (e.g. from an earlier launch).
 */
int entmax_attn_status(const void* workspace, void* stream, uint32_t* status);

/*
 * Diagnostics: copies the first n (1..8) work counters of `workspace` to
 * counters[] after synchronising `stream`.  [0] key tiles visited by the
 * forward's histogram pass, [1] by its tile refinement passes, [2] by its P.V
 * pass, [3] tile refinement passes summed over 128-row tiles, [4] active key
 * tiles per pass of the backward row kernel, [5] active query tiles of the
 * backward column kernel, [6] 128-row tiles whose candidate lists overflowed
 * (and which therefore refined by streaming the key tiles again); tiles are
 * 128 x 128.  Cleared by entmax_attn_fwd ([0]-[3], [6]) and entmax_attn_bwd
 * ([4]-[5]).
 */
int entmax_attn_counters(const void* workspace, void* stream, unsigned long long* counters, int n);

/*
 * Profiling aid, off by default and per calling thread.  entmax_attn_profile(1)
 * makes the thread's later fwd/bwd calls record CUDA events on their stream
 * around each kernel (it creates the events once; no memory is allocated);
 * entmax_attn_profile(0) stops recording.  entmax_attn_profile_read() waits for
 * the last recorded events and writes up to 5 durations in ms: [0] forward
 * kernel, [1] backward fp16 operand copies, [2] backward tile-mask preparation,
 * [3] backward row kernel (delta, dQ), [4] backward column kernel (dK, dV).
 */
int entmax_attn_profile(int enable);
int entmax_attn_profile_read(float* ms, int n);

/* Static, human-readable text for a return code. */
const char* entmax_attn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAX_ATTN_H */
