/*
 * dash_route.h -- C ABI of the DashAttention stage-0/1 entmax router (sm_100a).
 *
 * The Italian summary of DashAttention (gist.science/it/paper/2605.18753), which
 * the AdaSplash-2 pages carry, replaces top-k chunk routing with alpha-entmax:
 *   stage 0 ("Riassunto Locale dei Chunk"): every complete chunk of `chunk`
 *     keys gets a summary by local attention with a learned query qbar; at its
 *     initial value qbar = 0 the attention is uniform and the summary is the
 *     mean of the chunk's keys -- the form computed here;
 *   stage 1 ("Routing dei Chunk con Entmax"): per query, w = alpha-entmax(gamma
 *     zbar) over the chunk summaries, zbar = q . kbar / sqrt(D) (the scaling of
 *     the attention itself; the summary gives no formula), over the complete
 *     chunks before the query's own: chunk c is visible to row r iff
 *     c < floor(r / chunk) (the own chunk has no summary yet and belongs to the
 *     diagonal branch of stage 2);
 *   GQA ("Gestione GQA"): the probabilities of the query heads that share a KV
 *     head are averaged, wbar = mean over the group, one sparse support per KV
 *     head.
 * Stage 2 (prior-induced sparse softmax) and the backward are not provided.
 *
 * Conventions are those of entmax_attn.h (device pointers owned by the caller,
 * asynchronous on `stream`, arguments checked before any launch, ENTMAX_*
 * return codes, device conditions OR-ed into the status word at the start of
 * the workspace -- read it with entmax_attn_status).
 */
#ifndef DASH_ROUTE_H
#define DASH_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#include "entmax_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Most complete chunks a problem may have (N / chunk): the logits and the
 * GQA accumulator of a 128-row tile share the 512 columns of tensor memory. */
#define DASH_MAX_CHUNKS 256

/*
 * Bytes of device workspace for dash_route_fwd: status word (256 B), the chunk
 * summaries as two fp16 parts, hi + lo, [2][B*Hkv][Cp][D] (Cp = C rounded up to
 * a multiple of 128, C = N / chunk; the logits take one MMA per part, so they
 * keep fp32 accuracy), and an exact fp16 copy of q [B*Hq][N][D].  0 for
 * unsupported arguments.
 */
size_t dash_route_workspace_size(int B, int Hq, int Hkv, int N, int D, int chunk);

/*
 * Stages 0 and 1 with the GQA average.
 *   q           in   [B][Hq][N][D] bf16; query head h belongs to KV head h / (Hq / Hkv).
 *   k           in   [B][Hkv][N][D] bf16.
 *   chunk       in   chunk size, >= 1, with C = N / chunk <= DASH_MAX_CHUNKS
 *                    (a trailing partial chunk has no summary).
 *   gamma       in   > 0, the router's logit scale.
 *   alpha       in   [1.05, 3] as for entmax_attn_fwd (closed forms at 1.5 and 2).
 *   max_iter    in   cap on the threshold steps per row (0..ENTMAX_MAX_ITER);
 *                    rows stop once certified exact (closed forms) or converged.
 *   wbar        out  float32 [B][Hkv][N][C]: the averaged routing
 *                    probabilities; rows with no visible chunk are all zero.
 *   row_mask    out  uint32 [B][Hkv][N][W], W = ceil(C / 32): bit (c % 32) of
 *                    word c / 32 set iff wbar > 0 (least significant bit = lowest
 *                    chunk).
 *   block_mask  out  uint32 [B][Hkv][ceil(N / 128)][W]: the OR of row_mask over
 *                    each 128-row query block, the form a kernel that walks
 *                    active chunks per query tile reads.
 *   workspace   in/out  >= dash_route_workspace_size() bytes, 256-byte aligned;
 *                    its status word is cleared here.  ENTMAX_ST_NOT_CONVERGED
 *                    marks a row whose probabilities do not sum to 1 within 1e-3
 *                    per query head; q or k entries beyond the fp16 range raise
 *                    ENTMAX_ST_RANGE.
 * Returns ENTMAX_OK, or ENTMAX_E_NULL / _ALIGN (q, k 16-byte, outputs 4-byte,
 * workspace 256-byte) / _SHAPE (B, Hq, Hkv, N, chunk, Hq % Hkv, C) /
 * _UNSUPPORTED (D not 64 or 128) / _ALPHA / _MAXITER / _WORKSPACE / _CUDA.
 * With C = 0 (N < chunk) the outputs are empty (their pointers may be NULL)
 * and nothing is launched.
 */
int dash_route_fwd(const void* q, const void* k, int B, int Hq, int Hkv, int N, int D, int chunk,
                   float gamma, float alpha, int max_iter, float* wbar, uint32_t* row_mask,
                   uint32_t* block_mask, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DASH_ROUTE_H */
