/*
 * mot_attn_dev.h -- kernel-level entry points of the same library, for tests
 * that check one stage of the layer at a time. Same conventions as
 * mot_attn.h (device/host pointers, 16-byte alignment, stream = cudaStream_t,
 * host-side validation, no exceptions across the ABI).
 */
#ifndef MOT_ATTN_DEV_H
#define MOT_ATTN_DEV_H

#include <stddef.h>
#include <stdint.h>

#include "mot_attn.h"
#include "mot_mlp.h"

#ifdef __cplusplus
extern "C" {
#endif

/* d = A B^T on the tensor cores (the persistent tcgen05 GEMM used by the
 * layer's projections): a device [m, k], b device [n, k], both bf16
 * (is_bf16 != 0) or both f16; d device f32 [m, n]; output tiles 128 x tile_n
 * (tile_n 128 or 256). Requires k % 64 == 0, n % tile_n == 0, m >= 1. */
mot_status mot_dev_gemm(const void* a, const void* b, float* d, int32_t m, int32_t n, int32_t k,
                        int32_t is_bf16, int32_t tile_n, void* stream);

/* The other GEMM building blocks on the same operands (A [m, k], B and B2
 * [n, k], K-major, f16 or bf16; D = f32 [m, n]):
 *   variant 1: CTA pairs (cluster of 2, cta_group::2), 256 x 256 tiles;
 *              n a multiple of 256.
 *   variant 2: 128 x 64 tiles with split-K (f32 partial tiles summed in split
 *              order by the CTA that completes a tile last); n == 64.
 *   variant 3: as 2, with B2 as a second B operand of every A tile:
 *              D = A B^T + A B2^T; n == 64.
 *   variant 4: as 1, with B given transposed, [k, n] row-major (loaded as an
 *              MN-major operand): D = A B.
 * k a multiple of 64. Variants 2 and 3 allocate their split scratch and
 * synchronize `stream` before returning (test entry). */
mot_status mot_dev_gemm_variant(const void* a, const void* b, const void* b2, float* d, int32_t m, int32_t n,
                                int32_t k, int32_t is_bf16, int32_t variant, void* stream);

/* Byte offsets, inside the `saved` buffer of a training forward, of the
 * activations it keeps (all device, f16 unless noted):
 *   [0] q^      [B, Hq, N, dh]      normalised + rotated queries
 *   [1] K       [B, Hkv, Lcap, dh]  keys: prefix rows then self rows
 *   [2] V       [B, Hkv, Lcap, dh]
 *   [3] o       [B*N, Hq*dh]        attention output (o_proj input)
 *   [4] lse     f32 [B, Hq, N]      natural-log softmax normaliser
 *   [5] xhat    [B*N, (Hq+Hkv)*dh]  normalised pre-gain q/k
 *   [6] rstd    f32 [B*N, Hq+Hkv]
 *   [7] u_qkv   [B*N, 3*RP]         s x A^T per q/k/v (RP = rank rounded up to 64)
 *   [8] u_o     [B*N, RP]           s o A_o^T
 * lcap receives Lcap = round_up(P_max + N, 128). */
mot_status mot_dev_saved_layout(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens,
                                int32_t prefix_max, size_t offsets[9], int32_t* lcap);

/* Per-stage device timing. enable != 0: every later forward/backward call
 * records a CUDA event on its stream before its first launch and after each
 * launch (no synchronisation is added). mot_dev_stage_times waits for the
 * last call's final event and writes, for each launch of that call in order,
 * its stage id and its duration in milliseconds (at most `max` entries;
 * *count receives the number of launches). */
mot_status mot_dev_profile(mot_attn_t h, int32_t enable);
mot_status mot_dev_stage_times(mot_attn_t h, int32_t* ids, float* ms, int32_t max, int32_t* count);

/* The same launches placed on one clock: t0_ms[i] / t1_ms[i] are the times
 * of launch i's start and end events, in milliseconds after the first
 * launch's start event. Side-stream launches (the backward's LoRA gradients)
 * start at the side stream's own previous event, so overlap between the two
 * streams shows as intersecting intervals. Same argument rules as
 * mot_dev_stage_times. */
mot_status mot_dev_stage_timeline(mot_attn_t h, int32_t* ids, float* t0_ms, float* t1_ms, int32_t max,
                                  int32_t* count);

/* y[i] = 2^x[i] through the FMA-pipe exponential the attention softmax uses
 * for part of its probabilities (range reduction + degree-3 polynomial);
 * x, y device f32 [n], n even, x in [-125, 8]. For accuracy tests. */
mot_status mot_dev_exp2_poly(const float* x, float* y, int32_t n, void* stream);

/* Failure-detection check: enqueue on `stream` one kernel whose single wait
 * is on a barrier nothing ever completes, through the bounded wait all the
 * kernels use. The wait gives up after its limit (2 s), latches the timeout
 * in the handle's device status and the kernel exits normally, so the next
 * mot_attn_get_device_status returns MOT_ERR_TIMEOUT and the handle and the
 * context stay usable. For tests. */
mot_status mot_dev_wait_probe(mot_attn_t h, void* stream);

/* Split-KV count of the attention forward. The work is one unit per
 * (branch, query head, pair of 128-query tiles). splits == 0 (the default):
 * each forward plans from the call's shape (key tiles per branch, units, how
 * many clusters of S CTAs fit on the GPU at once): the units that fill whole
 * waves of one CTA per SM run unsplit, and the units of a partly empty last
 * wave may run split S ways in a second launch. splits in 1..8: every unit
 * of every later forward cuts its keys into exactly that many contiguous
 * ranges of whole 128-key tiles, one CTA each, merged in split order
 * (MOT_ERR_UNSUPPORTED_SHAPE from a forward whose shortest branch has fewer
 * 128-key tiles than splits; from this call if clusters of that size cannot
 * be resident). For tests and measurements. */
mot_status mot_dev_set_attn_splits(mot_attn_t h, int32_t splits);

/* Split count of the split units of the last forward (1 if none was split;
 * 0 before any forward), and how many units it ran unsplit ahead of them. */
int32_t mot_dev_last_attn_splits(mot_attn_t h);
int32_t mot_dev_last_attn_full_units(mot_attn_t h);

/* Static name of a stage id ("qkv_gemm", "attn_fwd", ...; "?" if unknown). */
const char* mot_dev_stage_name(int32_t id);

/* The same per-launch timing for an MLP handle (mot_mlp.h): enable, then
 * the last call's launches with their stage ids and durations (ms), and the
 * stage names ("mlp_gate_up", "mlp_down", ...). Same rules as
 * mot_dev_profile / mot_dev_stage_times. */
mot_status mot_dev_mlp_profile(mot_mlp_t h, int32_t enable);
mot_status mot_dev_mlp_stage_times(mot_mlp_t h, int32_t* ids, float* ms, int32_t max, int32_t* count);
const char* mot_dev_mlp_stage_name(int32_t id);

#ifdef __cplusplus
}
#endif

#endif /* MOT_ATTN_DEV_H */
