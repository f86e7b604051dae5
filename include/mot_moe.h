/*
 * mot_moe.h -- C ABI of the A3B gen-tower mixture-of-experts MLP on B200
 * (sm_100a).
 *
 *   "SenseNova-U1" (vLLM-Omni recipe), A3B (MoE) variant: a Qwen3-MoE
 *     backbone whose generation branch (mlp_mot_gen) routes over 32 experts,
 *     top-8, per-expert width moe_intermediate_size = 768; measured kernel
 *     table: fused_moe_kernel (top-8 expert GEMMs, 48% of the denoise step),
 *     MoE routing (top-k), act_and_mul.
 *
 * For each token x [d] (the already-normalised hidden state):
 *   p = softmax(x W_r^T) over the E experts; the top_k experts i_k by p
 *   (ties to the lower index) with weights w_k = p_{i_k} / sum_k p_{i_k};
 *   y = sum_k w_k (silu(x Wg_{i_k}^T) * (x Wu_{i_k}^T)) Wd_{i_k}^T
 * (k in rank order). Inference only, no adapters. Conventions as mot_attn.h.
 */
#ifndef MOT_MOE_H
#define MOT_MOE_H

#include <stddef.h>
#include <stdint.h>

#include "mot_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mot_moe* mot_moe_t; /* opaque handle */

/* Supported: hidden % 256 == 0, intermediate % 128 == 0, 1 <= experts <= 32,
 * 1 <= top_k <= min(8, experts). */
typedef struct {
  int32_t hidden;        /* d (2048 for the A3B tower)                 */
  int32_t intermediate;  /* expert width I (768)                       */
  int32_t experts;       /* E (32)                                     */
  int32_t top_k;         /* experts per token (8)                      */
  int32_t max_tokens;    /* largest T per call                         */
} mot_moe_config;

/* Weights, device bf16 (kept by pointer, unchanged while the handle lives):
 *   w_router [E, d]; w_gate, w_up [E, I, d]; w_down [E, d, I]
 * (each expert's nn.Linear weight, the experts stacked in the first axis). */
typedef struct {
  const void *w_router, *w_gate, *w_up, *w_down;
} mot_moe_weights;

/* Device workspace bytes of a call over `tokens` tokens. Host-only. */
mot_status mot_moe_query_workspace(const mot_moe_config* cfg, int32_t tokens, size_t* workspace_bytes);

/* Create: validates, makes the f16 copy of w_down (it meets the f16 expert
 * activations), the router GEMM's split-K scratch and the tensor maps. */
mot_status mot_moe_create(const mot_moe_config* cfg, const mot_moe_weights* weights, void* stream,
                          mot_moe_t* out);

/* Forward.
 *   x       device bf16 [T, d]
 *   y       device bf16 [T, d]; y_f32 device f32 [T, d] or NULL (y == RNE_bf16(y_f32))
 *   experts_out  device int32 [T, top_k] or NULL: the chosen experts per
 *           token in rank order (for checks of the routing)
 *   workspace device, workspace_bytes from mot_moe_query_workspace
 * The expert GEMMs run on M tiles of 256 rows of one expert each; their
 * count depends on the routing and is bounded by ceil(T top_k / 256) + E.
 * The experts' activations h and outputs are kept in f16 between the
 * kernels; an overflow there is latched as MOT_ERR_NUMERIC and reported by
 * mot_moe_get_device_status. */
mot_status mot_moe_forward(mot_moe_t h, const void* x, int32_t tokens, void* y, float* y_f32, int32_t* experts_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, return and clear the latched device status. */
mot_status mot_moe_get_device_status(mot_moe_t h, void* stream);

/* Free the handle. NULL is ignored. */
void mot_moe_destroy(mot_moe_t h);

#ifdef __cplusplus
}
#endif

#endif /* MOT_MOE_H */
