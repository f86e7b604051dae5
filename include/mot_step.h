/*
 * mot_step.h -- C ABI of one gen-tower flow-matching denoise step on B200
 * (sm_100a): the stack of generation-tower decoder layers (mot_attn.h
 * attention halves and mot_mlp.h MLP halves, each behind a pre-norm
 * residual) over the image tokens of a CFG batch, the flow head, the
 * guidance combine and the Euler update.
 *
 *   "SenseNova-U1" (DiffSynth-Studio docs), inference parameters: 50 steps,
 *     cfg_scale 4.0 with a fixed unconditional branch, shift 3.0, 32-pixel
 *     patches, pixel space (no VAE); architecture note: 42 decoder layers.
 *   "SenseNova-U1" (vLLM-Omni recipe), measured case: 50 Euler steps,
 *     cfg_norm none, timestep_shift 3.0, t_eps 0.02; image editing with dual
 *     CFG (img_cfg_scale) over three branches.
 *   "Setup notes" (LoRA trainer docs), default training config: x0 loss, a
 *     timestep/noise embedder, an fm_head.
 *
 * One step for one image (z: its N patch tokens of C = 3 * 32 * 32 pixel
 * values at noise level sigma) and B branches (1: cond; 2: cond, uncond;
 * 3: cond, image-cond, uncond), each with its prefix caches:
 *   h0 = z W_in^T + e(sigma)     e: cos / sin of 1000 sigma 10000^(-k/(d/2))
 *   for each layer l: h += Attn_l(RMSNorm(h) g_in[l]); h += MLP_l(RMSNorm(h) g_post[l])
 *   x0_b = (RMSNorm(h_b) g_out) W_out^T                  (the head predicts x0)
 *   x0 = x0_u + cfg (x0_c - x0_u)                        (B = 2; B = 3:
 *        x0_u + img_cfg (x0_i - x0_u) + cfg (x0_c - x0_i); B = 1: x0_c)
 *   z_next = z + (sigma_next - sigma) (z - x0) / max(sigma, t_eps)
 * The residual stream h is kept in f32; the layers' inputs are bf16.
 * Conventions as mot_attn.h. Device-detected conditions of the layers are
 * latched in their handles; the step's own embedding and head GEMMs latch
 * theirs in the first layer's attention handle (mot_attn_get_device_status
 * of attn[0]).
 */
#ifndef MOT_STEP_H
#define MOT_STEP_H

#include <stddef.h>
#include <stdint.h>

#include "mot_attn.h"
#include "mot_mlp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mot_step* mot_step_t; /* opaque handle */

typedef struct {
  int32_t n_layers;   /* decoder layers (42)                               */
  int32_t hidden;     /* d (4096), the attention and MLP handles' hidden    */
  int32_t patch_dim;  /* C (3 * 32 * 32 = 3072); a multiple of 256          */
  float rms_eps;      /* decoder-layer RMSNorm epsilon (1e-6)               */
} mot_step_config;

/* The tower. Handles are the caller's (made with mot_attn_create /
 * mot_mlp_create for each layer; they must outlive the step handle); the
 * arrays are read at create and may be freed afterwards. Weights: device
 * bf16, kept by pointer (unchanged while the handle lives).
 *   attn[n_layers], mlp[n_layers]
 *   norm_in[n_layers], norm_post[n_layers]   [d] each
 *   w_in [d, C], norm_out [d], w_out [C, d] */
typedef struct {
  const mot_attn_t* attn;
  const mot_mlp_t* mlp;
  const void* const* norm_in;
  const void* const* norm_post;
  const void* w_in;
  const void* norm_out;
  const void* w_out;
} mot_step_model;

/* Create: validates (hidden % 256 == 0, patch_dim % 256 == 0, n_layers >= 1)
 * and makes the f32 copies of the norm gains and the weight tensor maps. */
mot_status mot_step_create(const mot_step_config* cfg, const mot_step_model* model, void* stream,
                           mot_step_t* out);

/* Device workspace bytes of mot_step_forward for B branches of N tokens
 * over P_max cached prefix keys (host-only, reads the layer handles'
 * configurations). */
mot_status mot_step_query_workspace(mot_step_t h, int32_t batch, int32_t img_tokens, int32_t prefix_max,
                                    size_t* workspace_bytes);

/* One step.
 *   z          device f32 [N, C]    the image's patch tokens at sigma
 *   k_cache[l], v_cache[l]          device bf16 [B, Hkv, P_max, dh], layer l's
 *                                   prefix cache (as mot_attn_forward)
 *   prefix_len host int32 [B]
 *   z_next     device f32 [N, C]    (may alias z)
 *   z_next_bf16 device bf16 [N, C] or NULL: the same, rounded
 * Every layer handle must accept (B, N, P_max) (mot_attn_forward's rules)
 * and B * N tokens (mot_mlp_forward's). */
mot_status mot_step_forward(mot_step_t h, const float* z, int32_t batch, int32_t img_tokens,
                            const void* const* k_cache, const void* const* v_cache, const int32_t* prefix_len,
                            int32_t prefix_max, float sigma, float sigma_next, float cfg_scale,
                            float img_cfg_scale, float t_eps, float* z_next, void* z_next_bf16, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Free the handle (not the layer handles). NULL is ignored. */
void mot_step_destroy(mot_step_t h);

#ifdef __cplusplus
}
#endif

#endif /* MOT_STEP_H */
