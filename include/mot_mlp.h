/*
 * mot_mlp.h -- C ABI of the B200 (sm_100a) gen-tower SwiGLU MLP with LoRA.
 *
 * The MLP half of one generation-tower (`*_mot_gen`) decoder layer of the
 * Mixture-of-Transformers image model, the block that follows the attention
 * half of include/mot_attn.h:
 *
 *   "SenseNova-U1" (DiffSynth-Studio docs), training section: the LoRA
 *     targets of the generation branch include mlp_mot_gen.gate_proj,
 *     mlp_mot_gen.up_proj and mlp_mot_gen.down_proj.
 *   "SenseNova-U1" (vLLM-Omni recipe), measured kernel table: an
 *     act_and_mul (SwiGLU) step between the fused gate/up projection and
 *     down_proj.
 *
 * Per token x [d] (s = lora_alpha / lora_rank):
 *   g = x Wg^T + s (x Ag^T) Bg^T,   u = x Wu^T + s (x Au^T) Bu^T   [I]
 *   h = silu(g) * u,                silu(z) = z / (1 + e^-z)
 *   y = h Wd^T + s (h Ad^T) Bd^T                                   [d]
 * The gate is the activated half (the act_and_mul convention). x is the
 * already-normalised hidden state; y is the down_proj output (no residual).
 *
 * Conventions are those of mot_attn.h: "device" pointers are CUDA device
 * memory, "host" pointers plain host memory read before the call returns;
 * dense row-major tensors, 16-byte aligned (MOT_ERR_ALIGNMENT otherwise);
 * `stream` is a cudaStream_t; host validation before anything is enqueued;
 * device-detected f16 overflow or an expired bounded wait is latched in the
 * handle and returned by mot_mlp_get_device_status; the caller owns every
 * buffer it passes; a handle is used from one stream at a time.
 */
#ifndef MOT_MLP_H
#define MOT_MLP_H

#include <stddef.h>
#include <stdint.h>

#include "mot_attn.h" /* mot_status */

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mot_mlp* mot_mlp_t; /* opaque handle */

/* Supported: hidden % 256 == 0, intermediate % 128 == 0, lora_rank in
 * {0, 8, ..., 128} (a multiple of 8). */
typedef struct {
  int32_t hidden;          /* d (4096)                                        */
  int32_t intermediate;    /* I (12288)                                       */
  int32_t lora_rank;       /* r; 0 = no adapters                              */
  float lora_alpha;        /* alpha; s = alpha / r                            */
  int32_t max_tokens;      /* largest T (all CFG branches' image tokens) per call */
  int32_t enable_backward; /* nonzero: build what mot_mlp_backward needs      */
} mot_mlp_config;

/* Weights, device bf16, nn.Linear layout [out, in]; the handle keeps the
 * pointers (LoRA tensors may change in place between calls, base weights
 * may not) and makes f16 / transposed copies of the base weights at create.
 *   w_gate, w_up [I, d], w_down [d, I]
 *   a_gate, a_up [r, d], a_down [r, I]          (lora_down; NULL if r == 0)
 *   b_gate, b_up [I, r], b_down [d, r]          (lora_up) */
typedef struct {
  const void *w_gate, *w_up, *w_down;
  const void *a_gate, *a_up, *a_down;
  const void *b_gate, *b_up, *b_down;
} mot_mlp_weights;

/* Device bytes a call over `tokens` tokens needs: workspace (scratch of
 * forward and backward) and saved (activations a training forward keeps for
 * backward). Either pointer may be NULL. Host-only. */
mot_status mot_mlp_query_sizes(const mot_mlp_config* cfg, int32_t tokens, size_t* workspace_bytes,
                               size_t* saved_bytes);

/* Create a handle: validates cfg and the weights, allocates the f16 copy of
 * w_down (it meets the f16 h), split-K scratch for the LoRA-down GEMMs and,
 * with enable_backward, the transposed copies the backward GEMMs read
 * (w_down^T bf16, w_gate^T and w_up^T f16) and a side stream. */
mot_status mot_mlp_create(const mot_mlp_config* cfg, const mot_mlp_weights* weights, void* stream,
                          mot_mlp_t* out);

/* Forward.
 *   x      device bf16 [T, d]
 *   y      device bf16 [T, d];  y_f32 device f32 [T, d] or NULL
 *          (y == RNE_bf16(y_f32) bit for bit)
 *   saved  device, saved_bytes from query_sizes, or NULL for inference
 *   workspace device, workspace_bytes from query_sizes
 * 1 <= T <= max_tokens. */
mot_status mot_mlp_forward(mot_mlp_t h, const void* x, int32_t tokens, void* y, float* y_f32, void* saved,
                           size_t saved_bytes, void* workspace, size_t workspace_bytes, void* stream);

/* LoRA-training backward (base weights frozen).
 *   dy     device bf16 [T, d]; x as passed to the forward; saved: its buffer
 *   dx     device bf16 [T, d]; dx_f32 device f32 [T, d] or NULL
 *   d_a[3], d_b[3]  device f32, gate/up/down order, shapes of a_* / b_*;
 *          accumulate != 0 adds into them. All NULL allowed when r == 0.
 * Deterministic. Requires enable_backward. Like mot_attn_backward, the
 * LoRA-gradient GEMMs that feed nothing later run on the handle's second
 * stream, joined back into `stream` before the call returns. */
mot_status mot_mlp_backward(mot_mlp_t h, const void* dy, const void* x, int32_t tokens, const void* saved,
                            size_t saved_bytes, void* dx, float* dx_f32, float* const d_a[3],
                            float* const d_b[3], int32_t accumulate, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Synchronise `stream`, return and clear the latched device status
 * (MOT_OK, MOT_ERR_NUMERIC or MOT_ERR_TIMEOUT). */
mot_status mot_mlp_get_device_status(mot_mlp_t h, void* stream);

/* Number of kernels the last forward / backward enqueued. */
int32_t mot_mlp_last_launch_count(mot_mlp_t h);

/* Free the handle's own device memory. NULL is ignored. */
void mot_mlp_destroy(mot_mlp_t h);

#ifdef __cplusplus
}
#endif

#endif /* MOT_MLP_H */
