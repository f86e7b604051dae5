/*
 * mot_attn.h -- C ABI of the B200 (sm_100a) gen-tower attention layer.
 *
 * The layer is the attention half of one generation-tower (`*_mot_gen`)
 * decoder layer of a Mixture-of-Transformers unified image model during a
 * pixel-space flow-matching denoise step:
 *
 *   "SenseNova-U1" (DiffSynth-Studio docs), architecture note: each of the
 *     42 decoder layers holds an understanding and a generation weight set;
 *     the prompt is encoded once by the understanding branch into
 *     past_key_values, and at each denoise step the image tokens go through
 *     the generation branch and attend to that cache.
 *   "Setup notes" (LoRA trainer docs), "Why bf16 base on CPU + tower
 *     offload?": a static prefix-KV cache is computed once; the gen tower
 *     carries LoRA adapters; the base stays bf16.
 *   "SenseNova-U1" (DiffSynth-Studio docs), training section: LoRA targets
 *     q_proj_mot_gen, k_proj_mot_gen, v_proj_mot_gen, o_proj_mot_gen.
 *   "SenseNova-U1" (vLLM-Omni recipe), measured kernel table: attention in a
 *     flash kernel, q/k through a fused RMSNorm + RoPE kernel.
 *
 * Per CFG branch b (image tokens x_b [N, hidden], P_b = prefix_len[b]):
 *   q = x Wq^T + s (x Aq^T) Bq^T   (likewise k, v; s = lora_alpha / lora_rank)
 *   q^ = RoPE_p(RMSNorm_head(q) * q_norm), k^ likewise with k_norm,
 *        position of image token i is p = P_b + i (rotate-half pairs j, j+dh/2,
 *        inverse frequency rope_theta^(-2j/dh))
 *   o_h = softmax(q^_h [Kc_g ; k^_g]^T / sqrt(dh)) [Vc_g ; v_g],  g = h / (Hq/Hkv)
 *   y = o Wo^T + s (o Ao^T) Bo^T
 * Kc/Vc are the cached prefix keys/values (keys already normalised and
 * rotated). Rows of the cache at index >= P_b are ignored.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device (or managed) pointers; pointers
 *     marked "host" are ordinary host memory read before the call returns.
 *   - All tensors are dense, row-major, with the shapes given, and 16-byte
 *     aligned (MOT_ERR_ALIGNMENT otherwise).
 *   - bf16 = IEEE bfloat16, f16 = IEEE binary16, f32 = IEEE binary32.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). All device
 *     work is enqueued on it; no call synchronises the host unless stated.
 *   - Validation happens on the host before anything is enqueued; a non-OK
 *     status means nothing was enqueued (except MOT_ERR_CUDA from a launch).
 *   - Device-detected conditions (fp16 overflow of an intermediate, a bounded
 *     wait that expired) are latched in the handle and returned by the next
 *     call that checks them (mot_attn_get_device_status).
 *   - The caller owns every buffer it passes. A handle must not be used from
 *     two streams at the same time.
 */
#ifndef MOT_ATTN_H
#define MOT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOT_OK = 0,
  MOT_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad enum, negative size   */
  MOT_ERR_UNSUPPORTED_SHAPE = 2,  /* dims outside what the kernels support   */
  MOT_ERR_ALIGNMENT = 3,          /* a pointer is not 16-byte aligned        */
  MOT_ERR_WORKSPACE_TOO_SMALL = 4,/* workspace/saved smaller than queried    */
  MOT_ERR_NO_SAVED_STATE = 5,     /* backward without a forward's saved state*/
  MOT_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed       */
  MOT_ERR_NUMERIC = 7,            /* an f16 intermediate overflowed          */
  MOT_ERR_TIMEOUT = 8             /* a bounded in-kernel wait expired        */
} mot_status;

typedef struct mot_attn* mot_attn_t; /* opaque handle */

/* Layer configuration. Supported: head_dim == 128, hidden == n_q_heads *
 * head_dim, n_q_heads % n_kv_heads == 0, hidden % 64 == 0, lora_rank in
 * {0, 8, 16, ..., 128} (a multiple of 8), max_batch <= 64. */
typedef struct {
  int32_t hidden;          /* model width d (4096)                            */
  int32_t n_q_heads;       /* Hq (32)                                         */
  int32_t n_kv_heads;      /* Hkv (8)                                         */
  int32_t head_dim;        /* dh (128)                                        */
  int32_t lora_rank;       /* r; 0 = no adapters                              */
  float lora_alpha;        /* alpha; scale s = alpha / r                      */
  float rms_eps;           /* QK-RMSNorm epsilon (1e-6)                       */
  double rope_theta;       /* RoPE base (1e6)                                 */
  int32_t max_batch;       /* largest B (CFG branches) per call               */
  int32_t max_img_tokens;  /* largest N per call                              */
  int32_t max_prefix;      /* largest P_max per call                          */
  int32_t enable_backward; /* nonzero: build what mot_attn_backward needs     */
} mot_attn_config;

/* Weights, all device bf16, nn.Linear layout [out, in]. The handle keeps the
 * pointers (and makes an f16 copy of w_o and f32 copies of the norm gains at
 * create); the caller keeps them alive and unchanged, except the LoRA
 * tensors a_* / b_*, which may be updated in place between calls (training).
 *   w_q [Hq*dh, d], w_k [Hkv*dh, d], w_v [Hkv*dh, d], w_o [d, Hq*dh]
 *   q_norm, k_norm [dh]
 *   a_q, a_k, a_v [r, d], a_o [r, Hq*dh]         (lora_down; NULL if r == 0)
 *   b_q [Hq*dh, r], b_k, b_v [Hkv*dh, r], b_o [d, r]   (lora_up) */
typedef struct {
  const void *w_q, *w_k, *w_v, *w_o;
  const void *q_norm, *k_norm;
  const void *a_q, *a_k, *a_v, *a_o;
  const void *b_q, *b_k, *b_v, *b_o;
} mot_attn_weights;

/* Bytes of caller-provided device memory for one call shape.
 * workspace_bytes: scratch for forward and backward (contents undefined
 *   between calls). saved_bytes: activations a training forward keeps for
 *   backward. Either output pointer may be NULL. Host-only; no CUDA calls. */
mot_status mot_attn_query_sizes(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens,
                                int32_t prefix_max, size_t* workspace_bytes, size_t* saved_bytes);

/* Create a handle. Validates cfg (host) and the weight pointers, allocates
 * the handle's own device copies (f16 w_o, f32 norm gains, f32 RoPE cos/sin
 * table built in fp64 on the host for positions < max_prefix +
 * max_img_tokens) and enqueues their initialisation on `stream`. It also
 * allocates the split-K scratch of the LoRA-down GEMMs (f32 partial tiles
 * for up to max_batch * max_img_tokens rows, at most 32 MiB, when
 * lora_rank > 0) with its arrival counters, and, with enable_backward,
 * transposed copies of w_o (bf16) and w_q|w_k|w_v (f16) and a second stream
 * plus two events on which the backward runs the LoRA-gradient GEMMs that
 * feed nothing later in the call.
 * Returns MOT_OK and *out, or an error and *out = NULL. */
mot_status mot_attn_create(const mot_attn_config* cfg, const mot_attn_weights* weights,
                           void* stream, mot_attn_t* out);

/* Forward of the layer.
 *   x        device bf16 [B, N, d]          image-token hidden states
 *   k_cache  device bf16 [B, Hkv, P_max, dh] cached prefix keys (normed+rotated)
 *   v_cache  device bf16 [B, Hkv, P_max, dh] cached prefix values
 *   prefix_len host int32 [B], 0 <= prefix_len[b] <= P_max
 *   y        device bf16 [B, N, d]          output (o_proj output, no residual)
 *   y_f32    device f32 [B, N, d] or NULL   the same output before rounding
 *            (y == RNE_bf16(y_f32) bit for bit)
 *   saved    device, saved_bytes from query_sizes, or NULL for inference;
 *            when given, the activations backward needs are written there
 *   workspace device, workspace_bytes from query_sizes
 * Shapes must satisfy 1 <= B <= max_batch, 1 <= N <= max_img_tokens,
 * 0 <= P_max <= max_prefix. */
mot_status mot_attn_forward(mot_attn_t h, const void* x, int32_t batch, int32_t img_tokens,
                            const void* k_cache, const void* v_cache, const int32_t* prefix_len,
                            int32_t prefix_max, void* y, float* y_f32, void* saved, size_t saved_bytes,
                            void* workspace, size_t workspace_bytes, void* stream);

/* The prefix tower's attention layer over the prompt, which builds the
 * prefix-KV cache entry of this layer ("SenseNova-U1" DiffSynth-Studio docs,
 * architecture note: the prompt is encoded once by the understanding branch
 * into past_key_values; "Setup notes", "Why bf16 base on CPU + tower
 * offload?": the prefix tower computes the static cache once, in bf16). The
 * handle is created with that tower's weights (w_q .. w_o, q_norm, k_norm of
 * the *_mot modules; lora_rank 0 for the pages' setup, adapters are applied
 * if the handle has them). Per branch b, token i < lengths[b] at position i:
 *   q, k, v as mot_attn_forward; o_i = softmax over keys j <= i; y = o Wo^T;
 *   k_cache_out[b, g, i] = k^_i (normalised, rotated), v_cache_out[b, g, i] = v_i
 * so that k_cache_out / v_cache_out with prefix_len = lengths are exactly the
 * cache mot_attn_forward takes (the image tokens continue at position
 * lengths[b]).
 *   x           device bf16 [B, N, d]     prompt hidden states (N = padded length)
 *   lengths     host int32 [B], 1 <= lengths[b] <= N; rows at or beyond it
 *               are padding: their y and cache rows are unspecified
 *   y, y_f32    as mot_attn_forward (y_f32 may be NULL)
 *   k_cache_out, v_cache_out  device bf16 [B, Hkv, N, dh], each element one
 *               round to nearest of the f32 value
 *   workspace   device, workspace_bytes of mot_attn_query_sizes(cfg, B, N, 0)
 * 1 <= B <= max_batch, N <= max_img_tokens. Inference only. */
mot_status mot_attn_prefix_forward(mot_attn_t h, const void* x, int32_t batch, int32_t tokens,
                                   const int32_t* lengths, void* y, float* y_f32, void* k_cache_out,
                                   void* v_cache_out, void* workspace, size_t workspace_bytes, void* stream);

/* LoRA-training backward of the layer (base weights, norm gains and the
 * cache are frozen; no gradient flows into them).
 *   dy       device bf16 [B, N, d]     upstream gradient of y
 *   x, k_cache, v_cache, prefix_len, prefix_max: as passed to the forward
 *   saved    the buffer a forward with the same arguments filled
 *   dx       device bf16 [B, N, d]     gradient of x
 *   dx_f32   device f32 [B, N, d] or NULL  (dx == RNE_bf16(dx_f32))
 *   d_a[4], d_b[4]  device f32, q,k,v,o order, shapes of a_* / b_*;
 *            accumulate != 0 adds into their contents, else overwrites.
 *            All NULL is allowed when lora_rank == 0.
 * Requires cfg.enable_backward. Deterministic: same inputs, same bits.
 * Part of the work (the dB and dA GEMMs) runs on the handle's own stream,
 * which waits for `stream` where its inputs are produced; before returning,
 * the call makes `stream` wait for that work, so everything the call writes
 * is ordered before later work on `stream`, as if it all ran there. */
mot_status mot_attn_backward(mot_attn_t h, const void* dy, const void* x, int32_t batch,
                             int32_t img_tokens, const void* k_cache, const void* v_cache,
                             const int32_t* prefix_len, int32_t prefix_max, const void* saved,
                             size_t saved_bytes, void* dx, float* dx_f32, float* const d_a[4],
                             float* const d_b[4], int32_t accumulate, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Fold the adapters into the base ("SenseNova-U1.5" vLLM-Omni recipe,
 * 8-step distilled LoRA: fused into the gen tower at load):
 *   w_*_out = RNE_bf16(w_* + s * b_* a_*)   computed in f32, one rounding.
 * Outputs are device bf16 with the shapes of w_q, w_k, w_v, w_o and may alias
 * the inputs (in-place bake-in). On success the handle is rebound to the
 * merged weights with rank 0. */
mot_status mot_attn_merge_lora(mot_attn_t h, void* w_q_out, void* w_k_out, void* w_v_out,
                               void* w_o_out, void* stream);

/* Forward that allocates nothing and takes no workspace. The pages describe
 * no such call; it exists for callers that cannot call cudaMalloc per call:
 * plug-ins whose host owns all device memory (pre-reserved arenas where an
 * extra allocation fails or fragments the pool) and latency-critical loops
 * where cudaMalloc's implicit device-wide synchronisation is not acceptable.
 * Arguments are those of mot_attn_forward without saved/workspace
 * (inference only). The scratch lives in one 32 MiB device array inside this
 * library (every GPU that loads the library holds it until process exit);
 * a call whose scratch exceeds 32 MiB returns MOT_ERR_WORKSPACE_TOO_SMALL
 * before anything is enqueued. The scratch is what an inference forward of
 * the shape needs (its activations and the f16 copies of the LoRA tensors):
 * at hidden 4096, 32/8 heads, LoRA rank 32 and a 400-token prefix, up to
 * about 1450 image tokens in one branch.
 * The current CUDA device must be the one the handle was created on
 * (MOT_ERR_INVALID_ARGUMENT otherwise). The first call on a device resolves
 * the array's device address on the host; make that first call before any
 * stream capture. All calls share the
 * one array and leave their intermediates in it: calls that overlap on the
 * GPU (other streams, other handles, other threads) race and must be
 * serialised by the caller. Nothing in the array needs to start at zero:
 * every byte a call reads was written earlier in the same call. */
mot_status mot_attn_forward_noalloc(mot_attn_t h, const void* x, int32_t batch, int32_t img_tokens,
                                    const void* k_cache, const void* v_cache, const int32_t* prefix_len,
                                    int32_t prefix_max, void* y, float* y_f32, void* stream);

/* Device staging bytes mot_attn_forward_host needs for calls of this shape:
 * two slots, each holding one call's x, k_cache, v_cache and y. Host-only;
 * no CUDA calls. */
mot_status mot_attn_query_host_staging(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens,
                                       int32_t prefix_max, size_t* staging_bytes);

/* `steps` inference forwards whose inputs and outputs live in host memory
 * (the pages describe no such call: it is the host-buffer path a serving
 * loop or an end-to-end measurement drives).
 *   x_host[i]        host bf16 [B, N, d]              input of call i
 *   k_cache_host[i], v_cache_host[i]
 *                    host bf16 [B, Hkv, P_max, dh]     (NULL allowed when P_max == 0)
 *   prefix_len       host int32 [B], shared by all calls
 *   y_host[i]        host bf16 [B, N, d]              output of call i
 *   staging          device, staging_bytes from mot_attn_query_host_staging
 *   workspace        device, workspace_bytes from mot_attn_query_sizes
 * Call i uses staging slot i % 2: its inputs are copied into the slot on a
 * copy-in stream the handle owns, the layer runs on `stream` (as
 * mot_attn_forward), and y is copied back on a copy-out stream the handle
 * owns; the copy-in of call i+1 and the copy-out of call i-1 therefore
 * overlap the layer of call i (PCIe carries both directions at once). A slot
 * is refilled only after the layer two calls earlier has read it and its y
 * has been copied out. Exception to the host-pointer rule above: the host
 * buffers are read and written asynchronously, after this function returns;
 * they must stay valid and untouched until `stream` has completed the work
 * enqueued so far. Page-locked (pinned) host memory lets the copies overlap;
 * pageable memory gives the same results with the copies serialised.
 * Both copy streams first wait for the work already enqueued on `stream`,
 * and `stream` finally waits for the last copy-out, so every y_host[i] is
 * complete once `stream` reaches the end of this call's work. */
mot_status mot_attn_forward_host(mot_attn_t h, int32_t steps, const void* const* x_host, int32_t batch,
                                 int32_t img_tokens, const void* const* k_cache_host,
                                 const void* const* v_cache_host, const int32_t* prefix_len, int32_t prefix_max,
                                 void* const* y_host, void* staging, size_t staging_bytes, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Synchronise `stream` and return (and clear) the status latched on the
 * device by earlier calls: MOT_OK, MOT_ERR_NUMERIC or MOT_ERR_TIMEOUT. The
 * outputs of a call that timed out are undefined; after MOT_ERR_TIMEOUT the
 * handle's internal split-K counters are reset, so later calls are valid. */
mot_status mot_attn_get_device_status(mot_attn_t h, void* stream);

/* Free the handle's own device memory. NULL is ignored. */
void mot_attn_destroy(mot_attn_t h);

/* Static, human-readable name of a status. */
const char* mot_status_string(mot_status s);

/* Number of kernels the last forward / backward call enqueued (host-side
 * count, for launch accounting). */
int32_t mot_attn_last_launch_count(mot_attn_t h);

#ifdef __cplusplus
}
#endif

#endif /* MOT_ATTN_H */
