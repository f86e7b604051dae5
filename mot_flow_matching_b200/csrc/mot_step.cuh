// mot_step.cuh -- C ABI of one gen-tower flow-matching denoise step (see
// include/mot_step.h). Same translation unit as mot_attn.cu: it drives the
// attention and MLP forwards through their internal residual mode and reuses
// the tensor-map and launch helpers.
//
// Launch sequence on the caller's stream (d = hidden, C = patch_dim):
//   f32_to_bf16        z -> bf16 (the embedding GEMM's operand)
//   embed GEMM         e0 = z W_in^T (f32 [N, d]), CTA pairs
//   temb_kernel        e(sigma) (f32 [d])
//   per layer l:
//     rmsnorm_rows     h -> bf16 RMSNorm(h) g_in[l] (layer 0 first forms
//                      h = e0 + e(sigma) in every branch's rows)
//     attention layer  h += Attn_l(.)  (mot_attn forward, f32 accumulate)
//     rmsnorm_rows     h -> bf16 RMSNorm(h) g_post[l]
//     MLP              h += MLP_l(.)   (mot_mlp forward, f32 accumulate)
//   rmsnorm_rows       h -> bf16 RMSNorm(h) g_out
//   head GEMM          x0 = . W_out^T (f32 [B N, C]), CTA pairs
//   cfg_euler_kernel   guidance and the Euler update -> z_next
#pragma once

#include "mot_step.h"

struct mot_step {
  mot_step_config cfg;
  std::vector<mot_attn_t> attn;
  std::vector<mot_mlp_t> mlp;
  float* gains = nullptr;  // [n_layers][2][d] (in, post) then [d] (out), f32
  CUtensorMap win_map, wout_map;
  int num_sms = 148;
};

namespace {

struct StepLayout {
  size_t h = 0, e0 = 0, xn = 0, zb = 0, x0 = 0, temb = 0, layer = 0, layer_bytes = 0, total = 0;
};

mot_status make_step_layout(const mot_step* s, int B, int N, int P, StepLayout& L) {
  const size_t d = s->cfg.hidden, C = s->cfg.patch_dim, M = static_cast<size_t>(B) * N;
  size_t lw = 0;
  for (size_t l = 0; l < s->attn.size(); ++l) {
    size_t a = 0, m = 0;
    mot_status st = mot_attn_query_sizes(&s->attn[l]->cfg, B, N, P, &a, nullptr);
    if (st != MOT_OK) return st;
    st = mot_mlp_query_sizes(&s->mlp[l]->cfg, static_cast<int32_t>(M), &m, nullptr);
    if (st != MOT_OK) return st;
    lw = std::max({lw, a, m});
  }
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 1024);
    return o;
  };
  L.h = take(M * d * 4);
  L.e0 = take(static_cast<size_t>(N) * d * 4);
  L.xn = take(M * d * 2);
  L.zb = take(static_cast<size_t>(N) * C * 2);
  L.x0 = take(M * C * 4);
  L.temb = take(d * 4);
  L.layer = take(lw);
  L.layer_bytes = lw;
  L.total = off;
  return MOT_OK;
}

// one pair-kernel GEMM D (f32) = A (bf16 [M, K]) B^T (bf16 [Nout, K] map)
cudaError_t step_gemm(const CUtensorMap& bmap, const void* a, int M, int Nout, int K, float* d, int* status,
                      int num_sms, cudaStream_t st) {
  GemmCore core;
  core_init(core, M, Nout, 256, 128, status);
  core_pair(core);
  if (!map2d(&core.maps[0], a, true, K, M, K, 128)) return cudaErrorInvalidValue;
  core.maps[2] = bmap;
  core.segs[0] = seg1(0, 0, 2, K / 64, idesc_f16(256, 256, true, true), false, false);
  core.num_segs = 1;
  EpiStore::Params ep = store_params(M, Nout);
  ep.out32 = d;
  ep.ld32 = Nout;
  return launch_gemm2<256, 6, EpiStore>(core, ep, num_sms, st);
}

}  // namespace

extern "C" {

mot_status mot_step_create(const mot_step_config* cfg, const mot_step_model* model, void* stream, mot_step_t* out) {
  if (!out) return MOT_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!cfg || !model || cfg->n_layers < 1 || !model->attn || !model->mlp || !model->norm_in ||
      !model->norm_post || !model->w_in || !model->norm_out || !model->w_out || !(cfg->rms_eps >= 0.f))
    return MOT_ERR_INVALID_ARGUMENT;
  if (cfg->hidden <= 0 || cfg->hidden % 256 != 0 || cfg->patch_dim <= 0 || cfg->patch_dim % 256 != 0)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  for (int l = 0; l < cfg->n_layers; ++l) {
    if (!model->attn[l] || !model->mlp[l] || !model->norm_in[l] || !model->norm_post[l])
      return MOT_ERR_INVALID_ARGUMENT;
    if (model->attn[l]->cfg.hidden != cfg->hidden || model->mlp[l]->cfg.hidden != cfg->hidden)
      return MOT_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(model->norm_in[l]) || !aligned16(model->norm_post[l])) return MOT_ERR_ALIGNMENT;
  }
  if (!aligned16(model->w_in) || !aligned16(model->w_out) || !aligned16(model->norm_out)) return MOT_ERR_ALIGNMENT;
  if (!encode_ready()) return MOT_ERR_CUDA;
  mot_step* s = new (std::nothrow) mot_step();
  if (!s) return MOT_ERR_CUDA;
  s->cfg = *cfg;
  s->attn.assign(model->attn, model->attn + cfg->n_layers);
  s->mlp.assign(model->mlp, model->mlp + cfg->n_layers);
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&s->num_sms, cudaDevAttrMultiProcessorCount, dev);
  const int d = cfg->hidden, C = cfg->patch_dim, nl = cfg->n_layers;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMalloc(&s->gains, (static_cast<size_t>(nl) * 2 + 1) * d * sizeof(float)) == cudaSuccess;
  for (int l = 0; l < nl && ok; ++l) {
    bf16_to_f32_kernel<<<(d + 127) / 128, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(model->norm_in[l]),
                                                         s->gains + static_cast<size_t>(2 * l) * d, d);
    bf16_to_f32_kernel<<<(d + 127) / 128, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(model->norm_post[l]),
                                                         s->gains + static_cast<size_t>(2 * l + 1) * d, d);
  }
  if (ok)
    bf16_to_f32_kernel<<<(d + 127) / 128, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(model->norm_out),
                                                         s->gains + static_cast<size_t>(2 * nl) * d, d);
  ok = ok && cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(st) == cudaSuccess &&
       map2d(&s->win_map, model->w_in, true, C, d, C, 128) && map2d(&s->wout_map, model->w_out, true, d, C, d, 128);
  if (!ok) {
    cudaFree(s->gains);
    delete s;
    return MOT_ERR_CUDA;
  }
  *out = s;
  return MOT_OK;
}

void mot_step_destroy(mot_step_t h) {
  if (!h) return;
  cudaFree(h->gains);
  delete h;
}

mot_status mot_step_query_workspace(mot_step_t h, int32_t B, int32_t N, int32_t P, size_t* workspace_bytes) {
  if (!h || !workspace_bytes || B <= 0 || B > 3 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  StepLayout L;
  const mot_status st = make_step_layout(h, B, N, P, L);
  if (st != MOT_OK) return st;
  *workspace_bytes = L.total;
  return MOT_OK;
}

mot_status mot_step_forward(mot_step_t h, const float* z, int32_t B, int32_t N, const void* const* k_cache,
                            const void* const* v_cache, const int32_t* prefix_len, int32_t P, float sigma,
                            float sigma_next, float cfg_scale, float img_cfg_scale, float t_eps, float* z_next,
                            void* z_next_bf16, void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !z || !z_next || !prefix_len || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  if (B <= 0 || B > 3 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  const int nl = h->cfg.n_layers;
  if (P > 0 && (!k_cache || !v_cache)) return MOT_ERR_INVALID_ARGUMENT;
  if (!aligned16(z) || !aligned16(z_next) || !aligned16(workspace) || (z_next_bf16 && !aligned16(z_next_bf16)))
    return MOT_ERR_ALIGNMENT;
  if (!(t_eps > 0.f) || !(sigma >= 0.f)) return MOT_ERR_INVALID_ARGUMENT;
  StepLayout L;
  mot_status status = make_step_layout(h, B, N, P, L);
  if (status != MOT_OK) return status;
  if (workspace_bytes < L.total) return MOT_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* hs = reinterpret_cast<float*>(ws + L.h);
  float* e0 = reinterpret_cast<float*>(ws + L.e0);
  __nv_bfloat16* xn = reinterpret_cast<__nv_bfloat16*>(ws + L.xn);
  __nv_bfloat16* zb = reinterpret_cast<__nv_bfloat16*>(ws + L.zb);
  float* x0 = reinterpret_cast<float*>(ws + L.x0);
  float* temb = reinterpret_cast<float*>(ws + L.temb);
  void* lws = ws + L.layer;
  const int d = h->cfg.hidden, C = h->cfg.patch_dim, M = B * N;
  const float eps = h->cfg.rms_eps;
  const long long nzc = static_cast<long long>(N) * C;
  const int ew_grid = static_cast<int>(std::min<long long>((nzc + 255) / 256, 8LL * h->num_sms));
  const int norm_grid = std::min((M + 7) / 8, 16 * h->num_sms);  // 8 warps (rows) per block
  // the tower's own status word: the first layer's (every kernel here only
  // reports through the layers)
  int* status_word = h->attn[0]->status;
  cudaError_t e = launch_pdl(f32_to_bf16_kernel, dim3(ew_grid), dim3(256), 0, st, z, zb, nzc);
  if (e == cudaSuccess) e = step_gemm(h->win_map, zb, N, d, C, e0, status_word, h->num_sms, st);
  if (e == cudaSuccess)
    e = launch_pdl(temb_kernel, dim3((d / 2 + 127) / 128), dim3(128), 0, st, temb, d, static_cast<double>(sigma));
  if (e != cudaSuccess) return MOT_ERR_CUDA;
  for (int l = 0; l < nl; ++l) {
    const float* g_in = h->gains + static_cast<size_t>(2 * l) * d;
    const float* g_post = g_in + d;
    e = launch_pdl(rmsnorm_rows_kernel, dim3(norm_grid), dim3(256), 0, st, hs, l == 0 ? e0 : nullptr, N, temb, g_in,
                   xn, M, d, eps);
    if (e != cudaSuccess) return MOT_ERR_CUDA;
    status = forward_impl(h->attn[l], xn, B, N, P > 0 ? k_cache[l] : nullptr, P > 0 ? v_cache[l] : nullptr,
                          prefix_len, P, nullptr, hs, nullptr, 0, lws, L.layer_bytes, stream, nullptr, true);
    if (status != MOT_OK) return status;
    e = launch_pdl(rmsnorm_rows_kernel, dim3(norm_grid), dim3(256), 0, st, hs, static_cast<const float*>(nullptr), N,
                   static_cast<const float*>(nullptr), g_post, xn, M, d, eps);
    if (e != cudaSuccess) return MOT_ERR_CUDA;
    status = mlp_forward_impl(h->mlp[l], xn, M, nullptr, hs, nullptr, 0, lws, L.layer_bytes, stream, true);
    if (status != MOT_OK) return status;
  }
  e = launch_pdl(rmsnorm_rows_kernel, dim3(norm_grid), dim3(256), 0, st, hs, static_cast<const float*>(nullptr), N,
                 static_cast<const float*>(nullptr), h->gains + static_cast<size_t>(2 * nl) * d, xn, M, d, eps);
  if (e == cudaSuccess) e = step_gemm(h->wout_map, xn, M, C, d, x0, status_word, h->num_sms, st);
  const double c = (static_cast<double>(sigma_next) - sigma) / std::max(static_cast<double>(sigma),
                                                                         static_cast<double>(t_eps));
  if (e == cudaSuccess)
    e = launch_pdl(cfg_euler_kernel, dim3(ew_grid), dim3(256), 0, st, static_cast<const float*>(x0), nzc, B, z, z_next,
                   static_cast<__nv_bfloat16*>(z_next_bf16), cfg_scale, img_cfg_scale, static_cast<float>(c));
  return e == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

}  // extern "C"
