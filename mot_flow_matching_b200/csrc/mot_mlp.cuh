// mot_mlp.cuh -- C ABI of the gen-tower SwiGLU MLP with LoRA (see
// include/mot_mlp.h). Part of the same translation unit as mot_attn.cu: it
// reuses that file's tensor-map, launch and split-K helpers and the same
// kernel instantiations (the persistent tcgen05 GEMMs of gemm.cuh).
//
// Forward launch sequence on the caller's stream (r = LoRA rank, s = alpha/r,
// RP = r rounded up to 64):
//   [r>0] mlp_prep      A_down, B_down -> f16; B_gate, B_up -> zero-padded f16
//                       blocks of one [I, 2 RP] K extension each
//   [r>0] LoRA down     u_gu = s x [A_gate; A_up]^T                  (f16)
//   gate/up GEMM        CTA pairs, 256-column tiles of 128 gate + 128 up
//                       columns of the same intermediate indices (rank 0 of
//                       the pair stages W_gate rows, rank 1 W_up rows), LoRA up
//                       as the K extension; epilogue h = silu(g) u     (f16)
//   [r>0] LoRA down     u_d = s h A_down^T                            (f16)
//   down GEMM           y = h W_down^T + u_d B_down^T                 (bf16 + f32)
// Backward (LoRA training, base frozen):
//   [r>0] B_gate, B_up -> f16;  g_d = dy B_down
//   dh GEMM + epilogue  dh = dy W_down + s g_d A_down; dg = dh u silu'(g),
//                       du = dh silu(g)                               (f16 [T, 2I])
//   [r>0] dB_down = dy^T u_d ; dA_down = s g_d^T h          (side stream)
//   [r>0] g_gu = [dg B_gate | du B_up]
//   [r>0] dB_gate/up = [dg|du]^T u_gu ; dA_gate/up = s g_gu^T x (side stream)
//   dx GEMM             dx = dg W_gate + du W_up + s sum_j g_j A_j
#pragma once

#include "mot_mlp.h"

struct mot_mlp {
  mot_mlp_config cfg;
  mot_mlp_weights w;
  int rank = 0;
  float scale = 0.f;
  int RP = 0;
  int device = 0;
  int num_sms = 148;
  int last_launches = 0;
  __half* wd16 = nullptr;          // [d, I] f16 W_down (it meets the f16 h)
  __nv_bfloat16* wdT = nullptr;    // [I, d] W_down^T (backward: dh GEMM B operand, K-major)
  __half* wguT16 = nullptr;        // [d, 2I] [W_gate^T | W_up^T] f16 (backward: dx GEMM)
  int* status = nullptr;
  int* split_cnt = nullptr;        // [3][kSplitCounters]: caller's stream, side stream, forward
  void* fsplit = nullptr;          // forward split-K partials
  size_t fsplit_bytes = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  bool profile = false;
  cudaEvent_t ev[2 * kMaxStages + 2] = {};
  cudaEvent_t stage_start[kMaxStages] = {}, stage_end[kMaxStages] = {};
  int stage_ids[kMaxStages] = {};
  int stage_count = 0;
  CUtensorMap wg, wu, wd;          // K-major, box rows 128
  CUtensorMap ag, au;              // lora_down gate/up, box rows RP
  CUtensorMap wdT_k, wguT_k;       // backward K-major
  CUtensorMap ag_mn, au_mn, ad_mn, bd_mn;
};

namespace {

enum MlpStageId : int {
  MS_PREP = 0, MS_LORA_DOWN_GU = 1, MS_GATE_UP = 2, MS_LORA_DOWN_D = 3, MS_DOWN = 4, MS_BWD_PREP = 5,
  MS_BWD_G_D = 6, MS_BWD_DH = 7, MS_BWD_DB_D = 8, MS_BWD_DA_D = 9, MS_BWD_G_GU = 10, MS_BWD_DB_GU = 11,
  MS_BWD_DA_GU = 12, MS_BWD_DX = 13,
};
const char* const kMlpStageNames[] = {"mlp_prep", "mlp_lora_down_gu", "mlp_gate_up", "mlp_lora_down_d",
                                      "mlp_down", "mlp_bwd_prep", "mlp_bwd_g_d", "mlp_bwd_dh",
                                      "mlp_bwd_db_d", "mlp_bwd_da_d", "mlp_bwd_g_gu", "mlp_bwd_db_gu",
                                      "mlp_bwd_da_gu", "mlp_bwd_dx"};

struct MlpLayout {
  int T = 0, r = 0, RP = 0;
  // activations: in `saved` for training, else after the forward scratch
  size_t o_ugu = 0, o_h = 0, o_g = 0, o_u = 0, o_ud = 0, o_udhi = 0, o_udlo = 0, act_bytes = 0;
  // forward scratch: per-call f16 copies of the LoRA tensors
  size_t w_ad16 = 0, w_bd16 = 0, w_bg2 = 0, w_bu2 = 0, fwd_scratch = 0;
  // backward scratch
  size_t b_dgu = 0, b_gdhi = 0, b_gdlo = 0, b_gd16 = 0, b_ghi = 0, b_glo = 0, b_bg16 = 0, b_bu16 = 0, b_split = 0,
         bwd_scratch = 0;
};

MlpLayout make_mlp_layout(const mot_mlp_config& c, int T, bool train) {
  MlpLayout L;
  L.T = T;
  L.r = c.lora_rank;
  L.RP = L.r ? static_cast<int>(round_up(L.r, 64)) : 0;
  const size_t d = c.hidden, I = c.intermediate, r = L.r, RP = L.RP, t = T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 1024);
    return o;
  };
  L.o_ugu = take(r ? t * 2 * RP * 2 : 0);
  L.o_h = take(t * I * 2);
  L.o_g = take(train ? t * I * 2 : 0);
  L.o_u = take(train ? t * I * 2 : 0);
  L.o_ud = take(r ? t * RP * 2 : 0);
  L.o_udhi = take(train && r ? t * RP * 2 : 0);
  L.o_udlo = take(train && r ? t * RP * 2 : 0);
  L.act_bytes = off;
  off = 0;
  L.w_ad16 = take(r ? r * I * 2 : 0);
  L.w_bd16 = take(r ? d * r * 2 : 0);
  L.w_bg2 = take(r ? I * 2 * RP * 2 : 0);
  L.w_bu2 = take(r ? I * 2 * RP * 2 : 0);
  L.fwd_scratch = off;
  off = 0;
  L.b_dgu = take(t * 2 * I * 2);
  L.b_gdhi = take(r ? t * RP * 2 : 0);
  L.b_gdlo = take(r ? t * RP * 2 : 0);
  L.b_gd16 = take(r ? t * RP * 2 : 0);
  L.b_ghi = take(r ? t * 2 * RP * 2 : 0);
  L.b_glo = take(r ? t * 2 * RP * 2 : 0);
  L.b_bg16 = take(r ? I * r * 2 : 0);
  L.b_bu16 = take(r ? I * r * 2 : 0);
  L.b_split = take(r ? 2 * kSplitWsBytes : 0);
  L.bwd_scratch = c.enable_backward ? off : 0;
  return L;
}

mot_status check_mlp_config(const mot_mlp_config* c) {
  if (!c) return MOT_ERR_INVALID_ARGUMENT;
  if (c->hidden <= 0 || c->intermediate <= 0 || c->lora_rank < 0 || c->max_tokens <= 0)
    return MOT_ERR_INVALID_ARGUMENT;
  if (c->lora_rank > 0 && !(c->lora_alpha == c->lora_alpha)) return MOT_ERR_INVALID_ARGUMENT;
  if (c->hidden % 256 != 0 || c->intermediate % 128 != 0 || c->lora_rank % 8 != 0 || c->lora_rank > 128)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(c->max_tokens) > (1ll << 30)) return MOT_ERR_UNSUPPORTED_SHAPE;
  return MOT_OK;
}

mot_status build_mlp_maps(mot_mlp* h) {
  const mot_mlp_config& c = h->cfg;
  const uint64_t d = c.hidden, I = c.intermediate;
  bool ok = map2d(&h->wg, h->w.w_gate, true, d, I, d, 128) && map2d(&h->wu, h->w.w_up, true, d, I, d, 128) &&
            map2d(&h->wd, h->wd16, false, I, d, I, 128);
  if (ok && h->rank > 0) {
    const uint64_t r = h->rank;
    const uint32_t box_a = static_cast<uint32_t>(h->RP);
    ok = map2d(&h->ag, h->w.a_gate, true, d, r, d, box_a) && map2d(&h->au, h->w.a_up, true, d, r, d, box_a);
  }
  if (ok && c.enable_backward) {
    ok = map2d(&h->wdT_k, h->wdT, true, d, I, d, 128) && map2d(&h->wguT_k, h->wguT16, false, 2 * I, d, 2 * I, 128);
    if (ok && h->rank > 0) {
      const uint64_t r = h->rank;
      ok = map2d_mn(&h->ag_mn, h->w.a_gate, true, d, r, d) && map2d_mn(&h->au_mn, h->w.a_up, true, d, r, d) &&
           map2d_mn(&h->ad_mn, h->w.a_down, true, I, r, I) && map2d_mn(&h->bd_mn, h->w.b_down, true, r, d, r);
    }
  }
  return ok ? MOT_OK : MOT_ERR_CUDA;
}

void release_mlp(mot_mlp* h) {
  if (!h) return;
  for (cudaEvent_t e : h->ev)
    if (e) cudaEventDestroy(e);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  cudaFree(h->wd16);
  cudaFree(h->wdT);
  cudaFree(h->wguT16);
  cudaFree(h->status);
  cudaFree(h->split_cnt);
  cudaFree(h->fsplit);
  delete h;
}

using MlpLaunches = LaunchesT<mot_mlp>;

}  // namespace

extern "C" {

mot_status mot_mlp_query_sizes(const mot_mlp_config* cfg, int32_t tokens, size_t* workspace_bytes,
                               size_t* saved_bytes) {
  mot_status st = check_mlp_config(cfg);
  if (st != MOT_OK) return st;
  if (tokens <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (tokens > cfg->max_tokens) return MOT_ERR_UNSUPPORTED_SHAPE;
  const MlpLayout inf = make_mlp_layout(*cfg, tokens, false);
  const MlpLayout trn = make_mlp_layout(*cfg, tokens, true);
  if (workspace_bytes)
    *workspace_bytes = std::max({inf.fwd_scratch + inf.act_bytes, trn.fwd_scratch, trn.bwd_scratch});
  if (saved_bytes) *saved_bytes = trn.act_bytes;
  return MOT_OK;
}

mot_status mot_mlp_create(const mot_mlp_config* cfg, const mot_mlp_weights* wts, void* stream, mot_mlp_t* out) {
  if (!out) return MOT_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  mot_status st = check_mlp_config(cfg);
  if (st != MOT_OK) return st;
  if (!wts || !wts->w_gate || !wts->w_up || !wts->w_down) return MOT_ERR_INVALID_ARGUMENT;
  if (cfg->lora_rank > 0 && (!wts->a_gate || !wts->a_up || !wts->a_down || !wts->b_gate || !wts->b_up ||
                             !wts->b_down))
    return MOT_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {wts->w_gate, wts->w_up, wts->w_down, wts->a_gate, wts->a_up,
                        wts->a_down, wts->b_gate, wts->b_up, wts->b_down};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  if (!encode_ready()) return MOT_ERR_CUDA;

  mot_mlp* h = new (std::nothrow) mot_mlp();
  if (!h) return MOT_ERR_CUDA;
  h->cfg = *cfg;
  h->w = *wts;
  h->rank = cfg->lora_rank;
  h->scale = h->rank ? cfg->lora_alpha / static_cast<float>(h->rank) : 0.f;
  h->RP = h->rank ? static_cast<int>(round_up(h->rank, 64)) : 0;
  cudaGetDevice(&h->device);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t d = cfg->hidden, I = cfg->intermediate;
  bool ok = cudaMalloc(&h->wd16, d * I * 2) == cudaSuccess && cudaMalloc(&h->status, sizeof(int)) == cudaSuccess &&
            cudaMalloc(&h->split_cnt, 3 * kSplitCounters * sizeof(int)) == cudaSuccess &&
            cudaMemset(h->split_cnt, 0, 3 * kSplitCounters * sizeof(int)) == cudaSuccess;
  if (ok && h->rank > 0) {
    // the forward LoRA-down GEMMs' split-K partials: up to 4 splits of the
    // 128-row tiles of the largest call, 128 f32 columns each
    const size_t tiles = (static_cast<size_t>(cfg->max_tokens) + kBM - 1) / kBM;
    h->fsplit_bytes = std::min(kSplitWsBytes * 2, tiles * 4 * 2 * 128 * kBM * 4);
    ok = cudaMalloc(&h->fsplit, h->fsplit_bytes) == cudaSuccess;
  }
  if (ok && cfg->enable_backward)
    ok = cudaMalloc(&h->wdT, I * d * 2) == cudaSuccess && cudaMalloc(&h->wguT16, d * 2 * I * 2) == cudaSuccess &&
         cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    release_mlp(h);
    return MOT_ERR_CUDA;
  }
  ok = cudaMemsetAsync(h->status, 0, sizeof(int), s) == cudaSuccess;
  // frozen base: f16 W_down; for backward W_down^T (bf16) and [W_gate^T | W_up^T] (f16)
  CvtJobs jobs{};
  jobs.src[0] = static_cast<const __nv_bfloat16*>(wts->w_down);
  jobs.dst[0] = h->wd16;
  jobs.n8[0] = static_cast<long long>(d * I / 8);
  jobs.count = 1;
  cvt_multi_kernel<<<4 * h->num_sms, 256, 0, s>>>(jobs, h->status);
  if (cfg->enable_backward) {
    const dim3 blk(32, 8);
    transpose_copy_kernel<__nv_bfloat16><<<dim3((I + 31) / 32, (d + 31) / 32), blk, 0, s>>>(
        static_cast<const __nv_bfloat16*>(wts->w_down), static_cast<int>(d), static_cast<int>(I), h->wdT,
        static_cast<long long>(d), 0);
    const void* src[2] = {wts->w_gate, wts->w_up};
    for (int j = 0; j < 2; ++j)
      transpose_copy_kernel<__half><<<dim3((d + 31) / 32, (I + 31) / 32), blk, 0, s>>>(
          static_cast<const __nv_bfloat16*>(src[j]), static_cast<int>(I), static_cast<int>(d), h->wguT16,
          static_cast<long long>(2 * I), static_cast<int>(j * I));
  }
  ok = ok && cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess &&
       build_mlp_maps(h) == MOT_OK;
  if (!ok) {
    release_mlp(h);
    return MOT_ERR_CUDA;
  }
  *out = h;
  return MOT_OK;
}

void mot_mlp_destroy(mot_mlp_t h) { release_mlp(h); }

int32_t mot_mlp_last_launch_count(mot_mlp_t h) { return h ? h->last_launches : 0; }

mot_status mot_mlp_get_device_status(mot_mlp_t h, void* stream) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  int v = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return MOT_ERR_CUDA;
  if (v & DEV_ERR_TIMEOUT) {
    if (h->side && cudaStreamSynchronize(h->side) != cudaSuccess) return MOT_ERR_CUDA;
    if (cudaMemset(h->split_cnt, 0, 3 * kSplitCounters * sizeof(int)) != cudaSuccess) return MOT_ERR_CUDA;
    return MOT_ERR_TIMEOUT;
  }
  if (v & DEV_ERR_NUMERIC) return MOT_ERR_NUMERIC;
  return MOT_OK;
}

}  // extern "C"

namespace {

// residual: the block output is added into y_f32 (the caller's f32
// residual stream; y may then be NULL)
mot_status mlp_forward_impl(mot_mlp_t h, const void* x, int32_t T, void* y, float* y_f32, void* saved,
                            size_t saved_bytes, void* workspace, size_t workspace_bytes, void* stream,
                            bool residual) {
  if (!h || !x || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  if (residual ? !y_f32 : !y) return MOT_ERR_INVALID_ARGUMENT;
  const mot_mlp_config& c = h->cfg;
  if (T <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (T > c.max_tokens) return MOT_ERR_UNSUPPORTED_SHAPE;
  const void* ptrs[] = {x, y, y_f32, saved, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  const bool train = saved != nullptr;
  const MlpLayout L = make_mlp_layout(c, T, train);
  if (train && saved_bytes < L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (workspace_bytes < L.fwd_scratch + (train ? 0 : L.act_bytes)) return MOT_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* act = train ? static_cast<uint8_t*>(saved) : ws + L.fwd_scratch;
  __half* u_gu = reinterpret_cast<__half*>(act + L.o_ugu);
  __half* hh = reinterpret_cast<__half*>(act + L.o_h);
  __half* g_sv = train ? reinterpret_cast<__half*>(act + L.o_g) : nullptr;
  __half* u_sv = train ? reinterpret_cast<__half*>(act + L.o_u) : nullptr;
  __half* u_d = reinterpret_cast<__half*>(act + L.o_ud);
  __nv_bfloat16* u_dhi = train ? reinterpret_cast<__nv_bfloat16*>(act + L.o_udhi) : nullptr;
  __nv_bfloat16* u_dlo = train ? reinterpret_cast<__nv_bfloat16*>(act + L.o_udlo) : nullptr;
  __half* ad16 = reinterpret_cast<__half*>(ws + L.w_ad16);
  __half* bd16 = reinterpret_cast<__half*>(ws + L.w_bd16);
  __half* bg2 = reinterpret_cast<__half*>(ws + L.w_bg2);
  __half* bu2 = reinterpret_cast<__half*>(ws + L.w_bu2);

  const int d = c.hidden, I = c.intermediate, r = h->rank, RP = h->RP;
  MlpLaunches lz(h, st);

  // 1. f16 copies of the LoRA tensors that meet f16 operands (per call: a
  //    trainer updates them in place between calls)
  if (r > 0) {
    lz.stage = MS_PREP;
    CvtJobs cj{};
    cj.src[0] = static_cast<const __nv_bfloat16*>(h->w.a_down);
    cj.dst[0] = ad16;
    cj.n8[0] = static_cast<long long>(r) * I / 8;
    cj.src[1] = static_cast<const __nv_bfloat16*>(h->w.b_down);
    cj.dst[1] = bd16;
    cj.n8[1] = static_cast<long long>(d) * r / 8;
    cj.count = 2;
    PadJobs pj{};
    pj.src[0] = static_cast<const __nv_bfloat16*>(h->w.b_gate);
    pj.dst[0] = bg2;
    pj.col0[0] = 0;
    pj.src[1] = static_cast<const __nv_bfloat16*>(h->w.b_up);
    pj.dst[1] = bu2;
    pj.col0[1] = RP;
    pj.rows[0] = pj.rows[1] = I;
    pj.r = r;
    pj.ld = 2 * RP;
    pj.count = 2;
    lz.done(launch_pdl(mlp_prep_kernel, dim3(2 * h->num_sms), dim3(256), 0, st, cj, pj, h->status));
    // 2. LoRA down for gate/up: u_gu[:, j*RP:(j+1)*RP] = s x A_j^T (f16)
    lz.stage = MS_LORA_DOWN_GU;
    GemmCore core;
    core_init(core, T, 2 * RP, 128, RP, h->status);
    if (!map2d(&core.maps[0], x, true, d, T, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->ag;
    core.maps[3] = h->au;
    core.num_regions = 2;
    for (int j = 0; j <= 2; ++j) core.region_n0[j] = j * RP;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(128, 128, true, true), false, false);
    core.segs[0].b_map[1] = 3;
    core.num_segs = 1;
    EpiStore::Params ep = store_params(T, 2 * RP);
    set_out16(ep, 0, u_gu, 2 * RP, false, h->scale);
    ep.check_f16 = 1;
    enable_split(core, h->fsplit, h->split_cnt + 2 * kSplitCounters, h->fsplit_bytes);
    lz.done(launch_gemm<128, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  // 3. gate/up projection (+ LoRA up) with the SwiGLU epilogue: h (f16)
  lz.stage = MS_GATE_UP;
  {
    GemmCore core;
    core_init(core, T, 2 * I, 256, 128, h->status);
    core_pair(core);
    core.b_by_rank = 1;
    bool ok = map2d(&core.maps[0], x, true, d, T, d, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], u_gu, false, 2 * RP, T, 2 * RP, 128) &&
           map2d(&core.maps[4], bg2, false, 2 * RP, I, 2 * RP, 128) &&
           map2d(&core.maps[5], bu2, false, 2 * RP, I, 2 * RP, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wg;
    core.maps[3] = h->wu;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(256, 256, true, true), false, false);
    core.segs[0].b_map[1] = 3;
    core.num_segs = 1;
    if (r > 0) {
      core.segs[1] = seg1(1, 0, 4, 2 * RP / 64, idesc_f16(256, 256, false, false), false, false);
      core.segs[1].b_map[1] = 5;
      core.num_segs = 2;
    }
    EpiSwiGLU::Params ep{hh, g_sv, u_sv, T, I};
    lz.done(launch_gemm2<256, 6, EpiSwiGLU>(core, ep, h->num_sms, st));
  }
  // 4. LoRA down for down_proj: u_d = s h A_down^T (f16; training also bf16 hi + lo)
  if (r > 0) {
    lz.stage = MS_LORA_DOWN_D;
    GemmCore core;
    core_init(core, T, RP, RP, RP, h->status);
    if (!map2d(&core.maps[0], hh, false, I, T, I, 128) || !map2d(&core.maps[2], ad16, false, I, r, I, RP))
      return MOT_ERR_CUDA;
    core.segs[0] = seg1(0, 0, 2, I / 64, idesc_f16(128, RP, false, false), false, false);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(T, RP);
    set_out16(ep, 0, u_d, RP, false, h->scale);
    if (train) {
      set_out16(ep, 1, u_dhi, RP, true, h->scale);
      set_out16(ep, 2, u_dlo, RP, true, 1.0f, 1);
    }
    ep.check_f16 = 1;
    enable_split(core, h->fsplit, h->split_cnt + 2 * kSplitCounters, h->fsplit_bytes);
    lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
  }
  // 5. down projection (+ LoRA up): y bf16 and optional f32
  lz.stage = MS_DOWN;
  {
    GemmCore core;
    core_init(core, T, d, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], hh, false, I, T, I, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], u_d, false, RP, T, RP, 128) && map2d(&core.maps[3], bd16, false, r, d, r, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wd;
    core.segs[0] = seg1(0, 0, 2, I / 64, idesc_f16(256, 256, false, false), false, false);
    core.num_segs = 1;
    if (r > 0) {
      core.segs[1] = seg1(1, 0, 3, RP / 64, idesc_f16(256, 256, false, false), false, false);
      core.num_segs = 2;
    }
    EpiStore::Params ep = store_params(T, d);
    if (y) set_out16(ep, 0, y, d, true);
    ep.out32 = y_f32;
    ep.ld32 = d;
    ep.accumulate32 = residual ? 1 : 0;
    lz.done(launch_gemm2<256, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  return lz.finish();
}

}  // namespace

extern "C" {

mot_status mot_mlp_forward(mot_mlp_t h, const void* x, int32_t T, void* y, float* y_f32, void* saved,
                           size_t saved_bytes, void* workspace, size_t workspace_bytes, void* stream) {
  return mlp_forward_impl(h, x, T, y, y_f32, saved, saved_bytes, workspace, workspace_bytes, stream, false);
}

mot_status mot_mlp_backward(mot_mlp_t h, const void* dy, const void* x, int32_t T, const void* saved,
                            size_t saved_bytes, void* dx, float* dx_f32, float* const d_a[3], float* const d_b[3],
                            int32_t accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !dy || !x || !dx || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  const mot_mlp_config& c = h->cfg;
  if (!c.enable_backward) return MOT_ERR_INVALID_ARGUMENT;
  if (!saved) return MOT_ERR_NO_SAVED_STATE;
  if (T <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (T > c.max_tokens) return MOT_ERR_UNSUPPORTED_SHAPE;
  const int r = h->rank;
  if (r > 0) {
    if (!d_a || !d_b) return MOT_ERR_INVALID_ARGUMENT;
    for (int j = 0; j < 3; ++j)
      if (!d_a[j] || !d_b[j]) return MOT_ERR_INVALID_ARGUMENT;
  }
  const void* ptrs[] = {dy, x, dx, dx_f32, saved, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  if (r > 0)
    for (int j = 0; j < 3; ++j)
      if (!aligned16(d_a[j]) || !aligned16(d_b[j])) return MOT_ERR_ALIGNMENT;
  const MlpLayout L = make_mlp_layout(c, T, true);
  if (saved_bytes < L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (workspace_bytes < L.bwd_scratch) return MOT_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* act = static_cast<const uint8_t*>(saved);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const __half* u_gu = reinterpret_cast<const __half*>(act + L.o_ugu);
  const __half* hh = reinterpret_cast<const __half*>(act + L.o_h);
  const __half* g_sv = reinterpret_cast<const __half*>(act + L.o_g);
  const __half* u_sv = reinterpret_cast<const __half*>(act + L.o_u);
  const __nv_bfloat16* u_dhi = reinterpret_cast<const __nv_bfloat16*>(act + L.o_udhi);
  const __nv_bfloat16* u_dlo = reinterpret_cast<const __nv_bfloat16*>(act + L.o_udlo);
  __half* dgu = reinterpret_cast<__half*>(ws + L.b_dgu);
  __nv_bfloat16* gd_hi = reinterpret_cast<__nv_bfloat16*>(ws + L.b_gdhi);
  __nv_bfloat16* gd_lo = reinterpret_cast<__nv_bfloat16*>(ws + L.b_gdlo);
  __half* gd16 = reinterpret_cast<__half*>(ws + L.b_gd16);
  __nv_bfloat16* g_hi = reinterpret_cast<__nv_bfloat16*>(ws + L.b_ghi);
  __nv_bfloat16* g_lo = reinterpret_cast<__nv_bfloat16*>(ws + L.b_glo);
  __half* bg16 = reinterpret_cast<__half*>(ws + L.b_bg16);
  __half* bu16 = reinterpret_cast<__half*>(ws + L.b_bu16);
  void* split_ws = ws + L.b_split;
  void* split_ws_side = ws + L.b_split + kSplitWsBytes;
  int* split_cnt_side = h->split_cnt + kSplitCounters;

  const int d = c.hidden, I = c.intermediate, RP = h->RP;
  const int kb_tok = (T + 63) / 64;  // K blocks over tokens (zero-filled tail)
  MlpLaunches lz(h, st);

  if (r > 0) {
    // B_gate, B_up to f16 (they meet the f16 dg, du)
    lz.stage = MS_BWD_PREP;
    CvtJobs jobs{};
    jobs.src[0] = static_cast<const __nv_bfloat16*>(h->w.b_gate);
    jobs.dst[0] = bg16;
    jobs.src[1] = static_cast<const __nv_bfloat16*>(h->w.b_up);
    jobs.dst[1] = bu16;
    jobs.n8[0] = jobs.n8[1] = static_cast<long long>(I) * r / 8;
    jobs.count = 2;
    lz.done(launch_pdl(cvt_multi_kernel, dim3(64), dim3(256), 0, st, jobs, h->status));
    // g_d = dy B_down -> s g_d as bf16 hi + lo, and as f16
    lz.stage = MS_BWD_G_D;
    GemmCore core;
    core_init(core, T, RP, RP, RP, h->status);
    if (!map2d(&core.maps[0], dy, true, d, T, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->bd_mn;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(128, RP, true, true, false, true), false, true);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(T, RP);
    set_out16(ep, 0, gd_hi, RP, true, h->scale);
    set_out16(ep, 1, gd_lo, RP, true, 1.0f, 0);
    set_out16(ep, 2, gd16, RP, false, h->scale);
    ep.check_f16 = 1;
    enable_split(core, split_ws, h->split_cnt);
    lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
  }
  // dh = dy W_down + s g_d A_down, then dg = dh u silu'(g), du = dh silu(g) (f16 [T, 2I])
  lz.stage = MS_BWD_DH;
  {
    GemmCore core;
    core_init(core, T, I, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], dy, true, d, T, d, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], gd_hi, true, RP, T, RP, 128) && map2d(&core.maps[4], gd_lo, true, RP, T, RP, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wdT_k;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(256, 256, true, true), false, false);
    core.num_segs = 1;
    if (r > 0) {
      core.maps[3] = h->ad_mn;
      core.segs[1] = seg1(1, 0, 3, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      core.segs[2] = seg1(4, 0, 3, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      core.num_segs = 3;
    }
    EpiSwiGLUBwd::Params ep{dgu, g_sv, u_sv, T, I};
    lz.done(launch_gemm2<256, 6, EpiSwiGLUBwd>(core, ep, h->num_sms, st));
  }
  if (r > 0) {
    // dB_down and dA_down feed nothing later in this call: side stream
    lz.fork();
    // dB_down = dy^T u_d  [d, r], with u_d as its bf16 hi + lo pair
    lz.stage = MS_BWD_DB_D;
    {
      GemmCore core;
      core_init(core, d, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], dy, true, d, T, d) || !map2d_mn(&core.maps[2], u_dhi, true, RP, T, RP) ||
          !map2d_mn(&core.maps[3], u_dlo, true, RP, T, RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, true, true, true, true), true, true);
      set_dual(core.segs[0], 3);
      core.num_segs = 1;
      EpiStore::Params ep = store_params(d, r);
      ep.out32 = d_b[2];
      ep.ld32 = r;
      ep.accumulate32 = accumulate;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_dual<EpiStore>(RP, core, ep, h->num_sms, lz.cur));
    }
    // dA_down = (s g_d)^T h  [r, I], computed as its transpose h^T (s g_d)
    lz.stage = MS_BWD_DA_D;
    {
      GemmCore core;
      core_init(core, I, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], hh, false, I, T, I) || !map2d_mn(&core.maps[2], gd16, false, RP, T, RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, false, false, true, true), true, true);
      core.num_segs = 1;
      EpiStore::Params ep = store_params(I, r);
      ep.out32 = d_a[2];
      ep.ld32 = I;
      ep.accumulate32 = accumulate;
      ep.transpose32 = 1;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, lz.cur));
    }
    lz.to_main();
    // g_j = d{g,u} B_j for gate and up in one GEMM: column block j reads its
    // own K range of [dg | du] -> s g_j as bf16 hi + lo in columns [j RP, (j+1) RP)
    lz.stage = MS_BWD_G_GU;
    {
      GemmCore core;
      core_init(core, T, 2 * RP, RP, RP, h->status);
      if (!map2d(&core.maps[0], dgu, false, 2 * I, T, 2 * I, 128) ||
          !map2d_mn(&core.maps[2], bg16, false, r, I, r) || !map2d_mn(&core.maps[3], bu16, false, r, I, r))
        return MOT_ERR_CUDA;
      core.num_regions = 2;
      for (int j = 0; j <= 2; ++j) core.region_n0[j] = j * RP;
      core.segs[0] = seg1(0, 0, 2, I / 64, idesc_f16(128, RP, false, false, false, true), false, true);
      core.segs[0].a_k0[1] = I;
      core.segs[0].b_map[1] = 3;
      core.num_segs = 1;
      EpiStore::Params ep = store_params(T, 2 * RP);
      set_out16(ep, 0, g_hi, 2 * RP, true, h->scale);
      set_out16(ep, 1, g_lo, 2 * RP, true, 1.0f, 0);
      enable_split(core, split_ws, h->split_cnt);
      lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
    }
    lz.fork();
    // dB_j = d{g,u}^T u_j  [I, r] for gate and up in one GEMM: D rows are the
    // 2I columns of [dg | du], row block j meets u_gu's block j
    lz.stage = MS_BWD_DB_GU;
    {
      GemmCore core;
      core_init(core, 2 * I, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], dgu, false, 2 * I, T, 2 * I) ||
          !map2d_mn(&core.maps[2], u_gu, false, RP, T, 2 * RP) ||
          !map2d_mn(&core.maps[3], u_gu + RP, false, RP, T, 2 * RP))
        return MOT_ERR_CUDA;
      core.regions_on_m = 1;
      core.num_regions = 2;
      core.region_n0[0] = 0;
      core.region_n0[1] = I;
      core.region_n0[2] = 2 * I;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, false, false, true, true), true, true);
      core.segs[0].b_map[1] = 3;
      core.num_segs = 1;
      EpiRowBlocks::Params ep{};
      ep.out[0] = d_b[0];
      ep.out[1] = d_b[1];
      ep.row0[0] = 0;
      ep.row0[1] = I;
      ep.row0[2] = 2 * I;
      ep.row0[3] = 2 * I;
      ep.ld = r;
      ep.cols = r;
      ep.accumulate = accumulate;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_narrow<EpiRowBlocks>(RP, core, ep, h->num_sms, lz.cur));
    }
    // dA_j = (s g_j)^T x for gate and up in one GEMM over x^T, with (s g_j)
    // as its bf16 hi + lo pair; block j goes to dA_j transposed
    lz.stage = MS_BWD_DA_GU;
    {
      GemmCore core;
      const int bn = 2 * RP <= 192 ? 2 * RP : RP;
      core_init(core, d, 2 * RP, bn, RP, h->status);
      if (!map2d_mn(&core.maps[0], x, true, d, T, d) || !map2d_mn(&core.maps[2], g_hi, true, 2 * RP, T, 2 * RP) ||
          !map2d_mn(&core.maps[3], g_lo, true, 2 * RP, T, 2 * RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, bn, true, true, true, true), true, true);
      set_dual(core.segs[0], 3);
      core.num_segs = 1;
      EpiLoraGrad::Params ep{};
      ep.out[0] = d_a[0];
      ep.out[1] = d_a[1];
      ep.out[2] = nullptr;
      ep.ld = d;
      ep.RP = RP;
      ep.r = r;
      ep.M = d;
      ep.transpose = 1;
      ep.accumulate = accumulate;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_dual<EpiLoraGrad>(bn, core, ep, h->num_sms, lz.cur));
    }
    lz.to_main();
  }
  // dx = dg W_gate + du W_up + sum_j ((s g_j)_hi + (s g_j)_lo) A_j
  lz.stage = MS_BWD_DX;
  {
    GemmCore core;
    core_init(core, T, d, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], dgu, false, 2 * I, T, 2 * I, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], g_hi, true, 2 * RP, T, 2 * RP, 128) &&
           map2d(&core.maps[6], g_lo, true, 2 * RP, T, 2 * RP, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wguT_k;
    for (int j = 0; j < 2; ++j) {
      core.segs[j] = seg1(0, j * I, 2, I / 64, idesc_f16(256, 256, false, false), false, false);
      core.segs[j].b_k0 = j * I;
    }
    core.num_segs = 2;
    if (r > 0) {
      core.maps[4] = h->ag_mn;
      core.maps[5] = h->au_mn;
      for (int j = 0; j < 2; ++j) {
        core.segs[2 + j] = seg1(1, j * RP, 4 + j, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
        core.segs[4 + j] = seg1(6, j * RP, 4 + j, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      }
      core.num_segs = 6;
    }
    EpiStore::Params ep = store_params(T, d);
    set_out16(ep, 0, dx, d, true);
    ep.out32 = dx_f32;
    ep.ld32 = d;
    lz.done(launch_gemm2<256, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  return lz.finish();
}

mot_status mot_dev_mlp_profile(mot_mlp_t h, int32_t enable) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  if (enable && !h->ev[0])
    for (cudaEvent_t& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return MOT_ERR_CUDA;
  h->profile = enable != 0;
  h->stage_count = 0;
  return MOT_OK;
}

mot_status mot_dev_mlp_stage_times(mot_mlp_t h, int32_t* ids, float* ms, int32_t max, int32_t* count) {
  if (!h || !ids || !ms || max < 0 || !count) return MOT_ERR_INVALID_ARGUMENT;
  if (!h->profile) return MOT_ERR_INVALID_ARGUMENT;
  *count = h->stage_count;
  for (int i = 0; i < h->stage_count && i < max; ++i) {
    ids[i] = h->stage_ids[i];
    if (!h->stage_start[i] || !h->stage_end[i]) return MOT_ERR_CUDA;
    if (cudaEventSynchronize(h->stage_end[i]) != cudaSuccess ||
        cudaEventElapsedTime(&ms[i], h->stage_start[i], h->stage_end[i]) != cudaSuccess)
      return MOT_ERR_CUDA;
  }
  return MOT_OK;
}

const char* mot_dev_mlp_stage_name(int32_t id) {
  if (id >= 0 && id < static_cast<int32_t>(sizeof(kMlpStageNames) / sizeof(kMlpStageNames[0])))
    return kMlpStageNames[id];
  return "?";
}

}  // extern "C"
