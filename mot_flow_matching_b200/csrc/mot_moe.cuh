// mot_moe.cuh -- C ABI of the A3B gen-tower mixture-of-experts MLP (see
// include/mot_moe.h). Same translation unit as mot_attn.cu.
//
// Launch sequence on the caller's stream (T tokens, E experts, top K, width I):
//   router GEMM      logits = x W_r^T (f32 [T, E]), 1-CTA, split-K
//   moe_route        softmax, top K, renormalised weights, per-block numbering
//   moe_offsets      per-expert scan over the routing blocks, expert blocks
//                    padded to 256 rows, M-tile -> expert table
//   moe_dispatch     x rows gathered into their experts' slots, padding zeroed
//   gate/up GEMM     grouped CTA pairs (rank 0 W_gate rows, rank 1 W_up rows
//                    of the tile's expert) with the SwiGLU epilogue -> f16 h
//   down GEMM        grouped CTA pairs, h W_down^T (f16 copy) -> f16 per slot
//   moe_combine      y = sum_k w_k (slot rows) in f32; f32 and bf16 out
#pragma once

#include "mot_moe.h"
#include "moe.cuh"

struct mot_moe {
  mot_moe_config cfg;
  mot_moe_weights w;
  int num_sms = 148;
  int* status = nullptr;
  int* split_cnt = nullptr;
  void* fsplit = nullptr;
  size_t fsplit_bytes = 0;
  __half* wd16 = nullptr;  // [E, d, I] f16 copy of w_down
  CUtensorMap wr_map, wg_map, wu_map, wd_map;
};

namespace {

struct MoeLayout {
  int tiles = 0, rows = 0, nblk = 0;
  size_t logits = 0, idx = 0, wts = 0, pos = 0, blk_cnt = 0, blk_base = 0, small = 0, tile_expert = 0, slot = 0,
         xp = 0, hp = 0, yp = 0, total = 0;
};

MoeLayout make_moe_layout(const mot_moe_config& c, int T) {
  MoeLayout L;
  const size_t d = c.hidden, I = c.intermediate, E = c.experts, K = c.top_k, t = T;
  L.tiles = static_cast<int>((t * K + kMoeTileRows - 1) / kMoeTileRows + E);
  L.rows = L.tiles * kMoeTileRows;
  L.nblk = static_cast<int>((t + kMoeRouteTokens - 1) / kMoeRouteTokens);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 1024);
    return o;
  };
  L.logits = take(t * E * 4);
  L.idx = take(t * K * 4);
  L.wts = take(t * K * 4);
  L.pos = take(t * K * 4);
  L.blk_cnt = take(static_cast<size_t>(L.nblk) * E * 4);
  L.blk_base = take(static_cast<size_t>(L.nblk) * E * 4);
  L.small = take(2 * kMoeMaxExperts * 4);  // counts, offsets
  L.tile_expert = take(static_cast<size_t>(L.tiles) * 4);
  L.slot = take(t * K * 4);
  L.xp = take(static_cast<size_t>(L.rows) * d * 2);
  L.hp = take(static_cast<size_t>(L.rows) * I * 2);
  L.yp = take(static_cast<size_t>(L.rows) * d * 2);
  L.total = off;
  return L;
}

mot_status check_moe_config(const mot_moe_config* c) {
  if (!c || c->hidden <= 0 || c->intermediate <= 0 || c->experts <= 0 || c->top_k <= 0 || c->max_tokens <= 0)
    return MOT_ERR_INVALID_ARGUMENT;
  if (c->hidden % 256 != 0 || c->intermediate % 128 != 0 || c->experts > kMoeMaxExperts ||
      c->top_k > std::min(kMoeMaxTopK, c->experts) || static_cast<long long>(c->max_tokens) * c->top_k > (1ll << 28))
    return MOT_ERR_UNSUPPORTED_SHAPE;
  return MOT_OK;
}

void release_moe(mot_moe* h) {
  if (!h) return;
  cudaFree(h->status);
  cudaFree(h->split_cnt);
  cudaFree(h->fsplit);
  cudaFree(h->wd16);
  delete h;
}

}  // namespace

extern "C" {

mot_status mot_moe_query_workspace(const mot_moe_config* cfg, int32_t T, size_t* workspace_bytes) {
  const mot_status st = check_moe_config(cfg);
  if (st != MOT_OK) return st;
  if (!workspace_bytes || T <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (T > cfg->max_tokens) return MOT_ERR_UNSUPPORTED_SHAPE;
  *workspace_bytes = make_moe_layout(*cfg, T).total;
  return MOT_OK;
}

mot_status mot_moe_create(const mot_moe_config* cfg, const mot_moe_weights* wts, void* stream, mot_moe_t* out) {
  if (!out) return MOT_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  const mot_status st = check_moe_config(cfg);
  if (st != MOT_OK) return st;
  if (!wts || !wts->w_router || !wts->w_gate || !wts->w_up || !wts->w_down) return MOT_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {wts->w_router, wts->w_gate, wts->w_up, wts->w_down};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOT_ERR_ALIGNMENT;
  if (!encode_ready()) return MOT_ERR_CUDA;
  mot_moe* h = new (std::nothrow) mot_moe();
  if (!h) return MOT_ERR_CUDA;
  h->cfg = *cfg;
  h->w = *wts;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t d = cfg->hidden, I = cfg->intermediate, E = cfg->experts;
  // the router GEMM's split-K partials: up to 8 splits of every 128-row tile, 64 f32 columns
  const size_t tiles = (static_cast<size_t>(cfg->max_tokens) + kBM - 1) / kBM;
  h->fsplit_bytes = std::min(kSplitWsBytes * 2, tiles * 8 * 64 * kBM * 4);
  bool ok = cudaMalloc(&h->status, sizeof(int)) == cudaSuccess &&
            cudaMalloc(&h->split_cnt, kSplitCounters * sizeof(int)) == cudaSuccess &&
            cudaMemset(h->split_cnt, 0, kSplitCounters * sizeof(int)) == cudaSuccess &&
            cudaMalloc(&h->fsplit, h->fsplit_bytes) == cudaSuccess &&
            cudaMalloc(&h->wd16, E * d * I * 2) == cudaSuccess;
  if (ok) {
    ok = cudaMemsetAsync(h->status, 0, sizeof(int), s) == cudaSuccess;
    CvtJobs jobs{};
    jobs.src[0] = static_cast<const __nv_bfloat16*>(wts->w_down);
    jobs.dst[0] = h->wd16;
    jobs.n8[0] = static_cast<long long>(E * d * I / 8);
    jobs.count = 1;
    cvt_multi_kernel<<<4 * h->num_sms, 256, 0, s>>>(jobs, h->status);
    ok = ok && cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess &&
         map2d(&h->wr_map, wts->w_router, true, d, E, d, 64) &&
         map2d(&h->wg_map, wts->w_gate, true, d, E * I, d, 128) &&
         map2d(&h->wu_map, wts->w_up, true, d, E * I, d, 128) && map2d(&h->wd_map, h->wd16, false, I, E * d, I, 128);
  }
  if (!ok) {
    release_moe(h);
    return MOT_ERR_CUDA;
  }
  *out = h;
  return MOT_OK;
}

void mot_moe_destroy(mot_moe_t h) { release_moe(h); }

mot_status mot_moe_get_device_status(mot_moe_t h, void* stream) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  int v = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return MOT_ERR_CUDA;
  if (v & DEV_ERR_TIMEOUT) {
    if (cudaMemset(h->split_cnt, 0, kSplitCounters * sizeof(int)) != cudaSuccess) return MOT_ERR_CUDA;
    return MOT_ERR_TIMEOUT;
  }
  if (v & DEV_ERR_NUMERIC) return MOT_ERR_NUMERIC;
  return MOT_OK;
}

mot_status mot_moe_forward(mot_moe_t h, const void* x, int32_t T, void* y, float* y_f32, int32_t* experts_out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !x || !y || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  const mot_moe_config& c = h->cfg;
  if (T <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (T > c.max_tokens) return MOT_ERR_UNSUPPORTED_SHAPE;
  const void* ptrs[] = {x, y, y_f32, experts_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  const MoeLayout L = make_moe_layout(c, T);
  if (workspace_bytes < L.total) return MOT_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  int* idx = reinterpret_cast<int*>(ws + L.idx);
  float* wts = reinterpret_cast<float*>(ws + L.wts);
  int* pos = reinterpret_cast<int*>(ws + L.pos);
  int* blk_cnt = reinterpret_cast<int*>(ws + L.blk_cnt);
  int* blk_base = reinterpret_cast<int*>(ws + L.blk_base);
  int* counts = reinterpret_cast<int*>(ws + L.small);
  int* offsets = counts + kMoeMaxExperts;
  int* tile_expert = reinterpret_cast<int*>(ws + L.tile_expert);
  int* slot = reinterpret_cast<int*>(ws + L.slot);
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(ws + L.xp);
  __half* hp = reinterpret_cast<__half*>(ws + L.hp);
  __half* yp = reinterpret_cast<__half*>(ws + L.yp);
  const int d = c.hidden, I = c.intermediate, E = c.experts, K = c.top_k;
  cudaError_t e = cudaSuccess;
  // router logits
  {
    GemmCore core;
    core_init(core, T, E, 64, 64, h->status);
    if (!map2d(&core.maps[0], x, true, d, T, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->wr_map;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(128, 64, true, true), false, false);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(T, E);
    ep.out32 = logits;
    ep.ld32 = E;
    enable_split(core, h->fsplit, h->split_cnt, h->fsplit_bytes);
    e = launch_gemm_narrow<EpiStore>(64, core, ep, h->num_sms, st);
  }
  const int warps_grid = std::max(1, std::min((T + 7) / 8, 16 * h->num_sms));
  if (e == cudaSuccess)
    e = launch_pdl(moe_route_kernel, dim3(L.nblk), dim3(kMoeRouteWarps * 32), 0, st,
                   static_cast<const float*>(logits), T, E, K, idx, wts, pos, blk_cnt);
  if (e == cudaSuccess)
    e = launch_pdl(moe_offsets_kernel, dim3(1), dim3(1024), 0, st, static_cast<const int*>(blk_cnt), L.nblk, E,
                   L.tiles, blk_base, counts, offsets, tile_expert);
  if (e == cudaSuccess)
    e = launch_pdl(moe_dispatch_kernel, dim3(warps_grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), T,
                   K, E, d, L.nblk, static_cast<const int*>(idx), static_cast<const int*>(pos),
                   static_cast<const int*>(blk_base), static_cast<const int*>(offsets),
                   static_cast<const int*>(counts), xp, slot);
  // gate/up of every slot's expert, SwiGLU -> h (f16)
  if (e == cudaSuccess) {
    GemmCore core;
    core_init(core, L.rows, 2 * I, 256, 128, h->status);
    core_pair(core);
    core.b_by_rank = 1;
    core.tile_group = tile_expert;
    core.group_rows = I;
    if (!map2d(&core.maps[0], xp, true, d, L.rows, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->wg_map;
    core.maps[3] = h->wu_map;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(256, 256, true, true), false, false);
    core.segs[0].b_map[1] = 3;
    core.num_segs = 1;
    EpiSwiGLU::Params ep{hp, nullptr, nullptr, L.rows, I};
    e = launch_gemm2<256, 6, EpiSwiGLU>(core, ep, h->num_sms, st);
  }
  // down projection of every slot's expert -> f16 slot rows (overflow latched)
  if (e == cudaSuccess) {
    GemmCore core;
    core_init(core, L.rows, d, 256, 128, h->status);
    core_pair(core);
    core.tile_group = tile_expert;
    core.group_rows = d;
    if (!map2d(&core.maps[0], hp, false, I, L.rows, I, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->wd_map;
    core.segs[0] = seg1(0, 0, 2, I / 64, idesc_f16(256, 256, false, false), false, false);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(L.rows, d);
    set_out16(ep, 0, yp, d, false);
    ep.check_f16 = 1;
    e = launch_gemm2<256, 6, EpiStore>(core, ep, h->num_sms, st);
  }
  if (e == cudaSuccess)
    e = launch_pdl(moe_combine_kernel, dim3(warps_grid), dim3(256), 0, st, static_cast<const __half*>(yp), T, K, d,
                   static_cast<const int*>(slot), static_cast<const float*>(wts), static_cast<__nv_bfloat16*>(y),
                   y_f32);
  if (e == cudaSuccess && experts_out)
    e = cudaMemcpyAsync(experts_out, idx, static_cast<size_t>(T) * K * sizeof(int), cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

}  // extern "C"
