// moe.cuh -- routing, dispatch and combine kernels of the gen-tower
// mixture-of-experts MLP ("SenseNova-U1" vLLM-Omni recipe, A3B variant: the
// generation branch routes over 32 experts, top-8, expert width 768; kernel
// table: top-k routing, fused_moe expert GEMMs, act_and_mul). The expert
// GEMMs themselves are the grouped CTA-pair GEMMs of gemm.cuh.
//
// Layout of the expert rows ("slots"): the (token, rank) pairs routed to
// expert e occupy rows [offset[e], offset[e] + count[e]) of the permuted
// buffers, each expert's block padded with zero rows to a multiple of 256
// (one M tile of the pair GEMM), so an M tile never spans two experts.
// Slots are assigned in token order, without atomics: the routing kernel
// takes one block per 64 tokens and numbers each expert's selections within
// the block, a scan over the blocks gives every block's base within each
// expert, and dispatch adds the two; the slot layout is the same on every
// run.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr int kMoeMaxExperts = 32;  // one lane per expert
constexpr int kMoeMaxTopK = 8;
constexpr int kMoeTileRows = 256;

constexpr int kMoeRouteWarps = 8;                        // warps per routing block
constexpr int kMoeRouteTokensPerWarp = 8;                // tokens each warp routes
constexpr int kMoeRouteTokens = kMoeRouteWarps * kMoeRouteTokensPerWarp;  // tokens per routing block

// Softmax over the E router logits of each token, its top_k experts (ties to
// the lower index) and their probabilities renormalised to sum to one; lane e
// holds expert e, block b takes tokens [64 b, 64 b + 64), eight per warp
// (their logits loaded together). Each lane finds its expert's rank directly
// (how many experts have a larger logit, or an equal one at a lower index:
// the order of the probabilities, which exp keeps), so the selection has no
// dependent rounds; the lanes ranked below top_k write their slot. Every
// selection gets its number within its block and expert in token order
// (topk_pos): lane e keeps a bit per token of its warp that chose expert e,
// the warps' counts are scanned in shared memory, and the number is the
// warp's base plus the bits below the token's. blk_cnt[e][b] is the block's
// count.
__global__ void __launch_bounds__(kMoeRouteWarps * 32) moe_route_kernel(
    const float* __restrict__ logits, int T, int E, int K, int* __restrict__ topk_idx, float* __restrict__ topk_w,
    int* __restrict__ topk_pos, int* __restrict__ blk_cnt) {
  __shared__ int warp_counts[kMoeRouteWarps][kMoeMaxExperts];
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool live = lane < E;
  const int t0 = blockIdx.x * kMoeRouteTokens + warp * kMoeRouteTokensPerWarp;
  float vv[kMoeRouteTokensPerWarp];
#pragma unroll
  for (int i = 0; i < kMoeRouteTokensPerWarp; ++i)
    vv[i] = (live && t0 + i < T) ? logits[static_cast<long long>(t0 + i) * E + lane] : -INFINITY;
  unsigned chosen = 0u;  // bit i: token t0 + i chose this lane's expert
  int rank_of[kMoeRouteTokensPerWarp];
#pragma unroll
  for (int i = 0; i < kMoeRouteTokensPerWarp; ++i) {
    rank_of[i] = 0;
    const int t = t0 + i;
    if (t >= T) break;
    const float v = vv[i];
    float m = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float p = live ? expf(v - m) : 0.f;
    float s = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    p = p / s;
    int rank = 0;
    for (int j = 0; j < E; ++j) {
      const float vj = __shfl_sync(0xffffffffu, v, j);
      rank += (vj > v || (vj == v && j < lane)) ? 1 : 0;
    }
    const bool sel = live && rank < K;
    float ws = sel ? p : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
    if (sel) {
      const long long pr = static_cast<long long>(t) * K + rank;
      topk_idx[pr] = lane;
      topk_w[pr] = p / ws;
      chosen |= 1u << i;
      rank_of[i] = rank;
    }
  }
  warp_counts[warp][lane] = __popc(chosen);
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_counts[w][lane];
#pragma unroll
  for (int i = 0; i < kMoeRouteTokensPerWarp; ++i)
    if (chosen & (1u << i))
      topk_pos[static_cast<long long>(t0 + i) * K + rank_of[i]] = base + __popc(chosen & ((1u << i) - 1u));
  if (threadIdx.x < E) {
    int total = 0;
    for (int w = 0; w < kMoeRouteWarps; ++w) total += warp_counts[w][threadIdx.x];
    blk_cnt[static_cast<long long>(threadIdx.x) * gridDim.x + blockIdx.x] = total;
  }
}

// Per expert: the exclusive scan of the routing blocks' counts (blk_base,
// expert-major like blk_cnt) and the total count; then the expert block
// offsets (each count padded to a multiple of 256), the M-tile table of the
// grouped GEMMs (expert of each 256-row tile, -1 past the used rows, for all
// `tiles` entries). One block of 32 warps, warp e
// scanning expert e: lane l sums a contiguous chunk of blocks (independent
// loads), the lanes' sums are scanned by shuffles, and each lane writes its
// chunk's running bases.
__global__ void __launch_bounds__(1024) moe_offsets_kernel(const int* __restrict__ blk_cnt, int nblk, int E,
                                                           int tiles, int* __restrict__ blk_base,
                                                           int* __restrict__ counts, int* __restrict__ offsets,
                                                           int* __restrict__ tile_expert) {
  grid_dep_launch();
  grid_dep_wait();
  __shared__ int cnt[kMoeMaxExperts];
  __shared__ int off[kMoeMaxExperts + 1];
  const int lane = threadIdx.x & 31, e = threadIdx.x >> 5;
  if (e < E) {
    const int chunk = (nblk + 31) / 32;
    const int b_lo = min(nblk, lane * chunk), b_hi = min(nblk, b_lo + chunk);
    const int* src = blk_cnt + static_cast<long long>(e) * nblk;
    int sum = 0;
#pragma unroll 8
    for (int b = b_lo; b < b_hi; ++b) sum += src[b];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    int running = incl - sum;
    int* dst = blk_base + static_cast<long long>(e) * nblk;
#pragma unroll 8
    for (int b = b_lo; b < b_hi; ++b) {
      dst[b] = running;
      running += src[b];
    }
    if (lane == 31) cnt[e] = incl;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0;
    for (int j = 0; j < E; ++j) {
      off[j] = o;
      offsets[j] = o;
      counts[j] = cnt[j];
      o += (cnt[j] + kMoeTileRows - 1) / kMoeTileRows * kMoeTileRows;
    }
    off[E] = o;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < tiles; i += blockDim.x) {
    const int r = i * kMoeTileRows;
    int ex = -1;
    for (int j = 0; j < E; ++j)
      if (r >= off[j] && r < off[j + 1]) ex = j;
    tile_expert[i] = ex;
  }
}

// Copies each token's row into the slot of every expert it was routed to,
// slot = offset[e] + the routing block's base within e + the selection's
// number within the block, and records the slot per (token, rank); then
// zeroes the padding rows of every expert block. One warp per token: the
// row's first 256 16-byte chunks are loaded before the slot lookups (they do
// not depend on them), and the row is written K times.
__global__ void __launch_bounds__(256) moe_dispatch_kernel(const __nv_bfloat16* __restrict__ x, int T, int K, int E,
                                                           int d, int nblk, const int* __restrict__ topk_idx,
                                                           const int* __restrict__ topk_pos,
                                                           const int* __restrict__ blk_base,
                                                           const int* __restrict__ offsets,
                                                           const int* __restrict__ counts,
                                                           __nv_bfloat16* __restrict__ xp, int* __restrict__ slot) {
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  const int warp0 = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int n16 = d / 8;  // 16-byte chunks per row
  for (int t = warp0; t < T; t += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(t) * d);
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (lane + 32 * i < n16) v[i] = src[lane + 32 * i];
    int pos = 0;
    if (lane < K) {
      const long long pr = static_cast<long long>(t) * K + lane;
      const int e = topk_idx[pr];
      pos = offsets[e] + blk_base[static_cast<long long>(e) * nblk + t / kMoeRouteTokens] + topk_pos[pr];
      slot[pr] = pos;
    }
    // the K slot rows (as row numbers: half the registers of pointers)
    int rowk[kMoeMaxTopK];
#pragma unroll
    for (int k = 0; k < kMoeMaxTopK; ++k) rowk[k] = __shfl_sync(0xffffffffu, pos, k);
    uint4* const xp4 = reinterpret_cast<uint4*>(xp);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = lane + 32 * i;
      if (c >= n16) break;
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k) {
        if (k >= K) break;
        xp4[static_cast<long long>(rowk[k]) * n16 + c] = v[i];
      }
    }
    for (int c = lane + 256; c < n16; c += 32) {
      const uint4 w = src[c];
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k) {
        if (k >= K) break;
        xp4[static_cast<long long>(rowk[k]) * n16 + c] = w;
      }
    }
  }
  // padding rows [offset + count, offset + round_up(count, 256)) of each expert
  for (int e = 0; e < E; ++e) {
    const int lo = offsets[e] + counts[e];
    const int hi = offsets[e] + (counts[e] + kMoeTileRows - 1) / kMoeTileRows * kMoeTileRows;
    for (int r = lo + warp0; r < hi; r += nwarps) {
      uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<long long>(r) * d);
      for (int c = lane; c < n16; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    }
  }
}

// y[t] = sum over ranks k (in order) of w[t, k] * yp[slot[t, k]] (yp: the f16
// expert outputs): f32 and bf16 = RNE(f32). One warp per token, d a multiple
// of 256; lane l takes 8 columns of every 256, two such chunks at a time so
// that 2 K row loads of 16 bytes are in flight.
__device__ __forceinline__ void moe_acc8(float (&acc)[8], const uint4& raw, float w) {
  const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
  }
}

__device__ __forceinline__ void moe_store8(const float (&acc)[8], __nv_bfloat16* y, float* y32, long long o) {
  if (y32) {
    *reinterpret_cast<float4*>(y32 + o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(y32 + o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  *reinterpret_cast<uint4*>(y + o) = make_uint4(pack_bf162(acc[0], acc[1]), pack_bf162(acc[2], acc[3]),
                                                pack_bf162(acc[4], acc[5]), pack_bf162(acc[6], acc[7]));
}

__global__ void __launch_bounds__(256) moe_combine_kernel(const __half* __restrict__ yp, int T, int K, int d,
                                                          const int* __restrict__ slot,
                                                          const float* __restrict__ topk_w,
                                                          __nv_bfloat16* __restrict__ y, float* __restrict__ y32) {
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int t = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); t < T; t += nwarps) {
    const __half* rows[kMoeMaxTopK];
    float wk[kMoeMaxTopK];
#pragma unroll
    for (int k = 0; k < kMoeMaxTopK; ++k) {
      const long long pr = static_cast<long long>(t) * K + k;
      rows[k] = yp + static_cast<long long>(k < K ? slot[pr] : 0) * d;
      wk[k] = k < K ? topk_w[pr] : 0.f;
    }
    for (int c = lane * 8; c < d; c += 512) {
      const bool two = c + 256 < d;
      uint4 a[kMoeMaxTopK], b[kMoeMaxTopK];
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k) {
        if (k < K) {
          a[k] = *reinterpret_cast<const uint4*>(rows[k] + c);
          if (two) b[k] = *reinterpret_cast<const uint4*>(rows[k] + c + 256);
        }
      }
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k)
        if (k < K) moe_acc8(acc, a[k], wk[k]);
      moe_store8(acc, y, y32, static_cast<long long>(t) * d + c);
      if (two) {
        float acc2[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kMoeMaxTopK; ++k)
          if (k < K) moe_acc8(acc2, b[k], wk[k]);
        moe_store8(acc2, y, y32, static_cast<long long>(t) * d + c + 256);
      }
    }
  }
}

}  // namespace mot
