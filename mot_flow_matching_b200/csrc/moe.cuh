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
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr int kMoeMaxExperts = 32;  // one lane per expert
constexpr int kMoeMaxTopK = 8;
constexpr int kMoeTileRows = 256;

// Softmax over the E router logits of each token, its top_k experts (ties to
// the lower index) and their probabilities renormalised to sum to one; one
// warp per token, lane e holds expert e. Each lane finds its expert's rank
// directly (how many experts have a larger logit, or an equal one at a lower
// index: the order of the probabilities, which exp keeps), so the selection
// has no dependent rounds; the lanes ranked below top_k write their slot.
// counts[e] gains one per selection (summed per block in shared memory).
__global__ void __launch_bounds__(256) moe_route_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                        int* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                        int* __restrict__ counts) {
  __shared__ int block_counts[kMoeMaxExperts];
  if (threadIdx.x < kMoeMaxExperts) block_counts[threadIdx.x] = 0;
  __syncthreads();
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const bool live = lane < E;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int t = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); t < T; t += nwarps) {
    const float v = live ? logits[static_cast<long long>(t) * E + lane] : -INFINITY;
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
      topk_idx[static_cast<long long>(t) * K + rank] = lane;
      topk_w[static_cast<long long>(t) * K + rank] = p / ws;
      atomicAdd(&block_counts[lane], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < E && block_counts[threadIdx.x] > 0) atomicAdd(&counts[threadIdx.x], block_counts[threadIdx.x]);
}

// Expert block offsets (each count padded to a multiple of 256), the M-tile
// table of the grouped GEMMs (expert of each 256-row tile, -1 past the
// used rows, for all `tiles` entries), the total row count, and zeroed fill
// counters. One block.
__global__ void moe_offsets_kernel(const int* __restrict__ counts, int E, int tiles, int* __restrict__ offsets,
                                   int* __restrict__ tile_expert, int* __restrict__ total_rows,
                                   int* __restrict__ fill) {
  grid_dep_launch();
  grid_dep_wait();
  __shared__ int off[kMoeMaxExperts + 1];
  if (threadIdx.x == 0) {
    int o = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = o;
      offsets[e] = o;
      o += (counts[e] + kMoeTileRows - 1) / kMoeTileRows * kMoeTileRows;
      fill[e] = 0;
    }
    off[E] = o;
    *total_rows = o;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < tiles; i += blockDim.x) {
    const int r = i * kMoeTileRows;
    int e = -1;
    for (int j = 0; j < E; ++j)
      if (r >= off[j] && r < off[j + 1]) e = j;
    tile_expert[i] = e;
  }
}

// Copies each token's row into the slot of every expert it was routed to
// (slot order within an expert follows arrival; every row of an expert's
// GEMM is computed independently, so the block's result does not depend on
// it) and records the slot per (token, rank); then zeroes the padding rows
// of every expert block. One warp per token: lanes 0..K-1 claim the K slots
// at once, and the row is read once and written K times.
__global__ void __launch_bounds__(256) moe_dispatch_kernel(const __nv_bfloat16* __restrict__ x, int T, int K, int d,
                                                           const int* __restrict__ topk_idx,
                                                           const int* __restrict__ offsets,
                                                           const int* __restrict__ counts, int* __restrict__ fill,
                                                           const int* __restrict__ tile_expert,
                                                           const int* __restrict__ total_rows,
                                                           __nv_bfloat16* __restrict__ xp, int* __restrict__ slot) {
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  const int warp0 = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int n16 = d / 8;  // 16-byte chunks per row
  for (int t = warp0; t < T; t += nwarps) {
    int pos = 0;
    if (lane < K) {
      const long long pr = static_cast<long long>(t) * K + lane;
      const int e = topk_idx[pr];
      pos = offsets[e] + atomicAdd(&fill[e], 1);
      slot[pr] = pos;
    }
    uint4* dst[kMoeMaxTopK];
#pragma unroll
    for (int k = 0; k < kMoeMaxTopK; ++k)
      dst[k] = reinterpret_cast<uint4*>(xp + static_cast<long long>(__shfl_sync(0xffffffffu, pos, k)) * d);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(t) * d);
    for (int c = lane; c < n16; c += 32) {
      const uint4 v = src[c];
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k) {
        if (k >= K) break;
        dst[k][c] = v;
      }
    }
  }
  const int rows = *total_rows;
  for (int r = warp0; r < rows; r += nwarps) {
    const int e = tile_expert[r / kMoeTileRows];
    if (e < 0 || r - offsets[e] < counts[e]) continue;
    uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<long long>(r) * d);
    for (int c = lane; c < n16; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
  }
}

// y[t] = sum over ranks k (in order) of w[t, k] * yp[slot[t, k]] (yp: the f16
// expert outputs): f32 and bf16 = RNE(f32). One warp per token, d a multiple
// of 128.
__global__ void __launch_bounds__(256) moe_combine_kernel(const __half* __restrict__ yp, int T, int K, int d,
                                                          const int* __restrict__ slot,
                                                          const float* __restrict__ topk_w,
                                                          __nv_bfloat16* __restrict__ y, float* __restrict__ y32) {
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int t = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); t < T; t += nwarps) {
    int sl[kMoeMaxTopK];
    float wk[kMoeMaxTopK];
#pragma unroll
    for (int k = 0; k < kMoeMaxTopK; ++k) {
      const long long pr = static_cast<long long>(t) * K + k;
      sl[k] = k < K ? slot[pr] : 0;
      wk[k] = k < K ? topk_w[pr] : 0.f;
    }
    for (int c = lane * 4; c < d; c += 128) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kMoeMaxTopK; ++k) {
        if (k >= K) break;
        const uint2 raw = *reinterpret_cast<const uint2*>(yp + static_cast<long long>(sl[k]) * d + c);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        acc.x = fmaf(wk[k], a.x, acc.x);
        acc.y = fmaf(wk[k], a.y, acc.y);
        acc.z = fmaf(wk[k], b.x, acc.z);
        acc.w = fmaf(wk[k], b.y, acc.w);
      }
      const long long o = static_cast<long long>(t) * d + c;
      if (y32) *reinterpret_cast<float4*>(y32 + o) = acc;
      *reinterpret_cast<uint2*>(y + o) = make_uint2(pack_bf162(acc.x, acc.y), pack_bf162(acc.z, acc.w));
    }
  }
}

}  // namespace mot
