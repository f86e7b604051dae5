// gemm.cuh -- persistent tcgen05 GEMM for sm_100a.
//
//   D[M, N] = sum_k A[m, k] B[n, k]            (main segment, K = 64 * kb_main)
//           + sum_k A2[m, a2_col + k] B2[n, k] (extension segment, K = 64 * kb_ext)
//
// The extension segment is how the LoRA up-projection rides on the base
// projection: A2 = u = s x A^T (already computed), B2 = lora_up, so
// x W^T + s (x A^T) B^T comes out of one accumulator with no extra pass
// ("SenseNova-U1" DiffSynth-Studio docs, training section: LoRA on the
// q/k/v/o_proj_mot_gen projections).
//
// Design: one CTA per SM, persistent over 128 x BN output tiles. Warp 0
// issues TMA loads into a STAGES-deep ring of 128-byte-swizzled K-major
// tiles; warp 1 issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM
// accumulators; warps 2..5 drain the other accumulator through the epilogue,
// so the epilogue of tile i overlaps the main loop of tile i+1.
// D columns are split into up to four regions, each with its own B / B2
// tensor (e.g. the q, k and v projections), so separate weight tensors feed
// one GEMM without being concatenated.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr int kGemmThreads = 192;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxMaps = 10;
constexpr int kMaxRegions = 4;

struct GemmRegion {
  int n_begin, n_end;  // D columns [n_begin, n_end); B rows are n - n_begin
  int b_map;           // maps[] index of the main-segment B tensor
  int b2_map;          // maps[] index of the extension B tensor (-1: none)
  int a2_col;          // first A2 column read by this region's extension
};

struct GemmCore {
  CUtensorMap maps[kMaxMaps];  // [0] A, [1] A2, [2..] B / B2 tensors
  GemmRegion regions[kMaxRegions];
  int num_regions;
  int M, N;
  int kb_main, kb_ext;
  int tiles_m, tiles_n;
  int b_box_rows;  // rows per B TMA box; BN is a multiple of it
  uint32_t idesc_main, idesc_ext;
  int* status;
};

template <class Epi>
struct GemmArgs {
  GemmCore core;
  typename Epi::Params epi;
};

__device__ __forceinline__ const GemmRegion& region_of(const GemmCore& g, int n) {
  int i = 0;
#pragma unroll 1
  while (i + 1 < g.num_regions && n >= g.regions[i].n_end) ++i;
  return g.regions[i];
}

// grouped tile order: 8 M-tiles share each sweep over N (L2 reuse of A rows)
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& tm, int& tn) {
  constexpr int G = 8;
  const int per_group = G * tiles_n;
  const int group = tile / per_group;
  const int first_m = group * G;
  const int gm = min(tiles_m - first_m, G);
  const int r = tile - group * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kBarOffset = STAGES * (kABytes + kBBytes);
  static constexpr uint32_t kBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
};

template <int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs<Epi> args) {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  using L = GemmSmem<BN, STAGES>;
  constexpr uint32_t kTmemCols = tmem_cols_for(2 * BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const GemmCore& g = args.core;
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kMaxMaps; ++i)
      if (i < 2 + 2 * kMaxRegions) tma_prefetch_desc(&g.maps[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitGuard wg{abort_flag, g.status};

  const int num_tiles = g.tiles_m * g.tiles_n;
  const int kb_total = g.kb_main + g.kb_ext;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int boxes = BN / g.b_box_rows;
      const uint32_t box_bytes = static_cast<uint32_t>(g.b_box_rows) * kBK * 2;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int tm, tn;
        tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
        const int m0 = tm * kBM, n0 = tn * BN;
        const GemmRegion& reg0 = region_of(g, n0);
        for (int kb = 0; kb < kb_total; ++kb) {
          mbar_wait(&empty[stage], phase ^ 1u, wg);
          mbar_expect_tx(&full[stage], L::kABytes + L::kBBytes);
          uint8_t* a_dst = sA + stage * L::kABytes;
          uint8_t* b_dst = sB + stage * L::kBBytes;
          if (kb < g.kb_main) {
            tma_load_2d(a_dst, &g.maps[0], &full[stage], kb * kBK, m0);
            for (int i = 0; i < boxes; ++i) {
              const int n = n0 + i * g.b_box_rows;
              const GemmRegion& r = region_of(g, n);
              tma_load_2d(b_dst + i * box_bytes, &g.maps[r.b_map], &full[stage], kb * kBK, n - r.n_begin);
            }
          } else {
            const int ke = kb - g.kb_main;
            tma_load_2d(a_dst, &g.maps[1], &full[stage], reg0.a2_col + ke * kBK, m0);
            for (int i = 0; i < boxes; ++i) {
              const int n = n0 + i * g.b_box_rows;
              const GemmRegion& r = region_of(g, n);
              tma_load_2d(b_dst + i * box_bytes, &g.maps[r.b2_map], &full[stage], ke * kBK, n - r.n_begin);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        mbar_wait(&tempty[acc], acc_phase ^ 1u, wg);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kb_total; ++kb) {
          mbar_wait(&full[stage], phase, wg);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * L::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * L::kBBytes);
          const uint32_t idesc = kb < g.kb_main ? g.idesc_main : g.idesc_ext;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss(d_tmem, kmajor_desc(a_addr, kk, L::kABytes), kmajor_desc(b_addr, kk, L::kBBytes), idesc,
                    (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32)
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int tm, tn;
      tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
      mbar_wait(&tfull[acc], acc_phase, wg);
      tc_fence_after();
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
      Epi::template apply<BN>(args.epi, taddr, tm * kBM, tn * BN, row, g.status);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ epilogues
__device__ __forceinline__ void load_row32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// out = scale * acc, stored as bf16/f16 and/or f32 (f32 optionally added to
// what is there). Rows >= M and columns >= N are skipped.
struct EpiStore {
  struct Params {
    void* out16;
    int out16_bf16;  // 1: bf16, 0: f16
    long long ld16;
    float* out32;
    long long ld32;
    int accumulate32;
    float scale;
    int M, N;
    int check_f16;  // flag f16 overflow
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    const int m = m0 + row;
    bool overflow = false;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      load_row32(taddr + c, v);
      if (m >= p.M || n0 + c >= p.N) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= p.scale;
      if (p.out32) {
        float4* dst = reinterpret_cast<float4*>(p.out32 + m * p.ld32 + n0 + c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float4 w = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          if (p.accumulate32) {
            const float4 o = dst[i];
            w.x += o.x;
            w.y += o.y;
            w.z += o.z;
            w.w += o.w;
          }
          dst[i] = w;
        }
      }
      if (p.out16) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out16) + m * p.ld16 + n0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          if (p.out16_bf16) {
            w.x = pack_bf162(v[8 * i + 0], v[8 * i + 1]);
            w.y = pack_bf162(v[8 * i + 2], v[8 * i + 3]);
            w.z = pack_bf162(v[8 * i + 4], v[8 * i + 5]);
            w.w = pack_bf162(v[8 * i + 6], v[8 * i + 7]);
          } else {
            w.x = pack_half2(v[8 * i + 0], v[8 * i + 1]);
            w.y = pack_half2(v[8 * i + 2], v[8 * i + 3]);
            w.z = pack_half2(v[8 * i + 4], v[8 * i + 5]);
            w.w = pack_half2(v[8 * i + 6], v[8 * i + 7]);
          }
          dst[i] = w;
        }
        if (p.check_f16) {
#pragma unroll
          for (int i = 0; i < 32; ++i) overflow |= fabsf(v[i]) > 65504.f;
        }
      }
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

// QKV epilogue: for q and k heads, per-head RMSNorm (gain after
// normalisation) then rotate-half RoPE at position prefix_len[b] + i; v heads
// pass through. Writes f16 q^ [B, Hq, N, dh] and the self rows of the
// attention key/value buffers [B, Hkv, Lcap, dh] at row prefix_len[b] + i.
// "SenseNova-U1" (vLLM-Omni recipe), kernel table: the fused "RMSNorm +
// RoPE" step, here folded into the projection's epilogue.
struct EpiQkv {
  struct Params {
    __half* q_out;
    __half* k_out;
    __half* v_out;
    __half* xhat;  // [M, (Hq+Hkv)*dh] normalised pre-gain q/k (training) or null
    float* rstd;   // [M, Hq+Hkv] (training) or null
    const float* gamma_q;
    const float* gamma_k;
    const float2* rope;  // [positions][64] (cos, sin)
    int plen[kMaxBatch];
    int N, Hq, Hkv, Lcap, M;
    float eps;
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    static_assert(BN % 128 == 0, "whole heads per tile");
    const int m = m0 + row;
    const bool valid = m < p.M;
    const int b = valid ? m / p.N : 0;
    const int n = valid ? m - b * p.N : 0;
    const int pos = p.plen[b] + n;
    bool overflow = false;
#pragma unroll 1
    for (int hc = 0; hc < BN / 128; ++hc) {
      float v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + hc * 128 + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[c * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_ld_wait();
      if (!valid) continue;
      const int head = (n0 >> 7) + hc;
      __half* dst;
      if (head < p.Hq + p.Hkv) {
        const bool is_q = head < p.Hq;
        const float* gamma = is_q ? p.gamma_q : p.gamma_k;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) ss = fmaf(v[i], v[i], ss);
        const float rs = rsqrtf(ss * (1.0f / 128.0f) + p.eps);
        if (p.xhat) {
          uint4* xd = reinterpret_cast<uint4*>(p.xhat + static_cast<long long>(m) * (p.Hq + p.Hkv) * 128 + head * 128);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            uint4 w;
            w.x = pack_half2(v[8 * i + 0] * rs, v[8 * i + 1] * rs);
            w.y = pack_half2(v[8 * i + 2] * rs, v[8 * i + 3] * rs);
            w.z = pack_half2(v[8 * i + 4] * rs, v[8 * i + 5] * rs);
            w.w = pack_half2(v[8 * i + 6] * rs, v[8 * i + 7] * rs);
            xd[i] = w;
          }
          p.rstd[static_cast<long long>(m) * (p.Hq + p.Hkv) + head] = rs;
        }
        const float2* cs = p.rope + static_cast<long long>(pos) * 64;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float2 t = __ldg(cs + j);
          const float a = v[j] * rs * __ldg(gamma + j);
          const float c = v[j + 64] * rs * __ldg(gamma + j + 64);
          v[j] = a * t.x - c * t.y;
          v[j + 64] = c * t.x + a * t.y;
        }
        dst = is_q ? p.q_out + (static_cast<long long>(b * p.Hq + head) * p.N + n) * 128
                   : p.k_out + (static_cast<long long>(b * p.Hkv + head - p.Hq) * p.Lcap + pos) * 128;
      } else {
        dst = p.v_out + (static_cast<long long>(b * p.Hkv + head - p.Hq - p.Hkv) * p.Lcap + pos) * 128;
      }
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        uint4 w;
        w.x = pack_half2(v[8 * i + 0], v[8 * i + 1]);
        w.y = pack_half2(v[8 * i + 2], v[8 * i + 3]);
        w.z = pack_half2(v[8 * i + 4], v[8 * i + 5]);
        w.w = pack_half2(v[8 * i + 6], v[8 * i + 7]);
        d4[i] = w;
      }
#pragma unroll
      for (int i = 0; i < 128; ++i) overflow |= fabsf(v[i]) > 65504.f;
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

}  // namespace mot
