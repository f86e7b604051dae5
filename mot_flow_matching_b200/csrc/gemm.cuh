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
constexpr int kMaxSegs = 9;
constexpr uint32_t kMnBoxBytes = 64 * 64 * 2;  // MN-major TMA box: 64 MN x 64 K, 16-bit

// One K segment: D += A[:, a_k0 + k] B[:, b_k0 + k] over kb 64-wide blocks.
// A and B may each be K-major (row = M or N index, K contiguous) or MN-major
// (row = K index, M or N contiguous); MN-major tiles are loaded as 64 x 64
// TMA boxes and described to the tensor core as transposed operands.
struct GemmSeg {
  int a_map;
  int a_k0[kMaxRegions];   // per region (the LoRA extension reads a different u slice per region)
  int b_map[kMaxRegions];  // per region B tensor
  int b_k0;
  int kb;
  uint32_t idesc;
  int a_mn, b_mn;
  // dual (1-CTA kernel instantiated with kDual): every k-block also loads a
  // second B tile from b2_map and both products accumulate into D, so the A
  // tile is read once for two B operands (a bf16 hi + lo pair)
  int dual;
  int b2_map[kMaxRegions];
  // 1-CTA kernel: per-region k-block count (0 = kb), for regions that own
  // fewer K columns than the first
  int kb_r[kMaxRegions];
};

__device__ __forceinline__ int seg_kb(const GemmSeg& sg, int reg) { return sg.kb_r[reg] > 0 ? sg.kb_r[reg] : sg.kb; }

struct GemmCore {
  CUtensorMap maps[kMaxMaps];
  int region_n0[kMaxRegions + 1];  // region i covers D columns [region_n0[i], region_n0[i+1])
  int num_regions;
  int regions_on_m;  // 1-CTA kernel: regions split D rows instead (region_n0 then holds row bounds)
  GemmSeg segs[kMaxSegs];
  int num_segs;
  int M, N;
  int tiles_m, tiles_n;
  int b_box_rows;  // rows per K-major B TMA box; BN is a multiple of it
  int* status;
  // split-K (1-CTA kernel only): work item = (tile, split); split s of a
  // tile whose segments hold T k-blocks in its region takes k-blocks
  // [s T / k_splits, (s+1) T / k_splits) of the concatenated segments and
  // writes its f32 partial tile to split_ws; the CTA that finishes a tile
  // last (per-tile counter in split_cnt, which it resets) sums the partials
  // in split order into TMEM and runs the epilogue.
  // pair kernel: the B rows of CTA rank r come from b_map[r] of every
  // segment at rows [tn * BN/2, tn * BN/2 + BN/2) (regions unused), so one
  // 256-column tile holds BN/2 columns of two different weights for the same
  // output indices (the gate and up halves of a SwiGLU projection)
  int b_by_rank;
  // pair kernel, grouped GEMM (mixture of experts): M tile tm (256 rows)
  // belongs to group tile_group[tm] (device memory, written by an earlier
  // kernel; -1: an unused tile, skipped by every role), whose B rows start
  // at tile_group[tm] * group_rows of each B tensor (the experts' weights
  // stacked along rows)
  const int* tile_group;
  int group_rows;
  int k_splits;  // 1 = off
  int total_kb;  // host side: the smallest K-block total of any tile (bounds the split count)
  float4* split_ws;  // [tiles * k_splits][BN / 4][128]
  int* split_cnt;    // [tiles], zero between launches
  size_t split_cap;  // bytes at split_ws (host side: bounds the split count)
};

template <class Epi>
struct GemmArgs {
  GemmCore core;
  typename Epi::Params epi;
};

__device__ __forceinline__ int region_of(const GemmCore& g, int n) {
  int i = 0;
#pragma unroll 1
  while (i + 1 < g.num_regions && n >= g.region_n0[i + 1]) ++i;
  return i;
}

// grouped tile order: 16 M-tiles share each sweep over N, so A's rows stay in
// L2 across the sweep and B is streamed once per group (the 8192-row QKV
// projection reads its 50 MB of weights twice instead of four times)
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& tm, int& tn) {
  constexpr int G = 16;
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

template <int BN, int STAGES, bool kDual = false>
struct GemmSmem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kBBytes = BN * kBK * 2;                  // one B tile
  static constexpr uint32_t kBStage = kDual ? 2 * kBBytes : kBBytes;  // B tiles of a stage
  static constexpr uint32_t kBarOffset = STAGES * (kABytes + kBStage);
  static constexpr uint32_t kBytes = kBarOffset + 256 + 1024;  // barriers + alignment slack
};

template <int BN, int STAGES, class Epi, bool kDual = false>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs<Epi> args) {
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "UMMA N for M=128, whole 64-column boxes");
  using L = GemmSmem<BN, STAGES, kDual>;
  constexpr uint32_t kTmemCols = tmem_cols_for(2 * BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kABytes;  // stage s: B tile(s) at s * kBStage
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
    // pull every tensor map the segments use into the descriptor cache
    for (int si = 0; si < g.num_segs; ++si) {
      tma_prefetch_desc(&g.maps[g.segs[si].a_map]);
      for (int r = 0; r < g.num_regions; ++r) tma_prefetch_desc(&g.maps[g.segs[si].b_map[r]]);
    }
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
  grid_dep_launch();
  grid_dep_wait();  // every global access of this kernel comes after this

  const int num_tiles = g.tiles_m * g.tiles_n;
  const bool rows_reg = g.regions_on_m != 0;
  const int splits = g.k_splits > 1 ? g.k_splits : 1;
  const int num_items = num_tiles * splits;

  // Both issuing threads copy what they need out of the parameter block into
  // registers before their K loops: the TMA / MMA wrappers clobber memory, so
  // fields read through a reference would be re-fetched after every issue.
  const int num_segs = g.num_segs;
  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int b_box_rows = g.b_box_rows;
      for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
        const int tile = item / splits, split = item - tile * splits;
        int tm, tn;
        tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
        const int m0 = tm * kBM, n0 = tn * BN;
        const int reg0 = region_of(g, rows_reg ? m0 : n0);
        int tile_kb = 0;
        for (int si = 0; si < num_segs; ++si) tile_kb += seg_kb(g.segs[si], reg0);
        const int kb_lo = split * tile_kb / splits, kb_hi = (split + 1) * tile_kb / splits;
        int gk = 0;  // k-blocks of the segments before this one
        for (int si = 0; si < num_segs; ++si) {
          const GemmSeg& sg = g.segs[si];
          const int a_mn = sg.a_mn, b_mn = sg.b_mn, nkb = seg_kb(sg, reg0), a_k0 = sg.a_k0[reg0], b_k0 = sg.b_k0;
          const int kb0 = max(0, kb_lo - gk), kb1 = min(nkb, kb_hi - gk);
          gk += nkb;
          const bool dual = kDual && sg.dual;
          const CUtensorMap* amap = &g.maps[sg.a_map];
          // B boxes of this tile: up to 4 (map, row/column offset) pairs
          const int box_n = b_mn ? 64 : b_box_rows;
          const int nbox = BN / box_n;
          const CUtensorMap* bmap[4];
          const CUtensorMap* bmap2[4];
          int bcoord[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int n = n0 + (i < nbox ? i : 0) * box_n;
            const int r = rows_reg ? reg0 : region_of(g, n);
            bmap[i] = &g.maps[sg.b_map[r]];
            bmap2[i] = &g.maps[sg.b2_map[r]];
            bcoord[i] = rows_reg ? n : n - g.region_n0[r];
          }
          const uint32_t box_bytes = static_cast<uint32_t>(box_n) * kBK * 2;
          for (int kb = kb0; kb < kb1; ++kb) {
            mbar_wait(&empty[stage], phase ^ 1u, wg);
            mbar_expect_tx(&full[stage], L::kABytes + (dual ? 2 : 1) * L::kBBytes);
            uint8_t* a_dst = sA + stage * L::kABytes;
            uint8_t* b_dst = sB + stage * L::kBStage;
            const int ka = a_k0 + kb * kBK, kbk = b_k0 + kb * kBK;
            if (a_mn) {
              tma_load_2d(a_dst, amap, &full[stage], m0, ka);
              tma_load_2d(a_dst + kMnBoxBytes, amap, &full[stage], m0 + 64, ka);
            } else {
              tma_load_2d(a_dst, amap, &full[stage], ka, m0);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (i >= nbox) break;
              if (b_mn)
                tma_load_2d(b_dst + i * box_bytes, bmap[i], &full[stage], bcoord[i], kbk);
              else
                tma_load_2d(b_dst + i * box_bytes, bmap[i], &full[stage], kbk, bcoord[i]);
            }
            if (dual) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if (i >= nbox) break;
                uint8_t* d2 = b_dst + L::kBBytes + i * box_bytes;
                if (b_mn)
                  tma_load_2d(d2, bmap2[i], &full[stage], bcoord[i], kbk);
                else
                  tma_load_2d(d2, bmap2[i], &full[stage], kbk, bcoord[i]);
              }
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
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
      for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
        const int tile = item / splits, split = item - tile * splits;
        int tm, tn;
        tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
        const int reg0 = region_of(g, rows_reg ? tm * kBM : tn * BN);
        int tile_kb = 0;
        for (int si = 0; si < num_segs; ++si) tile_kb += seg_kb(g.segs[si], reg0);
        const int kb_lo = split * tile_kb / splits, kb_hi = (split + 1) * tile_kb / splits;
        mbar_wait(&tempty[acc], acc_phase ^ 1u, wg);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        uint32_t accumulate = 0u;
        int gk = 0;
        for (int si = 0; si < num_segs; ++si) {
          const GemmSeg& sg = g.segs[si];
          const int a_mn = sg.a_mn, b_mn = sg.b_mn, nkb = seg_kb(sg, reg0);
          const uint32_t idesc = sg.idesc;
          const bool dual = kDual && sg.dual;
          const int kb0 = max(0, kb_lo - gk), kb1 = min(nkb, kb_hi - gk);
          gk += nkb;
          for (int kb = kb0; kb < kb1; ++kb) {
            mbar_wait(&full[stage], phase, wg);
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * L::kABytes);
            const uint32_t b_addr = smem_u32(sB + stage * L::kBStage);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = a_mn ? mnmajor_desc(a_addr, kk, kMnBoxBytes) : kmajor_desc(a_addr, kk, L::kABytes);
              const uint64_t bd = b_mn ? mnmajor_desc(b_addr, kk, kMnBoxBytes) : kmajor_desc(b_addr, kk, L::kBBytes);
              umma_ss(d_tmem, ad, bd, idesc, accumulate);
              accumulate = 1u;
              if (dual) {
                const uint32_t b2 = b_addr + L::kBBytes;
                const uint64_t bd2 = b_mn ? mnmajor_desc(b2, kk, kMnBoxBytes) : kmajor_desc(b2, kk, L::kBBytes);
                umma_ss(d_tmem, ad, bd2, idesc, 1u);
              }
            }
            umma_commit(&empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
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
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
    for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
      const int tile = item / splits;
      int tm, tn;
      tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
      mbar_wait(&tfull[acc], acc_phase, wg);
      tc_fence_after();
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
      bool run_epi = true;
      if (splits > 1) {
        // this split's partial tile out, chunk-major so that a warp's stores are contiguous
        float4* part = g.split_ws + static_cast<long long>(item) * (BN / 4) * kBM + row;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(taddr + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            __stcg(part + ((c >> 2) + i) * kBM, make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                            __uint_as_float(r[4 * i + 2]),
                                                            __uint_as_float(r[4 * i + 3])));
        }
        __threadfence();
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) *last_flag = atomicAdd(g.split_cnt + tile, 1) == splits - 1;
        named_bar_sync(1, 128);
        run_epi = *last_flag != 0;
        if (run_epi) {
          // the tile's sum over splits, in split order, back into TMEM
          __threadfence();
          const float4* base = g.split_ws + static_cast<long long>(tile) * splits * (BN / 4) * kBM + row;
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
            // in split order; two splits' loads in flight at a time
            int sp = 0;
#pragma unroll 1
            for (; sp + 1 < splits; sp += 2) {
              const float4* q0 = base + static_cast<long long>(sp) * (BN / 4) * kBM + (c >> 2) * kBM;
              const float4* q1 = q0 + (BN / 4) * kBM;
              float4 f0[8], f1[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                f0[i] = __ldcg(q0 + i * kBM);
                f1[i] = __ldcg(q1 + i * kBM);
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                v[4 * i] = (v[4 * i] + f0[i].x) + f1[i].x;
                v[4 * i + 1] = (v[4 * i + 1] + f0[i].y) + f1[i].y;
                v[4 * i + 2] = (v[4 * i + 2] + f0[i].z) + f1[i].z;
                v[4 * i + 3] = (v[4 * i + 3] + f0[i].w) + f1[i].w;
              }
            }
            if (sp < splits) {
              const float4* q0 = base + static_cast<long long>(sp) * (BN / 4) * kBM + (c >> 2) * kBM;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 f = __ldcg(q0 + i * kBM);
                v[4 * i] += f.x;
                v[4 * i + 1] += f.y;
                v[4 * i + 2] += f.z;
                v[4 * i + 3] += f.w;
              }
            }
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
            tmem_st32(taddr + c, w);
          }
          tmem_st_wait();
          if (warp == 2 && lane == 0) g.split_cnt[tile] = 0;
        }
      }
      if (run_epi) Epi::template apply<BN>(args.epi, taddr, tm * kBM, tn * BN, row, g.status);
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

// ------------------------------------------------------------------ 2-SM variant
// The same GEMM on CTA pairs (clusters of 2, tcgen05 cta_group::2): a pair
// owns a 256 x BN output tile; CTA r of the pair stages rows [128r, 128r+128)
// of A and rows [r BN/2, (r+1) BN/2) of B in its own shared memory, the even
// CTA issues M=256 MMAs that read both CTAs' halves, and each CTA's TMEM
// receives its 128 rows of D (all BN columns). Per SM this halves the B bytes
// that TMA writes into, and the tensor core reads out of, shared memory.
// Both CTAs' TMA loads complete on the even CTA's "full" barrier; MMA
// completion is multicast to both CTAs' "empty" / "tfull" barriers; each
// epilogue warp reports a drained accumulator to the even CTA's "tempty".
template <int BN, int STAGES>
struct Gemm2Smem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;        // this CTA's 128 rows of A
  static constexpr uint32_t kBBytes = (BN / 2) * kBK * 2;   // this CTA's BN/2 rows of B
  static constexpr uint32_t kBarOffset = STAGES * (kABytes + kBBytes);
  static constexpr uint32_t kBytes = kBarOffset + 256 + 1024;
};

template <int BN, int STAGES, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm2_kernel(const __grid_constant__ GemmArgs<Epi> args) {
  static_assert(BN % 128 == 0 && BN <= 256, "two 64-column boxes of B per CTA half");
  using L = Gemm2Smem<BN, STAGES>;
  constexpr uint32_t kTmemCols = tmem_cols_for(2 * BN);
  constexpr int kHalfN = BN / 2;

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
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // the leader's expect_tx; both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast commit per round
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // one arrive per epilogue warp of both CTAs
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int si = 0; si < g.num_segs; ++si) {
      tma_prefetch_desc(&g.maps[g.segs[si].a_map]);
      for (int r = 0; r < (g.b_by_rank ? 2 : g.num_regions); ++r) tma_prefetch_desc(&g.maps[g.segs[si].b_map[r]]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barrier inits and the TMEM address visible to both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitGuard wg{abort_flag, g.status};
  grid_dep_launch();
  grid_dep_wait();  // every global access of this kernel comes after this

  const int num_tiles = g.tiles_m * g.tiles_n;  // 256-row tiles
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const int num_segs = g.num_segs;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int b_box_rows = g.b_box_rows;  // K-major B: rows per box (<= BN/2)
      for (int tile = cluster; tile < num_tiles; tile += clusters) {
        int tm, tn;
        tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
        int grp_off = 0;
        if (g.tile_group) {
          const int grp = g.tile_group[tm];
          if (grp < 0) continue;
          grp_off = grp * g.group_rows;
        }
        const int m0 = tm * 2 * kBM + static_cast<int>(rank) * kBM;
        const int n0 = tn * BN + static_cast<int>(rank) * kHalfN;
        const int reg0 = region_of(g, tn * BN);
        for (int si = 0; si < num_segs; ++si) {
          const GemmSeg& sg = g.segs[si];
          const int a_mn = sg.a_mn, b_mn = sg.b_mn, nkb = sg.kb, a_k0 = sg.a_k0[reg0], b_k0 = sg.b_k0;
          const CUtensorMap* amap = &g.maps[sg.a_map];
          const int box_n = b_mn ? 64 : b_box_rows;
          const int nbox = kHalfN / box_n;
          const CUtensorMap* bmap[2];
          int bcoord[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int n = n0 + (i < nbox ? i : 0) * box_n;
            if (g.b_by_rank) {
              bmap[i] = &g.maps[sg.b_map[rank]];
              bcoord[i] = tn * kHalfN + (i < nbox ? i : 0) * box_n + grp_off;
            } else {
              const int r = region_of(g, n);
              bmap[i] = &g.maps[sg.b_map[r]];
              bcoord[i] = n - g.region_n0[r] + grp_off;
            }
          }
          const uint32_t box_bytes = static_cast<uint32_t>(box_n) * kBK * 2;
          for (int kb = 0; kb < nkb; ++kb) {
            mbar_wait(&empty[stage], phase ^ 1u, wg);
            const uint32_t fbar = map_to_rank(smem_u32(&full[stage]), 0);
            if (leader) mbar_expect_tx(&full[stage], 2 * (L::kABytes + L::kBBytes));
            uint8_t* a_dst = sA + stage * L::kABytes;
            uint8_t* b_dst = sB + stage * L::kBBytes;
            const int ka = a_k0 + kb * kBK, kbk = b_k0 + kb * kBK;
            if (a_mn) {
              tma_load_2d_pair(a_dst, amap, fbar, m0, ka);
              tma_load_2d_pair(a_dst + kMnBoxBytes, amap, fbar, m0 + 64, ka);
            } else {
              tma_load_2d_pair(a_dst, amap, fbar, ka, m0);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              if (i >= nbox) break;
              if (b_mn)
                tma_load_2d_pair(b_dst + i * box_bytes, bmap[i], fbar, bcoord[i], kbk);
              else
                tma_load_2d_pair(b_dst + i * box_bytes, bmap[i], fbar, kbk, bcoord[i]);
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = cluster; tile < num_tiles; tile += clusters) {
        if (g.tile_group) {
          int tm, tn;
          tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
          if (g.tile_group[tm] < 0) continue;
        }
        mbar_wait(&tempty[acc], acc_phase ^ 1u, wg);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        uint32_t accumulate = 0u;
        for (int si = 0; si < num_segs; ++si) {
          const GemmSeg& sg = g.segs[si];
          const int a_mn = sg.a_mn, b_mn = sg.b_mn, nkb = sg.kb;
          const uint32_t idesc = sg.idesc;  // built for M = 256, N = BN
          for (int kb = 0; kb < nkb; ++kb) {
            mbar_wait(&full[stage], phase, wg);
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * L::kABytes);
            const uint32_t b_addr = smem_u32(sB + stage * L::kBBytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = a_mn ? mnmajor_desc(a_addr, kk, kMnBoxBytes) : kmajor_desc(a_addr, kk, L::kABytes);
              const uint64_t bd = b_mn ? mnmajor_desc(b_addr, kk, kMnBoxBytes) : kmajor_desc(b_addr, kk, L::kBBytes);
              umma_ss_pair(d_tmem, ad, bd, idesc, accumulate);
              accumulate = 1u;
            }
            umma_commit_pair(&empty[stage], 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        umma_commit_pair(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < num_tiles; tile += clusters) {
      int tm, tn;
      tile_coords(tile, g.tiles_m, g.tiles_n, tm, tn);
      if (g.tile_group && g.tile_group[tm] < 0) continue;
      mbar_wait(&tfull[acc], acc_phase, wg);
      tc_fence_after();
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
      Epi::template apply<BN>(args.epi, taddr, tm * 2 * kBM + static_cast<int>(rank) * kBM, tn * BN, row, g.status);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  tc_fence_before();
  cluster_sync();  // the peer's MMAs no longer read this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ epilogues
// 64 bytes of one row: two whole 32-byte sectors when the address allows,
// else four 16-byte stores (outputs are only required to be 16-byte aligned)
__device__ __forceinline__ void store_row64(void* dst, const uint32_t (&w)[16]) {
  if ((reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st_global_v8(static_cast<uint8_t*>(dst) + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
  } else {
    uint4* d = static_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

__device__ __forceinline__ void load_row32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Up to three 16-bit row-major outputs (each bf16 or f16 with its own scale)
// and an f32 output (own scale; optionally added to what is there;
// optionally transposed: element (m, n) at out32[n * ld32 + m]). A 16-bit
// output may instead hold the rounding residual of another one,
// bf16(w - float(bf16(w))) with w = acc * that output's scale, so that
// hi + lo carries about 16 significant bits through two bf16 operands.
// Rows >= M and columns >= N are skipped.
struct EpiStore {
  struct Out16 {
    void* ptr;
    long long ld;
    float scale;
    int bf16;
    int residual_of;  // -1, or the index of the output whose residual this is
  };
  struct Params {
    Out16 o16[3];
    float* out32;
    long long ld32;
    float scale32;
    int accumulate32;
    int transpose32;
    int M, N;
    int check_f16;  // flag f16 overflow of an f16 output
  };
  __device__ __forceinline__ static uint16_t round16(float w, int is_bf16) {
    if (is_bf16) {
      const __nv_bfloat16 h = __float2bfloat16_rn(w);
      return *reinterpret_cast<const uint16_t*>(&h);
    }
    const __half h = __float2half_rn(w);
    return *reinterpret_cast<const uint16_t*>(&h);
  }
  __device__ __forceinline__ static float value16(const Params& p, int i, float acc) {
    const Out16& o = p.o16[i];
    if (o.residual_of < 0) return acc * o.scale;
    const Out16& hi = p.o16[o.residual_of];
    const float w = acc * hi.scale;
    const uint16_t r = round16(w, hi.bf16);
    const float back = hi.bf16 ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&r))
                               : __half2float(*reinterpret_cast<const __half*>(&r));
    return w - back;
  }
  __device__ __forceinline__ static void store16(const Params& p, int i, int m, int n, const float (&v)[32],
                                                 int ncols, bool& overflow) {
    const Out16& o = p.o16[i];
    uint16_t* row = static_cast<uint16_t*>(o.ptr) + m * o.ld + n;
    if (ncols == 32) {
      uint4* dst = reinterpret_cast<uint4*>(row);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = value16(p, i, v[8 * q + 2 * k]), b = value16(p, i, v[8 * q + 2 * k + 1]);
          overflow |= p.check_f16 && !o.bf16 && !(fabsf(a) <= 65504.f && fabsf(b) <= 65504.f);
          w[k] = static_cast<uint32_t>(round16(a, o.bf16)) | (static_cast<uint32_t>(round16(b, o.bf16)) << 16);
        }
        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if (k >= ncols) continue;
        const float a = value16(p, i, v[k]);
        overflow |= p.check_f16 && !o.bf16 && !(fabsf(a) <= 65504.f);
        row[k] = round16(a, o.bf16);
      }
    }
  }
  // bf16 or f16 pair (a in the low half), round to nearest even
  template <bool kBf16>
  __device__ __forceinline__ static uint32_t pack2(float a, float b) {
    if constexpr (kBf16) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
      return *reinterpret_cast<const uint32_t*>(&h);
    } else {
      const __half2 h = __floats2half2_rn(a, b);
      return *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  // 32 full columns of one output, its type and kind fixed at compile time:
  // straight-line packed conversions and four 16-byte stores. kResid: the
  // bf16 residual of a bf16 output scaled by `scale`. f16: amax collects the
  // largest magnitude (NaN propagates) for the overflow check.
  template <bool kBf16, bool kResid>
  __device__ __forceinline__ static void store32(uint16_t* row, const float (&v)[32], float scale, float& amax) {
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a = v[2 * k] * scale, b = v[2 * k + 1] * scale;
      if constexpr (kResid) {
        const uint32_t hi = pack2<true>(a, b);
        a -= __uint_as_float(hi << 16);
        b -= __uint_as_float(hi & 0xffff0000u);
      }
      if constexpr (!kBf16) amax = fmax3_nan(amax, fabsf(a), fabsf(b));
      w[k] = pack2<kBf16>(a, b);
    }
    store_row64(row, w);
  }
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    const int m = m0 + row;
    bool overflow = false;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      const int n = n0 + c;
      if (n >= p.N) break;  // the same for every thread: no TMEM load for columns past N
      float v[32];
      load_row32(taddr + c, v);
      if (m >= p.M) continue;
      const int ncols = min(32, p.N - n);
#pragma unroll 1
      for (int i = 0; i < 3; ++i) {
        const Out16& o = p.o16[i];
        if (!o.ptr) continue;
        uint16_t* row16 = static_cast<uint16_t*>(o.ptr) + static_cast<long long>(m) * o.ld + n;
        const bool aligned = (reinterpret_cast<uintptr_t>(row16) & 15) == 0;
        const bool resid = o.residual_of >= 0;
        const Out16& hi = p.o16[resid ? o.residual_of : i];
        if (ncols == 32 && aligned && (!resid || (hi.bf16 && o.bf16))) {
          float amax = 0.f;
          if (resid)
            store32<true, true>(row16, v, hi.scale, amax);
          else if (o.bf16)
            store32<true, false>(row16, v, o.scale, amax);
          else
            store32<false, false>(row16, v, o.scale, amax);
          overflow |= p.check_f16 && !o.bf16 && !(amax <= 65504.f);
        } else {
          store16(p, i, m, n, v, ncols, overflow);
        }
      }
      if (p.out32) {
        const float s32 = p.scale32;
        if (p.transpose32) {
          // element (m, n + k) at out32[(n + k) ld32 + m]: for each k a warp
          // writes 32 consecutive floats; old values first, then the stores
          const long long ld = p.ld32;
          float* base = p.out32 + static_cast<long long>(n) * ld + m;
          float old[32];
          if (ncols == 32) {
#pragma unroll
            for (int k = 0; k < 32; ++k) old[k] = p.accumulate32 ? base[k * ld] : 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) base[k * ld] = fmaf(v[k], s32, old[k]);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) old[k] = (p.accumulate32 && k < ncols) ? base[k * ld] : 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < ncols) base[k * ld] = fmaf(v[k], s32, old[k]);
          }
        } else {
          float* o = p.out32 + static_cast<long long>(m) * p.ld32 + n;
          if (ncols == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
            float4* dst = reinterpret_cast<float4*>(o);
            float4 old[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) old[q] = p.accumulate32 ? dst[q] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(fmaf(v[4 * q], s32, old[q].x), fmaf(v[4 * q + 1], s32, old[q].y),
                                   fmaf(v[4 * q + 2], s32, old[q].z), fmaf(v[4 * q + 3], s32, old[q].w));
          } else {
            float old[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) old[k] = (p.accumulate32 && k < ncols) ? o[k] : 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < ncols) o[k] = fmaf(v[k], s32, old[k]);
          }
        }
      }
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

// LoRA gradients of q, k and v from one GEMM whose N columns are three
// rank-wide blocks (block j = columns [j*RP, (j+1)*RP), of which the first r
// are real): block j is added into (or written to) out[j], transposed
// (element (m, k) at out[j][k * ld + m]) or not (at out[j][m * ld + k]).
struct EpiLoraGrad {
  struct Params {
    float* out[3];
    long long ld;
    int RP, r, M;  // RP: a multiple of 32, so a 32-column chunk lies in one block
    int transpose, accumulate;
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    const int m = m0 + row;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      // block j and its first column k0: the same for every thread, so chunks
      // of padding columns (k0 >= r) or past the three blocks skip the TMEM load
      const int n = n0 + c;
      const int j = n / p.RP, k0 = n - j * p.RP;
      const int nv = j > 2 ? 0 : min(32, p.r - k0);
      if (nv <= 0) continue;
      float v[32];
      load_row32(taddr + c, v);
      if (m >= p.M) continue;
      float* out = j == 0 ? p.out[0] : j == 1 ? p.out[1] : p.out[2];
      float old[32];
      if (p.transpose) {
        // element (m, k) at out[k ld + m]: a warp's 32 rows are 32 consecutive floats
        const long long ld = p.ld;
        float* base = out + static_cast<long long>(k0) * ld + m;
        if (nv == 32) {
#pragma unroll
          for (int i = 0; i < 32; ++i) old[i] = p.accumulate ? base[i * ld] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) base[i * ld] = old[i] + v[i];
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) old[i] = (p.accumulate && i < nv) ? base[i * ld] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nv) base[i * ld] = old[i] + v[i];
        }
      } else {
        float* base = out + static_cast<long long>(m) * p.ld + k0;
        if (nv == 32 && (reinterpret_cast<uintptr_t>(base) & 15) == 0) {
          float4* dst = reinterpret_cast<float4*>(base);
          float4 o4[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) o4[q] = p.accumulate ? dst[q] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(o4[q].x + v[4 * q], o4[q].y + v[4 * q + 1], o4[q].z + v[4 * q + 2],
                                 o4[q].w + v[4 * q + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) old[i] = (p.accumulate && i < nv) ? base[i] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nv) base[i] = old[i] + v[i];
        }
      }
    }
  }
};

// D rows [row0[j], row0[j+1]) (j < 3) go to out[j], row m - row0[j], the
// first `cols` columns, row-major with leading dimension ld; accumulate adds
// into what is there (the three LoRA-up gradients of q, k, v in one GEMM).
struct EpiRowBlocks {
  struct Params {
    float* out[3];
    int row0[4];
    long long ld;
    int cols;
    int accumulate;
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    const int m = m0 + row;
    const int j = (m >= p.row0[1]) + (m >= p.row0[2]);
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      const int n = n0 + c;
      if (n >= p.cols) break;  // the same for every thread: no TMEM load for padding columns
      float v[32];
      load_row32(taddr + c, v);
      if (m >= p.row0[3]) continue;
      const int nv = min(32, p.cols - n);
      float* o = (j == 0 ? p.out[0] : j == 1 ? p.out[1] : p.out[2]) +
                 static_cast<long long>(m - p.row0[j]) * p.ld + n;
      if (nv == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
        float4* dst = reinterpret_cast<float4*>(o);
        float4 o4[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) o4[q] = p.accumulate ? dst[q] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(o4[q].x + v[4 * q], o4[q].y + v[4 * q + 1], o4[q].z + v[4 * q + 2],
                               o4[q].w + v[4 * q + 3]);
      } else {
        float old[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) old[i] = (p.accumulate && i < nv) ? o[i] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < nv) o[i] = old[i] + v[i];
      }
    }
  }
};

// Gradient of the attention output: stores dO = acc as f16 [M, Hq*dh] and,
// per (token, head), D = sum_j dO_j O_j with the forward's attention output O
// (the rowsum the softmax backward subtracts), taken over the f16-rounded dO
// the attention backward multiplies. Two heads per 256-column tile.
struct EpiDattn {
  struct Params {
    __half* dout;     // [M, Hq*dh]
    const __half* o;  // [M, Hq*dh]
    float* delta;     // [B, Hq, N]
    int M, N, Hq;
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    static_assert(BN % 128 == 0, "whole heads per tile");
    const int m = m0 + row;
    bool overflow = false;
#pragma unroll 1
    for (int hc = 0; hc < BN / 128; ++hc) {
      float dsum = 0.f;
      const int head = (n0 >> 7) + hc;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        load_row32(taddr + hc * 128 + c * 32, v);
        if (m >= p.M) continue;
        const long long off = static_cast<long long>(m) * p.Hq * 128 + head * 128 + c * 32;
        const uint4* o4 = reinterpret_cast<const uint4*>(p.o + off);
        uint4* d4 = reinterpret_cast<uint4*>(p.dout + off);
        uint4 ow4[4];  // loaded ahead of the dO stores
#pragma unroll
        for (int i = 0; i < 4; ++i) ow4[i] = o4[i];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 ow = ow4[i];
          const __half2* oh = reinterpret_cast<const __half2*>(&ow);
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            w[k] = pack_half2(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
            const float2 df = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
            const float2 of = __half22float2(oh[k]);
            dsum = fmaf(df.x, of.x, dsum);
            dsum = fmaf(df.y, of.y, dsum);
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) overflow |= !(fabsf(v[8 * i + k]) <= 65504.f);
          d4[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (m < p.M) {
        const int b = m / p.N, n = m - b * p.N;
        p.delta[(static_cast<long long>(b) * p.Hq + head) * p.N + n] = dsum;
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
    // prefix tower: the layer's cache entry, bf16 [B, Hkv, Pc, dh] keys
    // (normalised, rotated) and values at row n, rounded once from f32; null
    // for the gen tower
    __nv_bfloat16* kc_out;
    __nv_bfloat16* vc_out;
    int Pc;
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
      // 32 bytes at a time (few live registers beside the 128 values)
      const bool a32 = (reinterpret_cast<uintptr_t>(dst) & 31) == 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float* e = v + 16 * q;
        const uint32_t w0 = pack_half2(e[0], e[1]), w1 = pack_half2(e[2], e[3]), w2 = pack_half2(e[4], e[5]),
                       w3 = pack_half2(e[6], e[7]), w4 = pack_half2(e[8], e[9]), w5 = pack_half2(e[10], e[11]),
                       w6 = pack_half2(e[12], e[13]), w7 = pack_half2(e[14], e[15]);
        if (a32) {
          st_global_v8(dst + 16 * q, w0, w1, w2, w3, w4, w5, w6, w7);
        } else {
          uint4* d = reinterpret_cast<uint4*>(dst + 16 * q);
          d[0] = make_uint4(w0, w1, w2, w3);
          d[1] = make_uint4(w4, w5, w6, w7);
        }
      }
      if (p.kc_out && head >= p.Hq) {
        const bool is_k = head < p.Hq + p.Hkv;
        const int g = head - p.Hq - (is_k ? 0 : p.Hkv);
        uint4* c4 = reinterpret_cast<uint4*>((is_k ? p.kc_out : p.vc_out) +
                                             (static_cast<long long>(b * p.Hkv + g) * p.Pc + n) * 128);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          c4[i] = make_uint4(pack_bf162(v[8 * i + 0], v[8 * i + 1]), pack_bf162(v[8 * i + 2], v[8 * i + 3]),
                             pack_bf162(v[8 * i + 4], v[8 * i + 5]), pack_bf162(v[8 * i + 6], v[8 * i + 7]));
      }
#pragma unroll
      for (int i = 0; i < 128; ++i) overflow |= fabsf(v[i]) > 65504.f;
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

// SwiGLU epilogue of the gate/up projection (pair kernel with b_by_rank,
// BN = 256): D columns [0, 128) of the tile are the gate pre-activation g and
// [128, 256) the up pre-activation u of the same 128 intermediate indices
// j0 = n0 / 2 + [0, 128). Stores h = silu(g) u as f16 [M, I] and, for
// training, g and u themselves (f16, the backward's inputs). silu(g) =
// g / (1 + 2^(-g log2 e)) with the MUFU exponential and reciprocal; the
// exponent is capped so that 1 + e stays finite (silu -> 0 for g -> -inf).
// "SenseNova-U1" (vLLM-Omni recipe), measured kernel table: act_and_mul
// between the gate/up projection and down_proj, folded in here.
struct EpiSwiGLU {
  struct Params {
    __half* h;       // [M, I]
    __half* g_out;   // [M, I] or null
    __half* u_out;   // [M, I] or null
    int M, I;
  };
  __device__ __forceinline__ static float silu(float g) {
    const float e = ex2_approx(fminf(-g * 1.4426950408889634f, 126.0f));
    return g * __frcp_rn(1.0f + e);
  }
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    static_assert(BN == 256, "128 gate + 128 up columns per tile");
    const int m = m0 + row;
    const int j0 = n0 >> 1;
    bool overflow = false;
#pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
      uint32_t gr[32], ur[32];
      tmem_ld32(taddr + c, gr);
      tmem_ld32(taddr + 128 + c, ur);
      tmem_ld_wait();
      if (m >= p.M || j0 + c >= p.I) continue;
      const long long off = static_cast<long long>(m) * p.I + j0 + c;
      uint32_t hw[16];
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float g0 = __uint_as_float(gr[2 * k]), g1 = __uint_as_float(gr[2 * k + 1]);
        const float u0 = __uint_as_float(ur[2 * k]), u1 = __uint_as_float(ur[2 * k + 1]);
        const float h0 = silu(g0) * u0, h1 = silu(g1) * u1;
        amax = fmax3_nan(amax, fabsf(h0), fabsf(h1));
        hw[k] = pack_half2(h0, h1);
      }
      store_row64(p.h + off, hw);
      if (p.g_out) {
        uint32_t gw[16], uw[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          amax = fmax3_nan(amax, fabsf(__uint_as_float(gr[2 * k])), fabsf(__uint_as_float(gr[2 * k + 1])));
          amax = fmax3_nan(amax, fabsf(__uint_as_float(ur[2 * k])), fabsf(__uint_as_float(ur[2 * k + 1])));
          gw[k] = pack_half2(__uint_as_float(gr[2 * k]), __uint_as_float(gr[2 * k + 1]));
          uw[k] = pack_half2(__uint_as_float(ur[2 * k]), __uint_as_float(ur[2 * k + 1]));
        }
        store_row64(p.g_out + off, gw);
        store_row64(p.u_out + off, uw);
      }
      overflow |= !(amax <= 65504.f);
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

// SwiGLU backward epilogue of dh = dy W_down + s g_d A_down (pair kernel,
// BN = 256 columns of I): with the forward's g, u (f16) at the same (m, j),
//   dg = dh u silu'(g),  du = dh silu(g),
//   silu'(g) = sigma(g) (1 + g (1 - sigma(g))),  sigma(g) = 1 / (1 + e^-g),
// stored as f16 into one [M, 2I] tensor (dg in columns [0, I), du in
// [I, 2I)), which the dx GEMM and the LoRA-gradient GEMMs read.
struct EpiSwiGLUBwd {
  struct Params {
    __half* dgu;        // [M, 2I]
    const __half* g;    // [M, I]
    const __half* u;    // [M, I]
    int M, I;
  };
  template <int BN>
  __device__ __forceinline__ static void apply(const Params& p, uint32_t taddr, int m0, int n0, int row,
                                               int* status) {
    const int m = m0 + row;
    bool overflow = false;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      const int j = n0 + c;
      if (j >= p.I) break;  // the same for every thread
      uint32_t dr[32];
      tmem_ld32(taddr + c, dr);
      tmem_ld_wait();
      if (m >= p.M) continue;
      const long long off = static_cast<long long>(m) * p.I + j;
      const uint4* g4 = reinterpret_cast<const uint4*>(p.g + off);
      const uint4* u4 = reinterpret_cast<const uint4*>(p.u + off);
      uint4 gv[4], uv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gv[q] = g4[q];
        uv[q] = u4[q];
      }
      uint32_t dgw[16], duw[16];
      float amax = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __half2* gh = reinterpret_cast<const __half2*>(&gv[q]);
        const __half2* uh = reinterpret_cast<const __half2*>(&uv[q]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 gf = __half22float2(gh[k]);
          const float2 uf = __half22float2(uh[k]);
          const float d0 = __uint_as_float(dr[8 * q + 2 * k]), d1 = __uint_as_float(dr[8 * q + 2 * k + 1]);
          const float s0 = __frcp_rn(1.0f + ex2_approx(fminf(-gf.x * 1.4426950408889634f, 126.0f)));
          const float s1 = __frcp_rn(1.0f + ex2_approx(fminf(-gf.y * 1.4426950408889634f, 126.0f)));
          const float dg0 = d0 * uf.x * (s0 * (1.0f + gf.x * (1.0f - s0)));
          const float dg1 = d1 * uf.y * (s1 * (1.0f + gf.y * (1.0f - s1)));
          const float du0 = d0 * gf.x * s0, du1 = d1 * gf.y * s1;
          amax = fmax3_nan(amax, fabsf(dg0), fabsf(dg1));
          amax = fmax3_nan(amax, fabsf(du0), fabsf(du1));
          dgw[4 * q + k] = pack_half2(dg0, dg1);
          duw[4 * q + k] = pack_half2(du0, du1);
        }
      }
      uint4* gd = reinterpret_cast<uint4*>(p.dgu + static_cast<long long>(m) * 2 * p.I + j);
      uint4* ud = reinterpret_cast<uint4*>(p.dgu + static_cast<long long>(m) * 2 * p.I + p.I + j);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gd[q] = make_uint4(dgw[4 * q], dgw[4 * q + 1], dgw[4 * q + 2], dgw[4 * q + 3]);
        ud[q] = make_uint4(duw[4 * q], duw[4 * q + 1], duw[4 * q + 2], duw[4 * q + 3]);
      }
      overflow |= !(amax <= 65504.f);
    }
    if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
  }
};

}  // namespace mot
