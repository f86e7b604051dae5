// attn_bwd.cuh -- backward of the grouped-query attention over
// [prefix cache ; self] on sm_100a tensor cores, with the RoPE and QK-RMSNorm
// backward folded into the write-out.
//
// LoRA training through the gen tower ("Setup notes", LoRA trainer docs:
// frozen bf16 base, LoRA adapters on the gen tower, static prefix cache):
// gradients reach q^ over all L = prefix_len[b] + N keys, and k^, v only for
// the N self keys (the cache is constant). With P = softmax(q^K^T/sqrt(dh)),
// D = rowsum(dO * O) and dScore = P * (dO V^T - D):
//   dq^ = dScore K / sqrt(dh),  dk^ = dScore^T q^ / sqrt(dh),  dv = P^T dO.
// Two kernels keep every sum in a fixed order (no atomics, bitwise
// deterministic):
//   attn_bwd_dq_kernel  -- one CTA per (branch, query head, 128-query tile),
//                          loops over all key tiles: S, dP, then dQ += dS K.
//   attn_bwd_dkv_kernel -- one CTA per (branch, KV head, 128-self-key tile),
//                          loops over the group's query heads and query tiles:
//                          S^T, dP^T, then dV += P^T dO and dK += dS^T q^.
// The element-wise step needs no row reduction (lse and D were saved), so
// each row is split over two threads of 64 columns each (8 warps).
// dScore is multiplied by 2^10 (exact) before its f16 rounding so that small
// probabilities stay normal in f16; the write-out multiplies by 2^-10.
// The write-out applies RoPE^-1 (rotation by -angle) and the RMSNorm
// backward with the frozen gain: dx = rstd (g - xhat mean(g xhat)), g = gain dx^.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr float kDsScale = 1024.0f;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnBwdParams {
  CUtensorMap q_map;   // q^ 3D {dh, N, B*Hq} f16, box {64, 128, 1}
  CUtensorMap k_map;   // K  3D {dh, Lcap, B*Hkv} f16, box {64, 128, 1}
  CUtensorMap v_map;   // V  same
  CUtensorMap do_map;  // dO 3D {Hq*dh, N, B} f16, box {64, 128, 1}
  int B, N, Hq, Hkv, Lcap, q_tiles, kv_tiles;
  int plen[kMaxBatch];
  float scale_log2;  // log2(e) / sqrt(dh)
  float inv_sqrt_dh;
  const float* lse;    // [B, Hq, N] natural log
  const float* delta;  // [B, Hq, N]
  const __half* xhat;  // [B*N, (Hq+Hkv)*dh]
  const float* rstd;   // [B*N, Hq+Hkv]
  const float* gamma_q;
  const float* gamma_k;
  const float2* rope;  // [positions][64] (cos, sin)
  __half* dqkv;        // [B*N, (Hq+2Hkv)*dh] pre-norm gradients of q | k | v
  int* status;
};

constexpr int kAttnBwdThreads = 320;  // TMA warp, MMA warp, 8 element-wise warps

struct AttnBwdSmem {
  static constexpr uint32_t kTile = 32768;
  static constexpr uint32_t kBytes = 7 * kTile + 256 + 1024;
};

// RoPE^-1 and the RMSNorm backward of one head row whose gradient w.r.t. the
// rotated, normalised head sits in TMEM (128 f32 columns at taddr, times
// `scale`); writes the f16 pre-norm gradient to dst. Two passes over the
// rotation pairs (j, j+64), 16 pairs at a time: the first accumulates
// mean(g xhat), the second writes rstd (g - xhat mean), g = gain * RoPE^-1(dx^).
__device__ __forceinline__ void rot_chunk(uint32_t taddr, float scale, int c, const float2* cs, const float* gamma,
                                          float (&lo)[16], float (&hi)[16]) {
  uint32_t rl[16], rh[16];
  tmem_ld16(taddr + c * 16, rl);
  tmem_ld16(taddr + 64 + c * 16, rh);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int j = c * 16 + i;
    const float2 t = __ldg(cs + j);
    const float a = __uint_as_float(rl[i]) * scale, b = __uint_as_float(rh[i]) * scale;
    // rotation by -angle: in_j = o_j c + o_{j+64} s,  in_{j+64} = o_{j+64} c - o_j s
    lo[i] = (a * t.x + b * t.y) * __ldg(gamma + j);
    hi[i] = (b * t.x - a * t.y) * __ldg(gamma + j + 64);
  }
}

__device__ __forceinline__ void load_f16x16(const __half* src, float (&v)[16]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 w = s4[i];
    const __half2* h2 = reinterpret_cast<const __half2*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(h2[k]);
      v[8 * i + 2 * k] = f.x;
      v[8 * i + 2 * k + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void store_f16x16(__half* dst, const float (&v)[16], bool& overflow) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    d4[i] = make_uint4(pack_half2(v[8 * i], v[8 * i + 1]), pack_half2(v[8 * i + 2], v[8 * i + 3]),
                       pack_half2(v[8 * i + 4], v[8 * i + 5]), pack_half2(v[8 * i + 6], v[8 * i + 7]));
#pragma unroll
  for (int k = 0; k < 16; ++k) overflow |= !(fabsf(v[k]) <= 65504.f);
}

// All 32 lanes of the warp call this (TMEM loads are warp-collective);
// lanes with write == false skip every global access.
__device__ __forceinline__ void head_grad_writeout(uint32_t taddr, float scale, bool write, const float2* cs,
                                                   const float* gamma, const __half* xh, float rs, __half* dst,
                                                   bool& overflow) {
  float dot = 0.f;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float lo[16], hi[16], xl[16], xu[16];
    rot_chunk(taddr, scale, c, cs, gamma, lo, hi);
    if (!write) continue;
    load_f16x16(xh + c * 16, xl);
    load_f16x16(xh + 64 + c * 16, xu);
#pragma unroll
    for (int i = 0; i < 16; ++i) dot = fmaf(lo[i], xl[i], fmaf(hi[i], xu[i], dot));
  }
  const float mean = dot * (1.0f / 128.0f);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    float lo[16], hi[16], xl[16], xu[16];
    rot_chunk(taddr, scale, c, cs, gamma, lo, hi);
    if (!write) continue;
    load_f16x16(xh + c * 16, xl);
    load_f16x16(xh + 64 + c * 16, xu);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      lo[i] = rs * (lo[i] - xl[i] * mean);
      hi[i] = rs * (hi[i] - xu[i] * mean);
    }
    store_f16x16(dst + c * 16, lo, overflow);
    store_f16x16(dst + 64 + c * 16, hi, overflow);
  }
}

// write 64 f16 values (32 packed words) as columns [64 half, 64 half + 64) of
// row `row` of a 128x128 K-major 128-byte-swizzled tile (box `half`)
__device__ __forceinline__ void store_swizzled_half_row(uint8_t* tile, int row, int half, const uint32_t (&pk)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(tile + half * 16384 + row * 128 + ((c ^ (row & 7)) << 4)) =
        make_uint4(pk[c * 4 + 0], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
}

// write 128 f16 values (64 packed words) as row `row` of a 128x128 K-major
// 128-byte-swizzled tile (two 64-column boxes)
__device__ __forceinline__ void store_swizzled_row(uint8_t* tile, int row, const uint32_t (&pk)[64]) {
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 w = make_uint4(pk[hf * 32 + c * 4 + 0], pk[hf * 32 + c * 4 + 1], pk[hf * 32 + c * 4 + 2],
                           pk[hf * 32 + c * 4 + 3]);
      *reinterpret_cast<uint4*>(tile + hf * 16384 + row * 128 + ((c ^ (row & 7)) << 4)) = w;
    }
  }
}

// ------------------------------------------------------------------ dq
__global__ void __launch_bounds__(kAttnBwdThreads, 1) attn_bwd_dq_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t T32 = AttnBwdSmem::kTile;
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + T32;
  uint8_t* sK = smem + 2 * T32;   // 2 stages
  uint8_t* sV = smem + 4 * T32;   // 1 stage
  uint8_t* sDS = smem + 5 * T32;  // 2 buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 7 * T32);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* sdp_full = bars + 7;
  uint64_t* sdp_free = bars + 8;
  uint64_t* ds_full = bars + 9;   // [2]
  uint64_t* ds_free = bars + 11;  // [2]
  uint64_t* dq_full = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = warp_id(), lane = lane_id();
  int bid = blockIdx.x;
  const int qt = bid % p.q_tiles;
  bid /= p.q_tiles;
  const int h = bid % p.Hq;
  const int b = bid / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int L = p.plen[b] + p.N;
  const int T = (L + 127) >> 7;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&ds_full[i], 256);
      mbar_init(&ds_free[i], 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(sdp_full, 1);
    mbar_init(sdp_free, 256);
    mbar_init(dq_full, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + 128u, tDQ = tmem + 256u;
  const WaitGuard wg{abort_flag, p.status};

  if (warp == 0) {
    if (lane == 0) {
      const int qz = b * p.Hq + h, kz = b * p.Hkv + g;
      mbar_expect_tx(q_full, 2 * T32);
      tma_load_3d(sQ, &p.q_map, q_full, 0, qt * 128, qz);
      tma_load_3d(sQ + 16384, &p.q_map, q_full, 64, qt * 128, qz);
      tma_load_3d(sDO, &p.do_map, q_full, h * 128, qt * 128, b);
      tma_load_3d(sDO + 16384, &p.do_map, q_full, h * 128 + 64, qt * 128, b);
      for (int j = 0; j < T; ++j) {
        const int s = j & 1;
        mbar_wait(&k_empty[s], ((j >> 1) & 1) ^ 1u, wg);
        mbar_expect_tx(&k_full[s], T32);
        tma_load_3d(sK + s * T32, &p.k_map, &k_full[s], 0, j * 128, kz);
        tma_load_3d(sK + s * T32 + 16384, &p.k_map, &k_full[s], 64, j * 128, kz);
        mbar_wait(v_empty, (j & 1) ^ 1u, wg);
        mbar_expect_tx(v_full, T32);
        tma_load_3d(sV, &p.v_map, v_full, 0, j * 128, kz);
        tma_load_3d(sV + 16384, &p.v_map, v_full, 64, j * 128, kz);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t id_kmn = idesc_f16(128, 128, false, false, false, true);
      const uint32_t qa = smem_u32(sQ), da = smem_u32(sDO), va = smem_u32(sV);
      mbar_wait(q_full, 0, wg);
      for (int j = 0; j <= T; ++j) {
        if (j < T) {
          const int s = j & 1;
          mbar_wait(&k_full[s], (j >> 1) & 1, wg);
          mbar_wait(v_full, j & 1, wg);
          if (j >= 1) mbar_wait(sdp_free, (j - 1) & 1, wg);
          tc_fence_after();
          const uint32_t ka = smem_u32(sK + s * T32);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tS, kmajor_desc(qa, kk, 16384), kmajor_desc(ka, kk, 16384), id_kk, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tDP, kmajor_desc(da, kk, 16384), kmajor_desc(va, kk, 16384), id_kk, kk > 0);
          umma_commit(sdp_full);
          umma_commit(v_empty);
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj & 1;
          mbar_wait(&ds_full[s], (jj >> 1) & 1, wg);
          tc_fence_after();
          const uint32_t dsa = smem_u32(sDS + s * T32), ka = smem_u32(sK + s * T32);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tDQ, kmajor_desc(dsa, kk, 16384), mnmajor_desc(ka, kk, 16384), id_kmn, (jj | kk) != 0);
          umma_commit(&ds_free[s]);
          umma_commit(&k_empty[s]);
        }
      }
      umma_commit(dq_full);
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // key columns [64 half, 64 half + 64) of each tile
    const int row = quarter * 32 + lane;
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const int n = qt * 128 + row;
    const bool valid = n < p.N;
    const long long stat = (static_cast<long long>(b) * p.Hq + h) * p.N + n;
    const float lse2 = valid ? p.lse[stat] * kLog2e : 0.f;
    const float drow = valid ? p.delta[stat] : 0.f;
    bool overflow = false;
    for (int j = 0; j < T; ++j) {
      const int s = j & 1;
      mbar_wait(sdp_full, j & 1, wg);
      tc_fence_after();
      const int valid_keys = L - j * 128;
      uint32_t pk[32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = half * 2 + cc;
        uint32_t rs[32], rd[32];
        tmem_ld32(tS + lo + c * 32, rs);
        tmem_ld32(tDP + lo + c * 32, rd);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int col = c * 32 + i;
          float p0 = ex2_approx(fmaf(__uint_as_float(rs[i]), p.scale_log2, -lse2));
          float p1 = ex2_approx(fmaf(__uint_as_float(rs[i + 1]), p.scale_log2, -lse2));
          p0 = col < valid_keys ? p0 : 0.f;
          p1 = col + 1 < valid_keys ? p1 : 0.f;
          const float d0 = p0 * (__uint_as_float(rd[i]) - drow) * kDsScale;
          const float d1 = p1 * (__uint_as_float(rd[i + 1]) - drow) * kDsScale;
          overflow |= !(fabsf(d0) <= 65504.f) || !(fabsf(d1) <= 65504.f);
          pk[cc * 16 + i / 2] = pack_half2(d0, d1);
        }
      }
      tc_fence_before();
      mbar_arrive(sdp_free);
      if (j >= 2) mbar_wait(&ds_free[s], ((j - 2) >> 1) & 1, wg);
      store_swizzled_half_row(sDS + s * T32, row, half, pk);
      fence_proxy_async_smem();
      mbar_arrive(&ds_full[s]);
    }
    mbar_wait(dq_full, 0, wg);
    tc_fence_after();
    if (half == 0) {
      const long long m = static_cast<long long>(b) * p.N + (valid ? n : 0);
      const int pos = p.plen[b] + (valid ? n : 0);
      const int hk = p.Hq + p.Hkv;
      head_grad_writeout(tDQ + lo, p.inv_sqrt_dh / kDsScale, valid, p.rope + static_cast<long long>(pos) * 64,
                         p.gamma_q, p.xhat + (m * hk + h) * 128, valid ? p.rstd[m * hk + h] : 0.f,
                         p.dqkv + m * ((p.Hq + 2 * p.Hkv) * 128) + h * 128, overflow);
    }
    if (overflow) atomicOr(p.status, DEV_ERR_NUMERIC);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dk, dv
__global__ void __launch_bounds__(kAttnBwdThreads, 1) attn_bwd_dkv_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t T32 = AttnBwdSmem::kTile;
  uint8_t* sK = smem;
  uint8_t* sV = smem + T32;
  uint8_t* sQ = smem + 2 * T32;   // 2 stages, interleaved with dO: stage s at 2*T32 + s*2*T32
  uint8_t* sA = smem + 6 * T32;   // P^T, then dScore^T
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 7 * T32);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;   // [2]
  uint64_t* qd_empty = bars + 3;  // [2]
  uint64_t* sdp_full = bars + 5;
  uint64_t* sdp_free = bars + 6;
  uint64_t* pt_full = bars + 7;
  uint64_t* pt_free = bars + 8;
  uint64_t* dst_full = bars + 9;
  uint64_t* dst_free = bars + 10;
  uint64_t* acc_full = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = warp_id(), lane = lane_id();
  int bid = blockIdx.x;
  const int kt = bid % p.kv_tiles;
  bid /= p.kv_tiles;
  const int g = bid % p.Hkv;
  const int b = bid / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int I = G * p.q_tiles;
  const int pl = p.plen[b];

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(sdp_free, 256);
    mbar_init(pt_full, 256);
    mbar_init(pt_free, 1);
    mbar_init(dst_full, 256);
    mbar_init(dst_free, 1);
    mbar_init(acc_full, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tST = tmem, tDPT = tmem + 128u, tDK = tmem + 256u, tDV = tmem + 384u;
  const WaitGuard wg{abort_flag, p.status};

  if (warp == 0) {
    if (lane == 0) {
      const int kz = b * p.Hkv + g;
      mbar_expect_tx(kv_full, 2 * T32);
      tma_load_3d(sK, &p.k_map, kv_full, 0, pl + kt * 128, kz);
      tma_load_3d(sK + 16384, &p.k_map, kv_full, 64, pl + kt * 128, kz);
      tma_load_3d(sV, &p.v_map, kv_full, 0, pl + kt * 128, kz);
      tma_load_3d(sV + 16384, &p.v_map, kv_full, 64, pl + kt * 128, kz);
      for (int it = 0; it < I; ++it) {
        const int s = it & 1;
        const int h = g * G + it / p.q_tiles, qi = it % p.q_tiles;
        uint8_t* q_dst = sQ + s * 2 * T32;
        mbar_wait(&qd_empty[s], ((it >> 1) & 1) ^ 1u, wg);
        mbar_expect_tx(&qd_full[s], 2 * T32);
        tma_load_3d(q_dst, &p.q_map, &qd_full[s], 0, qi * 128, b * p.Hq + h);
        tma_load_3d(q_dst + 16384, &p.q_map, &qd_full[s], 64, qi * 128, b * p.Hq + h);
        tma_load_3d(q_dst + T32, &p.do_map, &qd_full[s], h * 128, qi * 128, b);
        tma_load_3d(q_dst + T32 + 16384, &p.do_map, &qd_full[s], h * 128 + 64, qi * 128, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t id_kmn = idesc_f16(128, 128, false, false, false, true);
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), aa = smem_u32(sA);
      mbar_wait(kv_full, 0, wg);
      for (int it = 0; it <= I; ++it) {
        if (it < I) {
          const int s = it & 1;
          mbar_wait(&qd_full[s], (it >> 1) & 1, wg);
          if (it >= 1) mbar_wait(sdp_free, (it - 1) & 1, wg);
          tc_fence_after();
          const uint32_t qa = smem_u32(sQ + s * 2 * T32), da = qa + T32;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tST, kmajor_desc(ka, kk, 16384), kmajor_desc(qa, kk, 16384), id_kk, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tDPT, kmajor_desc(va, kk, 16384), kmajor_desc(da, kk, 16384), id_kk, kk > 0);
          umma_commit(sdp_full);
        }
        if (it >= 1) {
          const int jj = it - 1, s = jj & 1;
          const uint32_t qa = smem_u32(sQ + s * 2 * T32), da = qa + T32;
          mbar_wait(pt_full, jj & 1, wg);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tDV, kmajor_desc(aa, kk, 16384), mnmajor_desc(da, kk, 16384), id_kmn, (jj | kk) != 0);
          umma_commit(pt_free);
          mbar_wait(dst_full, jj & 1, wg);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tDK, kmajor_desc(aa, kk, 16384), mnmajor_desc(qa, kk, 16384), id_kmn, (jj | kk) != 0);
          umma_commit(dst_free);
          umma_commit(&qd_empty[s]);
        }
      }
      umma_commit(acc_full);
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // query columns [64 half, 64 half + 64) of each tile
    const int row = quarter * 32 + lane;
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    bool overflow = false;
    for (int it = 0; it < I; ++it) {
      const int h = g * G + it / p.q_tiles, qi = it % p.q_tiles;
      const long long sbase = (static_cast<long long>(b) * p.Hq + h) * p.N + qi * 128;
      const int qvalid = p.N - qi * 128;
      // softmax statistics of this thread's 64 queries: lane l holds queries
      // 64 half + l and 64 half + 32 + l; column c is read from lane c%32 by a shuffle
      float lse_r[2], del_r[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = half * 64 + lane + 32 * k;
        lse_r[k] = q < qvalid ? p.lse[sbase + q] * kLog2e : 0.f;
        del_r[k] = q < qvalid ? p.delta[sbase + q] : 0.f;
      }
      mbar_wait(sdp_full, it & 1, wg);
      tc_fence_after();
      // the A buffer holds dScore^T of the previous iteration until its dK MMA is done
      if (it >= 1) mbar_wait(dst_free, (it - 1) & 1, wg);
      uint32_t dk[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16-column chunks of this half
        const int col0 = half * 64 + c * 16;
        uint32_t rs[16], rd[16];
        tmem_ld16(tST + lo + col0, rs);
        tmem_ld16(tDPT + lo + col0, rd);
        tmem_ld_wait();
        uint32_t pp[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const int lc = c * 16 + i;  // column within this half
          const int col = half * 64 + lc;
          const bool v0 = col < qvalid, v1 = col + 1 < qvalid;
          const float l0 = __shfl_sync(0xffffffffu, lse_r[lc >> 5], lc & 31);
          const float l1 = __shfl_sync(0xffffffffu, lse_r[(lc + 1) >> 5], (lc + 1) & 31);
          const float D0 = __shfl_sync(0xffffffffu, del_r[lc >> 5], lc & 31);
          const float D1 = __shfl_sync(0xffffffffu, del_r[(lc + 1) >> 5], (lc + 1) & 31);
          float p0 = ex2_approx(fmaf(__uint_as_float(rs[i]), p.scale_log2, -l0));
          float p1 = ex2_approx(fmaf(__uint_as_float(rs[i + 1]), p.scale_log2, -l1));
          p0 = v0 ? p0 : 0.f;
          p1 = v1 ? p1 : 0.f;
          const float d0 = p0 * (__uint_as_float(rd[i]) - D0) * kDsScale;
          const float d1 = p1 * (__uint_as_float(rd[i + 1]) - D1) * kDsScale;
          overflow |= !(fabsf(d0) <= 65504.f) || !(fabsf(d1) <= 65504.f);
          pp[i / 2] = pack_half2(p0, p1);
          dk[c * 8 + i / 2] = pack_half2(d0, d1);
        }
        // P^T columns [col0, col0+16) = two 16-byte chunks of box `half`
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int cc = c * 2 + q2;
          *reinterpret_cast<uint4*>(sA + half * 16384 + row * 128 + ((cc ^ (row & 7)) << 4)) =
              make_uint4(pp[q2 * 4 + 0], pp[q2 * 4 + 1], pp[q2 * 4 + 2], pp[q2 * 4 + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(sdp_free);
      fence_proxy_async_smem();
      mbar_arrive(pt_full);
      mbar_wait(pt_free, it & 1, wg);
      store_swizzled_half_row(sA, row, half, dk);
      fence_proxy_async_smem();
      mbar_arrive(dst_full);
    }
    mbar_wait(acc_full, 0, wg);
    tc_fence_after();
    const int n = kt * 128 + row;
    const bool valid = n < p.N;
    const long long m = static_cast<long long>(b) * p.N + (valid ? n : 0);
    const int hk = p.Hq + p.Hkv;
    const int ld = (p.Hq + 2 * p.Hkv) * 128;
    if (half == 0) {
      // dk: RoPE^-1 + RMSNorm backward
      head_grad_writeout(tDK + lo, p.inv_sqrt_dh / kDsScale, valid,
                         p.rope + static_cast<long long>(pl + (valid ? n : 0)) * 64, p.gamma_k,
                         p.xhat + (m * hk + p.Hq + g) * 128, valid ? p.rstd[m * hk + p.Hq + g] : 0.f,
                         p.dqkv + m * ld + (p.Hq + g) * 128, overflow);
    } else {
      // dv: stored as is
      __half* dv = p.dqkv + m * ld + (p.Hq + p.Hkv + g) * 128;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t r16[16];
        tmem_ld16(tDV + lo + c * 16, r16);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r16[i]);
        if (valid) store_f16x16(dv + c * 16, v, overflow);
      }
    }
    if (overflow) atomicOr(p.status, DEV_ERR_NUMERIC);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mot
