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
// Two kinds of CTA, in one launch, keep every sum in a fixed order (no
// atomics, bitwise deterministic):
//   dq CTAs  -- one CTA per (branch, query head, 128-query tile).
//       q^ and dO of the tile sit in TMEM as the A operands of S = q^ K^T and
//       dP = dO V^T, so only K and V stream through shared memory. dScore is
//       written over the dP columns and feeds dQ += dScore K from TMEM.
//   dk/dv CTAs -- one CTA per (branch, KV head, 128-self-key tile),
//       looping over the group's query heads and query tiles: S^T, dP^T, then
//       P^T written over S^T feeds dV += P^T dO and dScore^T written over dP^T
//       feeds dK += dScore^T q^, both with the A operand in TMEM.
// The MMA warp issues the next tile's score MMA before the current gradient
// MMA (S^T(j+1) ahead of dK(j); S(j+1) ahead of dQ(j)), so the tensor core
// works while the element-wise warps compute; a later MMA that overwrites a
// TMEM operand of an earlier one is issued after it by the same thread.
// The element-wise step needs no row reduction (lse and D were saved), so
// each row is split over two threads of 64 columns each (8 warps); each half
// writes its f16 operand over the first 32 of its own 64 f32 columns.
// Probabilities are formed as 2^10 P (exact power of two, folded into the
// exponent) so that dScore = 2^10 P (dP - D) keeps small values normal in
// f16; dV and the write-outs multiply by 2^-10.
// The write-out applies RoPE^-1 (rotation by -angle) and the RMSNorm
// backward with the frozen gain: dx = rstd (g - xhat mean(g xhat)), g = gain dx^.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr float kDsScale = 1024.0f;  // 2^10
constexpr float kDsScaleLog2 = 10.0f;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnBwdParams {
  CUtensorMap q_map;   // q^ 3D {dh, N, B*Hq} f16, box {64, 128, 1}
  CUtensorMap k_map;   // K  3D {dh, Lcap, B*Hkv} f16, box {64, 128, 1}
  CUtensorMap v_map;   // V  same
  CUtensorMap do_map;  // dO 3D {Hq*dh, N, B} f16, box {64, 128, 1}
  const __half* qhat;  // [B*Hq, N, dh]
  const __half* dout;  // [B*N, Hq*dh]
  int B, N, Hq, Hkv, Lcap, q_tiles, kv_tiles;
  int dkv_ctas;  // B * Hkv * kv_tiles
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
constexpr int kDqStages = 3;

struct AttnBwdDqSmem {
  static constexpr uint32_t kTile = 32768;  // 128 rows x 128 f16, two 64-column swizzled boxes
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kDqStages * kTile;
  static constexpr uint32_t kBar = kV + kDqStages * kTile;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;
};

struct AttnBwdDkvSmem {
  static constexpr uint32_t kTile = 32768;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kTile;
  static constexpr uint32_t kQD = 2 * kTile;          // 2 stages x (q^ tile, dO tile)
  static constexpr uint32_t kStat = kQD + 4 * kTile;  // per element-wise warp: 64 exponent offsets, 64 D
  static constexpr uint32_t kBar = kStat + 8 * 512;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;
};

// TMEM column of K-step kk (16 f16 values) of a 128-wide f16 operand whose
// halves were written at columns [0, 32) and [64, 96) of a 128-column region
__device__ __forceinline__ uint32_t split_col(int kk) { return static_cast<uint32_t>(kk * 8 + (kk >= 4 ? 32 : 0)); }

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

// 2^x of one score pair on the MUFU, or (sel) on the FMA pipe
__device__ __forceinline__ void exp2_pair(float& p0, float& p1, float x0, float x1, bool poly) {
  if (poly) {
    exp2_poly2(p0, p1, x0, x1);
  } else {
    p0 = ex2_approx(x0);
    p1 = ex2_approx(x1);
  }
}

// ------------------------------------------------------------------ dq
__device__ __forceinline__ void attn_bwd_dq_cta(const AttnBwdParams& p, int bid, uint8_t* smem) {
  constexpr uint32_t T32 = AttnBwdDqSmem::kTile;
  uint8_t* sK = smem + AttnBwdDqSmem::kK;
  uint8_t* sV = smem + AttnBwdDqSmem::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnBwdDqSmem::kBar);
  uint64_t* k_full = bars + 0;               // [kDqStages]
  uint64_t* k_empty = bars + kDqStages;      // [kDqStages]
  uint64_t* v_full = bars + 2 * kDqStages;   // [kDqStages]
  uint64_t* v_empty = bars + 3 * kDqStages;  // [kDqStages]
  uint64_t* qd_ready = bars + 4 * kDqStages + 0;  // q^ and dO rows stored in TMEM
  uint64_t* s_full = bars + 4 * kDqStages + 1;
  uint64_t* s_free = bars + 4 * kDqStages + 2;  // S read into registers
  uint64_t* dp_full = bars + 4 * kDqStages + 3;
  uint64_t* ds_full = bars + 4 * kDqStages + 4;  // dScore stored over dP
  uint64_t* dq_full = bars + 4 * kDqStages + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * kDqStages + 6);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = warp_id(), lane = lane_id();
  const int qt = bid % p.q_tiles;
  bid /= p.q_tiles;
  const int h = bid % p.Hq;
  const int b = bid / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int L = p.plen[b] + p.N;
  const int T = (L + 127) >> 7;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDqStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(qd_ready, 256);
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
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
  // q^ and dO as f16 operands (64 columns each), then S, dP (dScore over its
  // first columns) and the dQ accumulator (128 f32 columns each)
  const uint32_t tQ = tmem, tDO = tmem + 64u, tS = tmem + 128u, tDP = tmem + 256u, tDQ = tmem + 384u;
  const WaitGuard wg{abort_flag, p.status};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.k_map);
      tma_prefetch_desc(&p.v_map);
      const int kz = b * p.Hkv + g;
      for (int j = 0; j < T; ++j) {
        const int s = j % kDqStages;
        const uint32_t ph = (j / kDqStages) & 1;
        mbar_wait(&k_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&k_full[s], T32);
        tma_load_3d(sK + s * T32, &p.k_map, &k_full[s], 0, j * 128, kz);
        tma_load_3d(sK + s * T32 + 16384, &p.k_map, &k_full[s], 64, j * 128, kz);
        mbar_wait(&v_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&v_full[s], T32);
        tma_load_3d(sV + s * T32, &p.v_map, &v_full[s], 0, j * 128, kz);
        tma_load_3d(sV + s * T32 + 16384, &p.v_map, &v_full[s], 64, j * 128, kz);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t id_dq = idesc_f16(128, 128, false, false, false, true);
      auto issue_s = [&](int j) {
        const uint32_t ka = smem_u32(sK + (j % kDqStages) * T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) umma_ts(tS, tQ + kk * 8u, kmajor_desc(ka, kk, 16384), id_s, kk > 0);
        umma_commit(s_full);
      };
      auto issue_dp = [&](int j) {
        const int s = j % kDqStages;
        const uint32_t va = smem_u32(sV + s * T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) umma_ts(tDP, tDO + kk * 8u, kmajor_desc(va, kk, 16384), id_s, kk > 0);
        umma_commit(dp_full);
        umma_commit(&v_empty[s]);
      };
      mbar_wait(qd_ready, 0, wg);
      mbar_wait(&k_full[0], 0, wg);
      tc_fence_after();
      issue_s(0);
      mbar_wait(&v_full[0], 0, wg);
      tc_fence_after();
      issue_dp(0);
      for (int j = 0; j < T; ++j) {
        const int s = j % kDqStages;
        const bool more = j + 1 < T;
        const int s1 = (j + 1) % kDqStages;
        const uint32_t ph1 = ((j + 1) / kDqStages) & 1;
        if (more) {
          // S(j+1) overwrites S(j) once the element-wise warps hold it in registers
          mbar_wait(&k_full[s1], ph1, wg);
          mbar_wait(s_free, j & 1, wg);
          tc_fence_after();
          issue_s(j + 1);
        }
        mbar_wait(ds_full, j & 1, wg);
        tc_fence_after();
        const uint32_t ka = smem_u32(sK + s * T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDQ, tDP + split_col(kk), mnmajor_desc(ka, kk, 16384), id_dq, (j | kk) != 0);
        umma_commit(&k_empty[s]);
        if (more) {
          // dP(j+1) overwrites dScore(j) after the dQ MMA above has read it (in-order issue)
          mbar_wait(&v_full[s1], ph1, wg);
          tc_fence_after();
          issue_dp(j + 1);
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
    // 2^10 P = 2^(s log2(e)/sqrt(dh) + off), off = 10 - lse log2(e); rows past N get P = 0
    const float off = valid ? kDsScaleLog2 - p.lse[stat] * kLog2e : -INFINITY;
    const float drow = valid ? p.delta[stat] : 0.f;
    const float c = p.scale_log2;
    {
      // this thread's 64 q^ and dO values (dims [64 half, 64 half + 64)) into TMEM
      uint32_t w[32];
      const uint4* src = reinterpret_cast<const uint4*>(
          p.qhat + ((static_cast<long long>(b) * p.Hq + h) * p.N + (valid ? n : 0)) * 128 + half * 64);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = valid ? src[i] : make_uint4(0, 0, 0, 0);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
      tmem_st32(tQ + lo + half * 32, w);
      src = reinterpret_cast<const uint4*>(p.dout + (static_cast<long long>(b) * p.N + (valid ? n : 0)) * (p.Hq * 128) +
                                           h * 128 + half * 64);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = valid ? src[i] : make_uint4(0, 0, 0, 0);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
      tmem_st32(tDO + lo + half * 32, w);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(qd_ready);
    }
    float mx = 0.f;  // max |2^10 dScore| (NaN if any)
    for (int j = 0; j < T; ++j) {
      mbar_wait(s_full, j & 1, wg);
      tc_fence_after();
      uint32_t rs[2][32];
      tmem_ld32(tS + lo + half * 64, rs[0]);
      tmem_ld32(tS + lo + half * 64 + 32, rs[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free);
      const int valid_keys = L - j * 128 - half * 64;  // keys past L get P = 0
      float pv[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(rs[cc][i]), __uint_as_float(rs[cc][i + 1]), c, c, off, off);
          exp2_pair(pv[cc * 32 + i], pv[cc * 32 + i + 1], x0, x1, ((i >> 1) & 3) == 3);
        }
      }
      if (valid_keys < 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i) pv[i] = i < valid_keys ? pv[i] : 0.f;
      }
      mbar_wait(dp_full, j & 1, wg);
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t rd[32];
        tmem_ld32(tDP + lo + half * 64 + cc * 32, rd);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float d0, d1;
          fadd2(d0, d1, __uint_as_float(rd[i]), __uint_as_float(rd[i + 1]), -drow, -drow);
          fmul2(d0, d1, d0, d1, pv[cc * 32 + i], pv[cc * 32 + i + 1]);
          mx = fmax3_nan(mx, fabsf(d0), fabsf(d1));
          pk[i >> 1] = pack_half2(d0, d1);
        }
        tmem_st16(tDP + lo + half * 64 + cc * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    bool overflow = !(mx <= 65504.f);
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
__device__ __forceinline__ void attn_bwd_dkv_cta(const AttnBwdParams& p, int bid, uint8_t* smem) {
  constexpr uint32_t T32 = AttnBwdDkvSmem::kTile;
  uint8_t* sK = smem + AttnBwdDkvSmem::kK;
  uint8_t* sV = smem + AttnBwdDkvSmem::kV;
  uint8_t* sQD = smem + AttnBwdDkvSmem::kQD;  // stage s: q^ at s * 2 T32, dO at s * 2 T32 + T32
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnBwdDkvSmem::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;   // [2]
  uint64_t* qd_empty = bars + 3;  // [2]
  uint64_t* st_full = bars + 5;
  uint64_t* pt_full = bars + 6;   // P^T stored over S^T
  uint64_t* dpt_full = bars + 7;
  uint64_t* dst_full = bars + 8;  // dScore^T stored over dP^T
  uint64_t* acc_full = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = warp_id(), lane = lane_id();
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
    mbar_init(st_full, 1);
    mbar_init(pt_full, 256);
    mbar_init(dpt_full, 1);
    mbar_init(dst_full, 256);
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
      tma_prefetch_desc(&p.q_map);
      tma_prefetch_desc(&p.do_map);
      const int kz = b * p.Hkv + g;
      mbar_expect_tx(kv_full, 2 * T32);
      tma_load_3d(sK, &p.k_map, kv_full, 0, pl + kt * 128, kz);
      tma_load_3d(sK + 16384, &p.k_map, kv_full, 64, pl + kt * 128, kz);
      tma_load_3d(sV, &p.v_map, kv_full, 0, pl + kt * 128, kz);
      tma_load_3d(sV + 16384, &p.v_map, kv_full, 64, pl + kt * 128, kz);
      for (int it = 0; it < I; ++it) {
        const int s = it & 1;
        const int h = g * G + it / p.q_tiles, qi = it % p.q_tiles;
        uint8_t* q_dst = sQD + s * 2 * T32;
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
      constexpr uint32_t id_ss = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t id_ts = idesc_f16(128, 128, false, false, false, true);
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV);
      auto issue_st = [&](int it) {
        const uint32_t qa = smem_u32(sQD + (it & 1) * 2 * T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tST, kmajor_desc(ka, kk, 16384), kmajor_desc(qa, kk, 16384), id_ss, kk > 0);
        umma_commit(st_full);
      };
      auto issue_dpt = [&](int it) {
        const uint32_t da = smem_u32(sQD + (it & 1) * 2 * T32 + T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tDPT, kmajor_desc(va, kk, 16384), kmajor_desc(da, kk, 16384), id_ss, kk > 0);
        umma_commit(dpt_full);
      };
      mbar_wait(kv_full, 0, wg);
      mbar_wait(&qd_full[0], 0, wg);
      tc_fence_after();
      issue_st(0);
      issue_dpt(0);
      for (int it = 0; it < I; ++it) {
        const int s = it & 1;
        const bool more = it + 1 < I;
        const uint32_t qa = smem_u32(sQD + s * 2 * T32), da = qa + T32;
        mbar_wait(pt_full, it & 1, wg);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDV, tST + split_col(kk), mnmajor_desc(da, kk, 16384), id_ts, (it | kk) != 0);
        if (more) {
          // S^T(it+1) overwrites P^T(it) after the dV MMA above has read it (in-order issue)
          mbar_wait(&qd_full[(it + 1) & 1], ((it + 1) >> 1) & 1, wg);
          tc_fence_after();
          issue_st(it + 1);
        }
        mbar_wait(dst_full, it & 1, wg);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tDK, tDPT + split_col(kk), mnmajor_desc(qa, kk, 16384), id_ts, (it | kk) != 0);
        umma_commit(&qd_empty[s]);
        if (more) issue_dpt(it + 1);  // overwrites dScore^T(it) after the dK MMA above
      }
      umma_commit(acc_full);
    }
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // query columns [64 half, 64 half + 64) of each tile
    const int row = quarter * 32 + lane;
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    // this warp's copy of the per-query statistics of its 64 query columns:
    // [0, 64) exponent offset 10 - lse log2(e) (-inf past N), [64, 128) D
    float* stat = reinterpret_cast<float*>(smem + AttnBwdDkvSmem::kStat) + (warp - 2) * 128;
    auto fetch = [&](int it, float (&v)[4]) {
      const int h = g * G + it / p.q_tiles, qi = it % p.q_tiles;
      const long long sbase = (static_cast<long long>(b) * p.Hq + h) * p.N + qi * 128;
      const int qvalid = p.N - qi * 128;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = half * 64 + lane + 32 * k;
        v[k] = q < qvalid ? kDsScaleLog2 - p.lse[sbase + q] * kLog2e : -INFINITY;
        v[2 + k] = q < qvalid ? p.delta[sbase + q] : 0.f;
      }
    };
    float nxt[4];
    fetch(0, nxt);
    float mx = 0.f;
    for (int it = 0; it < I; ++it) {
      __syncwarp();
      stat[lane] = nxt[0];
      stat[32 + lane] = nxt[1];
      stat[64 + lane] = nxt[2];
      stat[96 + lane] = nxt[3];
      __syncwarp();
      if (it + 1 < I) fetch(it + 1, nxt);
      const float4* off4 = reinterpret_cast<const float4*>(stat);
      const float4* d4 = reinterpret_cast<const float4*>(stat + 64);
      mbar_wait(st_full, it & 1, wg);
      tc_fence_after();
      uint32_t rs[2][32];
      tmem_ld32(tST + lo + half * 64, rs[0]);
      tmem_ld32(tST + lo + half * 64 + 32, rs[1]);
      tmem_ld_wait();
      float pv[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 o = off4[(cc * 32 + i) >> 2];
          float x0, x1, x2, x3;
          ffma2(x0, x1, __uint_as_float(rs[cc][i]), __uint_as_float(rs[cc][i + 1]), c, c, o.x, o.y);
          ffma2(x2, x3, __uint_as_float(rs[cc][i + 2]), __uint_as_float(rs[cc][i + 3]), c, c, o.z, o.w);
          float* pp = pv + cc * 32 + i;
          exp2_pair(pp[0], pp[1], x0, x1, false);
          exp2_pair(pp[2], pp[3], x2, x3, ((i >> 2) & 1) == 1);
          pk[i >> 1] = pack_half2(pp[0], pp[1]);
          pk[(i >> 1) + 1] = pack_half2(pp[2], pp[3]);
        }
        tmem_st16(tST + lo + half * 64 + cc * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(pt_full);
      mbar_wait(dpt_full, it & 1, wg);
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t rd[32];
        tmem_ld32(tDPT + lo + half * 64 + cc * 32, rd);
        tmem_ld_wait();
        uint32_t pd[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 dd = d4[(cc * 32 + i) >> 2];
          float d0, d1, d2, d3;
          fadd2(d0, d1, __uint_as_float(rd[i]), __uint_as_float(rd[i + 1]), -dd.x, -dd.y);
          fadd2(d2, d3, __uint_as_float(rd[i + 2]), __uint_as_float(rd[i + 3]), -dd.z, -dd.w);
          const float* pp = pv + cc * 32 + i;
          fmul2(d0, d1, d0, d1, pp[0], pp[1]);
          fmul2(d2, d3, d2, d3, pp[2], pp[3]);
          mx = fmax3_nan(mx, fabsf(d0), fabsf(d1));
          mx = fmax3_nan(mx, fabsf(d2), fabsf(d3));
          pd[i >> 1] = pack_half2(d0, d1);
          pd[(i >> 1) + 1] = pack_half2(d2, d3);
        }
        tmem_st16(tDPT + lo + half * 64 + cc * 16, pd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(dst_full);
    }
    const int n = kt * 128 + row;
    const bool valid = n < p.N;
    // key rows past N (zero K, V) are never written out; their values do not count
    bool overflow = valid && !(mx <= 65504.f);
    mbar_wait(acc_full, 0, wg);
    tc_fence_after();
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
      // dv = 2^-10 (2^10 P)^T dO
      __half* dv = p.dqkv + m * ld + (p.Hq + p.Hkv + g) * 128;
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t r16[16];
        tmem_ld16(tDV + lo + cc * 16, r16);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r16[i]) * (1.0f / kDsScale);
        if (valid) store_f16x16(dv + cc * 16, v, overflow);
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

// One launch for both: blocks [0, dkv_ctas) take (branch, KV head, key
// tile), the rest (branch, query head, query tile); the long dk/dv CTAs are
// dispatched first and the short dq CTAs fill the SMs as they free up.
struct AttnBwdSmem {
  static constexpr uint32_t kBytes =
      AttnBwdDqSmem::kBytes > AttnBwdDkvSmem::kBytes ? AttnBwdDqSmem::kBytes : AttnBwdDkvSmem::kBytes;
};

__global__ void __launch_bounds__(kAttnBwdThreads, 1) attn_bwd_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bid = static_cast<int>(blockIdx.x);
  grid_dep_launch();
  grid_dep_wait();
  if (bid < p.dkv_ctas)
    attn_bwd_dkv_cta(p, bid, smem);
  else
    attn_bwd_dq_cta(p, bid - p.dkv_ctas, smem);
}

}  // namespace mot
