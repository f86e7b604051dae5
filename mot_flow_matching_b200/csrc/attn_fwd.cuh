// attn_fwd.cuh -- grouped-query attention forward over [prefix cache ; self]
// on sm_100a tensor cores.
//
// For one CFG branch b, query head h and a 128-row tile of image tokens:
//   o = softmax(q^ K^T / sqrt(dh)) V,  K, V = rows [0, prefix_len[b] + N) of the
//   KV head g = h / (Hq/Hkv) ("SenseNova-U1" DiffSynth-Studio docs,
//   architecture note: image tokens attend to the prefix cache; vLLM-Omni
//   "SenseNova-U1" recipe, kernel table: "dual-tower attention" in a flash
//   kernel). Non-causal; keys past prefix_len[b] + N are masked.
//
// Per CTA: warp 0 streams Q once and K/V tiles (128 keys x 128 dims, f16,
// 128-byte swizzle) by TMA into a 2-deep ring; warp 1 issues
//   S_j = Q K_j^T   into one of two TMEM buffers (M=128, N=128, K=16 x 8)
//   O  += P_j V_j   into a TMEM accumulator (V is the MN-major operand)
// in the order S0, S1, PV0, S2, PV1, ... so the tensor core computes S_{j+1}
// while warps 2..5 (one query row per thread) turn S_j into P_j:
// running max m and sum l in fp32, p = 2^(s*log2(e)/sqrt(dh) - m) written as
// f16 into a swizzled K-major smem tile. The running max is only raised
// (and O rescaled through TMEM) when a row's max grows by more than 2^8, so
// p <= 256 stays exact enough in f16 and the final o = O / l uses the same m
// as every p it summed: the result is unchanged by the laziness.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr int kAttnThreads = 192;
constexpr float kLazyRescaleLog2 = 8.0f;

struct AttnFwdParams {
  CUtensorMap q_map;  // 3D {dh, N, B*Hq} f16, box {64, 128, 1}
  CUtensorMap k_map;  // 3D {dh, Lcap, B*Hkv} f16, box {64, 128, 1}
  CUtensorMap v_map;  // same as k_map
  int B, N, Hq, Hkv, Lcap, q_tiles;
  int plen[kMaxBatch];
  float scale_log2;  // log2(e) / sqrt(dh)
  __half* out;       // [B*N, Hq*dh] token-major
  float* lse;        // [B, Hq, N] natural-log sum of exp(scores), or null
  int* status;
};

struct AttnSmem {
  static constexpr uint32_t kTile = 32768;  // 128 rows x 128 f16
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kV = kK + 2 * kTile;
  static constexpr uint32_t kP = kV + 2 * kTile;
  static constexpr uint32_t kBar = kP + 2 * kTile;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;
};

__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnFwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + AttnSmem::kQ;
  uint8_t* sK = smem + AttnSmem::kK;
  uint8_t* sV = smem + AttnSmem::kV;
  uint8_t* sP = smem + AttnSmem::kP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2]
  uint64_t* s_free = bars + 11;   // [2]
  uint64_t* p_full = bars + 13;   // [2]
  uint64_t* p_free = bars + 15;   // [2]
  uint64_t* o_full = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
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
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_full, 1);
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
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tO = tmem_base + 256u;
  const WaitGuard wg{abort_flag, p.status};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.q_map);
      tma_prefetch_desc(&p.k_map);
      tma_prefetch_desc(&p.v_map);
      const int qz = b * p.Hq + h, kz = b * p.Hkv + g;
      mbar_expect_tx(q_full, AttnSmem::kTile);
      tma_load_3d(sQ, &p.q_map, q_full, 0, qt * 128, qz);
      tma_load_3d(sQ + 16384, &p.q_map, q_full, 64, qt * 128, qz);
      for (int j = 0; j < T; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        mbar_wait(&k_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&k_full[s], AttnSmem::kTile);
        tma_load_3d(sK + s * AttnSmem::kTile, &p.k_map, &k_full[s], 0, j * 128, kz);
        tma_load_3d(sK + s * AttnSmem::kTile + 16384, &p.k_map, &k_full[s], 64, j * 128, kz);
        mbar_wait(&v_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&v_full[s], AttnSmem::kTile);
        tma_load_3d(sV + s * AttnSmem::kTile, &p.v_map, &v_full[s], 0, j * 128, kz);
        tma_load_3d(sV + s * AttnSmem::kTile + 16384, &p.v_map, &v_full[s], 64, j * 128, kz);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(128, 128, false, false, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      mbar_wait(q_full, 0, wg);
      for (int j = 0; j <= T; ++j) {
        if (j < T) {
          const int s = j & 1;
          mbar_wait(&k_full[s], (j >> 1) & 1, wg);
          if (j >= 2) mbar_wait(&s_free[s], ((j - 2) >> 1) & 1, wg);
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + s * AttnSmem::kTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem_base + static_cast<uint32_t>(s) * 128u, kmajor_desc(q_addr, kk, 16384), kmajor_desc(k_addr, kk, 16384), idesc_qk, kk > 0);
          umma_commit(&s_full[s]);
          umma_commit(&k_empty[s]);
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj & 1;
          const uint32_t ph = (jj >> 1) & 1;
          mbar_wait(&p_full[s], ph, wg);
          mbar_wait(&v_full[s], ph, wg);
          tc_fence_after();
          const uint32_t pa = smem_u32(sP + s * AttnSmem::kTile);
          const uint32_t va = smem_u32(sV + s * AttnSmem::kTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tO, kmajor_desc(pa, kk, 16384), mnmajor_desc(va, kk, 16384), idesc_pv, (jj | kk) != 0);
          umma_commit(&v_empty[s]);
          umma_commit(&p_free[s]);
        }
      }
      umma_commit(o_full);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < T; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      mbar_wait(&s_full[s], ph, wg);
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + static_cast<uint32_t>(s) * 128u + lane_off + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s_free[s]);

      const int valid = L - j * 128;  // keys of this tile that exist (>= 1)
      float mx = -INFINITY;
      if (valid >= 128) {
#pragma unroll
        for (int i = 0; i < 128; ++i) mx = fmaxf(mx, sv[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          if (i >= valid) sv[i] = -INFINITY;
          mx = fmaxf(mx, sv[i]);
        }
      }
      const float m_tile = mx * p.scale_log2;
      bool need = false;
      float m_new = m_run;
      if (j == 0) {
        m_new = m_tile;
      } else if (m_tile > m_run + kLazyRescaleLog2) {
        need = true;
        m_new = m_tile;
      }
      // the P buffer this tile writes was last read by PV_{j-2}
      if (j >= 2) mbar_wait(&p_free[s], ((j - 2) >> 1) & 1, wg);
      if (__any_sync(0xffffffffu, need)) {
        // O must be final up to PV_{j-1} before it is rescaled
        mbar_wait(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, wg);
        tc_fence_after();
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + lane_off + c * 32, r);
        }
        tmem_st_wait();
        l_run *= alpha;
      }
      m_run = m_new;
      float rowsum = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        sv[i] = ex2_approx(fmaf(sv[i], p.scale_log2, -m_run));
        rowsum += sv[i];
      }
      l_run += rowsum;
      uint8_t* pb = sP + s * AttnSmem::kTile + row * 128;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 w;
          const float* q = sv + hf * 64 + c * 8;
          w.x = pack_half2(q[0], q[1]);
          w.y = pack_half2(q[2], q[3]);
          w.z = pack_half2(q[4], q[5]);
          w.w = pack_half2(q[6], q[7]);
          *reinterpret_cast<uint4*>(pb + hf * 16384 + ((c ^ (row & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[s]);
    }
    // epilogue: o = O / l, token-major f16
    mbar_wait(o_full, 0, wg);
    tc_fence_after();
    const int qrow = qt * 128 + row;
    const float inv_l = 1.0f / l_run;
    __half* dst = p.out + (static_cast<long long>(b) * p.N + qrow) * (p.Hq * 128) + h * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tO + lane_off + c * 32, r);
      tmem_ld_wait();
      if (qrow < p.N) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_half2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l);
          w.y = pack_half2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l);
          w.z = pack_half2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l);
          w.w = pack_half2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l);
          d4[i] = w;
        }
      }
    }
    if (p.lse && qrow < p.N)
      p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace mot
