// attn_fwd.cuh -- grouped-query attention forward over [prefix cache ; self]
// on sm_100a tensor cores.
//
// For one CFG branch b, query head h and image tokens i:
//   o = softmax(q^ K^T / sqrt(dh)) V,  K, V = rows [0, prefix_len[b] + N) of the
//   KV head g = h / (Hq/Hkv) ("SenseNova-U1" DiffSynth-Studio docs,
//   architecture note: image tokens attend to the prefix cache; vLLM-Omni
//   "SenseNova-U1" recipe, kernel table: "dual-tower attention" in a flash
//   kernel). Non-causal; keys past prefix_len[b] + N are masked.
//
// One CTA owns two 128-query tiles (t = 0, 1) of one (b, h) and streams the
// key/value tiles (128 keys x 128 dims, f16, 128-byte swizzle) once for both
// through a 2-deep TMA ring. TMEM holds, per query tile, S_t (128 f32
// columns) and the output accumulator O_t (128 columns). Warp 1 issues, per
// key tile j,
//   S_0 = Q_0 K_j^T, S_1 = Q_1 K_j^T, then O_0 += P_0 V_j, S_0 <- next tile,
//   O_1 += P_1 V_j, S_1 <- next tile
// so the tensor core works on one query tile while the other's softmax runs.
// Warps 2-9 (tile 0) and 10-17 (tile 1) run the softmax, two threads per
// query row, 64 score columns each (the halves swap partial maxima through
// shared memory at a named barrier of the tile's 256 threads): they read S_t
// from TMEM, keep the running max m and sum l in f32, and write
// p = 2^(s log2(e)/sqrt(dh) - m) as f16 pairs back over the first 64 columns
// of S_t, where the P V MMA reads it as its TMEM operand (no shared-memory
// round trip). The running max is only raised, and O_t rescaled through
// TMEM, when a row's max grows by more than 2^8; p <= 256 is exact enough in
// f16 and the final o = O / l uses the same m as every p it summed.
//
// Split-KV: with `splits` = S > 1 the key tiles of one (b, h, query pair) are
// cut into S contiguous ranges, one per CTA of an S-CTA thread-block cluster.
// Each CTA ends with an unnormalised partial (O_s, m_s, l_s) of its range; it
// copies O_s (f32) from TMEM into its own shared memory (the Q and K staging
// areas, idle by then) and (m_s, l_s) beside it, and after a cluster barrier
// every CTA merges 256/S of the query rows by reading all S partials through
// distributed shared memory, in split order 0..S-1:
//   m = max_s m_s,  l = sum_s 2^(m_s - m) l_s,  o = sum_s 2^(m_s - m) O_s / l,
//   lse = (m + log2 l) ln 2
// (the log-sum-exp merge of partial softmax results; the same o and lse as
// one pass over all keys up to f32 summation order). A second cluster
// barrier keeps every CTA's shared memory alive until all reads are done.
// No global scratch, no atomics: the result is deterministic for a given S.
#pragma once

#include "ptx.cuh"

namespace mot {

constexpr int kAttnThreads = 576;  // TMA warp, MMA warp, 2 x 8 softmax warps
constexpr float kLazyRescaleLog2 = 8.0f;
constexpr int kMaxAttnSplits = 8;  // portable cluster size

struct AttnFwdParams {
  CUtensorMap q_map;  // 3D {dh, N, B*Hq} f16, box {64, 128, 1}
  CUtensorMap k_map;  // 3D {dh, Lcap, B*Hkv} f16, box {64, 128, 1}
  CUtensorMap v_map;  // same as k_map
  int B, N, Hq, Hkv, Lcap, q_pairs;  // q_pairs = ceil(N / 256)
  int splits;                        // S: key-range splits = cluster size (1..kMaxAttnSplits)
  int unit0;                         // first (b, h, query pair) unit of this launch
  // causal (prefix tower): plen[b] is the branch's token count L_b (keys and
  // queries are the same N-row sequence); query i attends to keys j <= i,
  // j < L_b. Otherwise keys are [cache ; self], L_b = plen[b] + N.
  int causal;
  int plen[kMaxBatch];
  float scale_log2;  // log2(e) / sqrt(dh)
  __half* out;       // [B*N, Hq*dh] token-major
  float* lse;        // [B, Hq, N] natural-log sum of exp(scores), or null
  int* status;
};

struct AttnSmem {
  static constexpr uint32_t kTile = 32768;  // 128 rows x 128 f16
  static constexpr uint32_t kQ = 0;         // two query tiles
  static constexpr uint32_t kK = kQ + 2 * kTile;
  static constexpr uint32_t kV = kK + 2 * kTile;
  static constexpr uint32_t kXch = kV + 2 * kTile;  // [2 tiles][2 buffers][2 halves][128] f32
  // split-KV partials (after the last MMA): O_t f32 [128 rows][128 cols] of
  // query tile t at kPart + t * 64 KB (over the Q and K areas), 16-byte chunks
  // of a row permuted by chunk ^ (row & 7); (m, l) per row at kStats
  static constexpr uint32_t kPart = kQ;
  static constexpr uint32_t kStats = kXch + 4096;  // [2 tiles][128 rows] float2
  static constexpr uint32_t kBar = kStats + 2048;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;
};

// Half a row of S (64 f32 scores) in registers: two TMEM loads, one wait.
struct HalfRowS {
  uint32_t r[2][32];
};

__device__ __forceinline__ void load_half_row(uint32_t taddr, HalfRowS& s) {
  tmem_ld32(taddr, s.r[0]);
  tmem_ld32(taddr + 32, s.r[1]);
  tmem_ld_wait();
}

// max over this thread's 64 scores (columns col0 + [0, 64); >= valid masked)
template <bool kFull>
__device__ __forceinline__ float half_row_max(const HalfRowS& s, int col0, int valid) {
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const int col = col0 + c * 32 + i;
      const float v0 = (kFull || col < valid) ? __uint_as_float(s.r[c][i]) : -INFINITY;
      const float v1 = (kFull || col + 1 < valid) ? __uint_as_float(s.r[c][i + 1]) : -INFINITY;
      mx[(i >> 1) & 3] = fmax3(mx[(i >> 1) & 3], v0, v1);
    }
  }
  return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// p = 2^(s c - m) for this thread's 64 scores, written as 32 f16 pairs at P
// columns [col0/2, col0/2 + 32) of S; returns their sum. Masked keys are
// zeroed after the exponential. One pair in four goes through the FMA-pipe
// exponential, the rest through the MUFU.
template <bool kFull>
__device__ __forceinline__ float half_row_exp_store(const HalfRowS& s, uint32_t taddr_p, int col0, int valid,
                                                    float scale, float neg_m) {
  float sa = 0.f, sb = 0.f, sc = 0.f, sd = 0.f;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const int col = col0 + c * 32 + i;
      float x0, x1;
      ffma2(x0, x1, __uint_as_float(s.r[c][i]), __uint_as_float(s.r[c][i + 1]), scale, scale, neg_m, neg_m);
      float p0, p1;
      if (((i >> 1) & 3) == 3) {
        exp2_poly2(p0, p1, x0, x1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      if (!kFull) {
        p0 = col < valid ? p0 : 0.f;
        p1 = col + 1 < valid ? p1 : 0.f;
      }
      if ((i >> 1) & 1)
        fadd2(sc, sd, sc, sd, p0, p1);
      else
        fadd2(sa, sb, sa, sb, p0, p1);
      pk[i >> 1] = pack_half2(p0, p1);
    }
    tmem_st16(taddr_p + c * 16, pk);
  }
  return (sa + sb) + (sc + sd);
}

// Merge of query rows over the S partials of its cluster (split-KV): a warp
// takes kRows rows at once, lane l owning output columns [4l, 4l + 4) of
// each; every distributed-shared-memory load of the group is issued before
// the first one is used, so the remote latency is paid once per group.
template <int kRows, int kMaxS>
__device__ __forceinline__ void merge_rows(const AttnFwdParams& p, uint8_t* smem, int S, const int (&R)[kRows],
                                           int nrows, int b, int h, int qp, int lane) {
  float ms[kRows][kMaxS], ls[kRows][kMaxS];
  float4 os[kRows][kMaxS];
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    if (i >= nrows) break;
    const int t = R[i] >> 7, row = R[i] & 127;
    const uint32_t stats = smem_u32(smem + AttnSmem::kStats) + static_cast<uint32_t>(t * 128 + row) * 8u;
    const int chunk = (lane & ~7) | ((lane & 7) ^ (row & 7));
    const uint32_t part = smem_u32(smem + AttnSmem::kPart) + static_cast<uint32_t>(t) * 65536u +
                          static_cast<uint32_t>(row) * 512u + static_cast<uint32_t>(chunk) * 16u;
#pragma unroll
    for (int s = 0; s < kMaxS; ++s) {
      if (s < S) {
        const float2 st = ld_cluster_f2(map_to_rank(stats, s));
        os[i][s] = ld_cluster_f4(map_to_rank(part, s));
        ms[i][s] = st.x;
        ls[i][s] = st.y;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    if (i >= nrows) break;
    const int qrow = qp * 256 + R[i];
    float m = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxS; ++s)
      if (s < S) m = fmaxf(m, ms[i][s]);
    float l = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxS; ++s) {
      if (s < S) {
        const float w = ex2_approx(ms[i][s] - m);
        l = fmaf(ls[i][s], w, l);
        o0 = fmaf(os[i][s].x, w, o0);
        o1 = fmaf(os[i][s].y, w, o1);
        o2 = fmaf(os[i][s].z, w, o2);
        o3 = fmaf(os[i][s].w, w, o3);
      }
    }
    if (qrow >= p.N) continue;
    const float inv_l = 1.0f / l;
    uint2 wv;
    wv.x = pack_half2(o0 * inv_l, o1 * inv_l);
    wv.y = pack_half2(o2 * inv_l, o3 * inv_l);
    __half* dst = p.out + (static_cast<long long>(b) * p.N + qrow) * (p.Hq * 128) + h * 128 + lane * 4;
    *reinterpret_cast<uint2*>(dst) = wv;
    if (p.lse && lane == 0)
      p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
  }
}

// This CTA's share of the cluster's merge: rows [r0, r1) of the 256, warp w
// taking rows r0 + w, r0 + w + 18, ... in groups of kRows.
template <int kRows, int kMaxS>
__device__ __forceinline__ void merge_share(const AttnFwdParams& p, uint8_t* smem, int S, int r0, int r1, int b,
                                            int h, int qp, int warp, int lane) {
  constexpr int kWarps = kAttnThreads / 32;
  for (int base = r0 + warp; base < r1; base += kRows * kWarps) {
    int R[kRows];
    int n = 0;
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      R[i] = base + i * kWarps;
      if (R[i] < r1) n = i + 1;
    }
    merge_rows<kRows, kMaxS>(p, smem, S, R, n, b, h, qp, lane);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnFwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr uint32_t T32 = AttnSmem::kTile;
  uint8_t* sQ = smem + AttnSmem::kQ;
  uint8_t* sK = smem + AttnSmem::kK;
  uint8_t* sV = smem + AttnSmem::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2] ring stages
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2] query tiles
  uint64_t* p_full = bars + 11;   // [2]
  uint64_t* o_done = bars + 13;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = warp_id(), lane = lane_id();
  const int S = p.splits;
  int bid = blockIdx.x;
  const int split = bid % S;  // = rank in the cluster (clusters are S consecutive CTAs along x)
  bid = p.unit0 + bid / S;
  const int qp = bid % p.q_pairs;
  bid /= p.q_pairs;
  const int h = bid % p.Hq;
  const int b = bid / p.Hq;
  const int g = h / (p.Hq / p.Hkv);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
      mbar_init(&o_done[i], 1);
    }
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
  grid_dep_launch();
  grid_dep_wait();  // inputs of this call (q^, K, V, prefix lengths) are final from here on
  const int L = p.causal ? p.plen[b] : p.plen[b] + p.N;
  // causal: no key past the unit's last query row is needed
  const int T = ((p.causal ? min(L, qp * 256 + 256) : L) + 127) >> 7;
  // this CTA's key tiles [j0, j0 + Ts); the host guarantees S <= T, so Ts >= 1
  const int j0 = split * T / S;
  const int Ts = (split + 1) * T / S - j0;
  const WaitGuard wg{abort_flag, p.status};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.q_map);
      tma_prefetch_desc(&p.k_map);
      tma_prefetch_desc(&p.v_map);
      const int qz = b * p.Hq + h, kz = b * p.Hkv + g;
      mbar_expect_tx(q_full, 2 * T32);
      for (int t = 0; t < 2; ++t) {
        tma_load_3d(sQ + t * T32, &p.q_map, q_full, 0, qp * 256 + t * 128, qz);
        tma_load_3d(sQ + t * T32 + 16384, &p.q_map, q_full, 64, qp * 256 + t * 128, qz);
      }
      for (int jj = 0; jj < Ts; ++jj) {
        const int s = jj & 1;
        const uint32_t ph = (jj >> 1) & 1;
        const int key0 = (j0 + jj) * 128;
        mbar_wait(&k_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&k_full[s], T32);
        tma_load_3d(sK + s * T32, &p.k_map, &k_full[s], 0, key0, kz);
        tma_load_3d(sK + s * T32 + 16384, &p.k_map, &k_full[s], 64, key0, kz);
        mbar_wait(&v_empty[s], ph ^ 1u, wg);
        mbar_expect_tx(&v_full[s], T32);
        tma_load_3d(sV + s * T32, &p.v_map, &v_full[s], 0, key0, kz);
        tma_load_3d(sV + s * T32 + 16384, &p.v_map, &v_full[s], 64, key0, kz);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(128, 128, false, false, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(128, 128, false, false, false, true);
      const uint32_t q_addr[2] = {smem_u32(sQ), smem_u32(sQ + T32)};
      auto issue_s = [&](int t, int jj) {
        const uint32_t k_addr = smem_u32(sK + (jj & 1) * T32);
        const uint32_t qa = t ? q_addr[1] : q_addr[0];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + t * 128u, kmajor_desc(qa, kk, 16384), kmajor_desc(k_addr, kk, 16384), idesc_qk, kk > 0);
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int jj) {
        const uint32_t va = smem_u32(sV + (jj & 1) * T32);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + 256u + t * 128u, tmem + t * 128u + kk * 8u, mnmajor_desc(va, kk, 16384), idesc_pv,
                  (jj | kk) != 0);
        umma_commit(&o_done[t]);
      };
      mbar_wait(q_full, 0, wg);
      mbar_wait(&k_full[0], 0, wg);
      tc_fence_after();
      issue_s(0, 0);
      issue_s(1, 0);
      umma_commit(&k_empty[0]);
      for (int jj = 0; jj < Ts; ++jj) {
        const int s = jj & 1;
        const bool more = jj + 1 < Ts;
        mbar_wait(&v_full[s], (jj >> 1) & 1, wg);
        mbar_wait(&p_full[0], jj & 1, wg);
        tc_fence_after();
        issue_pv(0, jj);
        if (more) {
          mbar_wait(&k_full[(jj + 1) & 1], ((jj + 1) >> 1) & 1, wg);
          tc_fence_after();
          issue_s(0, jj + 1);  // overwrites P_0 only after the P V MMA above (in-order issue)
        }
        mbar_wait(&p_full[1], jj & 1, wg);
        tc_fence_after();
        issue_pv(1, jj);
        umma_commit(&v_empty[s]);
        if (more) {
          issue_s(1, jj + 1);
          umma_commit(&k_empty[(jj + 1) & 1]);
        }
      }
    }
  } else {
    const int t = (warp - 2) >> 3;           // query tile of these 8 warps
    const int half = ((warp - 2) >> 2) & 1;  // score columns [64 half, 64 half + 64)
    const int quarter = warp & 3;            // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int col0 = half * 64;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + t * 128u + lane_off;
    const uint32_t tO = tmem + 256u + t * 128u + lane_off;
    float* xch = reinterpret_cast<float*>(smem + AttnSmem::kXch) + t * 512;  // [2 buffers][2 halves][128]
    const int bar_id = 1 + t;
    float m_run = -INFINITY, l_run = 0.f;  // l_run: this half's partial row sum
    // keys this row may see: all L, or (causal) those up to its own position
    const int key_end = p.causal ? min(L, qp * 256 + t * 128 + row + 1) : L;
    for (int jj = 0; jj < Ts; ++jj) {
      mbar_wait(&s_full[t], jj & 1, wg);
      tc_fence_after();
      const int valid = key_end - (j0 + jj) * 128;  // keys of this tile this row sees (>= 1 on the first tile)
      // warp-uniform: the exp/store path issues tcgen05.st, a warp-collective
      // instruction, so all 32 lanes must take the same template branch
      // (in causal mode `valid` differs from row to row)
      const bool full = __all_sync(0xffffffffu, valid >= 128);
      HalfRowS srow;
      load_half_row(tS + col0, srow);
      const float pm = full ? half_row_max<true>(srow, col0, valid) : half_row_max<false>(srow, col0, valid);
      float* xb = xch + (jj & 1) * 256;
      xb[half * 128 + row] = pm;
      // both halves hold their scores in registers past this barrier, so P
      // may overwrite S; the partial maxima are exchanged through smem
      named_bar_sync(bar_id, 256);
      const float m_tile = fmaxf(pm, xb[(half ^ 1) * 128 + row]) * p.scale_log2;
      bool need = false;
      float m_new = m_run;
      if (jj == 0) {
        m_new = m_tile;
      } else if (m_tile > m_run + kLazyRescaleLog2) {
        need = true;
        m_new = m_tile;
      }
      // o_done completes once per P V of this tile; waiting on every phase in
      // order keeps the parity unambiguous. S_t of this tile was issued after
      // the previous P V, so that P V is already complete here: O is stable.
      if (jj >= 1) {
        mbar_wait(&o_done[t], (jj - 1) & 1, wg);
        tc_fence_after();
      }
      const float m_old = m_run;
      m_run = m_new;
      const float part = full ? half_row_exp_store<true>(srow, tS + half * 32, col0, valid, p.scale_log2, -m_run)
                              : half_row_exp_store<false>(srow, tS + half * 32, col0, valid, p.scale_log2, -m_run);
      // this half's O columns move to the new max (the next P V waits for p_full)
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2_approx(m_old - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + col0 + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + col0 + c * 32, r);
        }
        l_run *= alpha;
      }
      tmem_st_wait();
      l_run += part;
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // epilogue: l = sum of the two halves
    mbar_wait(&o_done[t], (Ts - 1) & 1, wg);
    tc_fence_after();
    float* xb = xch + (Ts & 1) * 256;
    xb[half * 128 + row] = l_run;
    named_bar_sync(bar_id, 256);
    const float l_row = l_run + xb[(half ^ 1) * 128 + row];
    if (S == 1) {
      // o = O / l for this half's 64 columns
      const int qrow = qp * 256 + t * 128 + row;
      const float inv_l = 1.0f / l_row;
      __half* dst = p.out + (static_cast<long long>(b) * p.N + qrow) * (p.Hq * 128) + h * 128 + col0;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + col0 + c * 32, r);
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
      if (p.lse && half == 0 && qrow < p.N)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] = (m_run + __log2f(l_row)) * 0.69314718055994531f;
    } else {
      // split-KV partial: unnormalised O (this half's 64 columns) into this
      // CTA's shared memory; the last MMA of the CTA is complete (every MMA
      // reading Q or K was issued before the final P V of either tile)
      float* part = reinterpret_cast<float*>(smem + AttnSmem::kPart + t * 65536) + row * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + col0 + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int chunk = half * 16 + c * 8 + i;
          const int phys = (chunk & ~7) | ((chunk & 7) ^ (row & 7));
          *reinterpret_cast<uint4*>(part + phys * 4) =
              make_uint4(r[4 * i + 0], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
        }
      }
      if (half == 0)
        reinterpret_cast<float2*>(smem + AttnSmem::kStats)[t * 128 + row] = make_float2(m_run, l_row);
    }
  }
  if (S > 1) {
    // every CTA of the cluster has its partial in shared memory
    __syncwarp();
    cluster_sync();
    const int r0 = split * 256 / S, r1 = (split + 1) * 256 / S;
    if (S == 2)
      merge_share<4, 2>(p, smem, S, r0, r1, b, h, qp, warp, lane);
    else if (S <= 4)
      merge_share<2, 4>(p, smem, S, r0, r1, b, h, qp, warp, lane);
    else
      merge_share<1, kMaxAttnSplits>(p, smem, S, r0, r1, b, h, qp, warp, lane);
    // no CTA leaves (releasing its shared memory) before all reads are done
    __syncwarp();
    cluster_sync();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mot
