// mot_attn.cu -- C ABI of the gen-tower attention layer (see include/mot_attn.h).
//
// Forward launch sequence on the caller's stream (r = LoRA rank, s = alpha/r):
//   build_kv      prefix rows of the f16 key/value buffers, zero tail rows;
//                 [r>0] A_o and lora_up -> f16 (they meet f16 operands)
//   [r>0] lora-down GEMM    u_qkv = s x [A_q; A_k; A_v]^T           (bf16)
//   QKV GEMM + epilogue     x W_qkv^T + u B^T -> RMSNorm -> RoPE -> q^, K, V
//   attention               o = softmax(q^ K^T / sqrt(dh)) V         (f16)
//   [r>0] lora-down GEMM    u_o = s o A_o^T                          (bf16)
//   O GEMM                  y = o W_o^T + u_o B_o^T                  (bf16 + f32)
// Backward (LoRA training; frozen base, gains and cache):
//   [r>0] B_q/B_k/B_v -> f16;  g_o = dy B_o
//   dO GEMM + epilogue      dO = dy W_o + s g_o A_o ; D = rowsum(dO o)
//   [r>0] dB_o = dy^T u_o ;  dA_o = s g_o^T o
//   attention backward      dq^ (all keys), dk^, dv (self keys) -> RoPE^-1 ->
//                           RMSNorm backward -> pre-norm dq, dk, dv (f16)
//   [r>0] g_j = d{q,k,v} B_j ; dB_j = d{q,k,v}^T u_j ; dA_j = s g_j^T x
//   dX GEMM                 dx = dq W_q + dk W_k + dv W_v + s sum_j g_j A_j
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "mot_attn.h"
#include "mot_attn_dev.h"
#include "ptx.cuh"
#include "gemm.cuh"
#include "attn_fwd.cuh"
#include "attn_bwd.cuh"
#include "aux.cuh"

using namespace mot;

namespace {

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encode_ready() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

bool encode(CUtensorMap* m, const void* ptr, bool bf16, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  if (!encode_ready() || !ptr) return false;
  for (int i = 0; i < rank; ++i)
    if (dims[i] == 0) return false;
  const cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank,
                  const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major operand: row-major [outer, inner] 16-bit tensor (row stride `ld`
// elements), box = [box_outer rows, 64 columns], 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer, uint64_t ld,
           uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_outer};
  return encode(m, ptr, bf16, 2, dims, strides, box);
}

// MN-major operand: the same tensor read as 64 x 64 boxes (64 contiguous
// M/N elements by 64 K rows).
bool map2d_mn(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer, uint64_t ld) {
  return map2d(m, ptr, bf16, inner, outer, ld, 64);
}

// 3-D map over a contiguous f16 [outer, mid, inner] tensor, box [1, 128, 64].
bool map3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer) {
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner * 2, mid * inner * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  return encode(m, ptr, false, 3, dims, strides, box);
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// one staging slot of the host-buffer forward: x, y, k_cache, v_cache, each
// 256-byte aligned
struct HostStaging {
  size_t x, kv, slot;
};
HostStaging host_staging(const mot_attn_config& c, int B, int N, int P) {
  HostStaging s;
  s.x = round_up(static_cast<size_t>(B) * N * c.hidden * 2, 256);
  s.kv = round_up(static_cast<size_t>(B) * c.n_kv_heads * P * c.head_dim * 2, 256);
  s.slot = 2 * s.x + 2 * s.kv;
  return s;
}

// ------------------------------------------------------------------ layouts
// split-K partial tiles of the LoRA-gradient GEMMs (backward workspace)
constexpr size_t kSplitWsBytes = size_t(16) << 20;
constexpr int kSplitCounters = 1024;

struct Layout {
  int B = 0, N = 0, P = 0, M = 0, Lcap = 0, r = 0, RP = 0;
  // activations: in `saved` for training, else after the forward scratch
  size_t o_q = 0, o_k = 0, o_v = 0, o_attn = 0, o_lse = 0, o_xhat = 0, o_rstd = 0, o_uqkv = 0, o_uo = 0,
         o_uohi = 0, o_uolo = 0, act_bytes = 0;
  // forward scratch: f16 copies of the LoRA tensors that meet f16 operands
  size_t w_ao16 = 0, w_bo16 = 0, w_bqkv16 = 0, fwd_scratch = 0;
  // backward scratch (workspace)
  size_t b_do = 0, b_delta = 0, b_dqkv = 0, b_gohi = 0, b_golo = 0, b_go16 = 0, b_ghi = 0, b_glo = 0, b_bqkv16 = 0,
         b_split = 0, bwd_scratch = 0;
};

Layout make_layout(const mot_attn_config& c, int B, int N, int P, bool train) {
  Layout L;
  L.B = B;
  L.N = N;
  L.P = P;
  L.M = B * N;
  L.Lcap = static_cast<int>(round_up(static_cast<size_t>(P + N), 128));
  L.r = c.lora_rank;
  L.RP = L.r ? static_cast<int>(round_up(L.r, 64)) : 0;
  const size_t dh = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.hidden, M = L.M, r = L.r, RP = L.RP;
  const size_t nqkv = (Hq + 2 * Hkv) * dh;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 1024);
    return o;
  };
  L.o_q = take(B * Hq * N * dh * 2);
  L.o_k = take(B * Hkv * L.Lcap * dh * 2);
  L.o_v = take(B * Hkv * L.Lcap * dh * 2);
  L.o_attn = take(M * Hq * dh * 2);
  L.o_lse = take(train ? B * Hq * N * 4 : 0);
  L.o_xhat = take(train ? M * (Hq + Hkv) * dh * 2 : 0);
  L.o_rstd = take(train ? M * (Hq + Hkv) * 4 : 0);
  L.o_uqkv = take(r ? M * 3 * RP * 2 : 0);
  L.o_uo = take(r ? M * RP * 2 : 0);
  L.o_uohi = take(train && r ? M * RP * 2 : 0);
  L.o_uolo = take(train && r ? M * RP * 2 : 0);
  L.act_bytes = off;
  off = 0;
  L.w_ao16 = take(r ? r * Hq * dh * 2 : 0);
  L.w_bo16 = take(r ? d * r * 2 : 0);
  L.w_bqkv16 = take(r ? nqkv * r * 2 : 0);
  L.fwd_scratch = off;
  off = 0;
  L.b_do = take(M * Hq * dh * 2);
  L.b_delta = take(B * Hq * N * 4);
  L.b_dqkv = take(M * nqkv * 2);
  L.b_gohi = take(r ? M * RP * 2 : 0);
  L.b_golo = take(r ? M * RP * 2 : 0);
  L.b_go16 = take(r ? M * RP * 2 : 0);
  L.b_ghi = take(r ? M * 3 * RP * 2 : 0);
  L.b_glo = take(r ? M * 3 * RP * 2 : 0);
  L.b_bqkv16 = take(r ? nqkv * r * 2 : 0);
  L.b_split = take(r ? 2 * kSplitWsBytes : 0);  // caller's stream, side stream
  L.bwd_scratch = c.enable_backward ? off : 0;
  return L;
}

mot_status check_config(const mot_attn_config* c) {
  if (!c) return MOT_ERR_INVALID_ARGUMENT;
  if (c->hidden <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 || c->lora_rank < 0 ||
      c->max_batch <= 0 || c->max_img_tokens <= 0 || c->max_prefix < 0 || !(c->rms_eps >= 0.f) ||
      !(c->rope_theta > 0.0))
    return MOT_ERR_INVALID_ARGUMENT;
  if (c->lora_rank > 0 && !(c->lora_alpha == c->lora_alpha)) return MOT_ERR_INVALID_ARGUMENT;
  if (c->head_dim != 128 || c->hidden != c->n_q_heads * c->head_dim || c->n_q_heads % c->n_kv_heads != 0 ||
      (c->n_kv_heads * c->head_dim) % 256 != 0 || c->hidden % 256 != 0 || c->lora_rank % 8 != 0 ||
      c->lora_rank > 128 || c->max_batch > kMaxBatch)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(c->max_batch) * c->max_img_tokens > (1ll << 30)) return MOT_ERR_UNSUPPORTED_SHAPE;
  return MOT_OK;
}

template <class K>
void set_smem_attr(K kernel, size_t bytes) {
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

// Split count for a GEMM of `tiles` output tiles and total_kb k-blocks: the
// fewest splits that come close to the best SM balance ceil(items/SMs)/S,
// each split costing a little for its partial-tile round trip; at most 16,
// at least two k-blocks per split, partials within the split workspace.
int pick_splits(int tiles, int total_kb, int num_sms, int bn, size_t cap_bytes) {
  int best = 1;
  double best_cost = static_cast<double>((tiles + num_sms - 1) / num_sms);
  for (int sp = 2; sp <= 16 && 2 * sp <= total_kb; ++sp) {
    if (static_cast<size_t>(tiles) * sp * bn * kBM * 4 > cap_bytes) break;
    const double cost = static_cast<double>((tiles * sp + num_sms - 1) / num_sms) / sp + 0.02 * (sp - 1);
    if (cost < best_cost - 1e-9) {
      best = sp;
      best_cost = cost;
    }
  }
  return best;
}

// second B operand of a dual segment (same box coordinates, map b2 in every region)
void set_dual(GemmSeg& sg, int b2) {
  sg.dual = 1;
  for (int i = 0; i < kMaxRegions; ++i) sg.b2_map[i] = b2;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream drains (once all that kernel's CTAs
// are running) and runs its prologue (barriers, TMEM, descriptor prefetch);
// its grid_dep_wait then holds every global access until the previous grid
// has completed. Every kernel launched this way calls grid_dep_wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       const Args&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// launch_pdl for a kernel whose CTAs form clusters of `cluster` CTAs along x
// (grid.x a multiple of it); cluster 1 is a plain launch
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               int cluster, const Args&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Split-KV plan of the attention forward: how many clusters of S CTAs
// (split-KV ranges) fit on the GPU at once, per S (index 1 = plain CTAs,
// one per SM), queried once per handle from the occupancy calculator.
void attn_cluster_caps(int (&cap)[kMaxAttnSplits + 1], int num_sms) {
  set_smem_attr(attn_fwd_kernel, AttnSmem::kBytes);
  cap[0] = 0;
  cap[1] = num_sms;
  for (int S = 2; S <= kMaxAttnSplits; ++S) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(S * 64);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = AttnSmem::kBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_fwd_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cap[S] = n;
  }
}

// Split-KV plan of one attention forward. Units (b, h, query pair) run as
// one CTA each in waves of cap[1] (one CTA per SM); when the last wave is
// partly empty, the units of that tail may instead run as clusters of S
// CTAs, each taking 1/S of the keys, merged through distributed shared
// memory (a second launch, after the full waves). Cost in key steps (one
// 128-key tile for both query tiles of a CTA, ~2.2 us on B200): per CTA a
// fixed prologue/epilogue (kAttnFixedSteps) plus its key tiles, plus the
// merge for split CTAs (kAttnMergeSteps); per launch, waves of cap[S]
// clusters. Both constants come from timing forced split counts on the
// 512^2, 1024^2 and 2048^2 workloads (a split of every unit never paid off
// there: the fixed cost per CTA outweighs the balance it buys).
constexpr double kAttnFixedSteps = 2.2, kAttnMergeSteps = 1.5;

struct AttnPlan {
  int full_units;  // units [0, full_units) unsplit
  int splits;      // the rest as clusters of `splits` CTAs (1: none)
};

AttnPlan plan_attention(const int (&cap)[kMaxAttnSplits + 1], int units, int t_min, int t_max) {
  const double step_full = t_max + kAttnFixedSteps;
  const int waves = (units + cap[1] - 1) / cap[1];
  AttnPlan best{units, 1};
  double best_cost = waves * step_full;
  const int full = (units / cap[1]) * cap[1];
  const int tail = units - full;
  if (tail == 0) return best;
  for (int S = 2; S <= kMaxAttnSplits && S <= t_min; ++S) {
    if (cap[S] <= 0) continue;
    const double tail_waves = static_cast<double>((tail + cap[S] - 1) / cap[S]);
    const double per_cta = static_cast<double>((t_max + S - 1) / S) + kAttnFixedSteps + kAttnMergeSteps;
    const double cost = (full / cap[1]) * step_full + tail_waves * per_cta;
    if (cost < best_cost - 1e-9) {
      best = {full, S};
      best_cost = cost;
    }
  }
  return best;
}

// let launch_gemm split K (1-CTA kernel; partials in ws of cap bytes, counters in cnt)
void enable_split(GemmCore& c, void* ws, int* cnt, size_t cap = kSplitWsBytes) {
  c.k_splits = -1;
  c.split_ws = static_cast<float4*>(ws);
  c.split_cnt = cnt;
  c.split_cap = cap;
}

template <int BN, int STAGES, class Epi, bool kDual = false>
cudaError_t launch_gemm(const GemmCore& core, const typename Epi::Params& ep, int num_sms, cudaStream_t st) {
  static_assert(sizeof(GemmArgs<Epi>) <= 4096, "kernel parameter block");
  using L = GemmSmem<BN, STAGES, kDual>;
  static_assert(L::kBytes <= 232448, "shared memory");
  auto kern = gemm_kernel<BN, STAGES, Epi, kDual>;
  static std::once_flag once;
  std::call_once(once, [&] { set_smem_attr(kern, L::kBytes); });
  GemmArgs<Epi> args;
  args.core = core;
  args.epi = ep;
  const int tiles = core.tiles_m * core.tiles_n;
  // every split of every tile needs a k-block: bound by the smallest tile total
  int total_kb = 1 << 30;
  for (int r = 0; r < std::max(1, core.num_regions); ++r) {
    int t = 0;
    for (int i = 0; i < core.num_segs; ++i) t += core.segs[i].kb_r[r] > 0 ? core.segs[i].kb_r[r] : core.segs[i].kb;
    total_kb = std::min(total_kb, t);
  }
  args.core.total_kb = total_kb;
  args.core.k_splits =
      core.k_splits < 0 && tiles <= kSplitCounters ? pick_splits(tiles, total_kb, num_sms, BN, core.split_cap) : 1;
  const int items = tiles * args.core.k_splits;
  const int grid = std::max(1, std::min(items, num_sms));
  return launch_pdl(kern, dim3(grid), dim3(kGemmThreads), L::kBytes, st, args);
}

// CTA pairs a pair-kernel launch of `tiles` tiles uses: the fewest that
// finish in the same number of rounds of tiles as all SMs would, so every
// pair gets the same tile count and the SMs left over can run other work
// (the backward's side-stream GEMMs) for the whole duration
int pair_count(int tiles, int num_sms) {
  const int max_pairs = std::max(1, num_sms / 2);
  const int rounds = (tiles + max_pairs - 1) / max_pairs;
  return std::max(1, (tiles + rounds - 1) / rounds);
}

// 2-SM (CTA pair) launch: core.tiles_m counts 256-row tiles
template <int BN, int STAGES, class Epi>
cudaError_t launch_gemm2(const GemmCore& core, const typename Epi::Params& ep, int num_sms, cudaStream_t st) {
  static_assert(sizeof(GemmArgs<Epi>) <= 4096, "kernel parameter block");
  using L = Gemm2Smem<BN, STAGES>;
  static_assert(L::kBytes <= 232448, "shared memory");
  auto kern = gemm2_kernel<BN, STAGES, Epi>;
  static std::once_flag once;
  std::call_once(once, [&] { set_smem_attr(kern, L::kBytes); });
  GemmArgs<Epi> args;
  args.core = core;
  args.epi = ep;
  // the fewest pairs that finish in the same number of rounds of tiles: every
  // pair gets the same tile count, and the SMs left over can run other work
  // (the backward's side-stream GEMMs) for the whole duration
  const int pairs = pair_count(core.tiles_m * core.tiles_n, num_sms);
  return launch_pdl(kern, dim3(2 * pairs), dim3(kGemmThreads), L::kBytes, st, args);
}

// tiles of the pair kernel: 256 rows of D per CTA pair
void core_pair(GemmCore& c) { c.tiles_m = (c.M + 2 * kBM - 1) / (2 * kBM); }

// BN = 64 or 128 instantiation for the narrow (LoRA-rank-wide) GEMMs
template <class Epi>
cudaError_t launch_gemm_narrow(int BN, const GemmCore& core, const typename Epi::Params& ep, int num_sms,
                               cudaStream_t st) {
  return BN == 64 ? launch_gemm<64, 8, Epi>(core, ep, num_sms, st) : launch_gemm<128, 6, Epi>(core, ep, num_sms, st);
}

// the same with dual (hi + lo) B segments; BN = 64, 128 or 192
template <class Epi>
cudaError_t launch_gemm_dual(int BN, const GemmCore& core, const typename Epi::Params& ep, int num_sms,
                             cudaStream_t st) {
  if (BN == 64) return launch_gemm<64, 6, Epi, true>(core, ep, num_sms, st);
  if (BN == 128) return launch_gemm<128, 4, Epi, true>(core, ep, num_sms, st);
  return launch_gemm<192, 3, Epi, true>(core, ep, num_sms, st);
}

void core_init(GemmCore& c, int M, int N, int BN, int b_box_rows, int* status) {
  std::memset(static_cast<void*>(&c), 0, sizeof(c));
  c.M = M;
  c.N = N;
  c.tiles_m = (M + kBM - 1) / kBM;
  c.tiles_n = (N + BN - 1) / BN;
  c.b_box_rows = b_box_rows;
  c.num_regions = 1;
  c.region_n0[0] = 0;
  c.region_n0[1] = N;
  c.status = status;
}

// one K segment whose A offset and B tensor are the same for every region
GemmSeg seg1(int a_map, int a_k0, int b_map, int kb, uint32_t idesc, bool a_mn, bool b_mn) {
  GemmSeg s;
  std::memset(static_cast<void*>(&s), 0, sizeof(s));
  s.a_map = a_map;
  for (int i = 0; i < kMaxRegions; ++i) {
    s.a_k0[i] = a_k0;
    s.b_map[i] = b_map;
  }
  s.kb = kb;
  s.idesc = idesc;
  s.a_mn = a_mn;
  s.b_mn = b_mn;
  return s;
}

EpiStore::Params store_params(int M, int N) {
  EpiStore::Params p;
  std::memset(static_cast<void*>(&p), 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.scale32 = 1.0f;
  for (auto& o : p.o16) {
    o.scale = 1.0f;
    o.residual_of = -1;
  }
  return p;
}

void set_out16(EpiStore::Params& p, int i, void* ptr, long long ld, bool bf16, float scale = 1.0f,
               int residual_of = -1) {
  p.o16[i].ptr = ptr;
  p.o16[i].ld = ld;
  p.o16[i].bf16 = bf16 ? 1 : 0;
  p.o16[i].scale = scale;
  p.o16[i].residual_of = residual_of;
}

// K-major f16 maps over the per-call f16 copies of lora_up (box rows 128)
bool lora_up16_maps(CUtensorMap* m, const __half* b16, int r, const int (&rows)[3]) {
  long long off = 0;
  for (int j = 0; j < 3; ++j) {
    if (!map2d(&m[j], b16 + off, false, r, rows[j], r, 128)) return false;
    off += static_cast<long long>(rows[j]) * r;
  }
  return true;
}

}  // namespace

// ------------------------------------------------------------------ handle
constexpr int kMaxStages = 32;
enum StageId : int {
  ST_CVT_LORA_O = 0, ST_BUILD_KV = 1, ST_LORA_DOWN_QKV = 2, ST_QKV_GEMM = 3, ST_ATTN_FWD = 4,
  ST_LORA_DOWN_O = 5, ST_O_GEMM = 6, ST_BWD_CVT = 7, ST_BWD_G_O = 8, ST_BWD_DO = 9, ST_BWD_DB_O = 10,
  ST_BWD_DA_O = 11, ST_BWD_ATTN = 12, ST_BWD_G_QKV = 13, ST_BWD_DB_QKV = 14, ST_BWD_DA_QKV = 15, ST_BWD_DX = 16,
};
const char* const kStageNames[] = {"cvt_lora_o", "build_kv", "lora_down_qkv", "qkv_gemm", "attn_fwd",
                                   "lora_down_o", "o_gemm", "bwd_cvt_lora", "bwd_g_o", "bwd_do_gemm",
                                   "bwd_db_o", "bwd_da_o", "attn_bwd", "bwd_g_qkv",
                                   "bwd_db_qkv", "bwd_da_qkv", "bwd_dx_gemm"};

struct mot_attn {
  mot_attn_config cfg;
  mot_attn_weights w;
  int rank = 0;
  float scale = 0.f;
  int RP = 0;
  __half* wo16 = nullptr;
  // backward: the frozen weights transposed, so that the dO and dx GEMMs read
  // them as K-major operands
  __nv_bfloat16* woT = nullptr;  // [Hq*dh, d] bf16, W_o^T
  __half* wqkvT16 = nullptr;     // [d, Hq*dh + 2*Hkv*dh] f16, [W_q|W_k|W_v]^T
  float* gamma = nullptr;    // [2*dh]: q gain then k gain
  float2* rope = nullptr;
  int rope_len = 0;
  int* status = nullptr;
  int* split_cnt = nullptr;  // [3][kSplitCounters] split-K arrival counters: backward (caller's / side stream), forward
  void* fsplit = nullptr;    // forward split-K partials (LoRA down), sized for max_batch x max_img_tokens
  size_t fsplit_bytes = 0;
  int device = 0;  // the CUDA device the handle was created on
  int num_sms = 148;
  int last_launches = 0;
  // attention split-KV: clusters of S CTAs resident at once, per S; a forced
  // split count (0 = planned per call) and the count the last forward used
  int attn_cap[kMaxAttnSplits + 1] = {};
  int attn_splits_forced = 0;
  int last_attn_splits = 0;
  int last_attn_full_units = 0;
  // backward: a second stream for the gradient GEMMs nothing later depends on
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  // host-buffer forward: copy-in and copy-out streams and per-slot events,
  // made on first use
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t hev_start = nullptr, hev_in[2] = {}, hev_comp[2] = {}, hev_out[2] = {};
  // optional per-launch timing (mot_dev_profile): a start and an end event
  // per launch, on the stream it ran on
  bool profile = false;
  cudaEvent_t ev[2 * kMaxStages + 2] = {};
  cudaEvent_t stage_start[kMaxStages] = {}, stage_end[kMaxStages] = {};
  int stage_ids[kMaxStages] = {};
  int stage_count = 0;
  // forward weight maps (K-major)
  CUtensorMap wq, wk, wv, wo;  // box rows 128
  CUtensorMap aq, ak, av;      // lora_down q/k/v, box rows RP
  // backward weight maps (MN-major, 64 x 64 boxes)
  CUtensorMap woT_k, wqkvT_k;  // K-major maps over woT and wqkvT16, box rows 128
  CUtensorMap ao_mn, bo_mn, aq_mn, ak_mn, av_mn;
};

namespace {

mot_status build_weight_maps(mot_attn* h) {
  const mot_attn_config& c = h->cfg;
  const uint64_t d = c.hidden, qd = c.n_q_heads * 128, kvd = c.n_kv_heads * 128;
  bool ok = map2d(&h->wq, h->w.w_q, true, d, qd, d, 128) && map2d(&h->wk, h->w.w_k, true, d, kvd, d, 128) &&
            map2d(&h->wv, h->w.w_v, true, d, kvd, d, 128) && map2d(&h->wo, h->wo16, false, qd, d, qd, 128);
  if (ok && h->rank > 0) {
    const uint64_t r = h->rank;
    const uint32_t box_a = static_cast<uint32_t>(h->RP);
    ok = map2d(&h->aq, h->w.a_q, true, d, r, d, box_a) && map2d(&h->ak, h->w.a_k, true, d, r, d, box_a) &&
         map2d(&h->av, h->w.a_v, true, d, r, d, box_a);
  }
  if (ok && c.enable_backward) {
    const uint64_t nqkv = qd + 2 * kvd;
    ok = map2d(&h->woT_k, h->woT, true, d, qd, d, 128) && map2d(&h->wqkvT_k, h->wqkvT16, false, nqkv, d, nqkv, 128);
    if (ok && h->rank > 0) {
      const uint64_t r = h->rank;
      ok = map2d_mn(&h->ao_mn, h->w.a_o, true, qd, r, qd) && map2d_mn(&h->bo_mn, h->w.b_o, true, r, d, r) &&
           map2d_mn(&h->aq_mn, h->w.a_q, true, d, r, d) && map2d_mn(&h->ak_mn, h->w.a_k, true, d, r, d) &&
           map2d_mn(&h->av_mn, h->w.a_v, true, d, r, d);
    }
  }
  return ok ? MOT_OK : MOT_ERR_CUDA;
}

// copies the handle keeps of frozen weights: f16 W_o always; for backward
// W_o^T (bf16) and [W_q|W_k|W_v]^T (f16)
cudaError_t refresh_f16_copies(mot_attn* h, cudaStream_t s) {
  const mot_attn_config& c = h->cfg;
  const long long d = c.hidden, qd = c.n_q_heads * 128, kvd = c.n_kv_heads * 128;
  CvtJobs jobs{};
  jobs.src[0] = static_cast<const __nv_bfloat16*>(h->w.w_o);
  jobs.dst[0] = h->wo16;
  jobs.n8[0] = d * qd / 8;
  jobs.count = 1;
  cvt_multi_kernel<<<4 * h->num_sms, 256, 0, s>>>(jobs, h->status);
  if (c.enable_backward) {
    const dim3 blk(32, 8);
    transpose_copy_kernel<__nv_bfloat16><<<dim3((qd + 31) / 32, (d + 31) / 32), blk, 0, s>>>(
        static_cast<const __nv_bfloat16*>(h->w.w_o), static_cast<int>(d), static_cast<int>(qd), h->woT, d, 0);
    const void* src[3] = {h->w.w_q, h->w.w_k, h->w.w_v};
    const long long rows[3] = {qd, kvd, kvd};
    const long long nqkv = qd + 2 * kvd;
    long long off = 0;
    for (int i = 0; i < 3; ++i) {
      transpose_copy_kernel<__half><<<dim3((d + 31) / 32, (rows[i] + 31) / 32), blk, 0, s>>>(
          static_cast<const __nv_bfloat16*>(src[i]), static_cast<int>(rows[i]), static_cast<int>(d), h->wqkvT16,
          nqkv, static_cast<int>(off));
      off += rows[i];
    }
  }
  return cudaGetLastError();
}

void release(mot_attn* h) {
  if (!h) return;
  for (cudaEvent_t e : h->ev)
    if (e) cudaEventDestroy(e);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  const cudaEvent_t hev[] = {h->hev_start, h->hev_in[0], h->hev_in[1], h->hev_comp[0], h->hev_comp[1],
                             h->hev_out[0], h->hev_out[1]};
  for (cudaEvent_t e : hev)
    if (e) cudaEventDestroy(e);
  if (h->h2d) cudaStreamDestroy(h->h2d);
  if (h->d2h) cudaStreamDestroy(h->d2h);
  cudaFree(h->wo16);
  cudaFree(h->wqkvT16);
  cudaFree(h->woT);
  cudaFree(h->gamma);
  cudaFree(h->rope);
  cudaFree(h->status);
  cudaFree(h->split_cnt);
  cudaFree(h->fsplit);
  delete h;
}

// launch bookkeeping shared by forward and backward (of the attention and
// of the MLP handle): error capture, launch count and the optional
// per-launch events
template <class H>
struct LaunchesT {
  H* h;
  cudaStream_t st;   // the caller's stream
  cudaStream_t cur;  // where the next launch goes: st, or the handle's side stream
  int count = 0;
  int stage = 0;
  int nev = 0;
  bool side_pending = false;  // side-stream work not yet joined into st
  cudaEvent_t last[2] = {};   // latest profiling event on st / on the side stream
  cudaError_t err = cudaSuccess;
  LaunchesT(H* handle, cudaStream_t s) : h(handle), st(s), cur(s) {
    if (h->profile) last[0] = mark(st);
  }
  // every return path leaves st ordered after the side stream's work
  ~LaunchesT() {
    if (side_pending) join();
  }
  void note(cudaError_t e) {
    if (e != cudaSuccess && err == cudaSuccess) err = e;
  }
  cudaEvent_t mark(cudaStream_t s) {
    if (nev >= static_cast<int>(sizeof(h->ev) / sizeof(h->ev[0]))) return nullptr;
    cudaEvent_t e = h->ev[nev++];
    cudaEventRecord(e, s);
    return e;
  }
  // later launches go to the side stream, after all work issued so far on st
  void fork() {
    note(cudaEventRecord(h->ev_fork, st));
    note(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
    cur = h->side;
    side_pending = true;
    if (h->profile) last[1] = mark(h->side);
  }
  void to_main() { cur = st; }
  // st waits for all work issued on the side stream
  void join() {
    note(cudaEventRecord(h->ev_join, h->side));
    note(cudaStreamWaitEvent(st, h->ev_join, 0));
    cur = st;
    side_pending = false;
  }
  void done(cudaError_t e) {
    note(e);
    if (h->profile && count < kMaxStages) {
      const int k = cur == st ? 0 : 1;
      h->stage_ids[count] = stage;
      h->stage_start[count] = last[k];
      last[k] = h->stage_end[count] = mark(cur);
    }
    ++count;
  }
  mot_status finish() {
    if (side_pending) join();
    h->last_launches = count;
    h->stage_count = std::min(count, kMaxStages);
    return err == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
  }
};
using Launches = LaunchesT<mot_attn>;

}  // namespace

extern "C" {

const char* mot_status_string(mot_status s) {
  switch (s) {
    case MOT_OK: return "ok";
    case MOT_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOT_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOT_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MOT_ERR_WORKSPACE_TOO_SMALL: return "workspace or saved buffer too small";
    case MOT_ERR_NO_SAVED_STATE: return "backward needs the saved state of a training forward";
    case MOT_ERR_CUDA: return "CUDA error";
    case MOT_ERR_NUMERIC: return "f16 intermediate overflow";
    case MOT_ERR_TIMEOUT: return "bounded in-kernel wait expired";
  }
  return "unknown status";
}

mot_status mot_attn_query_host_staging(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens,
                                       int32_t prefix_max, size_t* staging_bytes) {
  mot_status st = check_config(cfg);
  if (st != MOT_OK) return st;
  if (!staging_bytes || batch <= 0 || img_tokens <= 0 || prefix_max < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (batch > cfg->max_batch || img_tokens > cfg->max_img_tokens || prefix_max > cfg->max_prefix)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  *staging_bytes = 2 * host_staging(*cfg, batch, img_tokens, prefix_max).slot;
  return MOT_OK;
}

mot_status mot_attn_query_sizes(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens, int32_t prefix_max,
                                size_t* workspace_bytes, size_t* saved_bytes) {
  mot_status st = check_config(cfg);
  if (st != MOT_OK) return st;
  if (batch <= 0 || img_tokens <= 0 || prefix_max < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (batch > cfg->max_batch || img_tokens > cfg->max_img_tokens || prefix_max > cfg->max_prefix)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  const Layout inf = make_layout(*cfg, batch, img_tokens, prefix_max, false);
  const Layout trn = make_layout(*cfg, batch, img_tokens, prefix_max, true);
  if (workspace_bytes) *workspace_bytes = std::max({inf.fwd_scratch + inf.act_bytes, trn.fwd_scratch, trn.bwd_scratch});
  if (saved_bytes) *saved_bytes = trn.act_bytes;
  return MOT_OK;
}

mot_status mot_attn_create(const mot_attn_config* cfg, const mot_attn_weights* wts, void* stream, mot_attn_t* out) {
  if (!out) return MOT_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  mot_status st = check_config(cfg);
  if (st != MOT_OK) return st;
  if (!wts || !wts->w_q || !wts->w_k || !wts->w_v || !wts->w_o || !wts->q_norm || !wts->k_norm)
    return MOT_ERR_INVALID_ARGUMENT;
  if (cfg->lora_rank > 0 && (!wts->a_q || !wts->a_k || !wts->a_v || !wts->a_o || !wts->b_q || !wts->b_k ||
                             !wts->b_v || !wts->b_o))
    return MOT_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {wts->w_q, wts->w_k, wts->w_v, wts->w_o, wts->q_norm, wts->k_norm,
                        wts->a_q, wts->a_k, wts->a_v, wts->a_o, wts->b_q, wts->b_k, wts->b_v, wts->b_o};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  if (!encode_ready()) return MOT_ERR_CUDA;

  mot_attn* h = new (std::nothrow) mot_attn();
  if (!h) return MOT_ERR_CUDA;
  h->cfg = *cfg;
  h->w = *wts;
  h->rank = cfg->lora_rank;
  h->scale = h->rank ? cfg->lora_alpha / static_cast<float>(h->rank) : 0.f;
  h->RP = h->rank ? static_cast<int>(round_up(h->rank, 64)) : 0;
  int dev = 0;
  cudaGetDevice(&dev);
  h->device = dev;
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const size_t dh = cfg->head_dim, d = cfg->hidden, qd = cfg->n_q_heads * dh, kvd = cfg->n_kv_heads * dh;
  h->rope_len = cfg->max_prefix + cfg->max_img_tokens;
  bool ok = cudaMalloc(&h->wo16, d * qd * 2) == cudaSuccess && cudaMalloc(&h->gamma, 2 * dh * 4) == cudaSuccess &&
            cudaMalloc(&h->rope, static_cast<size_t>(h->rope_len) * 64 * sizeof(float2)) == cudaSuccess &&
            cudaMalloc(&h->status, sizeof(int)) == cudaSuccess;
  ok = ok && cudaMalloc(&h->split_cnt, 3 * kSplitCounters * sizeof(int)) == cudaSuccess &&
       cudaMemset(h->split_cnt, 0, 3 * kSplitCounters * sizeof(int)) == cudaSuccess;
  if (ok && cfg->lora_rank > 0) {
    // the forward LoRA-down GEMMs' split-K partials: up to 4 splits of the
    // 128-row tiles of the largest call, 192 (or 128) f32 columns each
    const size_t tiles = (static_cast<size_t>(cfg->max_batch) * cfg->max_img_tokens + kBM - 1) / kBM;
    h->fsplit_bytes = std::min(kSplitWsBytes * 2, tiles * 4 * 192 * kBM * 4);
    ok = cudaMalloc(&h->fsplit, h->fsplit_bytes) == cudaSuccess;
  }
  if (ok && cfg->enable_backward)
    ok = cudaMalloc(&h->wqkvT16, (qd + 2 * kvd) * d * 2) == cudaSuccess &&
         cudaMalloc(&h->woT, qd * d * 2) == cudaSuccess &&
         cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    release(h);
    return MOT_ERR_CUDA;
  }
  // RoPE table: angle p * theta^(-2j/dh) in double, stored as f32 (cos, sin)
  std::vector<float2> tab(static_cast<size_t>(h->rope_len) * 64);
  for (int p = 0; p < h->rope_len; ++p)
    for (int j = 0; j < 64; ++j) {
      const double ang = static_cast<double>(p) * std::pow(cfg->rope_theta, -2.0 * j / 128.0);
      tab[static_cast<size_t>(p) * 64 + j] = make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
    }
  ok = cudaMemcpyAsync(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice, s) == cudaSuccess &&
       cudaMemsetAsync(h->status, 0, sizeof(int), s) == cudaSuccess;
  bf16_to_f32_kernel<<<1, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(wts->q_norm), h->gamma, 128);
  bf16_to_f32_kernel<<<1, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(wts->k_norm), h->gamma + 128, 128);
  ok = ok && cudaGetLastError() == cudaSuccess && refresh_f16_copies(h, s) == cudaSuccess &&
       cudaStreamSynchronize(s) == cudaSuccess;
  if (ok) ok = build_weight_maps(h) == MOT_OK;
  if (ok) attn_cluster_caps(h->attn_cap, h->num_sms);
  if (!ok) {
    release(h);
    return MOT_ERR_CUDA;
  }
  *out = h;
  return MOT_OK;
}

void mot_attn_destroy(mot_attn_t h) { release(h); }

int32_t mot_attn_last_launch_count(mot_attn_t h) { return h ? h->last_launches : 0; }

mot_status mot_attn_get_device_status(mot_attn_t h, void* stream) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return MOT_ERR_CUDA;
  if (v & DEV_ERR_TIMEOUT) {
    // a GEMM that gave up may have left split-K arrival counters behind:
    // zero them so that later calls on this handle start clean
    if (h->side && cudaStreamSynchronize(h->side) != cudaSuccess) return MOT_ERR_CUDA;
    if (h->split_cnt && cudaMemset(h->split_cnt, 0, 3 * kSplitCounters * sizeof(int)) != cudaSuccess)
      return MOT_ERR_CUDA;
    return MOT_ERR_TIMEOUT;
  }
  if (v & DEV_ERR_NUMERIC) return MOT_ERR_NUMERIC;
  return MOT_OK;
}

}  // extern "C"

namespace {

// The prefix tower's call (mot_attn_prefix_forward): the call's N tokens are
// the prompt itself, at positions 0..N-1, attending causally to each other
// (lengths[b] real tokens in branch b); the layer's cache entry (normalised,
// rotated keys and values) is written as bf16 [B, Hkv, N, dh].
struct PrefixCall {
  const int32_t* lengths;
  void* k_out;
  void* v_out;
};

// residual: the layer output is added into y_f32 (a residual stream the
// caller keeps in f32; y may then be NULL) instead of overwriting y / y_f32
mot_status forward_impl(mot_attn_t h, const void* x, int32_t B, int32_t N, const void* k_cache, const void* v_cache,
                        const int32_t* prefix_len, int32_t P, void* y, float* y_f32, void* saved, size_t saved_bytes,
                        void* workspace, size_t workspace_bytes, void* stream, const PrefixCall* pc,
                        bool residual = false) {
  if (!h || !x || !prefix_len || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  if (residual ? !y_f32 : !y) return MOT_ERR_INVALID_ARGUMENT;
  const mot_attn_config& c = h->cfg;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (B > c.max_batch || N > c.max_img_tokens || P > c.max_prefix) return MOT_ERR_UNSUPPORTED_SHAPE;
  if (P > 0 && (!k_cache || !v_cache)) return MOT_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < B; ++b) {
    if (prefix_len[b] < 0 || prefix_len[b] > P) return MOT_ERR_INVALID_ARGUMENT;
    // a forced split-KV count needs at least one key tile per split in every branch
    if (!pc && h->attn_splits_forced > (prefix_len[b] + N + 127) / 128) return MOT_ERR_UNSUPPORTED_SHAPE;
  }
  const void* ptrs[] = {x, y, y_f32, saved, workspace, k_cache, v_cache};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  const bool train = saved != nullptr;
  const Layout L = make_layout(c, B, N, P, train);
  if (train && saved_bytes < L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (workspace_bytes < L.fwd_scratch + (train ? 0 : L.act_bytes)) return MOT_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* act = train ? static_cast<uint8_t*>(saved) : ws + L.fwd_scratch;
  __half* q_hat = reinterpret_cast<__half*>(act + L.o_q);
  __half* k_all = reinterpret_cast<__half*>(act + L.o_k);
  __half* v_all = reinterpret_cast<__half*>(act + L.o_v);
  __half* attn = reinterpret_cast<__half*>(act + L.o_attn);
  float* lse = train ? reinterpret_cast<float*>(act + L.o_lse) : nullptr;
  __half* xhat = train ? reinterpret_cast<__half*>(act + L.o_xhat) : nullptr;
  float* rstd = train ? reinterpret_cast<float*>(act + L.o_rstd) : nullptr;
  __half* u_qkv = reinterpret_cast<__half*>(act + L.o_uqkv);
  __half* u_o = reinterpret_cast<__half*>(act + L.o_uo);
  __nv_bfloat16* u_ohi = train ? reinterpret_cast<__nv_bfloat16*>(act + L.o_uohi) : nullptr;
  __nv_bfloat16* u_olo = train ? reinterpret_cast<__nv_bfloat16*>(act + L.o_uolo) : nullptr;
  __half* ao16 = reinterpret_cast<__half*>(ws + L.w_ao16);
  __half* bo16 = reinterpret_cast<__half*>(ws + L.w_bo16);
  __half* bqkv16 = reinterpret_cast<__half*>(ws + L.w_bqkv16);

  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.hidden, M = L.M, r = h->rank, RP = h->RP;
  const int qd = Hq * 128, kvd = Hkv * 128, nqkv = qd + 2 * kvd;
  Launches lz(h, st);

  // 1. one launch: the f16 copies of A_o and of every lora_up (they meet f16
  //    operands; per call, since a trainer updates them in place between
  //    calls) and the key/value buffers' prefix rows (cache -> f16) and zero
  //    tail rows
  const int outj[3] = {qd, kvd, kvd};
  lz.stage = ST_BUILD_KV;
  {
    CvtJobs jobs{};
    if (r > 0) {
      const void* src[5] = {h->w.a_o, h->w.b_o, h->w.b_q, h->w.b_k, h->w.b_v};
      __half* dst[5] = {ao16, bo16, bqkv16, bqkv16 + static_cast<long long>(qd) * r,
                        bqkv16 + static_cast<long long>(qd + kvd) * r};
      const long long n[5] = {static_cast<long long>(r) * qd, static_cast<long long>(d) * r,
                              static_cast<long long>(qd) * r, static_cast<long long>(kvd) * r,
                              static_cast<long long>(kvd) * r};
      for (int i = 0; i < 5; ++i) {
        jobs.src[i] = static_cast<const __nv_bfloat16*>(src[i]);
        jobs.dst[i] = dst[i];
        jobs.n8[i] = n[i] / 8;
      }
      jobs.count = 5;
    }
    PlenArray pl{};
    for (int b = 0; b < B; ++b) pl.v[b] = prefix_len[b];
    // rows [0, plen) and [plen + N, Lcap) of every (branch, KV head), 16 chunks each
    const long long chunks = static_cast<long long>(B) * Hkv * (L.Lcap - N) * 16;
    const long long want = std::max<long long>((chunks + 255) / 256, r > 0 ? 2LL * h->num_sms : 1LL);
    const int grid = static_cast<int>(std::min<long long>(want, 16LL * h->num_sms));
    lz.done(launch_pdl(build_kv_kernel, dim3(grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(k_cache),
                       static_cast<const __nv_bfloat16*>(v_cache), k_all, v_all, Hkv, std::max(P, 1), N, L.Lcap,
                       chunks, pl, jobs, h->status));
  }
  // 3. LoRA down for q/k/v: u_qkv[:, j*RP:(j+1)*RP] = s x A_j^T (f16)
  lz.stage = ST_LORA_DOWN_QKV;
  if (r > 0) {
    GemmCore core;
    const int BN = RP == 64 ? 192 : 128;
    core_init(core, M, 3 * RP, BN, RP, h->status);
    if (!map2d(&core.maps[0], x, true, d, M, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->aq;
    core.maps[3] = h->ak;
    core.maps[4] = h->av;
    core.num_regions = 3;
    for (int j = 0; j <= 3; ++j) core.region_n0[j] = j * RP;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(128, BN, true, true), false, false);
    for (int j = 0; j < 3; ++j) core.segs[0].b_map[j] = 2 + j;
    core.num_segs = 1;
    EpiStore::Params ep = store_params(M, 3 * RP);
    set_out16(ep, 0, u_qkv, 3 * RP, false, h->scale);
    ep.check_f16 = 1;
    enable_split(core, h->fsplit, h->split_cnt + 2 * kSplitCounters, h->fsplit_bytes);
    if (BN == 192)
      lz.done(launch_gemm<192, 5, EpiStore>(core, ep, h->num_sms, st));
    else
      lz.done(launch_gemm<128, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  // 4. QKV projection (+ LoRA up) with RMSNorm + RoPE epilogue
  lz.stage = ST_QKV_GEMM;
  {
    GemmCore core;
    core_init(core, M, nqkv, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], x, true, d, M, d, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], u_qkv, false, 3 * RP, M, 3 * RP, 128) &&
           lora_up16_maps(&core.maps[5], bqkv16, r, outj);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wq;
    core.maps[3] = h->wk;
    core.maps[4] = h->wv;
    core.num_regions = 3;
    core.region_n0[0] = 0;
    core.region_n0[1] = qd;
    core.region_n0[2] = qd + kvd;
    core.region_n0[3] = nqkv;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(256, 256, true, true), false, false);
    for (int j = 0; j < 3; ++j) core.segs[0].b_map[j] = 2 + j;
    core.num_segs = 1;
    if (r > 0) {
      core.segs[1] = seg1(1, 0, 5, RP / 64, idesc_f16(256, 256, false, false), false, false);
      for (int j = 0; j < 3; ++j) {
        core.segs[1].a_k0[j] = j * RP;
        core.segs[1].b_map[j] = 5 + j;
      }
      core.num_segs = 2;
    }
    EpiQkv::Params ep{};
    ep.q_out = q_hat;
    ep.k_out = k_all;
    ep.v_out = v_all;
    ep.xhat = xhat;
    ep.rstd = rstd;
    ep.gamma_q = h->gamma;
    ep.gamma_k = h->gamma + 128;
    ep.rope = h->rope;
    for (int b = 0; b < B; ++b) ep.plen[b] = prefix_len[b];
    ep.N = N;
    ep.Hq = Hq;
    ep.Hkv = Hkv;
    ep.Lcap = L.Lcap;
    ep.M = M;
    ep.eps = c.rms_eps;
    if (pc) {
      ep.kc_out = static_cast<__nv_bfloat16*>(pc->k_out);
      ep.vc_out = static_cast<__nv_bfloat16*>(pc->v_out);
      ep.Pc = N;
    }
    lz.done(launch_gemm2<256, 6, EpiQkv>(core, ep, h->num_sms, st));
  }
  // 5. attention
  lz.stage = ST_ATTN_FWD;
  {
    AttnFwdParams ap{};
    if (!map3d(&ap.q_map, q_hat, 128, N, static_cast<uint64_t>(B) * Hq) ||
        !map3d(&ap.k_map, k_all, 128, L.Lcap, static_cast<uint64_t>(B) * Hkv) ||
        !map3d(&ap.v_map, v_all, 128, L.Lcap, static_cast<uint64_t>(B) * Hkv))
      return MOT_ERR_CUDA;
    ap.B = B;
    ap.N = N;
    ap.Hq = Hq;
    ap.Hkv = Hkv;
    ap.Lcap = L.Lcap;
    ap.q_pairs = (N + 255) / 256;
    int t_min = 1 << 30, t_max = 0;
    for (int b = 0; b < B; ++b) {
      ap.plen[b] = pc ? pc->lengths[b] : prefix_len[b];
      const int T = (prefix_len[b] + N + 127) / 128;
      t_min = std::min(t_min, T);
      t_max = std::max(t_max, T);
    }
    ap.causal = pc ? 1 : 0;
    const int units = B * Hq * ap.q_pairs;
    // causal units have unequal key ranges: they run unsplit
    const AttnPlan plan = pc ? AttnPlan{units, 1}
                          : h->attn_splits_forced > 0 ? AttnPlan{0, h->attn_splits_forced}
                                                      : plan_attention(h->attn_cap, units, t_min, t_max);
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
    ap.out = attn;
    ap.lse = lse;
    ap.status = h->status;
    h->last_attn_splits = plan.full_units < units ? plan.splits : 1;
    h->last_attn_full_units = plan.full_units;
    if (plan.full_units > 0) {
      ap.splits = 1;
      ap.unit0 = 0;
      lz.done(launch_pdl_cluster(attn_fwd_kernel, dim3(plan.full_units), dim3(kAttnThreads), AttnSmem::kBytes, st,
                                 1, ap));
    }
    if (plan.full_units < units) {
      ap.splits = plan.splits;
      ap.unit0 = plan.full_units;
      lz.done(launch_pdl_cluster(attn_fwd_kernel, dim3((units - plan.full_units) * plan.splits), dim3(kAttnThreads),
                                 AttnSmem::kBytes, st, plan.splits, ap));
    }
  }
  // 6. LoRA down for o: u_o = s o A_o^T (f16; training also keeps it as a bf16 hi + lo pair)
  lz.stage = ST_LORA_DOWN_O;
  if (r > 0) {
    GemmCore core;
    core_init(core, M, RP, RP, RP, h->status);
    if (!map2d(&core.maps[0], attn, false, qd, M, qd, 128) || !map2d(&core.maps[2], ao16, false, qd, r, qd, RP))
      return MOT_ERR_CUDA;
    core.segs[0] = seg1(0, 0, 2, qd / 64, idesc_f16(128, RP, false, false), false, false);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(M, RP);
    set_out16(ep, 0, u_o, RP, false, h->scale);
    if (train) {
      set_out16(ep, 1, u_ohi, RP, true, h->scale);
      set_out16(ep, 2, u_olo, RP, true, 1.0f, 1);
    }
    ep.check_f16 = 1;
    enable_split(core, h->fsplit, h->split_cnt + 2 * kSplitCounters, h->fsplit_bytes);
    lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
  }
  // 7. O projection (+ LoRA up): y bf16 and optional f32
  lz.stage = ST_O_GEMM;
  {
    GemmCore core;
    core_init(core, M, d, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], attn, false, qd, M, qd, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], u_o, false, RP, M, RP, 128) && map2d(&core.maps[3], bo16, false, r, d, r, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wo;
    core.segs[0] = seg1(0, 0, 2, qd / 64, idesc_f16(256, 256, false, false), false, false);
    core.num_segs = 1;
    if (r > 0) {
      core.segs[1] = seg1(1, 0, 3, RP / 64, idesc_f16(256, 256, false, false), false, false);
      core.num_segs = 2;
    }
    EpiStore::Params ep = store_params(M, d);
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

mot_status mot_attn_forward(mot_attn_t h, const void* x, int32_t B, int32_t N, const void* k_cache,
                            const void* v_cache, const int32_t* prefix_len, int32_t P, void* y, float* y_f32,
                            void* saved, size_t saved_bytes, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return forward_impl(h, x, B, N, k_cache, v_cache, prefix_len, P, y, y_f32, saved, saved_bytes, workspace,
                      workspace_bytes, stream, nullptr);
}

mot_status mot_attn_prefix_forward(mot_attn_t h, const void* x, int32_t B, int32_t N, const int32_t* lengths,
                                   void* y, float* y_f32, void* k_cache_out, void* v_cache_out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!h || !lengths || !k_cache_out || !v_cache_out) return MOT_ERR_INVALID_ARGUMENT;
  if (B <= 0 || B > kMaxBatch || N <= 0) return MOT_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < B; ++b)
    if (lengths[b] < 1 || lengths[b] > N) return MOT_ERR_INVALID_ARGUMENT;
  if (!aligned16(k_cache_out) || !aligned16(v_cache_out)) return MOT_ERR_ALIGNMENT;
  int32_t zeros[kMaxBatch] = {};
  const PrefixCall pc{lengths, k_cache_out, v_cache_out};
  return forward_impl(h, x, B, N, nullptr, nullptr, zeros, 0, y, y_f32, nullptr, 0, workspace, workspace_bytes,
                      stream, &pc);
}

mot_status mot_attn_backward(mot_attn_t h, const void* dy, const void* x, int32_t B, int32_t N, const void* k_cache,
                             const void* v_cache, const int32_t* prefix_len, int32_t P, const void* saved,
                             size_t saved_bytes, void* dx, float* dx_f32, float* const d_a[4], float* const d_b[4],
                             int32_t accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  (void)k_cache;
  (void)v_cache;  // the forward left the f16 key/value buffers in `saved`
  if (!h || !dy || !x || !dx || !prefix_len || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  if (!saved) return MOT_ERR_NO_SAVED_STATE;
  const mot_attn_config& c = h->cfg;
  if (!c.enable_backward) return MOT_ERR_INVALID_ARGUMENT;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (B > c.max_batch || N > c.max_img_tokens || P > c.max_prefix) return MOT_ERR_UNSUPPORTED_SHAPE;
  for (int b = 0; b < B; ++b)
    if (prefix_len[b] < 0 || prefix_len[b] > P) return MOT_ERR_INVALID_ARGUMENT;
  const int r = h->rank;
  if (r > 0) {
    if (!d_a || !d_b) return MOT_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < 4; ++i)
      if (!d_a[i] || !d_b[i] || !aligned16(d_a[i]) || !aligned16(d_b[i])) return d_a[i] && d_b[i] ? MOT_ERR_ALIGNMENT : MOT_ERR_INVALID_ARGUMENT;
  }
  const void* ptrs[] = {dy, x, dx, dx_f32, saved, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  const Layout L = make_layout(c, B, N, P, true);
  if (saved_bytes < L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (workspace_bytes < L.bwd_scratch) return MOT_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* act = static_cast<const uint8_t*>(saved);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const __half* q_hat = reinterpret_cast<const __half*>(act + L.o_q);
  const __half* k_all = reinterpret_cast<const __half*>(act + L.o_k);
  const __half* v_all = reinterpret_cast<const __half*>(act + L.o_v);
  const __half* attn = reinterpret_cast<const __half*>(act + L.o_attn);
  const float* lse = reinterpret_cast<const float*>(act + L.o_lse);
  const __half* xhat = reinterpret_cast<const __half*>(act + L.o_xhat);
  const float* rstd = reinterpret_cast<const float*>(act + L.o_rstd);
  const __half* u_qkv = reinterpret_cast<const __half*>(act + L.o_uqkv);          // s x A_j^T
  const __nv_bfloat16* u_ohi = reinterpret_cast<const __nv_bfloat16*>(act + L.o_uohi);  // s o A_o^T, hi + lo
  const __nv_bfloat16* u_olo = reinterpret_cast<const __nv_bfloat16*>(act + L.o_uolo);
  __half* dO = reinterpret_cast<__half*>(ws + L.b_do);
  float* delta = reinterpret_cast<float*>(ws + L.b_delta);
  __half* dqkv = reinterpret_cast<__half*>(ws + L.b_dqkv);
  // s g as bf16 hi + lo pairs (they meet bf16 x and lora_down), s g_o also in f16
  __nv_bfloat16* g_ohi = reinterpret_cast<__nv_bfloat16*>(ws + L.b_gohi);
  __nv_bfloat16* g_olo = reinterpret_cast<__nv_bfloat16*>(ws + L.b_golo);
  __half* g_o16 = reinterpret_cast<__half*>(ws + L.b_go16);
  __nv_bfloat16* g_hi = reinterpret_cast<__nv_bfloat16*>(ws + L.b_ghi);
  __nv_bfloat16* g_lo = reinterpret_cast<__nv_bfloat16*>(ws + L.b_glo);
  __half* b16 = reinterpret_cast<__half*>(ws + L.b_bqkv16);  // B_q|B_k|B_v in f16
  // split-K partials and counters: one set for the caller's stream, one for the side stream
  void* split_ws = ws + L.b_split;
  void* split_ws_side = ws + L.b_split + kSplitWsBytes;
  int* split_cnt_side = h->split_cnt + kSplitCounters;

  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.hidden, M = L.M, RP = h->RP;
  const int qd = Hq * 128, kvd = Hkv * 128, nqkv = qd + 2 * kvd;
  const int kb_tok = (M + 63) / 64;  // K blocks over tokens (zero-filled tail)
  const int col0[3] = {0, qd, qd + kvd}, outj[3] = {qd, kvd, kvd};
  Launches lz(h, st);

  if (r > 0) {
    // B_q, B_k, B_v to f16 (they meet the f16 pre-norm gradients)
    lz.stage = ST_BWD_CVT;
    CvtJobs jobs{};
    const void* src[3] = {h->w.b_q, h->w.b_k, h->w.b_v};
    for (int j = 0; j < 3; ++j) {
      jobs.src[j] = static_cast<const __nv_bfloat16*>(src[j]);
      jobs.dst[j] = b16 + static_cast<long long>(col0[j]) * r;
      jobs.n8[j] = static_cast<long long>(outj[j]) * r / 8;
    }
    jobs.count = 3;
    lz.done(launch_pdl(cvt_multi_kernel, dim3(64), dim3(256), 0, st, jobs, h->status));
    // g_o = dy B_o  -> s g_o as bf16 hi + lo, and as f16
    lz.stage = ST_BWD_G_O;
    GemmCore core;
    core_init(core, M, RP, RP, RP, h->status);
    if (!map2d(&core.maps[0], dy, true, d, M, d, 128)) return MOT_ERR_CUDA;
    core.maps[2] = h->bo_mn;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(128, RP, true, true, false, true), false, true);
    core.num_segs = 1;
    EpiStore::Params ep = store_params(M, RP);
    set_out16(ep, 0, g_ohi, RP, true, h->scale);
    set_out16(ep, 1, g_olo, RP, true, 1.0f, 0);
    set_out16(ep, 2, g_o16, RP, false, h->scale);
    ep.check_f16 = 1;
    enable_split(core, split_ws, h->split_cnt);
    lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
  }
  // dO = dy W_o + s g_o A_o (f16) and D = rowsum(dO o)
  lz.stage = ST_BWD_DO;
  {
    GemmCore core;
    core_init(core, M, qd, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], dy, true, d, M, d, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], g_ohi, true, RP, M, RP, 128) && map2d(&core.maps[4], g_olo, true, RP, M, RP, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->woT_k;
    core.segs[0] = seg1(0, 0, 2, d / 64, idesc_f16(256, 256, true, true), false, false);
    core.num_segs = 1;
    if (r > 0) {
      core.maps[3] = h->ao_mn;
      core.segs[1] = seg1(1, 0, 3, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      core.segs[2] = seg1(4, 0, 3, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      core.num_segs = 3;
    }
    EpiDattn::Params ep{dO, attn, delta, M, N, Hq};
    lz.done(launch_gemm2<256, 6, EpiDattn>(core, ep, h->num_sms, st));
  }
  if (r > 0) {
    // dB_o and dA_o feed nothing later in this call: side stream
    lz.fork();
    // dB_o = dy^T u_o   [d, r], with u_o as its bf16 hi + lo pair
    lz.stage = ST_BWD_DB_O;
    {
      GemmCore core;
      core_init(core, d, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], dy, true, d, M, d) || !map2d_mn(&core.maps[2], u_ohi, true, RP, M, RP) ||
          !map2d_mn(&core.maps[3], u_olo, true, RP, M, RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, true, true, true, true), true, true);
      set_dual(core.segs[0], 3);
      core.num_segs = 1;
      EpiStore::Params ep = store_params(d, r);
      ep.out32 = d_b[3];
      ep.ld32 = r;
      ep.accumulate32 = accumulate;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_dual<EpiStore>(RP, core, ep, h->num_sms, lz.cur));
    }
    // dA_o = (s g_o)^T o   [r, qd], computed as its transpose o^T (s g_o)
    lz.stage = ST_BWD_DA_O;
    {
      GemmCore core;
      core_init(core, qd, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], attn, false, qd, M, qd) || !map2d_mn(&core.maps[2], g_o16, false, RP, M, RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, false, false, true, true), true, true);
      core.num_segs = 1;
      EpiStore::Params ep = store_params(qd, r);
      ep.out32 = d_a[3];
      ep.ld32 = qd;
      ep.accumulate32 = accumulate;
      ep.transpose32 = 1;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, lz.cur));
    }
  }
  lz.to_main();
  // attention backward: dq^ over all keys, dk^, dv over the self keys
  {
    AttnBwdParams ap{};
    if (!map3d(&ap.q_map, q_hat, 128, N, static_cast<uint64_t>(B) * Hq) ||
        !map3d(&ap.k_map, k_all, 128, L.Lcap, static_cast<uint64_t>(B) * Hkv) ||
        !map3d(&ap.v_map, v_all, 128, L.Lcap, static_cast<uint64_t>(B) * Hkv) ||
        !map3d(&ap.do_map, dO, qd, N, B))
      return MOT_ERR_CUDA;
    ap.B = B;
    ap.N = N;
    ap.Hq = Hq;
    ap.Hkv = Hkv;
    ap.Lcap = L.Lcap;
    ap.q_tiles = (N + 127) / 128;
    ap.kv_tiles = (N + 127) / 128;
    ap.dkv_ctas = B * Hkv * ap.kv_tiles;
    for (int b = 0; b < B; ++b) ap.plen[b] = prefix_len[b];
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
    ap.inv_sqrt_dh = static_cast<float>(1.0 / std::sqrt(128.0));
    ap.lse = lse;
    ap.delta = delta;
    ap.xhat = xhat;
    ap.rstd = rstd;
    ap.gamma_q = h->gamma;
    ap.gamma_k = h->gamma + 128;
    ap.rope = h->rope;
    ap.dqkv = dqkv;
    ap.qhat = q_hat;
    ap.dout = dO;
    ap.status = h->status;
    static std::once_flag once;
    std::call_once(once, [] { set_smem_attr(attn_bwd_kernel, AttnBwdSmem::kBytes); });
    lz.stage = ST_BWD_ATTN;
    lz.done(launch_pdl(attn_bwd_kernel, dim3(ap.dkv_ctas + B * Hq * ap.q_tiles), dim3(kAttnBwdThreads),
                       AttnBwdSmem::kBytes, st, ap));
  }
  if (r > 0) {
    {
      // g_j = d{q,k,v}_pre B_j for the three projections in one GEMM: column
      // block j reads its own K range of d{q,k,v}_pre (B_k, B_v are zero past
      // their rows) -> s g_j as bf16 hi + lo in columns [j*RP, (j+1)*RP)
      lz.stage = ST_BWD_G_QKV;
      GemmCore core;
      core_init(core, M, 3 * RP, RP, RP, h->status);
      if (!map2d(&core.maps[0], dqkv, false, nqkv, M, nqkv, 128)) return MOT_ERR_CUDA;
      for (int j = 0; j < 3; ++j)
        if (!map2d_mn(&core.maps[2 + j], b16 + static_cast<long long>(col0[j]) * r, false, r, outj[j], r))
          return MOT_ERR_CUDA;
      core.num_regions = 3;
      for (int j = 0; j <= 3; ++j) core.region_n0[j] = j * RP;
      core.segs[0] = seg1(0, 0, 2, qd / 64, idesc_f16(128, RP, false, false, false, true), false, true);
      for (int j = 0; j < 3; ++j) {
        core.segs[0].a_k0[j] = col0[j];
        core.segs[0].b_map[j] = 2 + j;
        core.segs[0].kb_r[j] = outj[j] / 64;  // each block reads only its own K columns
      }
      core.num_segs = 1;
      EpiStore::Params ep = store_params(M, 3 * RP);
      set_out16(ep, 0, g_hi, 3 * RP, true, h->scale);
      set_out16(ep, 1, g_lo, 3 * RP, true, 1.0f, 0);
      enable_split(core, split_ws, h->split_cnt);
      lz.done(launch_gemm_narrow<EpiStore>(RP, core, ep, h->num_sms, st));
    }
    // dB_j and dA_j feed nothing later in this call: side stream
    lz.fork();
    {
      // dB_j = d{q,k,v}_pre^T u_j   [out_j, r] for the three projections in
      // one GEMM: D rows are the nqkv columns of d{q,k,v}_pre, and row block j
      // (a whole number of 128-row tiles) meets u_j
      lz.stage = ST_BWD_DB_QKV;
      GemmCore core;
      core_init(core, nqkv, RP, RP, RP, h->status);
      if (!map2d_mn(&core.maps[0], dqkv, false, nqkv, M, nqkv)) return MOT_ERR_CUDA;
      for (int j = 0; j < 3; ++j)
        if (!map2d_mn(&core.maps[2 + j], u_qkv + j * RP, false, RP, M, 3 * RP)) return MOT_ERR_CUDA;
      core.regions_on_m = 1;
      core.num_regions = 3;
      for (int j = 0; j < 3; ++j) core.region_n0[j] = col0[j];
      core.region_n0[3] = nqkv;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, RP, false, false, true, true), true, true);
      for (int j = 0; j < 3; ++j) core.segs[0].b_map[j] = 2 + j;
      core.num_segs = 1;
      EpiRowBlocks::Params ep{};
      for (int j = 0; j < 3; ++j) {
        ep.out[j] = d_b[j];
        ep.row0[j] = col0[j];
      }
      ep.row0[3] = nqkv;
      ep.ld = r;
      ep.cols = r;
      ep.accumulate = accumulate;
      enable_split(core, split_ws_side, split_cnt_side);
      lz.done(launch_gemm_narrow<EpiRowBlocks>(RP, core, ep, h->num_sms, lz.cur));
    }
    {
      // dA_j = (s g_j)^T x for the three projections in one GEMM over x^T,
      // with (s g_j) as its bf16 hi + lo pair; block j goes to dA_j transposed
      lz.stage = ST_BWD_DA_QKV;
      GemmCore core;
      // one 3 RP-wide tile when it fits the MMA (x^T read once), else RP-wide
      const int bn = 3 * RP <= 256 ? 3 * RP : RP;
      core_init(core, d, 3 * RP, bn, RP, h->status);
      if (!map2d_mn(&core.maps[0], x, true, d, M, d) || !map2d_mn(&core.maps[2], g_hi, true, 3 * RP, M, 3 * RP) ||
          !map2d_mn(&core.maps[3], g_lo, true, 3 * RP, M, 3 * RP))
        return MOT_ERR_CUDA;
      core.segs[0] = seg1(0, 0, 2, kb_tok, idesc_f16(128, bn, true, true, true, true), true, true);
      set_dual(core.segs[0], 3);
      core.num_segs = 1;
      EpiLoraGrad::Params ep{};
      for (int j = 0; j < 3; ++j) ep.out[j] = d_a[j];
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
  // dx = dq W_q + dk W_k + dv W_v + sum_j ((s g_j)_hi + (s g_j)_lo) A_j
  lz.stage = ST_BWD_DX;
  {
    GemmCore core;
    core_init(core, M, d, 256, 128, h->status);
    core_pair(core);
    bool ok = map2d(&core.maps[0], dqkv, false, nqkv, M, nqkv, 128);
    if (r > 0)
      ok = ok && map2d(&core.maps[1], g_hi, true, 3 * RP, M, 3 * RP, 128) &&
           map2d(&core.maps[8], g_lo, true, 3 * RP, M, 3 * RP, 128);
    if (!ok) return MOT_ERR_CUDA;
    core.maps[2] = h->wqkvT_k;
    for (int j = 0; j < 3; ++j) {
      core.segs[j] = seg1(0, col0[j], 2, outj[j] / 64, idesc_f16(256, 256, false, false), false, false);
      core.segs[j].b_k0 = col0[j];
    }
    core.num_segs = 3;
    if (r > 0) {
      core.maps[5] = h->aq_mn;
      core.maps[6] = h->ak_mn;
      core.maps[7] = h->av_mn;
      for (int j = 0; j < 3; ++j) {
        core.segs[3 + j] = seg1(1, j * RP, 5 + j, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
        core.segs[6 + j] = seg1(8, j * RP, 5 + j, RP / 64, idesc_f16(256, 256, true, true, false, true), false, true);
      }
      core.num_segs = 9;
    }
    EpiStore::Params ep = store_params(M, d);
    set_out16(ep, 0, dx, d, true);
    ep.out32 = dx_f32;
    ep.ld32 = d;
    lz.done(launch_gemm2<256, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  return lz.finish();
}

mot_status mot_attn_merge_lora(mot_attn_t h, void* w_q_out, void* w_k_out, void* w_v_out, void* w_o_out,
                               void* stream) {
  if (!h || !w_q_out || !w_k_out || !w_v_out || !w_o_out) return MOT_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {w_q_out, w_k_out, w_v_out, w_o_out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOT_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const mot_attn_config& c = h->cfg;
  const int d = c.hidden, qd = c.n_q_heads * 128, kvd = c.n_kv_heads * 128, r = h->rank;
  if (r > 0) {
    struct Job {
      const void *w, *a, *b;
      void* out;
      int rows, cols;
    } jobs[4] = {{h->w.w_q, h->w.a_q, h->w.b_q, w_q_out, qd, d},
                 {h->w.w_k, h->w.a_k, h->w.b_k, w_k_out, kvd, d},
                 {h->w.w_v, h->w.a_v, h->w.b_v, w_v_out, kvd, d},
                 {h->w.w_o, h->w.a_o, h->w.b_o, w_o_out, d, qd}};
    for (const Job& j : jobs) {
      dim3 grid((j.cols + 255) / 256, (j.rows + 7) / 8);
      merge_lora_kernel<<<grid, dim3(32, 8), 0, st>>>(
          static_cast<const __nv_bfloat16*>(j.w), static_cast<const __nv_bfloat16*>(j.a),
          static_cast<const __nv_bfloat16*>(j.b), static_cast<__nv_bfloat16*>(j.out), j.rows, j.cols, r, h->scale);
    }
  } else {
    const size_t sizes[4] = {static_cast<size_t>(qd) * d, static_cast<size_t>(kvd) * d,
                             static_cast<size_t>(kvd) * d, static_cast<size_t>(d) * qd};
    const void* src[4] = {h->w.w_q, h->w.w_k, h->w.w_v, h->w.w_o};
    void* dst[4] = {w_q_out, w_k_out, w_v_out, w_o_out};
    for (int i = 0; i < 4; ++i)
      if (src[i] != dst[i] && cudaMemcpyAsync(dst[i], src[i], sizes[i] * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MOT_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return MOT_ERR_CUDA;
  // rebind: merged base, no adapters; the f16 copies are rebuilt from the merged weights
  h->w.w_q = w_q_out;
  h->w.w_k = w_k_out;
  h->w.w_v = w_v_out;
  h->w.w_o = w_o_out;
  h->w.a_q = h->w.a_k = h->w.a_v = h->w.a_o = nullptr;
  h->w.b_q = h->w.b_k = h->w.b_v = h->w.b_o = nullptr;
  h->rank = 0;
  h->RP = 0;
  h->scale = 0.f;
  h->cfg.lora_rank = 0;
  if (refresh_f16_copies(h, st) != cudaSuccess) return MOT_ERR_CUDA;
  return build_weight_maps(h);
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation forward
// Scratch of mot_attn_forward_noalloc: one file-scope device array. In host
// code `g_noalloc_scratch` names a host-side stand-in, not device memory, so
// its device address is looked up with cudaGetSymbolAddress once per device
// (with that device current) and only that address is handed to kernels.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (resolved on the
// first call per device); nullptr on failure.
void* noalloc_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" mot_status mot_attn_forward_host(mot_attn_t h, int32_t steps, const void* const* x_host, int32_t B,
                                            int32_t N, const void* const* k_cache_host,
                                            const void* const* v_cache_host, const int32_t* prefix_len, int32_t P,
                                            void* const* y_host, void* staging, size_t staging_bytes,
                                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || steps <= 0 || !x_host || !y_host || !prefix_len || !staging || !workspace)
    return MOT_ERR_INVALID_ARGUMENT;
  const mot_attn_config& c = h->cfg;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (B > c.max_batch || N > c.max_img_tokens || P > c.max_prefix) return MOT_ERR_UNSUPPORTED_SHAPE;
  if (P > 0 && (!k_cache_host || !v_cache_host)) return MOT_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < steps; ++i) {
    if (!x_host[i] || !y_host[i]) return MOT_ERR_INVALID_ARGUMENT;
    if (P > 0 && (!k_cache_host[i] || !v_cache_host[i])) return MOT_ERR_INVALID_ARGUMENT;
  }
  for (int b = 0; b < B; ++b)
    if (prefix_len[b] < 0 || prefix_len[b] > P) return MOT_ERR_INVALID_ARGUMENT;
  if (!aligned16(staging) || !aligned16(workspace)) return MOT_ERR_ALIGNMENT;
  const HostStaging hs = host_staging(c, B, N, P);
  if (staging_bytes < 2 * hs.slot) return MOT_ERR_WORKSPACE_TOO_SMALL;
  const Layout L = make_layout(c, B, N, P, false);
  if (workspace_bytes < L.fwd_scratch + L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (!h->h2d) {
    bool ok = cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->hev_start, cudaEventDisableTiming) == cudaSuccess;
    for (int s = 0; s < 2 && ok; ++s)
      ok = cudaEventCreateWithFlags(&h->hev_in[s], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->hev_comp[s], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->hev_out[s], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return MOT_ERR_CUDA;  // what was made is released with the handle
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  auto note = [&err](cudaError_t e) {
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    return err == cudaSuccess;
  };
  // both copy streams start after the work already on the caller's stream
  note(cudaEventRecord(h->hev_start, st));
  note(cudaStreamWaitEvent(h->h2d, h->hev_start, 0));
  note(cudaStreamWaitEvent(h->d2h, h->hev_start, 0));
  const size_t xb = static_cast<size_t>(B) * N * c.hidden * 2;
  const size_t kvb = static_cast<size_t>(B) * c.n_kv_heads * P * c.head_dim * 2;
  uint8_t* base = static_cast<uint8_t*>(staging);
  mot_status status = MOT_OK;
  for (int i = 0; i < steps && err == cudaSuccess; ++i) {
    const int s = i & 1;
    uint8_t* slot = base + s * hs.slot;
    void* xd = slot;
    void* yd = slot + hs.x;
    void* kd = slot + 2 * hs.x;
    void* vd = slot + 2 * hs.x + hs.kv;
    // copy-in; the slot's inputs were last read by the layer of call i-2
    if (i >= 2) note(cudaStreamWaitEvent(h->h2d, h->hev_comp[s], 0));
    note(cudaMemcpyAsync(xd, x_host[i], xb, cudaMemcpyHostToDevice, h->h2d));
    if (P > 0) {
      note(cudaMemcpyAsync(kd, k_cache_host[i], kvb, cudaMemcpyHostToDevice, h->h2d));
      note(cudaMemcpyAsync(vd, v_cache_host[i], kvb, cudaMemcpyHostToDevice, h->h2d));
    }
    note(cudaEventRecord(h->hev_in[s], h->h2d));
    // the layer, once its inputs landed and call i-2's y has left the slot
    note(cudaStreamWaitEvent(st, h->hev_in[s], 0));
    if (i >= 2) note(cudaStreamWaitEvent(st, h->hev_out[s], 0));
    if (err != cudaSuccess) break;
    status = mot_attn_forward(h, xd, B, N, P > 0 ? kd : nullptr, P > 0 ? vd : nullptr, prefix_len, P, yd, nullptr,
                              nullptr, 0, workspace, workspace_bytes, stream);
    if (status != MOT_OK) break;
    note(cudaEventRecord(h->hev_comp[s], st));
    // copy-out
    note(cudaStreamWaitEvent(h->d2h, h->hev_comp[s], 0));
    note(cudaMemcpyAsync(y_host[i], yd, xb, cudaMemcpyDeviceToHost, h->d2h));
    note(cudaEventRecord(h->hev_out[s], h->d2h));
  }
  // on every path the caller's stream ends after all copies enqueued so far
  // (each copy stream runs in order, so its latest event covers the rest)
  cudaError_t e1 = cudaEventRecord(h->hev_out[0], h->d2h);
  cudaError_t e2 = cudaStreamWaitEvent(st, h->hev_out[0], 0);
  cudaError_t e3 = cudaEventRecord(h->hev_in[0], h->h2d);
  cudaError_t e4 = cudaStreamWaitEvent(st, h->hev_in[0], 0);
  note(e1);
  note(e2);
  note(e3);
  note(e4);
  if (status != MOT_OK) return status;
  return err == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

extern "C" mot_status mot_attn_forward_noalloc(mot_attn_t h, const void* x, int32_t B, int32_t N,
                                               const void* k_cache, const void* v_cache,
                                               const int32_t* prefix_len, int32_t P, void* y, float* y_f32,
                                               void* stream) {
  if (!h || !x || !y || !prefix_len) return MOT_ERR_INVALID_ARGUMENT;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  const mot_attn_config& c = h->cfg;
  if (B > c.max_batch || N > c.max_img_tokens || P > c.max_prefix) return MOT_ERR_UNSUPPORTED_SHAPE;
  // the scratch array is resolved for the current device: it must be the
  // handle's, where its weights and copies live
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return MOT_ERR_CUDA;
  if (cur != h->device) return MOT_ERR_INVALID_ARGUMENT;
  // what an inference forward of this shape needs (what mot_attn_forward checks)
  const Layout L = make_layout(c, B, N, P, false);
  if (L.fwd_scratch + L.act_bytes > kNoAllocScratchBytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return MOT_ERR_CUDA;
  return mot_attn_forward(h, x, B, N, k_cache, v_cache, prefix_len, P, y, y_f32, nullptr, 0, scratch,
                          kNoAllocScratchBytes, stream);
}

// ------------------------------------------------------------------ dev entry points
extern "C" {

mot_status mot_dev_gemm(const void* a, const void* b, float* dmat, int32_t m, int32_t n, int32_t k, int32_t is_bf16,
                        int32_t tile_n, void* stream) {
  if (!a || !b || !dmat || m <= 0 || n <= 0 || k <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (tile_n != 128 && tile_n != 256) return MOT_ERR_INVALID_ARGUMENT;
  if (k % 64 != 0 || n % tile_n != 0) return MOT_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(dmat)) return MOT_ERR_ALIGNMENT;
  GemmCore core;
  const bool bf = is_bf16 != 0;
  core_init(core, m, n, tile_n, tile_n, nullptr);
  if (!map2d(&core.maps[0], a, bf, k, m, k, 128) || !map2d(&core.maps[2], b, bf, k, n, k, tile_n)) return MOT_ERR_CUDA;
  core.segs[0] = seg1(0, 0, 2, k / 64, idesc_f16(128, tile_n, bf, bf), false, false);
  core.num_segs = 1;
  EpiStore::Params ep = store_params(m, n);
  ep.out32 = dmat;
  ep.ld32 = n;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const cudaError_t e = tile_n == 256 ? launch_gemm<256, 4, EpiStore>(core, ep, sms, static_cast<cudaStream_t>(stream))
                                      : launch_gemm<128, 6, EpiStore>(core, ep, sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

mot_status mot_dev_gemm_variant(const void* a, const void* b, const void* b2, float* dmat, int32_t m, int32_t n,
                                int32_t k, int32_t is_bf16, int32_t variant, void* stream) {
  if (!a || !b || !dmat || m <= 0 || n <= 0 || k <= 0 || variant < 1 || variant > 4) return MOT_ERR_INVALID_ARGUMENT;
  if (variant == 3 && !b2) return MOT_ERR_INVALID_ARGUMENT;
  if (k % 64 != 0 || ((variant == 1 || variant == 4) && n % 256 != 0) || ((variant == 2 || variant == 3) && n != 64))
    return MOT_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(dmat) || (b2 && !aligned16(b2))) return MOT_ERR_ALIGNMENT;
  const bool bf = is_bf16 != 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  GemmCore core;
  EpiStore::Params ep = store_params(m, n);
  ep.out32 = dmat;
  ep.ld32 = n;
  if (variant == 1 || variant == 4) {
    // variant 4: B given as [k, n] (MN-major operand, 64 x 64 boxes)
    const bool bmn = variant == 4;
    core_init(core, m, n, 256, 128, nullptr);
    core_pair(core);
    if (!map2d(&core.maps[0], a, bf, k, m, k, 128) ||
        !(bmn ? map2d_mn(&core.maps[2], b, bf, n, k, n) : map2d(&core.maps[2], b, bf, k, n, k, 128)))
      return MOT_ERR_CUDA;
    core.segs[0] = seg1(0, 0, 2, k / 64, idesc_f16(256, 256, bf, bf, false, bmn), false, bmn);
    core.num_segs = 1;
    return launch_gemm2<256, 6, EpiStore>(core, ep, sms, st) == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
  }
  // 64-wide tiles with split-K (variant 3: a second B operand on every A tile)
  core_init(core, m, n, 64, 64, nullptr);
  if (!map2d(&core.maps[0], a, bf, k, m, k, 128) || !map2d(&core.maps[2], b, bf, k, n, k, 64) ||
      (variant == 3 && !map2d(&core.maps[3], b2, bf, k, n, k, 64)))
    return MOT_ERR_CUDA;
  core.segs[0] = seg1(0, 0, 2, k / 64, idesc_f16(128, 64, bf, bf), false, false);
  if (variant == 3) set_dual(core.segs[0], 3);
  core.num_segs = 1;
  const int tiles = (m + kBM - 1) / kBM;
  if (tiles > kSplitCounters) return MOT_ERR_UNSUPPORTED_SHAPE;
  void* ws = nullptr;
  int* cnt = nullptr;
  if (cudaMalloc(&ws, kSplitWsBytes) != cudaSuccess) return MOT_ERR_CUDA;
  if (cudaMalloc(&cnt, kSplitCounters * sizeof(int)) != cudaSuccess || cudaMemsetAsync(cnt, 0, kSplitCounters * sizeof(int), st) != cudaSuccess) {
    cudaFree(ws);
    return MOT_ERR_CUDA;
  }
  enable_split(core, ws, cnt);
  const cudaError_t e = variant == 3 ? launch_gemm_dual<EpiStore>(64, core, ep, sms, st)
                                     : launch_gemm_narrow<EpiStore>(64, core, ep, sms, st);
  const cudaError_t e2 = cudaStreamSynchronize(st);
  cudaFree(ws);
  cudaFree(cnt);
  return (e == cudaSuccess && e2 == cudaSuccess) ? MOT_OK : MOT_ERR_CUDA;
}

mot_status mot_dev_exp2_poly(const float* x, float* y, int32_t n, void* stream) {
  if (!x || !y || n <= 0 || (n & 1)) return MOT_ERR_INVALID_ARGUMENT;
  exp2_poly_kernel<<<(n / 2 + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n / 2);
  return cudaGetLastError() == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

mot_status mot_dev_profile(mot_attn_t h, int32_t enable) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  if (enable && !h->ev[0])
    for (cudaEvent_t& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return MOT_ERR_CUDA;
  h->profile = enable != 0;
  h->stage_count = 0;
  return MOT_OK;
}

mot_status mot_dev_stage_times(mot_attn_t h, int32_t* ids, float* ms, int32_t max, int32_t* count) {
  if (!h || !ids || !ms || max < 0 || !count) return MOT_ERR_INVALID_ARGUMENT;
  if (!h->profile) return MOT_ERR_INVALID_ARGUMENT;
  *count = h->stage_count;
  if (h->stage_count == 0) return MOT_OK;
  for (int i = 0; i < h->stage_count && i < max; ++i) {
    ids[i] = h->stage_ids[i];
    if (!h->stage_start[i] || !h->stage_end[i]) return MOT_ERR_CUDA;
    if (cudaEventSynchronize(h->stage_end[i]) != cudaSuccess ||
        cudaEventElapsedTime(&ms[i], h->stage_start[i], h->stage_end[i]) != cudaSuccess)
      return MOT_ERR_CUDA;
  }
  return MOT_OK;
}

mot_status mot_dev_stage_timeline(mot_attn_t h, int32_t* ids, float* t0_ms, float* t1_ms, int32_t max,
                                  int32_t* count) {
  if (!h || !ids || !t0_ms || !t1_ms || max < 0 || !count) return MOT_ERR_INVALID_ARGUMENT;
  if (!h->profile) return MOT_ERR_INVALID_ARGUMENT;
  *count = h->stage_count;
  if (h->stage_count == 0) return MOT_OK;
  cudaEvent_t origin = h->stage_start[0];
  for (int i = 0; i < h->stage_count && i < max; ++i) {
    ids[i] = h->stage_ids[i];
    if (!origin || !h->stage_start[i] || !h->stage_end[i]) return MOT_ERR_CUDA;
    if (cudaEventSynchronize(h->stage_end[i]) != cudaSuccess ||
        cudaEventElapsedTime(&t0_ms[i], origin, h->stage_start[i]) != cudaSuccess ||
        cudaEventElapsedTime(&t1_ms[i], origin, h->stage_end[i]) != cudaSuccess)
      return MOT_ERR_CUDA;
  }
  return MOT_OK;
}

mot_status mot_dev_set_attn_splits(mot_attn_t h, int32_t splits) {
  if (!h || splits < 0 || splits > kMaxAttnSplits) return MOT_ERR_INVALID_ARGUMENT;
  if (splits > 1 && h->attn_cap[splits] <= 0) return MOT_ERR_UNSUPPORTED_SHAPE;
  h->attn_splits_forced = splits;
  return MOT_OK;
}

int32_t mot_dev_last_attn_splits(mot_attn_t h) { return h ? h->last_attn_splits : 0; }

int32_t mot_dev_last_attn_full_units(mot_attn_t h) { return h ? h->last_attn_full_units : 0; }

mot_status mot_dev_wait_probe(mot_attn_t h, void* stream) {
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->status);
  return cudaGetLastError() == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

const char* mot_dev_stage_name(int32_t id) {
  if (id >= 0 && id < static_cast<int32_t>(sizeof(kStageNames) / sizeof(kStageNames[0]))) return kStageNames[id];
  return "?";
}

mot_status mot_dev_saved_layout(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens, int32_t prefix_max,
                                size_t offsets[9], int32_t* lcap) {
  mot_status st = check_config(cfg);
  if (st != MOT_OK) return st;
  if (!offsets || batch <= 0 || img_tokens <= 0 || prefix_max < 0) return MOT_ERR_INVALID_ARGUMENT;
  const Layout L = make_layout(*cfg, batch, img_tokens, prefix_max, true);
  const size_t o[9] = {L.o_q, L.o_k, L.o_v, L.o_attn, L.o_lse, L.o_xhat, L.o_rstd, L.o_uqkv, L.o_uo};
  for (int i = 0; i < 9; ++i) offsets[i] = o[i];
  if (lcap) *lcap = L.Lcap;
  return MOT_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ the gen-tower MLP
#include "mot_mlp.cuh"

// ------------------------------------------------------------------ the denoise step
#include "mot_step.cuh"

// ------------------------------------------------------------------ the A3B mixture-of-experts MLP
#include "mot_moe.cuh"
