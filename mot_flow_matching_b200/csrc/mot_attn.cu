// mot_attn.cu -- C ABI of the gen-tower attention layer (see include/mot_attn.h).
//
// Forward launch sequence on the caller's stream (r = LoRA rank):
//   [r>0] bf16 -> f16 of lora_down/lora_up of o_proj (per call: they may change)
//   build_kv      prefix rows of the f16 key/value buffers, zero tail rows
//   [r>0] lora-down GEMM    u_qkv = s x [A_q; A_k; A_v]^T        (bf16)
//   QKV GEMM + epilogue     x W_qkv^T + u B^T -> RMSNorm -> RoPE -> q^, K, V
//   attention               o = softmax(q^ K^T / sqrt(dh)) V      (f16)
//   [r>0] lora-down GEMM    u_o = s o A_o^T                       (f16)
//   O GEMM                  y = o W_o^T + u_o B_o^T               (bf16 + f32)
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

// 2-D map over a row-major [outer, inner] 16-bit tensor with row stride
// `ld` elements; box = [box_outer rows, 64 columns], 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer, uint64_t ld,
           uint32_t box_outer) {
  if (!encode_ready() || inner == 0 || outer == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                  const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over a contiguous f16 [outer, mid, 128] tensor, box [1, 128, 64].
bool map3d_heads(CUtensorMap* m, const void* ptr, uint64_t mid, uint64_t outer) {
  if (!encode_ready() || mid == 0 || outer == 0) return false;
  cuuint64_t dims[3] = {128, mid, outer};
  cuuint64_t strides[2] = {256, mid * 256};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ layouts
struct Layout {
  int B = 0, N = 0, P = 0, M = 0, Lcap = 0, r = 0, RP = 0;
  size_t o_q = 0, o_k = 0, o_v = 0, o_attn = 0, o_lse = 0, o_xhat = 0, o_rstd = 0, o_uqkv = 0, o_uo = 0;
  size_t act_bytes = 0;    // activation region (in `saved`, else in the workspace)
  size_t w_ao16 = 0, w_bo16 = 0, scratch_bytes = 0;
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
  const size_t dh = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.hidden, M = L.M;
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
  L.o_uqkv = take(L.r ? M * 3 * L.RP * 2 : 0);
  L.o_uo = take(L.r ? M * L.RP * 2 : 0);
  L.act_bytes = off;
  off = 0;
  L.w_ao16 = take(L.r ? L.r * Hq * dh * 2 : 0);
  L.w_bo16 = take(L.r ? d * L.r * 2 : 0);
  L.scratch_bytes = off;
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

int g_grid_cap = 0;  // 0 = number of SMs

template <int BN, int STAGES, class Epi>
cudaError_t launch_gemm(const GemmCore& core, const typename Epi::Params& ep, int num_sms, cudaStream_t st) {
  static_assert(sizeof(GemmArgs<Epi>) <= 4096, "kernel parameter block");
  using L = GemmSmem<BN, STAGES>;
  static_assert(L::kBytes <= 232448, "shared memory");
  auto kern = gemm_kernel<BN, STAGES, Epi>;
  static std::once_flag once;
  std::call_once(once, [&] { set_smem_attr(kern, L::kBytes); });
  GemmArgs<Epi> args;
  args.core = core;
  args.epi = ep;
  const int tiles = core.tiles_m * core.tiles_n;
  const int cap = g_grid_cap > 0 ? g_grid_cap : num_sms;
  const int grid = std::max(1, std::min(tiles, cap));
  kern<<<grid, kGemmThreads, L::kBytes, st>>>(args);
  return cudaGetLastError();
}

void core_init(GemmCore& c, int M, int N, int BN, int kb_main, int kb_ext, int b_box_rows, uint32_t idesc_main,
               uint32_t idesc_ext, int* status) {
  std::memset(static_cast<void*>(&c), 0, sizeof(c));
  c.M = M;
  c.N = N;
  c.kb_main = kb_main;
  c.kb_ext = kb_ext;
  c.tiles_m = (M + kBM - 1) / kBM;
  c.tiles_n = (N + BN - 1) / BN;
  c.b_box_rows = b_box_rows;
  c.idesc_main = idesc_main;
  c.idesc_ext = idesc_ext;
  c.status = status;
}

}  // namespace

// ------------------------------------------------------------------ handle
constexpr int kMaxStages = 32;
enum StageId : int {
  ST_CVT_LORA_O = 0, ST_BUILD_KV = 1, ST_LORA_DOWN_QKV = 2, ST_QKV_GEMM = 3, ST_ATTN_FWD = 4,
  ST_LORA_DOWN_O = 5, ST_O_GEMM = 6,
};
const char* const kStageNames[] = {"cvt_lora_o", "build_kv", "lora_down_qkv", "qkv_gemm", "attn_fwd",
                                   "lora_down_o", "o_gemm"};

struct mot_attn {
  mot_attn_config cfg;
  mot_attn_weights w;
  int rank = 0;
  float scale = 0.f;
  int RP = 0;
  __half* wo16 = nullptr;
  float* gamma = nullptr;  // [2*dh]: q gain then k gain
  float2* rope = nullptr;
  int rope_len = 0;
  int* status = nullptr;
  int num_sms = 148;
  int last_launches = 0;
  // optional per-launch timing (mot_dev_profile)
  bool profile = false;
  cudaEvent_t ev[kMaxStages + 1] = {};
  int stage_ids[kMaxStages] = {};
  int stage_count = 0;
  CUtensorMap wq, wk, wv, wo;  // base weights, box rows 256
  CUtensorMap aq, ak, av;      // lora_down q/k/v, box rows RP
  CUtensorMap bq, bk, bv;      // lora_up q/k/v, box rows 256
};

namespace {

mot_status build_weight_maps(mot_attn* h) {
  const mot_attn_config& c = h->cfg;
  const uint64_t d = c.hidden, qd = c.n_q_heads * 128, kvd = c.n_kv_heads * 128;
  bool ok = map2d(&h->wq, h->w.w_q, true, d, qd, d, 256) && map2d(&h->wk, h->w.w_k, true, d, kvd, d, 256) &&
            map2d(&h->wv, h->w.w_v, true, d, kvd, d, 256) && map2d(&h->wo, h->wo16, false, qd, d, qd, 256);
  if (ok && h->rank > 0) {
    const uint64_t r = h->rank;
    const uint32_t box_a = static_cast<uint32_t>(h->RP);
    ok = map2d(&h->aq, h->w.a_q, true, d, r, d, box_a) && map2d(&h->ak, h->w.a_k, true, d, r, d, box_a) &&
         map2d(&h->av, h->w.a_v, true, d, r, d, box_a) && map2d(&h->bq, h->w.b_q, true, r, qd, r, 256) &&
         map2d(&h->bk, h->w.b_k, true, r, kvd, r, 256) && map2d(&h->bv, h->w.b_v, true, r, kvd, r, 256);
  }
  return ok ? MOT_OK : MOT_ERR_CUDA;
}

void release(mot_attn* h) {
  if (!h) return;
  for (cudaEvent_t e : h->ev)
    if (e) cudaEventDestroy(e);
  cudaFree(h->wo16);
  cudaFree(h->gamma);
  cudaFree(h->rope);
  cudaFree(h->status);
  delete h;
}

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

mot_status mot_attn_query_sizes(const mot_attn_config* cfg, int32_t batch, int32_t img_tokens, int32_t prefix_max,
                                size_t* workspace_bytes, size_t* saved_bytes) {
  mot_status st = check_config(cfg);
  if (st != MOT_OK) return st;
  if (batch <= 0 || img_tokens <= 0 || prefix_max < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (batch > cfg->max_batch || img_tokens > cfg->max_img_tokens || prefix_max > cfg->max_prefix)
    return MOT_ERR_UNSUPPORTED_SHAPE;
  const Layout inf = make_layout(*cfg, batch, img_tokens, prefix_max, false);
  const Layout trn = make_layout(*cfg, batch, img_tokens, prefix_max, true);
  if (workspace_bytes) *workspace_bytes = inf.scratch_bytes + inf.act_bytes;
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
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const size_t dh = cfg->head_dim, d = cfg->hidden, qd = cfg->n_q_heads * dh;
  h->rope_len = cfg->max_prefix + cfg->max_img_tokens;
  bool ok = cudaMalloc(&h->wo16, d * qd * 2) == cudaSuccess && cudaMalloc(&h->gamma, 2 * dh * 4) == cudaSuccess &&
            cudaMalloc(&h->rope, static_cast<size_t>(h->rope_len) * 64 * sizeof(float2)) == cudaSuccess &&
            cudaMalloc(&h->status, sizeof(int)) == cudaSuccess;
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
  bf16_to_f16_kernel<<<2 * h->num_sms, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(wts->w_o), h->wo16,
                                                     static_cast<long long>(d * qd / 8), h->status);
  ok = ok && cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess;
  if (ok) ok = build_weight_maps(h) == MOT_OK;
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
  if (v & DEV_ERR_TIMEOUT) return MOT_ERR_TIMEOUT;
  if (v & DEV_ERR_NUMERIC) return MOT_ERR_NUMERIC;
  return MOT_OK;
}

mot_status mot_attn_forward(mot_attn_t h, const void* x, int32_t B, int32_t N, const void* k_cache,
                            const void* v_cache, const int32_t* prefix_len, int32_t P, void* y, float* y_f32,
                            void* saved, size_t saved_bytes, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!h || !x || !y || !prefix_len || !workspace) return MOT_ERR_INVALID_ARGUMENT;
  const mot_attn_config& c = h->cfg;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  if (B > c.max_batch || N > c.max_img_tokens || P > c.max_prefix) return MOT_ERR_UNSUPPORTED_SHAPE;
  if (P > 0 && (!k_cache || !v_cache)) return MOT_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < B; ++b)
    if (prefix_len[b] < 0 || prefix_len[b] > P) return MOT_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {x, y, y_f32, saved, workspace, k_cache, v_cache};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOT_ERR_ALIGNMENT;
  const bool train = saved != nullptr;
  const Layout L = make_layout(c, B, N, P, train);
  if (train && saved_bytes < L.act_bytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  if (workspace_bytes < L.scratch_bytes + (train ? 0 : L.act_bytes)) return MOT_ERR_WORKSPACE_TOO_SMALL;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* act = train ? static_cast<uint8_t*>(saved) : ws + L.scratch_bytes;
  __half* q_hat = reinterpret_cast<__half*>(act + L.o_q);
  __half* k_all = reinterpret_cast<__half*>(act + L.o_k);
  __half* v_all = reinterpret_cast<__half*>(act + L.o_v);
  __half* attn = reinterpret_cast<__half*>(act + L.o_attn);
  float* lse = train ? reinterpret_cast<float*>(act + L.o_lse) : nullptr;
  __half* xhat = train ? reinterpret_cast<__half*>(act + L.o_xhat) : nullptr;
  float* rstd = train ? reinterpret_cast<float*>(act + L.o_rstd) : nullptr;
  __nv_bfloat16* u_qkv = reinterpret_cast<__nv_bfloat16*>(act + L.o_uqkv);
  __half* u_o = reinterpret_cast<__half*>(act + L.o_uo);
  __half* ao16 = reinterpret_cast<__half*>(ws + L.w_ao16);
  __half* bo16 = reinterpret_cast<__half*>(ws + L.w_bo16);

  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.hidden, M = L.M, r = h->rank, RP = h->RP;
  const int qd = Hq * 128, kvd = Hkv * 128, nqkv = qd + 2 * kvd;
  int launches = 0;
  cudaError_t e = cudaSuccess;
  int stage = 0;
  if (h->profile) cudaEventRecord(h->ev[0], st);
  auto chk = [&](cudaError_t err) {
    if (err != cudaSuccess && e == cudaSuccess) e = err;
    if (h->profile && launches < kMaxStages) {
      h->stage_ids[launches] = stage;
      cudaEventRecord(h->ev[launches + 1], st);
    }
    ++launches;
  };

  // 1. o-side LoRA tensors to f16 (they share the MMA with f16 activations)
  stage = ST_CVT_LORA_O;
  if (r > 0) {
    bf16_to_f16_kernel<<<64, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h->w.a_o), ao16,
                                           static_cast<long long>(r) * qd / 8, h->status);
    chk(cudaGetLastError());
    bf16_to_f16_kernel<<<64, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h->w.b_o), bo16,
                                           static_cast<long long>(d) * r / 8, h->status);
    chk(cudaGetLastError());
  }
  // 2. key/value buffers: prefix rows + zero tail
  stage = ST_BUILD_KV;
  {
    PlenArray pl{};
    for (int b = 0; b < B; ++b) pl.v[b] = prefix_len[b];
    const long long chunks = static_cast<long long>(B) * Hkv * L.Lcap * 16;
    const int grid = static_cast<int>(std::min<long long>((chunks + 255) / 256, 16LL * h->num_sms));
    build_kv_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k_cache),
                                          static_cast<const __nv_bfloat16*>(v_cache), k_all, v_all, Hkv,
                                          std::max(P, 1), N, L.Lcap, chunks, pl, h->status);
    chk(cudaGetLastError());
  }
  // 3. LoRA down for q/k/v: u_qkv[:, j*RP:(j+1)*RP] = s x A_j^T
  stage = ST_LORA_DOWN_QKV;
  if (r > 0) {
    GemmCore core;
    const int BN = RP == 64 ? 192 : 128;
    core_init(core, M, 3 * RP, BN, d / 64, 0, RP, idesc_f16(128, BN, true, true), 0, h->status);
    bool ok = map2d(&core.maps[0], x, true, d, M, d, 128);
    core.maps[2] = h->aq;
    core.maps[3] = h->ak;
    core.maps[4] = h->av;
    core.num_regions = 3;
    for (int j = 0; j < 3; ++j) core.regions[j] = GemmRegion{j * RP, (j + 1) * RP, 2 + j, -1, 0};
    EpiStore::Params ep{u_qkv, 1, 3 * RP, nullptr, 0, 0, h->scale, M, 3 * RP, 0};
    if (!ok) return MOT_ERR_CUDA;
    if (BN == 192)
      chk(launch_gemm<192, 5, EpiStore>(core, ep, h->num_sms, st));
    else
      chk(launch_gemm<128, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  // 4. QKV projection (+ LoRA up) with RMSNorm + RoPE epilogue
  stage = ST_QKV_GEMM;
  {
    GemmCore core;
    core_init(core, M, nqkv, 256, d / 64, r > 0 ? RP / 64 : 0, 256, idesc_f16(128, 256, true, true),
              idesc_f16(128, 256, true, true), h->status);
    bool ok = map2d(&core.maps[0], x, true, d, M, d, 128);
    if (r > 0) ok = ok && map2d(&core.maps[1], u_qkv, true, 3 * RP, M, 3 * RP, 128);
    core.maps[2] = h->wq;
    core.maps[3] = h->wk;
    core.maps[4] = h->wv;
    if (r > 0) {
      core.maps[5] = h->bq;
      core.maps[6] = h->bk;
      core.maps[7] = h->bv;
    }
    core.num_regions = 3;
    core.regions[0] = GemmRegion{0, qd, 2, r > 0 ? 5 : -1, 0};
    core.regions[1] = GemmRegion{qd, qd + kvd, 3, r > 0 ? 6 : -1, RP};
    core.regions[2] = GemmRegion{qd + kvd, nqkv, 4, r > 0 ? 7 : -1, 2 * RP};
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
    if (!ok) return MOT_ERR_CUDA;
    chk(launch_gemm<256, 4, EpiQkv>(core, ep, h->num_sms, st));
  }
  // 5. attention
  stage = ST_ATTN_FWD;
  {
    AttnFwdParams ap{};
    bool ok = map3d_heads(&ap.q_map, q_hat, N, static_cast<uint64_t>(B) * Hq) &&
              map3d_heads(&ap.k_map, k_all, L.Lcap, static_cast<uint64_t>(B) * Hkv) &&
              map3d_heads(&ap.v_map, v_all, L.Lcap, static_cast<uint64_t>(B) * Hkv);
    if (!ok) return MOT_ERR_CUDA;
    ap.B = B;
    ap.N = N;
    ap.Hq = Hq;
    ap.Hkv = Hkv;
    ap.Lcap = L.Lcap;
    ap.q_tiles = (N + 127) / 128;
    for (int b = 0; b < B; ++b) ap.plen[b] = prefix_len[b];
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
    ap.out = attn;
    ap.lse = lse;
    ap.status = h->status;
    static std::once_flag once;
    std::call_once(once, [] { set_smem_attr(attn_fwd_kernel, AttnSmem::kBytes); });
    attn_fwd_kernel<<<B * Hq * ap.q_tiles, kAttnThreads, AttnSmem::kBytes, st>>>(ap);
    chk(cudaGetLastError());
  }
  // 6. LoRA down for o: u_o = s o A_o^T (f16)
  stage = ST_LORA_DOWN_O;
  if (r > 0) {
    GemmCore core;
    core_init(core, M, RP, RP, qd / 64, 0, RP, idesc_f16(128, RP, false, false), 0, h->status);
    bool ok = map2d(&core.maps[0], attn, false, qd, M, qd, 128) &&
              map2d(&core.maps[2], ao16, false, qd, r, qd, RP);
    core.num_regions = 1;
    core.regions[0] = GemmRegion{0, RP, 2, -1, 0};
    EpiStore::Params ep{u_o, 0, RP, nullptr, 0, 0, h->scale, M, RP, 1};
    if (!ok) return MOT_ERR_CUDA;
    if (RP == 64)
      chk(launch_gemm<64, 8, EpiStore>(core, ep, h->num_sms, st));
    else
      chk(launch_gemm<128, 6, EpiStore>(core, ep, h->num_sms, st));
  }
  // 7. O projection (+ LoRA up): y bf16 and optional f32
  stage = ST_O_GEMM;
  {
    GemmCore core;
    core_init(core, M, d, 256, qd / 64, r > 0 ? RP / 64 : 0, 256, idesc_f16(128, 256, false, false),
              idesc_f16(128, 256, false, false), h->status);
    bool ok = map2d(&core.maps[0], attn, false, qd, M, qd, 128);
    if (r > 0) ok = ok && map2d(&core.maps[1], u_o, false, RP, M, RP, 128) && map2d(&core.maps[3], bo16, false, r, d, r, 256);
    core.maps[2] = h->wo;
    core.num_regions = 1;
    core.regions[0] = GemmRegion{0, d, 2, r > 0 ? 3 : -1, 0};
    EpiStore::Params ep{y, 1, d, y_f32, d, 0, 1.0f, M, d, 0};
    if (!ok) return MOT_ERR_CUDA;
    chk(launch_gemm<256, 4, EpiStore>(core, ep, h->num_sms, st));
  }
  h->last_launches = launches;
  h->stage_count = std::min(launches, kMaxStages);
  return e == cudaSuccess ? MOT_OK : MOT_ERR_CUDA;
}

mot_status mot_attn_backward(mot_attn_t h, const void* dy, const void* x, int32_t B, int32_t N, const void* k_cache,
                             const void* v_cache, const int32_t* prefix_len, int32_t P, const void* saved,
                             size_t saved_bytes, void* dx, float* dx_f32, float* const d_a[4], float* const d_b[4],
                             int32_t accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  (void)dy; (void)x; (void)B; (void)N; (void)k_cache; (void)v_cache; (void)prefix_len; (void)P; (void)saved_bytes;
  (void)dx; (void)dx_f32; (void)d_a; (void)d_b; (void)accumulate; (void)workspace; (void)workspace_bytes;
  (void)stream;
  if (!h) return MOT_ERR_INVALID_ARGUMENT;
  if (!saved) return MOT_ERR_NO_SAVED_STATE;
  return MOT_ERR_UNSUPPORTED_SHAPE;
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
  // rebind: merged base, no adapters; W_o's f16 copy is rebuilt from the merged W_o
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
  bf16_to_f16_kernel<<<2 * h->num_sms, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w_o_out), h->wo16,
                                                     static_cast<long long>(d) * qd / 8, h->status);
  if (cudaGetLastError() != cudaSuccess) return MOT_ERR_CUDA;
  return build_weight_maps(h);
}

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

extern "C" mot_status mot_attn_forward_noalloc(mot_attn_t h, const void* x, int32_t B, int32_t N,
                                               const void* k_cache, const void* v_cache,
                                               const int32_t* prefix_len, int32_t P, void* y, float* y_f32,
                                               void* stream) {
  if (!h || !x || !y || !prefix_len) return MOT_ERR_INVALID_ARGUMENT;
  if (B <= 0 || N <= 0 || P < 0) return MOT_ERR_INVALID_ARGUMENT;
  size_t need = 0;
  const mot_status st = mot_attn_query_sizes(&h->cfg, B, N, P, &need, nullptr);
  if (st != MOT_OK) return st;
  if (need > kNoAllocScratchBytes) return MOT_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return MOT_ERR_CUDA;
  return mot_attn_forward(h, x, B, N, k_cache, v_cache, prefix_len, P, y, y_f32, nullptr, 0, scratch,
                          kNoAllocScratchBytes, stream);
}

// ------------------------------------------------------------------ dev entry points
mot_status mot_dev_gemm(const void* a, const void* b, float* dmat, int32_t m, int32_t n, int32_t k, int32_t is_bf16,
                        void* stream) {
  if (!a || !b || !dmat || m <= 0 || n <= 0 || k <= 0) return MOT_ERR_INVALID_ARGUMENT;
  if (k % 64 != 0 || n % 256 != 0) return MOT_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(dmat)) return MOT_ERR_ALIGNMENT;
  GemmCore core;
  const bool bf = is_bf16 != 0;
  core_init(core, m, n, 256, k / 64, 0, 256, idesc_f16(128, 256, bf, bf), 0, nullptr);
  if (!map2d(&core.maps[0], a, bf, k, m, k, 128) || !map2d(&core.maps[2], b, bf, k, n, k, 256)) return MOT_ERR_CUDA;
  core.num_regions = 1;
  core.regions[0] = GemmRegion{0, n, 2, -1, 0};
  EpiStore::Params ep{nullptr, 0, 0, dmat, n, 0, 1.0f, m, n, 0};
  return launch_gemm<256, 4, EpiStore>(core, ep, 148, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOT_OK
             : MOT_ERR_CUDA;
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
  if (cudaEventSynchronize(h->ev[h->stage_count]) != cudaSuccess) return MOT_ERR_CUDA;
  for (int i = 0; i < h->stage_count && i < max; ++i) {
    ids[i] = h->stage_ids[i];
    if (cudaEventElapsedTime(&ms[i], h->ev[i], h->ev[i + 1]) != cudaSuccess) return MOT_ERR_CUDA;
  }
  return MOT_OK;
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
