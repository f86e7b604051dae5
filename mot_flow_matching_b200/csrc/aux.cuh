// aux.cuh -- bandwidth-bound helper kernels (no tensor cores).
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace mot {

struct PlenArray {
  int v[kMaxBatch];
};

// Build the attention key/value buffers [B, Hkv, Lcap, dh] (f16) around the
// self rows the QKV epilogue writes: rows [0, plen[b]) take the cached prefix
// (bf16 -> f16, exact for |x| <= 65504 apart from f16 subnormals), rows
// [plen[b] + N, Lcap) are zeroed so masked key tiles never hold NaN/Inf.
// "Setup notes" (LoRA trainer docs): the prefix-KV cache is static input.
// Only the rows this kernel owns are walked: Lcap - N per (branch, KV head),
// row r < plen[b] maps to r, the rest to r + N. One thread moves 8 elements
// (16 bytes). The same launch first converts the jobs in `cvt` (the f16
// copies of the LoRA tensors that meet f16 operands, per call since a
// trainer may update them in place), so a forward makes one launch for both.
struct CvtJobs {
  const __nv_bfloat16* src[6];
  __half* dst[6];
  long long n8[6];  // element count / 8
  int count;
};

__device__ __forceinline__ bool cvt_jobs_run(const CvtJobs& jobs) {
  bool overflow = false;
  for (int j = 0; j < jobs.count; ++j) {
    const uint4* src = reinterpret_cast<const uint4*>(jobs.src[j]);
    uint4* dst = reinterpret_cast<uint4*>(jobs.dst[j]);
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < jobs.n8[j];
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
      const uint4 r = src[i];
      const __nv_bfloat162* bv = reinterpret_cast<const __nv_bfloat162*>(&r);
      float2 f[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[k] = __bfloat1622float2(bv[k]);
        overflow |= fabsf(f[k].x) > 65504.f || fabsf(f[k].y) > 65504.f;
      }
      dst[i] = make_uint4(pack_half2(f[0].x, f[0].y), pack_half2(f[1].x, f[1].y), pack_half2(f[2].x, f[2].y),
                          pack_half2(f[3].x, f[3].y));
    }
  }
  return overflow;
}

__global__ void __launch_bounds__(256) build_kv_kernel(const __nv_bfloat16* __restrict__ kc,
                                                       const __nv_bfloat16* __restrict__ vc,
                                                       __half* __restrict__ kall, __half* __restrict__ vall,
                                                       int Hkv, int Pmax, int N, int Lcap, long long total_chunks,
                                                       PlenArray plen, const CvtJobs cvt, int* status) {
  grid_dep_launch();
  grid_dep_wait();
  bool overflow = cvt_jobs_run(cvt);
  const int own = Lcap - N;  // rows of one (branch, KV head) written here
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total_chunks;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int chunk = static_cast<int>(idx & 15);
    const long long rg = idx >> 4;
    const int r = static_cast<int>(rg % own);
    const long long bg = rg / own;
    const int b = static_cast<int>(bg / Hkv);
    const int pl = plen.v[b];
    const int row = r < pl ? r : r + N;
    const long long dst = (bg * Lcap + row) * 128 + chunk * 8;
    uint4* kd = reinterpret_cast<uint4*>(kall + dst);
    uint4* vd = reinterpret_cast<uint4*>(vall + dst);
    if (row < pl) {
      const long long src = (bg * Pmax + row) * 128 + chunk * 8;
      const uint4 kr = *reinterpret_cast<const uint4*>(kc + src);
      const uint4 vr = *reinterpret_cast<const uint4*>(vc + src);
      const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(&kr);
      const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(&vr);
      uint4 ko, vo;
      uint32_t* ko32 = reinterpret_cast<uint32_t*>(&ko);
      uint32_t* vo32 = reinterpret_cast<uint32_t*>(&vo);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float k0 = __bfloat162float(kb[2 * i]), k1 = __bfloat162float(kb[2 * i + 1]);
        const float v0 = __bfloat162float(vb[2 * i]), v1 = __bfloat162float(vb[2 * i + 1]);
        overflow |= fabsf(k0) > 65504.f || fabsf(k1) > 65504.f || fabsf(v0) > 65504.f || fabsf(v1) > 65504.f;
        ko32[i] = pack_half2(k0, k1);
        vo32[i] = pack_half2(v0, v1);
      }
      *kd = ko;
      *vd = vo;
    } else {
      *kd = make_uint4(0, 0, 0, 0);
      *vd = make_uint4(0, 0, 0, 0);
    }
  }
  if (overflow) atomicOr(status, DEV_ERR_NUMERIC);
}

// LoRA bake-in ("SenseNova-U1.5" vLLM-Omni recipe, 8-step distilled LoRA:
// fused into the gen tower at load):
//   out[i, j] = RNE_bf16(w[i, j] + s * sum_k b[i, k] a[k, j]),
// the sum over k ascending in f32, then one f32 fma and one rounding to bf16.
// out may alias w (each element reads its own w before writing it).
// Block: 32 x 8 threads over a 8-row x 256-column patch; b rows staged in smem.
__global__ void __launch_bounds__(256) merge_lora_kernel(const __nv_bfloat16* w, const __nv_bfloat16* __restrict__ a,
                                                         const __nv_bfloat16* __restrict__ bm, __nv_bfloat16* out,
                                                         int rows, int cols, int r, float s) {
  __shared__ float sb[8][128];
  const int i0 = blockIdx.y * 8;
  for (int t = threadIdx.y * 32 + threadIdx.x; t < 8 * r; t += 256) {
    const int ii = t / r, k = t % r;
    sb[ii][k] = (i0 + ii < rows) ? __bfloat162float(bm[static_cast<long long>(i0 + ii) * r + k]) : 0.f;
  }
  __syncthreads();
  const int i = i0 + threadIdx.y;
  if (i >= rows) return;
#pragma unroll 1
  for (int jj = 0; jj < 8; ++jj) {
    const int j = blockIdx.x * 256 + jj * 32 + threadIdx.x;
    if (j >= cols) break;
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < r; ++k) acc = fmaf(sb[threadIdx.y][k], __bfloat162float(a[static_cast<long long>(k) * cols + j]), acc);
    const long long o = static_cast<long long>(i) * cols + j;
    out[o] = __float2bfloat16_rn(fmaf(s, acc, __bfloat162float(w[o])));
  }
}

// Transposed copy of a bf16 [rows, cols] matrix into dst [cols, ...] at
// column offset col_off of rows of length ld_dst: dst[c * ld_dst + col_off + r]
// = src[r * cols + c], as bf16 or converted to f16 (exact for weights in the
// f16 range). 32 x 32 tiles through shared memory, reads and writes coalesced.
template <class OutT>
__global__ void __launch_bounds__(256) transpose_copy_kernel(const __nv_bfloat16* __restrict__ src, int rows, int cols,
                                                             OutT* __restrict__ dst, long long ld_dst, int col_off) {
  __shared__ float tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
#pragma unroll
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < rows && c < cols) ? __bfloat162float(src[static_cast<long long>(r) * cols + c]) : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows) {
      const float v = tile[threadIdx.x][i];
      OutT* o = dst + static_cast<long long>(c) * ld_dst + col_off + r;
      if constexpr (sizeof(OutT) == 2 && std::is_same<OutT, __half>::value)
        *o = __float2half_rn(v);
      else
        *o = __float2bfloat16_rn(v);
    }
  }
}

// bf16 -> f16 copies (tensors that meet f16 operands in an MMA), outside a forward
__global__ void __launch_bounds__(256) cvt_multi_kernel(const CvtJobs jobs, int* status) {
  grid_dep_launch();
  grid_dep_wait();
  const bool overflow = cvt_jobs_run(jobs);
  if (overflow && status) atomicOr(status, DEV_ERR_NUMERIC);
}

// Zero-padded f16 copies of lora_up tensors: dst [rows, ld] holds src
// [rows, r] (bf16) in columns [col0, col0 + r) and zeros elsewhere (col0, r
// and ld multiples of 8). The gate and up LoRA-up tensors of the SwiGLU MLP
// become the two blocks of a block-diagonal K extension this way: the gate
// copy in columns [0, r) and the up copy in [RP, RP + r) of [I, 2 RP] rows,
// against u = [s x A_gate^T | s x A_up^T].
struct PadJobs {
  const __nv_bfloat16* src[2];
  __half* dst[2];
  long long rows[2];
  int r, ld, col0[2];
  int count;
};

// Per-call preparation of the MLP's LoRA tensors in one launch: the plain
// conversions in `cvt`, then the padded copies in `pad`.
__global__ void __launch_bounds__(256) mlp_prep_kernel(const CvtJobs cvt, const PadJobs pad, int* status) {
  grid_dep_launch();
  grid_dep_wait();
  bool overflow = cvt_jobs_run(cvt);
  const int chunks_per_row = pad.ld / 8;
  for (int j = 0; j < pad.count; ++j) {
    const long long n = pad.rows[j] * chunks_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
      const long long row = i / chunks_per_row;
      const int col = static_cast<int>(i - row * chunks_per_row) * 8;
      uint4 o = make_uint4(0, 0, 0, 0);
      if (col >= pad.col0[j] && col < pad.col0[j] + pad.r) {
        const uint4 v = *reinterpret_cast<const uint4*>(pad.src[j] + row * pad.r + (col - pad.col0[j]));
        const __nv_bfloat162* bv = reinterpret_cast<const __nv_bfloat162*>(&v);
        float2 f[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          f[k] = __bfloat1622float2(bv[k]);
          overflow |= fabsf(f[k].x) > 65504.f || fabsf(f[k].y) > 65504.f;
        }
        o = make_uint4(pack_half2(f[0].x, f[0].y), pack_half2(f[1].x, f[1].y), pack_half2(f[2].x, f[2].y),
                       pack_half2(f[3].x, f[3].y));
      }
      *reinterpret_cast<uint4*>(pad.dst[j] + row * pad.ld + col) = o;
    }
  }
  if (overflow && status) atomicOr(status, DEV_ERR_NUMERIC);
}

// ------------------------------------------------------------------ denoise step
// RMSNorm of rows of the f32 residual stream into the bf16 input of the next
// block: out[m] = RNE_bf16(h[m] / sqrt(mean(h[m]^2) + eps) * gain). With
// `src` (the step's first norm) row m first becomes src[m % src_rows] + bias
// (the patch embedding plus the timestep embedding, the same for every
// branch) and is written back to h. One warp per row; d a multiple of 128.
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(float* __restrict__ h, const float* __restrict__ src,
                                                           int src_rows, const float* __restrict__ bias,
                                                           const float* __restrict__ gain,
                                                           __nv_bfloat16* __restrict__ out, int rows, int d,
                                                           float eps) {
  grid_dep_launch();
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int m = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); m < rows; m += nwarps) {
    float* hr = h + static_cast<long long>(m) * d;
    float ss = 0.f;
    if (src) {
      const float* sr = src + static_cast<long long>(m % src_rows) * d;
      for (int c = lane * 4; c < d; c += 128) {
        float4 v = *reinterpret_cast<const float4*>(sr + c);
        const float4 b4 = *reinterpret_cast<const float4*>(bias + c);
        v.x += b4.x;
        v.y += b4.y;
        v.z += b4.z;
        v.w += b4.w;
        *reinterpret_cast<float4*>(hr + c) = v;
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
    } else {
      for (int c = lane * 4; c < d; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(hr + c);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = rsqrtf(ss / static_cast<float>(d) + eps);
    __nv_bfloat16* orow = out + static_cast<long long>(m) * d;
    for (int c = lane * 4; c < d; c += 128) {
      const float4 v = *reinterpret_cast<const float4*>(hr + c);
      const float4 g = *reinterpret_cast<const float4*>(gain + c);
      *reinterpret_cast<uint2*>(orow + c) =
          make_uint2(pack_bf162(v.x * rs * g.x, v.y * rs * g.y), pack_bf162(v.z * rs * g.z, v.w * rs * g.w));
    }
  }
}

// Timestep embedding of the step (f32 [d]): cos(1000 sigma f_k) at k and
// sin(1000 sigma f_k) at d/2 + k, f_k = 10000^(-k/(d/2)), in double.
__global__ void temb_kernel(float* __restrict__ out, int d, double sigma) {
  grid_dep_launch();
  grid_dep_wait();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < d / 2) {
    const double ang = 1000.0 * sigma * pow(10000.0, -static_cast<double>(k) / (d / 2));
    out[k] = static_cast<float>(cos(ang));
    out[d / 2 + k] = static_cast<float>(sin(ang));
  }
}

// Guidance over the branches' x0 predictions (cfg_norm none; branch order
// cond, [image-cond,] uncond) and the Euler update of the image's patch
// tokens: z_next = z + c (z - x0), c = (sigma_next - sigma) / max(sigma,
// t_eps), also as bf16 for the next step's embedding GEMM. x0 [B, n], z [n].
__global__ void __launch_bounds__(256) cfg_euler_kernel(const float* __restrict__ x0, long long n, int B,
                                                        const float* __restrict__ z, float* __restrict__ z_next,
                                                        __nv_bfloat16* __restrict__ z_next16, float cfg,
                                                        float img_cfg, float c) {
  grid_dep_launch();
  grid_dep_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float x;
    if (B == 1)
      x = x0[i];
    else if (B == 2)
      x = x0[n + i] + cfg * (x0[i] - x0[n + i]);
    else
      x = x0[2 * n + i] + img_cfg * (x0[n + i] - x0[2 * n + i]) + cfg * (x0[i] - x0[n + i]);
    const float zi = z[i];
    const float zn = zi + c * (zi - x);
    z_next[i] = zn;
    if (z_next16) z_next16[i] = __float2bfloat16_rn(zn);
  }
}

// f32 -> bf16, round to nearest even (the patch tokens as a GEMM operand)
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ src,
                                                          __nv_bfloat16* __restrict__ dst, long long n) {
  grid_dep_launch();
  grid_dep_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// 2^x of a buffer through exp2_poly2 (accuracy tests of the softmax's FMA-pipe exponential)
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int npairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < npairs) exp2_poly2(y[2 * i], y[2 * i + 1], x[2 * i], x[2 * i + 1]);
}

// Failure-detection check of the bounded waits: one thread waits on an
// mbarrier that nothing ever arrives on, through the same bounded wait every
// kernel uses, so the wait gives up after its limit, latches DEV_ERR_TIMEOUT
// in `status` and the kernel exits normally (no trap, no fault).
__global__ void wait_probe_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitGuard wg{&abort_flag, status};
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, wg);  // phase 0 never completes
  __syncthreads();
}

// f32 copy of a bf16 vector (norm gains)
__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = __bfloat162float(src[i]);
}

}  // namespace mot
