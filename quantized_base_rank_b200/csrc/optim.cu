// The adapter optimiser steps. AdamW with paged states (QLoRA page, aizip.shop/methodologies/qlora,
// section "3. Paged Optimizer": optimiser states kept in unified memory, which the driver
// pages to host RAM when device memory runs short and back on access).
//
// ql_adamw_step updates one flat fp32 vector of adapter parameters (the trained copy),
// its first and second moments, and the bf16 copy the linear layers read: one pass over
// 30 bytes per parameter (read grad, theta, m, v; write theta, m, v, bf16), 16-byte
// vectors, grid sized to the SM count. Any of the arrays may be managed memory from
// ql_paged_alloc: the kernel is the same, and pages that were moved to the host migrate
// back as the kernel touches them (or ahead of it, with ql_paged_prefetch).
#include <cmath>

#include "common.cuh"

namespace qlb {

struct AdamwConst {
  float beta1, beta2, one_m_beta1, one_m_beta2;
  float step_size;      // lr / (1 - beta1^t)
  float inv_sqrt_bc2;   // 1 / sqrt(1 - beta2^t)
  float eps;
  float decay;          // 1 - lr * weight_decay
  float grad_scale;
};

__device__ __forceinline__ float adamw_one(const AdamwConst& c, float g, float& th, float& m, float& v) {
  g *= c.grad_scale;
  m = c.beta1 * m + c.one_m_beta1 * g;
  v = c.beta2 * v + c.one_m_beta2 * (g * g);
  const float denom = sqrtf(v) * c.inv_sqrt_bc2 + c.eps;
  th = th * c.decay - c.step_size * (m / denom);
  return g;
}

// VEC: all pointers 16-byte aligned (8 for the bf16 copy) and whole groups of 4; else one
// element per thread step.
template <bool VEC>
__global__ void __launch_bounds__(256)
adamw_kernel(float* __restrict__ theta, uint16_t* __restrict__ param, const float* __restrict__ grad,
             float* __restrict__ m, float* __restrict__ v, int64_t n, AdamwConst c, int* flag) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  bool bad = false;
  if (VEC) {
    const int64_t n4 = n >> 2;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
      float4 g = reinterpret_cast<const float4*>(grad)[i];
      float4 th = reinterpret_cast<float4*>(theta)[i];
      float4 mm = reinterpret_cast<float4*>(m)[i];
      float4 vv = reinterpret_cast<float4*>(v)[i];
      bad |= !isfinite(g.x) || !isfinite(g.y) || !isfinite(g.z) || !isfinite(g.w);
      adamw_one(c, g.x, th.x, mm.x, vv.x);
      adamw_one(c, g.y, th.y, mm.y, vv.y);
      adamw_one(c, g.z, th.z, mm.z, vv.z);
      adamw_one(c, g.w, th.w, mm.w, vv.w);
      reinterpret_cast<float4*>(theta)[i] = th;
      reinterpret_cast<float4*>(m)[i] = mm;
      reinterpret_cast<float4*>(v)[i] = vv;
      reinterpret_cast<uint2*>(param)[i] =
          make_uint2((uint32_t)float_to_bf16_bits(th.x) | ((uint32_t)float_to_bf16_bits(th.y) << 16),
                     (uint32_t)float_to_bf16_bits(th.z) | ((uint32_t)float_to_bf16_bits(th.w) << 16));
    }
  } else {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
      float th = theta[i], mm = m[i], vv = v[i];
      const float g = grad[i];
      bad |= !isfinite(g);
      adamw_one(c, g, th, mm, vv);
      theta[i] = th;
      m[i] = mm;
      v[i] = vv;
      param[i] = float_to_bf16_bits(th);
    }
  }
  if (bad) raise_flag(flag, kFlagNonfinite);
}

// ---- Lion with INT8 momentum (QFT page, gist.science/ko/paper/2310.07147, section 2.1) ----
//
// One warp per block of 64 parameters, two per lane. The momentum arrives as INT8 codes
// with the block's fp32 absmax, is decoded, used and re-encoded with the block's new
// absmax (a warp max). Every floating-point step is an explicitly rounded fp32 operation
// in a fixed order (no contraction into fused multiply-adds), because the new codes are
// integer decisions. 16 bytes per parameter (theta read and written, grad, the code read
// and written, the bf16 copy).
struct LionConst {
  float lr, beta1, beta2, omb1, omb2, decay;
};

// The step of one pair of parameters (elements e0, e0 + 1 of block b, as the lane's
// share), given the block's decoded scale; returns the new momentum values for the
// block's re-encoding.
__device__ __forceinline__ void lion_pair(const LionConst& c, float sc, const float (&t)[2], const float (&g)[2],
                                          const int (&q)[2], float (&tn)[2], float (&mn)[2]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float m = __fmul_rn((float)q[i], sc);
    const float cv = __fadd_rn(__fmul_rn(c.beta1, m), __fmul_rn(c.omb1, g[i]));
    const float u = cv > 0.0f ? 1.0f : (cv < 0.0f ? -1.0f : 0.0f);
    tn[i] = __fsub_rn(__fmul_rn(t[i], c.decay), __fmul_rn(c.lr, u));
    mn[i] = __fadd_rn(__fmul_rn(c.beta2, m), __fmul_rn(c.omb2, g[i]));
  }
}

// Re-encodes a block's new momentum (a warp max of |m'|, then one code per element).
__device__ __forceinline__ float lion_encode(const float (&mn)[2], int8_t (&q)[2]) {
  float a = fmaxf(fabsf(mn[0]), fabsf(mn[1]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  const float sn = __fdiv_rn(a, 127.0f);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float r = rintf(__fdiv_rn(mn[i], sn));
    q[i] = sn == 0.0f ? (int8_t)0 : (int8_t)fminf(fmaxf(r, -127.0f), 127.0f);
  }
  return a;
}

// VEC: theta and grad 8-byte aligned, param 4-byte, codes 2-byte: each lane moves its two
// elements with one load or store per array, and a warp takes two blocks per iteration
// with every load issued before any is used. The tail (a partial last block) and the
// unaligned case take the scalar path.
template <bool VEC>
__global__ void __launch_bounds__(256)
lion_int8_kernel(float* __restrict__ theta, uint16_t* __restrict__ param, const float* __restrict__ grad,
                 int8_t* __restrict__ codes, float* __restrict__ absmax, int64_t n, LionConst c, int* flag) {
  const int lane = threadIdx.x & 31;
  const int64_t nb = (n + 63) / 64;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  bool bad = false;
  if (VEC) {
    const int64_t nfull = n / 64;                       // whole blocks
    for (int64_t b0 = w; b0 < nfull; b0 += 2 * warps) {
      const int64_t b1 = b0 + warps;
      const bool two = b1 < nfull;
      const int64_t e0 = b0 * 64 + 2 * lane, e1 = b1 * 64 + 2 * lane;
      const float2 ta = reinterpret_cast<const float2*>(theta)[e0 >> 1];
      const float2 ga = reinterpret_cast<const float2*>(grad)[e0 >> 1];
      const uint16_t qa = reinterpret_cast<const uint16_t*>(codes)[e0 >> 1];
      const float aa = absmax[b0];
      float2 tb = make_float2(0.0f, 0.0f), gb = tb;
      uint16_t qb = 0;
      float ab = 0.0f;
      if (two) {
        tb = reinterpret_cast<const float2*>(theta)[e1 >> 1];
        gb = reinterpret_cast<const float2*>(grad)[e1 >> 1];
        qb = reinterpret_cast<const uint16_t*>(codes)[e1 >> 1];
        ab = absmax[b1];
      }
      {
        const float t[2] = {ta.x, ta.y}, g[2] = {ga.x, ga.y};
        const int q[2] = {(int)(int8_t)(qa & 0xFF), (int)(int8_t)(qa >> 8)};
        bad |= !isfinite(g[0]) || !isfinite(g[1]);
        float tn[2], mn[2];
        lion_pair(c, __fdiv_rn(aa, 127.0f), t, g, q, tn, mn);
        int8_t o[2];
        const float a = lion_encode(mn, o);
        reinterpret_cast<float2*>(theta)[e0 >> 1] = make_float2(tn[0], tn[1]);
        reinterpret_cast<uint16_t*>(codes)[e0 >> 1] = (uint16_t)((uint8_t)o[0] | ((uint16_t)(uint8_t)o[1] << 8));
        reinterpret_cast<uint32_t*>(param)[e0 >> 1] =
            (uint32_t)float_to_bf16_bits(tn[0]) | ((uint32_t)float_to_bf16_bits(tn[1]) << 16);
        if (lane == 0) absmax[b0] = a;
      }
      if (two) {                                        // warp-uniform
        const float t[2] = {tb.x, tb.y}, g[2] = {gb.x, gb.y};
        const int q[2] = {(int)(int8_t)(qb & 0xFF), (int)(int8_t)(qb >> 8)};
        bad |= !isfinite(g[0]) || !isfinite(g[1]);
        float tn[2], mn[2];
        lion_pair(c, __fdiv_rn(ab, 127.0f), t, g, q, tn, mn);
        int8_t o[2];
        const float a = lion_encode(mn, o);
        reinterpret_cast<float2*>(theta)[e1 >> 1] = make_float2(tn[0], tn[1]);
        reinterpret_cast<uint16_t*>(codes)[e1 >> 1] = (uint16_t)((uint8_t)o[0] | ((uint16_t)(uint8_t)o[1] << 8));
        reinterpret_cast<uint32_t*>(param)[e1 >> 1] =
            (uint32_t)float_to_bf16_bits(tn[0]) | ((uint32_t)float_to_bf16_bits(tn[1]) << 16);
        if (lane == 0) absmax[b1] = a;
      }
    }
  }
  // scalar path: every block (not VEC) or the partial last block (VEC)
  for (int64_t b = VEC ? n / 64 + w : w; b < nb; b += warps) {
    const int64_t e0 = b * 64 + 2 * lane;
    const bool in0 = e0 < n, in1 = e0 + 1 < n;
    const float t[2] = {in0 ? theta[e0] : 0.0f, in1 ? theta[e0 + 1] : 0.0f};
    const float g[2] = {in0 ? grad[e0] : 0.0f, in1 ? grad[e0 + 1] : 0.0f};
    const int q[2] = {in0 ? (int)codes[e0] : 0, in1 ? (int)codes[e0 + 1] : 0};
    bad |= !isfinite(g[0]) || !isfinite(g[1]);
    float tn[2], mn[2];
    lion_pair(c, __fdiv_rn(absmax[b], 127.0f), t, g, q, tn, mn);
    if (!in0) mn[0] = 0.0f;
    if (!in1) mn[1] = 0.0f;
    int8_t o[2];
    const float a = lion_encode(mn, o);
    if (in0) {
      theta[e0] = tn[0];
      codes[e0] = o[0];
      param[e0] = float_to_bf16_bits(tn[0]);
    }
    if (in1) {
      theta[e0 + 1] = tn[1];
      codes[e0 + 1] = o[1];
      param[e0 + 1] = float_to_bf16_bits(tn[1]);
    }
    if (lane == 0) absmax[b] = a;
  }
  if (bad) raise_flag(flag, kFlagNonfinite);
}

}  // namespace qlb

using namespace qlb;

extern "C" {

ql_status ql_adamw_step(float* theta, ql_bf16* param, const float* grad, float* m, float* v, int64_t n,
                        const ql_adamw* h, void* stream) {
  if (n < 0 || !h) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!theta || !param || !grad || !m || !v) return QL_ERR_INVALID_ARG;
  if (!aligned(theta, 4) || !aligned(grad, 4) || !aligned(m, 4) || !aligned(v, 4) || !aligned(param, 2))
    return QL_ERR_INVALID_ARG;
  if (h->step < 1 || !(h->lr >= 0.0f) || !(h->beta1 >= 0.0f && h->beta1 < 1.0f) ||
      !(h->beta2 >= 0.0f && h->beta2 < 1.0f) || !(h->eps > 0.0f) || !(h->weight_decay >= 0.0f) ||
      !std::isfinite(h->grad_scale))
    return QL_ERR_INVALID_ARG;
  AdamwConst c;
  const double t = (double)h->step;
  const double bc1 = 1.0 - std::pow((double)h->beta1, t), bc2 = 1.0 - std::pow((double)h->beta2, t);
  c.beta1 = h->beta1;
  c.beta2 = h->beta2;
  c.one_m_beta1 = (float)(1.0 - (double)h->beta1);
  c.one_m_beta2 = (float)(1.0 - (double)h->beta2);
  c.step_size = (float)((double)h->lr / bc1);
  c.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  c.eps = h->eps;
  c.decay = (float)(1.0 - (double)h->lr * (double)h->weight_decay);
  c.grad_scale = h->grad_scale;
  cudaStream_t st = as_stream(stream);
  const bool vec = n % 4 == 0 && aligned(theta, 16) && aligned(grad, 16) && aligned(m, 16) &&
                   aligned(v, 16) && aligned(param, 8);
  const int64_t work = vec ? n / 4 : n;
  const unsigned grid = (unsigned)imax64(1, imin64((work + 255) / 256, (int64_t)num_sms() * 8));
  ProfScope prof(PK_OPTIM, st, 1);
  if (vec)
    adamw_kernel<true><<<grid, 256, 0, st>>>(theta, param, grad, m, v, n, c, device_flag_ptr());
  else
    adamw_kernel<false><<<grid, 256, 0, st>>>(theta, param, grad, m, v, n, c, device_flag_ptr());
  QL_CHECK_LAUNCH();
  return QL_OK;
}

ql_status ql_lion_int8_step(float* theta, ql_bf16* param, const float* grad, int8_t* m_codes, float* m_absmax,
                            int64_t n, const ql_lion* h, void* stream) {
  if (n < 0 || !h) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!theta || !param || !grad || !m_codes || !m_absmax) return QL_ERR_INVALID_ARG;
  if (!aligned(theta, 4) || !aligned(grad, 4) || !aligned(m_absmax, 4) || !aligned(param, 2))
    return QL_ERR_INVALID_ARG;
  if (!(h->lr >= 0.0f) || !std::isfinite(h->lr) || !(h->beta1 >= 0.0f && h->beta1 <= 1.0f) ||
      !(h->beta2 >= 0.0f && h->beta2 <= 1.0f) || !(h->weight_decay >= 0.0f) || !std::isfinite(h->weight_decay))
    return QL_ERR_INVALID_ARG;
  // fp32, one rounding per operation, as the step defines them
  LionConst c;
  c.lr = h->lr;
  c.beta1 = h->beta1;
  c.beta2 = h->beta2;
  volatile float omb1 = 1.0f - h->beta1, omb2 = 1.0f - h->beta2;
  volatile float lr_wd = h->lr * h->weight_decay;
  volatile float decay = 1.0f - lr_wd;
  c.omb1 = omb1;
  c.omb2 = omb2;
  c.decay = decay;
  cudaStream_t st = as_stream(stream);
  const int64_t nb = (n + 63) / 64;
  const unsigned grid = (unsigned)imax64(1, imin64((nb + 7) / 8, (int64_t)num_sms() * 8));
  ProfScope prof(PK_OPTIM, st, 1);
  const bool vec = aligned(theta, 8) && aligned(grad, 8) && aligned(param, 4) && aligned(m_codes, 2);
  if (vec)
    lion_int8_kernel<true><<<grid, 256, 0, st>>>(theta, param, grad, m_codes, m_absmax, n, c, device_flag_ptr());
  else
    lion_int8_kernel<false><<<grid, 256, 0, st>>>(theta, param, grad, m_codes, m_absmax, n, c, device_flag_ptr());
  QL_CHECK_LAUNCH();
  return QL_OK;
}

ql_status ql_paged_alloc(size_t bytes, void** out) {
  if (!out) return QL_ERR_INVALID_ARG;
  *out = nullptr;
  if (bytes == 0) return QL_OK;
  if (cudaMallocManaged(out, bytes, cudaMemAttachGlobal) != cudaSuccess) {
    *out = nullptr;
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status ql_paged_free(void* p) {
  if (!p) return QL_OK;
  return cudaFree(p) == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status ql_paged_prefetch(const void* p, size_t bytes, int32_t to_host, void* stream) {
  if (!p) return bytes == 0 ? QL_OK : QL_ERR_INVALID_ARG;
  if (bytes == 0) return QL_OK;
  int dev = 0;
  if (!to_host && cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  const cudaError_t e = cudaMemPrefetchAsync(p, bytes, to_host ? cudaCpuDeviceId : dev, as_stream(stream));
  return e == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // extern "C"
