// The adapter optimiser step with paged states (QLoRA page, aizip.shop/methodologies/qlora,
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
