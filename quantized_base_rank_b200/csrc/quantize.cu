// Quantisation kernels: NF4 encode with blockwise absmax, double quantisation of the
// absmax constants, blockwise int8, and standalone dequantisation.
//
// QLoRA page (aizip.shop/methodologies/qlora): "1. 4-bit NormalFloat (NF4)" defines the
// quantile grid; "2. Double Quantization" the block size 64 and the re-quantised
// constants. The int8 format is the 8-bit option of AutoQRA's per-layer bit-width
// (gist.science/ko/paper/2602.22268, section 3.1).
//
// All of these are HBM-bound streaming passes: one thread owns one block of 64
// elements (128 B of bf16 read with eight 16-byte loads), so the decision data of a
// block (its absmax and boundaries) lives in registers and nothing is staged.
#include <math.h>

#include "common.cuh"

namespace qlb {

// ---------------------------------------------------------------------------------
// NF4 encode.
//
// Decision (exact): code = #{ j : x / a >= m_j } with m_j the exact midpoints of the
// grid, ties to the upper point, and code 8 for an all-zero block. With a > 0 and
// positive midpoints m_8..m_14, this is
//   x >= 0 (or -0):  code = 8 + #{k : |x| >= a*m_{7+k}}
//   x <  0       :  code = 7 - #{k : |x| >= a*m_{7+k}}
// because a*m is never exactly a bf16 value (a has at most 8 significant bits, every
// nonzero m at least 21), so |x| <= a*m and |x| < a*m agree. a*m is exact in fp64;
// rounding it up to bf16 gives a boundary C_k with |x| >= a*m  <=>  |x| >= C_k for
// bf16 |x|, and on positive bf16 values that is an integer comparison of bit patterns.
// ---------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t nf4_code(uint32_t x16, const uint32_t (&C)[7]) {
  const uint32_t mag = x16 & 0x7FFFu;
  uint32_t cnt = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) cnt += (mag >= C[k]) ? 1u : 0u;
  const bool neg = (x16 & 0x8000u) && mag;
  return neg ? 7u - cnt : 8u + cnt;
}

__device__ __forceinline__ void load_block(const uint16_t* __restrict__ W, int64_t base,
                                           int64_t n, bool vec, uint32_t (&v)[32]) {
  if (vec) {
    const uint4* p = reinterpret_cast<const uint4*>(W + base);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint4 t = __ldg(p + i);
      v[4 * i + 0] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int64_t e = base + 2 * i;
      const uint32_t lo = e < n ? (uint32_t)W[e] : 0u;
      const uint32_t hi = e + 1 < n ? (uint32_t)W[e + 1] : 0u;
      v[i] = lo | (hi << 16);
    }
  }
}

__device__ __forceinline__ uint32_t block_absmax_bits(const uint32_t (&v)[32]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = max(m, max(v[i] & 0x7FFFu, (v[i] >> 16) & 0x7FFFu));
  return m;   // bf16 bits of max |x|; >= 0x7F80 means inf or NaN somewhere
}

__global__ void __launch_bounds__(256)
nf4_quantize_kernel(const uint16_t* __restrict__ W, int64_t n, uint8_t* __restrict__ codes,
                    float* __restrict__ absmax, const Nf4Tables tab, int vec_ok, int* flag) {
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const int64_t base = b * kBlock;
    const bool full = base + kBlock <= n;
    uint32_t v[32];
    load_block(W, base, n, vec_ok && full, v);
    const uint32_t amax = block_absmax_bits(v);
    if (amax >= 0x7F80u) raise_flag(flag, kFlagNonfinite);
    const float a = __uint_as_float(amax << 16);
    absmax[b] = a;
    uint32_t C[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      const double prod = (double)a * tab.mid_pos[k];            // exact
      const uint32_t fb = __float_as_uint(__double2float_ru(prod));
      C[k] = amax ? ((fb + 0xFFFFu) >> 16) : 0xFFFFu;           // ceil to bf16
    }
    uint32_t out[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t pair = v[4 * w + j];
        const uint32_t byte = nf4_code(pair & 0xFFFFu, C) | (nf4_code(pair >> 16, C) << 4);
        word |= byte << (8 * j);
      }
      out[w] = word;
    }
    if (vec_ok && full) {
      uint4* dst = reinterpret_cast<uint4*>(codes + b * 32);
      dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
      dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    } else {
      const int64_t cnt = imin64(kBlock, n - base);
      const int64_t nbytes = (cnt + 1) / 2;
      for (int i = 0; i < nbytes; ++i) {
        uint8_t byte = (uint8_t)(out[i / 4] >> (8 * (i % 4)));
        if (2 * i + 1 >= cnt) byte &= 0x0F;                  // no element: nibble 0
        codes[b * 32 + i] = byte;
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// Blockwise int8: sc = fp32(a/127); c = clamp(rint_half_even(fp32(x/sc)), -127, 127).
// ---------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t int8_code(uint32_t x16, float sc) {
  if (sc == 0.0f) return 0u;
  float t = rintf(__fdiv_rn(bf16_bits_to_float(x16), sc));
  t = fminf(fmaxf(t, -127.0f), 127.0f);
  return (uint32_t)((int32_t)t) & 0xFFu;
}

__global__ void __launch_bounds__(256)
int8_quantize_kernel(const uint16_t* __restrict__ W, int64_t n, int8_t* __restrict__ codes,
                     float* __restrict__ absmax, int vec_ok, int* flag) {
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const int64_t base = b * kBlock;
    const bool full = base + kBlock <= n;
    uint32_t v[32];
    load_block(W, base, n, vec_ok && full, v);
    const uint32_t amax = block_absmax_bits(v);
    if (amax >= 0x7F80u) raise_flag(flag, kFlagNonfinite);
    const float a = __uint_as_float(amax << 16);
    absmax[b] = a;
    const float sc = __fdiv_rn(a, 127.0f);
    uint32_t out[16];
#pragma unroll
    for (int w = 0; w < 16; ++w) {
      const uint32_t p0 = v[2 * w], p1 = v[2 * w + 1];
      out[w] = int8_code(p0 & 0xFFFFu, sc) | (int8_code(p0 >> 16, sc) << 8) |
               (int8_code(p1 & 0xFFFFu, sc) << 16) | (int8_code(p1 >> 16, sc) << 24);
    }
    if (vec_ok && full) {
      uint4* dst = reinterpret_cast<uint4*>(codes + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    } else {
      const int64_t cnt = imin64(64, n - base);
      for (int i = 0; i < cnt; ++i) codes[base + i] = (int8_t)(out[i / 4] >> (8 * (i % 4)));
    }
  }
}

// ---------------------------------------------------------------------------------
// Double quantisation.
//
// The mean needs the exact sum of the constants, rounded once to fp64. It is
// accumulated exactly and order-independently in integer bins: a finite v >= 0 is
// m * 2^(p - 149) with a 24-bit integer m and p in [0, 253]; it adds m << (p % 16)
// (< 2^39) to bin p / 16, whose weight is 2^(16 * bin - 149). With at most 2^24
// values a bin stays below 2^63, and integer addition is associative, so thread and
// atomic order cannot change the result.
// ---------------------------------------------------------------------------------

constexpr int kSumBins = 16;

__global__ void __launch_bounds__(256)
dq_sum_kernel(const float* __restrict__ absmax, int64_t nb, unsigned long long* bins, int* flag) {
  __shared__ unsigned long long part[8][kSumBins];
  unsigned long long acc[kSumBins];
#pragma unroll
  for (int i = 0; i < kSumBins; ++i) acc[i] = 0ull;
  bool bad = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const uint32_t u = __float_as_uint(absmax[b]);
    const uint32_t e = (u >> 23) & 0xFFu;
    if ((u >> 31) || e == 0xFFu) { bad = true; continue; }
    const uint32_t m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    const uint32_t p = (e ? e : 1u) - 1u;
    const unsigned long long c = (unsigned long long)m << (p & 15u);
    const uint32_t bin = p >> 4;
#pragma unroll
    for (int i = 0; i < kSumBins; ++i) acc[i] += (bin == (uint32_t)i) ? c : 0ull;
  }
  if (bad) raise_flag(flag, kFlagNonfinite);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kSumBins; ++i) {
    unsigned long long x = acc[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xFFFFFFFFu, x, off);
    if (lane == 0) part[warp][i] = x;
  }
  __syncthreads();
  if (threadIdx.x < kSumBins) {
    unsigned long long x = 0ull;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) x += part[w][threadIdx.x];
    if (x) atomicAdd(bins + threadIdx.x, x);
  }
}

// One thread: turn the bins into the exact integer X (value X * 2^-149), round it to
// fp64 (nearest, ties to even), and form mean = fp32(fp64(S) / nb).
__global__ void dq_finalize_kernel(const unsigned long long* __restrict__ bins, int64_t nb,
                                   float* __restrict__ mean) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  uint32_t limb[12];                                   // 384-bit little-endian integer
  for (int i = 0; i < 12; ++i) limb[i] = 0u;
  for (int i = 0; i < kSumBins; ++i) {
    const unsigned long long v = bins[i];
    const int bit = 16 * i;
    const int li = bit / 32;
    const unsigned long long lo = (bit % 32) ? (v << 16) : v;
    const uint32_t parts[3] = {(uint32_t)lo, (uint32_t)(lo >> 32), (bit % 32) ? (uint32_t)(v >> 48) : 0u};
    unsigned long long carry = 0;
    for (int k = 0; li + k < 12; ++k) {
      const unsigned long long sum = (unsigned long long)limb[li + k] + (k < 3 ? parts[k] : 0u) + carry;
      limb[li + k] = (uint32_t)sum;
      carry = sum >> 32;
      if (k >= 2 && carry == 0) break;
    }
  }
  int top = -1;
  for (int i = 11; i >= 0; --i)
    if (limb[i]) { top = i; break; }
  double S = 0.0;
  if (top >= 0) {
    // 96-bit window of limbs top, top-1, top-2 (missing limbs are zero)
    const uint32_t l1 = top >= 1 ? limb[top - 1] : 0u, l2 = top >= 2 ? limb[top - 2] : 0u;
    const unsigned __int128 W = ((unsigned __int128)limb[top] << 64) | ((unsigned __int128)l1 << 32) | l2;
    const int tb = 95 - __clz(limb[top]);              // top set bit inside W (>= 64)
    const int base = 32 * (top - 2);                   // weight of bit 0 of W
    if (base + tb < 53) {
      S = ldexp((double)(unsigned long long)(W >> (base < 0 ? -base : 0)), base > 0 ? base - 149 : -149);
    } else {
      unsigned long long mant = (unsigned long long)(W >> (tb - 52));
      const uint32_t rbit = (uint32_t)(W >> (tb - 53)) & 1u;
      bool sticky = (W & ((((unsigned __int128)1) << (tb - 53)) - 1)) != 0;
      for (int i = 0; i < top - 2 && !sticky; ++i) sticky = limb[i] != 0u;
      if (rbit && (sticky || (mant & 1ull))) mant += 1ull;
      S = ldexp((double)mant, base + tb - 52 - 149);   // exact scaling
    }
  }
  *mean = __double2float_rn(__ddiv_rn(S, (double)nb));
}

// One warp per group of 256 blocks.
__global__ void __launch_bounds__(256)
dq_encode_kernel(const float* __restrict__ absmax, int64_t nb, const float* __restrict__ mean,
                 int8_t* __restrict__ qabsmax, float* __restrict__ group_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float mu = *mean;
  for (int64_t g = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); g < ng; g += warps) {
    float d[8];
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kGroup + i * 32 + lane;
      d[i] = b < nb ? __fsub_rn(absmax[b], mu) : 0.0f;
      mx = fmaxf(mx, fabsf(d[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    const float s = __fdiv_rn(mx, 127.0f);
    if (lane == 0) group_scale[g] = s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kGroup + i * 32 + lane;
      if (b >= nb) continue;
      int8_t c = 0;
      if (s != 0.0f) {
        float t = rintf(__fdiv_rn(d[i], s));
        c = (int8_t)(int32_t)fminf(fmaxf(t, -127.0f), 127.0f);
      }
      qabsmax[b] = c;
    }
  }
}

// ---------------------------------------------------------------------------------
// Standalone dequantisation (checks only; the linear kernels decode on the fly).
// ---------------------------------------------------------------------------------

__global__ void __launch_bounds__(256)
dequant_nf4_kernel(const uint8_t* __restrict__ codes, const int8_t* __restrict__ qabsmax,
                   const float* __restrict__ gscale, const float* __restrict__ mean, int64_t n,
                   uint16_t* __restrict__ out, const Nf4Tables tab) {
  __shared__ float q[16];
  if (threadIdx.x < 16) q[threadIdx.x] = tab.q[threadIdx.x];
  __syncthreads();
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const float mu = *mean;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const float ar = __fadd_rn(__fmul_rn((float)qabsmax[b], gscale[b / kGroup]), mu);
    const int64_t base = b * kBlock;
    const int cnt = (int)imin64(kBlock, n - base);
    for (int j = 0; j < cnt; ++j) {
      const uint8_t byte = codes[(base + j) >> 1];
      const uint32_t c = ((base + j) & 1) ? (byte >> 4) : (byte & 0xF);
      out[base + j] = (uint16_t)float_to_bf16_bits(__fmul_rn(q[c], ar));
    }
  }
}

__global__ void __launch_bounds__(256)
dequant_int8_kernel(const int8_t* __restrict__ codes, const float* __restrict__ absmax, int64_t n,
                    uint16_t* __restrict__ out) {
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const float sc = __fdiv_rn(absmax[b], 127.0f);
    const int64_t base = b * kBlock;
    const int cnt = (int)imin64(kBlock, n - base);
    for (int j = 0; j < cnt; ++j)
      out[base + j] = (uint16_t)float_to_bf16_bits(__fmul_rn((float)codes[base + j], sc));
  }
}

static int grid_for(int64_t items, int threads) {
  const int64_t need = (items + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 16;
  return (int)imax64(1, imin64(need, cap));
}

}  // namespace qlb

using namespace qlb;

extern "C" {

ql_status nf4_quantize(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax, void* stream) {
  if (n < 0) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!W || !codes || !absmax) return QL_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(codes, 4) || !aligned(absmax, 4)) return QL_ERR_INVALID_ARG;
  const int vec = aligned(W, 16) && aligned(codes, 16);
  const int64_t nb = (n + kBlock - 1) / kBlock;
  ProfScope prof(PK_NF4, as_stream(stream), 1);
  nf4_quantize_kernel<<<grid_for(nb, 256), 256, 0, as_stream(stream)>>>(
      W, n, codes, absmax, nf4_tables(), vec, device_flag_ptr());
  QL_CHECK_LAUNCH();
  return QL_OK;
}

ql_status int8_quantize(const ql_bf16* W, int64_t n, int8_t* codes, float* absmax, void* stream) {
  if (n < 0) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!W || !codes || !absmax) return QL_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(absmax, 4)) return QL_ERR_INVALID_ARG;
  const int vec = aligned(W, 16) && aligned(codes, 16);
  const int64_t nb = (n + kBlock - 1) / kBlock;
  ProfScope prof(PK_INT8, as_stream(stream), 1);
  int8_quantize_kernel<<<grid_for(nb, 256), 256, 0, as_stream(stream)>>>(
      W, n, codes, absmax, vec, device_flag_ptr());
  QL_CHECK_LAUNCH();
  return QL_OK;
}

ql_status dq_quantize(const float* absmax, int64_t nblocks, int8_t* qabsmax, float* group_scale,
                      float* mean, void* ws, size_t ws_bytes, void* stream) {
  if (nblocks < 1 || !absmax || !qabsmax || !group_scale || !mean || !ws) return QL_ERR_INVALID_ARG;
  if (nblocks > (int64_t(1) << 24)) return QL_ERR_UNSUPPORTED;
  if (!aligned(absmax, 4) || !aligned(group_scale, 4) || !aligned(mean, 4) || !aligned(ws, 16))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0)) return QL_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  unsigned long long* bins = static_cast<unsigned long long*>(ws);
  ProfScope prof(PK_DQ, st, 3);
  if (cudaMemsetAsync(bins, 0, kSumBins * sizeof(unsigned long long), st) != cudaSuccess)
    return QL_ERR_CUDA;
  dq_sum_kernel<<<(int)imin64((nblocks + 255) / 256, num_sms()), 256, 0, st>>>(absmax, nblocks, bins,
                                                                              device_flag_ptr());
  QL_CHECK_LAUNCH();
  dq_finalize_kernel<<<1, 32, 0, st>>>(bins, nblocks, mean);
  QL_CHECK_LAUNCH();
  const int64_t ng = (nblocks + kGroup - 1) / kGroup;
  dq_encode_kernel<<<grid_for(ng * 32, 256), 256, 0, st>>>(absmax, nblocks, mean, qabsmax, group_scale);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

ql_status ql_dequantize(const ql_weight* w, ql_bf16* Wout, void* stream) {
  if (!w || !Wout || w->N < 1 || w->K < 1 || !w->codes) return QL_ERR_INVALID_ARG;
  const int64_t n = w->N * w->K;
  const int64_t nb = (n + kBlock - 1) / kBlock;
  cudaStream_t st = as_stream(stream);
  ProfScope prof(PK_DEQ, st, 1);
  if (w->fmt == QL_FMT_NF4_DQ) {
    if (!w->qabsmax || !w->group_scale || !w->mean) return QL_ERR_INVALID_ARG;
    dequant_nf4_kernel<<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const uint8_t*>(w->codes), w->qabsmax, w->group_scale, w->mean, n, Wout,
        nf4_tables());
  } else if (w->fmt == QL_FMT_INT8_B64) {
    if (!w->absmax) return QL_ERR_INVALID_ARG;
    dequant_int8_kernel<<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const int8_t*>(w->codes), w->absmax, n, Wout);
  } else {
    return QL_ERR_INVALID_ARG;
  }
  QL_CHECK_LAUNCH();
  return QL_OK;
}

}  // extern "C"
