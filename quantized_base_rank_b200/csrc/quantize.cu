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
// bf16 |x|, an exact bf16 comparison done for two elements per instruction.
// ---------------------------------------------------------------------------------

// Two elements at a time in bf16x2 arithmetic: every value involved (the compare results
// 0/1, counts up to 7, codes up to 15, 128 + code) is a small integer, exact in bf16.
__device__ __forceinline__ uint32_t bf2_set_ge(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_set_lt(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.lt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_add(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Codes of the two elements of one bf16x2 word, as one byte (element 0 in the low
// nibble). Cp[k] holds the boundary C_k in both halves.
//   acc  = 8 + #{k : |x| >= C_k}                       (the code of a non-negative x)
//   code = acc + neg * (15 - 2 acc)  = 7 - #{...} when x < 0 (strictly; -0 is not)
__device__ __forceinline__ uint32_t nf4_code_pair(uint32_t w, const uint32_t (&Cp)[7]) {
  constexpr uint32_t kOne8 = 0x41004100u;        // 8.0, 8.0
  const uint32_t ax = w & 0x7FFF7FFFu;           // |x|, |x|
  uint32_t acc = bf2_add(kOne8, bf2_set_ge(ax, Cp[0]));
#pragma unroll
  for (int k = 1; k < 7; ++k) acc = bf2_add(acc, bf2_set_ge(ax, Cp[k]));
  const uint32_t neg = bf2_set_lt(w, 0u);                           // 1.0 where x < 0
  const uint32_t t = bf2_fma(acc, 0xC000C000u /* -2 */, 0x41704170u /* 15 */);
  const uint32_t code = bf2_fma(neg, t, acc);                        // 0..15
  const uint32_t r = bf2_add(code, 0x43004300u /* 128 */);           // bits 0x4300 | code
  return (r & 0xFu) | ((r >> 12) & 0xF0u);
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
  uint32_t m = 0;                                 // two 16-bit lanes of |x| bit patterns
#pragma unroll
  for (int i = 0; i < 32; ++i) m = __vmaxu2(m, v[i] & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);   // bf16 bits of max |x|; >= 0x7F80 means inf or NaN somewhere
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
    uint32_t Cp[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      const double prod = (double)a * tab.mid_pos[k];            // exact
      const uint32_t fb = __float_as_uint(__double2float_ru(prod));
      const uint32_t c = amax ? ((fb + 0xFFFFu) >> 16) : 0x7FC0u;   // ceil to bf16 (NaN: never >=)
      Cp[k] = c | (c << 16);
    }
    uint32_t out[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) word |= nf4_code_pair(v[4 * w + j], Cp) << (8 * j);
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

// Turn the bins into the exact integer X (value X * 2^-149), round it to fp64 (nearest,
// ties to even), and return mean = fp32(fp64(S) / nb). One thread's work.
__device__ float dq_mean_from_bins(const unsigned long long* __restrict__ bins, int64_t nb) {
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
  return __double2float_rn(__ddiv_rn(S, (double)nb));
}

// One warp per group of 256 blocks. Every CTA first rounds the exact sum to the mean
// itself (a few hundred instructions on one thread), so no separate launch is needed;
// CTA 0 also stores it.
__global__ void __launch_bounds__(256)
dq_encode_kernel(const float* __restrict__ absmax, int64_t nb, const unsigned long long* __restrict__ bins,
                 float* __restrict__ mean, int8_t* __restrict__ qabsmax, float* __restrict__ group_scale) {
  __shared__ float s_mu;
  if (threadIdx.x == 0) {
    s_mu = dq_mean_from_bins(bins, nb);
    if (blockIdx.x == 0) *mean = s_mu;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float mu = s_mu;
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
  ProfScope prof(PK_DQ, st, 2);
  if (cudaMemsetAsync(bins, 0, kSumBins * sizeof(unsigned long long), st) != cudaSuccess)
    return QL_ERR_CUDA;
  dq_sum_kernel<<<(int)imin64((nblocks + 255) / 256, num_sms()), 256, 0, st>>>(absmax, nblocks, bins,
                                                                              device_flag_ptr());
  QL_CHECK_LAUNCH();
  const int64_t ng = (nblocks + kGroup - 1) / kGroup;
  dq_encode_kernel<<<grid_for(ng * 32, 256), 256, 0, st>>>(absmax, nblocks, bins, mean, qabsmax, group_scale);
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
