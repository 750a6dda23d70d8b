// Quantisation kernels: NF4 encode with blockwise absmax, double quantisation of the
// absmax constants, blockwise int8, and standalone dequantisation.
//
// QLoRA page (aizip.shop/methodologies/qlora): "1. 4-bit NormalFloat (NF4)" defines the
// quantile grid; "2. Double Quantization" the block size 64 and the re-quantised
// constants. The int8 format is the 8-bit option of AutoQRA's per-layer bit-width
// (gist.science/ko/paper/2602.22268, section 3.1).
//
// All of these are HBM-bound streaming passes. The decision data of a block (its absmax
// and boundaries) lives in registers and nothing is staged.
#include <math.h>

#include <algorithm>
#include <vector>

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

// Packed compares that return masks: 0xFFFF in each half where the comparison holds.
__device__ __forceinline__ uint32_t bf2_ge_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_lt_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.lt.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// m ? a : b, bit by bit (one LOP3)
__device__ __forceinline__ uint32_t bit_select(uint32_t m, uint32_t a, uint32_t b) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xCA;" : "=r"(d) : "r"(m), "r"(a), "r"(b));
  return d;
}
// (a & b) ^ c (one LOP3)
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Codes of the two elements of one bf16x2 word, each in the low nibble of its half (the
// rest of the half zero). Cp[k] holds the boundary C_{k+1} in both halves, C_1 < ... < C_7.
// cnt = #{k : |x| >= C_k} by a three-step binary search over the sorted boundaries (three
// packed compares; the next boundary is chosen by bit selects), then
//   code = 8 + cnt = 8 ^ cnt  for x >= 0 (and -0),   7 - cnt = 7 ^ cnt  for x < 0.
// A zero block has NaN boundaries, which no compare passes: cnt = 0 and every code is 8.
__device__ __forceinline__ uint32_t nf4_code_pair(uint32_t w, const uint32_t (&Cp)[7]) {
  const uint32_t ax = w & 0x7FFF7FFFu;                       // |x|, |x|
  const uint32_t f1 = bf2_ge_mask(ax, Cp[3]);               // cnt >= 4
  const uint32_t t2 = bit_select(f1, Cp[5], Cp[1]);
  const uint32_t u = bit_select(f1, Cp[6], Cp[2]);
  const uint32_t v = bit_select(f1, Cp[4], Cp[0]);
  const uint32_t f2 = bf2_ge_mask(ax, t2);                  // the next bit of cnt
  const uint32_t f3 = bf2_ge_mask(ax, bit_select(f2, u, v));
  // bit 2 from f1, bit 1 from f2, bit 0 from f3 (higher bits hold copies, masked below)
  const uint32_t cnt = bit_select(0x00060006u, bit_select(0x00040004u, f1, f2), f3);
  const uint32_t base = and_xor(bf2_lt_mask(w, 0u), 0x000F000Fu, 0x00080008u);   // 7 if x < 0, else 8
  return and_xor(cnt, 0x00070007u, base);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Eight codes (four nf4_code_pair results, elements in order) -> one 32-bit word of
// nibbles, element i in bits 4i..4i+3. The low byte of each half holds a code.
__device__ __forceinline__ uint32_t nf4_pack8(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  const uint32_t t0 = prmt(r0, r1, 0x6420u);      // bytes: c0 c1 c2 c3
  const uint32_t t1 = prmt(r2, r3, 0x6420u);      // bytes: c4 c5 c6 c7
  // t + (t >> 4) == t | (t >> 4) (no overlapping bits): byte 0 = c0 | c1 << 4 and byte 2 =
  // c2 | c3 << 4; one multiply-add on the FMA pipe instead of a shift and an OR
  uint32_t y0, y1;
  asm("mad.hi.u32 %0, %1, 0x10000000, %1;" : "=r"(y0) : "r"(t0));
  asm("mad.hi.u32 %0, %1, 0x10000000, %1;" : "=r"(y1) : "r"(t1));
  return prmt(y0, y1, 0x6420u);
}

// The seven boundaries C_k = ceil_bf16(a * m_{8+k}) of a block with absmax bits `amax`
// (sign clear), in both halves of Cp[k]. Normal absmax with biased exponent >= 5 come
// from the shared-memory copy of the [1, 2) table plus an exponent shift (every boundary
// then stays normal); zero, subnormal, tiny and non-finite absmax take the fp64 product.
// A zero block gets NaN boundaries, which no comparison passes: every code is 8.
__device__ __forceinline__ void nf4_boundaries(uint32_t amax, const uint32_t* s_tab, const Nf4Tables& tab,
                                               uint32_t (&Cp)[7]) {
  const uint32_t e = amax >> 7;
  if (e >= 5u && e <= 254u) {
    const uint4* row = reinterpret_cast<const uint4*>(s_tab + (amax & 0x7Fu) * 8);
    const uint4 lo = row[0], hi = row[1];
    const uint32_t d = (uint32_t)(((int32_t)e - 127) * 128) * 0x10001u;
    Cp[0] = lo.x + d; Cp[1] = lo.y + d; Cp[2] = lo.z + d; Cp[3] = lo.w + d;
    Cp[4] = hi.x + d; Cp[5] = hi.y + d; Cp[6] = hi.z + d;
  } else {
    const float a = __uint_as_float(amax << 16);
#pragma unroll
    for (int k = 0; k < 7; ++k) {
      const double prod = (double)a * tab.mid_pos[k];            // exact
      const uint32_t fb = __float_as_uint(__double2float_ru(prod));
      const uint32_t c = amax ? ((fb + 0xFFFFu) >> 16) : 0x7FC0u;   // ceil to bf16 (NaN: never >=)
      Cp[k] = c | (c << 16);
    }
  }
}

// ---------------------------------------------------------------------------------
// Integer codes clamp(rint_half_even(fp32(x / sc)), -127, 127), shared by the blockwise
// int8 format and the double-quantised constants. The quotient comes from the reciprocal
// r = fp32(1/sc) and one residual correction (Markstein's method: q0 = x r, e = x - q0 sc
// exactly by FMA, q = q0 + e r rounded once), the correctly rounded quotient when nothing
// under- or overflows; scales below 2^-100 take the IEEE division. Rounding to an integer,
// half to even, is one add of 1.5 * 2^23, after which the low byte of the sum's bits is the
// code in two's complement.
// ---------------------------------------------------------------------------------

constexpr float kInt8FastMinScale = 7.888609052210118e-31f;   // 2^-100
constexpr float kRoundMagic = 12582912.0f;                     // 1.5 * 2^23

// Code byte (low 8 bits) of the element x given the block scale.
__device__ __forceinline__ uint32_t int8_byte(float x, float sc, float r, bool fast) {
  float q;
  if (fast) {
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q0, sc, x);
    q = __fmaf_rn(e, r, q0);
  } else {
    q = sc == 0.0f ? 0.0f : __fdiv_rn(x, sc);
  }
  return __float_as_uint(__fadd_rn(fminf(fmaxf(q, -127.0f), 127.0f), kRoundMagic));
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

// One constant's term of the exact sum, from its fp32 bits u: the bin and the integer
// added to it. A negative, infinite or NaN constant is left out (c = 0) and sets `bad`.
__device__ __forceinline__ void dq_term(uint32_t u, uint32_t& bin, unsigned long long& c, bool& bad) {
  const uint32_t e = (u >> 23) & 0xFFu;
  const bool ok = !(u >> 31) && e != 0xFFu;
  bad |= !ok;
  const uint32_t m = ok ? ((u & 0x7FFFFFu) | (e ? 0x800000u : 0u)) : 0u;
  const uint32_t p = (e ? e : 1u) - 1u;
  c = (unsigned long long)m << (p & 15u);
  bin = p >> 4;
}

// Adds one group of lanes' terms (all lanes whose `bin` equals the leader's) into the
// warp's shared bins. A lane's value c < 2^63 (a running sum of terms below 2^39) is split
// into 27-bit parts so that no 32-bit warp sum can wrap (32 * 2^27 = 2^32).
__device__ __forceinline__ void bins_warp_add(unsigned long long* wbins, uint32_t bin, unsigned long long c,
                                              int lane) {
  uint32_t pending = __ballot_sync(0xFFFFFFFFu, c != 0ull);
  while (pending) {                                   // one pass per distinct bin (<= 16)
    const int leader = __ffs(pending) - 1;
    const uint32_t lb = __shfl_sync(0xFFFFFFFFu, bin, leader);
    const bool mine = c != 0ull && bin == lb;
    constexpr unsigned long long kPart = (1ull << 27) - 1ull;
    const uint32_t p0 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)(c & kPart) : 0u);
    const uint32_t p1 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)((c >> 27) & kPart) : 0u);
    const uint32_t p2 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)(c >> 54) : 0u);
    if (lane == 0)
      wbins[lb] += (unsigned long long)p0 + ((unsigned long long)p1 << 27) + ((unsigned long long)p2 << 54);
    pending &= ~__ballot_sync(0xFFFFFFFFu, mine);
  }
}

// Turn the bins into the exact integer X (value X * 2^-149), round it to fp64 (nearest,
// ties to even), and return mean = fp32(fp64(S) / nb). One thread's work. Every array
// index is a compile-time constant (the loops are unrolled), so the big integer stays in
// registers: X < 16 * 2^63 * 2^240 = 2^307 fits five 64-bit limbs.
__device__ float dq_mean_from_bins(const unsigned long long (&bins)[16], int64_t nb) {
  unsigned __int128 acc[6] = {0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < kSumBins; ++i) {                // bin i has weight 2^(16 i)
    const unsigned __int128 v = (unsigned __int128)bins[i] << (16 * (i % 4));   // < 2^111
    acc[i / 4] += (unsigned long long)v;
    acc[i / 4 + 1] += (unsigned long long)(v >> 64);
  }
  unsigned long long limb[6];
#pragma unroll
  for (int j = 0; j < 6; ++j) {                       // each acc < 2^67 before its carry-in
    limb[j] = (unsigned long long)acc[j];
    if (j < 5) acc[j + 1] += acc[j] >> 64;
  }
  int top = -1;
#pragma unroll
  for (int j = 0; j < 6; ++j)
    if (limb[j]) top = j;
  double S = 0.0;
  if (top == 0) {
    S = ldexp(__ull2double_rn(limb[0]), -149);        // one rounding of a 64-bit integer
  } else if (top > 0) {
    // the 128-bit window of limbs top and top - 1, and whether anything below it is set
    unsigned long long hi = 0, lo = 0;
    bool sticky = false;
#pragma unroll
    for (int j = 0; j < 6; ++j) {
      if (j == top) hi = limb[j];
      if (j == top - 1) lo = limb[j];
      if (j < top - 1 && limb[j]) sticky = true;
    }
    const unsigned __int128 W = ((unsigned __int128)hi << 64) | lo;
    const int tb = 127 - __clzll((long long)hi);     // top set bit of W, >= 64
    unsigned long long mant = (unsigned long long)(W >> (tb - 52));
    const unsigned rbit = (unsigned)(W >> (tb - 53)) & 1u;
    sticky = sticky || (W & ((((unsigned __int128)1) << (tb - 53)) - 1)) != 0;
    if (rbit && (sticky || (mant & 1ull))) mant += 1ull;
    S = ldexp((double)mant, 64 * (top - 1) + tb - 52 - 149);   // exact scaling
  }
  return __double2float_rn(__ddiv_rn(S, (double)nb));
}

// End of the exact sum for one CTA (every thread calls it): the per-warp bins are
// combined, added to the global bins (one atomic per non-empty bin), and the CTA takes a
// ticket. The CTA that takes the last of `ctas` tickets (counted over every launch that
// shares the bins) rounds the sum and writes the mean, or, with bins_out (one shard of a
// weight split across ranks), copies the shard's exact bins out instead. No CTA waits
// for another. ws: bins[16], then the ticket counter; zeroed before the first launch.
__device__ __forceinline__ bool dq_bins_finish(unsigned long long (*s_bins)[kSumBins], int nwarps,
                                               unsigned long long* ws, unsigned int ctas, int64_t nb,
                                               float* mean, unsigned long long* bins_out) {
  __shared__ int s_last;
  __syncthreads();
  unsigned int* ticket = reinterpret_cast<unsigned int*>(ws + kSumBins);
  if (threadIdx.x < kSumBins) {
    unsigned long long x = 0ull;
    for (int w = 0; w < nwarps; ++w) x += s_bins[w][threadIdx.x];
    if (x) atomicAdd(ws + threadIdx.x, x);
    __threadfence();                                  // the bin atomics before the ticket
  }
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == ctas - 1;
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    unsigned long long v[kSumBins];
#pragma unroll
    for (int i = 0; i < kSumBins; ++i) v[i] = __ldcg(ws + i);
    if (bins_out) {
      for (int i = 0; i < kSumBins; ++i) bins_out[i] = v[i];
    } else {
      *mean = dq_mean_from_bins(v, nb);
    }
  }
  return s_last != 0;
}

// The mean from bins summed over the shards of a weight: one thread.
__global__ void dq_mean_kernel(const unsigned long long* __restrict__ bins, int64_t nb_total, float* mean) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  unsigned long long v[kSumBins];
#pragma unroll
  for (int i = 0; i < kSumBins; ++i) v[i] = bins[i];
  *mean = dq_mean_from_bins(v, nb_total);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One group of 256 constants by one warp: d = a - mean, s_g = max|d| / 127, code =
// clamp(rint(d / s_g)). CG: read the constants from L2 (they were written by other CTAs
// of the same grid).
template <bool CG>
__device__ __forceinline__ void dq_encode_group(const float* __restrict__ absmax, int64_t nb, float mu,
                                                int8_t* __restrict__ qabsmax, float* __restrict__ group_scale,
                                                int64_t g, int lane) {
  {
    float d[8];
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kGroup + i * 32 + lane;
      d[i] = b < nb ? __fsub_rn(CG ? __ldcg(absmax + b) : absmax[b], mu) : 0.0f;
      mx = fmaxf(mx, fabsf(d[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    const float s = __fdiv_rn(mx, 127.0f);
    if (lane == 0) group_scale[g] = s;
    const bool fast = s >= kInt8FastMinScale && s < 3.0e38f;
    const float r = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kGroup + i * 32 + lane;
      if (b >= nb) continue;
      qabsmax[b] = (int8_t)int8_byte(d[i], s, r, fast);
    }
  }
}

// Groups g[0..G-1] (a value >= ng is skipped) by one warp, as dq_encode_group<true>, with
// the loads of every group issued before any is used, so their round trips to L2 overlap.
template <int G>
__device__ __forceinline__ void dq_encode_groups_cg(const float* __restrict__ absmax, int64_t nb, float mu,
                                                    int8_t* __restrict__ qabsmax, float* __restrict__ group_scale,
                                                    const int64_t (&g)[G], int lane) {
  float d[G][8];
#pragma unroll
  for (int j = 0; j < G; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g[j] * kGroup + i * 32 + lane;
      d[j][i] = b < nb ? __ldcg(absmax + b) : mu;     // a value past the end gives d = 0
    }
#pragma unroll
  for (int j = 0; j < G; ++j) {
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      d[j][i] = __fsub_rn(d[j][i], mu);
      mx = fmaxf(mx, fabsf(d[j][i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    const float s = __fdiv_rn(mx, 127.0f);
    const int64_t ng = (nb + kGroup - 1) / kGroup;
    if (g[j] >= ng) continue;                        // warp-uniform
    if (lane == 0) group_scale[g[j]] = s;
    const bool fast = s >= kInt8FastMinScale && s < 3.0e38f;
    const float r = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g[j] * kGroup + i * 32 + lane;
      if (b >= nb) continue;
      qabsmax[b] = (int8_t)int8_byte(d[j][i], s, r, fast);
    }
  }
}

// NF4 encode kernel. One lane per block of 64 elements (128 bytes in, 32 bytes of codes
// out); the grid is persistent and the loop warp-uniform, so every lane takes part in the
// warp collectives. VEC = true covers whole blocks with 16-byte aligned input and codes,
// and each lane loads its next block while it encodes the current one; VEC = false (a
// ragged last block, or unaligned pointers) goes element by element with bounds checks.
// DQ = true also accumulates the exact sum of the block constants for double
// quantisation: each lane keeps a running sum for one bin of the exact integer sum (the
// constants of a weight rarely span more than one bin of 16 binades) and the warp adds it
// into its shared bins only when some lane's bin changes, and at the end (dq_bins_finish).
constexpr int kNf4Threads = 256;
constexpr uint64_t kDqWaitNs = 2000000000ull;   // bound of the fused quantise's wait for the mean

__device__ __forceinline__ uint64_t qt_globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
constexpr int kNf4Warps = kNf4Threads / 32;

struct Nf4Args {
  const uint16_t* W;
  int64_t n, blk_begin, blk_end;
  uint8_t* codes;
  float* absmax;
  int* flag;
  unsigned long long* dq_ws;   // DQ: bins + ticket
  float* mean;                 // DQ: output
  unsigned long long* bins_out;  // DQ, one shard: its exact bins instead of the mean
  unsigned int dq_ctas;        // DQ: CTAs over all launches sharing the bins
  int64_t nb_total;            // DQ: number of constants
  int8_t* qabsmax;             // FUSED: the DQ codes
  float* group_scale;          // FUSED: the group scales
};

__device__ __forceinline__ void nf4_load_vec(const uint16_t* __restrict__ W, int64_t base, bool live,
                                             uint4 (&x)[4]) {
  if (live) {
    const uint4* src = reinterpret_cast<const uint4*>(W + base);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __ldg(src + i);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// FUSED (a cooperative launch of the single whole-block VEC grid, with DQ): after the
// exact sum, the last CTA publishes the mean through a ready flag in the workspace; every
// CTA waits for it (bounded by globaltimer; all CTAs are co-resident by the cooperative
// launch) and the grid's warps then encode the groups of 256 constants, so no second
// launch is needed. The constants written by other CTAs are read from L2.
template <bool VEC, bool DQ, bool FUSED = false>
__global__ void __launch_bounds__(kNf4Threads, VEC ? 2 : 1)
nf4_quantize_kernel(const Nf4Args args, const Nf4Tables tab, const Nf4BoundTable btab) {
  __shared__ __align__(16) uint32_t s_tab[128 * 8];
  __shared__ unsigned long long s_bins[DQ ? kNf4Warps : 1][kSumBins];
  for (int i = threadIdx.x; i < 128 * 8 / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(s_tab)[i] = reinterpret_cast<const uint4*>(&btab.c[0][0])[i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (DQ) {
    if (lane < kSumBins) s_bins[warp][lane] = 0ull;
    if (!FUSED) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  __syncthreads();

  const uint16_t* __restrict__ W = args.W;
  const int64_t n = args.n;
  const int64_t nblk = args.blk_end - args.blk_begin;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  bool bad = false;
  uint32_t lbin = 0;                                  // DQ: this lane's running bin and sum
  unsigned long long lsum = 0ull;
  int64_t w0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  uint4 nx[8];
  if (VEC) {
    const int64_t it = w0 + lane;
    if (it < nblk) {
      const uint4* src = reinterpret_cast<const uint4*>(W + (args.blk_begin + it) * kBlock);
#pragma unroll
      for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
    }
  }
  for (; w0 < nblk; w0 += stride) {
    const int64_t it = w0 + lane;
    const bool live = it < nblk;
    const int64_t b = args.blk_begin + it;
    const int64_t base = b * kBlock;
    uint32_t v[32];
    if (VEC) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[4 * i + 0] = nx[i].x; v[4 * i + 1] = nx[i].y; v[4 * i + 2] = nx[i].z; v[4 * i + 3] = nx[i].w;
      }
      if (it + stride < nblk) {                        // this lane's next block
        const uint4* src = reinterpret_cast<const uint4*>(W + (b + stride) * kBlock);
#pragma unroll
        for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int64_t e = base + 2 * i;
        const uint32_t lo = live && e < n ? (uint32_t)W[e] : 0u;
        const uint32_t hi = live && e + 1 < n ? (uint32_t)W[e + 1] : 0u;
        v[i] = lo | (hi << 16);
      }
    }
    // two 16-bit lanes of max |x| by packed bf16 max (NaN-propagating; the sign bits of the
    // running value are meaningless and cleared after the loop): for non-NaN values the
    // order of |x| is the order of its bit patterns, so this is the bitwise maximum
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(m), "r"(v[i]));
    m &= 0x7FFF7FFFu;
    const uint32_t amax = max(m & 0xFFFFu, m >> 16);   // bf16 bits of the block's max |x|
    if (live) {
      if (amax >= 0x7F80u) raise_flag(args.flag, kFlagNonfinite);
      args.absmax[b] = __uint_as_float(amax << 16);
    }
    if (DQ) {
      uint32_t bin = 0;
      unsigned long long c = 0ull;
      if (live) dq_term(amax << 16, bin, c, bad);
      const bool move = c != 0ull && bin != lbin && lsum != 0ull;
      if (__any_sync(0xFFFFFFFFu, move)) {           // some lane changes bin: flush the old sums
        bins_warp_add(s_bins[warp], lbin, move ? lsum : 0ull, lane);
        if (move) lsum = 0ull;
      }
      if (c != 0ull) {
        lbin = bin;
        lsum += c;                                      // < 2^63: at most 2^24 terms below 2^39
      }
    }
    uint32_t Cp[7];
    nf4_boundaries(amax, s_tab, tab, Cp);
    uint32_t out[8];
#pragma unroll
    for (int w = 0; w < 8; ++w)
      out[w] = nf4_pack8(nf4_code_pair(v[4 * w + 0], Cp), nf4_code_pair(v[4 * w + 1], Cp),
                         nf4_code_pair(v[4 * w + 2], Cp), nf4_code_pair(v[4 * w + 3], Cp));
    uint8_t* dst = args.codes + b * 32;
    if (VEC) {
      if (live) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4*>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
      }
    } else if (live) {
      const int64_t cnt = imin64(64, n - base);        // elements of this block
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (2 * i >= cnt) break;
        uint8_t byte = (uint8_t)(out[i / 4] >> (8 * (i % 4)));
        if (2 * i + 1 >= cnt) byte &= 0x0F;              // no element: nibble 0
        dst[i] = byte;
      }
    }
  }
  if (DQ) {
    (void)bad;                                         // a non-finite absmax already raised the flag
    bins_warp_add(s_bins[warp], lbin, lsum, lane);
    const bool last =
        dq_bins_finish(s_bins, kNf4Warps, args.dq_ws, args.dq_ctas, args.nb_total, args.mean, args.bins_out);
    if (FUSED) {
      // the ready word: 1 in the low half once the mean is written, the mean's bits in the
      // high half, so the waiting CTAs get the mean with the same acquire load
      __shared__ int s_ok;
      __shared__ float s_mu;
      unsigned long long* ready = args.dq_ws + kSumBins + 1;
      if (threadIdx.x == 0) {
        if (last) {
          const unsigned long long word = 1ull | ((unsigned long long)__float_as_uint(*args.mean) << 32);
          asm volatile("st.release.gpu.global.u64 [%0], %1;" :: "l"(ready), "l"(word) : "memory");
        }
        unsigned long long v = 0ull;
        const uint64_t t0 = qt_globaltimer_ns();
        for (;;) {
          asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ready) : "memory");
          if ((v & 1ull) || qt_globaltimer_ns() - t0 > kDqWaitNs) break;
          __nanosleep(64);
        }
        s_ok = (v & 1ull) != 0ull;
        s_mu = __uint_as_float((uint32_t)(v >> 32));
        if (!s_ok) raise_flag(args.flag, kFlagTimeout);
      }
      __syncthreads();
      if (!s_ok) return;
      const float mu = s_mu;
      const int64_t ng = (args.nb_total + kGroup - 1) / kGroup;
      const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
      for (int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < ng; g += 2 * warps) {
        const int64_t gg[2] = {g, g + warps};
        dq_encode_groups_cg<2>(args.absmax, args.nb_total, mu, args.qabsmax, args.group_scale, gg, lane);
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// Blockwise int8: sc = fp32(a/127); c = clamp(rint_half_even(fp32(x/sc)), -127, 127).
//
// One lane per block of 64 elements. The quotient fp32(x/sc) is formed from the block's
// reciprocal r = fp32(1/sc) with one residual correction (Markstein's method: q0 = x r,
// e = x - q0 sc exactly by FMA, q = q0 + e r rounded once), which yields the correctly
// rounded quotient when nothing under- or overflows; blocks whose scale is below 2^-100
// take the IEEE division instead. Rounding to an integer, half to even, is one add of
// 1.5 * 2^23, after which the low byte of the sum's bits is the code in two's complement.
// All of it runs on the FMA pipe except the bf16 unpacking and the byte packing.
// ---------------------------------------------------------------------------------

// Four elements in two bf16x2 words -> one word of four code bytes, element order kept.
__device__ __forceinline__ uint32_t int8_word(uint32_t p0, uint32_t p1, float sc, float r, bool fast) {
  const uint32_t b0 = int8_byte(__uint_as_float(p0 << 16), sc, r, fast);
  const uint32_t b1 = int8_byte(__uint_as_float(p0 & 0xFFFF0000u), sc, r, fast);
  const uint32_t b2 = int8_byte(__uint_as_float(p1 << 16), sc, r, fast);
  const uint32_t b3 = int8_byte(__uint_as_float(p1 & 0xFFFF0000u), sc, r, fast);
  return __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u);
}

// VEC: whole blocks, 16-byte aligned W and codes; each lane loads its next block while it
// encodes the current one. Otherwise element loads with bounds checks (a ragged last
// block, or unaligned pointers).
template <bool VEC>
__global__ void __launch_bounds__(256)
int8_quantize_kernel(const uint16_t* __restrict__ W, int64_t n, int64_t nb, int8_t* __restrict__ codes,
                     float* __restrict__ absmax, int* flag) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint4 nx[8];
  if (VEC && b < nb) {
    const uint4* src = reinterpret_cast<const uint4*>(W + b * kBlock);
#pragma unroll
    for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
  }
  for (; b < nb; b += stride) {
    uint32_t v[32];
    const int64_t base = b * kBlock;
    if (VEC) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[4 * i] = nx[i].x; v[4 * i + 1] = nx[i].y; v[4 * i + 2] = nx[i].z; v[4 * i + 3] = nx[i].w;
      }
      if (b + stride < nb) {
        const uint4* src = reinterpret_cast<const uint4*>(W + (b + stride) * kBlock);
#pragma unroll
        for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
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
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(m), "r"(v[i]));
    m &= 0x7FFF7FFFu;
    const uint32_t amax = max(m & 0xFFFFu, m >> 16);
    if (amax >= 0x7F80u) raise_flag(flag, kFlagNonfinite);
    const float a = __uint_as_float(amax << 16);
    absmax[b] = a;
    const float sc = __fdiv_rn(a, 127.0f);
    const bool fast = sc >= kInt8FastMinScale && sc < 3.0e38f;
    const float r = fast ? __frcp_rn(sc) : 0.0f;
    uint32_t out[16];
#pragma unroll
    for (int w = 0; w < 16; ++w) out[w] = int8_word(v[2 * w], v[2 * w + 1], sc, r, fast);
    if (VEC) {
      uint4* dst = reinterpret_cast<uint4*>(codes + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    } else {
      const int64_t cnt = imin64(64, n - base);
      for (int i = 0; i < cnt; ++i) codes[base + i] = (int8_t)(out[i / 4] >> (8 * (i % 4)));
    }
  }
}

// Exact integer-bin sum of an array of constants (dq_quantize). Each thread reads
// kSumPerThread constants; a lane whose constants share one bin adds them first, and a
// warp whose lanes all use one bin needs one pass of bins_warp_add.
constexpr int kSumThreads = 256;
constexpr int kSumPerThread = 8;          // constants per thread (two 16-byte loads)

__global__ void __launch_bounds__(kSumThreads)
dq_sum_kernel(const float* __restrict__ absmax, int64_t nb, unsigned long long* ws, float* mean, int vec,
              int* flag) {
  __shared__ unsigned long long s_bins[kSumThreads / 32][kSumBins];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < kSumBins) s_bins[warp][lane] = 0ull;
  __syncwarp();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  bool bad = false;
  const int64_t chunk = (int64_t)kSumThreads * kSumPerThread;
  for (int64_t c0 = (int64_t)blockIdx.x * chunk; c0 < nb; c0 += (int64_t)gridDim.x * chunk) {
    const int64_t i0 = c0 + (int64_t)threadIdx.x * kSumPerThread;
    uint32_t u[kSumPerThread];
    if (vec && i0 + kSumPerThread <= nb) {
      const uint4* src = reinterpret_cast<const uint4*>(absmax + i0);
      const uint4 x = __ldg(src), y = __ldg(src + 1);
      u[0] = x.x; u[1] = x.y; u[2] = x.z; u[3] = x.w; u[4] = y.x; u[5] = y.y; u[6] = y.z; u[7] = y.w;
    } else {
#pragma unroll
      for (int k = 0; k < kSumPerThread; ++k) u[k] = i0 + k < nb ? __float_as_uint(absmax[i0 + k]) : 0u;
    }
    uint32_t bin[kSumPerThread];
    unsigned long long c[kSumPerThread];
#pragma unroll
    for (int k = 0; k < kSumPerThread; ++k) dq_term(u[k], bin[k], c[k], bad);
    // lane-level merge when every non-zero term of the lane falls in one bin
    uint32_t b0 = 0u;
    bool have = false;
#pragma unroll
    for (int k = 0; k < kSumPerThread; ++k)
      if (c[k] != 0ull && !have) { b0 = bin[k]; have = true; }
    bool one = true;
    unsigned long long csum = 0ull;
#pragma unroll
    for (int k = 0; k < kSumPerThread; ++k) {
      one &= (c[k] == 0ull) || (bin[k] == b0);
      csum += c[k];                                   // < 8 * 2^39 = 2^42: fits the split in bins_warp_add
    }
    if (__all_sync(0xFFFFFFFFu, one)) {
      bins_warp_add(s_bins[warp], b0, csum, lane);
    } else {
#pragma unroll
      for (int k = 0; k < kSumPerThread; ++k) bins_warp_add(s_bins[warp], bin[k], c[k], lane);
    }
  }
  if (bad) raise_flag(flag, kFlagNonfinite);
  dq_bins_finish(s_bins, kSumThreads / 32, ws, gridDim.x, nb, mean, nullptr);
}

// One warp per group of 256 blocks: d = a - mean, s_g = max|d| / 127, code =
// clamp(rint(d / s_g)). Launched as a programmatic dependent of dq_sum_kernel; it waits
// for that grid (and its mean) before reading anything.
__global__ void __launch_bounds__(256)
dq_encode_kernel(const float* __restrict__ absmax, int64_t nb, const float* __restrict__ mean,
                 int8_t* __restrict__ qabsmax, float* __restrict__ group_scale) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float mu = *mean;
  for (int64_t g = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); g < ng; g += warps)
    dq_encode_group<false>(absmax, nb, mu, qabsmax, group_scale, g, lane);
}

// ---------------------------------------------------------------------------------
// NF4 + double quantisation of a batch of weights (a model's linears at load time) in
// three launches instead of two per weight: one persistent pass over every block of every
// weight (NF4 codes, absmax, and each weight's exact DQ sum), one thread per weight for
// the means, and the group encode over every weight's groups. The arithmetic of each weight
// is that of nf4_dq_quantize, so the results are the same bit for bit.
// ---------------------------------------------------------------------------------

constexpr int kBatchMax = 128;      // weights per launch (the table travels as a kernel parameter)

struct BatchItem {
  const uint16_t* W;
  int64_t n;
  uint8_t* codes;
  float* absmax;
  int8_t* qabsmax;
  float* group_scale;
  float* mean;
};

struct BatchArgs {
  BatchItem item[kBatchMax];
  int64_t blk_start[kBatchMax + 1];   // prefix sums of the weights' blocks
  int64_t grp_start[kBatchMax + 1];   // prefix sums of their DQ groups
  int count;
  unsigned long long* bins;           // [count][16] exact sums, zeroed before the pass
  int* flag;
};

// Weight of flattened block (or group) x, starting the search at w (prefix sums ascending).
__device__ __forceinline__ int batch_find(const int64_t* start, int count, int64_t x, int w) {
  while (w + 1 < count && x >= start[w + 1]) ++w;
  return w;
}

// Adds the lanes' running sums, keyed by (weight, bin), into the global bins: one pass per
// distinct key, a three-part warp reduction (as bins_warp_add), one atomic per key.
__device__ __forceinline__ void batch_bins_flush(unsigned long long* gbins, uint32_t key, unsigned long long c) {
  uint32_t pending = __ballot_sync(0xFFFFFFFFu, c != 0ull);
  while (pending) {
    const int leader = __ffs(pending) - 1;
    const uint32_t lk = __shfl_sync(0xFFFFFFFFu, key, leader);
    const bool mine = c != 0ull && key == lk;
    constexpr unsigned long long kPart = (1ull << 27) - 1ull;
    const uint32_t p0 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)(c & kPart) : 0u);
    const uint32_t p1 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)((c >> 27) & kPart) : 0u);
    const uint32_t p2 = __reduce_add_sync(0xFFFFFFFFu, mine ? (uint32_t)(c >> 54) : 0u);
    if ((threadIdx.x & 31) == 0)
      atomicAdd(gbins + lk, (unsigned long long)p0 + ((unsigned long long)p1 << 27) + ((unsigned long long)p2 << 54));
    pending &= ~__ballot_sync(0xFFFFFFFFu, mine);
  }
}

// Every weight of the batch holds whole blocks, with 16-byte aligned source and codes. Each
// CTA takes a contiguous range of the flattened blocks, so it touches one or two weights;
// its lanes take consecutive blocks and load their next block while they encode.
__global__ void __launch_bounds__(kNf4Threads, 2)
nf4_batch_kernel(const __grid_constant__ BatchArgs args, const Nf4Tables tab, const Nf4BoundTable btab) {
  __shared__ __align__(16) uint32_t s_tab[128 * 8];
  for (int i = threadIdx.x; i < 128 * 8 / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(s_tab)[i] = reinterpret_cast<const uint4*>(&btab.c[0][0])[i];
  __syncthreads();
  const int64_t total = args.blk_start[args.count];
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t c0 = imin64(total, per * blockIdx.x), c1 = imin64(total, c0 + per);
  bool bad = false;
  uint32_t lkey = 0;                                  // this lane's running (weight, bin) and sum
  unsigned long long lsum = 0ull;
  int w = batch_find(args.blk_start, args.count, c0, 0);
  int64_t it = c0 + threadIdx.x;
  uint4 nx[8];
  if (it < c1) {
    w = batch_find(args.blk_start, args.count, it, w);
    const uint4* src = reinterpret_cast<const uint4*>(args.item[w].W + (it - args.blk_start[w]) * kBlock);
#pragma unroll
    for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
  }
  for (int64_t w0 = c0 + (threadIdx.x & ~31); w0 < c1; w0 += kNf4Threads, it += kNf4Threads) {
    const bool live = it < c1;
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[4 * i] = nx[i].x; v[4 * i + 1] = nx[i].y; v[4 * i + 2] = nx[i].z; v[4 * i + 3] = nx[i].w;
    }
    const int wc = w;                                 // this block's weight
    const int64_t b = it - args.blk_start[wc];
    if (it + kNf4Threads < c1) {                      // the next block, possibly of the next weight
      w = batch_find(args.blk_start, args.count, it + kNf4Threads, w);
      const uint4* src =
          reinterpret_cast<const uint4*>(args.item[w].W + (it + kNf4Threads - args.blk_start[w]) * kBlock);
#pragma unroll
      for (int i = 0; i < 8; ++i) nx[i] = __ldg(src + i);
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(m), "r"(v[i]));
    m &= 0x7FFF7FFFu;
    const uint32_t amax = max(m & 0xFFFFu, m >> 16);
    uint32_t bin = 0;
    unsigned long long c = 0ull;
    if (live) {
      if (amax >= 0x7F80u) raise_flag(args.flag, kFlagNonfinite);
      args.item[wc].absmax[b] = __uint_as_float(amax << 16);
      dq_term(amax << 16, bin, c, bad);
    }
    const uint32_t key = (uint32_t)wc * kSumBins + bin;
    const bool move = c != 0ull && key != lkey && lsum != 0ull;
    if (__any_sync(0xFFFFFFFFu, move)) {
      batch_bins_flush(args.bins, lkey, move ? lsum : 0ull);
      if (move) lsum = 0ull;
    }
    if (c != 0ull) {
      lkey = key;
      lsum += c;
    }
    uint32_t Cp[7];
    nf4_boundaries(amax, s_tab, tab, Cp);
    uint32_t out[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      out[q] = nf4_pack8(nf4_code_pair(v[4 * q + 0], Cp), nf4_code_pair(v[4 * q + 1], Cp),
                         nf4_code_pair(v[4 * q + 2], Cp), nf4_code_pair(v[4 * q + 3], Cp));
    if (live) {
      uint8_t* dst = args.item[wc].codes + b * 32;
      *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
      *reinterpret_cast<uint4*>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
    }
  }
  (void)bad;                                          // a non-finite absmax already raised the flag
  batch_bins_flush(args.bins, lkey, lsum);
}

// One thread per weight: the mean from its exact bins.
__global__ void nf4_batch_mean_kernel(const __grid_constant__ BatchArgs args) {
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= args.count) return;
  unsigned long long v[kSumBins];
#pragma unroll
  for (int i = 0; i < kSumBins; ++i) v[i] = args.bins[w * kSumBins + i];
  *args.item[w].mean = dq_mean_from_bins(v, args.blk_start[w + 1] - args.blk_start[w]);
}

// One warp per DQ group, over every weight's groups.
__global__ void __launch_bounds__(256) nf4_batch_dq_kernel(const __grid_constant__ BatchArgs args) {
  const int lane = threadIdx.x & 31;
  const int64_t total = args.grp_start[args.count];
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  int w = 0;
  for (int64_t gg = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; gg < total; gg += warps) {
    w = batch_find(args.grp_start, args.count, gg, w);
    const BatchItem& it = args.item[w];
    dq_encode_group<false>(it.absmax, args.blk_start[w + 1] - args.blk_start[w], *it.mean, it.qabsmax,
                           it.group_scale, gg - args.grp_start[w], lane);
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

// CTAs of `kernel` that fit on one SM at `threads` threads (at least 1), per device.
template <typename Kernel>
static int resident_ctas(Kernel kernel, int threads) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) return 1;
  return n;
}

static int grid_for(int64_t items, int threads) {
  const int64_t need = (items + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 16;
  return (int)imax64(1, imin64(need, cap));
}

// Kernels nf4_quantize launches: the vector kernel over whole blocks when W and codes are
// 16-byte aligned, and the element-wise kernel over the rest (a ragged last block, or
// everything when unaligned).
static int nf4_launches(const void* W, int64_t n, const void* codes) {
  const bool vec = aligned(W, 16) && aligned(codes, 16);
  const int64_t nb = (n + kBlock - 1) / kBlock, nb_vec = vec ? n / kBlock : 0;
  return (nb_vec > 0) + (nb_vec < nb);
}

// NF4 encode of W[0, n); with dq_ws (zeroed bins + ticket) also the exact sum of the block
// constants and, from the last CTA, the double-quantisation mean.
static ql_status launch_nf4(const uint16_t* W, int64_t n, uint8_t* codes, float* absmax,
                            unsigned long long* dq_ws, float* mean, cudaStream_t st,
                            unsigned long long* bins_out = nullptr) {
  const bool vec = aligned(W, 16) && aligned(codes, 16);
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t nb_vec = vec ? n / kBlock : 0;
  const bool dq = dq_ws != nullptr;
  int g_vec = 0, g_tail = 0;
  if (nb_vec > 0) {
    static const int per_sm = resident_ctas(nf4_quantize_kernel<true, true>, kNf4Threads);
    const int64_t need = (nb_vec + kNf4Threads - 1) / kNf4Threads;
    g_vec = (int)imax64(1, imin64(need, (int64_t)num_sms() * per_sm));
  }
  if (nb_vec < nb) {
    const int64_t need = (nb - nb_vec + kNf4Threads - 1) / kNf4Threads;
    g_tail = (int)imax64(1, imin64(need, (int64_t)num_sms() * 4));
  }
  Nf4Args a;
  a.W = W; a.n = n; a.codes = codes; a.absmax = absmax; a.flag = device_flag_ptr();
  a.dq_ws = dq_ws; a.mean = mean; a.bins_out = bins_out; a.dq_ctas = (unsigned)(g_vec + g_tail);
  a.nb_total = nb; a.qabsmax = nullptr; a.group_scale = nullptr;
  const Nf4Tables& tab = nf4_tables();
  const Nf4BoundTable& btab = nf4_bound_table();
  if (g_vec) {
    a.blk_begin = 0; a.blk_end = nb_vec;
    if (dq) nf4_quantize_kernel<true, true><<<g_vec, kNf4Threads, 0, st>>>(a, tab, btab);
    else nf4_quantize_kernel<true, false><<<g_vec, kNf4Threads, 0, st>>>(a, tab, btab);
    QL_CHECK_LAUNCH();
  }
  if (g_tail) {
    a.blk_begin = nb_vec; a.blk_end = nb;
    if (dq) nf4_quantize_kernel<false, true><<<g_tail, kNf4Threads, 0, st>>>(a, tab, btab);
    else nf4_quantize_kernel<false, false><<<g_tail, kNf4Threads, 0, st>>>(a, tab, btab);
    QL_CHECK_LAUNCH();
  }
  return QL_OK;
}

// Zeroes n 64-bit words of a workspace. A one-CTA kernel node costs about a microsecond
// in a chain of launches, a memset node about five (measured in a CUDA graph on B200).
__global__ void __launch_bounds__(256) ws_zero_kernel(unsigned long long* __restrict__ p, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0ull;
}

static ql_status zero_ws(unsigned long long* p, int64_t n, cudaStream_t st) {
  if (n <= 0) return QL_OK;
  ws_zero_kernel<<<(unsigned)imin64((n + 255) / 256, 64), 256, 0, st>>>(p, n);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

// NF4 + DQ in one cooperative launch: whole blocks, 16-byte aligned W and codes (the
// single VEC grid). The workspace holds the bins, the ticket and the ready flag, zeroed
// here by ws_zero_kernel. A refused cooperative launch (grid not co-resident) returns QL_ERR_UNSUPPORTED
// and the caller takes the two-kernel path.
static ql_status launch_nf4_dq_fused(const uint16_t* W, int64_t n, uint8_t* codes, float* absmax,
                                     int8_t* qabsmax, float* group_scale, float* mean,
                                     unsigned long long* dq_ws, cudaStream_t st) {
  auto kern = nf4_quantize_kernel<true, true, true>;
  static const int per_sm = resident_ctas(kern, kNf4Threads);
  const int64_t nb = n / kBlock;
  const int64_t need = (nb + kNf4Threads - 1) / kNf4Threads;
  const int grid = (int)imax64(1, imin64(need, (int64_t)num_sms() * per_sm));
  Nf4Args a;
  a.W = W; a.n = n; a.blk_begin = 0; a.blk_end = nb; a.codes = codes; a.absmax = absmax;
  a.flag = device_flag_ptr(); a.dq_ws = dq_ws; a.mean = mean; a.bins_out = nullptr;
  a.dq_ctas = (unsigned)grid; a.nb_total = nb; a.qabsmax = qabsmax; a.group_scale = group_scale;
  const Nf4Tables& tab = nf4_tables();
  const Nf4BoundTable& btab = nf4_bound_table();
  if (zero_ws(dq_ws, kSumBins + 2, st) != QL_OK) return QL_ERR_CUDA;
  void* params[] = {&a, const_cast<Nf4Tables*>(&tab), const_cast<Nf4BoundTable*>(&btab)};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(grid), dim3(kNf4Threads), params, 0, st) !=
      cudaSuccess) {
    (void)cudaGetLastError();                          // clear it; the two-kernel path follows
    return QL_ERR_UNSUPPORTED;
  }
  return QL_OK;
}

// The encode pass of double quantisation, launched as a programmatic dependent of the
// kernel before it on the stream (it waits for that grid before reading anything).
static ql_status launch_dq_encode(const float* absmax, int64_t nb, const float* mean, int8_t* qabsmax,
                                  float* group_scale, cudaStream_t st) {
  const int64_t ng = (nb + kGroup - 1) / kGroup;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_for(ng * 32, 256));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, dq_encode_kernel, absmax, nb, mean, qabsmax, group_scale) != cudaSuccess)
    return QL_ERR_CUDA;
  return QL_OK;
}

}  // namespace qlb

using namespace qlb;

extern "C" {

ql_status nf4_quantize(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax, void* stream) {
  if (n < 0) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!W || !codes || !absmax) return QL_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(codes, 4) || !aligned(absmax, 4)) return QL_ERR_INVALID_ARG;
  ProfScope prof(PK_NF4, as_stream(stream), nf4_launches(W, n, codes));
  return launch_nf4(W, n, codes, absmax, nullptr, nullptr, as_stream(stream));
}

ql_status int8_quantize(const ql_bf16* W, int64_t n, int8_t* codes, float* absmax, void* stream) {
  if (n < 0) return QL_ERR_INVALID_ARG;
  if (n == 0) return QL_OK;
  if (!W || !codes || !absmax) return QL_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(absmax, 4)) return QL_ERR_INVALID_ARG;
  const bool vec = aligned(W, 16) && aligned(codes, 16);
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t nb_full = vec ? n / kBlock : 0;       // whole blocks on the vector path
  cudaStream_t st = as_stream(stream);
  ProfScope prof(PK_INT8, st, (nb_full > 0) + (nb_full < nb));
  if (nb_full > 0) {
    // persistent: the CTAs that fit at once, each lane loading its next block while it
    // encodes the current one
    static const int per_sm = resident_ctas(int8_quantize_kernel<true>, 256);
    const int grid = (int)imax64(1, imin64((nb_full + 255) / 256, (int64_t)num_sms() * per_sm));
    int8_quantize_kernel<true><<<grid, 256, 0, st>>>(W, n, nb_full, codes, absmax, device_flag_ptr());
    QL_CHECK_LAUNCH();
  }
  if (nb_full < nb) {
    // the rest (a ragged last block, or every block when unaligned), offset to its first block
    const int64_t off = nb_full * kBlock;
    int8_quantize_kernel<false><<<grid_for(nb - nb_full, 256), 256, 0, st>>>(
        W + off, n - off, nb - nb_full, codes + off, absmax + nb_full, device_flag_ptr());
    QL_CHECK_LAUNCH();
  }
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
  if (zero_ws(bins, kSumBins + 1, st) != QL_OK) return QL_ERR_CUDA;
  const int64_t chunk = (int64_t)kSumThreads * kSumPerThread;
  const int sum_grid = (int)imax64(1, imin64((nblocks + chunk - 1) / chunk, (int64_t)num_sms() * 8));
  dq_sum_kernel<<<sum_grid, kSumThreads, 0, st>>>(absmax, nblocks, bins, mean, aligned(absmax, 16) ? 1 : 0,
                                                  device_flag_ptr());
  QL_CHECK_LAUNCH();
  return launch_dq_encode(absmax, nblocks, mean, qabsmax, group_scale, st);
}

ql_status nf4_dq_quantize(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax, int8_t* qabsmax,
                          float* group_scale, float* mean, void* ws, size_t ws_bytes, void* stream) {
  if (n < 1 || !W || !codes || !absmax || !qabsmax || !group_scale || !mean || !ws) return QL_ERR_INVALID_ARG;
  const int64_t nb = (n + kBlock - 1) / kBlock;
  if (nb > (int64_t(1) << 24)) return QL_ERR_UNSUPPORTED;
  if (!aligned(W, 2) || !aligned(codes, 4) || !aligned(absmax, 4) || !aligned(group_scale, 4) ||
      !aligned(mean, 4) || !aligned(ws, 16))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0)) return QL_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  unsigned long long* bins = static_cast<unsigned long long*>(ws);
  if (n % kBlock == 0 && aligned(W, 16) && aligned(codes, 16)) {
    // one cooperative launch: encode, exact sum, mean and DQ codes
    ProfScope prof(PK_NF4, st, 2);
    const ql_status s = launch_nf4_dq_fused(W, n, codes, absmax, qabsmax, group_scale, mean, bins, st);
    if (s != QL_ERR_UNSUPPORTED) return s;
  }
  {
    ProfScope prof(PK_NF4, st, nf4_launches(W, n, codes) + 1);
    if (zero_ws(bins, kSumBins + 1, st) != QL_OK) return QL_ERR_CUDA;
    const ql_status s = launch_nf4(W, n, codes, absmax, bins, mean, st);
    if (s != QL_OK) return s;
  }
  ProfScope prof(PK_DQ, st, 1);
  return launch_dq_encode(absmax, nb, mean, qabsmax, group_scale, st);
}

ql_status nf4_dq_quantize_batch(const ql_nf4_dq_item* items, int32_t count, void* ws, size_t ws_bytes,
                                void* stream) {
  if (count < 0 || (count > 0 && (!items || !ws))) return QL_ERR_INVALID_ARG;
  if (count == 0) return QL_OK;
  if (!aligned(ws, 16)) return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql_workspace_bytes(QL_OP_DQ_BATCH, count, 0, 0, 0)) return QL_ERR_WORKSPACE;
  for (int32_t i = 0; i < count; ++i) {
    const ql_nf4_dq_item& t = items[i];
    if (t.n < 1 || !t.W || !t.codes || !t.absmax || !t.qabsmax || !t.group_scale || !t.mean)
      return QL_ERR_INVALID_ARG;
    if ((t.n + kBlock - 1) / kBlock > (int64_t(1) << 24)) return QL_ERR_UNSUPPORTED;
    if (!aligned(t.W, 2) || !aligned(t.codes, 4) || !aligned(t.absmax, 4) || !aligned(t.group_scale, 4) ||
        !aligned(t.mean, 4))
      return QL_ERR_INVALID_ARG;
  }
  cudaStream_t st = as_stream(stream);
  unsigned long long* bins = static_cast<unsigned long long*>(ws);
  // items the batch kernel does not take (a ragged last block, unaligned source or codes)
  // go through the single-weight path, one after another on the stream
  std::vector<int32_t> batch;
  for (int32_t i = 0; i < count; ++i) {
    const ql_nf4_dq_item& t = items[i];
    if (t.n % kBlock == 0 && aligned(t.W, 16) && aligned(t.codes, 16)) {
      batch.push_back(i);
    } else {
      const ql_status e = nf4_dq_quantize(t.W, t.n, t.codes, t.absmax, t.qabsmax, t.group_scale, t.mean, ws,
                                          ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0), stream);
      if (e != QL_OK) return e;
    }
  }
  static const int per_sm = resident_ctas(nf4_batch_kernel, kNf4Threads);
  const Nf4Tables& tab = nf4_tables();
  const Nf4BoundTable& btab = nf4_bound_table();
  for (size_t s0 = 0; s0 < batch.size(); s0 += kBatchMax) {
    const int cnt = (int)std::min(batch.size() - s0, (size_t)kBatchMax);
    BatchArgs a{};
    a.count = cnt;
    a.bins = bins;
    a.flag = device_flag_ptr();
    a.blk_start[0] = a.grp_start[0] = 0;
    for (int j = 0; j < cnt; ++j) {
      const ql_nf4_dq_item& t = items[batch[s0 + j]];
      a.item[j] = BatchItem{t.W, t.n, t.codes, t.absmax, t.qabsmax, t.group_scale, t.mean};
      const int64_t nb = t.n / kBlock;
      a.blk_start[j + 1] = a.blk_start[j] + nb;
      a.grp_start[j + 1] = a.grp_start[j] + (nb + kGroup - 1) / kGroup;
    }
    ProfScope prof(PK_NF4, st, 4);
    if (zero_ws(reinterpret_cast<unsigned long long*>(bins), (int64_t)cnt * kSumBins, st) != QL_OK)
      return QL_ERR_CUDA;
    const int64_t total = a.blk_start[cnt];
    const int grid = (int)imax64(1, imin64((total + kNf4Threads - 1) / kNf4Threads, (int64_t)num_sms() * per_sm));
    nf4_batch_kernel<<<grid, kNf4Threads, 0, st>>>(a, tab, btab);
    QL_CHECK_LAUNCH();
    nf4_batch_mean_kernel<<<(cnt + 31) / 32, 32, 0, st>>>(a);
    QL_CHECK_LAUNCH();
    nf4_batch_dq_kernel<<<grid_for(a.grp_start[cnt] * 32, 256), 256, 0, st>>>(a);
    QL_CHECK_LAUNCH();
  }
  return QL_OK;
}

ql_status nf4_quantize_shard(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax, uint64_t* bins,
                             void* ws, size_t ws_bytes, void* stream) {
  if (n < 1 || !W || !codes || !absmax || !bins || !ws) return QL_ERR_INVALID_ARG;
  const int64_t nb = (n + kBlock - 1) / kBlock;
  if (nb > (int64_t(1) << 24)) return QL_ERR_UNSUPPORTED;
  if (!aligned(W, 2) || !aligned(codes, 4) || !aligned(absmax, 4) || !aligned(bins, 8) || !aligned(ws, 16))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0)) return QL_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  unsigned long long* wsb = static_cast<unsigned long long*>(ws);
  ProfScope prof(PK_NF4, st, nf4_launches(W, n, codes) + 1);
  if (zero_ws(wsb, kSumBins + 1, st) != QL_OK) return QL_ERR_CUDA;
  return launch_nf4(W, n, codes, absmax, wsb, nullptr, st, reinterpret_cast<unsigned long long*>(bins));
}

ql_status dq_quantize_shard(const float* absmax, int64_t nblocks, const uint64_t* bins, int64_t nblocks_total,
                            int8_t* qabsmax, float* group_scale, float* mean, void* stream) {
  if (nblocks < 1 || nblocks_total < nblocks || !absmax || !bins || !qabsmax || !group_scale || !mean)
    return QL_ERR_INVALID_ARG;
  if (nblocks_total > (int64_t(1) << 24)) return QL_ERR_UNSUPPORTED;
  if (!aligned(absmax, 4) || !aligned(bins, 8) || !aligned(group_scale, 4) || !aligned(mean, 4))
    return QL_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  ProfScope prof(PK_DQ, st, 2);
  dq_mean_kernel<<<1, 32, 0, st>>>(reinterpret_cast<const unsigned long long*>(bins), nblocks_total, mean);
  QL_CHECK_LAUNCH();
  return launch_dq_encode(absmax, nblocks, mean, qabsmax, group_scale, st);
}

ql_status ql_dequantize(const ql_weight* w, ql_bf16* Wout, void* stream) {
  if (!w || !Wout || w->N < 1 || w->K < 1 || !w->codes || !aligned(Wout, 2)) return QL_ERR_INVALID_ARG;
  if (w->N > (int64_t(1) << 40) / w->K) return QL_ERR_UNSUPPORTED;   // N*K stays far from overflow
  const bool nf4 = w->fmt == QL_FMT_NF4_DQ;
  if (nf4 ? !w->qabsmax || !w->group_scale || !w->mean || !aligned(w->group_scale, 4) || !aligned(w->mean, 4)
          : w->fmt != QL_FMT_INT8_B64 || !w->absmax || !aligned(w->absmax, 4))
    return QL_ERR_INVALID_ARG;
  const int64_t n = w->N * w->K;
  const int64_t nb = (n + kBlock - 1) / kBlock;
  cudaStream_t st = as_stream(stream);
  ProfScope prof(PK_DEQ, st, 1);                      // counts a launch: every check is above
  if (nf4)
    dequant_nf4_kernel<<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const uint8_t*>(w->codes), w->qabsmax, w->group_scale, w->mean, n, Wout,
        nf4_tables());
  else
    dequant_int8_kernel<<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const int8_t*>(w->codes), w->absmax, n, Wout);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

}  // extern "C"
