// Persistent warp-specialised tcgen05 GEMMs for the quantised linear layer.
//
//   C[R, Cn] = sum_k Aop[R, k] * Bop[Cn, k]  (+ sum_e Aext[R, e] * Bext[Cn, e])
//
// Tiles are 128 rows x BN columns; the contraction runs in chunks of 64 (one 128-byte
// swizzled smem row per operand row). Accumulators are double-buffered in TMEM so the
// epilogue of one tile overlaps the main loop of the next.
//
// qgemm_tma_kernel — both operands by TMA (the adapter-sized GEMMs). Warps:
//   0..3 epilogue, 4 TMA, 5 MMA issuer (also owns TMEM).
// qgemm_wdec_kernel — the weight operand is decoded from its quantised form (QLoRA page,
// "1. NF4" and "2. Double Quantization": w' = q[code] * a') into the swizzled UMMA layout
// and used as the MMA's M = 128 operand against 256 tokens (see below). Nothing in the
// decode warps reads global memory, so they never wait on it.
// The unmerged LoRA term enters as extra contraction chunks of the same accumulator.
//
// Every wait is bounded; a wait that gives up raises the CTA's abort word, every role then
// leaves its loop, copies and MMAs in flight are drained (bounded), TMEM is freed, and the
// kernel reports QL_ERR_TIMEOUT through the device flag.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace qlb {

enum class BSrc : int { NF4 = 1, INT8 = 2 };
enum Epi : int { EPI_BF16 = 0, EPI_LORA_T = 1, EPI_LORA_Q = 2, EPI_DA = 3, EPI_DB = 4 };

struct GemmArgs {
  int64_t R, Cn, Kc;     // rows, columns, main contraction length
  int32_t n_ext;         // number of 64-wide extension chunks
  int32_t r;             // adapter rank (epilogue masks)
  float q[16];           // NF4 grid
  // epilogue
  void* out;  int64_t ld_out;
  void* out2; int64_t ld_out2;
  float scale;
  uint64_t timeout_ns;
  int* flag;
  // split-K (TMA GEMM only): ksplit > 1 splits the contraction into slices of kc_per
  // 64-wide chunks; each (tile, slice) stores its fp32 partial into part [ksplit][R][ldp]
  // and reduce_partials_kernel applies the epilogue to their sum
  int32_t ksplit, kc_per;
  float* part;
  int64_t ldp;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// ---------------------------------------------------------------------------------
// NF4 decode. For a block with rebuilt scale a', the eight non-negative-index entries
// M[i] = bf16(fp32(q_{8+i} * a')) are formed with 8 multiplies; since the grid is
// symmetric (q_{7-i} = -q_{8+i} exactly) and rounding is symmetric, code c decodes to
// M[c-8] for c >= 8 and to -M[7-c] for c < 8. L/H hold the low/high bytes of M[0..7].
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void nf4_table(const float (&q)[16], float ar, uint32_t (&L)[2],
                                          uint32_t (&H)[2]) {
  const uint32_t P01 = pack_bf16x2(__fmul_rn(q[8], ar), __fmul_rn(q[9], ar));
  const uint32_t P23 = pack_bf16x2(__fmul_rn(q[10], ar), __fmul_rn(q[11], ar));
  const uint32_t P45 = pack_bf16x2(__fmul_rn(q[12], ar), __fmul_rn(q[13], ar));
  const uint32_t P67 = pack_bf16x2(__fmul_rn(q[14], ar), __fmul_rn(q[15], ar));
  L[0] = prmt(P01, P23, 0x6420u);
  H[0] = prmt(P01, P23, 0x7531u);
  L[1] = prmt(P45, P67, 0x6420u);
  H[1] = prmt(P45, P67, 0x7531u);
}

// 8 codes (one 32-bit word, element 0 in the low nibble) -> 8 bf16 (four bf16x2 words).
__device__ __forceinline__ uint4 nf4_decode8(uint32_t w, const uint32_t (&L)[2], const uint32_t (&H)[2]) {
  const uint32_t m8 = w & 0x88888888u;                     // bit 3 of every code
  const uint32_t f = m8 - (m8 >> 3);                       // 7 where the code is >= 8
  const uint32_t idx = (w ^ f ^ 0x77777777u) & 0x77777777u;  // c-8 (c >= 8) or 7-c (c < 8)
  const uint32_t m84 = m8 << 4;
  uint4 o;
  uint32_t s = prmt(m84, m8, 0xD9C8u);                     // 0xFF in byte i where code i >= 8
  uint32_t lo = prmt(L[0], L[1], idx);
  uint32_t hi = prmt(H[0], H[1], idx) ^ (~s & 0x80808080u);  // negate the codes below 8
  o.x = prmt(lo, hi, 0x5140u);
  o.y = prmt(lo, hi, 0x7362u);
  s = prmt(m84, m8, 0xFBEAu);
  const uint32_t idxh = idx >> 16;
  lo = prmt(L[0], L[1], idxh);
  hi = prmt(H[0], H[1], idxh) ^ (~s & 0x80808080u);
  o.z = prmt(lo, hi, 0x5140u);
  o.w = prmt(lo, hi, 0x7362u);
  return o;
}

// int8: w' = bf16(fp32(c * sc)); c is recovered exactly from a magic float (2^23 + c + 128).
__device__ __forceinline__ uint4 int8_decode8(uint32_t w0, uint32_t w1, float sc) {
  uint32_t o[4];
  const uint32_t kMagic = 0x4B000000u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t wv = (h ? w1 : w0) ^ 0x80808080u;
    float f[4];
    f[0] = __uint_as_float(prmt(wv, kMagic, 0x7540u));
    f[1] = __uint_as_float(prmt(wv, kMagic, 0x7541u));
    f[2] = __uint_as_float(prmt(wv, kMagic, 0x7542u));
    f[3] = __uint_as_float(prmt(wv, kMagic, 0x7543u));
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __fmul_rn(__fsub_rn(f[i], 8388736.0f), sc);
    o[2 * h] = pack_bf16x2(f[0], f[1]);
    o[2 * h + 1] = pack_bf16x2(f[2], f[3]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ---------------------------------------------------------------------------------
// Epilogues
// ---------------------------------------------------------------------------------
template <int EPI>
__device__ __forceinline__ void epilogue_store(const GemmArgs& a, int64_t row, int64_t col,
                                               const uint32_t (&v)[32]) {
  if (row >= a.R) return;
  if constexpr (EPI == EPI_BF16 || EPI == EPI_LORA_Q) {
    const float s = (EPI == EPI_LORA_Q) ? a.scale : 1.0f;
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      p[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * s, __uint_as_float(v[2 * j + 1]) * s);
    uint16_t* out = static_cast<uint16_t*>(a.out) + row * a.ld_out + col;
    if (col + 32 <= a.Cn) {
      uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
    } else {
      for (int j = 0; j < 32 && col + j < a.Cn; ++j)
        out[j] = (uint16_t)(p[j / 2] >> (16 * (j & 1)));
    }
  } else if constexpr (EPI == EPI_LORA_T) {
    // out2 = P = bf16(s * T) [R, ld_out2] (all padded columns); out = bf16(T) [R, r]
    uint16_t* P = static_cast<uint16_t*>(a.out2) + row * a.ld_out2 + col;
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      p[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * a.scale, __uint_as_float(v[2 * j + 1]) * a.scale);
    uint4* o = reinterpret_cast<uint4*>(P);
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
    if (a.out) {
      uint16_t* T = static_cast<uint16_t*>(a.out) + row * a.ld_out;
      for (int j = 0; j < 32; ++j)
        if (col + j < a.r) T[col + j] = (uint16_t)float_to_bf16_bits(__uint_as_float(v[j]));
    }
  } else if constexpr (EPI == EPI_DA) {
    // out = dA [r, ld_out] fp32; this tile's rows are input features k, columns j
    float* dA = static_cast<float*>(a.out);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col + j < a.r) dA[(col + j) * a.ld_out + row] = __uint_as_float(v[j]) * a.scale;
  } else {
    // EPI_DB: out = dB [R, r] fp32
    float* dB = static_cast<float*>(a.out) + row * a.ld_out;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col + j < a.r) dB[col + j] = __uint_as_float(v[j]) * a.scale;
  }
}

// Epilogue role shared by both kernels: warps 0..3, TMEM lanes 32*warp ..
template <int BN, int EPI>
__device__ __forceinline__ void run_epilogue(const GemmArgs& args, uint32_t tmem_base, uint32_t acc_full,
                                             uint32_t acc_empty, int64_t items, int64_t n_tiles,
                                             volatile int* abort_word) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = args.ksplit > 1 ? args.ksplit : 1;
  uint32_t tcount = 0;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x, ++tcount) {
    const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
    const bool okw = mbar_wait(acc_full + 8 * acc, aph, args.timeout_ns, abort_word);
    if (!__all_sync(0xFFFFFFFFu, okw)) break;
    tc_fence_after();
    const int64_t t = it / ks, split = it % ks;
    const int64_t r0 = (t / n_tiles) * 128, c0 = (t % n_tiles) * BN;
    const int64_t row = r0 + warp * 32 + lane;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * BN + cc, v);
      if (ks > 1) {
        if (row < args.R) {                          // the slice's partial, all BN columns
          float4* dst = reinterpret_cast<float4*>(args.part + (split * args.R + row) * args.ldp + c0 + cc);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
      } else if (c0 + cc < args.Cn) {
        epilogue_store<EPI>(args, row, c0 + cc, v);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty + 8 * acc);
  }
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < 200000000ull) {}
}

// Sum of the split-K partials in slice order (so the result does not depend on which CTA
// ran which slice), then the GEMM's own epilogue. One thread per (row, 32 columns).
template <int EPI>
__global__ void __launch_bounds__(256)
reduce_partials_kernel(const GemmArgs args) {
  const int64_t chunks = (args.Cn + 31) / 32;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= args.R * chunks) return;
  const int64_t row = i / chunks, c0 = (i % chunks) * 32;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
  for (int s = 0; s < args.ksplit; ++s) {
    const float4* src = reinterpret_cast<const float4*>(args.part + (s * args.R + row) * args.ldp + c0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = src[j];
      acc[4 * j] += v.x; acc[4 * j + 1] += v.y; acc[4 * j + 2] += v.z; acc[4 * j + 3] += v.w;
    }
  }
  uint32_t v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(acc[j]);
  epilogue_store<EPI>(args, row, c0, v);
}

// =================================================================================
// Both operands by TMA
// =================================================================================
template <int BN>
struct TmaCfg {
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStages = BN >= 192 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);   // power of two
  static constexpr size_t kSmem = (size_t)kStages * (kABytes + kBBytes) + 2048;
};

template <int BN, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(192, 1)
qgemm_tma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs args) {
  using Cfg = TmaCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * Cfg::kBBytes);
  const uint32_t full = smem_u32(bars);
  const uint32_t empty = full + 8 * S;
  const uint32_t acc_full = full + 16 * S;
  const uint32_t acc_empty = acc_full + 16;
  const uint32_t drain = acc_full + 32;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + 8 * s, 1); mbar_init(empty + 8 * s, 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full + 8 * i, 1); mbar_init(acc_empty + 8 * i, 4); }
    mbar_init(drain, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) { tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB); }
  if (warp == 5) tmem_alloc(smem_u32(tmem_holder), Cfg::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int64_t n_tiles = (args.Cn + BN - 1) / BN;
  const int64_t tiles = ((args.R + 127) / 128) * n_tiles;
  const int kc_total = (int)((args.Kc + 63) / 64);
  // work items: (tile, contraction slice); one slice of all chunks without split-K
  const int ks = args.ksplit > 1 ? args.ksplit : 1;
  const int kc_per = ks > 1 ? args.kc_per : kc_total;
  const int64_t items = tiles * ks;
  const uint64_t lim = args.timeout_ns;

  if (warp < 4) {
    run_epilogue<BN, EPI>(args, tmem_base, acc_full, acc_empty, items, n_tiles, abort_word);
  } else if (warp == 4 && lane == 0) {
    uint32_t g = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < items && ok; it += gridDim.x) {
      const int64_t t = it / ks;
      const int kb = (int)(it % ks) * kc_per, ke = kb + kc_per < kc_total ? kb + kc_per : kc_total;
      const int32_t r0 = (int32_t)((t / n_tiles) * 128), c0 = (int32_t)((t % n_tiles) * BN);
      for (int kc = kb; kc < ke; ++kc, ++g) {
        const uint32_t s = g % S, ph = (g / S) & 1;
        if (!mbar_wait(empty + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
        const uint32_t fb = full + 8 * s;
        const uint32_t dA = smem_u32(sA + s * Cfg::kABytes);
        const uint32_t dB = smem_u32(sB + s * Cfg::kBBytes);
        mbar_arrive_expect_tx(fb, Cfg::kABytes + Cfg::kBBytes);
        if (!A_MN) {
          tma_load_2d(dA, &tmA, fb, kc * 64, r0);
        } else {
          tma_load_2d(dA, &tmA, fb, r0, kc * 64);
          tma_load_2d(dA + 8192, &tmA, fb, r0 + 64, kc * 64);
        }
        if (!B_MN) {
          tma_load_2d(dB, &tmB, fb, kc * 64, c0);
        } else {
#pragma unroll
          for (int i = 0; i < BN / 64; ++i) tma_load_2d(dB + i * 8192, &tmB, fb, c0 + 64 * i, kc * 64);
        }
      }
    }
    if (!ok || *abort_word)
      for (uint32_t j = (g > (uint32_t)S ? g - S : 0); j < g; ++j) drain_wait(full + 8 * (j % S), (j / S) & 1);
  } else if (warp == 5 && lane == 0) {
    constexpr uint32_t kId = idesc_bf16_f32(128, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
    uint32_t g = 0, tcount = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < items && ok; it += gridDim.x, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      if (!mbar_wait(acc_empty + 8 * acc, aph ^ 1, lim, abort_word)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      const int kb = (int)(it % ks) * kc_per, ke = kb + kc_per < kc_total ? kb + kc_per : kc_total;
      for (int kc = kb; kc < ke; ++kc, ++g) {
        const uint32_t s = g % S, ph = (g / S) & 1;
        if (!mbar_wait(full + 8 * s, ph, lim, abort_word)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * Cfg::kABytes);
        const uint32_t b_base = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = !A_MN ? smem_desc_sw128(a_base + k * 32, 16, 1024)
                                    : smem_desc_sw128(a_base + k * 2048, 8192, 1024);
          const uint64_t bd = !B_MN ? smem_desc_sw128(b_base + k * 32, 16, 1024)
                                    : smem_desc_sw128(b_base + k * 2048, 8192, 1024);
          tc_mma(d_tmem, ad, bd, kId, (kc > kb || k > 0) ? 1u : 0u);
        }
        tc_commit(empty + 8 * s);
      }
      if (!ok) break;
      tc_commit(acc_full + 8 * acc);
    }
    if (!ok || *abort_word) { tc_commit(drain); drain_wait(drain, 0); }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) { tc_fence_after(); tmem_dealloc(tmem_base, Cfg::kTmemCols); }
  if (threadIdx.x == 0 && *abort_word) raise_flag(args.flag, kFlagTimeout);
}

// =================================================================================
// Weight operand decoded from NF4 / int8, as the M = 128 operand of the MMA
//
//   C^T[w, t] = sum_k W'[w, k] * T[t, k]   (w: 128 weight rows per tile, t: 256 tokens)
//
// Forward: w = output feature n, contraction over input features (W' K-major).
// dX:      w = input feature k,  contraction over output features (W'^T, MN-major).
// Each decoded weight row feeds 256 token columns, so a tile decodes 128 blocks per
// chunk for 2*128*256*64 flops. The result is stored transposed (lanes are consecutive
// weight rows, so every store instruction of a warp writes 64 contiguous bytes).
// Warps: 0..3 epilogue, 4 TMA for the token tiles (and the extension's token factor),
// 5 MMA issuer, 6 TMA for the weight codes + block scales, 7..14 decode (two lanes per
// 64-element block; they also issue the TMA of the extension's weight-side factor, so
// every ring has a single producer).
// =================================================================================
// DW: a ring of SW stages for the dense update's chunks, paid for with one token stage and
// fewer code stages.
template <BSrc BS, bool DW = false>
struct WdecCfg {
  static constexpr int BM = 128;                                 // weight rows per tile
  static constexpr int BN = 256;                                 // tokens per tile
  static constexpr int NP = 8;                                   // decode warps
  static constexpr int kDBytes = BM * 128;                       // decoded weight stage
  static constexpr int kTBytes = BN * 128;                       // token stage
  static constexpr int kCodeBytes = BM * (BS == BSrc::NF4 ? 32 : 64);
  static constexpr int kCBytes = kCodeBytes + 1024;              // codes + scales
  static constexpr int SD = 4, ST = DW ? 3 : 4;
  static constexpr int SC = DW ? (BS == BSrc::NF4 ? 3 : 2) : (BS == BSrc::NF4 ? 6 : 3);
  static constexpr int SW = DW ? (BS == BSrc::NF4 ? 3 : 2) : 0;  // update stages (kDBytes each)
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = (7 + NP) * 32;
  static constexpr size_t kSmem =
      (size_t)SD * kDBytes + (size_t)ST * kTBytes + (size_t)SC * kCBytes + (size_t)SW * kDBytes + 2048;
};

// EPI_BF16 stored transposed: element (weight row w, token t) -> out[t * ld_out + w]
__device__ __forceinline__ void epilogue_store_t(const GemmArgs& a, int64_t wrow, int64_t t0,
                                                 const uint32_t (&v)[32]) {
  if (wrow >= a.R) return;
  uint16_t* out = static_cast<uint16_t*>(a.out) + wrow;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (t0 + j < a.Cn) out[(t0 + j) * a.ld_out] = (uint16_t)float_to_bf16_bits(__uint_as_float(v[j]));
}

// bf16x2 sum with one rounding to nearest even per half.
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// W_MN = false: forward; true: dX (weight used transposed). DW (forward only, no extension
// chunks): a dense bf16 update dW [R, Kc] (tmDW, box 64 x 128 with the 128-byte swizzle, the
// decoded stage's own layout) is added to the decoded weight before the MMA, bf16(W' + dW)
// with one rounding: the codes' producer also loads each chunk of dW into a ring of its own,
// and the decode warps add it to their decoded values before storing them.
template <BSrc BS, bool W_MN, bool DW = false>
__global__ void __launch_bounds__(WdecCfg<BS, DW>::kThreads, 1)
qgemm_wdec_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmCodes,
                  const __grid_constant__ CUtensorMap tmScale, const __grid_constant__ CUtensorMap tmTe,
                  const __grid_constant__ CUtensorMap tmWe, const __grid_constant__ CUtensorMap tmDW,
                  const GemmArgs args) {
  static_assert(!(DW && W_MN), "the dense update is a forward-only operand");
  using Cfg = WdecCfg<BS, DW>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN, NP = Cfg::NP, SD = Cfg::SD, ST = Cfg::ST, SC = Cfg::SC;
  constexpr int SW = Cfg::SW;
  constexpr int SWm = SW > 0 ? SW : 1;                 // the update ring's modulus (DW only)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sD = smem;                                   // decoded weight (A operand)
  uint8_t* sT = sD + SD * Cfg::kDBytes;                 // tokens (B operand)
  uint8_t* sC = sT + ST * Cfg::kTBytes;                 // codes + scales
  uint8_t* sW = sC + SC * Cfg::kCBytes;                 // DW: the update's chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + SW * Cfg::kDBytes);
  const uint32_t full_d = smem_u32(bars);
  const uint32_t empty_d = full_d + 8 * SD;
  const uint32_t full_t = empty_d + 8 * SD;
  const uint32_t empty_t = full_t + 8 * ST;
  const uint32_t full_c = empty_t + 8 * ST;
  const uint32_t empty_c = full_c + 8 * SC;
  const uint32_t acc_full = empty_c + 8 * SC;
  const uint32_t acc_empty = acc_full + 16;
  const uint32_t drain = acc_full + 32;
  const uint32_t dw_full = drain + 8;                  // DW: the update's chunk has landed
  const uint32_t dw_empty = dw_full + 8 * SW;          // DW: the decode warps have read it
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * (SD + ST + SC) + 5 + 2 * SW);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SD; ++s) { mbar_init(full_d + 8 * s, NP); mbar_init(empty_d + 8 * s, 1); }
    for (int s = 0; s < ST; ++s) { mbar_init(full_t + 8 * s, 1); mbar_init(empty_t + 8 * s, 1); }
    for (int s = 0; s < SC; ++s) { mbar_init(full_c + 8 * s, 1); mbar_init(empty_c + 8 * s, NP); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full + 8 * i, 1); mbar_init(acc_empty + 8 * i, 4); }
    mbar_init(drain, 1);
    for (int s = 0; s < SW; ++s) { mbar_init(dw_full + 8 * s, 1); mbar_init(dw_empty + 8 * s, NP); }
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmT);
    if (args.n_ext) tma_prefetch_desc(&tmTe);
  }
  if (warp == 6 && lane == 0) {
    tma_prefetch_desc(&tmCodes);
    tma_prefetch_desc(&tmScale);
    if (DW) tma_prefetch_desc(&tmDW);
  }
  if (warp == 7 && lane == 0 && args.n_ext) tma_prefetch_desc(&tmWe);
  if (warp == 5) tmem_alloc(smem_u32(tmem_holder), Cfg::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // tiles: weight-row tiles fastest, so concurrently running CTAs share token tiles
  const int64_t w_tiles = (args.R + BM - 1) / BM;
  const int64_t tiles = w_tiles * ((args.Cn + BN - 1) / BN);
  const int kc_main = (int)((args.Kc + 63) / 64);
  const int kc_total = kc_main + args.n_ext;
  const uint64_t lim = args.timeout_ns;

  if (warp < 4) {
    // ---- epilogue: 128 weight rows (TMEM lanes) x 256 tokens ----
    uint32_t tcount = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      const bool okw = mbar_wait(acc_full + 8 * acc, aph, lim, abort_word);
      if (!__all_sync(0xFFFFFFFFu, okw)) break;
      tc_fence_after();
      const int64_t w0 = (t % w_tiles) * BM, t0 = (t / w_tiles) * BN;
      const int64_t wrow = w0 + warp * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * BN + cc, v);
        if (t0 + cc < args.Cn) epilogue_store_t(args, wrow, t0 + cc, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * acc);
    }
  } else if (warp == 4 && lane == 0) {
    // ---- token tiles -> T ring ----
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int32_t t0 = (int32_t)((t / w_tiles) * BN);
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t s = g % ST, ph = (g / ST) & 1;
        if (!mbar_wait(empty_t + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
        const uint32_t fb = full_t + 8 * s;
        mbar_arrive_expect_tx(fb, Cfg::kTBytes);
        if (kc < kc_main) tma_load_2d(smem_u32(sT + s * Cfg::kTBytes), &tmT, fb, kc * 64, t0);
        else tma_load_2d(smem_u32(sT + s * Cfg::kTBytes), &tmTe, fb, (kc - kc_main) * 64, t0);
      }
    }
    if (!ok || *abort_word)
      for (uint32_t j = (g > (uint32_t)ST ? g - ST : 0); j < g; ++j) drain_wait(full_t + 8 * (j % ST), (j / ST) & 1);
  } else if (warp == 6 && lane == 0) {
    // ---- weight codes + block scales -> C ring ----
    uint32_t gc = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int32_t w0 = (int32_t)((t % w_tiles) * BM);
      for (int kc = 0; kc < kc_main; ++kc, ++gc) {
        const uint32_t s = gc % SC, ph = (gc / SC) & 1;
        if (!mbar_wait(empty_c + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
        const uint32_t fb = full_c + 8 * s;
        const uint32_t dst = smem_u32(sC + s * Cfg::kCBytes);
        if (!W_MN) {
          // weight rows w0..w0+128, block column kc
          mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + BM * 4);
          tma_load_2d(dst, &tmCodes, fb, kc * (BS == BSrc::NF4 ? 32 : 64), w0);
          tma_load_2d(dst + Cfg::kCodeBytes, &tmScale, fb, w0, kc);
        } else {
          // weight rows kc*64..+64, weight columns w0..w0+128 (2 blocks per row); the
          // scale box starts at a multiple of 4 blocks (16-byte aligned) and spans 4
          mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + 1024);
          tma_load_2d(dst, &tmCodes, fb, BS == BSrc::NF4 ? w0 / 2 : w0, kc * 64);
          tma_load_2d(dst + Cfg::kCodeBytes, &tmScale, fb, (w0 / 64) & ~3, kc * 64);
        }
        if (DW) {
          // the update's rows w0..w0+128, columns kc*64..+64, into its own ring (the chunk
          // sequence, there being no extension chunks)
          const uint32_t sw = gc % SWm, pw = (gc / SWm) & 1;
          if (!mbar_wait(dw_empty + 8 * sw, pw ^ 1, lim, abort_word)) { ok = false; ++gc; break; }
          mbar_arrive_expect_tx(dw_full + 8 * sw, Cfg::kDBytes);
          tma_load_2d(smem_u32(sW + sw * Cfg::kDBytes), &tmDW, dw_full + 8 * sw, kc * 64, w0);
        }
      }
    }
    if (!ok || *abort_word) {
      for (uint32_t j = (gc > (uint32_t)SC ? gc - SC : 0); j < gc; ++j) drain_wait(full_c + 8 * (j % SC), (j / SC) & 1);
      if (DW) {
        // the update chunks issued: all but the last when a wait for the stage gave up
        const uint32_t gdw = ok ? gc : gc - 1;
        for (uint32_t j = (gdw > (uint32_t)SWm ? gdw - SWm : 0); j < gdw; ++j) drain_wait(dw_full + 8 * (j % SWm), (j / SWm) & 1);
      }
    }
  } else if (warp == 5 && lane == 0) {
    // ---- MMA issuer ----
    constexpr uint32_t kIdMain = idesc_bf16_f32(128, BN, W_MN ? 1 : 0, 0);
    constexpr uint32_t kIdExt = idesc_bf16_f32(128, BN, 0, 0);
    uint32_t g = 0, tcount = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      if (!mbar_wait(acc_empty + 8 * acc, aph ^ 1, lim, abort_word)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t sd = g % SD, pd = (g / SD) & 1;
        const uint32_t st = g % ST, pt = (g / ST) & 1;
        if (!mbar_wait(full_t + 8 * st, pt, lim, abort_word)) { ok = false; break; }
        if (!mbar_wait(full_d + 8 * sd, pd, lim, abort_word)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_base = smem_u32(sD + sd * Cfg::kDBytes);
        const uint32_t t_base = smem_u32(sT + st * Cfg::kTBytes);
        const bool ext = kc >= kc_main;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = (!W_MN || ext) ? smem_desc_sw128(d_base + k * 32, 16, 1024)
                                             : smem_desc_sw128(d_base + k * 2048, 8192, 1024);
          const uint64_t bd = smem_desc_sw128(t_base + k * 32, 16, 1024);
          tc_mma(d_tmem, ad, bd, ext ? kIdExt : kIdMain, (kc > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(empty_d + 8 * sd);
        tc_commit(empty_t + 8 * st);
      }
      if (!ok) break;
      tc_commit(acc_full + 8 * acc);
    }
    if (!ok || *abort_word) { tc_commit(drain); drain_wait(drain, 0); }
  } else if (warp >= 7) {
    // ---- decode: C ring -> D ring (bf16, swizzled UMMA layout), two lanes per block ----
    const int tid = threadIdx.x - 7 * 32;                        // 0..255
    const int blk = tid >> 1, half = tid & 1;                    // block 0..127
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = args.q[i];
    int code_off, j_row = 0, gi = 0;
    uint32_t d_off, key;
    if (!W_MN) {
      code_off = blk * (BS == BSrc::NF4 ? 32 : 64);
      d_off = blk * 128;
      key = blk & 7;
    } else {
      j_row = blk & 63;
      gi = blk >> 6;
      code_off = j_row * (BS == BSrc::NF4 ? 64 : 128) + gi * (BS == BSrc::NF4 ? 32 : 64);
      d_off = gi * 8192 + (j_row >> 3) * 1024 + (j_row & 7) * 128;
      key = j_row & 7;
    }
    uint32_t gc = 0, gd = 0, last_sd = 0, last_pd = 0;
    bool ok = true, ext_issued = false;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int32_t w0 = (int32_t)((t % w_tiles) * BM);
      const int scale_idx = !W_MN ? blk : j_row * 4 + ((w0 / 64) & 3) + gi;
      for (int kc = 0; kc < kc_total; ++kc, ++gd) {
        const uint32_t sd = gd % SD, pd = (gd / SD) & 1;
        if (kc >= kc_main) {
          const bool wb = mbar_wait(empty_d + 8 * sd, pd ^ 1, lim, abort_word);
          if (!__all_sync(0xFFFFFFFFu, wb)) { ok = false; break; }
          if (lane == 0) {
            const uint32_t fb = full_d + 8 * sd;
            if (warp == 7) {
              mbar_arrive_expect_tx(fb, Cfg::kDBytes);
              tma_load_2d(smem_u32(sD + sd * Cfg::kDBytes), &tmWe, fb, (kc - kc_main) * 64, w0);
              ext_issued = true;
              last_sd = sd;
              last_pd = pd;
            } else {
              mbar_arrive(fb);
            }
          }
          continue;
        }
        const uint32_t sc = gc % SC, pc = (gc / SC) & 1;
        const bool w1 = mbar_wait(full_c + 8 * sc, pc, lim, abort_word);
        // DW: the update's chunk gc has landed in its ring
        const uint32_t sw = DW ? gc % SWm : 0, pw = DW ? (gc / SWm) & 1 : 0;
        const bool w3 = w1 && (!DW || mbar_wait(dw_full + 8 * sw, pw, lim, abort_word));
        const bool w2 = w3 && mbar_wait(empty_d + 8 * sd, pd ^ 1, lim, abort_word);
        if (!__all_sync(0xFFFFFFFFu, w2)) { ok = false; break; }
        const uint8_t* cst = sC + sc * Cfg::kCBytes;
        const float sv = reinterpret_cast<const float*>(cst + Cfg::kCodeBytes)[scale_idx];
        uint4* d = reinterpret_cast<uint4*>(sD + sd * Cfg::kDBytes + d_off);
        const uint4* u = reinterpret_cast<const uint4*>(sW + sw * Cfg::kDBytes + d_off);
        auto put = [&](int i, uint4 v) {
          if (DW) {
            const uint4 x = u[i];
            v = make_uint4(add_bf16x2(v.x, x.x), add_bf16x2(v.y, x.y), add_bf16x2(v.z, x.z), add_bf16x2(v.w, x.w));
          }
          d[i] = v;
        };
        if constexpr (BS == BSrc::NF4) {
          const uint4 cv = reinterpret_cast<const uint4*>(cst + code_off)[half];
          uint32_t L[2], H[2];
          nf4_table(q, sv, L, H);
          const int c0i = 4 * half;
          put((c0i + 0) ^ key, nf4_decode8(cv.x, L, H));
          put((c0i + 1) ^ key, nf4_decode8(cv.y, L, H));
          put((c0i + 2) ^ key, nf4_decode8(cv.z, L, H));
          put((c0i + 3) ^ key, nf4_decode8(cv.w, L, H));
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(cst + code_off) + 2 * half;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 w = src[h];
            const int c = 4 * half + 2 * h;
            put(c ^ key, int8_decode8(w.x, w.y, sv));
            put((c + 1) ^ key, int8_decode8(w.z, w.w, sv));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(full_d + 8 * sd);
          mbar_arrive(empty_c + 8 * sc);
          if (DW) mbar_arrive(dw_empty + 8 * sw);
        }
        ++gc;
      }
    }
    if ((!ok || *abort_word) && warp == 7 && lane == 0 && ext_issued)
      drain_wait(full_d + 8 * last_sd, last_pd);       // our last extension copy (bounded)
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) { tc_fence_after(); tmem_dealloc(tmem_base, Cfg::kTmemCols); }
  if (threadIdx.x == 0 && *abort_word) raise_flag(args.flag, kFlagTimeout);
}

// =================================================================================
// The same decode GEMM on a CTA pair (cta_group::2): one MMA of 256 weight rows x 256
// tokens per 16-wide k step, issued by the even CTA. Each CTA decodes its own 128 weight
// rows into its own shared memory and loads its own 128 token rows by TMA, so per SM the
// token tile and its tensor-core reads are half of the single-CTA kernel's, which is
// what bounds that kernel (shared-memory bandwidth). Every ring stays local to its CTA;
// the odd CTA's MMA warp relays "stage s is full here" to the even CTA with one
// cluster-scope arrive per stage, and the even CTA's commits free the stages of both.
// =================================================================================
// DW: as WdecCfg, a ring of SW stages for the dense update's chunks (this CTA's 128 rows),
// paid for with token and code stages.
template <BSrc BS, bool DW = false>
struct WpairCfg {
  static constexpr int BM = 128;                                 // weight rows per CTA
  static constexpr int BN = 256;                                 // tokens per pair tile
  static constexpr int BNH = 128;                                // tokens per CTA
  static constexpr int NP = 8;                                   // decode warps
  static constexpr int kDBytes = BM * 128;                       // decoded weight stage
  static constexpr int kTBytes = BNH * 128;                      // token stage (this CTA's half)
  static constexpr int kCodeBytes = BM * (BS == BSrc::NF4 ? 32 : 64);
  static constexpr int kCBytes = kCodeBytes + 1024;              // codes + scales
  // decoded-weight stages (filled on this SM, short latency), token stages (TMA from L2,
  // long latency: the deeper ring), code stages
  static constexpr int SD = 4, ST = DW ? (BS == BSrc::NF4 ? 6 : 5) : 8;
  static constexpr int SC = DW ? 3 : (BS == BSrc::NF4 ? 6 : 3);
  static constexpr int SW = DW ? 3 : 0;                          // update stages (kDBytes each)
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = (7 + NP) * 32;
  static constexpr size_t kSmem =
      (size_t)SD * kDBytes + (size_t)ST * kTBytes + (size_t)SC * kCBytes + (size_t)SW * kDBytes + 2048;
  static_assert(kSmem + 1024 <= 232448, "shared memory");
};

// First weight row (or input feature, for dX) that a CTA of the pair loads. When the odd
// CTA's whole 128-row half lies past the end (R not a multiple of 256), it loads the even
// CTA's rows instead, so no box starts past the end of a tensor; the outputs of those
// rows are never stored.
__device__ __forceinline__ int32_t load_row0(int32_t w0, int64_t R) {
  return (int64_t)w0 >= R ? w0 - 128 : w0;
}

template <BSrc BS, bool W_MN, bool DW = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(WpairCfg<BS, DW>::kThreads, 1)
qgemm_wpair_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmCodes,
                   const __grid_constant__ CUtensorMap tmScale, const __grid_constant__ CUtensorMap tmTe,
                   const __grid_constant__ CUtensorMap tmWe, const __grid_constant__ CUtensorMap tmDW,
                   const GemmArgs args) {
  static_assert(!(DW && W_MN), "the dense update is a forward-only operand");
  using Cfg = WpairCfg<BS, DW>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BNH = Cfg::BNH, NP = Cfg::NP, SD = Cfg::SD, ST = Cfg::ST,
                SC = Cfg::SC;
  constexpr int SW = Cfg::SW, SWm = SW > 0 ? SW : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sD = smem;                                   // decoded weight (A operand rows of this CTA)
  uint8_t* sT = sD + SD * Cfg::kDBytes;                 // tokens (this CTA's half of B)
  uint8_t* sC = sT + ST * Cfg::kTBytes;                 // codes + scales
  uint8_t* sW = sC + SC * Cfg::kCBytes;                 // DW: this CTA's update chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + SW * Cfg::kDBytes);
  const uint32_t full_d = smem_u32(bars);
  const uint32_t empty_d = full_d + 8 * SD;
  const uint32_t full_t = empty_d + 8 * SD;
  const uint32_t empty_t = full_t + 8 * ST;
  const uint32_t peer_ready = empty_t + 8 * ST;         // even CTA: the odd CTA's chunk g is in
  const uint32_t full_c = peer_ready + 8 * ST;
  const uint32_t empty_c = full_c + 8 * SC;
  const uint32_t acc_full = empty_c + 8 * SC;
  const uint32_t acc_empty = acc_full + 16;             // even CTA: epilogue warps of both CTAs
  const uint32_t drain = acc_full + 32;
  const uint32_t dw_full = drain + 8, dw_empty = dw_full + 8 * SW;   // DW
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * SD + 3 * ST + 2 * SC + 5 + 2 * SW);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SD; ++s) { mbar_init(full_d + 8 * s, NP); mbar_init(empty_d + 8 * s, 1); }
    for (int s = 0; s < ST; ++s) {
      mbar_init(full_t + 8 * s, 1); mbar_init(empty_t + 8 * s, 1); mbar_init(peer_ready + 8 * s, 1);
    }
    for (int s = 0; s < SC; ++s) { mbar_init(full_c + 8 * s, 1); mbar_init(empty_c + 8 * s, NP); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full + 8 * i, 1); mbar_init(acc_empty + 8 * i, 8); }
    mbar_init(drain, 1);
    for (int s = 0; s < SW; ++s) { mbar_init(dw_full + 8 * s, 1); mbar_init(dw_empty + 8 * s, NP); }
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmT);
    if (args.n_ext) tma_prefetch_desc(&tmTe);
  }
  if (warp == 6 && lane == 0) {
    tma_prefetch_desc(&tmCodes);
    tma_prefetch_desc(&tmScale);
    if (DW) tma_prefetch_desc(&tmDW);
  }
  if (warp == 7 && lane == 0 && args.n_ext) tma_prefetch_desc(&tmWe);
  if (warp == 5) tmem_alloc_pair(smem_u32(tmem_holder), Cfg::kTmemCols);
  tc_fence_before();
  cluster_sync();                                       // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // pair tiles: 256 weight rows x 256 tokens, weight-row tiles fastest
  const int64_t w_tiles = (args.R + 2 * BM - 1) / (2 * BM);
  const int64_t tiles = w_tiles * ((args.Cn + BN - 1) / BN);
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int kc_main = (int)((args.Kc + 63) / 64);
  const int kc_total = kc_main + args.n_ext;
  const uint64_t lim = args.timeout_ns;
  const uint32_t row_off = rank * BM;                   // this CTA's rows within the pair tile

  if (warp < 4) {
    // ---- epilogue: this CTA's 128 weight rows (TMEM lanes) x the tile's 256 tokens ----
    const uint32_t acc_empty_lead = mapa_shared(acc_empty, 0);
    uint32_t tcount = 0;
    for (int64_t t = pair; t < tiles; t += npairs, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      const bool okw = mbar_wait(acc_full + 8 * acc, aph, lim, abort_word);
      if (!__all_sync(0xFFFFFFFFu, okw)) break;
      tc_fence_after();
      const int64_t w0 = (t % w_tiles) * 2 * BM + row_off, t0 = (t / w_tiles) * BN;
      const int64_t wrow = w0 + warp * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * BN + cc, v);
        if (t0 + cc < args.Cn) epilogue_store_t(args, wrow, t0 + cc, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_lead + 8 * acc);
    }
  } else if (warp == 4 && lane == 0) {
    // ---- this CTA's token rows -> T ring ----
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = pair; t < tiles && ok; t += npairs) {
      int32_t t0 = (int32_t)((t / w_tiles) * BN + rank * BNH);
      if (t0 >= args.Cn) t0 -= BNH;                      // whole half past the tokens: as load_row0
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t s = g % ST, ph = (g / ST) & 1;
        if (!mbar_wait(empty_t + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
        const uint32_t fb = full_t + 8 * s;
        mbar_arrive_expect_tx(fb, Cfg::kTBytes);
        if (kc < kc_main) tma_load_2d(smem_u32(sT + s * Cfg::kTBytes), &tmT, fb, kc * 64, t0);
        else tma_load_2d(smem_u32(sT + s * Cfg::kTBytes), &tmTe, fb, (kc - kc_main) * 64, t0);
      }
    }
    if (!ok || *abort_word)
      for (uint32_t j = (g > (uint32_t)ST ? g - ST : 0); j < g; ++j) drain_wait(full_t + 8 * (j % ST), (j / ST) & 1);
  } else if (warp == 6 && lane == 0) {
    // ---- this CTA's weight codes + block scales -> C ring ----
    uint32_t gc = 0;
    bool ok = true;
    for (int64_t t = pair; t < tiles && ok; t += npairs) {
      const int32_t w0 = load_row0((int32_t)((t % w_tiles) * 2 * BM + row_off), args.R);
      for (int kc = 0; kc < kc_main; ++kc, ++gc) {
        const uint32_t s = gc % SC, ph = (gc / SC) & 1;
        if (!mbar_wait(empty_c + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
        const uint32_t fb = full_c + 8 * s;
        const uint32_t dst = smem_u32(sC + s * Cfg::kCBytes);
        if (!W_MN) {
          mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + BM * 4);
          tma_load_2d(dst, &tmCodes, fb, kc * (BS == BSrc::NF4 ? 32 : 64), w0);
          tma_load_2d(dst + Cfg::kCodeBytes, &tmScale, fb, w0, kc);
        } else {
          mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + 1024);
          tma_load_2d(dst, &tmCodes, fb, BS == BSrc::NF4 ? w0 / 2 : w0, kc * 64);
          tma_load_2d(dst + Cfg::kCodeBytes, &tmScale, fb, (w0 / 64) & ~3, kc * 64);
        }
        if (DW) {
          // this CTA's 128 rows of the update, columns kc*64..+64, into its own ring
          const uint32_t sw = gc % SWm, pw = (gc / SWm) & 1;
          if (!mbar_wait(dw_empty + 8 * sw, pw ^ 1, lim, abort_word)) { ok = false; ++gc; break; }
          mbar_arrive_expect_tx(dw_full + 8 * sw, Cfg::kDBytes);
          tma_load_2d(smem_u32(sW + sw * Cfg::kDBytes), &tmDW, dw_full + 8 * sw, kc * 64, w0);
        }
      }
    }
    if (!ok || *abort_word) {
      for (uint32_t j = (gc > (uint32_t)SC ? gc - SC : 0); j < gc; ++j) drain_wait(full_c + 8 * (j % SC), (j / SC) & 1);
      if (DW) {
        const uint32_t gdw = ok ? gc : gc - 1;
        for (uint32_t j = (gdw > (uint32_t)SWm ? gdw - SWm : 0); j < gdw; ++j) drain_wait(dw_full + 8 * (j % SWm), (j / SWm) & 1);
      }
    }
  } else if (warp == 5 && lane == 0 && leader) {
    // ---- MMA issuer (even CTA) ----
    constexpr uint32_t kIdMain = idesc_bf16_f32(2 * BM, BN, W_MN ? 1 : 0, 0);
    constexpr uint32_t kIdExt = idesc_bf16_f32(2 * BM, BN, 0, 0);
    uint32_t g = 0, tcount = 0;
    bool ok = true;
    for (int64_t t = pair; t < tiles && ok; t += npairs, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      if (!mbar_wait(acc_empty + 8 * acc, aph ^ 1, lim, abort_word)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t sd = g % SD, pd = (g / SD) & 1, st = g % ST, pt = (g / ST) & 1;
        if (!mbar_wait(full_t + 8 * st, pt, lim, abort_word)) { ok = false; break; }
        if (!mbar_wait(full_d + 8 * sd, pd, lim, abort_word)) { ok = false; break; }
        if (!mbar_wait(peer_ready + 8 * st, pt, lim, abort_word)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_base = smem_u32(sD + sd * Cfg::kDBytes);
        const uint32_t t_base = smem_u32(sT + st * Cfg::kTBytes);
        const bool ext = kc >= kc_main;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = (!W_MN || ext) ? smem_desc_sw128(d_base + k * 32, 16, 1024)
                                             : smem_desc_sw128(d_base + k * 2048, 8192, 1024);
          const uint64_t bd = smem_desc_sw128(t_base + k * 32, 16, 1024);
          tc_mma_pair(d_tmem, ad, bd, ext ? kIdExt : kIdMain, (kc > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit_pair_mc(empty_d + 8 * sd, 0x3);
        tc_commit_pair_mc(empty_t + 8 * st, 0x3);
      }
      if (!ok) break;
      tc_commit_pair_mc(acc_full + 8 * acc, 0x3);
    }
    if (!ok || *abort_word) { tc_commit_pair(drain); drain_wait(drain, 0); }
  } else if (warp == 5 && lane == 0) {
    // ---- relay (odd CTA): tell the even CTA when a stage is full here ----
    const uint32_t ready_lead = mapa_shared(peer_ready, 0);
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = pair; t < tiles && ok; t += npairs) {
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t sd = g % SD, pd = (g / SD) & 1, st = g % ST, pt = (g / ST) & 1;
        if (!mbar_wait(full_t + 8 * st, pt, lim, abort_word)) { ok = false; break; }
        if (!mbar_wait(full_d + 8 * sd, pd, lim, abort_word)) { ok = false; break; }
        mbar_arrive_remote(ready_lead + 8 * st);      // never laps: the MMA frees slots first
      }
    }
  } else if (warp >= 7) {
    // ---- decode: C ring -> D ring (bf16, swizzled UMMA layout), two lanes per block ----
    const int tid = threadIdx.x - 7 * 32;                        // 0..255
    const int blk = tid >> 1, half = tid & 1;                    // block 0..127
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = args.q[i];
    int code_off, j_row = 0, gi = 0;
    uint32_t d_off, key;
    if (!W_MN) {
      code_off = blk * (BS == BSrc::NF4 ? 32 : 64);
      d_off = blk * 128;
      key = blk & 7;
    } else {
      j_row = blk & 63;
      gi = blk >> 6;
      code_off = j_row * (BS == BSrc::NF4 ? 64 : 128) + gi * (BS == BSrc::NF4 ? 32 : 64);
      d_off = gi * 8192 + (j_row >> 3) * 1024 + (j_row & 7) * 128;
      key = j_row & 7;
    }
    uint32_t gc = 0, gd = 0, last_s = 0, last_p = 0;
    bool ok = true, ext_issued = false;
    for (int64_t t = pair; t < tiles && ok; t += npairs) {
      const int32_t w0 = load_row0((int32_t)((t % w_tiles) * 2 * BM + row_off), args.R);
      const int scale_idx = !W_MN ? blk : j_row * 4 + ((w0 / 64) & 3) + gi;
      for (int kc = 0; kc < kc_total; ++kc, ++gd) {
        const uint32_t sd = gd % SD, pd = (gd / SD) & 1;
        if (kc >= kc_main) {
          const bool wb = mbar_wait(empty_d + 8 * sd, pd ^ 1, lim, abort_word);
          if (!__all_sync(0xFFFFFFFFu, wb)) { ok = false; break; }
          if (lane == 0) {
            const uint32_t fb = full_d + 8 * sd;
            if (warp == 7) {
              mbar_arrive_expect_tx(fb, Cfg::kDBytes);
              tma_load_2d(smem_u32(sD + sd * Cfg::kDBytes), &tmWe, fb, (kc - kc_main) * 64, w0);
              ext_issued = true;
              last_s = sd;
              last_p = pd;
            } else {
              mbar_arrive(fb);
            }
          }
          continue;
        }
        const uint32_t sc = gc % SC, pc = (gc / SC) & 1;
        const bool w1 = mbar_wait(full_c + 8 * sc, pc, lim, abort_word);
        const uint32_t sw = DW ? gc % SWm : 0, pw = DW ? (gc / SWm) & 1 : 0;
        const bool w3 = w1 && (!DW || mbar_wait(dw_full + 8 * sw, pw, lim, abort_word));
        const bool w2 = w3 && mbar_wait(empty_d + 8 * sd, pd ^ 1, lim, abort_word);
        if (!__all_sync(0xFFFFFFFFu, w2)) { ok = false; break; }
        const uint8_t* cst = sC + sc * Cfg::kCBytes;
        const float sv = reinterpret_cast<const float*>(cst + Cfg::kCodeBytes)[scale_idx];
        uint4* d = reinterpret_cast<uint4*>(sD + sd * Cfg::kDBytes + d_off);
        const uint4* u = reinterpret_cast<const uint4*>(sW + sw * Cfg::kDBytes + d_off);
        auto put = [&](int i, uint4 v) {
          if (DW) {
            const uint4 x = u[i];
            v = make_uint4(add_bf16x2(v.x, x.x), add_bf16x2(v.y, x.y), add_bf16x2(v.z, x.z), add_bf16x2(v.w, x.w));
          }
          d[i] = v;
        };
        if constexpr (BS == BSrc::NF4) {
          const uint4 cv = reinterpret_cast<const uint4*>(cst + code_off)[half];
          uint32_t L[2], H[2];
          nf4_table(q, sv, L, H);
          const int c0i = 4 * half;
          put((c0i + 0) ^ key, nf4_decode8(cv.x, L, H));
          put((c0i + 1) ^ key, nf4_decode8(cv.y, L, H));
          put((c0i + 2) ^ key, nf4_decode8(cv.z, L, H));
          put((c0i + 3) ^ key, nf4_decode8(cv.w, L, H));
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(cst + code_off) + 2 * half;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 w = src[h];
            const int c = 4 * half + 2 * h;
            put(c ^ key, int8_decode8(w.x, w.y, sv));
            put((c + 1) ^ key, int8_decode8(w.z, w.w, sv));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(full_d + 8 * sd);
          mbar_arrive(empty_c + 8 * sc);
          if (DW) mbar_arrive(dw_empty + 8 * sw);
        }
        ++gc;
      }
    }
    if ((!ok || *abort_word) && warp == 7 && lane == 0 && ext_issued)
      drain_wait(full_d + 8 * last_s, last_p);           // our last extension copy (bounded)
  }

  // Neither CTA leaves (or frees TMEM) while the pair's MMAs may still read its shared
  // memory or the other CTA may still arrive on its barriers.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 5) tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  if (threadIdx.x == 0 && *abort_word) raise_flag(args.flag, kFlagTimeout);
}

}  // namespace qlb
