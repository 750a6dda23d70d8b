// Persistent warp-specialised tcgen05 GEMM with an on-the-fly NF4 / int8 decoding
// producer for the weight operand and a K-extension for the unmerged LoRA term.
//
//   C[R, Cn] = sum_k Aop[R, k] * Bop[Cn, k]  (+ sum_e Aext[R, e] * Bext[Cn, e])
//
// Tiles: 128 rows x BN columns, contraction in chunks of 64 (one 128-byte swizzled
// smem row per operand row). Roles (warp index):
//   0..3  epilogue: TMEM -> registers -> global (one TMEM lane quarter each)
//   4     TMA producer for Aop (and Bop when it is plain bf16), and the extension
//   5     MMA issuer (one elected thread), also owns the TMEM allocation
//   6..   NP decode warps: weight codes -> bf16 rows written straight into the
//         swizzled UMMA layout of the stage's B tile (QLoRA page, "1. NF4" and
//         "2. Double Quantization": w' = q[code] * a', a' rebuilt from the 8-bit constant)
// Accumulators are double-buffered in TMEM so the epilogue of one tile overlaps the
// main loop of the next. Every wait is bounded; a wait that gives up raises the CTA's
// abort word, every role then leaves its loop, and the kernel reports QL_ERR_TIMEOUT
// through the device flag after freeing its TMEM.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace qlb {

enum class BSrc : int { TMA = 0, NF4 = 1, INT8 = 2 };
enum Epi : int { EPI_BF16 = 0, EPI_LORA_T = 1, EPI_LORA_Q = 2, EPI_DA = 3, EPI_DB = 4 };

struct GemmArgs {
  int64_t R, Cn, Kc;     // rows, columns, main contraction length
  int32_t n_ext;         // number of 64-wide extension chunks
  int32_t r;             // adapter rank (epilogue masks)
  // weight operand (decode modes): W [Nw, Kw]
  const uint8_t* codes;
  const int8_t* qabsmax;
  const float* gscale;
  const float* mean;
  const float* absmax;
  int64_t Nw, Kw;
  float q[16];
  // epilogue
  void* out;  int64_t ld_out;
  void* out2; int64_t ld_out2;
  float scale;
  uint64_t timeout_ns;
  int* flag;
};

template <int BN>
struct GemmCfg {
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStages = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr size_t kSmem = (size_t)kStages * (kABytes + kBBytes) + 2048;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// 16-entry bf16 table lookup of 4 nibbles (bits 0..15 of sel16), giving two packed
// bf16x2 words (elements 0,1 and 2,3). L/H hold the low/high bytes of entries
// 0..15 (entry c in byte c%4 of word c/4).
__device__ __forceinline__ void lut4(uint32_t sel16, const uint32_t (&L)[4],
                                     const uint32_t (&H)[4], uint32_t& w01, uint32_t& w23) {
  const uint32_t s7 = sel16 & 0x7777u;
  const uint32_t mask = prmt(sel16 << 4, sel16, 0xD9C8u);   // 0xFF where the code is >= 8
  const uint32_t lo = (prmt(L[2], L[3], s7) & mask) | (prmt(L[0], L[1], s7) & ~mask);
  const uint32_t hi = (prmt(H[2], H[3], s7) & mask) | (prmt(H[0], H[1], s7) & ~mask);
  w01 = prmt(lo, hi, 0x5140u);
  w23 = prmt(lo, hi, 0x7362u);
}

// Decode one block of 64 weight elements (row n of W, block kb of that row) into one
// 128-byte swizzled smem row (chunk c goes to position c ^ key). Rows past the end
// of W are written as zeros.
template <BSrc BS>
__device__ __forceinline__ void decode_block(const GemmArgs& a, float mean0, int64_t n, int64_t kb,
                                             uint8_t* dst, uint32_t key) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  if (n >= a.Nw || kb >= (a.Kw >> 6)) {
#pragma unroll
    for (int c = 0; c < 8; ++c) d[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int64_t blk = n * (a.Kw >> 6) + kb;
  if constexpr (BS == BSrc::NF4) {
    const uint4* src = reinterpret_cast<const uint4*>(a.codes + blk * 32);
    const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
    // a' = fp32(fp32(c8 * s_g) + mean)
    const float ar = __fadd_rn(__fmul_rn((float)__ldg(a.qabsmax + blk), __ldg(a.gscale + (blk >> 8))),
                               mean0);
    // entries 8..15: bf16(fp32(q_c * a')); entries 0..7 are their exact negatives
    const uint32_t P01 = pack_bf16x2(__fmul_rn(a.q[8], ar), __fmul_rn(a.q[9], ar));
    const uint32_t P23 = pack_bf16x2(__fmul_rn(a.q[10], ar), __fmul_rn(a.q[11], ar));
    const uint32_t P45 = pack_bf16x2(__fmul_rn(a.q[12], ar), __fmul_rn(a.q[13], ar));
    const uint32_t P67 = pack_bf16x2(__fmul_rn(a.q[14], ar), __fmul_rn(a.q[15], ar));
    uint32_t L[4], H[4];
    L[2] = prmt(P01, P23, 0x6420u);
    H[2] = prmt(P01, P23, 0x7531u);
    L[3] = prmt(P45, P67, 0x6420u);
    H[3] = prmt(P45, P67, 0x7531u);
    L[0] = prmt(L[3], 0u, 0x0123u);
    H[0] = prmt(H[3], 0u, 0x0123u) ^ 0x80808080u;
    L[1] = prmt(L[2], 0u, 0x0123u);
    H[1] = prmt(H[2], 0u, 0x0123u) ^ 0x80808080u;
    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 o;
      lut4(words[c] & 0xFFFFu, L, H, o.x, o.y);
      lut4(words[c] >> 16, L, H, o.z, o.w);
      d[c ^ key] = o;
    }
  } else {
    // int8: w' = bf16(fp32(c * fp32(a/127))); c recovered exactly from a magic float
    const float sc = __fdiv_rn(__ldg(a.absmax + blk), 127.0f);
    const uint4* src = reinterpret_cast<const uint4*>(a.codes + blk * 64);
    const uint4 q0 = __ldg(src), q1 = __ldg(src + 1), q2 = __ldg(src + 2), q3 = __ldg(src + 3);
    const uint32_t words[16] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w,
                                q2.x, q2.y, q2.z, q2.w, q3.x, q3.y, q3.z, q3.w};
    const uint32_t kMagic = 0x4B000000u;   // 2^23: low byte of the mantissa holds c + 128
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t wv = words[2 * c + h] ^ 0x80808080u;
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
      d[c ^ key] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

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

template <int BN, int NP, bool A_MN, BSrc BS, bool B_MN, int EPI>
__global__ void __launch_bounds__((6 + NP) * 32, 1)
qgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmAe, const __grid_constant__ CUtensorMap tmBe,
             const GemmArgs args) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr bool kDecode = BS != BSrc::TMA;
  static_assert(!kDecode || NP * 32 == BN, "one decode thread per B row");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * Cfg::kBBytes);
  const uint32_t full_a = smem_u32(bars);
  const uint32_t full_b = full_a + 8 * S;
  const uint32_t empty = full_a + 16 * S;
  const uint32_t acc_full = full_a + 24 * S;
  const uint32_t acc_empty = acc_full + 16;
  const uint32_t drain = acc_full + 32;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_a + 8 * s, 1);
      mbar_init(full_b + 8 * s, NP > 0 ? NP : 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + 8 * i, 1);
      mbar_init(acc_empty + 8 * i, 4);
    }
    mbar_init(drain, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    if (BS == BSrc::TMA) tma_prefetch_desc(&tmB);
    if (args.n_ext) { tma_prefetch_desc(&tmAe); tma_prefetch_desc(&tmBe); }
  }
  if (warp == 5) tmem_alloc(smem_u32(tmem_holder), Cfg::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int64_t m_tiles = (args.R + 127) / 128;
  const int64_t n_tiles = (args.Cn + BN - 1) / BN;
  const int64_t tiles = m_tiles * n_tiles;
  const int kc_main = (int)((args.Kc + 63) / 64);
  const int kc_total = kc_main + args.n_ext;
  const uint64_t lim = args.timeout_ns;

  if (warp < 4) {
    // ---------------- epilogue ----------------
    uint32_t tcount = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++tcount) {
      const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
      const bool okw = mbar_wait(acc_full + 8 * acc, aph, lim, abort_word);
      if (!__all_sync(0xFFFFFFFFu, okw)) break;
      tc_fence_after();
      const int64_t r0 = (t / n_tiles) * 128, c0 = (t % n_tiles) * BN;
      const int64_t row = r0 + warp * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * BN + cc, v);
        if (c0 + cc < args.Cn) epilogue_store<EPI>(args, row, c0 + cc, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * acc);
    }
  } else if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int32_t r0 = (int32_t)((t / n_tiles) * 128), c0 = (int32_t)((t % n_tiles) * BN);
        for (int kc = 0; kc < kc_total; ++kc, ++g) {
          const uint32_t s = g % S, ph = (g / S) & 1;
          if (!mbar_wait(empty + 8 * s, ph ^ 1, lim, abort_word)) { ok = false; break; }
          const uint32_t fa = full_a + 8 * s;
          const uint32_t dA = smem_u32(sA + s * Cfg::kABytes);
          const uint32_t dB = smem_u32(sB + s * Cfg::kBBytes);
          if (kc < kc_main) {
            mbar_arrive_expect_tx(fa, Cfg::kABytes + (kDecode ? 0 : Cfg::kBBytes));
            if (!A_MN) {
              tma_load_2d(dA, &tmA, fa, kc * 64, r0);
            } else {
              tma_load_2d(dA, &tmA, fa, r0, kc * 64);
              tma_load_2d(dA + 8192, &tmA, fa, r0 + 64, kc * 64);
            }
            if (!kDecode) {
              if (!B_MN) {
                tma_load_2d(dB, &tmB, fa, kc * 64, c0);
              } else {
#pragma unroll
                for (int i = 0; i < BN / 64; ++i) tma_load_2d(dB + i * 8192, &tmB, fa, c0 + 64 * i, kc * 64);
              }
            }
          } else {
            const int e = kc - kc_main;
            mbar_arrive_expect_tx(fa, Cfg::kABytes + Cfg::kBBytes);
            tma_load_2d(dA, &tmAe, fa, e * 64, r0);
            tma_load_2d(dB, &tmBe, fa, e * 64, c0);
          }
        }
      }
      if (!ok || *abort_word) {
        // let our own copies land before the CTA's shared memory goes away
        for (uint32_t j = (g > (uint32_t)S ? g - S : 0); j < g; ++j) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_a + 8 * (j % S), (j / S) & 1) && globaltimer_ns() - t0 < 200000000ull) {}
        }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t kIdMain = idesc_bf16_f32(128, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
      constexpr uint32_t kIdExt = idesc_bf16_f32(128, BN, 0, 0);
      uint32_t g = 0, tcount = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tcount) {
        const uint32_t acc = tcount & 1, aph = (tcount >> 1) & 1;
        if (!mbar_wait(acc_empty + 8 * acc, aph ^ 1, lim, abort_word)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kc = 0; kc < kc_total; ++kc, ++g) {
          const uint32_t s = g % S, ph = (g / S) & 1;
          if (!mbar_wait(full_a + 8 * s, ph, lim, abort_word)) { ok = false; break; }
          if (kDecode && !mbar_wait(full_b + 8 * s, ph, lim, abort_word)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * Cfg::kABytes);
          const uint32_t b_base = smem_u32(sB + s * Cfg::kBBytes);
          const bool ext = kc >= kc_main;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = (!A_MN || ext) ? smem_desc_sw128(a_base + k * 32, 16, 1024)
                                               : smem_desc_sw128(a_base + k * 2048, 8192, 1024);
            const uint64_t bd = (!B_MN || ext) ? smem_desc_sw128(b_base + k * 32, 16, 1024)
                                               : smem_desc_sw128(b_base + k * 2048, 8192, 1024);
            tc_mma(d_tmem, ad, bd, ext ? kIdExt : kIdMain, (kc > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(empty + 8 * s);
        }
        if (!ok) break;
        tc_commit(acc_full + 8 * acc);
      }
      if (!ok || *abort_word) {
        tc_commit(drain);                       // completes once every issued MMA is done
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 200000000ull) {}
      }
    }
  } else if (kDecode) {
    // ---------------- decode producers ----------------
    const int tid = threadIdx.x - 192;
    const float mean0 = (BS == BSrc::NF4) ? __ldg(args.mean) : 0.0f;
    uint32_t g = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int64_t c0 = (t % n_tiles) * BN;
      for (int kc = 0; kc < kc_total; ++kc, ++g) {
        const uint32_t s = g % S, ph = (g / S) & 1;
        const bool okw = mbar_wait(empty + 8 * s, ph ^ 1, lim, abort_word);
        if (!__all_sync(0xFFFFFFFFu, okw)) { ok = false; break; }
        if (kc < kc_main) {
          uint8_t* bst = sB + s * Cfg::kBBytes;
          if (!B_MN) {
            // K-major tile: smem row u = weight row c0 + u, block kc of that row
            const int u = tid;
            decode_block<BS>(args, mean0, c0 + u, kc, bst + u * 128, (uint32_t)(u & 7));
          } else {
            // MN-major tile: 64-wide groups of output columns (weight input features),
            // rows = weight rows kc*64 + j
            const int j = tid & 63, gi = tid >> 6;
            decode_block<BS>(args, mean0, (int64_t)kc * 64 + j, (c0 >> 6) + gi,
                             bst + gi * 8192 + (j >> 3) * 1024 + (j & 7) * 128, (uint32_t)(j & 7));
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(full_b + 8 * s);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_word) raise_flag(args.flag, kFlagTimeout);
}

}  // namespace qlb
