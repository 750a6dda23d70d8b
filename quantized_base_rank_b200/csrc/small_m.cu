// Decode-shaped forward (M <= 16 tokens): Y = X W'^T + s (X A^T) B^T in one launch.
//
// This is the HBM-bound case of the quantised linear (QLoRA page, aizip.shop/methodologies/
// qlora, "limitations": the dequantisation cost is paid at inference): the whole weight is
// read once as 4-bit codes and every byte must be decoded at memory speed.
//
// Layout of the work:
//  - a cluster of kCS = 8 CTAs owns 128 consecutive weight rows; its CTAs split K into
//    contiguous ranges of 256-wide units (4 quantisation blocks);
//  - each warp owns 16 weight rows; lane (g, q) = (lane / 4, lane % 4) decodes block q of
//    every unit for rows g and g+8, straight into the A fragments of mma.sync m16n8k16
//    (W' rows x k), with X as the 8-token B operand. The contraction order is permuted
//    consistently for both operands (step s of a unit uses k = 64q + 4s + {0..3}), so a
//    lane's 64 elements of a block come from one 32-byte code row and one table;
//  - the adapter term enters per K-range by linearity: each CTA forms T_kr = X_kr A_kr^T
//    and adds B (s T_kr) to its partial sums;
//  - the 8 partial sums of a row group are reduced in fixed rank order through
//    distributed shared memory, so the result is deterministic and no workspace or atomic
//    is needed. T = sum of the T_kr is reduced the same way for T_save.
// The codes of the next unit are loaded while the current one is decoded.
#include "common.cuh"

namespace qlb {

constexpr int kCS = 8;            // CTAs per cluster (K split)
constexpr int kRowsPerCta = 128;  // 8 warps x 16 rows

struct SmallArgs {
  const uint16_t* X; const uint16_t* A; const uint16_t* B;
  int64_t M, N, K;
  int r;
  float s;
  int fmt;
  const uint8_t* codes; const int8_t* qabsmax; const float* gscale; const float* mean;
  const float* absmax;
  uint16_t* Y; uint16_t* T_save;
  int kr_max;                      // max K-range per CTA, in elements
  float q[16];
};

__device__ __forceinline__ uint32_t prmt_s(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NF4 block table (symmetric fold, see gemm.cuh): low/high bytes of the 8 entries
// bf16(fp32(q_{8+i} * a')).
__device__ __forceinline__ void small_nf4_table(const float* q, float ar, uint32_t (&L)[2], uint32_t (&H)[2]) {
  const uint32_t P01 = pack_bf16x2(__fmul_rn(q[8], ar), __fmul_rn(q[9], ar));
  const uint32_t P23 = pack_bf16x2(__fmul_rn(q[10], ar), __fmul_rn(q[11], ar));
  const uint32_t P45 = pack_bf16x2(__fmul_rn(q[12], ar), __fmul_rn(q[13], ar));
  const uint32_t P67 = pack_bf16x2(__fmul_rn(q[14], ar), __fmul_rn(q[15], ar));
  L[0] = prmt_s(P01, P23, 0x6420u);
  H[0] = prmt_s(P01, P23, 0x7531u);
  L[1] = prmt_s(P45, P67, 0x6420u);
  H[1] = prmt_s(P45, P67, 0x7531u);
}

__device__ __forceinline__ uint4 small_nf4_decode8(uint32_t w, const uint32_t (&L)[2], const uint32_t (&H)[2]) {
  const uint32_t m8 = w & 0x88888888u;
  const uint32_t f = m8 - (m8 >> 3);
  const uint32_t idx = (w ^ f ^ 0x77777777u) & 0x77777777u;
  const uint32_t m84 = m8 << 4;
  uint4 o;
  uint32_t sg = prmt_s(m84, m8, 0xD9C8u);
  uint32_t lo = prmt_s(L[0], L[1], idx);
  uint32_t hi = prmt_s(H[0], H[1], idx) ^ (~sg & 0x80808080u);
  o.x = prmt_s(lo, hi, 0x5140u);
  o.y = prmt_s(lo, hi, 0x7362u);
  sg = prmt_s(m84, m8, 0xFBEAu);
  const uint32_t idxh = idx >> 16;
  lo = prmt_s(L[0], L[1], idxh);
  hi = prmt_s(H[0], H[1], idxh) ^ (~sg & 0x80808080u);
  o.z = prmt_s(lo, hi, 0x5140u);
  o.w = prmt_s(lo, hi, 0x7362u);
  return o;
}

// 4 int8 codes -> 2 bf16x2 words (exact code recovery through a magic float)
__device__ __forceinline__ uint2 small_int8_decode4(uint32_t w, float sc) {
  const uint32_t wv = w ^ 0x80808080u;
  float f0 = __uint_as_float(prmt_s(wv, 0x4B000000u, 0x7540u));
  float f1 = __uint_as_float(prmt_s(wv, 0x4B000000u, 0x7541u));
  float f2 = __uint_as_float(prmt_s(wv, 0x4B000000u, 0x7542u));
  float f3 = __uint_as_float(prmt_s(wv, 0x4B000000u, 0x7543u));
  f0 = __fmul_rn(__fsub_rn(f0, 8388736.0f), sc);
  f1 = __fmul_rn(__fsub_rn(f1, 8388736.0f), sc);
  f2 = __fmul_rn(__fsub_rn(f2, 8388736.0f), sc);
  f3 = __fmul_rn(__fsub_rn(f3, 8388736.0f), sc);
  return make_uint2(pack_bf16x2(f0, f1), pack_bf16x2(f2, f3));
}

// The codes and scale of one block (row, block index) for one lane.
template <int FMT>
struct UnitRegs {
  uint4 c[FMT == QL_FMT_NF4_DQ ? 2 : 4];
  float sc;
};

template <int FMT>
__device__ __forceinline__ void load_block_regs(const SmallArgs& a, int64_t row, int64_t kb, float mu,
                                                UnitRegs<FMT>& u) {
  const int64_t KB = a.K >> 6;
  constexpr int NV = FMT == QL_FMT_NF4_DQ ? 2 : 4;
  if (row >= a.N || kb >= KB) {
#pragma unroll
    for (int i = 0; i < NV; ++i) u.c[i] = make_uint4(0u, 0u, 0u, 0u);
    u.sc = 0.0f;
    return;
  }
  const int64_t blk = row * KB + kb;
  const uint4* src = reinterpret_cast<const uint4*>(a.codes + blk * (FMT == QL_FMT_NF4_DQ ? 32 : 64));
#pragma unroll
  for (int i = 0; i < NV; ++i) u.c[i] = __ldg(src + i);
  if (FMT == QL_FMT_NF4_DQ)
    u.sc = __fadd_rn(__fmul_rn((float)__ldg(a.qabsmax + blk), __ldg(a.gscale + (blk >> 8))), mu);
  else
    u.sc = __fdiv_rn(__ldg(a.absmax + blk), 127.0f);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local)), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <int NT, int FMT>
__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(256)
small_m_fwd_kernel(const SmallArgs a) {
  constexpr int NTT = NT / 8;                       // token tiles of 8
  extern __shared__ __align__(16) uint8_t sm[];
  const int RP = (a.r + 15) & ~15;                  // rank padded to the j-tile of 16
  uint16_t* sX = reinterpret_cast<uint16_t*>(sm);   // [NT][kr_max] bf16
  float* sTp = reinterpret_cast<float*>(sm + (size_t)NT * a.kr_max * 2);   // [8 warps][RP][NT]
  float* sT = sTp + 8 * RP * NT;                    // [RP][NT] this CTA's T_kr
  float* sD = sT + RP * NT;                         // [128 rows][NT] partial Y

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const uint32_t rank = cluster_rank();
  const int64_t n0 = (int64_t)(blockIdx.x / kCS) * kRowsPerCta;
  const int64_t U = (a.K + 255) / 256;
  const int64_t u0 = rank * U / kCS, u1 = (rank + 1) * U / kCS;
  const int64_t k0 = u0 * 256;
  const int kr = (int)((u1 - u0) * 256);
  const float mu = FMT == QL_FMT_NF4_DQ ? __ldg(a.mean) : 0.0f;

  // first unit's codes go out before anything else
  const int64_t row_g = n0 + warp * 16 + g, row_h = row_g + 8;
  UnitRegs<FMT> cg, ch;
  if (u0 < u1) {
    load_block_regs<FMT>(a, row_g, u0 * 4 + q, mu, cg);
    load_block_regs<FMT>(a, row_h, u0 * 4 + q, mu, ch);
  }

  // X[:, k0 : k0 + kr] -> smem, zero beyond M and K
  for (int i = threadIdx.x; i < NT * kr / 8; i += blockDim.x) {
    const int tok = i / (kr / 8), kk = (i % (kr / 8)) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    const int64_t k = k0 + kk;
    if (tok < a.M && k < a.K) v = *reinterpret_cast<const uint4*>(a.X + tok * a.K + k);
    *reinterpret_cast<uint4*>(sX + (size_t)tok * a.kr_max + kk) = v;
  }
  __syncthreads();

  // ---- T_kr = X_kr A_kr^T, k16 steps split over the 8 warps ----
  for (int jt = 0; jt < RP / 16; ++jt) {
    float dt[NTT][4];
#pragma unroll
    for (int t = 0; t < NTT; ++t) dt[t][0] = dt[t][1] = dt[t][2] = dt[t][3] = 0.0f;
    const int j_g = jt * 16 + g, j_h = j_g + 8;
    for (int st = warp; st < kr / 16; st += 8) {
      const int kl = st * 16 + 2 * q;
      const int64_t k = k0 + kl;
      uint32_t av[4] = {0u, 0u, 0u, 0u};
      if (k < a.K) {
        if (j_g < a.r) {
          av[0] = *reinterpret_cast<const uint32_t*>(a.A + j_g * a.K + k);
          av[2] = *reinterpret_cast<const uint32_t*>(a.A + j_g * a.K + k + 8);
        }
        if (j_h < a.r) {
          av[1] = *reinterpret_cast<const uint32_t*>(a.A + j_h * a.K + k);
          av[3] = *reinterpret_cast<const uint32_t*>(a.A + j_h * a.K + k + 8);
        }
      }
#pragma unroll
      for (int t = 0; t < NTT; ++t) {
        const uint16_t* xr = sX + (size_t)(t * 8 + g) * a.kr_max + kl;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(xr + 8);
        mma_bf16_16816(dt[t], av[0], av[1], av[2], av[3], b0, b1);
      }
    }
#pragma unroll
    for (int t = 0; t < NTT; ++t) {
      float* p = sTp + ((size_t)warp * RP) * NT;
      p[(j_g)*NT + t * 8 + 2 * q] = dt[t][0];
      p[(j_g)*NT + t * 8 + 2 * q + 1] = dt[t][1];
      p[(j_h)*NT + t * 8 + 2 * q] = dt[t][2];
      p[(j_h)*NT + t * 8 + 2 * q + 1] = dt[t][3];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < RP * NT; i += blockDim.x) {
    float acc = 0.0f;
    for (int w = 0; w < 8; ++w) acc += sTp[(size_t)w * RP * NT + i];
    sT[i] = acc;
  }

  // ---- main loop: decode into A fragments, X from smem as the B fragments ----
  float d[NTT][4];
#pragma unroll
  for (int t = 0; t < NTT; ++t) d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.0f;
  for (int64_t u = u0; u < u1; ++u) {
    UnitRegs<FMT> ng, nh;
    if (u + 1 < u1) {
      load_block_regs<FMT>(a, row_g, (u + 1) * 4 + q, mu, ng);
      load_block_regs<FMT>(a, row_h, (u + 1) * 4 + q, mu, nh);
    }
    const uint16_t* xb = sX + (u - u0) * 256 + 64 * q;
    if constexpr (FMT == QL_FMT_NF4_DQ) {
      uint32_t Lg[2], Hg[2], Lh[2], Hh[2];
      small_nf4_table(a.q, cg.sc, Lg, Hg);
      small_nf4_table(a.q, ch.sc, Lh, Hh);
      const uint32_t wg[8] = {cg.c[0].x, cg.c[0].y, cg.c[0].z, cg.c[0].w, cg.c[1].x, cg.c[1].y, cg.c[1].z, cg.c[1].w};
      const uint32_t wh[8] = {ch.c[0].x, ch.c[0].y, ch.c[0].z, ch.c[0].w, ch.c[1].x, ch.c[1].y, ch.c[1].z, ch.c[1].w};
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) {
        const uint4 eg = small_nf4_decode8(wg[w8], Lg, Hg);
        const uint4 eh = small_nf4_decode8(wh[w8], Lh, Hh);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int s = 2 * w8 + half;
          const uint32_t a0 = half ? eg.z : eg.x, a2 = half ? eg.w : eg.y;
          const uint32_t a1 = half ? eh.z : eh.x, a3 = half ? eh.w : eh.y;
#pragma unroll
          for (int t = 0; t < NTT; ++t) {
            const uint2 bx = *reinterpret_cast<const uint2*>(xb + (size_t)(t * 8 + g) * a.kr_max + 4 * s);
            mma_bf16_16816(d[t], a0, a1, a2, a3, bx.x, bx.y);
          }
        }
      }
    } else {
      const uint32_t wg[16] = {cg.c[0].x, cg.c[0].y, cg.c[0].z, cg.c[0].w, cg.c[1].x, cg.c[1].y, cg.c[1].z, cg.c[1].w,
                               cg.c[2].x, cg.c[2].y, cg.c[2].z, cg.c[2].w, cg.c[3].x, cg.c[3].y, cg.c[3].z, cg.c[3].w};
      const uint32_t wh[16] = {ch.c[0].x, ch.c[0].y, ch.c[0].z, ch.c[0].w, ch.c[1].x, ch.c[1].y, ch.c[1].z, ch.c[1].w,
                               ch.c[2].x, ch.c[2].y, ch.c[2].z, ch.c[2].w, ch.c[3].x, ch.c[3].y, ch.c[3].z, ch.c[3].w};
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        const uint2 eg = small_int8_decode4(wg[s], cg.sc);
        const uint2 eh = small_int8_decode4(wh[s], ch.sc);
#pragma unroll
        for (int t = 0; t < NTT; ++t) {
          const uint2 bx = *reinterpret_cast<const uint2*>(xb + (size_t)(t * 8 + g) * a.kr_max + 4 * s);
          mma_bf16_16816(d[t], eg.x, eh.x, eg.y, eh.y, bx.x, bx.y);
        }
      }
    }
    if (u + 1 < u1) { cg = ng; ch = nh; }
  }

  // ---- adapter term of this K-range: D += B[rows, :] (s T_kr) ----
  __syncthreads();
  for (int jt = 0; jt < RP / 16; ++jt) {
    const int j0 = jt * 16 + 2 * q;
    auto bload = [&](int64_t row, int j) -> uint32_t {
      if (row >= a.N) return 0u;
      const uint32_t lo = j < a.r ? a.B[row * a.r + j] : 0u;
      const uint32_t hi = j + 1 < a.r ? a.B[row * a.r + j + 1] : 0u;
      return lo | (hi << 16);
    };
    const uint32_t a0 = bload(row_g, j0), a1 = bload(row_h, j0);
    const uint32_t a2 = bload(row_g, j0 + 8), a3 = bload(row_h, j0 + 8);
#pragma unroll
    for (int t = 0; t < NTT; ++t) {
      const int tok = t * 8 + g;
      const uint32_t b0 = pack_bf16x2(a.s * sT[j0 * NT + tok], a.s * sT[(j0 + 1) * NT + tok]);
      const uint32_t b1 = pack_bf16x2(a.s * sT[(j0 + 8) * NT + tok], a.s * sT[(j0 + 9) * NT + tok]);
      mma_bf16_16816(d[t], a0, a1, a2, a3, b0, b1);
    }
  }

  // ---- partial sums -> smem, then the fixed-order cluster reduction ----
#pragma unroll
  for (int t = 0; t < NTT; ++t) {
    const int rg = warp * 16 + g;
    sD[rg * NT + t * 8 + 2 * q] = d[t][0];
    sD[rg * NT + t * 8 + 2 * q + 1] = d[t][1];
    sD[(rg + 8) * NT + t * 8 + 2 * q] = d[t][2];
    sD[(rg + 8) * NT + t * 8 + 2 * q + 1] = d[t][3];
  }
  cluster_sync_all();
  {
    constexpr int kRowsPerRank = kRowsPerCta / kCS;    // 16
    for (int i = threadIdx.x; i < kRowsPerRank * NT; i += blockDim.x) {
      const int rr = (int)rank * kRowsPerRank + i / NT, tok = i % NT;
      float acc = 0.0f;
      for (uint32_t c = 0; c < kCS; ++c) acc += ld_cluster_f32(sD + rr * NT + tok, c);
      const int64_t row = n0 + rr;
      if (tok < a.M && row < a.N) a.Y[tok * a.N + row] = (uint16_t)float_to_bf16_bits(acc);
    }
    if (a.T_save && blockIdx.x < (unsigned)kCS) {        // first cluster also reduces T
      for (int i = threadIdx.x; i < RP * NT; i += blockDim.x) {
        const int j = i / NT, tok = i % NT;
        if ((int)(j % kCS) != (int)rank) continue;
        float acc = 0.0f;
        for (uint32_t c = 0; c < kCS; ++c) acc += ld_cluster_f32(sT + j * NT + tok, c);
        if (tok < a.M && j < a.r) a.T_save[tok * a.r + j] = (uint16_t)float_to_bf16_bits(acc);
      }
    }
  }
  cluster_sync_all();                                   // keep smem alive for the readers
}

size_t small_m_smem(int NT, int kr_max, int r) {
  const int RP = (r + 15) & ~15;
  return (size_t)NT * kr_max * 2 + (size_t)(8 * RP * NT + RP * NT + kRowsPerCta * NT) * 4;
}

template <int NT, int FMT>
static ql_status launch_small(const SmallArgs& a, cudaStream_t st) {
  auto kern = small_m_fwd_kernel<NT, FMT>;
  const size_t smem = small_m_smem(NT, a.kr_max, a.r);
  if (smem > 227 * 1024) return QL_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const int groups = (int)((a.N + kRowsPerCta - 1) / kRowsPerCta);
  kern<<<groups * kCS, 256, smem, st>>>(a);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

// Host entry used by qlora_linear_fwd when M <= 16.
ql_status small_m_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                          const uint16_t* B, int r, float alpha, uint16_t* Y, uint16_t* T_save,
                          cudaStream_t st) {
  SmallArgs a{};
  a.X = X; a.A = A; a.B = B; a.M = M; a.N = w->N; a.K = w->K; a.r = r; a.s = alpha / (float)r;
  a.fmt = w->fmt;
  a.codes = static_cast<const uint8_t*>(w->codes);
  a.qabsmax = w->qabsmax; a.gscale = w->group_scale; a.mean = w->mean; a.absmax = w->absmax;
  a.Y = Y; a.T_save = T_save;
  const int64_t U = (w->K + 255) / 256;
  a.kr_max = (int)(((U + kCS - 1) / kCS) * 256);
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) a.q[i] = t.q[i];
  ProfScope prof(PK_FWD_SMALL, st, 1);
  if (w->fmt == QL_FMT_NF4_DQ)
    return M <= 8 ? launch_small<8, QL_FMT_NF4_DQ>(a, st) : launch_small<16, QL_FMT_NF4_DQ>(a, st);
  return M <= 8 ? launch_small<8, QL_FMT_INT8_B64>(a, st) : launch_small<16, QL_FMT_INT8_B64>(a, st);
}

}  // namespace qlb
