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
//  - the adapter term enters per K-range by linearity: T_kr = X_kr A_kr^T is formed in the
//    same loop from the same token fragments (adapter rows staged like the tokens), and
//    B (s T_kr) is added to the partial sums;
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
  // Walsh-Hadamard adapter (QW instantiations): F in compressed rows and the transformed
  // tokens Zs [K][16] (bf16, token-contiguous), written by the grid just before
  const int32_t* q_row_ptr; const uint16_t* q_col; const uint16_t* q_c; int64_t q_nnz;
  const uint16_t* q_Zs;
  int* flag;                       // the device status flag (bad sparse indices)
  int kr_max;                      // max K-range per CTA, in elements
  int b_pairs;                     // r even and B 4-byte aligned
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

// The codes and the raw constants of one block (row, block index) for one lane. Loading
// does no arithmetic on the loaded values, so several units' loads can be in flight at
// once; unit_scale() turns the constants into the block scale at first use.
template <int FMT>
struct UnitRegs {
  uint4 c[FMT == QL_FMT_NF4_DQ ? 2 : 4];
  int qa;         // NF4: the int8 double-quantised constant
  float f;        // NF4: the group scale; int8: the fp32 absmax
};

template <int FMT>
__device__ __forceinline__ void load_block_regs(const SmallArgs& a, int64_t row, int64_t kb, UnitRegs<FMT>& u) {
  const int64_t KB = a.K >> 6;
  constexpr int NV = FMT == QL_FMT_NF4_DQ ? 2 : 4;
  if (row >= a.N || kb >= KB) {
#pragma unroll
    for (int i = 0; i < NV; ++i) u.c[i] = make_uint4(0u, 0u, 0u, 0u);
    u.qa = 0;
    u.f = 0.0f;
    return;
  }
  const int64_t blk = row * KB + kb;
  const uint4* src = reinterpret_cast<const uint4*>(a.codes + blk * (FMT == QL_FMT_NF4_DQ ? 32 : 64));
#pragma unroll
  for (int i = 0; i < NV; ++i) u.c[i] = __ldg(src + i);
  if (FMT == QL_FMT_NF4_DQ) {
    u.qa = __ldg(a.qabsmax + blk);
    u.f = __ldg(a.gscale + (blk >> 8));
  } else {
    u.qa = 0;
    u.f = __ldg(a.absmax + blk);
  }
}

// NF4: a' = fp32(fp32(qabsmax * group_scale) + mean); int8: fp32(absmax / 127). Zero for a
// block outside the weight.
template <int FMT>
__device__ __forceinline__ float unit_scale(const UnitRegs<FMT>& u, float mu) {
  if (FMT == QL_FMT_NF4_DQ) return __fadd_rn(__fmul_rn((float)u.qa, u.f), mu);
  return __fdiv_rn(u.f, 127.0f);
}

// Warm L2 with bytes [lo, hi) of each of rows [0, rows) of a byte array whose rows are
// `pitch` bytes apart: one prefetch per 128-byte line, threads t, t + nt, ... taking
// successive lines. Every prefetched address lies inside a requested span.
__device__ __forceinline__ void l2_prefetch_rows(const void* p, int64_t pitch, int64_t rows, int64_t lo,
                                                 int64_t hi, int t, int nt) {
  if (rows <= 0 || hi <= lo) return;
  const int lpr = (int)((hi - lo + 127) >> 7) + 1;   // lines that can touch one row's span
  const int total = (int)rows * lpr;
  for (int i = t; i < total; i += nt) {
    const int row = i / lpr, l = i - row * lpr;
    const uintptr_t b = reinterpret_cast<uintptr_t>(p) + (uintptr_t)(row * pitch + lo);
    const uintptr_t e = b + (uintptr_t)(hi - lo);
    uintptr_t x = ((b >> 7) + (uintptr_t)l) << 7;
    if (x >= e) continue;
    if (x < b) x = b;
    asm volatile("prefetch.global.L2 [%0];" :: "l"(x));
  }
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The last barrier only keeps every CTA's shared memory alive until the other CTAs have
// read it; each of those remote loads is consumed (summed) before the arrive, so the
// arrive needs no release ordering.
__device__ __forceinline__ void cluster_sync_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store two floats at the same shared-memory offset in CTA `rank` of the cluster (8-byte
// aligned). Visible to that CTA after a release/acquire cluster barrier.
__device__ __forceinline__ void st_cluster_f32x2(float* local, uint32_t rank, float x, float y) {
  uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local)), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" :: "r"(remote), "f"(x), "f"(y) : "memory");
}

// Read a float from the same shared-memory offset in CTA `rank` of the cluster. The loads
// stay in program order after the cluster barrier; callers issue several before using any,
// so they are in flight together.
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(local)), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Shared-memory layout of the token rows and adapter rows of a CTA's K-range: the four
// elements a lane feeds to one MMA step (k = 64q + 4s + e of unit ul) are 8 contiguous
// bytes at  row * kRowPitch(units) + ul * 512 + (4s + q) * 8.  With a row pitch of 32 mod 128
// bytes, the 16 lanes of a half-warp (rows g = 0..3, q = 0..3) hit 16 different bank pairs.
__host__ __device__ __forceinline__ int small_row_pitch(int units) { return units * 512 + 32; }

// Adds sum_j c_j Zs[col_j][tok] over each of the 16 rows [r0, r0 + 16) of F (compressed
// rows) to out[(row - r0) * NT + tok] for the NT tokens. Each warp takes two rows, and the
// first batch of both is requested before either is used. Lane = (stream, token pair tp),
// NT/2 token pairs and 64/NT streams; a row's values are read 32 per chunk, U chunks at a
// time, and handed to the streams by shuffles; each lane gathers
// its value's two tokens (one 4-byte load from the token-contiguous Zs) and keeps their
// fp32 sums; a fixed xor butterfly combines the streams. Columns at or past K and row
// offsets outside [0, nnz] are skipped and raise the bad-index flag. Call after the
// dependency wait (Zs is the previous grid's output) and a __syncthreads.
template <int NT>
__device__ __forceinline__ void qwha_rows_add(const SmallArgs& a, int64_t r0, float* out) {
  constexpr int TP = NT / 2, NS = 32 / TP;
  constexpr int U = NT == 8 ? 8 : 4;                 // chunks in flight per row: 256 / 128 values
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stream = lane / TP, tp = lane % TP;
  bool bad = false;
  // the warp's two rows: bounds, then the first batch of both rows, before any is used
  int jb[2], je[2];
  uint32_t wv[2][U];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t n = r0 + 2 * warp + i;
    jb[i] = je[i] = 0;
    if (n < a.N) {
      jb[i] = __ldg(a.q_row_ptr + n);
      je[i] = __ldg(a.q_row_ptr + n + 1);
      if (jb[i] < 0 || (int64_t)je[i] > a.q_nnz || jb[i] > je[i]) {
        bad = true;
        jb[i] = je[i] = 0;
      }
    }
  }
  auto load_batch = [&](int i, int jc, uint32_t (&w)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int jj = jc + 32 * u + lane;
      w[u] = jj < je[i] ? (uint32_t)__ldg(a.q_col + jj) | ((uint32_t)__ldg(a.q_c + jj) << 16) : 0u;
      if ((int64_t)(w[u] & 0xFFFFu) >= a.K) {
        bad = true;
        w[u] = 0u;
      }
    }
  };
  load_batch(0, jb[0], wv[0]);
  load_batch(1, jb[1], wv[1]);
  // the gathers of CH chunks, all issued before any is used (a value of 0 gathers column 0
  // and adds nothing)
  auto gather = [&](const uint32_t* w, int CHn, float& a0, float& a1) {
    uint32_t z[U * TP];
    uint32_t we[U * TP];
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int it = 0; it < TP; ++it) {
        if (u < CHn) {
          we[u * TP + it] = __shfl_sync(0xffffffffu, w[u], it * NS + stream);
          z[u * TP + it] =
              __ldg(reinterpret_cast<const uint32_t*>(a.q_Zs + (size_t)(we[u * TP + it] & 0xFFFFu) * 16) + tp);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int it = 0; it < TP; ++it) {
        if (u < CHn) {
          const float cv = __uint_as_float(we[u * TP + it] & 0xFFFF0000u);
          a0 = fmaf(cv, __uint_as_float(z[u * TP + it] << 16), a0);
          a1 = fmaf(cv, __uint_as_float(z[u * TP + it] & 0xFFFF0000u), a1);
        }
      }
    }
  };
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float a0 = 0.0f, a1 = 0.0f;
    for (int jc = jb[i]; jc < je[i]; jc += 32 * U) {
      if (jc != jb[i]) load_batch(i, jc, wv[i]);
      // warp-uniform: a short batch (most rows) takes the two-chunk form
      if (je[i] - jc <= 64) gather(wv[i], 2, a0, a1);
      else gather(wv[i], U, a0, a1);
    }
#pragma unroll
    for (int off = TP; off < 32; off <<= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, off);
      a1 += __shfl_xor_sync(0xffffffffu, a1, off);
    }
    const int rr = 2 * warp + i;
    if (stream == 0 && r0 + rr < a.N) {
      out[rr * NT + 2 * tp] += a0;
      out[rr * NT + 2 * tp + 1] += a1;
    }
  }
  if (bad) raise_flag(a.flag, kFlagBadIndex);
}

// QW: the Walsh-Hadamard adapter's sparse sums (QWHA page, gist.science/ko/paper/2509.17428,
// section 2.1: Delta W x = F (H^{-1} x)) for the 16 rows this CTA reduces are added to its
// partial sums before the cluster reduction, so they reach Y with its one rounding. Only
// with JT = 0 (no LoRA part).
template <int NT, int FMT, int JT, bool QW = false>
__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(256, 2)
small_m_fwd_kernel(const SmallArgs a) {
  constexpr int NTT = NT / 8;                       // token tiles of 8
  constexpr int RP = JT * 16;                       // rank padded to j-tiles of 16
  extern __shared__ __align__(16) uint8_t sm[];
  const int64_t U = (a.K + 255) / 256;
  const int units_max = (int)((U + kCS - 1) / kCS);
  const int pitch = small_row_pitch(units_max);
  uint8_t* sX = sm;                                 // [NT][pitch]
  uint8_t* sA = sX + (size_t)NT * pitch;            // [RP][pitch]
  float* sTw = reinterpret_cast<float*>(sA + (size_t)RP * pitch);   // [8 warps][RP][NT]
  float* sD = sTw + 8 * RP * NT;                    // [128 rows][NT] partial Y

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const uint32_t rank = cluster_rank();
  const int64_t n0 = (int64_t)(blockIdx.x / kCS) * kRowsPerCta;
  const int64_t u0 = rank * U / kCS, u1 = (rank + 1) * U / kCS;
  const int nunits = (int)(u1 - u0);
  const int64_t k0 = u0 * 256;

  // The next launch on the stream may start now and warm L2 with its own weight while
  // this one finishes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // First half of a cluster barrier whose wait, just before the partial sums are stored
  // into other CTAs' shared memory, guarantees that every CTA of the cluster has started.
  if constexpr (!QW) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // Before the dependency wait this grid only warms L2 with what it is about to read: the
  // codes and constants of its blocks, the adapter rows of its K-range, its rows of B and
  // the token rows. The grid before it on the stream (a quantise, an adapter expansion,
  // the previous layer) may still be writing any of these, and its writes are visible
  // only after the wait; L2 is the point of coherence, so a prefetch never makes a later
  // load return stale data. Every load proper comes after the wait.
  {
    const int64_t rows = a.N - n0 < kRowsPerCta ? a.N - n0 : kRowsPerCta;
    const int64_t KB = a.K >> 6, kend = u1 * 256 < a.K ? u1 * 256 : a.K;
    const int t = threadIdx.x;
    if (FMT == QL_FMT_NF4_DQ) {
      l2_prefetch_rows(a.codes + n0 * (a.K >> 1), a.K >> 1, rows, k0 >> 1, kend >> 1, t, 256);
      l2_prefetch_rows(a.qabsmax + n0 * KB, KB, rows, u0 * 4, (kend + 63) >> 6, t, 256);
      const int64_t g0 = (n0 * KB) >> 8, g1 = ((n0 + rows) * KB - 1) >> 8;
      l2_prefetch_rows(a.gscale, 0, 1, g0 * 4, g1 * 4 + 4, t, 256);
    } else {
      l2_prefetch_rows(a.codes + n0 * a.K, a.K, rows, k0, kend, t, 256);
      l2_prefetch_rows(a.absmax + n0 * KB, KB * 4, rows, u0 * 16, ((kend + 63) >> 6) * 4, t, 256);
    }
    l2_prefetch_rows(a.A, a.K * 2, a.r, k0 * 2, kend * 2, t, 256);
    l2_prefetch_rows(a.B + n0 * a.r, 0, 1, 0, rows * a.r * 2, t, 256);
    l2_prefetch_rows(a.X, a.K * 2, a.M < NT ? a.M : NT, k0 * 2, kend * 2, t, 256);
    if (QW) {
      // this CTA's rows of F: the offsets, then the values they bound. The grid before
      // this one (the transform) never writes F, and it is launched without programmatic
      // serialisation, so everything that wrote F has completed: reading two offsets
      // here is safe. Only Zs waits.
      const int64_t r0 = n0 + rank * (kRowsPerCta / kCS);
      const int64_t r1 = imin64(r0 + kRowsPerCta / kCS, a.N);
      if (r0 < r1) {
        l2_prefetch_rows(a.q_row_ptr + r0, 0, 1, 0, (r1 - r0 + 1) * 4, t, 256);
        const int64_t j0 = __ldg(a.q_row_ptr + r0), j1 = __ldg(a.q_row_ptr + r1);
        if (j0 >= 0 && j1 <= a.q_nnz && j0 < j1) {
          l2_prefetch_rows(a.q_col, 0, 1, j0 * 2, j1 * 2, t, 256);
          l2_prefetch_rows(a.q_c, 0, 1, j0 * 2, j1 * 2, t, 256);
        }
      }
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float mu = FMT == QL_FMT_NF4_DQ ? __ldg(a.mean) : 0.0f;

  const int64_t row_g = n0 + warp * 16 + g, row_h = row_g + 8;
  // adapter right factor for this warp's rows (A fragments of the final MMA)
  auto bload = [&](int64_t row, int j) -> uint32_t {
    if (a.b_pairs)                                  // even r, 4-byte aligned B: j, j+1 in one word
      return row < a.N && j < a.r ? __ldg(reinterpret_cast<const uint32_t*>(a.B + row * a.r + j)) : 0u;
    if (row >= a.N) return 0u;
    const uint32_t lo = j < a.r ? a.B[row * a.r + j] : 0u;
    const uint32_t hi = j + 1 < a.r ? a.B[row * a.r + j + 1] : 0u;
    return lo | (hi << 16);
  };
  uint32_t bfr[JT > 0 ? JT : 1][4];                 // JT = 0: no adapter
#pragma unroll
  for (int jt = 0; jt < JT; ++jt) {
    const int j0 = jt * 16 + 2 * q;
    bfr[jt][0] = bload(row_g, j0);
    bfr[jt][1] = bload(row_h, j0);
    bfr[jt][2] = bload(row_g, j0 + 8);
    bfr[jt][3] = bload(row_h, j0 + 8);
  }
  UnitRegs<FMT> cg, ch, ng, nh;
  if (nunits > 0) {
    load_block_regs<FMT>(a, row_g, u0 * 4 + q, cg);
    load_block_regs<FMT>(a, row_h, u0 * 4 + q, ch);
  }
  if (nunits > 1) {
    load_block_regs<FMT>(a, row_g, (u0 + 1) * 4 + q, ng);
    load_block_regs<FMT>(a, row_h, (u0 + 1) * 4 + q, nh);
  }
  // rows [row_begin, row_end) of the staged block (tokens 0..NT-1, then adapter rows) ->
  // smem in fragment order (zero beyond the tokens, the rank and K): one 16-byte global
  // load feeds two 8-byte fragment slots. The loads of a batch are all issued before any
  // of its stores, so their latencies overlap.
  const int per_row = nunits * 32;                  // 16-byte vectors per row
  auto stage_rows = [&](int row_begin, int row_end) {
    const int total = (row_end - row_begin) * per_row;
    constexpr int kBatch = 8;
    for (int v0 = 0; v0 < total; v0 += kBatch * 256) {
      uint4 val[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int v = v0 + b * 256 + threadIdx.x;
        val[b] = make_uint4(0u, 0u, 0u, 0u);
        if (v < total) {
          const int row = row_begin + v / per_row, rem = v % per_row;
          const int64_t k = k0 + (rem >> 5) * 256 + 64 * ((rem >> 3) & 3) + 8 * (rem & 7);
          if (row < NT) {
            if (row < a.M && k < a.K) val[b] = __ldg(reinterpret_cast<const uint4*>(a.X + row * a.K + k));
          } else if (row - NT < a.r && k < a.K) {
            val[b] = __ldg(reinterpret_cast<const uint4*>(a.A + (row - NT) * a.K + k));
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int v = v0 + b * 256 + threadIdx.x;
        if (v < total) {
          const int row = row_begin + v / per_row, rem = v % per_row;
          const int ul = rem >> 5, qq = (rem >> 3) & 3, ii = rem & 7;
          uint8_t* p = (row < NT ? sX + (size_t)row * pitch : sA + (size_t)(row - NT) * pitch) + ul * 512;
          *reinterpret_cast<uint2*>(p + ((2 * ii) * 4 + qq) * 8) = make_uint2(val[b].x, val[b].y);
          *reinterpret_cast<uint2*>(p + ((2 * ii + 1) * 4 + qq) * 8) = make_uint2(val[b].z, val[b].w);
        }
      }
    }
  };
  stage_rows(0, NT + RP);                           // token rows, then adapter rows
  __syncthreads();

  // ---- main loop: W' rows (decoded) and, for the adapter, A rows against the tokens ----
  float d[NTT][4];
  float dt[JT > 0 ? JT : 1][NTT][4];                 // T_kr = X_kr A_kr^T, per j-tile
#pragma unroll
  for (int t = 0; t < NTT; ++t) {
    d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.0f;
#pragma unroll
    for (int jt = 0; jt < JT; ++jt) dt[jt][t][0] = dt[jt][t][1] = dt[jt][t][2] = dt[jt][t][3] = 0.0f;
  }
  // Register ring of the codes: units ul and ul + 1 are held; with DEPTH 3 unit ul + 2 is
  // loaded at the top of iteration ul, with DEPTH 2 at its end (fewer registers).
  constexpr int DEPTH = (FMT == QL_FMT_NF4_DQ && NT * JT <= 16) ? 3 : 2;
  for (int ul = 0; ul < nunits; ++ul) {
    UnitRegs<FMT> mg, mh;                            // unit ul + 2
    if (DEPTH == 3 && ul + 2 < nunits) {
      load_block_regs<FMT>(a, row_g, (u0 + ul + 2) * 4 + q, mg);
      load_block_regs<FMT>(a, row_h, (u0 + ul + 2) * 4 + q, mh);
    }
    const uint8_t* xu = sX + ul * 512 + q * 8;
    const uint8_t* au = sA + ul * 512 + q * 8;
    auto step = [&](int s, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
      uint2 bx[NTT];
#pragma unroll
      for (int t = 0; t < NTT; ++t) {
        bx[t] = *reinterpret_cast<const uint2*>(xu + (size_t)(t * 8 + g) * pitch + s * 32);
        mma_bf16_16816(d[t], a0, a1, a2, a3, bx[t].x, bx[t].y);
      }
#pragma unroll
      for (int jt = 0; jt < JT; ++jt) {
        {
          const uint2 ag = *reinterpret_cast<const uint2*>(au + (size_t)(jt * 16 + g) * pitch + s * 32);
          const uint2 ah = *reinterpret_cast<const uint2*>(au + (size_t)(jt * 16 + g + 8) * pitch + s * 32);
#pragma unroll
          for (int t = 0; t < NTT; ++t) mma_bf16_16816(dt[jt][t], ag.x, ah.x, ag.y, ah.y, bx[t].x, bx[t].y);
        }
      }
    };
    if constexpr (FMT == QL_FMT_NF4_DQ) {
      uint32_t Lg[2], Hg[2], Lh[2], Hh[2];
      small_nf4_table(a.q, unit_scale<FMT>(cg, mu), Lg, Hg);
      small_nf4_table(a.q, unit_scale<FMT>(ch, mu), Lh, Hh);
      const uint32_t wg[8] = {cg.c[0].x, cg.c[0].y, cg.c[0].z, cg.c[0].w, cg.c[1].x, cg.c[1].y, cg.c[1].z, cg.c[1].w};
      const uint32_t wh[8] = {ch.c[0].x, ch.c[0].y, ch.c[0].z, ch.c[0].w, ch.c[1].x, ch.c[1].y, ch.c[1].z, ch.c[1].w};
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) {
        const uint4 eg = small_nf4_decode8(wg[w8], Lg, Hg);
        const uint4 eh = small_nf4_decode8(wh[w8], Lh, Hh);
        step(2 * w8, eg.x, eh.x, eg.y, eh.y);
        step(2 * w8 + 1, eg.z, eh.z, eg.w, eh.w);
      }
    } else {
      const uint32_t wg[16] = {cg.c[0].x, cg.c[0].y, cg.c[0].z, cg.c[0].w, cg.c[1].x, cg.c[1].y, cg.c[1].z, cg.c[1].w,
                               cg.c[2].x, cg.c[2].y, cg.c[2].z, cg.c[2].w, cg.c[3].x, cg.c[3].y, cg.c[3].z, cg.c[3].w};
      const uint32_t wh[16] = {ch.c[0].x, ch.c[0].y, ch.c[0].z, ch.c[0].w, ch.c[1].x, ch.c[1].y, ch.c[1].z, ch.c[1].w,
                               ch.c[2].x, ch.c[2].y, ch.c[2].z, ch.c[2].w, ch.c[3].x, ch.c[3].y, ch.c[3].z, ch.c[3].w};
      const float scg = unit_scale<FMT>(cg, mu), sch = unit_scale<FMT>(ch, mu);
#pragma unroll
      for (int st = 0; st < 16; ++st) {
        const uint2 eg = small_int8_decode4(wg[st], scg);
        const uint2 eh = small_int8_decode4(wh[st], sch);
        step(st, eg.x, eh.x, eg.y, eh.y);
      }
    }
    if (ul + 1 < nunits) { cg = ng; ch = nh; }
    if (ul + 2 < nunits) {
      if (DEPTH == 3) {
        ng = mg; nh = mh;
      } else {
        load_block_regs<FMT>(a, row_g, (u0 + ul + 2) * 4 + q, ng);
        load_block_regs<FMT>(a, row_h, (u0 + ul + 2) * 4 + q, nh);
      }
    }
  }

  // ---- adapter term of this K-range: D += B[rows, :] (s T_kr) ----
  // every warp holds the same T_kr; it goes through the warp's own smem slice to reach the
  // B-fragment layout (j along k, tokens along n)
  float* tw = sTw + (size_t)warp * RP * NT;
#pragma unroll
  for (int jt = 0; jt < JT; ++jt) {
    {
#pragma unroll
      for (int t = 0; t < NTT; ++t) {
        tw[(jt * 16 + g) * NT + t * 8 + 2 * q] = dt[jt][t][0];
        tw[(jt * 16 + g) * NT + t * 8 + 2 * q + 1] = dt[jt][t][1];
        tw[(jt * 16 + g + 8) * NT + t * 8 + 2 * q] = dt[jt][t][2];
        tw[(jt * 16 + g + 8) * NT + t * 8 + 2 * q + 1] = dt[jt][t][3];
      }
    }
  }
  __syncwarp();
#pragma unroll
  for (int jt = 0; jt < JT; ++jt) {
    {
      const int j0 = jt * 16 + 2 * q;
#pragma unroll
      for (int t = 0; t < NTT; ++t) {
        const int tok = t * 8 + g;
        const uint32_t b0 = pack_bf16x2(a.s * tw[j0 * NT + tok], a.s * tw[(j0 + 1) * NT + tok]);
        const uint32_t b1 = pack_bf16x2(a.s * tw[(j0 + 8) * NT + tok], a.s * tw[(j0 + 9) * NT + tok]);
        mma_bf16_16816(d[t], bfr[jt][0], bfr[jt][1], bfr[jt][2], bfr[jt][3], b0, b1);
      }
    }
  }

  // ---- partial sums, then the fixed-order cluster reduction ----
  // CTA c reduces the weight rows [16c, 16c + 16) of the cluster's 128, which warp c of
  // every CTA holds. For each such row and token, Y is the sum of the eight CTAs' partials
  // taken in cluster-rank order, so the result does not depend on timing.
  constexpr int kRowsPerRank = kRowsPerCta / kCS;      // 16
  if constexpr (QW) {
    // pull form: partials in the CTA's own sD (rows in the cluster's order), the sparse
    // sums added to the CTA's own rows, then every CTA reads its rows from all eight
#pragma unroll
    for (int t = 0; t < NTT; ++t) {
      const int rg = warp * 16 + g;
      sD[rg * NT + t * 8 + 2 * q] = d[t][0];
      sD[rg * NT + t * 8 + 2 * q + 1] = d[t][1];
      sD[(rg + 8) * NT + t * 8 + 2 * q] = d[t][2];
      sD[(rg + 8) * NT + t * 8 + 2 * q + 1] = d[t][3];
    }
    __syncthreads();
    qwha_rows_add<NT>(a, n0 + rank * kRowsPerRank, sD + (size_t)rank * kRowsPerRank * NT);
    cluster_sync_all();
    for (int i = threadIdx.x; i < kRowsPerRank * NT; i += blockDim.x) {
      const int rr = (int)rank * kRowsPerRank + i / NT, tok = i % NT;
      float part[kCS];
#pragma unroll
      for (int c = 0; c < kCS; ++c) part[c] = ld_cluster_f32(sD + rr * NT + tok, (uint32_t)c);
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < kCS; ++c) acc += part[c];
      const int64_t row = n0 + rr;
      if (tok < a.M && row < a.N) a.Y[tok * a.N + row] = (uint16_t)float_to_bf16_bits(acc);
    }
  } else {
    // push form: warp w stores its partials straight into CTA w's sD, in the slot of this
    // source CTA (sD row 16 * rank + i holds this CTA's partial of the owner's row i); after
    // one release/acquire barrier each CTA sums its eight slots from its own shared memory.
    // Nothing reads another CTA's shared memory after that barrier (outside the T reduction
    // below), so no second barrier is needed before the CTA exits.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    const int rs = (int)rank * kRowsPerRank + g;
#pragma unroll
    for (int t = 0; t < NTT; ++t) {
      st_cluster_f32x2(sD + rs * NT + t * 8 + 2 * q, (uint32_t)warp, d[t][0], d[t][1]);
      st_cluster_f32x2(sD + (rs + 8) * NT + t * 8 + 2 * q, (uint32_t)warp, d[t][2], d[t][3]);
    }
    cluster_sync_all();
    for (int i = threadIdx.x; i < kRowsPerRank * NT; i += blockDim.x) {
      const int rr = i / NT, tok = i % NT;
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < kCS; ++c) acc += sD[(c * kRowsPerRank + rr) * NT + tok];
      const int64_t row = n0 + (int64_t)rank * kRowsPerRank + rr;
      if (tok < a.M && row < a.N) a.Y[tok * a.N + row] = (uint16_t)float_to_bf16_bits(acc);
    }
  }
  const bool reduce_T = a.T_save && blockIdx.x < (unsigned)kCS;   // uniform over the cluster
  {
    if (reduce_T) {                                       // first cluster also reduces T
      for (int i = threadIdx.x; i < RP * NT; i += blockDim.x) {
        const int j = i / NT, tok = i % NT;
        if ((int)(j % kCS) != (int)rank) continue;
        float part[kCS];
#pragma unroll
        for (int c = 0; c < kCS; ++c) part[c] = ld_cluster_f32(sTw + j * NT + tok, (uint32_t)c);
        float acc = 0.0f;
#pragma unroll
        for (int c = 0; c < kCS; ++c) acc += part[c];
        if (tok < a.M && j < a.r) a.T_save[tok * a.r + j] = (uint16_t)float_to_bf16_bits(acc);
      }
    }
  }
  // keep shared memory alive for the readers of the pull reductions
  if (QW || reduce_T) cluster_sync_relaxed();
}

size_t small_m_smem(int NT, int units_max, int r) {
  const int jt = (r + 15) / 16;
  const int RP = (jt == 3 ? 4 : jt) * 16;
  return (size_t)(NT + RP) * small_row_pitch(units_max) + (size_t)(8 * RP * NT + kRowsPerCta * NT) * 4;
}

template <int NT, int FMT, int JT, bool QW = false>
static ql_status launch_small(const SmallArgs& a, cudaStream_t st) {
  auto kern = small_m_fwd_kernel<NT, FMT, JT, QW>;
  SmallArgs b = a;
  const size_t smem = small_m_smem(NT, a.kr_max / 256, JT * 16);
  if (smem > 227 * 1024) return QL_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const int groups = (int)((a.N + kRowsPerCta - 1) / kRowsPerCta);
  // programmatic dependent launch: this grid may begin (and warm L2 with its inputs) while
  // the previous grid on the stream finishes; the kernel waits before loading any input
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(groups * kCS);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, b) != cudaSuccess) return QL_ERR_CUDA;
  QL_CHECK_LAUNCH();
  return QL_OK;
}

bool small_m_supported(int64_t K, int r) {
  if (r < 0 || r > 64) return false;
  const int64_t U = (K + 255) / 256;
  const int units_max = (int)((U + kCS - 1) / kCS);
  return small_m_smem(16, units_max, r) <= 200 * 1024;
}

// Host entry used by qlora_linear_fwd when M <= 16.
ql_status small_m_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                          const uint16_t* B, int r, float alpha, uint16_t* Y, uint16_t* T_save,
                          cudaStream_t st, const QwhaRows* qw) {
  if (r < 0 || r > 64) return QL_ERR_UNSUPPORTED;
  SmallArgs a{};
  a.flag = device_flag_ptr();
  if (qw) {
    if (r != 0) return QL_ERR_UNSUPPORTED;
    a.q_row_ptr = qw->row_ptr; a.q_col = qw->col; a.q_c = qw->c; a.q_nnz = qw->nnz; a.q_Zs = qw->Zs;
  }
  a.X = X; a.A = A; a.B = B; a.M = M; a.N = w->N; a.K = w->K; a.r = r; a.s = r > 0 ? alpha / (float)r : 0.0f;
  a.fmt = w->fmt;
  a.codes = static_cast<const uint8_t*>(w->codes);
  a.qabsmax = w->qabsmax; a.gscale = w->group_scale; a.mean = w->mean; a.absmax = w->absmax;
  a.Y = Y; a.T_save = T_save;
  const int64_t U = (w->K + 255) / 256;
  a.kr_max = (int)(((U + kCS - 1) / kCS) * 256);
  a.b_pairs = (r % 2 == 0 && aligned(B, 4)) ? 1 : 0;
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) a.q[i] = t.q[i];
  ProfScope prof(PK_FWD_SMALL, st, 1);
  const int jt = (r + 15) / 16;
  const bool nf4 = w->fmt == QL_FMT_NF4_DQ;
  if (jt == 0 && qw) {                             // no LoRA part; the Walsh-Hadamard sums
    if (M <= 8)
      return nf4 ? launch_small<8, QL_FMT_NF4_DQ, 0, true>(a, st) : launch_small<8, QL_FMT_INT8_B64, 0, true>(a, st);
    return nf4 ? launch_small<16, QL_FMT_NF4_DQ, 0, true>(a, st) : launch_small<16, QL_FMT_INT8_B64, 0, true>(a, st);
  }
  if (jt == 0) {                                   // no adapter: the base product alone
    if (M <= 8) return nf4 ? launch_small<8, QL_FMT_NF4_DQ, 0>(a, st) : launch_small<8, QL_FMT_INT8_B64, 0>(a, st);
    return nf4 ? launch_small<16, QL_FMT_NF4_DQ, 0>(a, st) : launch_small<16, QL_FMT_INT8_B64, 0>(a, st);
  }
  if (M <= 8) {
    if (nf4) return jt == 1 ? launch_small<8, QL_FMT_NF4_DQ, 1>(a, st) : jt == 2 ? launch_small<8, QL_FMT_NF4_DQ, 2>(a, st)
                                                                              : launch_small<8, QL_FMT_NF4_DQ, 4>(a, st);
    return jt == 1 ? launch_small<8, QL_FMT_INT8_B64, 1>(a, st) : jt == 2 ? launch_small<8, QL_FMT_INT8_B64, 2>(a, st)
                                                                        : launch_small<8, QL_FMT_INT8_B64, 4>(a, st);
  }
  if (nf4) return jt == 1 ? launch_small<16, QL_FMT_NF4_DQ, 1>(a, st) : jt == 2 ? launch_small<16, QL_FMT_NF4_DQ, 2>(a, st)
                                                                             : launch_small<16, QL_FMT_NF4_DQ, 4>(a, st);
  return jt == 1 ? launch_small<16, QL_FMT_INT8_B64, 1>(a, st) : jt == 2 ? launch_small<16, QL_FMT_INT8_B64, 2>(a, st)
                                                                       : launch_small<16, QL_FMT_INT8_B64, 4>(a, st);
}

}  // namespace qlb
