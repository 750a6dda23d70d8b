// Walsh-Hadamard adapter in the quantised linear (QWHA page,
// gist.science/ko/paper/2509.17428, section 2.1 "Walsh-Hadamard adaptation"):
//
//   Y = X deq(W)^T + X (F H^{-1})^T = base + Z F^T,    Z = X H^{-T} = X H
//
// H is the orthonormal Sylvester-order Walsh-Hadamard matrix, block-diagonal in blocks of
// b = the largest power of two dividing K (H = H^T = H^{-1}); F [N, K] is sparse, held as
// compressed rows (row_ptr, col, c). The adapter stays unmerged.
//
//  * qwha_wht_kernel forms Z = X H per token and block by the fast butterfly recursion,
//    adds and subtracts only, in fp32 (the page's point: no multiplies by H).
//  * Decode-shaped calls (M <= 16): Z goes to one token slab Zs[k][16] (a column of the
//    slab is one 32-byte sector); the decode-shaped base kernel gathers it by column index
//    for its rows (sum_j c_j Z[m, col_j]) and adds the sums before the cluster reduction,
//    so they reach Y with its one bf16 rounding (small_m.cu, qwha_rows_add).
//  * Larger M: Z F^T = X (F H)^T since H is symmetric. qwha_update_kernel forms dW = F H
//    [N, K] bf16 straight from the compressed rows (blocks up to 4096 wide; wider blocks:
//    qwha_densify_kernel writes the dense F and the row transform follows), and the fused
//    tcgen05 GEMM adds dW to the decoded weight in shared memory before the MMA, so the
//    adapter costs one bf16 add per weight element instead of a second contraction of K.
//    The gather has no tensor-core form (F's positions are arbitrary), and on the FMA
//    pipes it needs a shared-memory read per multiply-add.
#include <cmath>

#include "common.cuh"
#include "weight_check.cuh"

namespace qlb {

constexpr int kQwSlab = 16;          // tokens per slab of Z

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t f2_to_bf16x2(float lo, float hi) {
  return (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
}

// In-register butterflies over the index bits [0, NB) of v[0 .. 2^NB): after it,
// v[i] = sum_j (-1)^popcount(i & j) v_in[j] (unnormalised, natural order).
template <int NB>
__device__ __forceinline__ void butterflies(float* v) {
#pragma unroll
  for (int h = 1; h < (1 << NB); h <<= 1) {
#pragma unroll
    for (int i = 0; i < (1 << NB); ++i) {
      if ((i & h) == 0) {
        const float a = v[i], c = v[i + h];
        v[i] = a + c;
        v[i + h] = a - c;
      }
    }
  }
}

// Row elements live at phys(e) = e + e/16 in shared memory: one spare word after every 16
// floats, so that 32 threads storing 16 consecutive elements each (pass 0) and 32 threads
// touching one element of 32 consecutive groups (the later passes) hit 32 different banks.
__device__ __forceinline__ int phys(int e) { return e + (e >> 4); }
__host__ __device__ __forceinline__ int qwha_pitch(int b) { return b + (b >> 4) + 4; }

// Where element e of the transformed row of token m lands in global memory: row-major
// Z [M][K], or the token slabs Zs[m / 16][k][m % 16].
template <bool SLAB>
__device__ __forceinline__ size_t z_index(int64_t m, int64_t k, int64_t K) {
  return SLAB ? (size_t)(((m / kQwSlab) * K + k) * kQwSlab + (m % kQwSlab)) : (size_t)(m * K + k);
}

// One pass over the index bits [lo, lo + NB) of every length-bs row held in shared memory
// (rows of `pitch` floats, TT rows). A group is the 2^NB elements that differ only in
// those bits; consecutive threads take groups with consecutive low bits, so a warp's
// accesses to one element of its groups are consecutive words. FINAL: the pass that
// completes the transform writes its results (times `scale`, rounded to bf16) straight
// to global memory instead of back to shared memory; a warp's 32 stores of one element
// index are then 32 consecutive columns.
template <int NB, bool FINAL, bool SLAB>
__device__ __forceinline__ void smem_pass(float* sm, int TT, int bs, int pitch, int lo, float scale,
                                          uint16_t* Z, int64_t m0, int64_t M, int64_t K, int64_t kbase) {
  const int per_row = bs >> NB;                  // groups per row
  const int total = TT * per_row;
  const int low_mask = (1 << lo) - 1;
  for (int gi = threadIdx.x; gi < total; gi += blockDim.x) {
    const int t = gi / per_row, rest = gi - t * per_row;
    const int base = ((rest >> lo) << (lo + NB)) | (rest & low_mask);
    float* row = sm + (size_t)t * pitch;
    float v[1 << NB];
#pragma unroll
    for (int j = 0; j < (1 << NB); ++j) v[j] = row[phys(base + (j << lo))];
    butterflies<NB>(v);
    if (FINAL) {
      const int64_t m = m0 + t;
      if (m < M) {
#pragma unroll
        for (int j = 0; j < (1 << NB); ++j)
          Z[z_index<SLAB>(m, kbase + base + (j << lo), K)] = float_to_bf16_bits(v[j] * scale);
      }
    } else {
#pragma unroll
      for (int j = 0; j < (1 << NB); ++j) row[phys(base + (j << lo))] = v[j];
    }
  }
}

template <bool FINAL, bool SLAB>
__device__ __forceinline__ void smem_pass_n(int nb, float* sm, int TT, int bs, int pitch, int lo, float scale,
                                            uint16_t* Z, int64_t m0, int64_t M, int64_t K, int64_t kbase) {
  switch (nb) {
    case 4: smem_pass<4, FINAL, SLAB>(sm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase); break;
    case 3: smem_pass<3, FINAL, SLAB>(sm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase); break;
    case 2: smem_pass<2, FINAL, SLAB>(sm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase); break;
    default: smem_pass<1, FINAL, SLAB>(sm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase); break;
  }
}

// Z = X H for TT tokens [m0, m0 + TT) and one slice of one Walsh-Hadamard block of the
// input width: block blockIdx.y >> SL (b = 2^L elements), slice j = blockIdx.y & (2^SL - 1)
// of its outputs (bs = b / 2^SL consecutive columns). Sylvester's matrix factors as
// H_b = H_{2^SL} (x) H_bs, so slice j is H_bs applied to u_j = sum_r (-1)^popcount(j & r)
// x[r * bs ...]: the 2^SL input slices combined with signs, then a transform of length bs
// (2^SL CTAs share one token's block; SL = 0 is the plain transform). log2(bs) >= 5.
// Tokens at or past M read as zero and are not written.
template <bool SLAB>
__global__ void __launch_bounds__(256)
qwha_wht_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K, int L, int SL, int TT, float scale,
                uint16_t* __restrict__ Z) {
  extern __shared__ __align__(16) float wsm[];
  const int Ls = L - SL, bs = 1 << Ls;
  const int b = 1 << L;
  const int pitch = qwha_pitch(bs);
  const int64_t m0 = (int64_t)blockIdx.x * TT;
  const int j = (int)(blockIdx.y & ((1u << SL) - 1));
  const int64_t kblk = (int64_t)(blockIdx.y >> SL) << L;
  const int S = 1 << SL;
  // the next grid (the decode-shaped base kernel) may start now and warm L2 with its own
  // inputs; it waits for this grid before reading Z
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the raw bf16 input tile [TT][b] sits after the fp32 rows; every thread issues all of
  // its 16-byte copies before any is waited for (tokens past M are zero-filled)
  uint16_t* raw = reinterpret_cast<uint16_t*>(wsm + (size_t)TT * pitch);
  {
    const int per_row = b >> 3;
    for (int gi = threadIdx.x; gi < TT * per_row; gi += blockDim.x) {
      const int t = gi / per_row, e = (gi - t * per_row) << 3;
      const int64_t m = m0 + t;
      const uint16_t* src = m < M ? X + m * K + kblk + e : X;
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(raw + (size_t)t * b + e));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(m < M ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }

  // pass 0: 16 contiguous elements of u per thread, bits 0..3 in registers
  {
    const int per_row = bs >> 4;
    for (int gi = threadIdx.x; gi < TT * per_row; gi += blockDim.x) {
      const int t = gi / per_row, e0 = (gi - t * per_row) << 4;
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
      {
        for (int r = 0; r < S; ++r) {
          const uint4* src = reinterpret_cast<const uint4*>(raw + (size_t)t * b + r * bs + e0);
          const uint4 u0 = src[0], u1 = src[1];
          const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          if (__popc(j & r) & 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[2 * i] -= bf16_lo(w[i]);
              v[2 * i + 1] -= bf16_hi(w[i]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[2 * i] += bf16_lo(w[i]);
              v[2 * i + 1] += bf16_hi(w[i]);
            }
          }
        }
      }
      butterflies<4>(v);
      float* dst = wsm + (size_t)t * pitch + phys(e0);
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[i] = v[i];
    }
  }
  __syncthreads();
  // the remaining bits of the slice, up to four per pass; the last pass stores to global
  const int64_t kbase = kblk + (int64_t)j * bs;
  for (int lo = 4; lo < Ls; lo += 4) {
    const int nb = Ls - lo >= 4 ? 4 : Ls - lo;
    if (lo + nb < Ls) {
      smem_pass_n<false, SLAB>(nb, wsm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase);
      __syncthreads();
    } else {
      smem_pass_n<true, SLAB>(nb, wsm, TT, bs, pitch, lo, scale, Z, m0, M, K, kbase);
    }
  }
}

// F written out densely for the tensor cores: Fd [N, K] bf16 holds c_j at (n, col_j) and
// zero elsewhere. A CTA builds `rows` (<= 64) consecutive rows in shared memory: zero,
// then all its threads scatter the rows' values together (the values of the CTA's rows
// are one contiguous range, so a long row is spread over every thread), then the rows go
// out once with 16-byte stores. The same index checks as the sparse product.
__global__ void __launch_bounds__(256)
qwha_densify_kernel(const int32_t* __restrict__ row_ptr, const uint16_t* __restrict__ col,
                    const uint16_t* __restrict__ cval, int64_t nnz, int64_t N, int64_t K, int rows,
                    uint16_t* __restrict__ Fd, int* flag) {
  extern __shared__ __align__(16) uint16_t drow[];
  __shared__ int s_off[65];
  const int64_t n0 = (int64_t)blockIdx.x * rows;
  const int nr = (int)imin64(rows, N - n0);
  const int64_t n16 = (int64_t)nr * K / 8;             // 16-byte words (K % 64 == 0)
  uint4* d4 = reinterpret_cast<uint4*>(drow);
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) d4[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x <= nr) s_off[threadIdx.x] = __ldg(row_ptr + n0 + threadIdx.x);
  __syncthreads();
  bool bad = false;
  {
    const int t = threadIdx.x;
    const bool row_bad = t < nr && (s_off[t] < 0 || s_off[t] > s_off[t + 1] || (int64_t)s_off[t + 1] > nnz);
    bad = __syncthreads_or(row_bad) != 0;             // inconsistent offsets: scatter nothing
  }
  if (!bad) {
    const int jb = s_off[0], je = s_off[nr];
    for (int jj = jb + (int)threadIdx.x; jj < je; jj += blockDim.x) {
      int lo = 0, hi = nr - 1;                         // the row holding jj: s_off[lo] <= jj < s_off[lo + 1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= jj) lo = mid; else hi = mid - 1;
      }
      const uint32_t k = __ldg(col + jj);
      if (k >= (uint64_t)K) {
        bad = true;
        continue;
      }
      drow[(int64_t)lo * K + k] = __ldg(cval + jj);
    }
  }
  __syncthreads();
  uint4* g4 = reinterpret_cast<uint4*>(Fd + n0 * K);
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) g4[i] = d4[i];
  if (bad) raise_flag(flag, kFlagBadIndex);
}

// The update dW = F H (QWHA page, section 2.1: Delta W = F H^{-1}, H symmetric and
// orthogonal) straight from the compressed rows of F, for transform blocks of b = 64 << LB
// columns (b <= 4096), on the tensor cores. Each warp takes one (row n, super-tile st) item:
// the 4096 columns [4096 st, 4096 st + 4096) of row n as a 64 x 64 tile R[a][j] (column
// 4096 st + 64 a + j), which holds 64 >> LB whole blocks of 2^LB tile rows. In Sylvester
// order H_b = H_{2^LB} (x) H_64, so the tile's transform is Q = G R H_64 with G = I (x) H_{2^LB}
// (64 x 64, entries 0 and +-1) and H_64 the 64-point matrix: two 64 x 64 x 64 products by
// mma.sync (m16n8k16, bf16 in, fp32 out). R holds F's bf16 values and G, H_64 are exact in
// bf16, so P = G R is exact up to fp32 summation; P enters the second product as
// bf16 hi + lo (hi = bf16(P), lo = bf16(P - hi)), a relative error near 2^-16. Q is scaled
// by 1 / sqrt(b), rounded to bf16 and stored. The scatter writes F's values into a zeroed
// bf16 tile and writes zeros back to the same places afterwards. The same index checks as
// the densified form; a repeated column keeps one of its values, as there.
constexpr int kUpdPitch = 72;            // bf16 per tile row (144 bytes): conflict-free ldmatrix rows
constexpr int kUpdWarps = 6;
constexpr int kUpdWarpBytes = (64 + 16) * kUpdPitch * 2;   // the tile, then 16 output rows

__device__ __forceinline__ void upd_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// +-1 (or 0) as bf16 bits
__device__ __forceinline__ uint32_t pm1_bf16(bool nonzero, int parity) {
  return nonzero ? (parity & 1 ? 0xBF80u : 0x3F80u) : 0u;
}

template <int LB>
__global__ void __launch_bounds__(kUpdWarps * 32)
qwha_update_kernel(const int32_t* __restrict__ row_ptr, const uint16_t* __restrict__ col,
                   const uint16_t* __restrict__ cval, int64_t nnz, int64_t N, int64_t K, float scale,
                   uint16_t* __restrict__ dW, int* flag) {
  extern __shared__ __align__(16) uint16_t usm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  uint16_t* R = usm + (size_t)warp * (kUpdWarpBytes / 2);
  uint16_t* O = R + 64 * kUpdPitch;                      // one 16-row block of Q, bf16
  for (int i = lane; i < 64 * kUpdPitch / 8; i += 32) reinterpret_cast<uint4*>(R)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  // G's 16 x 16 diagonal-position block as an A fragment: element (r, c) is nonzero when r
  // and c lie in the same 2^LB block, with sign (-1)^popcount(r & c & (2^LB - 1)); a block
  // (ib, ka) of G is this one with the sign (-1)^popcount(ib & ka & (2^(LB-4) - 1)) when
  // LB >= 4 and ib, ka share a 2^LB block, and zero otherwise.
  constexpr int m = (1 << LB) - 1;
  auto gel = [&](int r, int c) -> uint32_t { return pm1_bf16(((r ^ c) & ~m & 15) == 0, __popc(r & c & m)); };
  uint32_t Ad[4];
  Ad[0] = gel(g, 2 * q) | (gel(g, 2 * q + 1) << 16);
  Ad[1] = gel(g + 8, 2 * q) | (gel(g + 8, 2 * q + 1) << 16);
  Ad[2] = gel(g, 2 * q + 8) | (gel(g, 2 * q + 9) << 16);
  Ad[3] = gel(g + 8, 2 * q + 8) | (gel(g + 8, 2 * q + 9) << 16);
  // H_64 as the B operand: rows 16 kn + {2q, 2q+1} (b0) and 16 kn + 8 + {2q, 2q+1} (b1) of
  // column 8 jt + g carry the signs of H_8 entries (2q.., g) times (-1)^popcount(kn & (jt >> 1))
  // (and (-1)^(jt & 1) for b1).
  const uint32_t B0 = pm1_bf16(true, __popc((2 * q) & g)) | (pm1_bf16(true, __popc((2 * q + 1) & g)) << 16);
  const int64_t ST = (K + 4095) / 4096;
  const int64_t items = N * ST;
  const int64_t stride = (int64_t)gridDim.x * kUpdWarps;
  const uint32_t rbase = static_cast<uint32_t>(__cvta_generic_to_shared(R));
  bool bad = false;
  // The warp's items it0, it0 + stride, ... are software-pipelined so that no global load
  // waits in front of the tensor cores: the row bounds are requested two items ahead, and
  // the first 64 (column, value) pairs of a row (two per lane) one item ahead; a longer
  // row loads the rest when it is scattered.
  auto row_bounds = [&](int64_t it, int& jb, int& je) {
    jb = je = 0;
    if (it < items) {
      const int64_t n = it / ST;
      jb = __ldg(row_ptr + n);
      je = __ldg(row_ptr + n + 1);
    }
  };
  auto first_pairs = [&](int jb, int je, uint32_t (&kv)[2]) {
    const bool ok = jb >= 0 && jb <= je && (int64_t)je <= nnz;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int jj = jb + 32 * u + lane;
      kv[u] = ok && jj < je ? (uint32_t)__ldg(col + jj) | ((uint32_t)__ldg(cval + jj) << 16) : 0xFFFFFFFFu;
    }
  };
  int64_t it = (int64_t)blockIdx.x * kUpdWarps + warp;
  int jb_c, je_c, jb_n, je_n;
  uint32_t kv_c[2];
  row_bounds(it, jb_c, je_c);
  row_bounds(it + stride, jb_n, je_n);
  first_pairs(jb_c, je_c, kv_c);
  for (; it < items; it += stride) {
    int jb_nn, je_nn;
    uint32_t kv_n[2];
    row_bounds(it + 2 * stride, jb_nn, je_nn);
    first_pairs(jb_n, je_n, kv_n);
    const int64_t n = it / ST, c0 = (it % ST) * 4096;
    const int rows = (int)imin64(64, (K - c0) >> 6);     // tile rows present: whole blocks (b | K)
    int jb = jb_c, je = je_c;
    if (jb < 0 || je < jb || (int64_t)je > nnz) {
      bad = true;
      jb = je = 0;
    }
    auto scatter = [&](uint32_t kc) {
      const uint32_t k = kc & 0xFFFFu;
      if ((int64_t)k >= K) {
        bad = true;
        return;
      }
      const int64_t e = (int64_t)k - c0;
      if (e >= 0 && e < 4096) R[(e >> 6) * kUpdPitch + (e & 63)] = (uint16_t)(kc >> 16);
    };
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (jb + 32 * u + lane < je) scatter(kv_c[u]);
    for (int jj = jb + 64 + lane; jj < je; jj += 32)
      scatter((uint32_t)__ldg(col + jj) | ((uint32_t)__ldg(cval + jj) << 16));
    __syncwarp();
#pragma unroll 1
    for (int ib = 0; ib < 4; ++ib) {
      if (16 * ib >= rows) break;
      // P[ib] (16 x 64) = sum over ka of G[ib, ka] R[ka, :]
      float P[8][4];
#pragma unroll
      for (int jt = 0; jt < 8; ++jt) P[jt][0] = P[jt][1] = P[jt][2] = P[jt][3] = 0.f;
#pragma unroll
      for (int ka = 0; ka < 4; ++ka) {
        if (LB < 6 && ((ib ^ ka) >> (LB > 4 ? LB - 4 : 0)) != 0) continue;   // a zero block of G
        if (LB < 4 && ka != ib) continue;
        const int sg = LB >= 4 ? __popc(ib & ka & ((1 << (LB > 4 ? LB - 4 : 0)) - 1)) & 1 : 0;
        uint32_t A[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) A[i] = Ad[i] ^ (sg ? 0x80008000u : 0u);
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {                 // j-tiles 2 jp, 2 jp + 1
          const int mi = lane >> 3, r = lane & 7;
          const uint32_t addr = rbase + (uint32_t)(((16 * ka + 8 * (mi & 1) + r) * kUpdPitch + 8 * (2 * jp + (mi >> 1))) * 2);
          uint32_t b[4];
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                       : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]) : "r"(addr));
          upd_mma(P[2 * jp], A, b[0], b[1]);
          upd_mma(P[2 * jp + 1], A, b[2], b[3]);
        }
      }
      // P as A fragments of the second product, split into bf16 hi + lo
      uint32_t Ah[4][4], Al[4][4];
#pragma unroll
      for (int kn = 0; kn < 4; ++kn) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float* c = P[2 * kn + h];
          const uint32_t hi01 = pack_bf16x2(c[0], c[1]), hi23 = pack_bf16x2(c[2], c[3]);
          const uint32_t lo01 = pack_bf16x2(c[0] - __uint_as_float(hi01 << 16), c[1] - __uint_as_float(hi01 & 0xFFFF0000u));
          const uint32_t lo23 = pack_bf16x2(c[2] - __uint_as_float(hi23 << 16), c[3] - __uint_as_float(hi23 & 0xFFFF0000u));
          Ah[kn][2 * h] = hi01; Ah[kn][2 * h + 1] = hi23;
          Al[kn][2 * h] = lo01; Al[kn][2 * h + 1] = lo23;
        }
      }
      // Q[ib] (16 x 64) = P[ib] H_64, eight independent accumulators per step, then scaled
      // and stored
      float Q[8][4];
#pragma unroll
      for (int jt = 0; jt < 8; ++jt) Q[jt][0] = Q[jt][1] = Q[jt][2] = Q[jt][3] = 0.f;
#pragma unroll
      for (int kn = 0; kn < 4; ++kn) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int jt = 0; jt < 8; ++jt) {
            const int s0 = __popc(kn & (jt >> 1)) & 1, s1 = (s0 + (jt & 1)) & 1;
            const uint32_t b0 = B0 ^ (s0 ? 0x80008000u : 0u), b1 = B0 ^ (s1 ? 0x80008000u : 0u);
            upd_mma(Q[jt], h ? Al[kn] : Ah[kn], b0, b1);
          }
        }
      }
      // through shared memory, so that the block's 16 tile rows (2 KB, contiguous in dW) go
      // out as whole 16-byte vectors, 512 contiguous bytes per warp store
#pragma unroll
      for (int jt = 0; jt < 8; ++jt) {
        const int col0 = 8 * jt + 2 * q;
        *reinterpret_cast<uint32_t*>(O + g * kUpdPitch + col0) = pack_bf16x2(Q[jt][0] * scale, Q[jt][1] * scale);
        *reinterpret_cast<uint32_t*>(O + (g + 8) * kUpdPitch + col0) = pack_bf16x2(Q[jt][2] * scale, Q[jt][3] * scale);
      }
      __syncwarp();
      const int vrows = rows - 16 * ib < 16 ? rows - 16 * ib : 16;
      uint4* dst = reinterpret_cast<uint4*>(dW + n * K + c0 + 64 * 16 * ib);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int idx = v * 32 + lane, r = idx >> 3, c = idx & 7;   // row r, 16-byte column c
        if (r < vrows) dst[idx] = *reinterpret_cast<const uint4*>(O + r * kUpdPitch + 8 * c);
      }
      __syncwarp();
    }
    __syncwarp();
    for (int i = lane; i < 64 * kUpdPitch / 8; i += 32)   // the tile back to zero
      reinterpret_cast<uint4*>(R)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    jb_c = jb_n; je_c = je_n; jb_n = jb_nn; je_n = je_nn;
    kv_c[0] = kv_n[0]; kv_c[1] = kv_n[1];
  }
  if (bad) raise_flag(flag, kFlagBadIndex);
}

// ---- host side -------------------------------------------------------------------------

static int log2_exact(int64_t b) {
  int L = 0;
  while ((int64_t(1) << L) < b) ++L;
  return L;
}

// tokens per WHT block: about 32 KB of fp32 rows (plus the raw tile) per CTA, so four
// CTAs share an SM and one's loads overlap another's butterflies (measured 8% faster than
// twice that per CTA at 8192 x 4096)
static int wht_tokens(int64_t b) {
  int tt = 16;
  while (tt > 1 && (int64_t)tt * b > 8192) tt >>= 1;
  return tt;
}

// fp32 rows of the transform (length bs) plus the raw bf16 input tile (length b)
static size_t wht_smem(int64_t b, int64_t bs, int tt) {
  return (size_t)tt * qwha_pitch((int)bs) * 4 + (size_t)tt * b * 2;
}

static bool qwha_decode_shaped(int64_t M, int64_t K) { return M <= kSmallMMax && small_m_supported(K, 0); }

// dW straight from the compressed rows when the transform blocks are at most 4096 wide;
// wider blocks go through the densified F and the row transform.
static bool qwha_update_direct(int64_t K) { return (K & (-K)) <= 4096; }

// Workspace: decode-shaped, the one slab of Z; otherwise dW = F H (bf16 [N, K]), the dense
// F as well when the blocks are wider than 4096, plus the fused GEMM's scratch.
int64_t qwha_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (qwha_decode_shaped(M, K)) return round_up(K * kQwSlab * 2, 256);
  return (qwha_update_direct(K) ? 1 : 2) * round_up(N * K * 2, 256) + ext_fwd_ws_bytes(M, N, K, 0);
}

// Z = X H, SLAB (decode-shaped: one token per CTA and blocks of more than 512 split into
// 512-column slices over several CTAs, so one token's transform is spread over the GPU;
// tokens < M only, the slab's other columns are never added to Y) or row-major [M, K].
template <bool SLAB>
static ql_status launch_wht(const uint16_t* X, int64_t M, int64_t K, uint16_t* Z, cudaStream_t st) {
  const int64_t b = K & (-K);
  const int L = log2_exact(b);
  const int SL = SLAB && L > 9 ? L - 9 : 0;
  const int tt = SLAB ? 1 : wht_tokens(b);
  const size_t smem = wht_smem(b, b >> SL, tt);
  if (L < 6 || L > 16 || L - SL < 5 || smem > 200 * 1024) return QL_ERR_UNSUPPORTED;
  auto kern = qwha_wht_kernel<SLAB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  if ((M + tt - 1) / tt > 0x7fffffff || (K / b) << SL > 65535) return QL_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)((M + tt - 1) / tt), (unsigned)((K / b) << SL));
  const float scale = (float)(1.0 / std::sqrt((double)b));
  kern<<<grid, 256, smem, st>>>(X, M, K, L, SL, tt, scale, Z);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

// rows of the dense F per CTA: about 16 KB of shared memory, so several CTAs share an SM
// and their zero / scatter / write phases overlap
static int densify_rows(int64_t K) { return (int)imax64(1, imin64(64, 16384 / (2 * K))); }

}  // namespace qlb

using namespace qlb;

extern "C" {

ql_status qlora_linear_fwd_qwha(const ql_weight* w, const ql_bf16* X, int64_t M, const ql_qwha* f, ql_bf16* Y,
                                void* ws, size_t ws_bytes, void* stream) {
  // every refusal of the wrapped forward is made here, before the transform or the update
  // is launched
  const ql_status ws0 = weight_desc_status(w);
  if (ws0 != QL_OK) return ws0;
  if (!f || !X || !Y || M < 1 || !aligned(X, 16) || !aligned(Y, 16)) return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!f->row_ptr || f->nnz < 0 || (f->nnz > 0 && (!f->col || !f->c))) return QL_ERR_INVALID_ARG;
  if (!aligned(f->row_ptr, 4) || !aligned(f->col, 2) || !aligned(f->c, 2)) return QL_ERR_INVALID_ARG;
  if (f->nnz >= (int64_t(1) << 31) || w->K > 65536) return QL_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  if ((int64_t)ws_bytes < qwha_ws_bytes(M, N, K)) return QL_ERR_WORKSPACE;
  {
    const int64_t b = K & (-K);
    if (wht_smem(b, b, wht_tokens(b)) > 200 * 1024) return QL_ERR_UNSUPPORTED;
  }
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  ql_status e;
  if (qwha_decode_shaped(M, K)) {
    // Z = X H into one token slab, then the decode-shaped base kernel, which adds the
    // sparse sums of its rows before the cluster reduction (a programmatic dependent of
    // the transform: it warms L2 with its weight and its rows of F while the transform
    // runs)
    uint16_t* Zs = reinterpret_cast<uint16_t*>(wsb);
    {
      ProfScope prof(PK_FWD_ADAPTER, st, 1);
      e = launch_wht<true>(X, M, K, Zs, st);
      if (e != QL_OK) return e;
    }
    const QwhaRows rows{f->row_ptr, f->col, reinterpret_cast<const uint16_t*>(f->c), f->nnz, Zs};
    return ext_forward(w, X, M, nullptr, nullptr, 0, Y, nullptr, 0, st, &rows);
  }
  // tensor cores: Z F^T = X (F H)^T (H symmetric), so the update dW = F H is formed once
  // (straight from the compressed rows for blocks up to 4096 wide, else F densified and
  // then the row transform) and added to the decoded weight inside the fused GEMM:
  // Y = X bf16(W' + dW)^T, one contraction of K.
  const int64_t fb = round_up(N * K * 2, 256);
  uint16_t* dW = reinterpret_cast<uint16_t*>(wsb);
  if (qwha_update_direct(K)) {
    const int64_t b = K & (-K);
    const int LB = log2_exact(b) - 6;
    const size_t usm = (size_t)kUpdWarps * kUpdWarpBytes;
    const float scale = (float)(1.0 / std::sqrt((double)b));
    const int64_t items = N * ((K + 4095) / 4096);
    const int grid = (int)imin64((items + kUpdWarps - 1) / kUpdWarps, (int64_t)num_sms() * 3);
    auto launch = [&](auto kern) -> ql_status {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)usm) != cudaSuccess)
        return QL_ERR_CUDA;
      kern<<<grid, kUpdWarps * 32, usm, st>>>(f->row_ptr, f->col, reinterpret_cast<const uint16_t*>(f->c), f->nnz,
                                              N, K, scale, dW, device_flag_ptr());
      QL_CHECK_LAUNCH();
      return QL_OK;
    };
    {
      ProfScope prof(PK_FWD_ADAPTER, st, 1);
      switch (LB) {
        case 0: e = launch(qwha_update_kernel<0>); break;
        case 1: e = launch(qwha_update_kernel<1>); break;
        case 2: e = launch(qwha_update_kernel<2>); break;
        case 3: e = launch(qwha_update_kernel<3>); break;
        case 4: e = launch(qwha_update_kernel<4>); break;
        case 5: e = launch(qwha_update_kernel<5>); break;
        default: e = launch(qwha_update_kernel<6>); break;
      }
    }
    if (e != QL_OK) return e;
    return dw_forward(w, X, M, dW, Y, wsb + fb, ws_bytes - (size_t)fb, st);
  }
  uint16_t* Fd = reinterpret_cast<uint16_t*>(wsb + fb);
  {
    ProfScope prof(PK_FWD_ADAPTER, st, 2);
    const int rows = densify_rows(K);
    const size_t dsm = (size_t)rows * K * 2;
    if (cudaFuncSetAttribute(qwha_densify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm) !=
        cudaSuccess)
      return QL_ERR_CUDA;
    qwha_densify_kernel<<<(unsigned)((N + rows - 1) / rows), 256, dsm, st>>>(f->row_ptr, f->col, f->c, f->nnz,
                                                                          N, K, rows, Fd, device_flag_ptr());
    QL_CHECK_LAUNCH();
    e = launch_wht<false>(Fd, N, K, dW, st);
    if (e != QL_OK) return e;
  }
  return dw_forward(w, X, M, dW, Y, wsb + 2 * fb, ws_bytes - (size_t)(2 * fb), st);
}

ql_status ql_wht(const ql_bf16* X, int64_t M, int64_t K, ql_bf16* Z, void* stream) {
  if (!X || !Z || M < 1 || K < 64) return QL_ERR_INVALID_ARG;
  if (K % 64 != 0 || M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!aligned(X, 16) || !aligned(Z, 16)) return QL_ERR_INVALID_ARG;
  const int64_t b = K & (-K);
  if (wht_smem(b, b, wht_tokens(b)) > 200 * 1024) return QL_ERR_UNSUPPORTED;
  ProfScope prof(PK_FWD_ADAPTER, as_stream(stream), 1);
  return launch_wht<false>(X, M, K, Z, as_stream(stream));
}

}  // extern "C"
