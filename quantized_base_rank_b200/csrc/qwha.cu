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
//  * Larger M: Z row-major; qwha_densify_kernel writes F as a dense bf16 [N, K] and the
//    fused tcgen05 GEMM takes Z F^T as K/64 extension chunks, beside X W'^T. The gather
//    has no tensor-core form (F's positions are arbitrary), and on the FMA pipes it needs
//    a shared-memory read per multiply-add; the extension chunks are faster at the
//    budgets of a rank-64 LoRA.
#include <cmath>

#include "common.cuh"

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

// Workspace: decode-shaped, the one slab of Z; otherwise Z [M, K] and the dense F [N, K]
// (bf16) plus the fused GEMM's scratch.
int64_t qwha_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (qwha_decode_shaped(M, K)) return round_up(K * kQwSlab * 2, 256);
  return round_up(M * K * 2, 256) + round_up(N * K * 2, 256) + ext_fwd_ws_bytes(M, N, K, K);
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
  if (!w || !f || !X || !Y || M < 1 || !aligned(X, 16) || !aligned(Y, 16)) return QL_ERR_INVALID_ARG;
  if (!f->row_ptr || f->nnz < 0 || (f->nnz > 0 && (!f->col || !f->c))) return QL_ERR_INVALID_ARG;
  if (!aligned(f->row_ptr, 4) || !aligned(f->col, 2) || !aligned(f->c, 2)) return QL_ERR_INVALID_ARG;
  if (f->nnz >= (int64_t(1) << 31) || w->K > 65536) return QL_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  if (K < 64 || K % 64 != 0 || N % 8 != 0) return QL_ERR_UNSUPPORTED;
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
  // tensor cores: Y = [X | Z] [W' | F]^T, the adapter as K extension chunks of the fused GEMM
  uint16_t* Z = reinterpret_cast<uint16_t*>(wsb);
  const int64_t zb = round_up(M * K * 2, 256);
  uint16_t* Fd = reinterpret_cast<uint16_t*>(wsb + zb);
  const int64_t fb = round_up(N * K * 2, 256);
  {
    ProfScope prof(PK_FWD_ADAPTER, st, 2);
    e = launch_wht<false>(X, M, K, Z, st);
    if (e != QL_OK) return e;
    const int rows = densify_rows(K);
    const size_t dsm = (size_t)rows * K * 2;
    if (cudaFuncSetAttribute(qwha_densify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm) !=
        cudaSuccess)
      return QL_ERR_CUDA;
    qwha_densify_kernel<<<(unsigned)((N + rows - 1) / rows), 256, dsm, st>>>(f->row_ptr, f->col, f->c, f->nnz,
                                                                          N, K, rows, Fd, device_flag_ptr());
    QL_CHECK_LAUNCH();
  }
  return ext_forward(w, X, M, Z, Fd, K, Y, wsb + zb + fb, ws_bytes - (size_t)(zb + fb), st);
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
