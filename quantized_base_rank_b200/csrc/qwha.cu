// Walsh-Hadamard adapter in the quantised linear (QWHA page,
// gist.science/ko/paper/2509.17428, section 2.1 "Walsh-Hadamard adaptation"):
//
//   Y = X deq(W)^T + X (F H^{-1})^T = base + Z F^T,    Z = X H^{-T} = X H
//
// H is the orthonormal Sylvester-order Walsh-Hadamard matrix, block-diagonal in blocks of
// b = the largest power of two dividing K (H = H^T = H^{-1}); F [N, K] is sparse, held as
// compressed rows (row_ptr, col, c). The adapter stays unmerged: after the base product,
//
//  * qwha_wht_kernel forms Z = X H per token and block by the fast butterfly recursion,
//    adds and subtracts only, in fp32 (the page's point: no multiplies by H), and writes
//    it once as bf16 in a token-slab layout Zs[slab][k][16]: the 16 tokens of a slab are
//    contiguous, so column k of a slab is one 32-byte sector;
//  * qwha_spmm_kernel adds, for every output row n and token m,
//    sum_j c_j Z[m, col_j] over row n's stored values, in fp32, into Y in place.
//
// The gather of Z by column index has no tensor-core form (F's positions are arbitrary),
// so the second kernel runs on the FMA pipes, its slab of Z staged in shared memory when
// it fits.
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

// One pass over the index bits [lo, lo + NB) of every length-b row held in shared memory
// (rows of `pitch` floats, TT rows). A group is the 2^NB elements that differ only in
// those bits; consecutive threads take groups with consecutive low bits, so a warp's
// accesses to one element of its groups are consecutive words.
template <int NB>
__device__ __forceinline__ void smem_pass(float* sm, int TT, int b, int pitch, int lo) {
  const int per_row = b >> NB;                   // groups per row
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
#pragma unroll
    for (int j = 0; j < (1 << NB); ++j) row[phys(base + (j << lo))] = v[j];
  }
}

// Z = X H for TT tokens [m0, m0 + TT) and one Walsh-Hadamard block [bi*b, bi*b + b) of the
// input width. L = log2(b) >= 6 (K is a multiple of 64). Tokens at or past M read as zero,
// so a slab's tail is written as zeros. SLAB: Zs[m / 16][k][m % 16]; otherwise Z [M][K].
template <bool SLAB>
__global__ void __launch_bounds__(256)
qwha_wht_kernel(const uint16_t* __restrict__ X, int64_t M, int64_t K, int L, int TT, float scale,
                uint16_t* __restrict__ Z) {
  extern __shared__ __align__(16) float wsm[];
  const int b = 1 << L;
  const int pitch = qwha_pitch(b);
  const int64_t m0 = (int64_t)blockIdx.x * TT;
  const int64_t k0 = (int64_t)blockIdx.y * b;

  // pass 0: 16 contiguous elements per thread from global, bits 0..3 in registers
  {
    const int per_row = b >> 4;
    for (int gi = threadIdx.x; gi < TT * per_row; gi += blockDim.x) {
      const int t = gi / per_row, e0 = (gi - t * per_row) << 4;
      const int64_t m = m0 + t;
      uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
      if (m < M) {
        const uint4* src = reinterpret_cast<const uint4*>(X + m * K + k0 + e0);
        u0 = __ldg(src);
        u1 = __ldg(src + 1);
      }
      float v[16] = {bf16_lo(u0.x), bf16_hi(u0.x), bf16_lo(u0.y), bf16_hi(u0.y),
                     bf16_lo(u0.z), bf16_hi(u0.z), bf16_lo(u0.w), bf16_hi(u0.w),
                     bf16_lo(u1.x), bf16_hi(u1.x), bf16_lo(u1.y), bf16_hi(u1.y),
                     bf16_lo(u1.z), bf16_hi(u1.z), bf16_lo(u1.w), bf16_hi(u1.w)};
      butterflies<4>(v);
      float* dst = wsm + (size_t)t * pitch + phys(e0);
#pragma unroll
      for (int j = 0; j < 16; ++j) dst[j] = v[j];
    }
  }
  __syncthreads();
  // the remaining bits, up to four per pass
  for (int lo = 4; lo < L; lo += 4) {
    switch (L - lo >= 4 ? 4 : L - lo) {
      case 4: smem_pass<4>(wsm, TT, b, pitch, lo); break;
      case 3: smem_pass<3>(wsm, TT, b, pitch, lo); break;
      case 2: smem_pass<2>(wsm, TT, b, pitch, lo); break;
      default: smem_pass<1>(wsm, TT, b, pitch, lo); break;
    }
    __syncthreads();
  }

  if (SLAB) {
    // one column k per thread: the TT tokens' values, contiguous in the slab
    const int64_t slab = m0 / kQwSlab;
    const int t0 = (int)(m0 % kQwSlab);
    for (int k = threadIdx.x; k < b; k += blockDim.x) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = 2 * i < TT ? wsm[(size_t)(2 * i) * pitch + phys(k)] * scale : 0.0f;
        const float c = 2 * i + 1 < TT ? wsm[(size_t)(2 * i + 1) * pitch + phys(k)] * scale : 0.0f;
        w[i] = f2_to_bf16x2(a, c);
      }
      uint16_t* dst = Z + ((slab * K + k0 + k) * kQwSlab + t0);
      if (TT == 16) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
      } else if (TT == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      } else if (TT == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
      } else if (TT == 2) {
        *reinterpret_cast<uint32_t*>(dst) = w[0];
      } else {
        *dst = (uint16_t)(w[0] & 0xFFFFu);
      }
    }
  } else {
    // eight consecutive k of one token per thread
    const int per_row = b >> 3;
    for (int gi = threadIdx.x; gi < TT * per_row; gi += blockDim.x) {
      const int t = gi / per_row, e0 = (gi - t * per_row) << 3;
      const int64_t m = m0 + t;
      if (m >= M) continue;
      const float* src = wsm + (size_t)t * pitch + phys(e0);   // e0 % 8 == 0: no gap inside
      const uint4 o = make_uint4(f2_to_bf16x2(src[0] * scale, src[1] * scale),
                                 f2_to_bf16x2(src[2] * scale, src[3] * scale),
                                 f2_to_bf16x2(src[4] * scale, src[5] * scale),
                                 f2_to_bf16x2(src[6] * scale, src[7] * scale));
      *reinterpret_cast<uint4*>(Z + m * K + k0 + e0) = o;
    }
  }
}

// Decode-shaped sparse product (M <= 16, one slab):
//   Y[m, n] += sum_j c_j Z[m, col_j], j over row n's stored values.
// A warp takes 8 consecutive rows (N is a multiple of 8). Each row's values are read 32 at
// a time, one (col, c) pair per lane, and handed out by shuffles: lane = (stream
// s = lane / 8, token pair tp = lane % 8), stream s takes values s, s + 4, ... of the
// chunk, so each chunk issues 8 independent 4-byte gathers of Z per lane. Each lane keeps
// two tokens' fp32 sums per row; the streams are combined by a fixed xor butterfly (the
// result does not depend on scheduling) and the sum is added to the base product with
// one bf16 rounding. Columns at or past K, or row offsets outside [0, nnz], are skipped
// and raise the device's bad-index flag.
__global__ void __launch_bounds__(256)
qwha_spmm_kernel(const uint16_t* __restrict__ Zs, int64_t M, int64_t N, int64_t K,
                 const int32_t* __restrict__ row_ptr, const uint16_t* __restrict__ col,
                 const uint16_t* __restrict__ cval, int64_t nnz, uint16_t* __restrict__ Y, int* flag) {
  const int64_t slab = blockIdx.y;
  const uint16_t* zsrc = Zs + slab * K * kQwSlab;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = lane >> 3, tp = lane & 7;
  const int64_t rg = (int64_t)blockIdx.x * 64 + warp * 8;
  if (rg >= N) return;                               // whole warp: its 8 rows are all outside
  bool bad = false;
  int off = 0;                                       // lanes 0..8: the 9 row offsets
  if (lane < 9) off = __ldg(row_ptr + rg + lane);
  float acc[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[i][0] = acc[i][1] = 0.0f;
    int j0 = __shfl_sync(0xffffffffu, off, i), j1 = __shfl_sync(0xffffffffu, off, i + 1);
    if (j0 < 0 || (int64_t)j1 > nnz || j0 > j1) {
      bad = true;
      j0 = j1 = 0;
    }
    for (int jc = j0; jc < j1; jc += 32) {
      uint32_t wv = 0u;                              // col | c << 16; 0 adds nothing
      if (jc + lane < j1) wv = (uint32_t)__ldg(col + jc + lane) | ((uint32_t)__ldg(cval + jc + lane) << 16);
      if ((int64_t)(wv & 0xFFFFu) >= K) {
        bad = true;
        wv = 0u;
      }
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const uint32_t we = __shfl_sync(0xffffffffu, wv, 4 * it + s);
        const uint32_t z = __ldg(reinterpret_cast<const uint32_t*>(zsrc + (size_t)(we & 0xFFFFu) * kQwSlab) + tp);
        const float cv = __uint_as_float(we & 0xFFFF0000u);
        acc[i][0] = fmaf(cv, bf16_lo(z), acc[i][0]);
        acc[i][1] = fmaf(cv, bf16_hi(z), acc[i][1]);
      }
    }
  }
  // combine the four streams (lanes tp, tp + 8, tp + 16, tp + 24)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 8);
      acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 16);
    }
  }
  // stream 0 adds token 2tp, stream 1 token 2tp + 1 into the base product (8 rows = 16 B)
  if (s < 2) {
    const int64_t m = slab * kQwSlab + 2 * tp + s;
    if (m < M) {
      uint4* py = reinterpret_cast<uint4*>(Y + m * N + rg);
      const uint4 y = *py;
      const uint32_t yw[4] = {y.x, y.y, y.z, y.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = f2_to_bf16x2(bf16_lo(yw[q]) + (s ? acc[2 * q][1] : acc[2 * q][0]),
                            bf16_hi(yw[q]) + (s ? acc[2 * q + 1][1] : acc[2 * q + 1][0]));
      *py = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (bad) raise_flag(flag, kFlagBadIndex);
}

// F written out densely for the tensor cores: Fd [N, K] bf16 (zeroed beforehand) gets c_j
// at (n, col_j). One warp per row; the same index checks as the sparse product.
__global__ void __launch_bounds__(256)
qwha_densify_kernel(const int32_t* __restrict__ row_ptr, const uint16_t* __restrict__ col,
                    const uint16_t* __restrict__ cval, int64_t nnz, int64_t N, int64_t K,
                    uint16_t* __restrict__ Fd, int* flag) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t n = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; n < N; n += warps) {
    int64_t j0 = __ldg(row_ptr + n), j1 = __ldg(row_ptr + n + 1);
    if (j0 < 0 || j1 > nnz || j0 > j1) {
      bad = true;
      continue;
    }
    for (int64_t j = j0 + lane; j < j1; j += 32) {
      const uint32_t k = __ldg(col + j);
      if (k >= (uint64_t)K) {
        bad = true;
        continue;
      }
      Fd[n * K + k] = __ldg(cval + j);
    }
  }
  if (bad) raise_flag(flag, kFlagBadIndex);
}

// ---- host side -------------------------------------------------------------------------

static int log2_exact(int64_t b) {
  int L = 0;
  while ((int64_t(1) << L) < b) ++L;
  return L;
}

// tokens per WHT block: about 64 KB of fp32 rows per CTA, so two CTAs share an SM
static int wht_tokens(int64_t b) {
  int tt = 16;
  while (tt > 1 && (int64_t)tt * b > 16384) tt >>= 1;
  return tt;
}

static size_t wht_smem(int64_t b, int tt) { return (size_t)tt * qwha_pitch((int)b) * 4; }

static bool qwha_decode_shaped(int64_t M, int64_t K) { return M <= kSmallMMax && small_m_supported(K, 0); }

// Workspace: decode-shaped, the one slab of Z; otherwise Z [M, K] and the dense F [N, K]
// (bf16) plus the fused GEMM's scratch.
int64_t qwha_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (qwha_decode_shaped(M, K)) return round_up(K * kQwSlab * 2, 256);
  return round_up(M * K * 2, 256) + round_up(N * K * 2, 256) + ext_fwd_ws_bytes(M, N, K, K);
}

// Z = X H: SLAB (decode-shaped, one token per CTA, tokens < M only: the slab's other
// columns are never added to Y) or row-major [M, K].
template <bool SLAB>
static ql_status launch_wht(const uint16_t* X, int64_t M, int64_t K, uint16_t* Z, cudaStream_t st) {
  const int64_t b = K & (-K);
  const int L = log2_exact(b);
  const int tt = SLAB ? 1 : wht_tokens(b);
  const size_t smem = wht_smem(b, tt);
  if (L < 6 || L > 15 || smem > 200 * 1024) return QL_ERR_UNSUPPORTED;
  auto kern = qwha_wht_kernel<SLAB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const dim3 grid((unsigned)((M + tt - 1) / tt), (unsigned)(K / b));
  if ((M + tt - 1) / tt > 0x7fffffff) return QL_ERR_UNSUPPORTED;
  const float scale = (float)(1.0 / std::sqrt((double)b));
  kern<<<grid, 256, smem, st>>>(X, M, K, L, tt, scale, Z);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

}  // namespace qlb

using namespace qlb;

extern "C" {

ql_status qlora_linear_fwd_qwha(const ql_weight* w, const ql_bf16* X, int64_t M, const ql_qwha* f, ql_bf16* Y,
                                void* ws, size_t ws_bytes, void* stream) {
  if (!w || !f || !X || !Y || M < 1) return QL_ERR_INVALID_ARG;
  if (!f->row_ptr || f->nnz < 0 || (f->nnz > 0 && (!f->col || !f->c))) return QL_ERR_INVALID_ARG;
  if (!aligned(f->row_ptr, 4) || !aligned(f->col, 2) || !aligned(f->c, 2)) return QL_ERR_INVALID_ARG;
  if (f->nnz >= (int64_t(1) << 31) || w->K > 65536) return QL_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  if (K < 64 || K % 64 != 0 || N % 8 != 0) return QL_ERR_UNSUPPORTED;
  if ((int64_t)ws_bytes < qwha_ws_bytes(M, N, K)) return QL_ERR_WORKSPACE;
  {
    const int64_t b = K & (-K);
    if (wht_smem(b, wht_tokens(b)) > 200 * 1024) return QL_ERR_UNSUPPORTED;
  }
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  ql_status e;
  if (qwha_decode_shaped(M, K)) {
    // the base product (decode-shaped kernel), then Z = X H and the sparse product
    uint16_t* Zs = reinterpret_cast<uint16_t*>(wsb);
    e = ext_forward(w, X, M, nullptr, nullptr, 0, Y, nullptr, 0, st);
    if (e != QL_OK) return e;
    ProfScope prof(PK_FWD_ADAPTER, st, 2);
    e = launch_wht<true>(X, M, K, Zs, st);
    if (e != QL_OK || f->nnz == 0) return e;
    const dim3 grid((unsigned)((N + 63) / 64), 1u);
    qwha_spmm_kernel<<<grid, 256, 0, st>>>(Zs, M, N, K, f->row_ptr, f->col, f->c, f->nnz, Y, device_flag_ptr());
    QL_CHECK_LAUNCH();
    return QL_OK;
  }
  // tensor cores: Y = [X | Z] [W' | F]^T, the adapter as K extension chunks of the fused GEMM
  uint16_t* Z = reinterpret_cast<uint16_t*>(wsb);
  const int64_t zb = round_up(M * K * 2, 256);
  uint16_t* Fd = reinterpret_cast<uint16_t*>(wsb + zb);
  const int64_t fb = round_up(N * K * 2, 256);
  {
    ProfScope prof(PK_FWD_ADAPTER, st, 3);
    e = launch_wht<false>(X, M, K, Z, st);
    if (e != QL_OK) return e;
    if (cudaMemsetAsync(Fd, 0, (size_t)(N * K * 2), st) != cudaSuccess) return QL_ERR_CUDA;
    if (f->nnz > 0) {
      qwha_densify_kernel<<<(unsigned)imin64((N + 7) / 8, (int64_t)num_sms() * 8), 256, 0, st>>>(
          f->row_ptr, f->col, f->c, f->nnz, N, K, Fd, device_flag_ptr());
      QL_CHECK_LAUNCH();
    }
  }
  return ext_forward(w, X, M, Z, Fd, K, Y, wsb + zb + fb, ws_bytes - (size_t)(zb + fb), st);
}

ql_status ql_wht(const ql_bf16* X, int64_t M, int64_t K, ql_bf16* Z, void* stream) {
  if (!X || !Z || M < 1 || K < 64) return QL_ERR_INVALID_ARG;
  if (K % 64 != 0 || M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!aligned(X, 16) || !aligned(Z, 16)) return QL_ERR_INVALID_ARG;
  const int64_t b = K & (-K);
  if (wht_smem(b, wht_tokens(b)) > 200 * 1024) return QL_ERR_UNSUPPORTED;
  ProfScope prof(PK_FWD_ADAPTER, as_stream(stream), 1);
  return launch_wht<false>(X, M, K, Z, as_stream(stream));
}

}  // extern "C"
