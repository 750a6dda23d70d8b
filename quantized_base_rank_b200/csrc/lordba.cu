// The LoRDBA double-binary adapter branch of the quantised linear (LoRDBA page,
// gist.science/ko/paper/2605.24058, section "2. Methodology", core architecture):
//     Delta W = sum_i diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i),
// with 1-bit sign carriers B1 [N, R], B2 [R, K] and fp16 channel scales.
//
// Algebraically the branch is a low-rank adapter of rank ell*R: stacking the envelope
// terms, Delta W = B_eff A_eff with A_eff rows diag(beta_i) B2 diag(gamma_i) and B_eff
// columns diag(alpha_i) B1. On the tensor cores a sign multiply costs the same as any
// other, so the page's add/subtract kernel buys nothing here. What the format does buy
// is its size, and that is kept: the carriers stay packed in HBM (1 bit per entry).
// Every call expands them with their scales into the bf16 operands of the fused GEMM:
// ell*R*(N + K) bf16, small next to the weight and L2-resident. The second accumulation
// into the GEMM's tile is then the same as for a dense adapter.
#include <cuda_fp16.h>

#include "common.cuh"
#include "weight_check.cuh"

namespace qlb {

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint32_t sign_bit(const uint32_t* __restrict__ row, int j) {
  return (__ldg(row + (j >> 5)) >> (j & 31)) & 1u;
}

// One launch expands both operands, A_eff first, then B_eff (grid-stride over the two
// ranges): the branch costs one small kernel before the GEMM, not two.
//   A_eff [ell*R, K]: element (i*R + j, k) = sign(B2[j][k]) * bf16(beta_i[j] * gamma_i[k])
//   B_eff [N, ell*R]: element (n, i*R + j) = sign(B1[n][j]) * bf16(alpha_i[n])
// The fp16 x fp16 product is exact in fp32; negating a rounded value is exact.
__global__ void __launch_bounds__(256)
lordba_expand_kernel(const uint32_t* __restrict__ B1, const uint32_t* __restrict__ B2,
                     const uint16_t* __restrict__ alpha, const uint16_t* __restrict__ beta,
                     const uint16_t* __restrict__ gamma, int R, int ell, int64_t N, int64_t K,
                     uint16_t* __restrict__ A, uint16_t* __restrict__ Bo) {
  const int64_t wk = (K + 31) / 32;
  const int wr = (R + 31) / 32;
  const int r = ell * R;
  const int64_t ea = (int64_t)r * K, total = ea + N * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    if (e < ea) {
      const int64_t row = e / K, k = e % K;
      const int i = (int)(row / R), j = (int)(row % R);
      const float v = __fmul_rn(half_bits_to_float(beta[i * R + j]), half_bits_to_float(gamma[(int64_t)i * K + k]));
      const uint32_t b = float_to_bf16_bits(v);
      A[e] = (uint16_t)(sign_bit(B2 + j * wk, (int)k) ? b : (b ^ 0x8000u));
    } else {
      const int64_t f = e - ea;
      const int64_t n = f / r;
      const int c = (int)(f % r), i = c / R, j = c % R;
      const uint32_t b = float_to_bf16_bits(half_bits_to_float(alpha[(int64_t)i * N + n]));
      Bo[f] = (uint16_t)(sign_bit(B1 + n * wr, j) ? b : (b ^ 0x8000u));
    }
  }
}

static int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

// Workspace of the LoRDBA forward: A_eff, B_eff, then the forward's own workspace.
int64_t lordba_ws_bytes(int64_t M, int64_t N, int64_t K, int r) {
  return round256(r * K * 2) + round256(N * r * 2) + (int64_t)ql_workspace_bytes(QL_OP_FWD, M, N, K, r);
}

}  // namespace qlb

using namespace qlb;

extern "C" ql_status qlora_linear_fwd_lordba(const ql_weight* w, const ql_bf16* X, int64_t M,
                                             const ql_lordba* ad, ql_bf16* Y, void* ws, size_t ws_bytes,
                                             void* stream) {
  // every refusal of the wrapped forward is made here, before the expansion is launched
  const ql_status ws0 = weight_desc_status(w);
  if (ws0 != QL_OK) return ws0;
  if (!ad || !X || !Y || M < 1 || !aligned(X, 16) || !aligned(Y, 16)) return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (ad->R < 1 || ad->ell < 1 || !ad->B1 || !ad->B2 || !ad->alpha || !ad->beta || !ad->gamma)
    return QL_ERR_INVALID_ARG;
  const int64_t r64 = (int64_t)ad->R * ad->ell;
  if (r64 > 256) return QL_ERR_UNSUPPORTED;
  const int r = (int)r64;
  if (!aligned(ad->B1, 4) || !aligned(ad->B2, 4) || !aligned(ad->alpha, 2) || !aligned(ad->beta, 2) ||
      !aligned(ad->gamma, 2))
    return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes < lordba_ws_bytes(M, N, K, r)) return QL_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* A_eff = reinterpret_cast<uint16_t*>(wsb);
  uint16_t* B_eff = reinterpret_cast<uint16_t*>(wsb + round256(r * K * 2));
  uint8_t* fwd_ws = wsb + round256(r * K * 2) + round256(N * r * 2);
  const size_t fwd_bytes = ws_bytes - (size_t)(fwd_ws - wsb);
  {
    ProfScope prof(PK_FWD_PREP, st, 1);
    const int64_t total = r64 * K + N * r64;
    lordba_expand_kernel<<<(int)imin64((total + 255) / 256, (int64_t)num_sms() * 8), 256, 0, st>>>(
        ad->B1, ad->B2, ad->alpha, ad->beta, ad->gamma, ad->R, ad->ell, N, K, A_eff, B_eff);
    QL_CHECK_LAUNCH();
  }
  // s = alpha / r = 1: the scales are already in A_eff and B_eff
  return qlora_linear_fwd(w, X, M, A_eff, B_eff, r, (float)r, Y, nullptr, fwd_ws, fwd_bytes, stream);
}
