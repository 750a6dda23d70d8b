// Shared device/host helpers of the B200 quantised-linear library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "qlora.h"

namespace qlb {

constexpr int kBlock = 64;        // elements per quantisation block
constexpr int kGroup = 256;       // blocks per double-quantisation group
constexpr int kFlagNonfinite = 1;
constexpr int kFlagTimeout = 2;
constexpr int kFlagBadIndex = 4;    // a sparse index read on the device was out of range

// NF4 grid and its exact decision points, computed once on the host by this
// library (runtime.cu) and passed to kernels by value.
struct Nf4Tables {
  float q[16];          // grid points q_0 < ... < q_15, fp32
  double mid_pos[7];    // positive midpoints (q_j + q_{j+1})/2, j = 8..14, exact in fp64
};

const Nf4Tables& nf4_tables();          // host, computed on first use

// The encoder's decision boundaries for the 128 normal bf16 absmax values in [1, 2),
// a = 1 + f/128: c[f][k] holds the bf16 bits of ceil_bf16(a * m_{8+k}) (the product is
// exact in fp64) in both 16-bit halves; c[f][7] = 0. Rounding to bf16 commutes with a
// power-of-two scale while the result stays normal, so for a = 2^(e-127) (1 + f/128) the
// boundaries are these bits with (e - 127) added to the exponent field.
struct Nf4BoundTable {
  uint32_t c[128][8];
};

const Nf4BoundTable& nf4_bound_table();  // host, computed on first use

// Decode-shaped forward (M <= 16), small_m.cu.
// A Walsh-Hadamard adapter's rows of F (compressed rows) and the transformed tokens Zs
// ([K][16] bf16, token-contiguous) for the decode-shaped kernel.
struct QwhaRows {
  const int32_t* row_ptr;
  const uint16_t* col;
  const uint16_t* c;
  int64_t nnz;
  const uint16_t* Zs;
};
// qw (optional, r = 0 only): the adapter's sparse sums are added before Y's rounding; Zs
// may be written by the grid just before on the stream (it is read after the dependency
// wait), provided that grid was launched without programmatic serialisation.
ql_status small_m_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* A,
                          const uint16_t* B, int r, float alpha, uint16_t* Y, uint16_t* T_save,
                          cudaStream_t st, const QwhaRows* qw = nullptr);
constexpr int64_t kSmallMMax = 16;
bool small_m_supported(int64_t K, int r);   // 0 <= rank <= 64 (0: no adapter), staging fits in smem
int64_t lordba_ws_bytes(int64_t M, int64_t N, int64_t K, int r);   // lordba.cu
// Y = X deq(W)^T + Zext Wext^T (linear.cu): the fused forward GEMM with caller-given
// extension operands [M, kext] and [N, kext] (kext % 64 == 0; 0 = the base product alone);
// scratch of ext_fwd_ws_bytes, 256-aligned
int64_t ext_fwd_ws_bytes(int64_t M, int64_t N, int64_t K, int64_t kext);
ql_status ext_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* Zext,
                      const uint16_t* Wext, int64_t kext, uint16_t* Y, void* ws, size_t ws_bytes,
                      cudaStream_t st, const QwhaRows* qw = nullptr);
// Y = X bf16(deq(W) + dW)^T, dW a dense bf16 [N, K] update added to the decoded weight in
// the fused GEMM (M > 16); scratch of ext_fwd_ws_bytes(M, N, K, 0), 256-aligned (linear.cu)
ql_status dw_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* dW, uint16_t* Y, void* ws,
                     size_t ws_bytes, cudaStream_t st);
int64_t qwha_ws_bytes(int64_t M, int64_t N, int64_t K);             // qwha.cu
int* device_flag_ptr();                 // device address of the sticky flag (current device)
int num_sms();                          // SM count of the current device

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

// Kernel groups that can be timed with CUDA events (ql_profile_enable / ql_profile_read).
enum ProfKind : int {
  PK_NF4 = 0, PK_DQ = 1, PK_INT8 = 2, PK_DEQ = 3, PK_FWD_PREP = 4, PK_FWD_T = 5, PK_FWD_MAIN = 6,
  PK_BWD_PREP = 7, PK_BWD_U = 8, PK_BWD_DB = 9, PK_BWD_DA = 10, PK_BWD_DX = 11, PK_FWD_SMALL = 12,
  PK_FWD_ADAPTER = 13, PK_OPTIM = 14, PK_COUNT = 15
};

// Counts the kernels a scope launches and, when profiling is on, brackets them with a
// pair of CUDA events recorded on the launch stream.
class ProfScope {
 public:
  ProfScope(int kind, cudaStream_t st, int nlaunch);
  ~ProfScope();
 private:
  int kind_;
  cudaStream_t st_;
  bool on_;
  cudaEvent_t a_;
};

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

#define QL_CHECK_LAUNCH()                                         \
  do {                                                            \
    if (cudaGetLastError() != cudaSuccess) return QL_ERR_CUDA;    \
  } while (0)

// ---- device helpers -------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

// fp32 -> bf16 bits, round to nearest even (the hardware conversion).
__device__ __forceinline__ uint32_t float_to_bf16_bits(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void raise_flag(int* flag, int bits) {
  if (flag) atomicOr(flag, bits);
}

}  // namespace qlb
