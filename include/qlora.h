/*
 * qlora.h — C ABI of the B200 (sm_100a) QLoRA-style quantised linear library.
 *
 * The library implements one layer: a frozen weight W [N, K] stored 4-bit (NF4 with
 * double-quantised constants) or 8-bit (blockwise int8), and an unmerged low-rank
 * adapter A [r, K], B [N, r], computing
 *
 *     Y  = X W'^T + s (X A^T) B^T,             s = alpha / r
 *     dX = dY W' + s (dY B) A,  dA = s (dY B)^T X,  dB = s dY^T (X A^T)
 *
 * where W' is the dequantised weight. The formats follow the QLoRA explainer page
 * (aizip.shop/methodologies/qlora): section "1. 4-bit NormalFloat (NF4)" for the grid
 * and section "2. Double Quantization" for blocks of 64 and re-quantised constants;
 * its "memory decomposition" section for the frozen 4-bit base with bf16 adapters.
 * The per-layer choice of bit-width and rank is the allocation C = {(q_l, r_l)} of the
 * AutoQRA page (gist.science/ko/paper/2602.22268), section 3.1.
 *
 * Beside the low-rank adapter, the same quantised linear takes two other unmerged
 * adapters in its forward: LoRDBA's double-binary adapter (qlora_linear_fwd_lordba) and
 * QWHA's Walsh-Hadamard adapter (qlora_linear_fwd_qwha, ql_wht). The adapter's training
 * step has two optimisers: AdamW with states in paged (managed) memory, after the QLoRA
 * page's paged optimiser (ql_adamw_step, ql_paged_*), and Lion with INT8 momentum, after
 * the QFT page (ql_lion_int8_step).
 *
 * Conventions, for every entry point:
 *  - Pointers named "device" are CUDA device pointers owned by the caller. Apart from
 *    ql_paged_alloc / ql_paged_free, which allocate and free managed memory when asked,
 *    the library never allocates or frees caller-visible memory; scratch comes from the
 *    caller's workspace (size from ql_workspace_bytes).
 *  - bf16 tensors are passed as uint16_t bit patterns, row-major, densely packed.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    asynchronous on it; outputs are valid once the stream reaches that point.
 *  - Arguments are checked before anything is launched; a bad argument returns an
 *    error status and launches nothing. No exception crosses the ABI.
 *  - Data-dependent faults found on the device (non-finite inputs, a bounded wait that
 *    gave up) set a sticky device flag instead of trapping; ql_get_device_status
 *    reads and clears it.
 *  - Device pointers must be 16-byte aligned unless stated otherwise.
 *  - The library looks up the device addresses of its own device-side objects (the
 *    status flag, the no-allocation forward's scratch) once per device and keeps them
 *    for the life of the process: do not use it across a cudaDeviceReset.
 */
#ifndef QLORA_B200_H
#define QLORA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t ql_bf16;   /* bf16 bit pattern */

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, bad enum */
  QL_ERR_UNSUPPORTED = 2,   /* well-formed but outside what the kernels handle */
  QL_ERR_WORKSPACE = 3,     /* workspace smaller than ql_workspace_bytes() */
  QL_ERR_NONFINITE = 4,     /* device flag: an input held inf or NaN */
  QL_ERR_TIMEOUT = 5,       /* device flag: a bounded wait inside a kernel gave up */
  QL_ERR_CUDA = 6           /* a CUDA runtime call failed */
} ql_status;

typedef enum {
  QL_FMT_NF4_DQ = 0,        /* 4-bit NF4 codes + double-quantised absmax */
  QL_FMT_INT8_B64 = 1       /* int8 codes + fp32 absmax per block of 64 */
} ql_format;

/* A quantised weight W [N, K] (row-major flattening, blocks of 64 consecutive
 * elements, groups of 256 consecutive blocks). All pointers are device pointers.
 *   NF4_DQ : codes   uint8 [ceil(N*K/2)]   element 2j in the low nibble of byte j
 *            qabsmax int8  [N*K/64]        double-quantised block absmax
 *            group_scale fp32 [ceil(N*K/64/256)]
 *            mean    fp32  [1]             per-tensor mean of the block absmax
 *            absmax  unused (may be NULL)
 *   INT8_B64: codes  int8  [N*K]
 *            absmax  fp32  [N*K/64]
 *            qabsmax, group_scale, mean unused (may be NULL)                       */
typedef struct {
  int32_t fmt;              /* ql_format */
  int32_t reserved;
  int64_t N, K;
  void*   codes;
  float*  absmax;
  int8_t* qabsmax;
  float*  group_scale;
  float*  mean;
} ql_weight;

/* NF4 blockwise quantisation (QLoRA page, "1. 4-bit NormalFloat (NF4)").
 * W: device bf16 [n]. For every block b of 64 consecutive elements (the last block
 * may be partial): absmax[b] = max |W_j| (fp32, exact), and each element's code is the
 * index of the grid point q_i = Q_N((i+1/2)/16)/Q_N(31/32) nearest to W_j/absmax[b]
 * (exact decision, ties to the upper point; an all-zero block gives code 8).
 * codes: device uint8 [ceil(n/2)], absmax: device fp32 [ceil(n/64)].
 * W needs 2-byte alignment; codes and absmax 4-byte. n = 0 is a no-op.
 * Non-finite elements set QL_ERR_NONFINITE on the device flag. */
ql_status nf4_quantize(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax,
                       void* stream);

/* Double quantisation of the block constants (QLoRA page, "2. Double Quantization").
 * absmax: device fp32 [nblocks], finite and >= 0. mean[0] = fp32(S / nblocks), S the
 * exact sum of absmax rounded once to fp64. Per group g of 256 blocks:
 * d = fp32(a - mean), group_scale[g] = fp32(max|d| / 127),
 * qabsmax[b] = clamp(rint_half_even(fp32(d / group_scale[g])), -127, 127)
 * (0 when group_scale[g] == 0).
 * ws: device workspace of at least ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0) bytes.
 * nblocks must be in [1, 2^24]. */
ql_status dq_quantize(const float* absmax, int64_t nblocks, int8_t* qabsmax,
                      float* group_scale, float* mean, void* ws, size_t ws_bytes,
                      void* stream);

/* NF4 with double quantisation in one call (QLoRA page, "1. 4-bit NormalFloat (NF4)"
 * followed by "2. Double Quantization"): the results are bit-identical to nf4_quantize
 * followed by dq_quantize on its absmax. The encode pass also accumulates the exact sum
 * of the block constants, so the constants are not read a second time for the mean.
 * codes, absmax as in nf4_quantize (absmax is still written: the double quantisation
 * reads it); qabsmax [ceil(n/64)], group_scale [ceil(ceil(n/64)/256)], mean [1] as in
 * dq_quantize. ws: at least ql_workspace_bytes(QL_OP_DQ, 0, 0, 0, 0) bytes.
 * n must be in [1, 2^30] (at most 2^24 blocks). */
ql_status nf4_dq_quantize(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax,
                          int8_t* qabsmax, float* group_scale, float* mean, void* ws,
                          size_t ws_bytes, void* stream);

/* One weight of nf4_dq_quantize_batch: the arguments of nf4_dq_quantize (device
 * pointers; W bf16 [n], codes uint8 [ceil(n/2)], absmax fp32 [ceil(n/64)], qabsmax int8
 * [ceil(n/64)], group_scale fp32 [ceil(ceil(n/64)/256)], mean fp32 [1]).               */
typedef struct {
  const ql_bf16* W;
  int64_t n;
  uint8_t* codes;
  float*   absmax;
  int8_t*  qabsmax;
  float*   group_scale;
  float*   mean;
} ql_nf4_dq_item;

/* NF4 + double quantisation of `count` weights, each exactly as nf4_dq_quantize would
 * quantise it (QLoRA page, "1. 4-bit NormalFloat (NF4)" and "2. Double Quantization": one
 * mean per tensor), for quantising a model's linears together. Weights with whole blocks
 * and 16-byte aligned W and codes share four launches per 128 weights: the workspace's
 * sums zeroed, one pass over all their blocks (codes, absmax and each weight's exact DQ
 * sum), the means, and the group encode; any other weight takes the single-weight path on
 * the stream. Every output is
 * bit-identical to nf4_dq_quantize of that weight.
 * items: HOST array of count descriptors (read before the call returns). count = 0 is a
 * no-op. Each item is checked as nf4_dq_quantize checks its arguments; a bad item returns
 * an error before anything is launched.
 * ws: device workspace of ql_workspace_bytes(QL_OP_DQ_BATCH, count, 0, 0, 0) bytes,
 * 16-byte aligned. */
ql_status nf4_dq_quantize_batch(const ql_nf4_dq_item* items, int32_t count, void* ws,
                                size_t ws_bytes, void* stream);

/* NF4 + double quantisation of a weight split across ranks (QLoRA page, "2. Double
 * Quantization": one mean per tensor, so the ranks must agree on the sum of all block
 * constants). Every rank holds a contiguous shard of the flattened weight; every shard
 * but the last holds a multiple of 16384 elements (whole groups of 256 blocks).
 *  1. nf4_quantize_shard: NF4 codes and absmax of the shard as in nf4_quantize, and the
 *     exact sum of its block constants as 16 unsigned 64-bit bins: a finite v >= 0 is
 *     m * 2^(p - 149) with 24-bit m and p in [0, 253], and adds m << (p % 16) to bin
 *     p / 16. bins: device uint64 [16], overwritten. ws as for nf4_dq_quantize.
 *  2. The caller sums the bins over the ranks: an integer all-reduce, exact whatever
 *     the order (each bin stays below 2^63 for at most 2^24 blocks in all).
 *  3. dq_quantize_shard: the mean from the summed bins and the total block count, as in
 *     dq_quantize, then the shard's groups.
 * The result on every rank is bit-identical to nf4_dq_quantize of the whole weight. */
ql_status nf4_quantize_shard(const ql_bf16* W, int64_t n, uint8_t* codes, float* absmax,
                             uint64_t* bins, void* ws, size_t ws_bytes, void* stream);
ql_status dq_quantize_shard(const float* absmax, int64_t nblocks, const uint64_t* bins,
                            int64_t nblocks_total, int8_t* qabsmax, float* group_scale,
                            float* mean, void* stream);

/* Blockwise int8 (the 8-bit choice of the per-layer bit-width, AutoQRA page 3.1):
 * absmax[b] as in nf4_quantize; sc = fp32(absmax[b]/127);
 * codes[j] = clamp(rint_half_even(fp32(W_j / sc)), -127, 127) (0 when sc == 0).
 * W: device bf16 [n]; codes: device int8 [n]; absmax: device fp32 [ceil(n/64)]. */
ql_status int8_quantize(const ql_bf16* W, int64_t n, int8_t* codes, float* absmax,
                        void* stream);

/* Dequantise a whole weight into bf16 W' [N, K] (device). NF4_DQ:
 * a' = fp32(fp32(qabsmax*group_scale) + mean), W'_j = bf16(fp32(q[code_j] * a'));
 * INT8_B64: W'_j = bf16(fp32(code_j * fp32(absmax/127))). Used for checks; the
 * linear kernels dequantise on the fly and never materialise W'. Wout needs 2-byte
 * alignment; the constants (group_scale, mean, absmax) 4-byte. */
ql_status ql_dequantize(const ql_weight* w, ql_bf16* Wout, void* stream);

/* Forward of the quantised linear with an unmerged adapter (QLoRA page, "memory
 * decomposition": frozen 4-bit base + bf16 adapters).
 *   X [M, K] bf16, A [r, K] bf16, B [N, r] bf16 (device), s = alpha / r.
 *   T = X A^T (fp32 accumulate); P = bf16(s T);
 *   Y [M, N] bf16 = bf16(X W'^T + P B^T), fp32 accumulation.
 *   T_save [M, r] bf16 = bf16(T) if non-NULL (needed by qlora_linear_bwd).
 * K % 64 == 0, N % 8 == 0, 1 <= r <= 256, M >= 1. ws: ql_workspace_bytes(QL_OP_FWD, M, N, K, r)
 * bytes (zero, and ws may be NULL, for M <= 16: that decode-shaped case runs as one
 * kernel that splits K over a cluster of 8 CTAs and adds the adapter term per K-range,
 * so its rounding differs from the large-M path within the stated tolerance). */
ql_status qlora_linear_fwd(const ql_weight* w, const ql_bf16* X, int64_t M,
                           const ql_bf16* A, const ql_bf16* B, int32_t r, float alpha,
                           ql_bf16* Y, ql_bf16* T_save, void* ws, size_t ws_bytes,
                           void* stream);

/* Backward with the base frozen: U = dY B (fp32), Q = bf16(s U),
 *   dX [M, K] bf16 = bf16(dY W' + Q A)          (fp32 accumulation)
 *   dA [r, K] fp32 = s U^T X,   dB [N, r] fp32 = s dY^T T_saved
 * X, dY [M, N], T_saved [M, r] from the forward; dA, dB are overwritten.
 * Same shape limits as the forward. ws: ql_workspace_bytes(QL_OP_BWD, M, N, K, r). */
ql_status qlora_linear_bwd(const ql_weight* w, const ql_bf16* X, const ql_bf16* dY,
                           int64_t M, const ql_bf16* A, const ql_bf16* B,
                           const ql_bf16* T_saved, int32_t r, float alpha,
                           ql_bf16* dX, float* dA, float* dB, void* ws,
                           size_t ws_bytes, void* stream);

/* The forward above, for callers that cannot allocate device memory where they run it:
 * a plugin whose host framework owns every device allocation (a private cudaMalloc would
 * escape its pool and accounting), or a latency-bound loop that must not touch the
 * allocator after start-up (cudaMalloc and cudaFree may synchronise the whole device).
 * It has no counterpart on the pages: it
 * only changes where the scratch lives. Instead of a caller workspace it uses one fixed
 * 8 MiB array in the library's device image, which every GPU that loads the library holds
 * until the process exits. Shapes whose ql_workspace_bytes(QL_OP_FWD, ...) exceeds 8 MiB
 * are refused with QL_ERR_WORKSPACE, after the same argument checks as qlora_linear_fwd
 * (so both return the same status for arguments that both refuse). A decode-shaped call
 * (M <= 16, with a K and r that the decode-shaped path supports, i.e. where
 * ql_workspace_bytes returns 0) needs no scratch at all. The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress) and caches it for the life of the
 * process, so the library must not be used across a cudaDeviceReset; make that first call
 * before any stream capture. A failed lookup returns QL_ERR_CUDA. All calls share the one array and nothing
 * in it needs to start at zero (every call rewrites what it reads), but calls that
 * overlap on the GPU (different streams, or different threads) race on it: serialise
 * them. Arguments and outputs are as for qlora_linear_fwd. */
ql_status qlora_linear_fwd_static(const ql_weight* w, const ql_bf16* X, int64_t M,
                                  const ql_bf16* A, const ql_bf16* B, int32_t r, float alpha,
                                  ql_bf16* Y, ql_bf16* T_save, void* stream);

/* A LoRDBA double-binary adapter (LoRDBA page, gist.science/ko/paper/2605.24058, section
 * "2. Methodology", core architecture):
 *     Delta W = sum_{i < ell} diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i)
 * with sign carriers B1 in {+-1}^{N x R} and B2 in {+-1}^{R x K} shared by the ell
 * envelope terms, stored 1 bit per entry, and fp16 channel scales (the page's storage).
 *   B1:    device uint32 [N][ceil(R/32)]: bit j%32 of word j/32 of row n is B1[n][j]
 *          (1 = +1, 0 = -1); unused high bits of a row's last word are ignored.
 *   B2:    device uint32 [R][ceil(K/32)], the same packing for B2[j][k].
 *   alpha: device fp16 bits [ell][N]; beta: [ell][R]; gamma: [ell][K].          */
typedef struct {
  int32_t R, ell;
  const uint32_t* B1;
  const uint32_t* B2;
  const uint16_t* alpha;
  const uint16_t* beta;
  const uint16_t* gamma;
} ql_lordba;

/* Forward of the quantised linear with a LoRDBA adapter branch, unmerged (the page's
 * "adapter mode"): Y [M, N] bf16 = bf16(X W'^T + X Delta W^T), fp32 accumulation.
 * The carriers are expanded with their scales into the bf16 operands of the same
 * fused GEMM as qlora_linear_fwd, at rank ell*R with s = 1:
 *   A_eff[i*R + j][k] = sign(B2[j][k]) * bf16(beta_i[j] * gamma_i[k])
 *   B_eff[n][i*R + j] = sign(B1[n][j]) * bf16(alpha_i[n])
 * (the fp16 x fp16 product is exact in fp32; one rounding to bf16). The adapter's
 * left factor X A_eff^T is rounded to bf16 as in qlora_linear_fwd. Shapes as in
 * qlora_linear_fwd with r = ell*R in [1, 256] (at most 64 for M <= 16).
 * ws: ql_workspace_bytes(QL_OP_FWD_LORDBA, M, N, K, ell*R) bytes. */
ql_status qlora_linear_fwd_lordba(const ql_weight* w, const ql_bf16* X, int64_t M,
                                  const ql_lordba* adapter, ql_bf16* Y, void* ws,
                                  size_t ws_bytes, void* stream);

/* A Walsh-Hadamard adapter (QWHA page, gist.science/ko/paper/2509.17428, section 2.1
 * "Walsh-Hadamard adaptation"): Delta W = F H^{-1}, F [N, K] sparse with values c at the
 * positions of an index list E, H the Walsh-Hadamard transform. E is held in
 * compressed-row form:
 *   row_ptr: device int32 [N + 1], row_ptr[0] = 0, nondecreasing, row_ptr[N] = nnz;
 *   col:     device uint16 [nnz], the column k of each value; within a row, distinct;
 *   c:       device bf16 [nnz], the values (row n holds j in [row_ptr[n], row_ptr[n+1])).
 * H is the orthonormal Sylvester-order Walsh-Hadamard matrix when K is a power of two;
 * otherwise block-diagonal, with blocks of the largest power of two dividing K (so
 * H = H^T = H^{-1}). The caller keeps the arrays alive until the stream passes the call;
 * nothing is copied. col and c may be NULL when nnz = 0. */
typedef struct {
  const int32_t* row_ptr;
  const uint16_t* col;
  const ql_bf16* c;
  int64_t nnz;
} ql_qwha;

/* Forward of the quantised linear with a Walsh-Hadamard adapter, unmerged:
 *   Y [M, N] = bf16( X W'^T + sum over row n's values of c_j * Z[m, col_j] ),
 *   Z = X H^{-T} = X H  (H^{-1} x per token), computed in fp32 by the add/subtract
 *   recursion and rounded once to bf16; products and sums accumulate in fp32 and Y is
 *   rounded once (the large-M form below rounds W' + dW to bf16 first).
 * Shapes and formats as qlora_linear_fwd (K a multiple of 64, K <= 65536, N a multiple
 * of 8); the Walsh-Hadamard block (the largest power of two dividing K) is at most
 * 16384, else QL_ERR_UNSUPPORTED. M <= 16: the transform of the tokens into one slab of
 * Z, then the decode-shaped kernel, which adds each row's sparse sum (Z gathered by
 * column index) to its partial sums before the cluster reduction. M > 16: since H is
 * symmetric, Z F^T = X (F H)^T, so the update dW = bf16(F H) [N, K] is formed (straight
 * from the compressed rows for blocks up to 4096 wide, else from F written out dense and
 * transformed row by row) and the fused GEMM of qlora_linear_fwd adds it to the decoded
 * weight before the product: Y = bf16(X bf16(W' + dW)^T). Column indices >= K and row
 * offsets outside [0, nnz] are skipped on the device and reported as QL_ERR_INVALID_ARG
 * by ql_get_device_status; the contents of the index arrays are not read on the host.
 * Every argument check, the weight's included, is made before the first launch.
 * ws: ql_workspace_bytes(QL_OP_FWD_QWHA, M, N, K, 0) bytes, 256-byte aligned (M <= 16:
 * one slab of Z, [K][16] bf16; otherwise dW [N, K], the dense F [N, K] as well for blocks
 * wider than 4096, and the GEMM's block scales). */
ql_status qlora_linear_fwd_qwha(const ql_weight* w, const ql_bf16* X, int64_t M,
                                const ql_qwha* adapter, ql_bf16* Y, void* ws,
                                size_t ws_bytes, void* stream);

/* The Walsh-Hadamard transform of each token row alone: Z [M, K] bf16 = bf16(X H^{-T})
 * with the H of ql_qwha (orthonormal, blockwise for K not a power of two), by the
 * add/subtract recursion in fp32 (QWHA page, section 2.1, the fast WHT kernel).
 * X and Z are 16-byte aligned, K a multiple of 64, the block at most 16384. */
ql_status ql_wht(const ql_bf16* X, int64_t M, int64_t K, ql_bf16* Z, void* stream);

enum { QL_OP_DQ = 0, QL_OP_FWD = 1, QL_OP_BWD = 2, QL_OP_FWD_LORDBA = 3, QL_OP_FWD_QWHA = 4,
       QL_OP_DQ_BATCH = 5 /* M = the number of weights */ };

/* The adapter optimiser step with paged states (QLoRA page, aizip.shop/methodologies/qlora,
 * section "3. Paged Optimizer": optimiser states held in unified memory, paged to host RAM
 * when device memory runs short). The page names no optimiser; the step is AdamW with
 * bias-corrected moments and weight decay decoupled from the gradient. With
 * g = grad_scale * grad and t = step (1 for the first):
 *   m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2,
 *   theta <- theta (1 - lr weight_decay) - (lr / (1 - beta1^t)) m / (sqrt(v / (1 - beta2^t)) + eps),
 *   param <- bf16(theta)  (round to nearest even),
 * all in fp32 (the bias corrections are formed on the host in fp64). grad_scale folds a
 * data-parallel average (1/world) into the step. */
typedef struct {
  float lr, beta1, beta2, eps, weight_decay, grad_scale;
  int64_t step;
} ql_adamw;

/* One step over n adapter parameters held as one flat vector: theta, grad, m, v fp32
 * [n] (theta the trained copy, m and v zero before step 1), param bf16 [n] (written).
 * Every array is device memory or managed memory from ql_paged_alloc; 4-byte aligned
 * (2 for param); 16-byte alignment and n % 4 == 0 take the vector path. The arrays must
 * not overlap. A non-finite gradient element sets QL_ERR_NONFINITE on the device flag
 * (the step still runs). Hyperparameters outside their domain (step < 1, beta not in
 * [0, 1), eps <= 0, negative lr or weight decay) return QL_ERR_INVALID_ARG. */
ql_status ql_adamw_step(float* theta, ql_bf16* param, const float* grad, float* m, float* v, int64_t n,
                        const ql_adamw* hparams, void* stream);

/* Lion with INT8 momentum (QFT page, gist.science/ko/paper/2310.07147, section 2.1: Lion
 * keeps only a momentum, its update is a sign of fixed size, and the momentum is stored in
 * INT8). With fp32 values and one IEEE rounding per operation, omb = 1 - beta and
 * decay = 1 - lr * weight_decay:
 *   m      = code * (absmax_block / 127)           (the stored momentum, decoded)
 *   c      = beta1 m + omb1 g
 *   theta <- theta decay - lr sign(c)              (sign(0) = 0)
 *   m'     = beta2 m + omb2 g, re-encoded per block of 64: absmax' = max |m'|,
 *            code' = clamp(rint(m' / (absmax' / 127)), -127, 127) (0 for a zero block)
 *   param <- bf16(theta)                          (round to nearest even)
 * The page names no INT8 scheme for the momentum; this is the blockwise absmax code of the
 * int8 weight format. */
typedef struct {
  float lr, beta1, beta2, weight_decay;
} ql_lion;

/* One step over n parameters: theta, grad fp32 [n]; m_codes int8 [n] and m_absmax fp32
 * [ceil(n/64)] (all zero before the first step), both updated; param bf16 [n] written.
 * Device or paged memory. A non-finite gradient sets QL_ERR_NONFINITE on the device flag. */
ql_status ql_lion_int8_step(float* theta, ql_bf16* param, const float* grad, int8_t* m_codes,
                            float* m_absmax, int64_t n, const ql_lion* hparams, void* stream);

/* Paged memory for optimiser states: `bytes` of CUDA managed (unified) memory, usable by
 * the kernels and the host alike, whose pages the driver migrates between device and host
 * memory on demand (and evicts to the host when device memory is oversubscribed).
 * *out = NULL for bytes = 0. Free with ql_paged_free. The caller owns the memory. */
ql_status ql_paged_alloc(size_t bytes, void** out);
ql_status ql_paged_free(void* ptr);

/* Move the pages of [ptr, ptr + bytes) of paged memory to the host (to_host != 0) or to
 * the current device, asynchronously on `stream`: the explicit form of the paging, ahead
 * of the step that touches them (or away from the device between steps). */
ql_status ql_paged_prefetch(const void* ptr, size_t bytes, int32_t to_host, void* stream);

/* Workspace bytes that op (QL_OP_*) needs for these sizes (0 if none). */
size_t ql_workspace_bytes(int32_t op, int64_t M, int64_t N, int64_t K, int32_t r);

/* Synchronise `stream`, then return and clear the sticky device flag of the current
 * device (QL_OK, QL_ERR_NONFINITE, QL_ERR_TIMEOUT, or QL_ERR_INVALID_ARG when a sparse
 * index read on the device was out of range). */
ql_status ql_get_device_status(void* stream);

/* Which fused weight GEMM the linear uses for M > 16: 0 (the default) runs it on single
 * CTAs (128 weight rows x 256 tokens per tile), 1 on CTA pairs (two SMs share each tcgen05
 * MMA, cta_group::2, 256 weight rows x 256 tokens). Both give the same results up to fp32
 * summation order. Process-wide; meant for comparisons. */
void ql_set_gemm_pair(int on);

/* Upper bound, in nanoseconds, on every wait inside the GEMM kernels (0 restores the
 * default of 2 s). A wait that exceeds it makes the kernel give up cleanly and report
 * QL_ERR_TIMEOUT through ql_get_device_status. Process-wide; meant for diagnostics. */
void ql_set_wait_timeout_ns(uint64_t ns);

/* Measurement hooks. When enabled, every kernel group launched by the entry points is
 * bracketed by two CUDA events on its launch stream; ql_profile_read synchronises on
 * them and returns (then forgets) the summed milliseconds and the number of launches of
 * one group. Groups: 0 nf4 encode, 1 double quantisation, 2 int8 encode, 3 dequantise,
 * 4 forward layout prep, 5 forward X A^T, 6 forward main GEMM, 7 backward layout prep,
 * 8 backward dY B, 9 dB, 10 dA, 11 dX, 12 small-M forward, 13 Walsh-Hadamard adapter
 * (transform and sparse product), 14 optimiser step. ql_launch_count is the
 * running number of kernels the library has launched in this process. Returns 0, or -1
 * for an unknown group. */
void ql_profile_enable(int on);
int ql_profile_read(int kind, double* total_ms, int64_t* count);
uint64_t ql_launch_count(void);

/* Static description of a status code. */
const char* ql_status_string(ql_status s);

/* The 16 NF4 grid points as the library computes them (host memory, fp32[16]). */
void ql_nf4_codebook(float* out16);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_B200_H */
