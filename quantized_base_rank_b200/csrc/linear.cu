// The quantised linear layer with an unmerged LoRA branch: forward, input-backward and
// adapter gradients, built from instances of the tcgen05 GEMM in gemm.cuh.
//
// QLoRA page (aizip.shop/methodologies/qlora), "memory decomposition": the frozen base
// is stored 4-bit and the adapters stay bf16 and unmerged. AutoQRA page
// (gist.science/ko/paper/2602.22268) section 3.1: each layer picks its bit-width
// (NF4+DQ or int8 here) and its rank r.
//
// Forward  (3 launches): pad B -> Bp;  [T | P] = X A^T  (P = bf16(s T));
//                        Y = X W'^T + P Bp^T  (W' decoded in the producer warps, P Bp^T
//                        as extra contraction chunks of the same accumulator)
// Backward (5 launches): prep (B^T, A^T padded, T padded); Q = bf16(s dY B);
//                        dB = s dY^T T;  dA = Q^T X;  dX = dY W' + Q A.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"

namespace qlb {

static std::atomic<uint64_t> g_wait_timeout_ns{2000000000ull};

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor [outer, inner] with row stride `ld_bytes`; box {box_inner, box_outer}.
static bool make_map_t(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* ptr,
                       uint64_t inner, uint64_t outer, uint64_t ld_bytes, uint32_t box_inner,
                       uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  (void)esize;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 matrix [outer, inner] with row stride `ld` elements; box {64, box_outer} with the
// 128-byte swizzle (one 128-byte smem row per box row).
static bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_outer) {
  return make_map_t(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, inner, outer, ld * 2, 64, box_outer,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BN, bool A_MN, bool B_MN, int EPI>
static ql_status launch_tma(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args,
                            cudaStream_t st) {
  auto kern = qgemm_tma_kernel<BN, A_MN, B_MN, EPI>;
  const size_t smem = TmaCfg<BN>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const int64_t items = ((args.R + 127) / 128) * ((args.Cn + BN - 1) / BN) * (args.ksplit > 1 ? args.ksplit : 1);
  const int grid = (int)imin64(items, num_sms());
  if (grid <= 0) return QL_OK;
  kern<<<grid, 192, smem, st>>>(a, b, args);
  QL_CHECK_LAUNCH();
  if (args.ksplit > 1) {
    const int64_t threads = args.R * ((args.Cn + 31) / 32);
    reduce_partials_kernel<EPI><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(args);
    QL_CHECK_LAUNCH();
  }
  return QL_OK;
}

template <int EPI, bool A_MN, bool B_MN>
static ql_status launch_tma_rp(int rp, const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args,
                               cudaStream_t st) {
  if (rp == 64) return launch_tma<64, A_MN, B_MN, EPI>(a, b, args, st);
  if (rp == 128) return launch_tma<128, A_MN, B_MN, EPI>(a, b, args, st);
  if (rp == 192) return launch_tma<192, A_MN, B_MN, EPI>(a, b, args, st);
  return launch_tma<256, A_MN, B_MN, EPI>(a, b, args, st);
}

// Process-wide choice of the fused weight GEMM: 1 = CTA pair (cta_group::2), 0 = one CTA
// (the default: on the 8192 x 11008 x 4096 up-projection the two measure within a few
// percent of each other, the single-CTA kernel ahead).
static std::atomic<int> g_gemm_pair{0};

template <BSrc BS, bool W_MN, bool DW = false>
static ql_status launch_wpair(const CUtensorMap& tok, const CUtensorMap& codes, const CUtensorMap& scale,
                              const CUtensorMap& tok_ext, const CUtensorMap& w_ext, const GemmArgs& args,
                              cudaStream_t st, const CUtensorMap* dw = nullptr) {
  auto kern = qgemm_wpair_kernel<BS, W_MN, DW>;
  if (DW && (!dw || args.n_ext != 0)) return QL_ERR_INVALID_ARG;
  const size_t smem = WpairCfg<BS, DW>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const int64_t tiles = ((args.R + 255) / 256) * ((args.Cn + 255) / 256);
  const int pairs = (int)imin64(tiles, num_sms() / 2);
  if (pairs <= 0) return QL_OK;
  kern<<<2 * pairs, WpairCfg<BS, DW>::kThreads, smem, st>>>(tok, codes, scale, tok_ext, w_ext, dw ? *dw : tok, args);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

// dw: the dense update added to the decoded weight (forward, no extension chunks), or null
template <BSrc BS, bool W_MN, bool DW = false>
static ql_status launch_wdec(const CUtensorMap& tok, const CUtensorMap& codes, const CUtensorMap& scale,
                             const CUtensorMap& tok_ext, const CUtensorMap& w_ext, const GemmArgs& args,
                             cudaStream_t st, const CUtensorMap* dw = nullptr) {
  auto kern = qgemm_wdec_kernel<BS, W_MN, DW>;
  if (DW && (!dw || args.n_ext != 0)) return QL_ERR_INVALID_ARG;
  const size_t smem = WdecCfg<BS, DW>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QL_ERR_CUDA;
  const int64_t tiles = ((args.R + 127) / 128) * ((args.Cn + 255) / 256);
  const int grid = (int)imin64(tiles, num_sms());
  if (grid <= 0) return QL_OK;
  kern<<<grid, WdecCfg<BS, DW>::kThreads, smem, st>>>(tok, codes, scale, tok_ext, w_ext, dw ? *dw : tok, args);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

// ---- small layout kernels (adapter-sized tensors only) ----------------------------

// dst[i, j] = j < r ? src[i, j] : 0, dst [rows, rp]
__global__ void pad_cols_kernel(const uint16_t* __restrict__ src, int64_t rows, int r, int rp,
                                uint16_t* __restrict__ dst) {
  const int64_t total = rows * rp;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / rp;
    const int j = (int)(i % rp);
    dst[i] = j < r ? src[row * r + j] : (uint16_t)0;
  }
}

// dst[c, j] = j < r ? src[j, c] : 0, src [r, cols], dst [cols, rp]
__global__ void transpose_pad_kernel(const uint16_t* __restrict__ src, int r, int64_t cols, int rp,
                                     uint16_t* __restrict__ dst) {
  const int64_t total = cols * rp;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i / rp;
    const int j = (int)(i % rp);
    dst[i] = j < r ? src[(int64_t)j * cols + c] : (uint16_t)0;
  }
}

// dst[j, n] = src[n, j], src [rows, r], dst [r, rows]
__global__ void transpose_kernel(const uint16_t* __restrict__ src, int64_t rows, int r,
                                 uint16_t* __restrict__ dst) {
  const int64_t total = rows * r;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(i / rows);
    const int64_t n = i % rows;
    dst[i] = src[n * r + j];
  }
}

// Rebuilt block scales, fp32, one per block of 64 weight elements:
//   NF4+DQ: a' = fp32(fp32(c8 * s_g) + mean);  int8: sc = fp32(absmax / 127).
// major == 0: block-major copy out[kb * N + n] (forward: a stage reads 256 consecutive rows
// of one block column); major == 1: row-major out[n * ld + kb] (dX: a stage reads 4
// consecutive blocks of 64 rows). ld is padded so TMA row strides are 16-byte multiples.
__global__ void block_scale_kernel(int fmt, const int8_t* __restrict__ qabsmax,
                                   const float* __restrict__ gscale, const float* __restrict__ mean,
                                   const float* __restrict__ absmax, int64_t N, int64_t KB, int major,
                                   int64_t ld, float* __restrict__ out) {
  const int64_t total = N * KB;
  const float mu = fmt == QL_FMT_NF4_DQ ? *mean : 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t n, kb;
    if (major == 0) { kb = i / N; n = i % N; } else { n = i / KB; kb = i % KB; }
    const int64_t blk = n * KB + kb;
    float v;
    if (fmt == QL_FMT_NF4_DQ) v = __fadd_rn(__fmul_rn((float)qabsmax[blk], gscale[blk >> 8]), mu);
    else v = __fdiv_rn(absmax[blk], 127.0f);
    out[major == 0 ? kb * N + n : n * ld + kb] = v;
  }
}

static int small_grid(int64_t n) { return (int)imax64(1, imin64((n + 255) / 256, (int64_t)num_sms() * 8)); }


struct WsLayout {
  int64_t off[6];
  int64_t total;
};

// Split-K for the adapter GEMMs of the backward, which stream a whole activation (dY or
// X) against a narrow factor and have few 128-row tiles: the number of contraction
// slices ks <= 8 that minimises the busiest CTA's share, ceil(tiles * ks / 148) / ks
// (148 SMs; a fixed count keeps the workspace size independent of the device), the
// smaller ks on ties, and never more slices than 64-wide chunks.
struct SplitK {
  int ks, kc_per;
};

static SplitK split_k(int64_t R, int64_t Cn, int64_t Kc, int BN) {
  const int64_t tiles = ((R + 127) / 128) * ((Cn + BN - 1) / BN);
  const int64_t kc_total = (Kc + 63) / 64;
  int best = 1;
  double best_share = 1.0;
  for (int ks = 2; ks <= 8; ++ks) {
    const double share = (double)((tiles * ks + 147) / 148) / ks;
    if (share < best_share - 1e-9) { best = ks; best_share = share; }
  }
  if (best > kc_total) best = (int)imax64(1, kc_total);
  const int kc_per = (int)((kc_total + best - 1) / best);
  SplitK k{(int)((kc_total + kc_per - 1) / kc_per), kc_per};   // no empty slice
  return k;
}

static int rp_bn(int64_t rp) { return rp <= 64 ? 64 : rp <= 128 ? 128 : rp <= 192 ? 192 : 256; }

// Bytes of split-K partials of one adapter GEMM: [ks][R][columns of its tiles] fp32.
static int64_t partial_bytes(int64_t R, int64_t rp, int64_t Kc) {
  const int bn = rp_bn(rp);
  const SplitK k = split_k(R, rp, Kc, bn);
  return k.ks > 1 ? (int64_t)k.ks * R * round_up(rp, bn) * 4 : 0;
}

// Turn on split-K for an adapter GEMM of padded rank rp, with its partials at `part`.
// Returns the number of kernels the GEMM then launches (1 or 2).
static int apply_split(GemmArgs& a, float* part, int64_t rp) {
  const int bn = rp_bn(rp);
  const SplitK k = split_k(a.R, a.Cn, a.Kc, bn);
  a.ksplit = k.ks;
  a.kc_per = k.kc_per;
  a.part = part;
  a.ldp = round_up(a.Cn, bn);
  return k.ks > 1 ? 2 : 1;
}

static WsLayout ws_layout(int op, int64_t M, int64_t N, int64_t K, int r) {
  WsLayout L{};
  const int64_t rp = round_up(r, 64);
  int64_t sz[6] = {0, 0, 0, 0, 0, 0};
  if (op == QL_OP_FWD) {
    sz[0] = M * rp * 2;        // P
    sz[1] = N * rp * 2;        // B padded
    sz[4] = (K / 64) * N * 4;  // block scales, block-major
  } else if (op == QL_OP_BWD) {
    sz[0] = M * rp * 2;        // Q
    sz[1] = (int64_t)r * N * 2;  // B^T
    sz[2] = K * rp * 2;        // A^T padded
    sz[3] = M * rp * 2;        // T padded
    sz[4] = N * round_up(K / 64, 4) * 4;  // block scales, row-major (padded rows)
    // split-K partials, shared by dY B (rows M, contraction N), dB (rows N, over M) and
    // dA (rows K, over M), which run one after another
    sz[5] = imax64(partial_bytes(M, rp, N), imax64(partial_bytes(N, rp, M), partial_bytes(K, rp, M)));
  } else if (op == QL_OP_DQ) {
    sz[0] = 256;
  }
  int64_t o = 0;
  for (int i = 0; i < 6; ++i) {
    L.off[i] = o;
    o += round_up(sz[i], 256);
  }
  L.total = o;
  return L;
}

static GemmArgs base_args() {
  GemmArgs a{};
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) a.q[i] = t.q[i];
  a.timeout_ns = g_wait_timeout_ns.load();
  a.flag = device_flag_ptr();
  return a;
}

// Tensor maps of the quantised weight for the decode GEMM (tiles of 128 weight rows).
// Forward: codes box {bytes per block, 128 rows}, scales from the block-major copy, box
// {128, 1}. dX: codes box {2 blocks of bytes, 64 rows}, scales row-major, box {4, 64}
// (the kernel starts it at a multiple of 4 blocks to keep TMA coordinates aligned).
static bool make_weight_maps(const ql_weight* w, const float* scales, bool transposed,
                                  CUtensorMap* mc, CUtensorMap* ms) {
  const int64_t N = w->N, K = w->K, KB = K / 64;
  const bool nf4 = w->fmt == QL_FMT_NF4_DQ;
  const uint64_t row_bytes = nf4 ? K / 2 : K;
  const uint32_t blk_bytes = nf4 ? 32 : 64;
  if (!transposed) {
    return make_map_t(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, row_bytes, N, row_bytes, blk_bytes,
                      128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           make_map_t(ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scales, N, KB, N * 4, 128, 1,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  const int64_t ld = round_up(KB, 4);
  return make_map_t(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, row_bytes, N, row_bytes, 2 * blk_bytes,
                    64, CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map_t(ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, scales, KB, N, ld * 4, 4, 64,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
}

static ql_status launch_block_scales(const ql_weight* w, bool transposed, float* out, cudaStream_t st) {
  const int64_t N = w->N, KB = w->K / 64;
  const int64_t ld = transposed ? round_up(KB, 4) : 0;
  block_scale_kernel<<<small_grid(N * KB), 256, 0, st>>>(w->fmt, w->qabsmax, w->group_scale, w->mean,
                                                         w->absmax, N, KB, transposed ? 1 : 0, ld, out);
  QL_CHECK_LAUNCH();
  return QL_OK;
}

static ql_status check_weight(const ql_weight* w) {
  if (!w || w->N < 1 || w->K < 64 || !w->codes || !aligned(w->codes, 16)) return QL_ERR_INVALID_ARG;
  if (w->K % 64 != 0 || w->N % 8 != 0) return QL_ERR_UNSUPPORTED;
  if (w->fmt == QL_FMT_NF4_DQ) {
    if (!w->qabsmax || !w->group_scale || !w->mean) return QL_ERR_INVALID_ARG;
  } else if (w->fmt == QL_FMT_INT8_B64) {
    if (!w->absmax || !aligned(w->absmax, 4)) return QL_ERR_INVALID_ARG;
  } else {
    return QL_ERR_INVALID_ARG;
  }
  return QL_OK;
}

// Y = X deq(W)^T + Zext Wext^T, with Zext [M, kext] and Wext [N, kext] bf16 row-major
// (kext a multiple of 64, 0 for the base product alone): the fused GEMM of the forward,
// its extension chunks taken from the caller's operands. M <= 16 with kext = 0 runs the
// decode-shaped kernel without its adapter part, adding a Walsh-Hadamard adapter's sparse
// sums when qw is given. The only scratch is the block-scale copy.
int64_t ext_fwd_ws_bytes(int64_t M, int64_t N, int64_t K, int64_t kext) {
  if (kext == 0 && M <= kSmallMMax && small_m_supported(K, 0)) return 0;
  return round_up((K / 64) * N * 4, 256);
}

ql_status ext_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* Zext,
                      const uint16_t* Wext, int64_t kext, uint16_t* Y, void* ws, size_t ws_bytes,
                      cudaStream_t st, const QwhaRows* qw) {
  ql_status e = check_weight(w);
  if (e != QL_OK) return e;
  if (!X || !Y || M < 1 || !aligned(X, 16) || !aligned(Y, 16)) return QL_ERR_INVALID_ARG;
  if (kext < 0 || kext % 64 != 0 || (kext > 0 && (!Zext || !Wext || !aligned(Zext, 16) || !aligned(Wext, 16))))
    return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  const int64_t N = w->N, K = w->K;
  if (kext == 0 && M <= kSmallMMax && small_m_supported(K, 0))
    return small_m_forward(w, X, M, nullptr, nullptr, 0, 0.0f, Y, nullptr, st, qw);
  if (qw) return QL_ERR_UNSUPPORTED;                // the sparse sums exist on the decode-shaped path only
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes < ext_fwd_ws_bytes(M, N, K, kext)) return QL_ERR_WORKSPACE;
  float* scales = static_cast<float*>(ws);
  const bool pair = g_gemm_pair.load() != 0;
  const uint32_t tbox = pair ? 128 : 256;
  CUtensorMap mXt, mc, ms, mZt, mWe;
  if (!make_map(&mXt, X, K, M, K, tbox) || !make_weight_maps(w, scales, false, &mc, &ms)) return QL_ERR_CUDA;
  if (kext > 0) {
    if (!make_map(&mZt, Zext, kext, M, kext, tbox) || !make_map(&mWe, Wext, kext, N, kext, 128)) return QL_ERR_CUDA;
  } else {
    mZt = mXt;                                      // never read with no extension chunks
    mWe = mXt;
  }
  {
    ProfScope prof(PK_FWD_PREP, st, 1);
    e = launch_block_scales(w, false, scales, st);
    if (e != QL_OK) return e;
  }
  GemmArgs y = base_args();
  y.R = N; y.Cn = M; y.Kc = K; y.n_ext = (int32_t)(kext / 64); y.r = 0;
  y.out = Y; y.ld_out = N; y.scale = 1.0f;
  ProfScope prof(PK_FWD_MAIN, st, 1);
  if (pair) {
    if (w->fmt == QL_FMT_NF4_DQ) return launch_wpair<BSrc::NF4, false>(mXt, mc, ms, mZt, mWe, y, st);
    return launch_wpair<BSrc::INT8, false>(mXt, mc, ms, mZt, mWe, y, st);
  }
  if (w->fmt == QL_FMT_NF4_DQ) return launch_wdec<BSrc::NF4, false>(mXt, mc, ms, mZt, mWe, y, st);
  return launch_wdec<BSrc::INT8, false>(mXt, mc, ms, mZt, mWe, y, st);
}

// Y = X bf16(deq(W) + dW)^T with a dense bf16 update dW [N, K] (row-major, 16-byte
// aligned) added to the decoded weight inside the fused GEMM (M > 16 only; the scratch is
// the block-scale copy of ext_fwd_ws_bytes(M, N, K, 0)).
ql_status dw_forward(const ql_weight* w, const uint16_t* X, int64_t M, const uint16_t* dW, uint16_t* Y, void* ws,
                     size_t ws_bytes, cudaStream_t st) {
  ql_status e = check_weight(w);
  if (e != QL_OK) return e;
  if (!X || !Y || !dW || M < 1 || !aligned(X, 16) || !aligned(Y, 16) || !aligned(dW, 16)) return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  const int64_t N = w->N, K = w->K;
  if (!ws || !aligned(ws, 256)) return QL_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes < ext_fwd_ws_bytes(M, N, K, 0)) return QL_ERR_WORKSPACE;
  float* scales = static_cast<float*>(ws);
  const bool pair = g_gemm_pair.load() != 0;
  CUtensorMap mXt, mc, ms, mdw;
  if (!make_map(&mXt, X, K, M, K, pair ? 128 : 256) || !make_weight_maps(w, scales, false, &mc, &ms) ||
      !make_map(&mdw, dW, K, N, K, 128))
    return QL_ERR_CUDA;
  {
    ProfScope prof(PK_FWD_PREP, st, 1);
    e = launch_block_scales(w, false, scales, st);
    if (e != QL_OK) return e;
  }
  GemmArgs y = base_args();
  y.R = N; y.Cn = M; y.Kc = K; y.n_ext = 0; y.r = 0;
  y.out = Y; y.ld_out = N; y.scale = 1.0f;
  ProfScope prof(PK_FWD_MAIN, st, 1);
  if (pair) {
    if (w->fmt == QL_FMT_NF4_DQ) return launch_wpair<BSrc::NF4, false, true>(mXt, mc, ms, mXt, mXt, y, st, &mdw);
    return launch_wpair<BSrc::INT8, false, true>(mXt, mc, ms, mXt, mXt, y, st, &mdw);
  }
  if (w->fmt == QL_FMT_NF4_DQ) return launch_wdec<BSrc::NF4, false, true>(mXt, mc, ms, mXt, mXt, y, st, &mdw);
  return launch_wdec<BSrc::INT8, false, true>(mXt, mc, ms, mXt, mXt, y, st, &mdw);
}

}  // namespace qlb

using namespace qlb;

extern "C" {

size_t ql_workspace_bytes(int32_t op, int64_t M, int64_t N, int64_t K, int32_t r) {
  if (op == QL_OP_DQ) return 256;
  if (op == QL_OP_DQ_BATCH) {                         // 16 exact-sum bins per weight of a launch
    if (M < 0) return 0;
    return (size_t)imax64(256, imin64(M, 128) * 16 * 8);
  }
  if (op == QL_OP_FWD_QWHA) {
    if (M < 1 || N < 1 || K < 64 || K % 64 != 0) return 0;
    return (size_t)qwha_ws_bytes(M, N, K);
  }
  if (op == QL_OP_FWD_LORDBA) {
    if (M < 0 || N < 0 || K < 0 || r < 1 || r > 256) return 0;
    return (size_t)lordba_ws_bytes(M, N, K, r);
  }
  if ((op != QL_OP_FWD && op != QL_OP_BWD) || M < 0 || N < 0 || K < 0 || r < 1 || r > 256) return 0;
  if (op == QL_OP_FWD && M <= kSmallMMax && small_m_supported(K, r)) return 0;   // decode-shaped path
  return (size_t)ws_layout(op, M, N, K, r).total;
}

void ql_set_wait_timeout_ns(uint64_t ns) {
  g_wait_timeout_ns.store(ns ? ns : 2000000000ull);
}

ql_status qlora_linear_fwd(const ql_weight* w, const ql_bf16* X, int64_t M, const ql_bf16* A,
                           const ql_bf16* B, int32_t r, float alpha, ql_bf16* Y, ql_bf16* T_save,
                           void* ws, size_t ws_bytes, void* stream) {
  ql_status st0 = check_weight(w);
  if (st0 != QL_OK) return st0;
  if (!X || !A || !B || !Y || M < 1 || r < 1) return QL_ERR_INVALID_ARG;
  if (r > 256 || M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!aligned(X, 16) || !aligned(A, 16) || !aligned(B, 2) || !aligned(Y, 16) ||
      (T_save && !aligned(T_save, 2)))
    return QL_ERR_INVALID_ARG;
  if (!(M <= kSmallMMax && small_m_supported(w->K, r)) && (!ws || !aligned(ws, 256))) return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  cudaStream_t st = as_stream(stream);
  if (M <= kSmallMMax && small_m_supported(w->K, r)) return small_m_forward(w, X, M, A, B, r, alpha, Y, T_save, st);
  const WsLayout L = ws_layout(QL_OP_FWD, M, N, K, r);
  if ((int64_t)ws_bytes < L.total) return QL_ERR_WORKSPACE;
  const int rp = (int)round_up(r, 64);
  const float s = alpha / (float)r;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* P = reinterpret_cast<uint16_t*>(wsb + L.off[0]);
  uint16_t* Bp = reinterpret_cast<uint16_t*>(wsb + L.off[1]);
  float* scales = reinterpret_cast<float*>(wsb + L.off[4]);

  // token boxes: 128 rows per CTA for the pair GEMM, 256 for the single-CTA one
  const bool pair = g_gemm_pair.load() != 0;
  const uint32_t tbox = pair ? 128 : 256;
  CUtensorMap mX, mXt, mA, mPt, mBp, mc, ms;
  if (!make_map(&mX, X, K, M, K, 128) || !make_map(&mXt, X, K, M, K, tbox) ||
      !make_map(&mA, A, K, r, K, rp) || !make_map(&mPt, P, rp, M, rp, tbox) ||
      !make_map(&mBp, Bp, rp, N, rp, 128) || !make_weight_maps(w, scales, false, &mc, &ms))
    return QL_ERR_CUDA;

  {
    ProfScope prof(PK_FWD_PREP, st, 2);
    pad_cols_kernel<<<small_grid(N * rp), 256, 0, st>>>(B, N, r, rp, Bp);
    QL_CHECK_LAUNCH();
    ql_status e = launch_block_scales(w, false, scales, st);
    if (e != QL_OK) return e;
  }

  // [T | P] = X A^T
  GemmArgs t = base_args();
  t.R = M; t.Cn = rp; t.Kc = K; t.n_ext = 0; t.r = r;
  t.out = T_save; t.ld_out = r; t.out2 = P; t.ld_out2 = rp; t.scale = s;
  ql_status e;
  {
    ProfScope prof(PK_FWD_T, st, 1);
    e = launch_tma_rp<EPI_LORA_T, false, false>(rp, mX, mA, t, st);
  }
  if (e != QL_OK) return e;

  // Y^T = W' X^T + Bp P^T  (weight rows as the MMA's M, tokens as its N)
  GemmArgs y = base_args();
  y.R = N; y.Cn = M; y.Kc = K; y.n_ext = rp / 64; y.r = r;
  y.out = Y; y.ld_out = N; y.scale = 1.0f;
  ProfScope prof(PK_FWD_MAIN, st, 1);
  if (pair) {
    if (w->fmt == QL_FMT_NF4_DQ) return launch_wpair<BSrc::NF4, false>(mXt, mc, ms, mPt, mBp, y, st);
    return launch_wpair<BSrc::INT8, false>(mXt, mc, ms, mPt, mBp, y, st);
  }
  if (w->fmt == QL_FMT_NF4_DQ) return launch_wdec<BSrc::NF4, false>(mXt, mc, ms, mPt, mBp, y, st);
  return launch_wdec<BSrc::INT8, false>(mXt, mc, ms, mPt, mBp, y, st);
}

void ql_set_gemm_pair(int on) { g_gemm_pair.store(on ? 1 : 0); }

ql_status qlora_linear_bwd(const ql_weight* w, const ql_bf16* X, const ql_bf16* dY, int64_t M,
                           const ql_bf16* A, const ql_bf16* B, const ql_bf16* T_saved, int32_t r,
                           float alpha, ql_bf16* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                           void* stream) {
  ql_status st0 = check_weight(w);
  if (st0 != QL_OK) return st0;
  if (!X || !dY || !A || !B || !T_saved || !dX || !dA || !dB || !ws || M < 1 || r < 1)
    return QL_ERR_INVALID_ARG;
  if (r > 256 || M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!aligned(X, 16) || !aligned(dY, 16) || !aligned(A, 2) || !aligned(B, 2) || !aligned(T_saved, 2) ||
      !aligned(dX, 16) || !aligned(dA, 4) || !aligned(dB, 4) || !aligned(ws, 256))
    return QL_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  const WsLayout L = ws_layout(QL_OP_BWD, M, N, K, r);
  if ((int64_t)ws_bytes < L.total) return QL_ERR_WORKSPACE;
  const int rp = (int)round_up(r, 64);
  const float s = alpha / (float)r;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* Q = reinterpret_cast<uint16_t*>(wsb + L.off[0]);
  uint16_t* Bt = reinterpret_cast<uint16_t*>(wsb + L.off[1]);
  uint16_t* At = reinterpret_cast<uint16_t*>(wsb + L.off[2]);
  uint16_t* Tp = reinterpret_cast<uint16_t*>(wsb + L.off[3]);
  float* scales = reinterpret_cast<float*>(wsb + L.off[4]);
  float* part = reinterpret_cast<float*>(wsb + L.off[5]);

  const bool pair = g_gemm_pair.load() != 0;
  const uint32_t tbox = pair ? 128 : 256;
  CUtensorMap mdY_k, mdYt, mBt, mQt, mAt, mdY_mn, mTp_mn, mX_mn, mQ_mn, mc, ms;
  if (!make_map(&mdY_k, dY, N, M, N, 128) || !make_map(&mdYt, dY, N, M, N, tbox) ||
      !make_map(&mBt, Bt, N, r, N, rp) ||
      !make_map(&mQt, Q, rp, M, rp, tbox) || !make_map(&mAt, At, rp, K, rp, 128) ||
      !make_map(&mdY_mn, dY, N, M, N, 64) || !make_map(&mTp_mn, Tp, rp, M, rp, 64) ||
      !make_map(&mX_mn, X, K, M, K, 64) || !make_map(&mQ_mn, Q, rp, M, rp, 64) ||
      !make_weight_maps(w, scales, true, &mc, &ms))
    return QL_ERR_CUDA;

  {
    ProfScope prof(PK_BWD_PREP, st, 4);
    transpose_kernel<<<small_grid(N * r), 256, 0, st>>>(B, N, r, Bt);
    QL_CHECK_LAUNCH();
    transpose_pad_kernel<<<small_grid(K * rp), 256, 0, st>>>(A, r, K, rp, At);
    QL_CHECK_LAUNCH();
    pad_cols_kernel<<<small_grid(M * rp), 256, 0, st>>>(T_saved, M, r, rp, Tp);
    QL_CHECK_LAUNCH();
    ql_status e = launch_block_scales(w, true, scales, st);
    if (e != QL_OK) return e;
  }
  ql_status e;

  // Q = bf16(s dY B)
  GemmArgs u = base_args();
  u.R = M; u.Cn = rp; u.Kc = N; u.r = r; u.out = Q; u.ld_out = rp; u.scale = s;
  {
    ProfScope prof(PK_BWD_U, st, apply_split(u, part, rp));
    e = launch_tma_rp<EPI_LORA_Q, false, false>(rp, mdY_k, mBt, u, st);
  }
  if (e != QL_OK) return e;

  // dB = s dY^T T     (rows n, columns j, contraction over tokens)
  GemmArgs b = base_args();
  b.R = N; b.Cn = rp; b.Kc = M; b.r = r; b.out = dB; b.ld_out = r; b.scale = s;
  {
    ProfScope prof(PK_BWD_DB, st, apply_split(b, part, rp));
    e = launch_tma_rp<EPI_DB, true, true>(rp, mdY_mn, mTp_mn, b, st);
  }
  if (e != QL_OK) return e;

  // dA = Q^T X        (computed as dA^T: rows k, columns j)
  GemmArgs a = base_args();
  a.R = K; a.Cn = rp; a.Kc = M; a.r = r; a.out = dA; a.ld_out = K; a.scale = 1.0f;
  {
    ProfScope prof(PK_BWD_DA, st, apply_split(a, part, rp));
    e = launch_tma_rp<EPI_DA, true, true>(rp, mX_mn, mQ_mn, a, st);
  }
  if (e != QL_OK) return e;

  // dX^T = W'^T dY^T + A^T-padded Q^T  (input features as the MMA's M, tokens as its N)
  GemmArgs x = base_args();
  x.R = K; x.Cn = M; x.Kc = N; x.n_ext = rp / 64; x.r = r; x.out = dX; x.ld_out = K; x.scale = 1.0f;
  ProfScope prof(PK_BWD_DX, st, 1);
  if (pair) {
    if (w->fmt == QL_FMT_NF4_DQ) return launch_wpair<BSrc::NF4, true>(mdYt, mc, ms, mQt, mAt, x, st);
    return launch_wpair<BSrc::INT8, true>(mdYt, mc, ms, mQt, mAt, x, st);
  }
  if (w->fmt == QL_FMT_NF4_DQ) return launch_wdec<BSrc::NF4, true>(mdYt, mc, ms, mQt, mAt, x, st);
  return launch_wdec<BSrc::INT8, true>(mdYt, mc, ms, mQt, mAt, x, st);
}

}  // extern "C"

// ---- forward without a caller-supplied workspace -------------------------------------
//
// Some callers cannot allocate device memory at the point where they run the layer:
// plugins hosted by a framework that owns every device allocation (a private cudaMalloc
// escapes its pool and its memory accounting), and latency-bound loops that must not touch
// the allocator after start-up (cudaMalloc and cudaFree may synchronise the whole device).
// For them the forward can use a fixed scratch array
// that lives in this library's own device image. It is sized for the fine-tune-shaped
// layers this library targets (the 8192 x 11008 x 4096, r = 64 forward needs 5.2 MiB);
// larger shapes are refused with QL_ERR_WORKSPACE.
namespace qlb {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device, looked up once per device and
// kept for the life of the process (so the library must not be used across a
// cudaDeviceReset, which may load the module at a new address).
static void* static_scratch_ptr() {
  static std::mutex mu;
  static void* ptrs[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace qlb

extern "C" ql_status qlora_linear_fwd_static(const ql_weight* w, const ql_bf16* X, int64_t M,
                                             const ql_bf16* A, const ql_bf16* B, int32_t r, float alpha,
                                             ql_bf16* Y, ql_bf16* T_save, void* stream) {
  // the same refusals, in the same order, as qlora_linear_fwd, so the two entry points
  // return the same status for the same arguments; only then the scratch-size limit
  ql_status st0 = check_weight(w);
  if (st0 != QL_OK) return st0;
  if (!X || !A || !B || !Y || M < 1 || r < 1) return QL_ERR_INVALID_ARG;
  if (r > 256 || M > (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED;
  if (!aligned(X, 16) || !aligned(A, 16) || !aligned(B, 2) || !aligned(Y, 16) ||
      (T_save && !aligned(T_save, 2)))
    return QL_ERR_INVALID_ARG;
  const size_t need = ql_workspace_bytes(QL_OP_FWD, M, w->N, w->K, r);
  if (need > kStaticScratchBytes) return QL_ERR_WORKSPACE;
  void* ws = static_scratch_ptr();
  if (!ws) return QL_ERR_CUDA;
  return qlora_linear_fwd(w, X, M, A, B, r, alpha, Y, T_save, ws, kStaticScratchBytes, stream);
}
