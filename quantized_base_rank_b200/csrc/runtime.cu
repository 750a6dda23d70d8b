// Host-side runtime pieces: the NF4 tables, the sticky device flag, status strings.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace qlb {

// Standard normal CDF through the complementary error function.
static double norm_cdf(double z) { return 0.5 * erfc(-z / 1.4142135623730950488); }

// Q_N(p): the standard normal quantile, by bisection on the CDF until the bracket is
// two adjacent doubles (erfc is accurate to about one ulp, which puts the quantile
// within a few ulps of the true value for the probabilities used here).
static double norm_quantile(double p) {
  double lo = -12.0, hi = 12.0;
  for (int it = 0; it < 400; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (norm_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

// The NF4 grid of the QLoRA page ("1. 4-bit NormalFloat (NF4)"): quantiles of N(0,1)
// at the centres (i + 1/2)/16 of 16 equal-probability bins, normalised so the largest
// magnitude is 1, each rounded once to fp32.
static Nf4Tables build_tables() {
  Nf4Tables t;
  const double zmax = norm_quantile(31.0 / 32.0);
  for (int i = 0; i < 16; ++i) t.q[i] = (float)(norm_quantile((i + 0.5) / 16.0) / zmax);
  // exact midpoints of adjacent fp32 points (sum and halving are exact in fp64)
  for (int k = 0; k < 7; ++k) t.mid_pos[k] = ((double)t.q[8 + k] + (double)t.q[9 + k]) * 0.5;
  return t;
}

const Nf4Tables& nf4_tables() {
  static const Nf4Tables t = build_tables();
  return t;
}

// Smallest bf16 value >= d, for a positive double d whose bf16 rounding is normal: round
// the fp64 bit pattern up at the 8th significant bit (a carry moves into the exponent
// on its own), then move the exponent from the fp64 bias to the bf16 bias.
static uint32_t ceil_bf16_bits(double d) {
  uint64_t bits;
  memcpy(&bits, &d, sizeof bits);
  const uint64_t r = (bits + ((uint64_t(1) << 45) - 1)) >> 45;   // sign | exp11 | top 7 bits
  return (uint32_t)(r - (uint64_t(1023 - 127) << 7));
}

static Nf4BoundTable build_bound_table() {
  const Nf4Tables& t = nf4_tables();
  Nf4BoundTable b;
  for (int f = 0; f < 128; ++f) {
    const double a = 1.0 + f / 128.0;
    for (int k = 0; k < 7; ++k) {
      const uint32_t c = ceil_bf16_bits(a * t.mid_pos[k]);          // exact product
      b.c[f][k] = c | (c << 16);
    }
    b.c[f][7] = 0u;
  }
  return b;
}

const Nf4BoundTable& nf4_bound_table() {
  static const Nf4BoundTable b = build_bound_table();
  return b;
}

__device__ int g_ql_flag;

int* device_flag_ptr() {
  static std::mutex mu;
  static int* ptrs[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ql_flag) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

int num_sms() {
  static std::mutex mu;
  static int cache[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

// ---- profiling events and launch counting -------------------------------------------

static std::atomic<int> g_prof_on{0};
static std::atomic<uint64_t> g_launches{0};
static std::mutex g_prof_mu;
static std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof[PK_COUNT];
static std::vector<cudaEvent_t> g_ev_pool;

static cudaEvent_t take_event() {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

ProfScope::ProfScope(int kind, cudaStream_t st, int nlaunch)
    : kind_(kind), st_(st), on_(g_prof_on.load() != 0), a_(nullptr) {
  g_launches += (uint64_t)nlaunch;
  if (on_) {
    a_ = take_event();
    cudaEventRecord(a_, st_);
  }
}

ProfScope::~ProfScope() {
  if (!on_) return;
  cudaEvent_t b = take_event();
  cudaEventRecord(b, st_);
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof[kind_].push_back({a_, b});
}

}  // namespace qlb

extern "C" {

void ql_profile_enable(int on) { qlb::g_prof_on.store(on ? 1 : 0); }

uint64_t ql_launch_count(void) { return qlb::g_launches.load(); }

int ql_profile_read(int kind, double* total_ms, int64_t* count) {
  if (kind < 0 || kind >= qlb::PK_COUNT) return -1;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> v;
  {
    std::lock_guard<std::mutex> lock(qlb::g_prof_mu);
    v.swap(qlb::g_prof[kind]);
  }
  double tot = 0.0;
  for (auto& p : v) {
    float ms = 0.0f;
    if (cudaEventSynchronize(p.second) == cudaSuccess && cudaEventElapsedTime(&ms, p.first, p.second) == cudaSuccess)
      tot += ms;
  }
  {
    std::lock_guard<std::mutex> lock(qlb::g_prof_mu);
    for (auto& p : v) {
      qlb::g_ev_pool.push_back(p.first);
      qlb::g_ev_pool.push_back(p.second);
    }
  }
  if (total_ms) *total_ms = tot;
  if (count) *count = (int64_t)v.size();
  return 0;
}

ql_status ql_get_device_status(void* stream) {
  if (cudaStreamSynchronize(qlb::as_stream(stream)) != cudaSuccess) return QL_ERR_CUDA;
  int* p = qlb::device_flag_ptr();
  if (!p) return QL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QL_ERR_CUDA;
  if (v) {
    int z = 0;
    if (cudaMemcpy(p, &z, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return QL_ERR_CUDA;
  }
  if (v & qlb::kFlagTimeout) return QL_ERR_TIMEOUT;
  if (v & qlb::kFlagNonfinite) return QL_ERR_NONFINITE;
  if (v & qlb::kFlagBadIndex) return QL_ERR_INVALID_ARG;
  return QL_OK;
}

const char* ql_status_string(ql_status s) {
  switch (s) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument";
    case QL_ERR_UNSUPPORTED: return "unsupported shape or format";
    case QL_ERR_WORKSPACE: return "workspace too small";
    case QL_ERR_NONFINITE: return "non-finite input";
    case QL_ERR_TIMEOUT: return "bounded device wait timed out";
    case QL_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

void ql_nf4_codebook(float* out16) {
  if (!out16) return;
  const qlb::Nf4Tables& t = qlb::nf4_tables();
  for (int i = 0; i < 16; ++i) out16[i] = t.q[i];
}

}  // extern "C"
