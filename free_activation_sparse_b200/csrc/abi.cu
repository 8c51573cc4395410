// Host-only entry points of the C ABI: version, status strings, the normal quantile
// used by the Spark threshold, workspace sizes and workspace views.
#include <math.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace wina {

// Small per-process caches of device facts, so that a launch does not query the
// driver each time (the decode path is launch-latency sensitive).
namespace {
constexpr int kMaxDev = 64;
constexpr int kCacheSlots = 128;
struct OccEntry {
  int dev;
  const void* kern;
  int threads;
  size_t smem;
  int per_sm;
};
struct SmemEntry {
  int dev;
  const void* kern;
  size_t smem;
};
std::mutex g_mu;
int g_sms[kMaxDev] = {0};
OccEntry g_occ[kCacheSlots];
int g_nocc = 0;
SmemEntry g_smem[kCacheSlots];
int g_nsmem = 0;
SmemEntry g_l1[kCacheSlots];
int g_nl1 = 0;
}  // namespace

namespace {
SideStream g_side[kMaxDev];
bool g_side_ok[kMaxDev];
std::mutex g_side_mu;
}  // namespace

bool side_stream(cudaStream_t main, SideStream* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_side_ok[dev]) {
    // not while `main` is being captured into a graph: creating a stream then is left out
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(main, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    SideStream ss;
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&ss.fork_ev, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join_ev, cudaEventDisableTiming) != cudaSuccess)
      return false;
    g_side[dev] = ss;
    g_side_ok[dev] = true;
  }
  *out = g_side[dev];
  return true;
}

std::unique_lock<std::mutex> side_stream_lock() { return std::unique_lock<std::mutex>(g_side_mu); }

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sms[dev] > 0) return g_sms[dev];
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxDev) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_sms[dev] = sms;
  }
  return sms;
}

cudaError_t ensure_smem_limit(const void* kern, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_nsmem; ++i)
      if (g_smem[i].dev == dev && g_smem[i].kern == kern && g_smem[i].smem >= smem) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < g_nsmem; ++i)
    if (g_smem[i].dev == dev && g_smem[i].kern == kern) {
      if (g_smem[i].smem < smem) g_smem[i].smem = smem;
      return cudaSuccess;
    }
  if (g_nsmem < kCacheSlots) g_smem[g_nsmem++] = SmemEntry{dev, kern, smem};
  return cudaSuccess;
}

cudaError_t ensure_carveout(const void* kern, int pct) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_nl1; ++i)
      if (g_l1[i].dev == dev && g_l1[i].kern == kern && g_l1[i].smem == (size_t)pct) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < g_nl1; ++i)
    if (g_l1[i].dev == dev && g_l1[i].kern == kern) {
      g_l1[i].smem = (size_t)pct;
      return cudaSuccess;
    }
  if (g_nl1 < kCacheSlots) g_l1[g_nl1++] = SmemEntry{dev, kern, (size_t)pct};
  return cudaSuccess;
}

cudaError_t ensure_prefer_l1(const void* kern) { return ensure_carveout(kern, (int)cudaSharedmemCarveoutMaxL1); }

int blocks_per_sm(const void* kern, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_nocc; ++i)
      if (g_occ[i].dev == dev && g_occ[i].kern == kern && g_occ[i].threads == threads && g_occ[i].smem == smem)
        return g_occ[i].per_sm;
  }
  if (ensure_smem_limit(kern, smem) != cudaSuccess) return 0;  // static shared memory comes on top
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_nocc < kCacheSlots) g_occ[g_nocc++] = OccEntry{dev, kern, threads, smem, per_sm};
  return per_sm;
}

namespace {
std::atomic<unsigned long long> g_wait_ns{kBarrierTimeoutNs};
}  // namespace

unsigned long long wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

// Phi(z) = P(Z <= z) for a standard normal Z, via the complementary error function.
static double normal_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

}  // namespace wina

using namespace wina;

extern "C" int32_t wina_abi_version(void) { return WINA_ABI_VERSION; }

extern "C" void wina_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns ? (unsigned long long)ns : kBarrierTimeoutNs, std::memory_order_relaxed);
}

extern "C" const char* wina_status_string(wina_status_t s) {
  switch (s) {
    case WINA_OK: return "ok";
    case WINA_ERR_INVALID_ARG: return "invalid argument";
    case WINA_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case WINA_ERR_WORKSPACE: return "workspace too small";
    case WINA_ERR_CAPACITY: return "more kept channels than the output capacity";
    case WINA_ERR_CUDA: return "CUDA runtime error";
    case WINA_ERR_TIMEOUT: return "grid barrier wait timed out";
  }
  return "unknown status";
}

// Standard normal quantile: solve Phi(z) = q on the lower tail (q = min(p, 1 - p), z <= 0,
// where erfc has full relative precision) by bisection on [-40, 0] down to the spacing
// of doubles, then two Newton steps z -= (Phi(z) - q) / phi(z); mirror for p > 1/2.
extern "C" double wina_normal_quantile(double p) {
  if (!(p > 0.0 && p < 1.0)) return NAN;
  if (p == 0.5) return 0.0;
  const double q = p < 0.5 ? p : 1.0 - p;
  double lo = -40.0, hi = 0.0;
  for (int it = 0; it < 200 && hi - lo > 0.0; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (normal_cdf(mid) < q)
      lo = mid;
    else
      hi = mid;
  }
  double z = 0.5 * (lo + hi);
  const double inv_sqrt_2pi = 0.39894228040143267794;
  for (int it = 0; it < 2; ++it) {
    const double pdf = inv_sqrt_2pi * exp(-0.5 * z * z);
    if (pdf <= 0.0) break;
    z -= (normal_cdf(z) - q) / pdf;
  }
  return p < 0.5 ? z : -z;
}

extern "C" size_t wina_workspace_size(wina_op_t op, int64_t n, int64_t m, int64_t k, int64_t batch) {
  (void)k;
  if (n < 1 || m < 1 || batch < 1) return 0;
  switch (op) {
    case WINA_OP_SPARSE_MATVEC: return spmv_total_ws(n, m, batch);
    case WINA_OP_FFN_SWIGLU: return ffn_ws_layout(n, m, batch).total;
    case WINA_OP_SPARK_FFN: return batch == 1 ? spark_ws_size(n, m) : 0;
    case WINA_OP_DENSE_FFN: return batch == 1 ? dense_ws_size(n, m) : 0;
    default: return 0;
  }
}

extern "C" wina_status_t wina_ffn_ws_view(int64_t d, int64_t ffn, int64_t batch, wina_ffn_ws_view_t* out) {
  if (d < 1 || ffn < 1 || batch < 1 || !out) return WINA_ERR_INVALID_ARG;
  const FfnWs L = ffn_ws_layout(d, ffn, batch);
  out->h = L.h;
  out->keep_gate = L.keep_g;
  out->keep_up = L.keep_u;
  out->keep_down = L.keep_d;
  out->stamps = L.stamps;
  out->cta_t = L.cta_t;
  return WINA_OK;
}
