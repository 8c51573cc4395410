// Per-token gates: the WINA top-K gate and the Spark statistical threshold.
//
//  * wina_select_topk ("WINA" article, section 一): score_i = |x_i * c_i| in float32,
//    keep the K largest (ties to the lower index), written as an ascending index list.
//    Vectors of up to 16384 channels: one CTA of 1024 threads per token keeps the scores'
//    bit patterns in registers and finds the kept set by a radix select on them; longer
//    vectors: one CTA per token with the scores in SMEM, a histogram select finds the
//    K-th largest as a threshold, a two-walk warp-ballot compaction emits the kept
//    indices in ascending order.
//  * stat_topk_threshold ("Spark Transformer", section 2.2): mu, sigma^2 (divisor n) in
//    one pass (Welford per thread, Chan's merge across threads, float64), then
//    t = mu + sigma * z with z = Phi^-1(1 - s) from the host, keep {i : v_i > t}.
#include <math.h>

#include "internal.h"
#include "regsel.cuh"

namespace wina {

// The kept set as bytes (optional): keep[j] = 1 or 0 for every channel j < n, and the
// union flags uflag[j] = 1 for the kept channels (several tokens may store the same 1).
template <int NT, typename Pred>
__device__ __forceinline__ void put_keep(int n, Pred kept, uint8_t* __restrict__ keep, uint8_t* __restrict__ uflag) {
  if (!keep && !uflag) return;
  for (int j = threadIdx.x; j < n; j += NT) {
    const bool k = kept(j);
    if (keep) keep[j] = (uint8_t)(k ? 1 : 0);
    if (uflag && k) uflag[j] = 1;
  }
}

template <int NT>
__global__ void __launch_bounds__(NT) k_select_topk(const void* __restrict__ x, int xdt, const float* __restrict__ c,
                                                    int n, int K, int ld, int32_t* __restrict__ idx,
                                                    float* __restrict__ xs, float* __restrict__ scores,
                                                    uint8_t* __restrict__ keep, uint8_t* __restrict__ uflag) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* keys = sm;                 // [n]
  uint32_t* hist = sm + n;             // [kSelBins]
  uint32_t* cand = hist + kSelBins;    // [2 * kSelCand]
  __shared__ uint32_t red[2 * NT / 32 + 8];
  const int64_t b = blockIdx.x;
  const int64_t off = b * (int64_t)n;
  for (int i = threadIdx.x; i < n; i += NT) {
    const float xv = load_elem(x, xdt, off + i);
    const float s = c ? fabsf(xv * __ldg(c + i)) : fabsf(xv);
    keys[i] = __float_as_uint(s);
    if (scores) scores[off + i] = s;
  }
  __syncthreads();
  const Threshold t = select_threshold<NT>(keys, n, K, hist, cand, red);
  const int64_t ob = b * (int64_t)ld;
  compact_pred<NT>(
      n, [&](int i) { return kept_by(t, keys[i], i); },
      [&](uint32_t, uint32_t* lo, uint32_t* hi) {
        *lo = 0;
        *hi = (uint32_t)K;
      },
      red,
      [&](int i, uint32_t pos) {
        idx[ob + pos] = i;
        if (xs) xs[ob + pos] = load_elem(x, xdt, off + i);
      });
  put_keep<NT>(n, [&](int i) { return kept_by(t, keys[i], i); }, keep ? keep + off : nullptr, uflag);
}

// The same gate for vectors of up to 16384 channels: one CTA of 1024 threads per token with
// the keys in registers (radix select on their bits), then the kept channels' flags, a
// block scan of the flag words' counts and each word's kept channels written in order.
template <int KMAX>
__global__ void __launch_bounds__(kDT, 1) k_select_topk_regs(const void* __restrict__ x, int xdt,
                                                             const float* __restrict__ c, int n, int K, int ld,
                                                             int32_t* __restrict__ idx, float* __restrict__ xs,
                                                             float* __restrict__ scores, uint8_t* __restrict__ keep,
                                                             uint8_t* __restrict__ uflag) {
  __shared__ uint32_t hist[kSelBins + 256];
  __shared__ uint32_t flags[kDMaxN / 32];
  __shared__ uint32_t red[kDW + 1];
  const int t = threadIdx.x;
  const int64_t off = (int64_t)blockIdx.x * n;
  const int kpt = (n + kDT - 1) / kDT;
  clear_hist(hist);
  uint32_t key[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    const int j = t + i * kDT;
    key[i] = 0u;
    if (i < kpt && j < n) {
      const float xv = load_elem(x, xdt, off + j);
      const float sv = c ? fabsf(xv * __ldg(c + j)) : fabsf(xv);
      key[i] = __float_as_uint(sv);
      if (scores) scores[off + j] = sv;
    }
  }
  __syncthreads();  // the histogram is zero
  const Threshold th = radix_select_regs(key, kpt, n, K, hist);
  flags_from_keys(key, kpt, n, th, flags);
  __syncthreads();
  const int nw = (n + 31) / 32;  // <= 512 < kDT: one word per thread
  const uint32_t f = t < nw ? flags[t] : 0u;
  uint32_t at = block_excl_scan<kDT>((uint32_t)__popc(f), red, nullptr);
  const int64_t ob = (int64_t)blockIdx.x * ld;
  for (uint32_t bits = f; bits; bits &= bits - 1u) {
    const int j = t * 32 + __ffs(bits) - 1;
    idx[ob + at] = j;
    if (xs) xs[ob + at] = load_elem(x, xdt, off + j);
    ++at;
  }
  put_keep<kDT>(n, [&](int j) { return ((flags[j >> 5] >> (j & 31)) & 1u) != 0u; }, keep ? keep + off : nullptr,
                uflag);
}

template <int NT>
__global__ void __launch_bounds__(NT) k_stat_threshold(const void* __restrict__ v, int vdt, int n, double z,
                                                       int32_t* __restrict__ idx, float* __restrict__ xs,
                                                       int32_t* __restrict__ count, float* __restrict__ tout, int cap,
                                                       int32_t* status, uint8_t* __restrict__ keep,
                                                       uint8_t* __restrict__ uflag) {
  extern __shared__ __align__(16) float vals[];  // [n]
  __shared__ double dred[NT / 32];
  __shared__ uint32_t wsm[2 * NT / 32 + 1];
  const int64_t b = blockIdx.x;
  const int64_t off = b * (int64_t)n;
  // mu = mean, sigma^2 = mean of (v - mu)^2: two passes, float64 sums in a fixed order
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += NT) {
    const float f = load_elem(v, vdt, off + i);
    vals[i] = f;
    s += (double)f;
  }
  const double mu = block_sum_f64<NT>(s, dred) / (double)n;  // contains __syncthreads
  double q = 0.0;
  for (int i = threadIdx.x; i < n; i += NT) {
    const double dl = (double)vals[i] - mu;
    q += dl * dl;
  }
  const double var = block_sum_f64<NT>(q, dred) / (double)n;
  const double t = mu + sqrt(var) * z;
  const int64_t ob = b * (int64_t)cap;
  const uint32_t total = compact_pred<NT>(
      n, [&](int i) { return (double)vals[i] > t; },
      [&](uint32_t, uint32_t* lo, uint32_t* hi) {
        *lo = 0;
        *hi = (uint32_t)cap;
      },
      wsm,
      [&](int i, uint32_t pos) {
        idx[ob + pos] = i;
        if (xs) xs[ob + pos] = vals[i];
      });
  if (threadIdx.x == 0) {
    count[b] = (int32_t)total;
    if (tout) tout[b] = (float)t;
    if ((int64_t)total > cap) record_status(status, WINA_ERR_CAPACITY);
  }
  put_keep<NT>(n, [&](int i) { return (double)vals[i] > t; }, keep ? keep + off : nullptr, uflag);
}

wina_status_t launch_select_topk(const void* x, int xdt, const float* c, int n, int k, int batch, int32_t* idx,
                                 float* xs, int ld, float* scores, cudaStream_t s, uint8_t* keep, uint8_t* uflag) {
  if (n <= kDMaxN) {
    const int kpt = (n + kDT - 1) / kDT;
    void (*kern)(const void*, int, const float*, int, int, int, int32_t*, float*, float*, uint8_t*, uint8_t*) =
        kpt <= 4 ? k_select_topk_regs<4> : kpt <= 8 ? k_select_topk_regs<8> : kpt <= 12 ? k_select_topk_regs<12>
                                                                                     : k_select_topk_regs<16>;
    kern<<<batch, kDT, 0, s>>>(x, xdt, c, n, k, ld, idx, xs, scores, keep, uflag);
    return cuda_status(cudaGetLastError());
  }
  const size_t smem = (size_t)(n + kSelBins + 2 * kSelCand) * 4;
  return cuda_status(launch_kernel(k_select_topk<kNT>, dim3(batch), dim3(kNT), smem, s, false, x, xdt, c, n, k, ld,
                                   idx, xs, scores, keep, uflag));
}

wina_status_t launch_stat_threshold(const void* v, int vdt, int n, double z, int batch, int32_t* idx, float* xs,
                                    int32_t* count, float* t, int cap, int32_t* status_dev, cudaStream_t s,
                                    uint8_t* keep, uint8_t* uflag) {
  const size_t smem = (size_t)n * 4;
  return cuda_status(launch_kernel(k_stat_threshold<kNT>, dim3(batch), dim3(kNT), smem, s, false, v, vdt, n, z, idx,
                                   xs, count, t, cap, status_dev, keep, uflag));
}

}  // namespace wina

using namespace wina;

extern "C" wina_status_t wina_select_topk(const void* x, wina_dtype_t xdt, const float* c, int64_t n, int64_t k,
                                          int64_t batch, int32_t* idx, float* xs, float* scores,
                                          wina_stream_t stream) {
  if (!valid_dtype(xdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (n < 1 || n > kMaxN || k < 0 || k > n || batch < 1 || batch > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!x || (k > 0 && !idx)) return WINA_ERR_INVALID_ARG;
  if (!aligned(x, elem_size(xdt)) || (c && !aligned(c, 4)) || (idx && !aligned(idx, 4)) || (xs && !aligned(xs, 4)) ||
      (scores && !aligned(scores, 4)))
    return WINA_ERR_INVALID_ARG;
  return launch_select_topk(x, xdt, c, (int)n, (int)k, (int)batch, idx, xs, (int)k, scores, (cudaStream_t)stream);
}

extern "C" wina_status_t stat_topk_threshold(const void* v, wina_dtype_t vdt, int64_t n, double s, int64_t batch,
                                             int32_t* idx, float* xs, int32_t* count, float* t, int64_t cap,
                                             int32_t* status_dev, wina_stream_t stream) {
  if (!valid_dtype(vdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (n < 1 || n > kMaxN || batch < 1 || batch > INT32_MAX || cap < 0 || cap > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!(s > 0.0 && s < 1.0)) return WINA_ERR_INVALID_ARG;
  if (!v || !count || (cap > 0 && !idx)) return WINA_ERR_INVALID_ARG;
  if (!aligned(v, elem_size(vdt)) || !aligned(count, 4) || (idx && !aligned(idx, 4)) || (xs && !aligned(xs, 4)) ||
      (t && !aligned(t, 4)) || (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  const double z = wina_normal_quantile(1.0 - s);
  return launch_stat_threshold(v, vdt, (int)n, z, (int)batch, idx, xs, count, t, (int)cap, status_dev,
                               (cudaStream_t)stream);
}
