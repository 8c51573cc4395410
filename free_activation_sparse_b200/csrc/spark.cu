// The Spark FFN as a key-value lookup ("Spark Transformer", section 2.1: y = sum_i
// f(q . k_i) v_i; the query's dot product with every key, the statistical top-k of
// section 2.2 on those scores, only the selected neurons activated), for a SwiGLU FFN,
// one token:
//   g = W_gate x                          dense GEMV over the output-major W_gate
//   S = { i : g_i > mu + sigma z }        statistical threshold on the signed scores
//   h_i = silu(g_i) * (W_up[i] . x)       only the selected rows of the output-major W_up
//   y = sum over i in S of h_i Wt_down[i] the sparse product over the input-major W_down
#include <math.h>

#include "internal.h"

namespace wina {

constexpr int kKT = 256;  // threads per CTA of the row-gather kernel

// h[r] = silu(g[idx[r]]) * (W_up[idx[r]] . x) for r < count (capped at cap): one warp per
// selected row, 16-byte streaming loads.
template <bool BF16>
__global__ void __launch_bounds__(kKT) k_spark_up(const void* __restrict__ Wu, int d, const float* __restrict__ x,
                                                   const float* __restrict__ g, const int32_t* __restrict__ idx,
                                                   const int32_t* __restrict__ count, int cap, float* __restrict__ h) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const uint64_t pol = l2_evict_first_policy();
  const int lane = threadIdx.x & 31;
  const int nsel = min(__ldg(count), cap);
  const int warps = gridDim.x * (kKT / 32);
  const size_t rb = (size_t)d * (BF16 ? 2 : 4);
  for (int r = blockIdx.x * (kKT / 32) + (threadIdx.x >> 5); r < nsel; r += warps) {
    const int i = __ldg(idx + r);
    const uint4* rp = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(Wu) + (size_t)i * rb);
    float acc = 0.f;
    for (int v = lane; v < d / EPV; v += 32) {
      float w[EPV];
#pragma unroll
      for (int e = 0; e < EPV; ++e) w[e] = 0.f;
      VecOps<BF16>::fma(w, ld_stream_u4(rp + v, pol), 1.0f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc = fmaf(w[e], __ldg(x + v * EPV + e), acc);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float gi = __ldg(g + i);
      h[r] = gi / (1.0f + expf(-gi)) * acc;
    }
  }
}

struct SparkWs {
  size_t xf, g, h, spmv, total;
};

static SparkWs spark_ws_layout(int64_t d, int64_t ffn) {
  SparkWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = round_up(o + bytes, kAlign);
    return at;
  };
  w.xf = take((size_t)d * 4);
  w.g = take((size_t)ffn * 4);
  w.h = take((size_t)ffn * 4);
  w.spmv = take(spmv_total_ws(ffn, d, 1));
  w.total = o;
  return w;
}

size_t spark_ws_size(int64_t d, int64_t ffn) { return spark_ws_layout(d, ffn).total; }

wina_status_t launch_dense_gemv(const void* W, int wdt, int m, int n, const void* x, int xdt, float* y, float* xbuf,
                                cudaStream_t s);
wina_status_t launch_widen(const void* x, int xdt, int n, float* xf, cudaStream_t s);

}  // namespace wina

using namespace wina;

extern "C" wina_status_t spark_ffn_swiglu(const void* W_gate, const void* W_up, const void* Wt_down,
                                          wina_dtype_t wdt, int64_t d, int64_t ffn, const void* x, wina_dtype_t xdt,
                                          double s, float* y, float* g_out, int32_t* idx, int32_t* count, void* ws,
                                          size_t ws_bytes, int32_t* status_dev, wina_stream_t stream) {
  if (!valid_dtype(wdt) || !valid_dtype(xdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (d < epv || ffn < 1 || d % epv || ffn > kMaxN || d > kMaxN) return WINA_ERR_INVALID_ARG;
  if (d / epv > (int64_t)kNT * 8) return WINA_ERR_INVALID_ARG;
  if (!(s > 0.0 && s < 1.0)) return WINA_ERR_INVALID_ARG;
  if (!W_gate || !W_up || !Wt_down || !x || !y || !idx || !count || !ws) return WINA_ERR_INVALID_ARG;
  if (!aligned(W_gate, 16) || !aligned(W_up, 16) || !aligned(Wt_down, 16) || !aligned(y, 16) || !aligned(ws, 16) ||
      !aligned(x, elem_size(xdt)) || !aligned(idx, 4) || !aligned(count, 4) || (g_out && !aligned(g_out, 4)) ||
      (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  if (ws_bytes < spark_ws_size(d, ffn)) return WINA_ERR_WORKSPACE;
  const SparkWs L = spark_ws_layout(d, ffn);
  char* w = (char*)ws;
  float* xf = reinterpret_cast<float*>(w + L.xf);
  float* g = g_out ? g_out : reinterpret_cast<float*>(w + L.g);
  float* h = reinterpret_cast<float*>(w + L.h);
  cudaStream_t st = (cudaStream_t)stream;
  wina_status_t r;
  if ((r = launch_widen(x, xdt, (int)d, xf, st))) return r;  // for the up rows
  if ((r = launch_dense_gemv(W_gate, wdt, (int)ffn, (int)d, x, xdt, g, xf, st))) return r;
  const double z = wina_normal_quantile(1.0 - s);
  if ((r = launch_stat_threshold(g, WINA_F32, (int)ffn, z, 1, idx, nullptr, count, nullptr, (int)ffn, status_dev, st)))
    return r;
  const int grid = device_sm_count() * 4;
  if (wdt == WINA_BF16)
    k_spark_up<true><<<grid, kKT, 0, st>>>(W_up, (int)d, xf, g, idx, count, (int)ffn, h);
  else
    k_spark_up<false><<<grid, kKT, 0, st>>>(W_up, (int)d, xf, g, idx, count, (int)ffn, h);
  if ((r = cuda_status(cudaGetLastError()))) return r;
  return launch_sparse_matvec(Wt_down, wdt, ffn, d, idx, h, -1, count, (int)ffn, 1, y, w + L.spmv, status_dev, st);
}
