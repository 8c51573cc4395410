// The dense comparator: the unsparsified layer y = W x and the unsparsified SwiGLU FFN,
// on the output-major weights W[m][n] (each output is one contiguous row, so no sum across
// CTAs is needed). One warp per output row: the lanes stream the row with 16-byte
// read-only loads (several in flight per lane), multiply by x (read through L1, it is
// small and shared by every row) and reduce with shuffles; the grid covers the SMs
// several times over so that enough rows are in flight to keep HBM busy.
#include <math.h>

#include "internal.h"

namespace wina {

constexpr int kGT = 256;  // threads per CTA (8 warps)
constexpr int kGU = 4;    // 16-byte loads of each row in flight per lane

// R rows' dot products with x (all of n elements), by one warp: kGU 16-byte loads of
// every row in flight per lane, x read through L1; the sums are reduced with shuffles
// and every lane receives them.
template <bool BF16, int R>
__device__ __forceinline__ void warp_rows_dot(const char* const (&rows)[R], const float* __restrict__ x, int n,
                                              uint64_t pol, float (&out)[R]) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int lane = threadIdx.x & 31;
  const int V = n / EPV;
  float acc[R][EPV];
#pragma unroll
  for (int q = 0; q < R; ++q)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[q][e] = 0.f;
  auto step = [&](const uint4 (&w)[R], int v) {
    const float4* xv = reinterpret_cast<const float4*>(x + (int64_t)v * EPV);
    float xe[EPV];
#pragma unroll
    for (int q = 0; q < EPV / 4; ++q) {
      const float4 f = __ldg(xv + q);
      xe[4 * q] = f.x;
      xe[4 * q + 1] = f.y;
      xe[4 * q + 2] = f.z;
      xe[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
      float wv[EPV];
#pragma unroll
      for (int e = 0; e < EPV; ++e) wv[e] = 0.f;
      VecOps<BF16>::fma(wv, w[q], 1.0f);  // widen the weights
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[q][e] = fmaf(wv[e], xe[e], acc[q][e]);
    }
  };
  int v = lane;
  for (; v + 32 * (kGU - 1) < V; v += 32 * kGU) {
    uint4 w[kGU][R];
#pragma unroll
    for (int u = 0; u < kGU; ++u)
#pragma unroll
      for (int q = 0; q < R; ++q) w[u][q] = ld_stream_u4(reinterpret_cast<const uint4*>(rows[q]) + v + 32 * u, pol);
#pragma unroll
    for (int u = 0; u < kGU; ++u) step(w[u], v + 32 * u);
  }
  for (; v < V; v += 32) {
    uint4 w[R];
#pragma unroll
    for (int q = 0; q < R; ++q) w[q] = ld_stream_u4(reinterpret_cast<const uint4*>(rows[q]) + v, pol);
    step(w, v);
  }
#pragma unroll
  for (int q = 0; q < R; ++q) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPV; ++e) s += acc[q][e];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    out[q] = s;
  }
}

// x (of dtype xdt) widened to float32 into xf (n elements).
__global__ void k_widen(const void* __restrict__ x, int xdt, int n, float* __restrict__ xf) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) xf[i] = load_elem(x, xdt, i);
}

// y[i] = W[i][:] . x for i < m, warps over rows.
template <bool BF16>
__global__ void __launch_bounds__(kGT) k_dense_gemv(const void* __restrict__ W, int m, int n,
                                                     const float* __restrict__ x, float* __restrict__ y) {
  const uint64_t pol = l2_evict_first_policy();
  const int warps = gridDim.x * (kGT / 32);
  const size_t rb = (size_t)n * (BF16 ? 2 : 4);
  for (int i = blockIdx.x * (kGT / 32) + (threadIdx.x >> 5); i < m; i += warps) {
    const char* rows[1] = {reinterpret_cast<const char*>(W) + (size_t)i * rb};
    float s[1];
    warp_rows_dot<BF16, 1>(rows, x, n, pol, s);
    if ((threadIdx.x & 31) == 0) y[i] = s[0];
  }
}

// h[i] = silu(Wg[i] . x) * (Wu[i] . x) for i < ffn.
template <bool BF16>
__global__ void __launch_bounds__(kGT) k_dense_gate_up(const void* __restrict__ Wg, const void* __restrict__ Wu,
                                                        int ffn, int d, const float* __restrict__ x,
                                                        float* __restrict__ h) {
  const uint64_t pol = l2_evict_first_policy();
  const int warps = gridDim.x * (kGT / 32);
  const size_t rb = (size_t)d * (BF16 ? 2 : 4);
  for (int i = blockIdx.x * (kGT / 32) + (threadIdx.x >> 5); i < ffn; i += warps) {
    const char* rows[2] = {reinterpret_cast<const char*>(Wg) + (size_t)i * rb,
                           reinterpret_cast<const char*>(Wu) + (size_t)i * rb};
    float gu[2];
    warp_rows_dot<BF16, 2>(rows, x, d, pol, gu);  // the gate and up rows of neuron i together
    if ((threadIdx.x & 31) == 0) h[i] = gu[0] / (1.0f + expf(-gu[0])) * gu[1];
  }
}

static int dense_grid() { return device_sm_count() * 8; }  // 8 CTAs of 8 warps per SM

wina_status_t launch_widen(const void* x, int xdt, int n, float* xf, cudaStream_t s) {
  k_widen<<<32, 256, 0, s>>>(x, xdt, n, xf);
  return cuda_status(cudaGetLastError());
}

wina_status_t launch_dense_gemv(const void* W, int wdt, int m, int n, const float* xf, float* y, cudaStream_t s) {
  if (wdt == WINA_BF16)
    k_dense_gemv<true><<<dense_grid(), kGT, 0, s>>>(W, m, n, xf, y);
  else
    k_dense_gemv<false><<<dense_grid(), kGT, 0, s>>>(W, m, n, xf, y);
  return cuda_status(cudaGetLastError());
}

}  // namespace wina

using namespace wina;

extern "C" wina_status_t wina_dense_matvec(const void* W, wina_dtype_t wdt, int64_t m, int64_t n, const void* x,
                                           wina_dtype_t xdt, float* y, float* xbuf, wina_stream_t stream) {
  if (!valid_dtype(wdt) || !valid_dtype(xdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (m < 1 || n < epv || n % epv || m > INT32_MAX || n > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!W || !x || !y || !xbuf || !aligned(W, 16) || !aligned(xbuf, 16) || !aligned(x, elem_size(xdt)) ||
      !aligned(y, 4))
    return WINA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  k_widen<<<32, 256, 0, s>>>(x, xdt, (int)n, xbuf);
  if (wdt == WINA_BF16)
    k_dense_gemv<true><<<dense_grid(), kGT, 0, s>>>(W, (int)m, (int)n, xbuf, y);
  else
    k_dense_gemv<false><<<dense_grid(), kGT, 0, s>>>(W, (int)m, (int)n, xbuf, y);
  return cuda_status(cudaGetLastError());
}

extern "C" wina_status_t wina_dense_ffn_swiglu(const void* W_gate, const void* W_up, const void* W_down,
                                               wina_dtype_t wdt, int64_t d, int64_t ffn, const void* x,
                                               wina_dtype_t xdt, float* y, float* buf, wina_stream_t stream) {
  if (!valid_dtype(wdt) || !valid_dtype(xdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (d < epv || ffn < epv || d % epv || ffn % epv || d > INT32_MAX || ffn > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!W_gate || !W_up || !W_down || !x || !y || !buf || !aligned(W_gate, 16) || !aligned(W_up, 16) ||
      !aligned(W_down, 16) || !aligned(buf, 16) || !aligned(x, elem_size(xdt)) || !aligned(y, 4))
    return WINA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  float* xf = buf;                                    // [d]
  float* h = buf + ((d + 3) / 4 * 4);                 // [ffn]
  k_widen<<<32, 256, 0, s>>>(x, xdt, (int)d, xf);
  if (wdt == WINA_BF16) {
    k_dense_gate_up<true><<<dense_grid(), kGT, 0, s>>>(W_gate, W_up, (int)ffn, (int)d, xf, h);
    k_dense_gemv<true><<<dense_grid(), kGT, 0, s>>>(W_down, (int)d, (int)ffn, h, y);
  } else {
    k_dense_gate_up<false><<<dense_grid(), kGT, 0, s>>>(W_gate, W_up, (int)ffn, (int)d, xf, h);
    k_dense_gemv<false><<<dense_grid(), kGT, 0, s>>>(W_down, (int)d, (int)ffn, h, y);
  }
  return cuda_status(cudaGetLastError());
}
