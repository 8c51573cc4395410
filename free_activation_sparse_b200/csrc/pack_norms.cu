// Offline weight preparation (untimed): the input-channel-major layout and the
// column-norm statistic of the WINA gate.
//
//  * wina_pack_in_major: W[m][n] -> Wt[n][m], so that input channel j of W is the
//    contiguous run Wt[j][0..m) ("Spark Transformer", section 3.1: the SVMM loop reads
//    W[j] whole for each active j).
//  * wina_col_norms: c_j = ||W[:, j]||_2 ("WINA" article, section 一), float64
//    accumulation, one rounding to float32 at the end.
#include "internal.h"

namespace wina {

// 32x32 tiles through SMEM; block (32, 8). Bit-exact copy of the elements.
template <typename T>
__global__ void __launch_bounds__(256) k_transpose(const T* __restrict__ W, T* __restrict__ Wt, int64_t m,
                                                   int64_t n) {
  __shared__ T tile[32][33];
  const int64_t c0 = (int64_t)blockIdx.x * 32;  // columns of W (= rows of Wt)
  const int64_t r0 = (int64_t)blockIdx.y * 32;  // rows of W
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int64_t r = r0 + j, c = c0 + threadIdx.x;
    if (r < m && c < n) tile[j][threadIdx.x] = W[r * n + c];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int64_t r = c0 + j, c = r0 + threadIdx.x;  // Wt[r][c] = W[c][r]
    if (r < n && c < m) Wt[r * m + c] = tile[threadIdx.x][j];
  }
}

template <typename T>
__device__ __forceinline__ double as_f64(T v);
template <>
__device__ __forceinline__ double as_f64<uint16_t>(uint16_t v) {
  return (double)bf16_bits_to_f32(v);
}
template <>
__device__ __forceinline__ double as_f64<float>(float v) {
  return (double)v;
}

// Column norms of W[m][n] (output-major): block (32, 16); threadIdx.x picks a column,
// threadIdx.y a residue class of rows; the 16 partial sums are added in fixed order.
template <typename T>
__global__ void __launch_bounds__(512) k_col_norms_out_in(const T* __restrict__ W, int64_t m, int64_t n,
                                                          float* __restrict__ c) {
  __shared__ double part[16][32];
  const int64_t j = (int64_t)blockIdx.x * 32 + threadIdx.x;
  double s = 0.0;
  if (j < n) {
    for (int64_t i = threadIdx.y; i < m; i += 16) {
      const double v = as_f64<T>(W[i * n + j]);
      s = fma(v, v, s);
    }
  }
  part[threadIdx.y][threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.y == 0 && j < n) {
    double t = 0.0;
    for (int q = 0; q < 16; ++q) t += part[q][threadIdx.x];
    c[j] = (float)sqrt(t);
  }
}

// Row norms of the packed Wt[n][m]: one block of 256 threads per input channel j.
template <typename T>
__global__ void __launch_bounds__(256) k_col_norms_in_major(const T* __restrict__ Wt, int64_t m, int64_t n,
                                                            float* __restrict__ c) {
  __shared__ double part[256];
  const int64_t j = blockIdx.x;
  const T* row = Wt + j * m;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < m; i += 256) {
    const double v = as_f64<T>(row[i]);
    s = fma(v, v, s);
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) c[j] = (float)sqrt(part[0]);
}

}  // namespace wina

using namespace wina;

extern "C" wina_status_t wina_pack_in_major(const void* W, wina_dtype_t dt, int64_t m, int64_t n, void* Wt,
                                            wina_stream_t stream) {
  if (!valid_dtype(dt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (m < 1 || n < 1 || !W || !Wt) return WINA_ERR_INVALID_ARG;
  if (!aligned(W, elem_size(dt)) || !aligned(Wt, elem_size(dt))) return WINA_ERR_INVALID_ARG;
  const int64_t bytes = m * n * elem_size(dt);
  const char* a = (const char*)W;
  const char* b = (const char*)Wt;
  if (a < b + bytes && b < a + bytes) return WINA_ERR_INVALID_ARG;  // overlap
  if ((n + 31) / 32 > INT32_MAX || (m + 31) / 32 > 65535) return WINA_ERR_INVALID_ARG;
  dim3 grid((unsigned)((n + 31) / 32), (unsigned)((m + 31) / 32));
  dim3 block(32, 8);
  cudaStream_t s = (cudaStream_t)stream;
  if (dt == WINA_BF16)
    k_transpose<uint16_t><<<grid, block, 0, s>>>((const uint16_t*)W, (uint16_t*)Wt, m, n);
  else
    k_transpose<float><<<grid, block, 0, s>>>((const float*)W, (float*)Wt, m, n);
  return cuda_status(cudaGetLastError());
}

extern "C" wina_status_t wina_col_norms(const void* W, wina_dtype_t dt, int64_t m, int64_t n, wina_layout_t layout,
                                        float* c, wina_stream_t stream) {
  if (!valid_dtype(dt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (m < 1 || n < 1 || !W || !c) return WINA_ERR_INVALID_ARG;
  if (layout != WINA_LAYOUT_OUT_IN && layout != WINA_LAYOUT_IN_MAJOR) return WINA_ERR_INVALID_ARG;
  if (!aligned(W, elem_size(dt)) || !aligned(c, 4)) return WINA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (layout == WINA_LAYOUT_OUT_IN) {
    if ((n + 31) / 32 > INT32_MAX) return WINA_ERR_INVALID_ARG;
    dim3 grid((unsigned)((n + 31) / 32)), block(32, 16);
    if (dt == WINA_BF16)
      k_col_norms_out_in<uint16_t><<<grid, block, 0, s>>>((const uint16_t*)W, m, n, c);
    else
      k_col_norms_out_in<float><<<grid, block, 0, s>>>((const float*)W, m, n, c);
  } else {
    if (n > INT32_MAX) return WINA_ERR_INVALID_ARG;
    if (dt == WINA_BF16)
      k_col_norms_in_major<uint16_t><<<(unsigned)n, 256, 0, s>>>((const uint16_t*)W, m, n, c);
    else
      k_col_norms_in_major<float><<<(unsigned)n, 256, 0, s>>>((const float*)W, m, n, c);
  }
  return cuda_status(cudaGetLastError());
}
