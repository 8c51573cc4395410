// The sparse product over kept channels ("Spark Transformer", section 3.1, SVMM):
//     y[b][:] = sum over r < k_b of xs[b][r] * Wt[idx[b][r]][:]
// with the input-channel-major weight Wt[n][m], so each kept channel is one
// contiguous run of m elements streamed from HBM with 16-byte cache-hinted loads.
//
// Work split: token b gets P CTAs (P = co-resident grid / batch); CTA p of token b
// takes kept rows [k_b*p/P, k_b*(p+1)/P) (split-K), accumulates all m outputs in float32
// registers and writes one partial row. When P > 1 the launch is cooperative: after a
// grid barrier (bounded wait) every CTA sums a slice of the outputs over the P partials
// in a fixed order, so results are bit-reproducible. When P == 1 the CTA writes y.
//
// One token: a grid of CG column groups x RG row groups (colstream.cuh). CTA (cg, rg)
// streams the column slice of group cg of every kept row of rank = rg (mod RG), and the
// last CTA of a column group to finish sums the group's RG partial rows in order; no
// grid barrier, and the result is bit-reproducible.

#include <algorithm>

#include "colstream.cuh"
#include "internal.h"

namespace wina {

template <bool BF16, int VPT, int U>
__device__ __forceinline__ void spmv_rows(const void* __restrict__ Wt, int64_t n, const RowLayout& L,
                                          const int32_t* __restrict__ idx_b, const float* __restrict__ xs_b, int lo,
                                          int hi, int32_t* rows, float* vals, float* red, float* __restrict__ out,
                                          uint64_t pol, int32_t* status) {
  constexpr int EPV = VecOps<BF16>::EPV;
  float acc[VPT][EPV];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[j][e] = 0.f;
  for (int r0 = lo; r0 < hi; r0 += kRowChunk) {
    const int nr = min(kRowChunk, hi - r0);
    __syncthreads();
    for (int i = threadIdx.x; i < nr; i += kNT) {
      int32_t row = __ldg(idx_b + r0 + i);
      float v = __ldg(xs_b + r0 + i);
      if (row < 0 || (int64_t)row >= n) {  // never read outside Wt
        record_status(status, WINA_ERR_INVALID_ARG);
        row = 0;
        v = 0.f;
      }
      rows[i] = row;
      vals[i] = v;
    }
    __syncthreads();
    accumulate_rows<BF16, VPT, U>(Wt, L, rows, vals, nr, acc, pol);
  }
  store_partial<BF16, VPT>(out, L, acc, red);
}

// out4[q] = sum over pp < P of part4[(token(q) * P + pp) * m4 + col(q)] for q in [q0, q1),
// fixed summation order per output. `red4` is SMEM of kNT float4.
__device__ __forceinline__ void reduce_partials(const float4* __restrict__ part4, int64_t m4, int P, int64_t q0,
                                                int64_t q1, float4* __restrict__ out4, float4* red4) {
  const int64_t nq = q1 - q0;
  for (int64_t qb = 0; qb < nq; qb += kNT) {
    const int w = (int)min((int64_t)kNT, nq - qb);
    const int groups = kNT / w;
    const int t = threadIdx.x;
    const int qi = t % w, grp = t / w;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grp < groups) {
      const int64_t q = q0 + qb + qi;
      const int64_t tok = q / m4, c4 = q % m4;
      for (int pp = grp; pp < P; pp += groups) {
        const float4 v = __ldcg(part4 + (tok * P + pp) * m4 + c4);
        a.x += v.x;
        a.y += v.y;
        a.z += v.z;
        a.w += v.w;
      }
    }
    red4[t] = a;
    __syncthreads();
    if (t < w) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int g = 0; g < groups; ++g) {
        const float4 v = red4[g * w + t];
        s.x += v.x;
        s.y += v.y;
        s.z += v.z;
        s.w += v.w;
      }
      out4[q0 + qb + t] = s;
    }
    __syncthreads();
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kNT, 1)
    k_sparse_matvec(const void* __restrict__ Wt, int64_t n, int64_t m, const int32_t* __restrict__ idx,
                    const float* __restrict__ xs, int k_fixed, const int32_t* __restrict__ count, int ld_idx, int P,
                    float* __restrict__ y, float* __restrict__ partials, GridBarrier* bar, int32_t* status) {
  constexpr int EPV = VecOps<BF16>::EPV;
  extern __shared__ __align__(16) unsigned char smraw[];
  int32_t* rows = reinterpret_cast<int32_t*>(smraw);      // [kRowChunk]
  float* vals = reinterpret_cast<float*>(rows + kRowChunk);  // [kRowChunk]
  float* red = vals + kRowChunk;                            // [kNT * 8]
  const int cta = blockIdx.x;
  const int b = cta / P, p = cta % P;
  int kb = k_fixed;
  if (kb < 0) kb = max(0, min(__ldg(count + b), ld_idx));
  const int lo = (int)((int64_t)kb * p / P);
  const int hi = (int)((int64_t)kb * (p + 1) / P);
  const RowLayout L = make_row_layout<kNT>(m, EPV);
  const uint64_t pol = l2_evict_first_policy();
  const int32_t* idx_b = idx + (int64_t)b * ld_idx;
  const float* xs_b = xs + (int64_t)b * ld_idx;
  float* out = (P == 1) ? y + (int64_t)b * m : partials + (int64_t)cta * m;
  switch (L.VPT) {
    case 1: spmv_rows<BF16, 1, 8>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 2: spmv_rows<BF16, 2, 4>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 3: spmv_rows<BF16, 3, 4>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 4: spmv_rows<BF16, 4, 3>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 5: spmv_rows<BF16, 5, 2>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 6: spmv_rows<BF16, 6, 2>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    case 7: spmv_rows<BF16, 7, 1>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
    default: spmv_rows<BF16, 8, 1>(Wt, n, L, idx_b, xs_b, lo, hi, rows, vals, red, out, pol, status); break;
  }
  if (P == 1) return;
  if (!grid_sync(bar, gridDim.x, status)) return;
  const int64_t m4 = m / 4;
  const int64_t C4 = (int64_t)(gridDim.x / P) * m4;
  const int64_t q0 = C4 * cta / gridDim.x, q1 = C4 * (cta + 1) / gridDim.x;
  reduce_partials(reinterpret_cast<const float4*>(partials), m4, P, q0, q1, reinterpret_cast<float4*>(y),
                  reinterpret_cast<float4*>(red));
}

__global__ void k_silu_mul(const float* __restrict__ g, const float* __restrict__ u, float* __restrict__ h,
                           int64_t count) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    const float gv = g[i];
    h[i] = gv / (1.0f + expf(-gv)) * u[i];
  }
}

static size_t spmv_smem() { return (size_t)kRowChunk * 8 + (size_t)kNT * 8 * 4; }

uint8_t* union_flags_for(void* ws, int wdt, int64_t n, int64_t m, int64_t batch) {
  if (batch < kUnionMinBatch || batch > kUnionBlock || !union_path_takes(wdt, n, m, batch)) return nullptr;
  return reinterpret_cast<uint8_t*>((char*)ws + spmv_ws_layout(m, batch).total + union_ws_layout(n, batch).flag);
}

// One token, column slices: CTA b = (cg = b % CG, rg = b / CG). Dynamic SMEM: the CTA's list
// entries (rows, values) [cap] each, then kCT * 4 floats for the pass sums.
template <bool BF16, int U>
__global__ void __launch_bounds__(kCT, 1)
    k_spmv_cols(const void* __restrict__ Wt, int64_t n, int64_t V, const int32_t* __restrict__ idx,
                const float* __restrict__ xs, int k_fixed, const int32_t* __restrict__ count, int ld, int CG, int RG,
                int cap, float* __restrict__ y, float* __restrict__ part, int pstride, unsigned* counters,
                int32_t* status) {
  constexpr int EPV = VecOps<BF16>::EPV;
  extern __shared__ __align__(16) unsigned char smraw[];
  int32_t* lrow = reinterpret_cast<int32_t*>(smraw);
  float* lval = reinterpret_cast<float*>(lrow + cap);
  float* red = lval + cap;  // 16-byte aligned: cap % 4 == 0
  const int t = threadIdx.x;
  const int cg = blockIdx.x % CG, rg = blockIdx.x / CG;
  const int v0 = (int)(V * cg / CG), v1 = (int)(V * (cg + 1) / CG), nv = v1 - v0;
  int kb = k_fixed;
  if (kb < 0) kb = max(0, min(__ldg(count), ld));
  const int cnt = kb > rg ? min(cap, (kb - rg + RG - 1) / RG) : 0;  // cap holds every entry (launcher)
  for (int i = t; i < cnt; i += kCT) {
    const int e = rg + i * RG;
    int32_t row = __ldg(idx + e);
    float v = __ldg(xs + e);
    if (row < 0 || (int64_t)row >= n) {  // never read outside Wt
      record_status(status, WINA_ERR_INVALID_ARG);
      row = 0;
      v = 0.f;
    }
    lrow[i] = row;
    lval[i] = v;
  }
  __syncthreads();
  float out[EPV];
  stream_cols<BF16, U>(Wt, V, v0, nv, cnt, [&](int i) { return lrow[i]; }, [&](int i) { return lval[i]; }, red,
                       l2_evict_first_policy(), out);
  if (t < nv) {
    float4* o = reinterpret_cast<float4*>(part + (int64_t)rg * pstride + (int64_t)(v0 + t) * EPV);
#pragma unroll
    for (int q = 0; q < EPV / 4; ++q) __stcg(o + q, make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]));
  }
  if (!group_arrive_last(counters + cg, RG)) return;
  // the last of the group: y over its columns = the RG partial rows summed in order
  if (t < nv) {
    float s[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) s[e] = 0.f;
    for (int r = 0; r < RG; ++r) {
      const float4* o = reinterpret_cast<const float4*>(part + (int64_t)r * pstride + (int64_t)(v0 + t) * EPV);
#pragma unroll
      for (int q = 0; q < EPV / 4; ++q) {
        const float4 v = __ldcg(o + q);
        s[4 * q] += v.x; s[4 * q + 1] += v.y; s[4 * q + 2] += v.z; s[4 * q + 3] += v.w;
      }
    }
    float4* yo = reinterpret_cast<float4*>(y + (int64_t)(v0 + t) * EPV);
#pragma unroll
    for (int q = 0; q < EPV / 4; ++q) yo[q] = make_float4(s[4 * q], s[4 * q + 1], s[4 * q + 2], s[4 * q + 3]);
  }
}

// The single-token column-slice launch; WINA_ERR_UNSUPPORTED_DTYPE (no launch) when the
// shape is outside what it takes.
static wina_status_t launch_spmv_cols(const void* Wt, int wdt, int64_t n, int64_t m, const int32_t* idx,
                                      const float* xs, int k, const int32_t* count, int ld, float* y, void* ws,
                                      int32_t* status, cudaStream_t s) {
  const bool bf16 = wdt == WINA_BF16;
  const int64_t V = m * (bf16 ? 2 : 4) / 16;
  const int sms = device_sm_count();
  if (sms < 1) return WINA_ERR_CUDA;
  // CG column groups of RG row groups, about one CTA per SM: slices of about 32 vectors
  // (512 bytes, long enough for full-rate streaming), the rest of the SMs as row groups
  const int CG = (int)std::max<int64_t>(1, std::min<int64_t>(sms / 4, V / 32));
  const int RG = std::max(1, std::min(64, sms / CG));
  if ((V + CG - 1) / CG > kCT || CG > kGridCap || RG > 64) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int kmax = k >= 0 ? k : ld;
  const int cap = std::max(4, ((kmax + RG - 1) / RG + 3) / 4 * 4);
  const size_t smem = (size_t)cap * 8 + (size_t)kCT * 4 * 4;
  if (smem > 200 * 1024) return WINA_ERR_UNSUPPORTED_DTYPE;
  const SpmvWs L = spmv_ws_layout(m, 1);
  float* part = reinterpret_cast<float*>((char*)ws + L.partials);
  unsigned* counters = reinterpret_cast<unsigned*>((char*)ws + L.counters);
  const int pstride = (int)(m + 4);  // rows offset by 4 floats: one column of successive rows spreads over L2 slices
  void (*kern)(const void*, int64_t, int64_t, const int32_t*, const float*, int, const int32_t*, int, int, int, int,
               float*, float*, int, unsigned*, int32_t*) = bf16 ? k_spmv_cols<true, 4> : k_spmv_cols<false, 4>;
  cudaError_t e = ensure_prefer_l1((const void*)kern);  // the loads in flight live in L1
  if (e != cudaSuccess) return cuda_status(e);
  e = launch_kernel(kern, dim3((unsigned)(CG * RG)), dim3(kCT), smem, s, false, Wt, n, V, idx, xs, k, count, ld, CG,
                    RG, cap, y, part, pstride, counters, status);
  return cuda_status(e);
}

wina_status_t launch_sparse_matvec(const void* Wt, int wdt, int64_t n, int64_t m, const int32_t* idx,
                                   const float* xs, int k, const int32_t* count, int ld_idx, int batch, float* y,
                                   void* ws, int32_t* status_dev, cudaStream_t s, bool premarked) {
  if (batch >= kUnionMinBatch && union_path_takes(wdt, n, m, batch))
    return launch_union_matvec(Wt, n, m, idx, xs, k, count, ld_idx, batch, y,
                               (char*)ws + spmv_ws_layout(m, batch).total, status_dev, s, premarked);
  if (batch == 1) {  // one token: column slices, when the shape fits
    const wina_status_t r1 = launch_spmv_cols(Wt, wdt, n, m, idx, xs, k, count, ld_idx, y, ws, status_dev, s);
    if (r1 != WINA_ERR_UNSUPPORTED_DTYPE) return r1;
  }
  const bool bf16 = wdt == WINA_BF16;
  const size_t smem = spmv_smem();
  const int gmax = bf16 ? max_coresident_grid(k_sparse_matvec<true>, kNT, smem)
                        : max_coresident_grid(k_sparse_matvec<false>, kNT, smem);
  if (gmax < 1) return WINA_ERR_CUDA;
  int P = batch < gmax ? gmax / batch : 1;
  const int kmax = k >= 0 ? k : ld_idx;
  const int want = (kmax + 7) / 8;  // at least ~8 kept rows per CTA
  if (P > want) P = want > 0 ? want : 1;
  const SpmvWs L = spmv_ws_layout(m, batch);
  GridBarrier* bar = reinterpret_cast<GridBarrier*>((char*)ws + L.bar);
  float* part = reinterpret_cast<float*>((char*)ws + L.partials);
  const bool coop = P > 1;
  const dim3 grid((unsigned)((int64_t)batch * P));
  cudaError_t e;
  if (bf16)
    e = launch_kernel(k_sparse_matvec<true>, grid, dim3(kNT), smem, s, coop, Wt, n, m, idx, xs, k, count, ld_idx, P,
                      y, part, bar, status_dev);
  else
    e = launch_kernel(k_sparse_matvec<false>, grid, dim3(kNT), smem, s, coop, Wt, n, m, idx, xs, k, count, ld_idx, P,
                      y, part, bar, status_dev);
  return cuda_status(e);
}

wina_status_t launch_silu_mul(const float* g, const float* u, float* h, int64_t count, cudaStream_t s) {
  int64_t blocks = (count + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  k_silu_mul<<<(unsigned)blocks, 256, 0, s>>>(g, u, h, count);
  return cuda_status(cudaGetLastError());
}

}  // namespace wina

using namespace wina;

extern "C" wina_status_t sparse_matvec(const void* Wt, wina_dtype_t wdt, int64_t n, int64_t m, const int32_t* idx,
                                       const float* xs, int64_t k, const int32_t* count, int64_t ld_idx,
                                       int64_t batch, float* y, void* ws, size_t ws_bytes, int32_t* status_dev,
                                       wina_stream_t stream) {
  if (!valid_dtype(wdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (n < 1 || n > INT32_MAX || m < epv || m % epv != 0 || m / epv > (int64_t)kNT * 8) return WINA_ERR_INVALID_ARG;
  if (batch < 1 || batch > INT32_MAX || ld_idx < 0 || ld_idx > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (k < -1 || k > ld_idx || (k == -1 && !count)) return WINA_ERR_INVALID_ARG;
  if (!Wt || !y || !ws || (ld_idx > 0 && (!idx || !xs))) return WINA_ERR_INVALID_ARG;
  if (!aligned(Wt, 16) || !aligned(y, 16) || !aligned(ws, 16) || (idx && !aligned(idx, 4)) ||
      (xs && !aligned(xs, 4)) || (count && !aligned(count, 4)) || (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  if (ws_bytes < wina_workspace_size(WINA_OP_SPARSE_MATVEC, n, m, ld_idx, batch)) return WINA_ERR_WORKSPACE;
  return launch_sparse_matvec(Wt, wdt, n, m, idx, xs, (int)k, count, (int)ld_idx, (int)batch, y, ws, status_dev,
                              (cudaStream_t)stream);
}

// ------------------------------------------------------------------------------------
// sparse_matvec_noalloc: the same product with library-owned scratch
// ------------------------------------------------------------------------------------
//
// Some callers cannot hand the library a workspace: code that runs where device
// allocation is forbidden or too costly (a fixed memory pool owned by a host framework,
// a latency-critical loop in which cudaMalloc could synchronise the device and stall
// other streams, a plugin that only receives input and output buffers). For them this
// entry point keeps its scratch (one grid-barrier word pair and the split-K partial
// rows) in a fixed array in device memory that the library itself declares; every GPU
// that loads the library holds it until the process exits.

namespace wina {

constexpr int64_t kNoAllocPartialFloats = (int64_t)1 << 21;  // 8 MiB of partial sums
constexpr int64_t kNoAllocMaxOutputs = kNoAllocPartialFloats / 2;  // batch * m limit

// [GridBarrier (256 B)][partials: kNoAllocPartialFloats float32]
static __device__ __align__(256) unsigned char g_noalloc_scratch[256 + kNoAllocPartialFloats * 4];

// Device address of g_noalloc_scratch in the current context. In host code the array's
// name is only a host-side stand-in, so the address is looked up on every call (a cheap
// runtime query), which stays right across a device reset or a new primary context.
// Returns nullptr on error.
static void* noalloc_scratch_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace wina

extern "C" wina_status_t sparse_matvec_noalloc(const void* Wt, wina_dtype_t wdt, int64_t n, int64_t m,
                                               const int32_t* idx, const float* xs, int64_t k, const int32_t* count,
                                               int64_t ld_idx, int64_t batch, float* y, int32_t* status_dev,
                                               wina_stream_t stream) {
  if (!valid_dtype(wdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (n < 1 || n > INT32_MAX || m < epv || m % epv != 0 || m / epv > (int64_t)kNT * 8) return WINA_ERR_INVALID_ARG;
  if (batch < 1 || batch > INT32_MAX || ld_idx < 0 || ld_idx > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (k < -1 || k > ld_idx || (k == -1 && !count)) return WINA_ERR_INVALID_ARG;
  if (!Wt || !y || (ld_idx > 0 && (!idx || !xs))) return WINA_ERR_INVALID_ARG;
  if (!aligned(Wt, 16) || !aligned(y, 16) || (idx && !aligned(idx, 4)) || (xs && !aligned(xs, 4)) ||
      (count && !aligned(count, 4)) || (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  char* scratch = (char*)noalloc_scratch_ptr();
  if (!scratch) return WINA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const bool bf16 = wdt == WINA_BF16;
  const size_t smem = spmv_smem();
  const int gmax = bf16 ? max_coresident_grid(k_sparse_matvec<true>, kNT, smem)
                        : max_coresident_grid(k_sparse_matvec<false>, kNT, smem);
  if (gmax < 1) return WINA_ERR_CUDA;
  const int B = (int)batch;
  // With at least one co-resident CTA per token (P == 1) every CTA writes its token's y
  // directly and the scratch is not used, whatever the size. Otherwise the split-K
  // partial rows must fit in the fixed array: at least two per token.
  if (B < gmax && batch * m > kNoAllocMaxOutputs) return WINA_ERR_INVALID_ARG;
  int P = B < gmax ? gmax / B : 1;
  const int kmax = k >= 0 ? (int)k : (int)ld_idx;
  const int want = (kmax + 7) / 8;
  if (P > want) P = want > 0 ? want : 1;
  if (P > 1) {
    const int64_t fit = kNoAllocPartialFloats / (batch * m);  // partial rows per token that fit
    if (P > fit) P = (int)fit;                                // >= 2 by the size check above
  }
  // The barrier words must start at zero: clear them on the stream (the partial rows
  // are always written before they are read). Calls that overlap on the GPU share this
  // scratch and race.
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(GridBarrier), s);
  if (e != cudaSuccess) return cuda_status(e);
  GridBarrier* bar = reinterpret_cast<GridBarrier*>(scratch);
  float* part = reinterpret_cast<float*>(scratch + 256);
  const bool coop = P > 1;
  const dim3 grid((unsigned)((int64_t)B * P));
  if (bf16)
    e = launch_kernel(k_sparse_matvec<true>, grid, dim3(kNT), smem, s, coop, Wt, n, m, idx, xs, (int)k, count,
                      (int)ld_idx, P, y, part, bar, status_dev);
  else
    e = launch_kernel(k_sparse_matvec<false>, grid, dim3(kNT), smem, s, coop, Wt, n, m, idx, xs, (int)k, count,
                      (int)ld_idx, P, y, part, bar, status_dev);
  return cuda_status(e);
}
