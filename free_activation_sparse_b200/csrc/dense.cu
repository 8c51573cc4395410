// The dense comparator: the unsparsified layer y = W x and the unsparsified SwiGLU FFN,
// on the output-major weights W[m][n] (each output is one contiguous row).
//
// The weights are read as one flat stream of 512-byte slabs (32 16-byte vectors, one per
// lane: a row of n elements is n / (32 * EPV) slabs). Every warp of the grid takes an
// equal contiguous range of slabs, keeps 4 loads per matrix (gate and up together) in
// flight per lane and multiplies by x, which each CTA stages once in shared memory in an
// order that makes every lane's float4 reads conflict-free. A warp's range is at least one
// row long, so a row is shared by at most two warps: each adds its part of the dot product
// into a zeroed output with one atomic add, and two float additions onto zero give the
// same bits in either order (the result does not depend on timing).
//
// Rows that are not a whole number of slabs, or too long to stage x in shared memory,
// take the warp-per-row kernels below, which read x through L1.
#include <math.h>

#include <algorithm>

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

constexpr int kST = 512;                 // threads per CTA of the slab kernels
constexpr int kSlabMaxSmem = 96 * 1024;  // x staged in shared memory up to this size

// Position of element e of x in shared memory: slab j (32 * EPV elements, EPV per lane) is
// stored as EPV / 4 planes of 32 float4s, plane p holding elements 4p..4p+3 of every
// lane's vector, so that a warp's float4 reads of a plane are 512 consecutive bytes.
template <int EPV>
__device__ __forceinline__ int xs_pos(int e) {
  const int slab = e / (32 * EPV), r = e - slab * (32 * EPV);
  const int lane = r / EPV, k = r - lane * EPV;
  return slab * 32 * EPV + (k >> 2) * 128 + lane * 4 + (k & 3);
}

// x into shared memory (positions xs_pos): kQ groups of 4 elements per thread per round,
// all of a round's loads issued before any is used, so that staging costs one round trip to L2.
// x is x[0..n) of dtype xdt, or silu(gin) * uin when gin is given; n % 4 == 0.
template <int EPV, int kQ>
__device__ __forceinline__ void stage_x(float* xs, int n, const void* __restrict__ x, int xdt,
                                        const float* __restrict__ gin, const float* __restrict__ uin) {
  const int nq = n / 4;
  for (int q0 = 0; q0 < nq; q0 += kQ * kST) {
    float4 a[kQ], b[kQ];
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = q0 + k * kST + (int)threadIdx.x;
      a[k] = b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (q < nq) {
        if (gin) {
          a[k] = __ldcg(reinterpret_cast<const float4*>(gin) + q);  // written by this or the last launch
          b[k] = __ldcg(reinterpret_cast<const float4*>(uin) + q);
        } else if (xdt == WINA_F32) {
          a[k] = __ldg(reinterpret_cast<const float4*>(x) + q);
        } else {
          const uint2 h = __ldg(reinterpret_cast<const uint2*>(x) + q);
          a[k] = make_float4(__uint_as_float(h.x << 16), __uint_as_float(h.x & 0xffff0000u),
                             __uint_as_float(h.y << 16), __uint_as_float(h.y & 0xffff0000u));
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = q0 + k * kST + (int)threadIdx.x;
      if (q < nq) {
        float v[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
        if (gin) {
          const float u[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = v[j] / (1.0f + expf(-v[j])) * u[j];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) xs[xs_pos<EPV>(4 * q + j)] = v[j];
      }
    }
  }
}

// One warp's share of the flat slab stream of a matrix of m rows of n elements, rows a
// whole number of slabs (n % (32 EPV) == 0), so that slab s starts at byte 512 s: slabs
// [s0, s1) of T = m * spr (spr slabs per row) among wuse = min(warps, m) warps, so that a
// share is at least one row long. The slabs are loaded U at a time into two register
// buffers in turn, at fixed offsets from one running address, the next batch always in
// flight while the current one is multiplied; the first batch can be issued early
// (first()) so that its loads are in flight while x is staged or a barrier is waited on.
template <bool BF16, int U>
struct SlabStream {
  static constexpr int EPV = VecOps<BF16>::EPV;
  const uint4* p;  // this lane's vector of the next slab to load
  int spr, ns, row, col;
  bool active;
  uint64_t pol;
  uint4 wa[U], wb[U];

  __device__ __forceinline__ SlabStream(const void* W, int m, int n, int gw, int warps) {
    spr = n / (32 * EPV);
    const int64_t T = (int64_t)m * spr;
    const int wuse = (int)min((int64_t)warps, (int64_t)m);
    active = gw < wuse;
    const int64_t s0 = active ? T * gw / wuse : 0, s1 = active ? T * (gw + 1) / wuse : 0;
    ns = (int)(s1 - s0);
    row = (int)(s0 / spr);
    col = (int)(s0 - (int64_t)row * spr);
    p = reinterpret_cast<const uint4*>(W) + s0 * 32 + (threadIdx.x & 31);
    pol = l2_evict_first_policy();
  }

  // the next U slabs into w (only the first `left` exist)
  __device__ __forceinline__ void load(uint4 (&w)[U], int left) {
    if (left >= U) {
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = ld_stream_u4(p + u * 32, pol);
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = u < left ? ld_stream_u4(p + u * 32, pol) : make_uint4(0u, 0u, 0u, 0u);
    }
    p += U * 32;
  }

  __device__ __forceinline__ void first() {
    if (active) load(wa, ns);
  }

  // one slab: acc += w . x over this lane's EPV elements
  __device__ __forceinline__ void fma_slab(float (&acc)[EPV], const uint4& w, const float4* xp) {
#pragma unroll
    for (int q = 0; q < EPV / 4; ++q) {
      const float4 f = xp[q * 32];
      float wv[4];
      if (BF16) {
        const uint32_t a = q == 0 ? w.x : w.z, b = q == 0 ? w.y : w.w;
        wv[0] = __uint_as_float(a << 16);
        wv[1] = __uint_as_float(a & 0xffff0000u);
        wv[2] = __uint_as_float(b << 16);
        wv[3] = __uint_as_float(b & 0xffff0000u);
      } else {
        wv[0] = __uint_as_float(w.x);
        wv[1] = __uint_as_float(w.y);
        wv[2] = __uint_as_float(w.z);
        wv[3] = __uint_as_float(w.w);
      }
      acc[4 * q] = fmaf(wv[0], f.x, acc[4 * q]);
      acc[4 * q + 1] = fmaf(wv[1], f.y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(wv[2], f.z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(wv[3], f.w, acc[4 * q + 3]);
    }
  }

  // The whole share (first() issued before): out[row] += partial dot products with x
  // (xs: positions xs_pos), one atomic add per row.
  __device__ __forceinline__ void run(const float* xs, float* __restrict__ out) {
    if (!active) return;
    const int lane = threadIdx.x & 31;
    float acc[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
    const float4* xl = reinterpret_cast<const float4*>(xs) + lane;
    // the slabs of one buffer (cnt of them), the row's sum flushed whenever a row ends
    auto consume = [&](const uint4 (&w)[U], int cnt) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u < cnt) {
          fma_slab(acc, w[u], xl + col * (8 * EPV));  // 32 EPV floats per slab
          if (++col == spr) {  // the row is complete in this warp's part
            float t = 0.f;
#pragma unroll
            for (int e = 0; e < EPV; ++e) {
              t += acc[e];
              acc[e] = 0.f;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) t += __shfl_down_sync(0xffffffffu, t, o);
            if (lane == 0) atomicAdd(out + row, t);
            col = 0;
            ++row;
          }
        }
      }
    };
    int left = ns;  // slabs not yet multiplied; wa holds the next U of them
    while (left > 0) {
      if (left > U) load(wb, left - U);
      consume(wa, left);
      left -= U;
      if (left <= 0) break;
      if (left > U) load(wa, left - U);
      consume(wb, left);
      left -= U;
    }
    if (col > 0) {  // the share ends inside a row
      float t = 0.f;
#pragma unroll
      for (int e = 0; e < EPV; ++e) t += acc[e];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) t += __shfl_down_sync(0xffffffffu, t, o);
      if (lane == 0) atomicAdd(out + row, t);
    }
  }
};

// y[row] = W[row][:] . x over the grid's slab stream (y zeroed before the launch); x of
// dtype xdt.
template <bool BF16, int U>
__global__ void __launch_bounds__(kST, 2)
    k_dense_slabs(const void* __restrict__ W, int m, int n, const void* __restrict__ x, int xdt,
                  float* __restrict__ y) {
  extern __shared__ __align__(16) float xs[];
  SlabStream<BF16, U> st(W, m, n, blockIdx.x * (kST / 32) + (threadIdx.x >> 5), gridDim.x * (kST / 32));
  st.first();  // in flight while x is staged
  stage_x<VecOps<BF16>::EPV, 4>(xs, n, x, xdt, nullptr, nullptr);
  __syncthreads();
  st.run(xs, y);
}

struct DenseFfnParams {
  const void* wg;
  const void* wu;
  const void* wd;
  int d, ffn;
  const void* x;
  int xdt;
  float* gu[2];  // two copies of [g (ffn, padded to 4) | u (ffn)], used by alternate calls
  unsigned* parity;  // which copy this call uses
  float* y;          // [d]
  GridBarrier* bar;
  unsigned long long wait_ns;
  int32_t* status;
};

// The dense FFN in one cooperative launch. W_gate is streamed into g by half of the warps
// and W_up into u by the other half; y is zeroed on the way; a grid barrier (the first
// down loads already in flight); h = silu(g) * u staged by every CTA; W_down streamed into
// y. g and u are added into a copy that the previous call zeroed, and this call zeroes the
// other copy for the next one, so that no barrier is needed before the first adds (the
// copies alternate by a parity word that CTA 0 flips once every CTA has read it).
template <bool BF16>
__global__ void __launch_bounds__(kST, 2) k_dense_ffn(DenseFfnParams p) {
  constexpr int EPV = VecOps<BF16>::EPV;
  extern __shared__ __align__(16) float xs[];
  const int G = gridDim.x, warps = G * (kST / 32);
  const int gw = blockIdx.x * (kST / 32) + (threadIdx.x >> 5);
  const unsigned par = __ldcg(p.parity) & 1u;
  float* g = par ? p.gu[1] : p.gu[0];
  float* u = g + ((p.ffn + 3) & ~3);
  {
    float* other = par ? p.gu[0] : p.gu[1];
    const int n2 = ((p.ffn + 3) & ~3) + p.ffn;
    for (int e = blockIdx.x * kST + threadIdx.x; e < n2; e += G * kST) other[e] = 0.f;
  }
  for (int e = blockIdx.x * kST + threadIdx.x; e < p.d; e += G * kST) p.y[e] = 0.f;
  {
    // the first half of the warps streams W_gate into g, the second half W_up into u
    const int half = warps / 2;
    const bool gate = gw < half;
    SlabStream<BF16, 3> st(gate ? p.wg : p.wu, p.ffn, p.d, gate ? gw : gw - half, gate ? half : warps - half);
    st.first();
    stage_x<EPV, 4>(xs, p.d, p.x, p.xdt, nullptr, nullptr);
    __syncthreads();
    st.run(xs, gate ? g : u);
  }
  SlabStream<BF16, 3> dn(p.wd, p.d, p.ffn, gw, warps);
  dn.first();  // in flight across the barrier
  if (!grid_sync_fixed(p.bar, G, p.status, p.wait_ns)) return;  // g, u complete; y zeroed
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.parity = par ^ 1u;  // every CTA has read it
  stage_x<EPV, 4>(xs, p.ffn, nullptr, WINA_F32, g, u);
  __syncthreads();
  dn.run(xs, p.y);
}

static size_t slab_smem(int n, int epv) { return (size_t)n * 4; }
// rows of whole slabs whose x fits in shared memory
static bool slab_path(int n, int epv) { return n % (32 * epv) == 0 && slab_smem(n, epv) <= (size_t)kSlabMaxSmem; }

template <bool BF16, int U>
static wina_status_t launch_slabs(const void* W, int m, int n, const void* x, int xdt, float* y, cudaStream_t s) {
  const void* kern = (const void*)k_dense_slabs<BF16, U>;
  const size_t smem = slab_smem(n, VecOps<BF16>::EPV);
  {  // always: static shared memory comes on top of the dynamic part
    const cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // the smallest carveout that holds two CTAs (the rest of the SM's 256 KB is L1, where
  // the loads in flight land)
  const int pct = (int)std::min<size_t>(100, (2 * (smem + 1024) * 100 + 228 * 1024 - 1) / (228 * 1024));
  const cudaError_t e = ensure_carveout(kern, pct);
  if (e != cudaSuccess) return cuda_status(e);
  k_dense_slabs<BF16, U><<<device_sm_count() * 2, kST, smem, s>>>(W, m, n, x, xdt, y);
  return cuda_status(cudaGetLastError());
}

static int dense_grid() { return device_sm_count() * 8; }  // 8 CTAs of 8 warps per SM

wina_status_t launch_widen(const void* x, int xdt, int n, float* xf, cudaStream_t s) {
  k_widen<<<32, 256, 0, s>>>(x, xdt, n, xf);
  return cuda_status(cudaGetLastError());
}

// y = W x (y[0..m) written; x of dtype xdt, n elements); xbuf: n floats of scratch, used
// only when the rows are too long for the slab kernel.
wina_status_t launch_dense_gemv(const void* W, int wdt, int m, int n, const void* x, int xdt, float* y, float* xbuf,
                                cudaStream_t s) {
  const bool bf16 = wdt == WINA_BF16;
  if (slab_path(n, bf16 ? 8 : 4) && aligned(x, 4 * elem_size(xdt))) {  // x staged 4 elements at a time
    const cudaError_t e = cudaMemsetAsync(y, 0, (size_t)m * sizeof(float), s);
    if (e != cudaSuccess) return cuda_status(e);
    return bf16 ? launch_slabs<true, 3>(W, m, n, x, xdt, y, s) : launch_slabs<false, 3>(W, m, n, x, xdt, y, s);
  }
  k_widen<<<32, 256, 0, s>>>(x, xdt, n, xbuf);
  if (bf16)
    k_dense_gemv<true><<<dense_grid(), kGT, 0, s>>>(W, m, n, xbuf, y);
  else
    k_dense_gemv<false><<<dense_grid(), kGT, 0, s>>>(W, m, n, xbuf, y);
  return cuda_status(cudaGetLastError());
}

struct DenseWs {
  size_t bar, parity, gu0, gu1, total;  // gu0, gu1: the two [g | u] copies (or x widened and
                                        // h on the warp-per-row path)
};

static DenseWs dense_ws_layout(int64_t d, int64_t ffn) {
  DenseWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = round_up(o + bytes, kAlign);
    return at;
  };
  const size_t gub = (size_t)(round_up((size_t)std::max(d, ffn), 4) + ffn) * 4;
  w.bar = take(sizeof(GridBarrier));
  w.parity = take(4);
  w.gu0 = take(gub);
  w.gu1 = take(gub);
  w.total = o;
  return w;
}

size_t dense_ws_size(int64_t d, int64_t ffn) { return dense_ws_layout(d, ffn).total; }

// The fused cooperative kernel when it fits (x and h staged in shared memory, two CTAs of
// 512 threads per SM co-resident); WINA_ERR_UNSUPPORTED_DTYPE (no launch) when it does not.
static wina_status_t launch_dense_ffn_fused(const DenseFfnParams& p0, bool bf16, cudaStream_t s) {
  const int epv = bf16 ? 8 : 4;
  if (!slab_path(p0.d, epv) || !slab_path(p0.ffn, epv) || !aligned(p0.x, 4 * elem_size(p0.xdt)))
    return WINA_ERR_UNSUPPORTED_DTYPE;
  void* kern = bf16 ? (void*)k_dense_ffn<true> : (void*)k_dense_ffn<false>;
  const size_t smem = std::max(slab_smem(p0.d, epv), slab_smem(p0.ffn, epv));
  {  // always: static shared memory comes on top of the dynamic part
    const cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
  }
  const int pct = (int)std::min<size_t>(100, (2 * (smem + 1024) * 100 + 228 * 1024 - 1) / (228 * 1024));
  cudaError_t e = ensure_carveout(kern, pct);
  if (e != cudaSuccess) return cuda_status(e);
  const int bps = std::min(2, blocks_per_sm(kern, kST, smem));
  if (bps < 1) return WINA_ERR_UNSUPPORTED_DTYPE;
  DenseFfnParams p = p0;
  p.wait_ns = wait_limit_ns();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(device_sm_count() * bps));
  cfg.blockDim = dim3(kST);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&p};
  return cuda_status(cudaLaunchKernelExC(&cfg, kern, args));
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
  return launch_dense_gemv(W, wdt, (int)m, (int)n, x, xdt, y, xbuf, (cudaStream_t)stream);
}

extern "C" wina_status_t wina_dense_ffn_swiglu(const void* W_gate, const void* W_up, const void* W_down,
                                               wina_dtype_t wdt, int64_t d, int64_t ffn, const void* x,
                                               wina_dtype_t xdt, float* y, void* ws, size_t ws_bytes,
                                               int32_t* status_dev, wina_stream_t stream) {
  if (!valid_dtype(wdt) || !valid_dtype(xdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int epv = wdt == WINA_BF16 ? 8 : 4;
  if (d < epv || ffn < epv || d % epv || ffn % epv || d > INT32_MAX || ffn > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!W_gate || !W_up || !W_down || !x || !y || !ws || !aligned(W_gate, 16) || !aligned(W_up, 16) ||
      !aligned(W_down, 16) || !aligned(ws, 16) || !aligned(x, elem_size(xdt)) || !aligned(y, 4) ||
      (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  if (ws_bytes < dense_ws_size(d, ffn)) return WINA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const bool bf16 = wdt == WINA_BF16;
  const DenseWs L = dense_ws_layout(d, ffn);
  char* w = (char*)ws;
  DenseFfnParams p{W_gate, W_up, W_down, (int)d, (int)ffn, x, (int)xdt,
                   {reinterpret_cast<float*>(w + L.gu0), reinterpret_cast<float*>(w + L.gu1)},
                   reinterpret_cast<unsigned*>(w + L.parity), y, reinterpret_cast<GridBarrier*>(w + L.bar), 0,
                   status_dev};
  const wina_status_t rf = launch_dense_ffn_fused(p, bf16, s);
  if (rf != WINA_ERR_UNSUPPORTED_DTYPE) return rf;
  // rows not a whole number of slabs, too long for shared memory, or x not 4-element
  // aligned: separate launches
  float* xf = reinterpret_cast<float*>(w + L.gu0);                          // [d]
  float* h = reinterpret_cast<float*>(w + L.gu0) + round_up((size_t)d, 4);  // [ffn]
  k_widen<<<32, 256, 0, s>>>(x, xdt, (int)d, xf);
  if (bf16) {
    k_dense_gate_up<true><<<dense_grid(), kGT, 0, s>>>(W_gate, W_up, (int)ffn, (int)d, xf, h);
    k_dense_gemv<true><<<dense_grid(), kGT, 0, s>>>(W_down, (int)d, (int)ffn, h, y);
  } else {
    k_dense_gate_up<false><<<dense_grid(), kGT, 0, s>>>(W_gate, W_up, (int)ffn, (int)d, xf, h);
    k_dense_gemv<false><<<dense_grid(), kGT, 0, s>>>(W_down, (int)d, (int)ffn, h, y);
  }
  return cuda_status(cudaGetLastError());
}
