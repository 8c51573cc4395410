// Double Sparsity decode attention ("大模型DoubleSparse稀疏化技术原理", section 技术原理):
//
//  * offline calibration (离线校准): the mean |K| of every channel of a key/value head over
//    the calibration tokens (the K-outlier strategy; the r largest are then picked by the
//    top-K gate kernel), and the label cache, the chosen channels of every token copied
//    into a contiguous [token][r] array;
//  * the decode step (在线前向计算): per query head, the query's important channels, their
//    approximate scores against every token's label row, the top-k tokens by those
//    scores, and full softmax attention of the full query over those tokens' keys and
//    values.
//
// The decode kernel runs one CTA per (sequence, query head). The scores are float32 sums
// in channel order (each product rounded, then added), so that the kept set is a
// deterministic function of the inputs; they are turned into order-preserving 32-bit
// keys in shared memory, the exact top-k (ties to the lower token index) is found as a
// threshold, and the kept tokens are compacted in ascending order. Attention over them:
// one warp per token for the logits, a fixed-order block max and sum, and per-warp
// partial outputs summed in warp order (the result does not depend on timing).
#include <math.h>

#include <algorithm>
#include <cmath>

#include "internal.h"

namespace wina {

constexpr int kAT = 512;  // threads per CTA of the decode kernel
constexpr int kAW = kAT / 32;
constexpr int kDsMaxR = 256;                   // important channels per head, at most
constexpr size_t kDsMaxSmem = 225 * 1024;     // dynamic shared memory of one CTA, at most (2 KB static)

// float -> key whose unsigned order is the float order (+0 and -0 map to one key)
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// EPL consecutive elements of one row held as raw words (loaded now, widened when used), so
// that many rows' loads can be in flight at once.
template <bool BF16, int EPL>
struct Lane {
  static constexpr int BYTES = EPL * (BF16 ? 2 : 4);
  static constexpr int W = BYTES < 4 ? 1 : BYTES / 4;
  uint32_t w[W];
  // elements [off, off + EPL) of p (EPL-element aligned)
  __device__ __forceinline__ void load(const void* p, int64_t off) {
    const char* s = reinterpret_cast<const char*>(p) + off * (BF16 ? 2 : 4);
    if constexpr (BYTES == 2) {
      w[0] = __ldg(reinterpret_cast<const uint16_t*>(s));
    } else if constexpr (BYTES == 4) {
      w[0] = __ldg(reinterpret_cast<const uint32_t*>(s));
    } else if constexpr (BYTES == 8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(s));
      w[0] = v.x;
      w[1] = v.y;
    } else {
#pragma unroll
      for (int q = 0; q < BYTES / 16; ++q) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(s) + q);
        w[4 * q] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
      }
    }
  }
  __device__ __forceinline__ float get(int e) const {
    if constexpr (BF16) return __uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
    else return __uint_as_float(w[e]);
  }
};

struct DsParams {
  const void* q;
  int qdt;
  const void* K;
  const void* V;
  const void* label;
  int kvdt;
  const int32_t* channels;  // [Hkv][r]
  const int32_t* seq_len;   // [B]
  int B, Hq, Hkv, Tmax, dh, r, k;
  float scale;
  float* out;        // [B][Hq][dh]
  int32_t* idx_out;  // [B][Hq][k] or null
  float* scores_out; // [B][Hq][Tmax] or null
  int32_t* status;
};

// Dynamic shared memory: keys [Tmax] | sel [kcap] | logits [kcap] | hist [kSelBins] |
// cand [2 kSelCand] | q [dh] | part [kAW][dh]. EPL = dh / 32 channels per lane.
template <bool BF16, int EPL>
__global__ void __launch_bounds__(kAT, 1) k_ds_decode(DsParams p) {
  constexpr int LV = BF16 ? 8 : 4;                    // label elements per 16-byte piece
  constexpr int TPT = 8;                              // tokens a thread scores per pass
  constexpr int SPW = Lane<BF16, EPL>::W >= 8 ? 4 : (Lane<BF16, EPL>::W >= 4 ? 8 : 16);  // kept tokens per warp per pass
  extern __shared__ __align__(16) uint32_t dsm[];
  const int kcap = min(p.k, p.Tmax);
  uint32_t* keys = dsm;
  int32_t* sel = reinterpret_cast<int32_t*>(keys + p.Tmax);
  float* logits = reinterpret_cast<float*>(sel + kcap);
  uint32_t* hist = reinterpret_cast<uint32_t*>(logits + kcap);
  uint32_t* cand = hist + kSelBins;
  float* qf = reinterpret_cast<float*>(cand + 2 * kSelCand);
  float* part = qf + p.dh;
  __shared__ uint32_t red[2 * kAW + 8];
  __shared__ float fred[kAW];
  __shared__ float qc[kDsMaxR];
  const int b = blockIdx.x / p.Hq, h = blockIdx.x % p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int T = __ldg(p.seq_len + b);
  if (T < 0 || T > p.Tmax) {
    if (tid == 0) record_status(p.status, WINA_ERR_INVALID_ARG);
    T = max(0, min(T, p.Tmax));
  }
  const int64_t head = (int64_t)b * p.Hkv + g;  // key/value head of this sequence
  float* out = p.out + ((int64_t)b * p.Hq + h) * p.dh;

  // step 1: the full query and its important channels
  for (int d = tid; d < p.dh; d += kAT) qf[d] = load_elem(p.q, p.qdt, ((int64_t)b * p.Hq + h) * p.dh + d);
  __syncthreads();
  for (int j = tid; j < p.r; j += kAT) qc[j] = qf[__ldg(p.channels + (int64_t)g * p.r + j)];
  __syncthreads();

  // step 2: approximate scores against the label rows, as order-preserving keys. A thread
  // takes tokens tid + u * kAT (u < TPT) per pass; each 16-byte piece of their label rows
  // is loaded for all of them at once, and every token's products are summed in channel
  // order.
  for (int t0 = tid; t0 < T; t0 += kAT * TPT) {
    float s[TPT];
#pragma unroll
    for (int u = 0; u < TPT; ++u) s[u] = 0.f;
    for (int j0 = 0; j0 < p.r; j0 += LV) {
      Lane<BF16, LV> lab[TPT];
#pragma unroll
      for (int u = 0; u < TPT; ++u)
        if (t0 + u * kAT < T) lab[u].load(p.label, (head * p.Tmax + t0 + u * kAT) * p.r + j0);
#pragma unroll
      for (int u = 0; u < TPT; ++u)
        if (t0 + u * kAT < T) {
#pragma unroll
          for (int e = 0; e < LV; ++e) s[u] = __fadd_rn(s[u], __fmul_rn(qc[j0 + e], lab[u].get(e)));
        }
    }
#pragma unroll
    for (int u = 0; u < TPT; ++u) {
      const int t = t0 + u * kAT;
      if (t < T) {
        keys[t] = order_key(s[u]);
        if (p.scores_out) p.scores_out[((int64_t)b * p.Hq + h) * p.Tmax + t] = s[u];
      }
    }
  }
  __syncthreads();

  // step 3: the top-k tokens (ties to the lower index), ascending
  const int kk = min(p.k, T);
  if (kk == 0) {
    for (int d = tid; d < p.dh; d += kAT) out[d] = 0.f;
    return;
  }
  const Threshold th = select_threshold<kAT>(keys, T, kk, hist, cand, red);
  compact_pred<kAT>(
      T, [&](int i) { return kept_by(th, keys[i], i); },
      [&](uint32_t, uint32_t* lo, uint32_t* hi) {
        *lo = 0;
        *hi = (uint32_t)kk;
      },
      red, [&](int i, uint32_t pos) { sel[pos] = i; });
  if (p.idx_out)
    for (int i = tid; i < kk; i += kAT) p.idx_out[((int64_t)b * p.Hq + h) * p.k + i] = sel[i];

  // attention over the kept tokens. Warp w takes kept tokens w + u * kAW (u < SPW) per
  // pass, lanes over channels; their key and value pieces are loaded together, the
  // logits go to SMEM, and the value pieces wait in registers for the softmax weights.
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const int npass = (kk + kAW * SPW - 1) / (kAW * SPW);
  float mx = -INFINITY, sum = 0.f;
  for (int ps = 0; ps < npass; ++ps) {
    const int i0 = ps * kAW * SPW + warp;
    Lane<BF16, EPL> kr[SPW], vr[SPW];
#pragma unroll
    for (int u = 0; u < SPW; ++u) {
      const int i = i0 + u * kAW;
      if (i < kk) {
        const int64_t row = (head * p.Tmax + sel[i]) * p.dh + (int64_t)lane * EPL;
        kr[u].load(p.K, row);
        vr[u].load(p.V, row);
      }
    }
#pragma unroll
    for (int u = 0; u < SPW; ++u) {
      const int i = i0 + u * kAW;
      if (i < kk) {  // warp-uniform
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) dot = fmaf(qf[lane * EPL + e], kr[u].get(e), dot);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane == 0) logits[i] = dot * p.scale;
      }
    }
    // the softmax needs every logit: with one pass (kk <= kAW * SPW) the value pieces stay
    // in registers across it; with several, the max and sum come after the last pass and
    // the weighted values are added in a second sweep below
    if (npass == 1) {
      __syncthreads();
      for (int i = tid; i < kk; i += kAT) mx = fmaxf(mx, logits[i]);
      {
        float m = mx;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) fred[warp] = m;
        __syncthreads();
        m = fred[0];
        for (int w = 1; w < kAW; ++w) m = fmaxf(m, fred[w]);
        __syncthreads();
        mx = m;
      }
      for (int i = tid; i < kk; i += kAT) {
        const float e = expf(logits[i] - mx);
        logits[i] = e;
        sum += e;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) fred[warp] = sum;
      __syncthreads();
      {
        float s2 = 0.f;
        for (int w = 0; w < kAW; ++w) s2 += fred[w];
        sum = s2;
      }
#pragma unroll
      for (int u = 0; u < SPW; ++u) {
        const int i = i0 + u * kAW;
        if (i < kk) {
          const float wgt = logits[i];
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wgt, vr[u].get(e), acc[e]);
        }
      }
    }
  }
  if (npass > 1) {
    // several passes: softmax over all logits, then the weighted value rows again in
    // batches (their loads issued together per pass)
    __syncthreads();
    for (int i = tid; i < kk; i += kAT) mx = fmaxf(mx, logits[i]);
    {
      float m = mx;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) fred[warp] = m;
      __syncthreads();
      m = fred[0];
      for (int w = 1; w < kAW; ++w) m = fmaxf(m, fred[w]);
      __syncthreads();
      mx = m;
    }
    for (int i = tid; i < kk; i += kAT) {
      const float e = expf(logits[i] - mx);
      logits[i] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) fred[warp] = sum;
    __syncthreads();
    {
      float s2 = 0.f;
      for (int w = 0; w < kAW; ++w) s2 += fred[w];
      sum = s2;
    }
    for (int ps = 0; ps < npass; ++ps) {
      const int i0 = ps * kAW * SPW + warp;
      Lane<BF16, EPL> vr[SPW];
#pragma unroll
      for (int u = 0; u < SPW; ++u) {
        const int i = i0 + u * kAW;
        if (i < kk) vr[u].load(p.V, (head * p.Tmax + sel[i]) * p.dh + (int64_t)lane * EPL);
      }
#pragma unroll
      for (int u = 0; u < SPW; ++u) {
        const int i = i0 + u * kAW;
        if (i < kk) {
          const float wgt = logits[i];
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wgt, vr[u].get(e), acc[e]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) part[warp * p.dh + lane * EPL + e] = acc[e];
  __syncthreads();
  for (int d = tid; d < p.dh; d += kAT) {
    float s2 = 0.f;
    for (int w = 0; w < kAW; ++w) s2 += part[w * p.dh + d];
    out[d] = s2 / sum;
  }
}

// label[b][g][t][j] = K[b][g][t][channels[g][j]] for t0 <= t < t1 (and t < seq_len[b])
__global__ void k_ds_label_build(const void* __restrict__ K, int kdt, int B, int Hkv, int Tmax, int dh,
                                 const int32_t* __restrict__ seq_len, const int32_t* __restrict__ channels, int r,
                                 int t0, int t1, void* __restrict__ label) {
  const int64_t per_head = (int64_t)(t1 - t0) * r;
  const int64_t total = (int64_t)B * Hkv * per_head;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t head = e / per_head;
    const int64_t rem = e - head * per_head;
    const int t = t0 + (int)(rem / r), j = (int)(rem % r);
    const int b = (int)(head / Hkv), g = (int)(head % Hkv);
    if (t >= __ldg(seq_len + b)) continue;
    const int64_t src = (head * Tmax + t) * dh + __ldg(channels + (int64_t)g * r + j);
    const int64_t dst = (head * Tmax + t) * r + j;
    if (kdt == WINA_BF16)
      reinterpret_cast<uint16_t*>(label)[dst] = reinterpret_cast<const uint16_t*>(K)[src];
    else
      reinterpret_cast<float*>(label)[dst] = reinterpret_cast<const float*>(K)[src];
  }
}

// absmean[g][c] = mean over every sequence's valid tokens of |K[b][g][t][c]|: one CTA per
// (g, c), float64 sums in a fixed order (thread strides, then a fixed tree), rounded
// once to float32.
__global__ void __launch_bounds__(256) k_ds_absmean(const void* __restrict__ K, int kdt, int B, int Hkv, int Tmax,
                                                    int dh, const int32_t* __restrict__ seq_len,
                                                    float* __restrict__ absmean) {
  __shared__ double red[8];
  const int g = blockIdx.x / dh, c = blockIdx.x % dh;
  double s = 0.0;
  long long cnt = 0;
  for (int b = 0; b < B; ++b) {
    const int T = min(max(__ldg(seq_len + b), 0), Tmax);
    cnt += T;
    const int64_t base = ((int64_t)b * Hkv + g) * Tmax * dh + c;
    for (int t = threadIdx.x; t < T; t += 256) s += fabs((double)load_elem(K, kdt, base + (int64_t)t * dh));
  }
  const double tot = block_sum_f64<256>(s, red);
  if (threadIdx.x == 0) absmean[(int64_t)g * dh + c] = cnt > 0 ? (float)(tot / (double)cnt) : 0.f;
}

}  // namespace wina

using namespace wina;

static bool ds_dtype_ok(wina_dtype_t t) { return t == WINA_BF16 || t == WINA_F32; }

extern "C" wina_status_t ds_channel_absmean(const void* K, wina_dtype_t kdt, int64_t B, int64_t Hkv, int64_t Tmax,
                                            int64_t dh, const int32_t* seq_len, float* absmean,
                                            wina_stream_t stream) {
  if (!ds_dtype_ok(kdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (B < 1 || Hkv < 1 || Tmax < 1 || dh < 1 || B * Hkv * Tmax * dh > ((int64_t)1 << 40) || Hkv * dh > INT32_MAX)
    return WINA_ERR_INVALID_ARG;
  if (!K || !seq_len || !absmean || !aligned(K, elem_size(kdt)) || !aligned(absmean, 4) || !aligned(seq_len, 4))
    return WINA_ERR_INVALID_ARG;
  k_ds_absmean<<<(unsigned)(Hkv * dh), 256, 0, (cudaStream_t)stream>>>(K, kdt, (int)B, (int)Hkv, (int)Tmax, (int)dh,
                                                                       seq_len, absmean);
  return cuda_status(cudaGetLastError());
}

extern "C" wina_status_t ds_label_build(const void* K, wina_dtype_t kdt, int64_t B, int64_t Hkv, int64_t Tmax,
                                        int64_t dh, const int32_t* seq_len, const int32_t* channels, int64_t r,
                                        int64_t t0, int64_t t1, void* label, wina_stream_t stream) {
  if (!ds_dtype_ok(kdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  if (B < 1 || Hkv < 1 || Tmax < 1 || dh < 1 || r < 1 || r > dh || t0 < 0 || t1 > Tmax || t0 > t1 ||
      Tmax > INT32_MAX || B * Hkv * Tmax * dh > ((int64_t)1 << 40))
    return WINA_ERR_INVALID_ARG;
  if (!K || !seq_len || !channels || !label || !aligned(K, elem_size(kdt)) || !aligned(label, elem_size(kdt)))
    return WINA_ERR_INVALID_ARG;
  if (t0 == t1) return WINA_OK;
  const int64_t total = B * Hkv * (t1 - t0) * r;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)device_sm_count() * 8);
  k_ds_label_build<<<grid, 256, 0, (cudaStream_t)stream>>>(K, kdt, (int)B, (int)Hkv, (int)Tmax, (int)dh, seq_len,
                                                           channels, (int)r, (int)t0, (int)t1, label);
  return cuda_status(cudaGetLastError());
}

extern "C" size_t ds_decode_smem_bytes(int64_t Tmax, int64_t dh, int64_t k) {
  if (Tmax < 1 || dh < 1 || k < 0) return 0;
  const int64_t kcap = std::min(k, Tmax);
  return (size_t)(Tmax + 2 * kcap + kSelBins + 2 * kSelCand + dh + kAW * dh) * 4;
}

extern "C" wina_status_t ds_decode_attention(const void* q, wina_dtype_t qdt, const void* K, const void* V,
                                             const void* label, wina_dtype_t kvdt, const int32_t* channels,
                                             int64_t B, int64_t Hq, int64_t Hkv, int64_t Tmax, int64_t dh, int64_t r,
                                             const int32_t* seq_len, int64_t k, float scale, float* out,
                                             int32_t* idx_out, float* scores_out, int32_t* status_dev,
                                             wina_stream_t stream) {
  if (!ds_dtype_ok(qdt) || !ds_dtype_ok(kvdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int vec = kvdt == WINA_BF16 ? 8 : 4;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || Tmax < 1 || Tmax > INT32_MAX || k < 0) return WINA_ERR_INVALID_ARG;
  if (dh != 32 && dh != 64 && dh != 128 && dh != 256) return WINA_ERR_INVALID_ARG;  // 1, 2, 4 or 8 per lane
  if (r < 1 || r > dh || r % vec) return WINA_ERR_INVALID_ARG;
  if (B * Hq > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (!q || !K || !V || !label || !channels || !seq_len || !out) return WINA_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(label, 16) || !aligned(q, elem_size(qdt)) || !aligned(out, 4) ||
      (idx_out && !aligned(idx_out, 4)) || (scores_out && !aligned(scores_out, 4)) ||
      (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  DsParams p;
  p.q = q;
  p.qdt = qdt;
  p.K = K;
  p.V = V;
  p.label = label;
  p.kvdt = kvdt;
  p.channels = channels;
  p.seq_len = seq_len;
  p.B = (int)B;
  p.Hq = (int)Hq;
  p.Hkv = (int)Hkv;
  p.Tmax = (int)Tmax;
  p.dh = (int)dh;
  p.r = (int)r;
  p.k = (int)std::min<int64_t>(k, INT32_MAX);
  p.scale = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)dh));
  p.out = out;
  p.idx_out = idx_out;
  p.scores_out = scores_out;
  p.status = status_dev;
  const size_t smem = ds_decode_smem_bytes(Tmax, dh, k);
  if (smem > kDsMaxSmem) return WINA_ERR_INVALID_ARG;  // Tmax and min(k, Tmax) too large together
  void (*kern)(DsParams) = nullptr;
  const bool bf = kvdt == WINA_BF16;
  switch (dh) {
    case 32: kern = bf ? k_ds_decode<true, 1> : k_ds_decode<false, 1>; break;
    case 64: kern = bf ? k_ds_decode<true, 2> : k_ds_decode<false, 2>; break;
    case 128: kern = bf ? k_ds_decode<true, 4> : k_ds_decode<false, 4>; break;
    default: kern = bf ? k_ds_decode<true, 8> : k_ds_decode<false, 8>; break;
  }
  {
    // always: the kernel's static shared memory comes on top of the dynamic part
    const cudaError_t e = ensure_smem_limit((const void*)kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
  }
  kern<<<(unsigned)(B * Hq), kAT, smem, (cudaStream_t)stream>>>(p);
  return cuda_status(cudaGetLastError());
}
