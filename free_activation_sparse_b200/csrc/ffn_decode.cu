// Single-token SwiGLU FFN decode with the gate on every projection ("WAS" article, core
// innovations: the gate is applied per component, gate/up/down among them; "WINA"
// article, section 一: each projection scores with the column norms of its own weight and
// keeps its own K; "Spark Transformer", section 2.2: the statistical threshold variant).
//
// One persistent cooperative launch, one CTA of 1024 threads per SM, little shared
// memory, so that most of each SM's L1 is free to hold the weight loads in flight. The
// sparse products are split over the grid in two dimensions (colstream.cuh): column groups
// of the output times row groups of the kept rows, so that each output column has only a
// few partial sums, added by the last CTA of its column group.
//   A  Every CTA scores x against its projection's c with the keys held in registers
//      (thread t owns channels t, t + 1024, ...), finds the kept set by a radix select on
//      the float32 key bits (histogram of the top 12 bits, then 8, 8 and 3 bits only while
//      needed; equal keys resolved by index), and lists the kept channels of its row
//      group: those whose rank in ascending channel order is congruent to it.
//   B  Column group cg of the ffn outputs has RG_g gate and RG_u up CTAs. Each streams the
//      cg slice of its listed rows (16-byte read-only loads, several rows in flight per
//      thread), times x, into a partial row of those columns. The last of the group's CTAs
//      to finish adds the partials of g and of u in row-group order and writes h =
//      silu(g) * u and the down scores |h * c_down| for the slice.
//   -- grid barrier --
//   C2 Every CTA loads all down scores into registers, selects and lists the down rows of
//      its row group the same way.
//   E  Column group cg of the d outputs has RG_e CTAs; each streams its slice of its rows
//      times h, and the group's last CTA adds the RG_e partials in order into y.
// The one wait (the grid barrier) has a time limit. Selections are exact and identical on
// every CTA, and every sum is taken in a fixed order, so the results are bit-reproducible.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "colstream.cuh"
#include "regsel.cuh"

namespace wina {


struct DecodeParams {
  const void* wt_gate;
  const void* wt_up;
  const void* wt_down;
  const float* c_gate;
  const float* c_up;
  const float* c_down;
  const void* x;
  int xdt;
  int d, ffn;
  int mode;
  int k_gate, k_up, k_down;
  double z;
  float* y;
  int cgb, rgg, rgu;  // phase B: column groups of ffn; gate and up row groups per column group
  int cge, rge;       // phase E: column groups of d; row groups per column group
  int list_cap;       // list entries per CTA at most
  uint32_t sm_flags, sm_wpre, sm_lrow;  // SMEM offsets (the histogram is at 0)
  GridBarrier* bar;
  unsigned long long wait_ns;  // time limit of the barrier wait
  float* part;      // partial rows [rgg + rgu + rge][pstride] float32: g, u, then y
  int pstride;      // floats per partial row (>= max(d, ffn), a multiple of 4)
  unsigned* groups;  // [cgb] then [cge] arrival counters of the column groups (zero between calls)
  uint32_t* dkeys;  // [ffn] down-gate scores (float32 bits), written by column group
  float* h;
  uint8_t* keep_g;
  uint8_t* keep_u;
  uint8_t* keep_d;
  long long* stamps;
  unsigned long long* cta_t;
  int32_t* status;
};

// Dynamic SMEM: hist [kSelBins + 256] | flags [nw] | word prefix [nw] | list rows [cap];
// the streams' pass sums (red, kCT * 4 floats) overlay hist.
struct DecodeSmem {
  uint32_t hist, flags, wpre, lrow, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int n_max, int cap) {
  DecodeSmem L;
  const uint32_t nw = (uint32_t)(n_max + 31) / 32;
  const uint32_t hist_bytes = (uint32_t)(kSelBins + 256) * 4u;
  const uint32_t red_bytes = (uint32_t)kCT * 16u;
  uint32_t o = 0;
  L.hist = o;
  o += (hist_bytes > red_bytes ? hist_bytes : red_bytes);
  o = (o + 15u) & ~15u;
  L.flags = o;
  o += nw * 4u;
  o = (o + 15u) & ~15u;
  L.wpre = o;
  o += nw * 4u;
  o = (o + 15u) & ~15u;
  L.lrow = o;
  o += (uint32_t)cap * 4u;
  L.total = (o + 127u) & ~127u;
  return L;
}

__device__ __forceinline__ float silu_d(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ void dstamp(long long* s, int i) {
  if (blockIdx.x == 0 && threadIdx.x == 0) s[i] = clock64();
}
__device__ __forceinline__ void dcta_time(unsigned long long* t, int i) {
  if (threadIdx.x == 0) t[blockIdx.x * 4 + i] = globaltimer_ns();
}

// Spark's statistical threshold on the CTA's n values (thread t holds v[i] = element
// t + i * kDT): mu = mean, sigma^2 = mean of (v - mu)^2 (two passes over the registers,
// float64 sums), kept = v > mu + sigma z, as flag words.
template <int KMAX>
__device__ __forceinline__ void flags_from_stat(const float (&v)[KMAX], int kpt, int n, double z,
                                                uint32_t* flags) {
  __shared__ double dred[kDW];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < KMAX; ++i)
    if (i < kpt && t + i * kDT < n) s += (double)v[i];
  const double mu = block_sum_f64<kDT>(s, dred) / (double)n;
  double q = 0.0;
#pragma unroll
  for (int i = 0; i < KMAX; ++i)
    if (i < kpt && t + i * kDT < n) {
      const double dl = (double)v[i] - mu;
      q += dl * dl;
    }
  const double var = block_sum_f64<kDT>(q, dred) / (double)n;
  const double th = mu + sqrt(var) * z;
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    if (i < kpt) {
      const int j = t + i * kDT;
      const bool k = j < n && (double)v[i] > th;
      const uint32_t bits = __ballot_sync(0xffffffffu, k);
      const int w = i * kDW + warp;
      if (lane == 0 && w < (n + 31) / 32) flags[w] = bits;
    }
  }
}

__device__ __forceinline__ void flags_all_d(int n, uint32_t* flags) {
  const int nw = (n + 31) / 32;
  for (int w = threadIdx.x; w < nw; w += kDT) {
    const int rem = n - w * 32;
    flags[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  }
}

// This CTA's rows: the kept channels whose rank (ascending channel order) is congruent
// to `part` modulo `parts`, in ascending order, into lrow[0..count). The flag words'
// exclusive prefix counts go to wpre; each listed rank is then found by a binary search
// over the words and the position of its set bit within the word. Returns the count
// (capped at cap; WINA_ERR_CAPACITY is recorded if it does not fit).
__device__ int list_rows(const uint32_t* flags, int n, int parts, int part, uint32_t* wpre, int* lrow, int cap,
                         int32_t* status) {
  __shared__ uint32_t red[kDW + 1];
  __shared__ uint32_t s_total;
  const int t = threadIdx.x;
  const int nw = (n + 31) / 32;  // <= kDMaxN / 32 = 512 < kDT: one word per thread
  const uint32_t f = t < nw ? flags[t] : 0u;
  uint32_t tot;
  const uint32_t pre = block_excl_scan<kDT>((uint32_t)__popc(f), red, &tot);
  if (t < nw) wpre[t] = pre;
  if (t == 0) s_total = tot;
  __syncthreads();
  const uint32_t total = s_total;
  int cnt = (int)total > part ? (int)((total - (uint32_t)part + (uint32_t)parts - 1u) / (uint32_t)parts) : 0;
  if (cnt > cap) {
    if (t == 0) record_status(status, WINA_ERR_CAPACITY);
    cnt = cap;
  }
  for (int i = t; i < cnt; i += kDT) {
    const uint32_t rank = (uint32_t)part + (uint32_t)i * (uint32_t)parts;
    int lo = 0, hi = nw - 1;  // the last word whose prefix count is <= rank holds it
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (wpre[mid] <= rank) lo = mid;
      else hi = mid - 1;
    }
    lrow[i] = lo * 32 + (int)__fns(flags[lo], 0u, (int)(rank - wpre[lo]) + 1);
  }
  __syncthreads();
  return cnt;
}

__device__ __forceinline__ void touch_pages_d(const void* p, size_t bytes) {
  const char* c = reinterpret_cast<const char*>(p);
  for (size_t o = (size_t)threadIdx.x << 21; o < bytes; o += (size_t)kDT << 21)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(c + o));
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------

// KA / KC: channels per thread of x (d) and of h (ffn), at most.
template <bool BF16, int KA, int KC>
__global__ void __launch_bounds__(kDT, 1) k_ffn_decode(DecodeParams a) {
  constexpr uint32_t ESZ = BF16 ? 2u : 4u;
  constexpr int EPV = VecOps<BF16>::EPV;
  constexpr int U = 4;  // rows in flight per thread
  extern __shared__ __align__(128) unsigned char smraw[];
  const int d = a.d, ffn = a.ffn;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smraw);
  float* red = reinterpret_cast<float*>(smraw);  // overlays hist while streaming
  uint32_t* flags = reinterpret_cast<uint32_t*>(smraw + a.sm_flags);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smraw + a.sm_wpre);
  int* lrow = reinterpret_cast<int*>(smraw + a.sm_lrow);
  const int G = gridDim.x, b = blockIdx.x, t = threadIdx.x;
  const uint64_t pol = l2_evict_first_policy();
  dstamp(a.stamps, 0);
  clear_hist(hist);  // for the first selection (the loads of x and c are in flight meanwhile)

  // ---------------- A: this CTA's projection, its kept set, its rows ----------------
  const int rgs = a.rgg + a.rgu;
  const bool inb = b < a.cgb * rgs;             // CTAs beyond the phase-B grid only wait
  const int cgb = b % a.cgb, kb = b / a.cgb;    // column group; row group among gate then up
  const bool gate = kb < a.rgg;
  const int parts = gate ? a.rgg : a.rgu;
  const int part = gate ? kb : kb - a.rgg;
  const void* wt = gate ? a.wt_gate : a.wt_up;
  const int kpt_a = (d + kDT - 1) / kDT;
  if (a.mode == WINA_GATE_TOPK) {
    const float* c = gate ? a.c_gate : a.c_up;
    uint32_t key[KA];
#pragma unroll
    for (int i = 0; i < KA; ++i) {
      const int j = t + i * kDT;
      key[i] = 0u;
      if (i < kpt_a && j < d) key[i] = __float_as_uint(fabsf(load_elem(a.x, a.xdt, j) * __ldg(c + j)));
    }
    touch_pages_d(wt, (size_t)d * ffn * ESZ);
    __syncthreads();  // the histogram is zero
    dstamp(a.stamps, 1);
    const Threshold th = radix_select_regs(key, kpt_a, d, gate ? a.k_gate : a.k_up, hist);
    dstamp(a.stamps, 2);
    flags_from_keys(key, kpt_a, d, th, flags);
  } else if (a.mode == WINA_GATE_STAT) {
    float v[KA];
#pragma unroll
    for (int i = 0; i < KA; ++i) {
      const int j = t + i * kDT;
      v[i] = (i < kpt_a && j < d) ? load_elem(a.x, a.xdt, j) : 0.f;
    }
    touch_pages_d(wt, (size_t)d * ffn * ESZ);
    flags_from_stat(v, kpt_a, d, a.z, flags);
  } else {
    touch_pages_d(wt, (size_t)d * ffn * ESZ);
    flags_all_d(d, flags);
  }
  __syncthreads();
  int cnt = inb ? list_rows(flags, d, parts, part, wpre, lrow, a.list_cap, a.status) : 0;
  if (inb && cgb == 0 && part == parts - 1) {
    uint8_t* kbytes = gate ? a.keep_g : a.keep_u;
    for (int j = t; j < d; j += kDT) kbytes[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
  }
  dstamp(a.stamps, 3);
  dcta_time(a.cta_t, 0);

  // ---------------- B: this CTA's column slice of its rows; the group's last adds up ----------------
  if (inb) {
    const int Vb = ffn * (int)ESZ / 16;
    const int v0 = (int)((int64_t)Vb * cgb / a.cgb), nv = (int)((int64_t)Vb * (cgb + 1) / a.cgb) - v0;
    float out[EPV];
    stream_cols<BF16, U>(wt, Vb, v0, nv, cnt, [&](int i) { return lrow[i]; },
                         [&](int i) { return load_elem(a.x, a.xdt, lrow[i]); }, red, pol, out);
    dstamp(a.stamps, 4);
    if (t == 0) a.cta_t[b * 4 + 1] = globaltimer_ns();
    if (t < nv) {
      float4* o = reinterpret_cast<float4*>(a.part + (size_t)kb * a.pstride + (size_t)(v0 + t) * EPV);
#pragma unroll
      for (int q = 0; q < EPV / 4; ++q) __stcg(o + q, make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]));
    }
    dstamp(a.stamps, 5);
    // h and the down scores of the slice, if this CTA is its group's last: float4 columns
    // [q0, q0 + nq); the first down-gate norms are read before the arrival
    const int q0 = v0 * EPV / 4, nq = nv * EPV / 4;
    float4 c4t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < nq && a.mode == WINA_GATE_TOPK) c4t = __ldg(reinterpret_cast<const float4*>(a.c_down) + q0 + t);
    touch_pages_d(a.wt_down, (size_t)d * ffn * ESZ);
    if (group_arrive_last(a.groups + cgb, rgs)) {
      for (int i = t; i < nq; i += kDT) {
        const int q = q0 + i;
        float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f), u4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < a.rgg; ++r) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part + (size_t)r * a.pstride) + q);
          g4.x += v.x; g4.y += v.y; g4.z += v.z; g4.w += v.w;
        }
        for (int r = 0; r < a.rgu; ++r) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part + (size_t)(a.rgg + r) * a.pstride) + q);
          u4.x += v.x; u4.y += v.y; u4.z += v.z; u4.w += v.w;
        }
        const float4 h4 = make_float4(silu_d(g4.x) * u4.x, silu_d(g4.y) * u4.y, silu_d(g4.z) * u4.z,
                                      silu_d(g4.w) * u4.w);
        __stcg(reinterpret_cast<float4*>(a.h) + q, h4);
        if (a.mode == WINA_GATE_TOPK) {
          const float4 c4 = i == t ? c4t : __ldg(reinterpret_cast<const float4*>(a.c_down) + q);
          __stcg(reinterpret_cast<uint4*>(a.dkeys) + q,
                 make_uint4(__float_as_uint(fabsf(h4.x * c4.x)), __float_as_uint(fabsf(h4.y * c4.y)),
                            __float_as_uint(fabsf(h4.z * c4.z)), __float_as_uint(fabsf(h4.w * c4.w))));
        }
      }
    }
  }
  dstamp(a.stamps, 6);
  clear_hist(hist);  // for the down selection (red overlays it)
  dstamp(a.stamps, 7);
  if (!grid_sync_fixed(a.bar, G, a.status, a.wait_ns)) return;
  dstamp(a.stamps, 8);

  // ---------------- C2: the down kept set and this CTA's rows ----------------
  const bool ine = b < a.cge * a.rge;
  const int cge = b % a.cge, rge = b / a.cge;
  const int kpt_c = (ffn + kDT - 1) / kDT;
  if (a.mode == WINA_GATE_TOPK) {
    uint32_t key[KC];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
      const int j = t + i * kDT;
      key[i] = (i < kpt_c && j < ffn) ? __ldcg(a.dkeys + j) : 0u;
    }
    dstamp(a.stamps, 9);
    const Threshold th = radix_select_regs(key, kpt_c, ffn, a.k_down, hist);
    dstamp(a.stamps, 10);
    flags_from_keys(key, kpt_c, ffn, th, flags);
  } else if (a.mode == WINA_GATE_STAT) {
    float hv[KC];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
      const int j = t + i * kDT;
      hv[i] = (i < kpt_c && j < ffn) ? __ldcg(a.h + j) : 0.f;
    }
    flags_from_stat(hv, kpt_c, ffn, a.z, flags);
  } else {
    flags_all_d(ffn, flags);
  }
  __syncthreads();
  cnt = ine ? list_rows(flags, ffn, a.rge, rge, wpre, lrow, a.list_cap, a.status) : 0;
  if (b == G - 1)
    for (int j = t; j < ffn; j += kDT) a.keep_d[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
  dstamp(a.stamps, 11);
  dcta_time(a.cta_t, 2);

  // ---------------- E: this CTA's column slice of its down rows; the group's last sums y ----------------
  if (!ine) return;
  const int Ve = d * (int)ESZ / 16;
  const int v0 = (int)((int64_t)Ve * cge / a.cge), nv = (int)((int64_t)Ve * (cge + 1) / a.cge) - v0;
  float out[EPV];
  stream_cols<BF16, U>(a.wt_down, Ve, v0, nv, cnt, [&](int i) { return lrow[i]; },
                       [&](int i) { return __ldcg(a.h + lrow[i]); }, red, pol, out);
  dstamp(a.stamps, 12);
  if (t == 0) a.cta_t[b * 4 + 3] = globaltimer_ns();
  float* pe = a.part + (size_t)rgs * a.pstride;  // the row groups' partial rows of y
  if (t < nv) {
    float4* o = reinterpret_cast<float4*>(pe + (size_t)rge * a.pstride + (size_t)(v0 + t) * EPV);
#pragma unroll
    for (int q = 0; q < EPV / 4; ++q) __stcg(o + q, make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]));
  }
  dstamp(a.stamps, 13);
  const bool last = group_arrive_last(a.groups + a.cgb + cge, a.rge);
  dstamp(a.stamps, 14);
  if (last) {  // y over the slice: the group's partial rows added in row-group order
    const int q0 = v0 * EPV / 4, nq = nv * EPV / 4;
    for (int i = t; i < nq; i += kDT) {
      float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = 0; r < a.rge; ++r) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(pe + (size_t)r * a.pstride) + q0 + i);
        s4.x += v.x; s4.y += v.y; s4.z += v.z; s4.w += v.w;
      }
      reinterpret_cast<float4*>(a.y)[q0 + i] = s4;
    }
  }
  dstamp(a.stamps, 15);
}

// Instantiations: the channel counts of the workloads' decode shapes fixed at compile time
// (the keys held in registers: 4 per thread for d <= 4096, 12 or 16 for ffn); every other
// shape up to 16384 channels takes the general one.
static void* decode_kernel_for(bool bf16, int ka, int kc) {
  if (bf16) {
    if (ka <= 4 && kc <= 12) return (void*)k_ffn_decode<true, 4, 12>;  // Llama-7B, Gemma-2-2B
    if (ka <= 4 && kc <= 16) return (void*)k_ffn_decode<true, 4, 16>;  // Llama-3-8B
    return (void*)k_ffn_decode<true, 16, 16>;
  }
  return (void*)k_ffn_decode<false, 16, 16>;
}

// Launch the single-token kernel if it takes this shape; returns WINA_ERR_UNSUPPORTED_DTYPE
// (no launch) when it does not, so that the caller can use the batched path.
wina_status_t launch_ffn_decode(const wina_ffn_t* f, const void* x, int xdt, int mode, int k_gate, int k_up,
                                int k_down, double z, float* y, const FfnWs& L, char* w, int32_t* status,
                                cudaStream_t st) {
  const bool bf16 = f->wdt == WINA_BF16;
  const int esz = bf16 ? 2 : 4;
  const int d = (int)f->d, ffn = (int)f->ffn;
  if (d > kDMaxN || ffn > kDMaxN) return WINA_ERR_UNSUPPORTED_DTYPE;
  void* kern = decode_kernel_for(bf16, (d + kDT - 1) / kDT, (ffn + kDT - 1) / kDT);
  const int sms = device_sm_count();
  const int G = std::min(sms, kGridCap);
  if (G < 8) return WINA_ERR_UNSUPPORTED_DTYPE;
  // phase B: four row groups per column group (slices of 37 vectors of a Llama-7B row),
  // split between gate and up in proportion to their kept rows (two each when unknown)
  const int rgs = 4;  // row groups per column group in phase B
  int rgg = rgs / 2;
  if (mode == WINA_GATE_TOPK && k_gate + k_up > 0)
    rgg = (int)((rgs * (int64_t)k_gate + (k_gate + k_up) / 2) / (k_gate + k_up));
  rgg = std::max(1, std::min(rgs - 1, rgg));
  const int rgu = rgs - rgg;
  const int cgb = G / rgs;
  // phase E: slices of about 64 vectors (1 KB), at most 16 row groups (8 x 16 CTAs for
  // Llama-7B's d = 4096; 16 x 9 slices of 512 B streamed slower)
  const int cge = std::max(1, std::min(G / 4, d * esz / 16 / 64));
  const int rge = std::min(16, G / cge);
  const int V_b = ffn * esz / 16, V_e = d * esz / 16;
  if ((V_b + cgb - 1) / cgb > kCT || (V_e + cge - 1) / cge > kCT || V_b < cgb || V_e < cge)
    return WINA_ERR_UNSUPPORTED_DTYPE;
  const int nmax = std::max(d, ffn);
  const int cap = std::max((d + std::min(rgg, rgu) - 1) / std::min(rgg, rgu), (ffn + rge - 1) / rge) + 1;
  const DecodeSmem SL = decode_smem(nmax, cap);
  const size_t smem = SL.total;
  if (smem > 96 * 1024) return WINA_ERR_UNSUPPORTED_DTYPE;  // keep most of the L1 for the loads in flight
  if (rgg + rgu + rge > kDecodeRows) return WINA_ERR_UNSUPPORTED_DTYPE;
  {
    cudaError_t e = ensure_smem_limit(kern, smem);  // static shared memory comes on top of the dynamic part
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (blocks_per_sm(kern, kDT, smem) < 1) return WINA_ERR_UNSUPPORTED_DTYPE;
  DecodeParams p;
  p.wt_gate = f->wt_gate;
  p.wt_up = f->wt_up;
  p.wt_down = f->wt_down;
  p.c_gate = f->c_gate;
  p.c_up = f->c_up;
  p.c_down = f->c_down;
  p.x = x;
  p.xdt = xdt;
  p.d = d;
  p.ffn = ffn;
  p.mode = mode;
  p.k_gate = k_gate;
  p.k_up = k_up;
  p.k_down = k_down;
  p.z = z;
  p.y = y;
  p.cgb = cgb;
  p.rgg = rgg;
  p.rgu = rgu;
  p.cge = cge;
  p.rge = rge;
  p.list_cap = cap;
  p.sm_flags = SL.flags;
  p.sm_wpre = SL.wpre;
  p.sm_lrow = SL.lrow;
  p.bar = reinterpret_cast<GridBarrier*>(w + L.bar);
  p.wait_ns = wait_limit_ns();
  p.part = reinterpret_cast<float*>(w + L.part);
  p.pstride = (int)L.pstride;
  p.groups = reinterpret_cast<unsigned*>(w + L.groups);
  p.dkeys = reinterpret_cast<uint32_t*>(w + L.dkeys);
  p.h = reinterpret_cast<float*>(w + L.h);
  p.keep_g = reinterpret_cast<uint8_t*>(w + L.keep_g);
  p.keep_u = reinterpret_cast<uint8_t*>(w + L.keep_u);
  p.keep_d = reinterpret_cast<uint8_t*>(w + L.keep_d);
  p.stamps = reinterpret_cast<long long*>(w + L.stamps);
  p.cta_t = reinterpret_cast<unsigned long long*>(w + L.cta_t);
  p.status = status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)G);
  cfg.blockDim = dim3(kDT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    cudaError_t e = ensure_prefer_l1(kern);  // the weight loads in flight live in L1
    if (e != cudaSuccess) return cuda_status(e);
  }
  void* args[] = {&p};
  return cuda_status(cudaLaunchKernelExC(&cfg, kern, args));
}

}  // namespace wina
