// Single-token SwiGLU FFN decode with the gate on every projection ("WAS" article, core
// innovations: the gate is applied per component, gate/up/down among them; "WINA"
// article, section 一: each projection scores with the column norms of its own weight and
// keeps its own K; "Spark Transformer", section 2.2: the statistical threshold variant).
//
// One persistent cooperative launch, one CTA of 1024 threads per SM, little shared
// memory, so that most of each SM's L1 is free to hold the weight loads in flight:
//   A  CTAs [0, Gg) take the gate projection, the rest up. Every CTA scores x against its
//      projection's c with the keys held in registers (thread t owns channels
//      t, t + 1024, ...), finds the kept set by a radix select on the float32 key bits
//      (histogram of the top 12 bits, then 8, 8 and 3 bits only while needed; equal keys
//      resolved by index), and lists the kept channels whose rank r in ascending channel
//      order satisfies r mod parts == its part: the kept rows are dealt out round robin,
//      so at any moment all SMs read rows from the same neighbourhood of the weight.
//   B  The CTA streams its rows with 16-byte read-only loads (several rows in flight per
//      thread), accumulates x_j * row_j in float32 registers and stores its partial row
//      of g or u (plain stores: float atomics from every SM onto the same addresses
//      serialise in L2 for microseconds).
//   -- grid barrier --
//   C1 CTA b sums its slice of the channels over all partial rows in a fixed order and
//      writes h = silu(g) * u and the down scores |h * c_down| for that slice.
//   -- grid barrier --
//   C2 Every CTA loads all down scores into registers, selects and lists its share of
//      the down rows the same way.
//   E  Streams them into its partial row of y.
//   -- grid barrier --
//   E2 CTA b sums its slice of y over the partial rows in a fixed order.
// Every wait is a grid barrier with a time limit. Selections are exact and identical on
// every CTA, and every sum is taken in a fixed order, so the results are bit-reproducible.
#include <math.h>

#include <algorithm>

#include "internal.h"
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
  int Gg;        // CTAs on the gate projection
  int list_cap;  // rows per CTA list
  uint32_t sm_flags, sm_wpre, sm_lrow;  // SMEM offsets (the histogram is at 0)
  GridBarrier* bar;
  unsigned long long wait_ns;  // time limit of each barrier wait
  float* part;      // [G][pstride] float32 partial rows (g / u in phase B, y in phase E)
  int pstride;      // floats per partial row (>= max(d, ffn), a multiple of 4)
  uint32_t* dkeys;  // [ffn] down-gate scores (float32 bits), written in slices in C1
  float* h;
  uint8_t* keep_g;
  uint8_t* keep_u;
  uint8_t* keep_d;
  long long* stamps;
  unsigned long long* cta_t;
  int32_t* status;
};

// Dynamic SMEM: hist [kSelBins + 256] | flags [nw] | word prefix [nw] | list rows [cap];
// the group and slice reductions (red) overlay hist.
struct DecodeSmem {
  uint32_t hist, flags, wpre, lrow, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int n_max, int cap, int red_floats) {
  DecodeSmem L;
  const uint32_t nw = (uint32_t)(n_max + 31) / 32;
  const uint32_t hist_bytes = (uint32_t)(kSelBins + 256) * 4u;
  const uint32_t red_bytes = (uint32_t)red_floats * 4u;
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

// Threads per row and row groups of a row of V 16-byte vectors: rows of more than 256
// vectors take 512 threads (two groups), shorter rows a power of two >= V.
__host__ __device__ inline int decode_tpr(int V) {
  int t = 32;
  while (t < V && t < kDT / 2) t <<= 1;
  return t;
}

__device__ __forceinline__ float silu_d(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

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

// ------------------------------------------------------------------------------------
// streaming the listed rows
// ------------------------------------------------------------------------------------

// This CTA's partial row(s) of sum over the listed rows r of val(lrow[r], r) *
// Wt[lrow[r]][0..m), read with 16-byte loads, stored in `part` (row stride pstride floats).
// The CTA is split into NG = kDT / TPR groups of TPR threads; group g takes list entries
// g, g + NG, ...; thread l of a group owns VPT vectors of each row, those of index l,
// l + TPR, ... rotated by an offset that differs from CTA to CTA. Rows are loaded U at a
// time, with DB into two register buffers in turn so that the next rows are in flight
// while the current ones are multiplied; the last batch is predicated (no row-by-row
// tail). A row's input value val(channel) is loaded with its weights. The groups' sums
// are stored as partial rows blockIdx.x * P + g (P = decode_partials(V) = 2 when two
// groups of 512 threads take the rows), or, with more groups, combined in SMEM in group
// order first (red: at least (NG - 1) * TPR * EPV floats) and stored as row blockIdx.x;
// fixed order throughout, so the result is bit-reproducible.
template <bool BF16, int VPT, int U, bool DB, typename Val>
__device__ void stream_rows(const void* __restrict__ Wt, int m, const int* lrow, Val val, int cnt,
                            float* __restrict__ part, int pstride, float* red, uint64_t pol, long long* stamp_loop,
                            unsigned long long* t_loop) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int V = m / EPV;
  const int TPR = decode_tpr(V);
  const int NG = kDT / TPR;
  const int t = threadIdx.x, g = t / TPR, l = t % TPR;
  const uint4* base = reinterpret_cast<const uint4*>(Wt);
  const int rot = (int)(((int64_t)blockIdx.x * V) / gridDim.x);
  int vid[VPT];  // this thread's vectors of a row (-1: none)
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = l + j * TPR;
    vid[j] = v < V ? (v + rot < V ? v + rot : v + rot - V) : -1;
  }
  float acc[VPT][EPV];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[j][e] = 0.f;
  const int mine = cnt > g ? (cnt - g + NG - 1) / NG : 0;  // this group's rows
  uint4 wa[U][VPT], wb[U][VPT];
  float xa[U], xb[U];
  // rows i0 .. i0 + U - 1 of this group (those below `mine`) into (w, xv)
  auto load = [&](uint4 (&w)[U][VPT], float (&xv)[U], int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < mine) {
        const int row = lrow[g + (i0 + u) * NG];
        xv[u] = val(row, g + (i0 + u) * NG);
        const uint4* rp = base + (int64_t)row * V;
#pragma unroll
        for (int j = 0; j < VPT; ++j)
          if (vid[j] >= 0) w[u][j] = ld_stream_u4(rp + vid[j], pol);
      }
    }
  };
  auto consume = [&](const uint4 (&w)[U][VPT], const float (&xv)[U], int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < mine) {
#pragma unroll
        for (int j = 0; j < VPT; ++j)
          if (vid[j] >= 0) VecOps<BF16>::fma(acc[j], w[u][j], xv[u]);
      }
    }
  };
  if (DB) {
    load(wa, xa, 0);
    for (int i0 = 0; i0 < mine; i0 += 2 * U) {
      if (i0 + U < mine) load(wb, xb, i0 + U);
      consume(wa, xa, i0);
      if (i0 + U >= mine) break;
      if (i0 + 2 * U < mine) load(wa, xa, i0 + 2 * U);
      consume(wb, xb, i0 + U);
    }
  } else {
    for (int i0 = 0; i0 < mine; i0 += U) {
      load(wa, xa, i0);
      consume(wa, xa, i0);
    }
  }
  if (t == 0) {
    if (blockIdx.x == 0) *stamp_loop = clock64();
    *t_loop = globaltimer_ns();
  }
  if (NG == 2) {  // each group stores its own partial row (no wait for the other group)
    float* out = part + (size_t)(blockIdx.x * 2 + g) * pstride;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      if (vid[j] >= 0) {
        float4* o = reinterpret_cast<float4*>(out + (int64_t)vid[j] * EPV);
#pragma unroll
        for (int q = 0; q < EPV / 4; ++q)
          __stcg(o + q, make_float4(acc[j][4 * q], acc[j][4 * q + 1], acc[j][4 * q + 2], acc[j][4 * q + 3]));
      }
    }
    return;
  }
  // more (narrower) groups: their sums are combined in SMEM in group order first
  float* out = part + (size_t)blockIdx.x * pstride;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    __syncthreads();
    if (g > 0 && vid[j] >= 0) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) red[((g - 1) * TPR + l) * EPV + e] = acc[j][e];
    }
    __syncthreads();
    if (g == 0 && vid[j] >= 0) {
      for (int gg = 1; gg < NG; ++gg)
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[j][e] += red[((gg - 1) * TPR + l) * EPV + e];
      float4* o = reinterpret_cast<float4*>(out + (int64_t)vid[j] * EPV);
#pragma unroll
      for (int q = 0; q < EPV / 4; ++q)
        __stcg(o + q, make_float4(acc[j][4 * q], acc[j][4 * q + 1], acc[j][4 * q + 2], acc[j][4 * q + 3]));
    }
  }
  __syncthreads();  // red (which overlays the selection histogram) is free again
}

// Partial rows a CTA stores for rows of V vectors: the two row groups of a CTA whose rows
// take 512 threads store one each; narrower rows (more groups) are summed into one.
__host__ __device__ inline int decode_partials(int V) { return decode_tpr(V) == kDT / 2 ? 2 : 1; }

// Reduce-scatter of the partial rows: for this CTA's nq (<= 32) float4 columns
// q0 .. q0 + nq - 1, the sums over rows p in [0, split) and in [split, end) of
// part[p][4q .. 4q + 3]. Warp w reads rows w, w + 32, ... in turn (lane i column q0 + i, so
// that each load instruction takes a few whole cache lines of one row); the warps' sums
// are then added in warp order through SMEM (red: 32 * 32 float4). Fixed order
// throughout, so the result is bit-reproducible. Thread i < nq receives the column's two
// sums. Every thread must call it.
__device__ void reduce_scatter(const float* __restrict__ part, int pstride, int q0, int nq, int split, int end,
                               float4* red, float4* sa, float4* sb) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane < nq) {
    const float4* col = reinterpret_cast<const float4*>(part) + q0 + lane;
    const int rs = pstride / 4;
#pragma unroll 8
    for (int p = warp; p < end; p += 32) {
      const float4 v = __ldcg(col + (size_t)p * rs);
      if (p < split) {  // warp-uniform
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
      } else {
        c.x += v.x; c.y += v.y; c.z += v.z; c.w += v.w;
      }
    }
  }
  float4 r2[2] = {a, c};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && split >= end) break;  // uniform
    red[warp * 32 + lane] = r2[h];
    __syncthreads();
    if (t < nq) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < 32; ++w) {
        const float4 v = red[w * 32 + t];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      if (h == 0) *sa = s;
      else *sb = s;
    }
    __syncthreads();
  }
}

__device__ __forceinline__ void touch_pages_d(const void* p, size_t bytes) {
  const char* c = reinterpret_cast<const char*>(p);
  for (size_t o = (size_t)threadIdx.x << 21; o < bytes; o += (size_t)kDT << 21)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(c + o));
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------

// VB / VE: 16-byte vectors per thread of a gate/up row and of a down row; UB / UE: rows in
// flight per thread; KA / KC: channels per thread of x (d) and of h (ffn), at most.
template <bool BF16, int VB, int UB, int VE, int UE, int KA, int KC>
__global__ void __launch_bounds__(kDT, 1) k_ffn_decode(DecodeParams a) {
  constexpr uint32_t ESZ = BF16 ? 2u : 4u;
  extern __shared__ __align__(128) unsigned char smraw[];
  const int d = a.d, ffn = a.ffn;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smraw);
  float* red = reinterpret_cast<float*>(smraw);  // overlays hist while streaming
  uint32_t* flags = reinterpret_cast<uint32_t*>(smraw + a.sm_flags);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smraw + a.sm_wpre);
  int* lrow = reinterpret_cast<int*>(smraw + a.sm_lrow);
  const int G = gridDim.x, b = blockIdx.x, t = threadIdx.x;
  const uint64_t pol = l2_evict_first_policy();
  const int npb = decode_partials(ffn * (int)ESZ / 16), npe = decode_partials(d * (int)ESZ / 16);
  dstamp(a.stamps, 0);
  clear_hist(hist);  // for the first selection (the loads of x and c are in flight meanwhile)

  // ---------------- A: this CTA's projection, its kept set, its rows ----------------
  const bool gate = b < a.Gg;
  const int parts = gate ? a.Gg : G - a.Gg;
  const int part = gate ? b : b - a.Gg;
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
  int cnt = list_rows(flags, d, parts, part, wpre, lrow, a.list_cap, a.status);
  if (part == parts - 1) {
    uint8_t* kb = gate ? a.keep_g : a.keep_u;
    for (int j = t; j < d; j += kDT) kb[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
  }
  __syncthreads();
  dstamp(a.stamps, 3);
  dcta_time(a.cta_t, 0);

  // ---------------- B: stream the gate / up rows into this CTA's partial row ----------------
  stream_rows<BF16, VB, UB, (VB <= 2)>(wt, ffn, lrow, [&](int j, int) { return load_elem(a.x, a.xdt, j); }, cnt,
                                       a.part, a.pstride, red, pol, a.stamps + 4, a.cta_t + b * 4 + 1);
  dstamp(a.stamps, 5);
  // this CTA's columns of h: float4 columns [qc0, qc0 + nqc); their down-gate norms are
  // read now and used after the barrier
  const int qc0 = (int)((int64_t)(ffn / 4) * b / G);
  const int nqc = (int)((int64_t)(ffn / 4) * (b + 1) / G) - qc0;
  float4 c4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (t < nqc && a.mode == WINA_GATE_TOPK) c4 = __ldg(reinterpret_cast<const float4*>(a.c_down) + qc0 + t);
  if (!grid_sync_fixed(a.bar, G, a.status, a.wait_ns)) return;
  dstamp(a.stamps, 6);

  // ---------------- C1: this CTA's slice of g and u, h and the down scores ----------------
  touch_pages_d(a.wt_down, (size_t)d * ffn * ESZ);
  {
    float4 g4, u4;
    reduce_scatter(a.part, a.pstride, qc0, nqc, a.Gg * npb, G * npb, reinterpret_cast<float4*>(red), &g4,
                             &u4);
    if (t < nqc) {
      const int q = qc0 + t;
      const float4 h4 = make_float4(silu_d(g4.x) * u4.x, silu_d(g4.y) * u4.y, silu_d(g4.z) * u4.z,
                                    silu_d(g4.w) * u4.w);
      __stcg(reinterpret_cast<float4*>(a.h) + q, h4);
      if (a.mode == WINA_GATE_TOPK)
        __stcg(reinterpret_cast<uint4*>(a.dkeys) + q,
               make_uint4(__float_as_uint(fabsf(h4.x * c4.x)), __float_as_uint(fabsf(h4.y * c4.y)),
                          __float_as_uint(fabsf(h4.z * c4.z)), __float_as_uint(fabsf(h4.w * c4.w))));
    }
  }
  clear_hist(hist);  // for the down selection (red overlays it)
  dstamp(a.stamps, 7);
  if (!grid_sync_fixed(a.bar, G, a.status, a.wait_ns)) return;
  dstamp(a.stamps, 8);

  // ---------------- C2: the down kept set and this CTA's rows ----------------
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
  cnt = list_rows(flags, ffn, G, b, wpre, lrow, a.list_cap, a.status);
  if (b == G - 1)
    for (int j = t; j < ffn; j += kDT) a.keep_d[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
  __syncthreads();
  dstamp(a.stamps, 11);
  dcta_time(a.cta_t, 2);

  // ---------------- E: stream the down rows into this CTA's partial row of y ----------------
  stream_rows<BF16, VE, UE, (VE <= 2)>(a.wt_down, d, lrow, [&](int j, int) { return __ldcg(a.h + j); }, cnt, a.part,
                                       a.pstride, red, pol, a.stamps + 12, a.cta_t + b * 4 + 3);
  dstamp(a.stamps, 13);
  if (!grid_sync_fixed(a.bar, G, a.status, a.wait_ns)) return;
  dstamp(a.stamps, 14);

  // ---------------- E2: this CTA's slice of y ----------------
  {
    const int q0 = (int)((int64_t)(d / 4) * b / G);
    const int nq = (int)((int64_t)(d / 4) * (b + 1) / G) - q0;
    float4 y4, unused;
    reduce_scatter(a.part, a.pstride, q0, nq, G * npe, G * npe, reinterpret_cast<float4*>(red), &y4,
                             &unused);
    if (t < nq) reinterpret_cast<float4*>(a.y)[q0 + t] = y4;
  }
  dstamp(a.stamps, 15);
}

// rows in flight per thread for a row of VPT vectors per thread (64 registers per thread
// at 1024 threads)
template <int VPT>
struct RowsInFlight {
  // rows per batch: two register buffers of this many rows for 1 or 2 vectors per thread,
  // one buffer beyond (the 64 registers of a 1024-thread CTA)
  static constexpr int value = VPT == 1 ? 4 : (VPT == 2 ? 2 : (VPT == 3 ? 2 : 1));
};

template <bool BF16, int VB, int VE, int KA, int KC>
static void* decode_kernel() {
  return (void*)k_ffn_decode<BF16, VB, RowsInFlight<VB>::value, VE, RowsInFlight<VE>::value, KA, KC>;
}

// Instantiations: the decode shapes of the workloads get their own (the row widths and
// channel counts fixed at compile time, so that the 64 registers of a 1024-thread CTA hold
// the keys and the rows in flight without spilling); every other shape up to 16384
// channels and rows of up to 2048 16-byte vectors takes the general one.
static void* decode_kernel_for(bool bf16, int vb, int ve, int ka, int kc) {
  if (bf16) {
    if (vb == 3 && ve == 1 && ka <= 4 && kc <= 12) return decode_kernel<true, 3, 1, 4, 12>();  // Llama-7B, Gemma-2-2B
    if (vb == 4 && ve == 1 && ka <= 4 && kc <= 16) return decode_kernel<true, 4, 1, 4, 16>();  // Llama-3-8B
    return decode_kernel<true, 4, 4, 16, 16>();
  }
  return decode_kernel<false, 4, 4, 16, 16>();
}

// Vectors per thread of a row of m elements (0 if the row is too long for this kernel).
static int decode_vpt(int64_t m, int esz) {
  const int64_t V = m * esz / 16;
  const int tpr = decode_tpr((int)std::min<int64_t>(V, 1 << 20));
  const int64_t vpt = (V + tpr - 1) / tpr;
  return vpt <= 4 ? (int)vpt : 0;
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
  const int vb = decode_vpt(ffn, esz), ve = decode_vpt(d, esz);
  if (vb == 0 || ve == 0) return WINA_ERR_UNSUPPORTED_DTYPE;
  void* kern = decode_kernel_for(bf16, vb, ve, (d + kDT - 1) / kDT, (ffn + kDT - 1) / kDT);
  if (!kern) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int sms = device_sm_count();
  if (sms < 2) return WINA_ERR_CUDA;
  // gate/up CTA split in proportion to the kept rows (half each when unknown)
  int G = std::min(sms, kGridCap);
  int Gg = G / 2;
  if (mode == WINA_GATE_TOPK && k_gate + k_up > 0) Gg = (int)(((int64_t)G * k_gate + (k_gate + k_up) / 2) / (k_gate + k_up));
  Gg = std::max(1, std::min(G - 1, Gg));
  const int nmax = std::max(d, ffn);
  const int min_parts = std::min(Gg, G - Gg);
  const int cap = (nmax + min_parts - 1) / min_parts + 1;
  const int V_b = ffn * esz / 16, V_e = d * esz / 16;
  const int tb = decode_tpr(V_b), te = decode_tpr(V_e);
  const int epv = 16 / esz;
  const int red_floats = std::max((kDT / tb - 1) * tb * epv, (kDT / te - 1) * te * epv);
  const DecodeSmem SL = decode_smem(nmax, cap, std::max(red_floats, 32 * 32 * 4));
  const size_t smem = SL.total;
  // a CTA's slice of the columns must fit one lane each in reduce_scatter
  if ((ffn / 4 + G - 1) / G > 32 || (d / 4 + G - 1) / G > 32) return WINA_ERR_UNSUPPORTED_DTYPE;
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
  p.Gg = Gg;
  p.list_cap = cap;
  p.sm_flags = SL.flags;
  p.sm_wpre = SL.wpre;
  p.sm_lrow = SL.lrow;
  p.bar = reinterpret_cast<GridBarrier*>(w + L.bar);
  p.wait_ns = wait_limit_ns();
  p.part = reinterpret_cast<float*>(w + L.part);
  p.pstride = (int)L.pstride;
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
  {  // always: static shared memory comes on top of the dynamic part
    cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return cuda_status(e);
  }
  {
    cudaError_t e = ensure_prefer_l1(kern);  // the weight loads in flight live in L1
    if (e != cudaSuccess) return cuda_status(e);
  }
  void* args[] = {&p};
  return cuda_status(cudaLaunchKernelExC(&cfg, kern, args));
}

// ------------------------------------------------------------------------------------
// one token's sparse product on the same row stream
// ------------------------------------------------------------------------------------
//
// y[:] = sum over r < k of xs[r] * Wt[idx[r]][:] ("Spark Transformer", section 3.1, SVMM)
// for a single token: one cooperative launch of one 1024-thread CTA per SM. CTA c takes
// list entries c, c + G, c + 2G, ... (the kept rows dealt out round robin, so that all SMs
// read rows from the same neighbourhood of the weight at any moment), streams them as the
// FFN kernel's phase B does and stores its partial rows; after a grid barrier CTA c sums
// its slice of the columns over all partial rows in a fixed order. Bit-reproducible.

struct SpmvOneParams {
  const void* Wt;
  int64_t n;
  int m;
  const int32_t* idx;
  const float* xs;
  int k_fixed;            // >= 0: entries of the list; -1: count[0], clamped to ld
  const int32_t* count;
  int ld;
  float* y;
  float* part;            // [2G][m + 4] float32 partial rows
  GridBarrier* bar;
  int cap;                // list entries per CTA at most
  unsigned long long wait_ns;
  int32_t* status;
};

template <bool BF16, int VPT>
__global__ void __launch_bounds__(kDT, 1) k_spmv_one(SpmvOneParams a) {
  constexpr int U = RowsInFlight<VPT>::value;
  extern __shared__ __align__(128) unsigned char smraw[];
  int* lrow = reinterpret_cast<int*>(smraw);            // [cap]
  float* lval = reinterpret_cast<float*>(lrow + a.cap);  // [cap]
  float* red = lval + a.cap;                             // reduction scratch (16-byte aligned: cap % 4 == 0)
  const int G = gridDim.x, c = blockIdx.x, t = threadIdx.x;
  const uint64_t pol = l2_evict_first_policy();
  int kb = a.k_fixed;
  if (kb < 0) kb = max(0, min(__ldg(a.count), a.ld));
  int cnt = kb > c ? (kb - c + G - 1) / G : 0;
  if (cnt > a.cap) {  // cannot happen with the launcher's cap; kept as a guard
    if (t == 0) record_status(a.status, WINA_ERR_CAPACITY);
    cnt = a.cap;
  }
  for (int i = t; i < cnt; i += kDT) {
    const int r = c + i * G;
    int32_t row = __ldg(a.idx + r);
    float v = __ldg(a.xs + r);
    if (row < 0 || (int64_t)row >= a.n) {  // never read outside Wt
      record_status(a.status, WINA_ERR_INVALID_ARG);
      row = 0;
      v = 0.f;
    }
    lrow[i] = row;
    lval[i] = v;
  }
  __syncthreads();
  unsigned long long unused_t;
  long long unused_s;
  const int pstride = a.m + 4;  // rows offset by 4 floats: one column of successive rows spreads over L2 slices
  stream_rows<BF16, VPT, U, (VPT <= 2)>(a.Wt, a.m, lrow, [&](int, int pos) { return lval[pos]; }, cnt, a.part,
                                        pstride, red, pol, &unused_s, &unused_t);
  if (!grid_sync_fixed(a.bar, G, a.status, a.wait_ns)) return;
  constexpr uint32_t ESZ = BF16 ? 2u : 4u;
  const int np = decode_partials(a.m * (int)ESZ / 16);
  const int q0 = (int)((int64_t)(a.m / 4) * c / G);
  const int nq = (int)((int64_t)(a.m / 4) * (c + 1) / G) - q0;
  float4 y4, unused;
  reduce_scatter(a.part, pstride, q0, nq, G * np, G * np, reinterpret_cast<float4*>(red), &y4, &unused);
  if (t < nq) reinterpret_cast<float4*>(a.y)[q0 + t] = y4;
}

template <bool BF16, int VPT>
static wina_status_t launch_spmv_one_t(SpmvOneParams p, int G, cudaStream_t st) {
  void* kern = (void*)k_spmv_one<BF16, VPT>;
  const int esz = BF16 ? 2 : 4;
  const int V = p.m * esz / 16;
  const int tpr = decode_tpr(V);
  const int red_floats = std::max((kDT / tpr - 1) * tpr * (16 / esz), 32 * 32 * 4);
  const size_t smem = (size_t)p.cap * 8 + (size_t)red_floats * 4;
  cudaError_t e = ensure_smem_limit(kern, smem);
  if (e != cudaSuccess) return cuda_status(e);
  e = ensure_prefer_l1(kern);  // the weight loads in flight live in L1
  if (e != cudaSuccess) return cuda_status(e);
  if (blocks_per_sm(kern, kDT, smem) < 1) return WINA_ERR_UNSUPPORTED_DTYPE;
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
  void* args[] = {&p};
  return cuda_status(cudaLaunchKernelExC(&cfg, kern, args));
}

wina_status_t launch_spmv_one(const void* Wt, int wdt, int64_t n, int64_t m, const int32_t* idx, const float* xs,
                              int k, const int32_t* count, int ld, float* y, float* part, GridBarrier* bar,
                              int32_t* status, cudaStream_t st) {
  const bool bf16 = wdt == WINA_BF16;
  const int esz = bf16 ? 2 : 4;
  const int vpt = decode_vpt(m, esz);
  const int sms = device_sm_count();
  const int G = std::min(sms, kGridCap / 2);  // 2G partial rows fit the workspace's kGridCap
  if (vpt == 0 || G < 2 || m > INT32_MAX) return WINA_ERR_UNSUPPORTED_DTYPE;
  if ((m / 4 + G - 1) / G > 32) return WINA_ERR_UNSUPPORTED_DTYPE;  // one lane per float4 column
  const int kmax = k >= 0 ? k : ld;
  SpmvOneParams p;
  p.Wt = Wt;
  p.n = n;
  p.m = (int)m;
  p.idx = idx;
  p.xs = xs;
  p.k_fixed = k;
  p.count = count;
  p.ld = ld;
  p.y = y;
  p.part = part;
  p.bar = bar;
  p.cap = ((kmax + G - 1) / G + 3) / 4 * 4;
  if (p.cap < 4) p.cap = 4;
  p.wait_ns = wait_limit_ns();
  p.status = status;
  if ((size_t)p.cap * 8 > 64 * 1024) return WINA_ERR_UNSUPPORTED_DTYPE;  // list beyond SMEM: the general path
  if (bf16) {
    switch (vpt) {
      case 1: return launch_spmv_one_t<true, 1>(p, G, st);
      case 2: return launch_spmv_one_t<true, 2>(p, G, st);
      case 3: return launch_spmv_one_t<true, 3>(p, G, st);
      default: return launch_spmv_one_t<true, 4>(p, G, st);
    }
  }
  switch (vpt) {
    case 1: return launch_spmv_one_t<false, 1>(p, G, st);
    case 2: return launch_spmv_one_t<false, 2>(p, G, st);
    case 3: return launch_spmv_one_t<false, 3>(p, G, st);
    default: return launch_spmv_one_t<false, 4>(p, G, st);
  }
}

}  // namespace wina
