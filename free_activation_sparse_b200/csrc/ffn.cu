// SwiGLU FFN decode with the gate on every projection ("WAS" article, core innovations:
// weight-aware sparsity per component, gate/up/down among them; "WINA" article,
// section 一: each projection scores with its own column norms and its own K).
//
// One token: a single persistent cooperative kernel, one CTA per SM.
//   A  every CTA scores x against c_gate and c_up in SMEM and selects both kept sets
//      (radix select; or the Spark threshold; or all channels). The kept gate rows
//      followed by the kept up rows form one list of Kg + Ku rows; CTA b takes the
//      b-th of G equal slices of it.
//   B  stream those rows of Wt_gate / Wt_up (ffn wide) and write float32 partial rows.
//   -- grid barrier --
//   C  CTA b sums its slice of columns over the partials (fixed order): g, u, then
//      h = silu(g) * u and the down gate's score |h_j * c_down_j| (or h itself).
//   -- grid barrier --
//   D  every CTA selects the kept down channels from all ffn scores; CTA b takes its
//      slice of the Kd kept rows.
//   E  stream those rows of Wt_down (d wide) and write partial rows.
//   -- grid barrier --
//   F  CTA b sums its slice of y over the partials.
// Barrier waits are bounded (WINA_ERR_TIMEOUT). Several tokens: the batched calls
// (select, sparse_matvec, silu*mul, select, sparse_matvec) in sequence.
#include <math.h>

#include "internal.h"

namespace wina {

constexpr int kFfnRowCap = 512;             // kept rows one CTA stages per projection
constexpr size_t kMaxSmem = 227 * 1024;     // dynamic SMEM one CTA may use on sm_100

struct FfnParams {
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
  GridBarrier* bar;
  float* h;
  uint32_t* keys_d;
  int32_t* idx_gate;
  int32_t* idx_up;
  int32_t* idx_down;
  int32_t* cnt;
  long long* stamps;
  unsigned long long* cta_t;
  float* part_g;
  float* part_u;
  float* part_d;
  int32_t* status;
};

struct Slice {
  int lo, hi;
};
__device__ __forceinline__ Slice slice_of(int total, int G, int p) {
  return Slice{(int)((int64_t)total * p / G), (int)((int64_t)total * (p + 1) / G)};
}

// The gate part and the up part of CTA p's slice of the list [gate rows | up rows].
struct GateUpSplit {
  int g_lo, g_hi, u_lo, u_hi;
};
__device__ __forceinline__ GateUpSplit gate_up_split(int Kg, int Ku, int G, int p) {
  const Slice s = slice_of(Kg + Ku, G, p);
  GateUpSplit r;
  r.g_lo = min(s.lo, Kg);
  r.g_hi = min(s.hi, Kg);
  r.u_lo = max(s.lo, Kg) - Kg;
  r.u_hi = max(s.hi, Kg) - Kg;
  return r;
}

template <bool BF16, int VPT, int U>
__device__ __forceinline__ void project_t(const void* __restrict__ Wt, const RowLayout& L, const int32_t* rows,
                                          const float* vals, int nrows, float* __restrict__ out, float* red,
                                          uint64_t pol) {
  constexpr int EPV = VecOps<BF16>::EPV;
  float acc[VPT][EPV];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[j][e] = 0.f;
  accumulate_rows<BF16, VPT, U>(Wt, L, rows, vals, nrows, acc, pol);
  store_partial<BF16, VPT>(out, L, acc, red);
}

// Partial row out[0..m) = sum over the staged rows of vals[r] * Wt[rows[r]][:].
template <bool BF16>
__device__ void project(const void* __restrict__ Wt, const RowLayout& L, const int32_t* rows, const float* vals,
                        int nrows, float* __restrict__ out, float* red, uint64_t pol) {
  switch (L.VPT) {
    case 1: project_t<BF16, 1, 8>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 2: project_t<BF16, 2, 4>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 3: project_t<BF16, 3, 4>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 4: project_t<BF16, 4, 3>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 5: project_t<BF16, 5, 2>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 6: project_t<BF16, 6, 2>(Wt, L, rows, vals, nrows, out, red, pol); break;
    case 7: project_t<BF16, 7, 1>(Wt, L, rows, vals, nrows, out, red, pol); break;
    default: project_t<BF16, 8, 1>(Wt, L, rows, vals, nrows, out, red, pol); break;
  }
}

// Fixed-order column sums over the partial rows of the CTAs in `list` (nl entries,
// ascending), for NP projections at once: for t < w, out[q] = sum over e of
// part4[q][list[q][e] * m4 + c0 + t]. Thread (grp, ci) takes list entries grp,
// grp + groups, ... and issues its loads eight at a time; the groups' sums are then
// added in group order. `red4` is SMEM of NP * kNT float4. All threads must call it.
template <int NP>
__device__ __forceinline__ void reduce_lists(const float4* const (&part4)[NP], const int* const (&list)[NP],
                                             const int (&nl)[NP], int64_t m4, int64_t c0, int w, float4* red4,
                                             float4 (&out)[NP]) {
  const int groups = kNT / w;
  const int t = threadIdx.x;
  const int ci = t % w, grp = t / w;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grp < groups) {
      const float4* base = part4[q] + c0 + ci;
      const int* L = list[q];
      for (int e0 = grp; e0 < nl[q]; e0 += 8 * groups) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // up to 8 independent loads in flight
          const int e = e0 + u * groups;
          v[u] = e < nl[q] ? __ldcg(base + (int64_t)L[e] * m4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          a.x += v[u].x;
          a.y += v[u].y;
          a.z += v[u].z;
          a.w += v[u].w;
        }
      }
    }
    red4[q * kNT + t] = a;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < w) {
      for (int g = 0; g < groups; ++g) {
        const float4 v = red4[q * kNT + g * w + t];
        s.x += v.x;
        s.y += v.y;
        s.z += v.z;
        s.w += v.w;
      }
    }
    out[q] = s;
  }
  __syncthreads();
}

// Ascending list of the CTAs pp < G for which wrote(pp) holds; returns its length.
template <typename Wrote>
__device__ __forceinline__ int writer_list(int G, Wrote wrote, int* list, uint32_t* wsm) {
  return (int)compact_pred<kNT>(
      G, wrote,
      [&](uint32_t total, uint32_t* lo, uint32_t* hi) {
        *lo = 0;
        *hi = total;
      },
      wsm, [&](int pp, uint32_t pos) { list[pos] = pp; });
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// CTA 0 records its SM clock at phase boundaries; every CTA records the global timer at
// the end of its four main phases (diagnostic views of the workspace).
__device__ __forceinline__ void stamp(long long* stamps, int i) {
  if (blockIdx.x == 0 && threadIdx.x == 0) stamps[i] = clock64();
}
__device__ __forceinline__ void cta_time(unsigned long long* t, int i) {
  if (threadIdx.x == 0) t[blockIdx.x * 4 + i] = globaltimer_ns();
}

template <bool BF16>
__global__ void __launch_bounds__(kNT, 1) k_ffn_fused(FfnParams a) {
  constexpr int EPV = VecOps<BF16>::EPV;
  extern __shared__ __align__(16) unsigned char smraw[];
  const int d = a.d, ffn = a.ffn;
  const int nkeys = max(2 * d, ffn);
  const int nvals = max(d, ffn);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smraw);          // [nkeys] scores (uint32 bits)
  float* xv = reinterpret_cast<float*>(keys + nkeys);           // [nvals] x, then h
  uint32_t* hist = reinterpret_cast<uint32_t*>(xv + nvals);     // [2 * 2 * 256] select histograms
  int32_t* rows = reinterpret_cast<int32_t*>(hist + 1024);      // [kFfnRowCap]
  float* vals = reinterpret_cast<float*>(rows + kFfnRowCap);    // [kFfnRowCap]
  int* wl = reinterpret_cast<int*>(vals + kFfnRowCap);          // [2 * kGridCap] writer lists
  float* red = reinterpret_cast<float*>(wl + 2 * kGridCap);     // [kNT * 8]
  __shared__ uint32_t wsm[2 * kNT / 32 + 1];
  __shared__ double dred[3 * kNT / 32];

  const int G = gridDim.x, b = blockIdx.x;
  const uint64_t pol = l2_evict_first_policy();
  stamp(a.stamps, 0);

  // ---------------- A: gate / up selection ----------------
  int Kg, Ku;
  GateUpSplit sp;
  if (a.mode == WINA_GATE_STAT) {
    Moments mo{0.0, 0.0, 0.0};
    for (int i = threadIdx.x; i < d; i += kNT) {
      const float f = load_elem(a.x, a.xdt, i);
      xv[i] = f;
      mo.n += 1.0;
      const double dl = (double)f - mo.mean;
      mo.mean += dl / mo.n;
      mo.m2 += dl * ((double)f - mo.mean);
    }
    const Moments tot = block_moments<kNT>(mo, dred);
    const double t = tot.mean + sqrt(tot.m2 / (double)d) * a.z;
    auto pred = [&](int i) { return (double)xv[i] > t; };
    // the kept count is known only after the first walk; every thread computes the
    // same split from it (no shared state needed)
    int kept = 0;
    GateUpSplit gs{0, 0, 0, 0};
    compact_pred<kNT>(
        d, pred,
        [&](uint32_t total, uint32_t* lo, uint32_t* hi) {
          kept = (int)total;
          gs = gate_up_split(kept, kept, G, b);
          *lo = gs.g_lo;
          *hi = gs.g_hi;
        },
        wsm,
        [&](int i, uint32_t pos) {
          rows[pos - gs.g_lo] = i;
          vals[pos - gs.g_lo] = xv[i];
          a.idx_gate[pos] = i;
        });
    Kg = Ku = kept;
    sp = gate_up_split(Kg, Ku, G, b);
    const int ng = sp.g_hi - sp.g_lo;
    compact_pred<kNT>(
        d, pred,
        [&](uint32_t, uint32_t* lo, uint32_t* hi) {
          *lo = sp.u_lo;
          *hi = sp.u_hi;
        },
        wsm,
        [&](int i, uint32_t pos) {
          rows[ng + pos - sp.u_lo] = i;
          vals[ng + pos - sp.u_lo] = xv[i];
          a.idx_up[pos] = i;
        });
  } else {
    Selection sel[2];
    if (a.mode == WINA_GATE_TOPK) {
      for (int i = threadIdx.x; i < d; i += kNT) {
        const float f = load_elem(a.x, a.xdt, i);
        xv[i] = f;
        keys[i] = __float_as_uint(fabsf(f * __ldg(a.c_gate + i)));
        keys[d + i] = __float_as_uint(fabsf(f * __ldg(a.c_up + i)));
      }
      __syncthreads();
      Kg = a.k_gate;
      Ku = a.k_up;
      const uint32_t* ks[2] = {keys, keys + d};
      const int kk[2] = {Kg, Ku};
      select_topk_multi<kNT, 2>(ks, d, kk, hist, sel);
    } else {  // dense: every channel
      for (int i = threadIdx.x; i < d; i += kNT) {
        xv[i] = load_elem(a.x, a.xdt, i);
        keys[i] = 0u;
        keys[d + i] = 0u;
      }
      __syncthreads();
      Kg = Ku = d;
      sel[0] = sel[1] = Selection{0u, 0u, (uint32_t)d};
    }
    sp = gate_up_split(Kg, Ku, G, b);
    const int ng = sp.g_hi - sp.g_lo;
    compact_selection<kNT>(keys, d, sel[0], (uint32_t)sp.g_lo, (uint32_t)sp.g_hi, wsm, [&](int i, uint32_t pos) {
      rows[pos - sp.g_lo] = i;
      vals[pos - sp.g_lo] = xv[i];
      a.idx_gate[pos] = i;
    });
    compact_selection<kNT>(keys + d, d, sel[1], (uint32_t)sp.u_lo, (uint32_t)sp.u_hi, wsm,
                           [&](int i, uint32_t pos) {
                             rows[ng + pos - sp.u_lo] = i;
                             vals[ng + pos - sp.u_lo] = xv[i];
                             a.idx_up[pos] = i;
                           });
  }
  __syncthreads();
  stamp(a.stamps, 1);
  cta_time(a.cta_t, 0);

  // ---------------- B: stream kept gate / up rows ----------------
  const RowLayout Lf = make_row_layout<kNT>(ffn, EPV);
  const int ng = sp.g_hi - sp.g_lo, nu = sp.u_hi - sp.u_lo;
  if (ng > 0) project<BF16>(a.wt_gate, Lf, rows, vals, ng, a.part_g + (int64_t)b * ffn, red, pol);
  if (nu > 0) project<BF16>(a.wt_up, Lf, rows + ng, vals + ng, nu, a.part_u + (int64_t)b * ffn, red, pol);
  stamp(a.stamps, 2);
  cta_time(a.cta_t, 1);

  if (!grid_sync_fixed(a.bar, G, a.status)) return;
  stamp(a.stamps, 3);

  // ---------------- C: g, u, h and the down scores for this CTA's columns ----------------
  {
    int* lg = wl;
    int* lu = wl + kGridCap;
    const int ngl = writer_list(
        G,
        [&](int pp) {
          const GateUpSplit s = gate_up_split(Kg, Ku, G, pp);
          return s.g_hi > s.g_lo;
        },
        lg, wsm);
    const int nul = writer_list(
        G,
        [&](int pp) {
          const GateUpSplit s = gate_up_split(Kg, Ku, G, pp);
          return s.u_hi > s.u_lo;
        },
        lu, wsm);
    stamp(a.stamps, 10);
    const int64_t m4 = ffn / 4;
    const int64_t q0 = m4 * b / G, q1 = m4 * (b + 1) / G;
    const float4* parts[2] = {reinterpret_cast<const float4*>(a.part_g), reinterpret_cast<const float4*>(a.part_u)};
    const int* lists[2] = {lg, lu};
    const int nls[2] = {ngl, nul};
    for (int64_t qb = q0; qb < q1; qb += kNT) {
      const int w = (int)min((int64_t)kNT, q1 - qb);
      float4 gu[2];
      reduce_lists<2>(parts, lists, nls, m4, qb, w, reinterpret_cast<float4*>(red), gu);
      if ((int)threadIdx.x < w) {
        const int64_t j = (qb + threadIdx.x) * 4;
        float4 h4;
        h4.x = silu_f(gu[0].x) * gu[1].x;
        h4.y = silu_f(gu[0].y) * gu[1].y;
        h4.z = silu_f(gu[0].z) * gu[1].z;
        h4.w = silu_f(gu[0].w) * gu[1].w;
        *reinterpret_cast<float4*>(a.h + j) = h4;
        if (a.mode == WINA_GATE_TOPK) {
          const float4 c4 = __ldg(reinterpret_cast<const float4*>(a.c_down + j));
          uint4 k4;
          k4.x = __float_as_uint(fabsf(h4.x * c4.x));
          k4.y = __float_as_uint(fabsf(h4.y * c4.y));
          k4.z = __float_as_uint(fabsf(h4.z * c4.z));
          k4.w = __float_as_uint(fabsf(h4.w * c4.w));
          *reinterpret_cast<uint4*>(a.keys_d + j) = k4;
        }
      }
    }
  }

  stamp(a.stamps, 4);
  if (!grid_sync_fixed(a.bar, G, a.status)) return;
  stamp(a.stamps, 5);

  // ---------------- D: down selection ----------------
  int Kd;
  Slice sd;
  for (int i = threadIdx.x; i < ffn; i += kNT) {
    xv[i] = __ldcg(a.h + i);
    if (a.mode == WINA_GATE_TOPK) keys[i] = __ldcg(a.keys_d + i);
  }
  __syncthreads();
  stamp(a.stamps, 11);
  if (a.mode == WINA_GATE_STAT) {
    Moments mo{0.0, 0.0, 0.0};
    for (int i = threadIdx.x; i < ffn; i += kNT) {
      const double f = (double)xv[i];
      mo.n += 1.0;
      const double dl = f - mo.mean;
      mo.mean += dl / mo.n;
      mo.m2 += dl * (f - mo.mean);
    }
    const Moments tot = block_moments<kNT>(mo, dred);
    const double t = tot.mean + sqrt(tot.m2 / (double)ffn) * a.z;
    int kept = 0;
    Slice ds{0, 0};
    compact_pred<kNT>(
        ffn, [&](int i) { return (double)xv[i] > t; },
        [&](uint32_t total, uint32_t* lo, uint32_t* hi) {
          kept = (int)total;
          ds = slice_of(kept, G, b);
          *lo = ds.lo;
          *hi = ds.hi;
        },
        wsm,
        [&](int i, uint32_t pos) {
          rows[pos - ds.lo] = i;
          vals[pos - ds.lo] = xv[i];
          a.idx_down[pos] = i;
        });
    Kd = kept;
    sd = slice_of(Kd, G, b);
  } else {
    Selection sel;
    if (a.mode == WINA_GATE_TOPK) {
      Kd = a.k_down;
      sel = select_topk_block<kNT>(keys, ffn, Kd, hist);
      stamp(a.stamps, 12);
    } else {
      Kd = ffn;
      sel = Selection{0u, 0u, (uint32_t)ffn};
    }
    sd = slice_of(Kd, G, b);
    compact_selection<kNT>(keys, ffn, sel, (uint32_t)sd.lo, (uint32_t)sd.hi, wsm, [&](int i, uint32_t pos) {
      rows[pos - sd.lo] = i;
      vals[pos - sd.lo] = xv[i];
      a.idx_down[pos] = i;
    });
  }
  __syncthreads();
  if (b == 0 && threadIdx.x == 0) {
    a.cnt[0] = Kg;
    a.cnt[1] = Ku;
    a.cnt[2] = Kd;
  }
  stamp(a.stamps, 6);
  cta_time(a.cta_t, 2);

  // ---------------- E: stream kept down rows ----------------
  const RowLayout Ld = make_row_layout<kNT>(d, EPV);
  const int nd = sd.hi - sd.lo;
  if (nd > 0) project<BF16>(a.wt_down, Ld, rows, vals, nd, a.part_d + (int64_t)b * d, red, pol);
  stamp(a.stamps, 7);
  cta_time(a.cta_t, 3);

  if (!grid_sync_fixed(a.bar, G, a.status)) return;
  stamp(a.stamps, 8);

  // ---------------- F: y for this CTA's columns ----------------
  {
    int* ld = wl;
    const int ndl = writer_list(
        G,
        [&](int pp) {
          const Slice s = slice_of(Kd, G, pp);
          return s.hi > s.lo;
        },
        ld, wsm);
    const int64_t m4 = d / 4;
    const int64_t q0 = m4 * b / G, q1 = m4 * (b + 1) / G;
    const float4* parts[1] = {reinterpret_cast<const float4*>(a.part_d)};
    const int* lists[1] = {ld};
    const int nls[1] = {ndl};
    for (int64_t qb = q0; qb < q1; qb += kNT) {
      const int w = (int)min((int64_t)kNT, q1 - qb);
      float4 y4[1];
      reduce_lists<1>(parts, lists, nls, m4, qb, w, reinterpret_cast<float4*>(red), y4);
      if ((int)threadIdx.x < w) reinterpret_cast<float4*>(a.y)[qb + threadIdx.x] = y4[0];
    }
  }
  stamp(a.stamps, 9);
}

static size_t ffn_fused_smem(int64_t d, int64_t ffn) {
  const int64_t nkeys = 2 * d > ffn ? 2 * d : ffn;
  const int64_t nvals = d > ffn ? d : ffn;
  return (size_t)nkeys * 4 + (size_t)nvals * 4 + (size_t)1024 * 4 + (size_t)kFfnRowCap * 8 +
         (size_t)2 * kGridCap * 4 + (size_t)kNT * 8 * 4;
}

}  // namespace wina

using namespace wina;

extern "C" wina_status_t sparse_ffn_swiglu(const wina_ffn_t* f, const void* x, wina_dtype_t xdt, int64_t batch,
                                           wina_gate_mode_t mode, int64_t k_gate, int64_t k_up, int64_t k_down,
                                           double s, float* y, void* ws, size_t ws_bytes, int32_t* status_dev,
                                           wina_stream_t stream) {
  if (!f) return WINA_ERR_INVALID_ARG;
  if (!valid_dtype(xdt) || !valid_dtype(f->wdt)) return WINA_ERR_UNSUPPORTED_DTYPE;
  const int64_t d = f->d, ffn = f->ffn;
  const int epv = f->wdt == WINA_BF16 ? 8 : 4;
  if (d < epv || ffn < epv || d % epv || ffn % epv || d > kMaxN || ffn > kMaxN) return WINA_ERR_INVALID_ARG;
  if (d / epv > (int64_t)kNT * 8 || ffn / epv > (int64_t)kNT * 8) return WINA_ERR_INVALID_ARG;  // register tile
  if (batch < 1 || batch > INT32_MAX) return WINA_ERR_INVALID_ARG;
  if (mode != WINA_GATE_TOPK && mode != WINA_GATE_STAT && mode != WINA_GATE_DENSE) return WINA_ERR_INVALID_ARG;
  if (mode == WINA_GATE_TOPK) {
    if (k_gate < 0 || k_gate > d || k_up < 0 || k_up > d || k_down < 0 || k_down > ffn) return WINA_ERR_INVALID_ARG;
    if (!f->c_gate || !f->c_up || !f->c_down) return WINA_ERR_INVALID_ARG;
  }
  if (mode == WINA_GATE_STAT && !(s > 0.0 && s < 1.0)) return WINA_ERR_INVALID_ARG;
  if (!f->wt_gate || !f->wt_up || !f->wt_down || !x || !y || !ws) return WINA_ERR_INVALID_ARG;
  if (!aligned(f->wt_gate, 16) || !aligned(f->wt_up, 16) || !aligned(f->wt_down, 16) || !aligned(y, 16) ||
      !aligned(ws, 16) || !aligned(x, elem_size(xdt)) || (f->c_gate && !aligned(f->c_gate, 16)) ||
      (f->c_up && !aligned(f->c_up, 16)) || (f->c_down && !aligned(f->c_down, 16)) ||
      (status_dev && !aligned(status_dev, 4)))
    return WINA_ERR_INVALID_ARG;
  if (ws_bytes < wina_workspace_size(WINA_OP_FFN_SWIGLU, d, ffn, 0, batch)) return WINA_ERR_WORKSPACE;
  if (mode == WINA_GATE_DENSE) {
    k_gate = k_up = d;
    k_down = ffn;
  }
  const double z = mode == WINA_GATE_STAT ? wina_normal_quantile(1.0 - s) : 0.0;
  cudaStream_t st = (cudaStream_t)stream;
  const FfnWs L = ffn_ws_layout(d, ffn, batch);
  char* w = (char*)ws;

  if (batch == 1 && 2 * d <= kMaxN && ffn_fused_smem(d, ffn) <= kMaxSmem) {
    const bool bf16 = f->wdt == WINA_BF16;
    const size_t smem = ffn_fused_smem(d, ffn);
    const int G = bf16 ? max_coresident_grid(k_ffn_fused<true>, kNT, smem)
                       : max_coresident_grid(k_ffn_fused<false>, kNT, smem);
    const int64_t lmax = 2 * d > ffn ? 2 * d : ffn;
    if (G >= 1 && (lmax + G - 1) / G <= kFfnRowCap) {
      FfnParams p;
      p.wt_gate = f->wt_gate;
      p.wt_up = f->wt_up;
      p.wt_down = f->wt_down;
      p.c_gate = f->c_gate;
      p.c_up = f->c_up;
      p.c_down = f->c_down;
      p.x = x;
      p.xdt = xdt;
      p.d = (int)d;
      p.ffn = (int)ffn;
      p.mode = mode;
      p.k_gate = (int)k_gate;
      p.k_up = (int)k_up;
      p.k_down = (int)k_down;
      p.z = z;
      p.y = y;
      p.bar = reinterpret_cast<GridBarrier*>(w + L.bar);
      p.h = reinterpret_cast<float*>(w + L.h);
      p.keys_d = reinterpret_cast<uint32_t*>(w + L.keys_d);
      p.idx_gate = reinterpret_cast<int32_t*>(w + L.idx_gate);
      p.idx_up = reinterpret_cast<int32_t*>(w + L.idx_up);
      p.idx_down = reinterpret_cast<int32_t*>(w + L.idx_down);
      p.cnt = reinterpret_cast<int32_t*>(w + L.cnt);
      p.stamps = reinterpret_cast<long long*>(w + L.stamps);
      p.cta_t = reinterpret_cast<unsigned long long*>(w + L.cta_t);
      p.part_g = reinterpret_cast<float*>(w + L.part_g);
      p.part_u = reinterpret_cast<float*>(w + L.part_u);
      p.part_d = reinterpret_cast<float*>(w + L.part_d);
      p.status = status_dev;
      cudaError_t e = bf16 ? launch_kernel(k_ffn_fused<true>, dim3(G), dim3(kNT), smem, st, true, p)
                           : launch_kernel(k_ffn_fused<false>, dim3(G), dim3(kNT), smem, st, true, p);
      return cuda_status(e);
    }
  }

  // Several tokens (or shapes the fused kernel does not take): batched calls.
  float* h = reinterpret_cast<float*>(w + L.h);
  int32_t* ig = reinterpret_cast<int32_t*>(w + L.idx_gate);
  int32_t* iu = reinterpret_cast<int32_t*>(w + L.idx_up);
  int32_t* idn = reinterpret_cast<int32_t*>(w + L.idx_down);
  int32_t* cnt = reinterpret_cast<int32_t*>(w + L.cnt);
  float* xg = reinterpret_cast<float*>(w + L.xs_gate);
  float* xu = reinterpret_cast<float*>(w + L.xs_up);
  float* xd = reinterpret_cast<float*>(w + L.xs_down);
  float* g = reinterpret_cast<float*>(w + L.g);
  float* u = reinterpret_cast<float*>(w + L.u);
  void* sw = w + L.spmv;
  const int B = (int)batch;
  wina_status_t r;
  if (mode == WINA_GATE_STAT) {
    if ((r = launch_stat_threshold(x, xdt, (int)d, z, B, ig, xg, cnt, nullptr, (int)d, status_dev, st))) return r;
    if ((r = launch_stat_threshold(x, xdt, (int)d, z, B, iu, xu, cnt + B, nullptr, (int)d, status_dev, st))) return r;
    if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, -1, cnt, (int)d, B, g, sw, status_dev, st)))
      return r;
    if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, iu, xu, -1, cnt + B, (int)d, B, u, sw, status_dev, st)))
      return r;
    if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
    if ((r = launch_stat_threshold(h, WINA_F32, (int)ffn, z, B, idn, xd, cnt + 2 * B, nullptr, (int)ffn, status_dev,
                                   st)))
      return r;
    return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, -1, cnt + 2 * B, (int)ffn, B, y, sw, status_dev,
                                st);
  }
  const float* cg = mode == WINA_GATE_TOPK ? f->c_gate : nullptr;
  const float* cu = mode == WINA_GATE_TOPK ? f->c_up : nullptr;
  const float* cd = mode == WINA_GATE_TOPK ? f->c_down : nullptr;
  if ((r = launch_select_topk(x, xdt, cg, (int)d, (int)k_gate, B, ig, xg, (int)d, nullptr, st))) return r;
  if ((r = launch_select_topk(x, xdt, cu, (int)d, (int)k_up, B, iu, xu, (int)d, nullptr, st))) return r;
  if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, (int)k_gate, nullptr, (int)d, B, g, sw,
                                status_dev, st)))
    return r;
  if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, iu, xu, (int)k_up, nullptr, (int)d, B, u, sw, status_dev,
                                st)))
    return r;
  if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
  if ((r = launch_select_topk(h, WINA_F32, cd, (int)ffn, (int)k_down, B, idn, xd, (int)ffn, nullptr, st))) return r;
  return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, (int)k_down, nullptr, (int)ffn, B, y, sw,
                              status_dev, st);
}
