// Device building blocks shared by the kernels of the WINA sparse-linear library.
//
//  * element loads (bf16 / f32) and cache-hinted streaming loads of weight rows;
//  * block-wide exclusive scan;
//  * exact top-K by radix select on float32 score bits (scores are >= 0, so their
//    uint32 bit patterns order like the floats), ties to the lower index;
//  * warp-ballot compaction of a selection into an ascending index list;
//  * a grid barrier with a time limit, for cooperative (co-resident) launches;
//  * the split-K row accumulation of the sparse product (SVMM).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "wina.h"

namespace wina {

constexpr int kMaxN = 32768;                          // longest vector a gate handles in SMEM
constexpr unsigned long long kBarrierTimeoutNs = 1000000000ull;  // 1 s per barrier wait

// ------------------------------------------------------------------------------------
// loads and status
// ------------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Element i of a vector stored as dtype dt, widened to float32 (exact).
__device__ __forceinline__ float load_elem(const void* p, int dt, int64_t i) {
  if (dt == WINA_BF16) return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
  return __ldg(reinterpret_cast<const float*>(p) + i);
}

// L2 policy: weight rows are read once per call; let them leave L2 first so that the
// small cross-CTA buffers (partials, h) stay resident.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint4 ld_stream_u4(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// First error wins; 0 means no error.
__device__ __forceinline__ void record_status(int32_t* st, int code) {
  if (st) atomicCAS(reinterpret_cast<int*>(st), 0, code);
}

// ------------------------------------------------------------------------------------
// block scan
// ------------------------------------------------------------------------------------

// Exclusive prefix sum of one uint32 per thread over the block (NT a multiple of 32,
// <= 1024). `red` is SMEM scratch of >= 32 words. Returns the thread's exclusive
// prefix; *total (if given) receives the block total. Contains __syncthreads().
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* red, uint32_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NW ? red[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) red[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t before = warp ? red[warp - 1] : 0u;
  if (total) *total = red[NW - 1];
  __syncthreads();  // red may be reused right after
  return before + x - v;
}

// ------------------------------------------------------------------------------------
// exact top-K selection on non-negative float32 keys
// ------------------------------------------------------------------------------------

// Ballot compaction of a predicate (ascending index order): first counts, then calls
// range(total, &lo, &hi) on every thread to choose the window of positions wanted, then
// emit(i, pos) for kept channels with lo <= pos < hi. Returns the total kept count.
template <int NT, typename Pred, typename Range, typename Emit>
__device__ uint32_t compact_pred(int n, Pred pred, Range range, uint32_t* wsm, Emit emit) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (((n + NW - 1) / NW) + 31) & ~31;
  const int b0 = warp * seg;
  const int b1 = min(n, b0 + seg);
  uint32_t cs = 0;
  for (int base = b0; base < b1; base += 32) {
    const int i = base + lane;
    cs += __popc(__ballot_sync(0xffffffffu, i < b1 && pred(i)));
  }
  if (lane == 0) wsm[warp] = cs;
  __syncthreads();
  if (warp == 0) {
    const uint32_t a = lane < NW ? wsm[lane] : 0u;
    uint32_t ia = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ia, o);
      if (lane >= o) ia += y;
    }
    if (lane < NW) wsm[lane] = ia - a;
    if (lane == NW - 1) wsm[NW] = ia;
  }
  __syncthreads();
  const uint32_t total = wsm[NW];
  uint32_t lo = 0, hi = 0;
  range(total, &lo, &hi);
  uint32_t sbase = wsm[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = b0; base < b1; base += 32) {
    const int i = base + lane;
    const bool k = i < b1 && pred(i);
    const uint32_t sb = __ballot_sync(0xffffffffu, k);
    const uint32_t pos = sbase + __popc(sb & lt);
    if (k && pos >= lo && pos < hi) emit(i, pos);
    sbase += __popc(sb);
  }
  __syncthreads();
  return total;
}

// ------------------------------------------------------------------------------------
// top-K as a threshold: kept(j) <=> key_j > T, or key_j == T and j <= cut
// ------------------------------------------------------------------------------------

struct Threshold {
  uint32_t T;  // key of the K-th largest channel
  int cut;     // its index: among keys equal to T, those with index <= cut are kept
};

__device__ __forceinline__ bool kept_by(const Threshold& t, uint32_t key, int j) {
  return key > t.T || (key == t.T && j <= t.cut);
}

constexpr int kSelBins = 4096;   // histogram bins of select_threshold
constexpr int kSelCand = 512;    // candidates resolved exactly by ranking

// Block-wide min and max of v (all threads receive them). `red` >= 2 * NT/32 words.
template <int NT>
__device__ __forceinline__ void block_minmax_u32(uint32_t v_min, uint32_t v_max, uint32_t* red, uint32_t& mn,
                                                 uint32_t& mx) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v_min = __reduce_min_sync(0xffffffffu, v_min);
  v_max = __reduce_max_sync(0xffffffffu, v_max);
  if (lane == 0) {
    red[warp] = v_min;
    red[NW + warp] = v_max;
  }
  __syncthreads();
  mn = 0xffffffffu;
  mx = 0u;
  for (int w = 0; w < NW; ++w) {
    mn = min(mn, red[w]);
    mx = max(mx, red[NW + w]);
  }
  __syncthreads();
}

// Exact top-K of keys[0..n) in SMEM (ties to the lower index), found as a threshold.
// The candidates (initially every key) are spread over kSelBins bins by a linear map
// of their bit patterns between the candidates' min and max key; the map is monotone,
// so the bins are ordered like the keys. One histogram pass and a scan find the bin
// holding the K-th key; if that bin holds at most kSelCand keys they are ranked
// exactly, otherwise the search repeats inside the bin's key range. Equal keys are
// ordered by index. Buffers in SMEM: hist [kSelBins], cand [2 * kSelCand] words,
// red [>= 2 * NT/32 + 4] words. Every thread of the block must call it.
template <int NT>
__device__ Threshold select_threshold(const uint32_t* __restrict__ keys, int n, int K, uint32_t* __restrict__ hist,
                                      uint32_t* __restrict__ cand, uint32_t* __restrict__ red) {
  constexpr int CH = 8;  // keys a thread loads into registers before it updates counts
  __shared__ uint32_t s_bin, s_above, s_cnt, s_ncand;
  __shared__ Threshold s_res;
  if (K <= 0) return Threshold{0xffffffffu, -1};
  if (K >= n) return Threshold{0u, n - 1};
  uint32_t lo = 0u, hi = 0xffffffffu;  // key range of the candidates
  uint32_t r = (uint32_t)K;            // rank (1-based, from the top) sought among them
#pragma unroll 1
  for (int iter = 0; iter < 8; ++iter) {
    // candidates' min / max
    uint32_t a = 0xffffffffu, b = 0u;
    for (int i0 = threadIdx.x; i0 < n; i0 += CH * NT) {
      uint32_t k[CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int i = i0 + u * NT;
        k[u] = i < n ? keys[i] : lo;  // lo never widens [a, b] beyond the candidates
      }
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (k[u] >= lo && k[u] <= hi) {
          a = min(a, k[u]);
          b = max(b, k[u]);
        }
    }
    uint32_t mn, mx;
    block_minmax_u32<NT>(a, b, red, mn, mx);
    if (mn == mx) {
      // every candidate has the same key: the r-th of them by index is the cut
      if (threadIdx.x == 0) s_res = Threshold{mn, n - 1};
      compact_pred<NT>(
          n, [&](int i) { return keys[i] == mn; },
          [&](uint32_t, uint32_t* l, uint32_t* h) {
            *l = r - 1;
            *h = r;
          },
          red, [&](int i, uint32_t) { s_res.cut = i; });
      const Threshold t = s_res;
      __syncthreads();
      return t;
    }
    const float scale = (float)kSelBins / ((float)(mx - mn) + 1.0f);
    auto bin_of = [&](uint32_t k) { return min(kSelBins - 1, (int)((float)(k - mn) * scale)); };
    for (int i = threadIdx.x; i < kSelBins; i += NT) hist[i] = 0u;
    if (threadIdx.x == 0) s_ncand = 0u;
    __syncthreads();
    for (int i0 = threadIdx.x; i0 < n; i0 += CH * NT) {
      uint32_t k[CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int i = i0 + u * NT;
        k[u] = i < n ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (i0 + u * NT < n && k[u] >= mn && k[u] <= mx) atomicAdd(&hist[bin_of(k[u])], 1u);
    }
    __syncthreads();
    // bins from the top: thread t owns descending bins [t*per, (t+1)*per)
    constexpr int per = (kSelBins + NT - 1) / NT;
    const int q0 = threadIdx.x * per, q1 = min(q0 + per, kSelBins);
    uint32_t local = 0u;
    for (int q = q0; q < q1; ++q) local += hist[kSelBins - 1 - q];
    const uint32_t above = block_excl_scan<NT>(local, red, nullptr);
    if (above < r && above + local >= r) {  // exactly one thread holds the crossing
      uint32_t cum = above;
      for (int q = q0; q < q1; ++q) {
        const uint32_t c = hist[kSelBins - 1 - q];
        if (cum + c >= r) {
          s_bin = (uint32_t)(kSelBins - 1 - q);
          s_above = cum;
          s_cnt = c;
          break;
        }
        cum += c;
      }
    }
    __syncthreads();
    const int bin = (int)s_bin;
    const uint32_t cnt = s_cnt;
    r -= s_above;
    if (cnt <= (uint32_t)kSelCand) {
      // gather the bin's keys and rank them exactly: (key desc, index asc)
      for (int i0 = threadIdx.x; i0 < n; i0 += CH * NT) {
        uint32_t k[CH];
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          const int i = i0 + u * NT;
          k[u] = i < n ? keys[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          const int i = i0 + u * NT;
          if (i < n && k[u] >= mn && k[u] <= mx && bin_of(k[u]) == bin) {
            const uint32_t at = atomicAdd(&s_ncand, 1u);
            cand[2 * at] = k[u];
            cand[2 * at + 1] = (uint32_t)i;
          }
        }
      }
      __syncthreads();
      const int nc = (int)s_ncand;
      for (int c = threadIdx.x; c < nc; c += NT) {
        const uint32_t kc = cand[2 * c];
        const int ic = (int)cand[2 * c + 1];
        uint32_t rank = 0u;
        for (int o = 0; o < nc; ++o) {
          const uint32_t ko = cand[2 * o];
          const int io = (int)cand[2 * o + 1];
          rank += (ko > kc || (ko == kc && io < ic)) ? 1u : 0u;
        }
        if (rank == r - 1) s_res = Threshold{kc, ic};
      }
      __syncthreads();
      const Threshold t = s_res;
      __syncthreads();
      return t;
    }
    // too many keys in the bin: narrow the range to the bin's members and repeat
    uint32_t a2 = 0xffffffffu, b2 = 0u;
    for (int i0 = threadIdx.x; i0 < n; i0 += CH * NT) {
      uint32_t k[CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int i = i0 + u * NT;
        k[u] = i < n ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < CH; ++u)
        if (i0 + u * NT < n && k[u] >= mn && k[u] <= mx && bin_of(k[u]) == bin) {
          a2 = min(a2, k[u]);
          b2 = max(b2, k[u]);
        }
    }
    block_minmax_u32<NT>(a2, b2, red, lo, hi);
  }
  return Threshold{lo, n - 1};  // not reached for 32-bit keys (each round shrinks the range)
}

// Bin holding the r-th largest of kSelBins counts, scanned from the top in two levels:
// warp w (< 16) sums its 256 contiguous bins with conflict-free loads, warp 0 scans
// the 16 totals, and the warp whose chunk holds the crossing scans its 8 rows of 32
// bins. Results in *bin (the bin), *above (count in higher bins), *cnt (the bin's
// count). Requires NT >= 512. Every thread must call it.
template <int NT>
__device__ void hist_crossing(const uint32_t* __restrict__ hist, uint32_t r, uint32_t* red, int* bin,
                              uint32_t* above, uint32_t* cnt) {
  static_assert(NT >= 512, "needs 16 warps");
  __shared__ uint32_t s_w, s_wabove, s_bin, s_above, s_cnt;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < 16) {
    const int top = kSelBins - 1 - warp * 256;  // the warp's bins top, top-1, ..., top-255
    uint32_t t = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) t += hist[top - (j * 32 + lane)];
    t = __reduce_add_sync(0xffffffffu, t);
    if (lane == 0) red[warp] = t;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < 16 ? red[lane] : 0u;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const bool hit = lane < 16 && inc - v < r && inc >= r;
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    const int w = __ffs(m) - 1;
    if (lane == w) {
      s_w = (uint32_t)w;
      s_wabove = inc - v;
    }
  }
  __syncthreads();
  if (warp == (int)s_w) {
    const int top = kSelBins - 1 - warp * 256;
    uint32_t base = s_wabove;
    for (int j = 0; j < 8; ++j) {
      const uint32_t v = hist[top - (j * 32 + lane)];
      uint32_t inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t ab = base + inc - v;
      const uint32_t m = __ballot_sync(0xffffffffu, ab < r && ab + v >= r);
      if (m) {
        const int l = __ffs(m) - 1;
        if (lane == l) {
          s_bin = (uint32_t)(top - (j * 32 + l));
          s_above = ab;
          s_cnt = v;
        }
        break;
      }
      base = __shfl_sync(0xffffffffu, base + inc, 31);
    }
  }
  __syncthreads();
  *bin = (int)s_bin;
  *above = s_above;
  *cnt = s_cnt;
}

// ------------------------------------------------------------------------------------
// one-pass mean / variance (Welford per thread, Chan's pairwise merge across threads)
// ------------------------------------------------------------------------------------

// Block-wide sum of one double per thread in a fixed order: a shuffle tree inside each
// warp, then the warps' sums by a butterfly in which every pairwise add is commutative, so
// that all threads receive the same bits. `red` SMEM of >= NT/32 doubles. Contains two
// __syncthreads.
template <int NT>
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 32, "one warp combines the warps' sums");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = lane < NW ? red[lane] : 0.0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  __syncthreads();
  return t;
}

// ------------------------------------------------------------------------------------
// grid barriers (cooperative launches only: all CTAs must be co-resident)
// ------------------------------------------------------------------------------------

// Lives in the caller's workspace; zero-filled before first use.
struct GridBarrier {
  unsigned count;            // grid_sync: arrivals of the current barrier (back to 0 after each)
  unsigned gen;              // grid_sync: completed barriers
  unsigned long long total;  // grid_sync_fixed: arrivals ever made
  unsigned pad[28];
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long atom_add_release_u64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

// Sense-counting barrier that works for any grid size: the last arriver resets `count`
// and bumps `gen`. Returns false if this CTA gave up waiting (WINA_ERR_TIMEOUT is
// recorded); the caller must then return without touching shared results.
__device__ __forceinline__ bool grid_sync(GridBarrier* bar, unsigned nblocks, int32_t* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned g0 = ld_acquire_u32(&bar->gen);
    __threadfence();
    const unsigned old = atomicAdd(&bar->count, 1u);
    if (old == nblocks - 1u) {
      atomicExch(&bar->count, 0u);
      __threadfence();
      atomicAdd(&bar->gen, 1u);
    } else {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_u32(&bar->gen) == g0) {
        if (globaltimer_ns() - t0 > kBarrierTimeoutNs) {
          ok = 0;
          record_status(status, WINA_ERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// Barrier for kernels whose grid size never changes for a given workspace: arrivals
// accumulate in a 64-bit counter, so barrier k of the workspace's life completes when
// the counter reaches (k + 1) * nblocks. One release atomic per CTA and acquire polls;
// the last arriver does no extra round trip. Same failure contract as grid_sync, with
// the wait limit given by the caller.
__device__ __forceinline__ bool grid_sync_fixed(GridBarrier* bar, unsigned nblocks, int32_t* status,
                                                unsigned long long limit_ns = kBarrierTimeoutNs) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned long long old = atom_add_release_u64(&bar->total, 1ull);
    const unsigned long long target = old - old % nblocks + nblocks;
    if (ld_acquire_u64(&bar->total) < target) {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_u64(&bar->total) < target) {
        if (globaltimer_ns() - t0 > limit_ns) {
          ok = 0;
          record_status(status, WINA_ERR_TIMEOUT);
          break;
        }
        __nanosleep(20);
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// ------------------------------------------------------------------------------------
// the sparse product's inner loop (SVMM over a CTA's share of kept rows)
// ------------------------------------------------------------------------------------

// One 16-byte vector of weights times a scalar, accumulated in float32.
template <bool BF16>
struct VecOps;

template <>
struct VecOps<true> {
  static constexpr int EPV = 8;  // bf16 per 16 bytes
  __device__ __forceinline__ static void fma(float* acc, const uint4& w, float x) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] = fmaf(__uint_as_float(ws[q] << 16), x, acc[2 * q]);
      acc[2 * q + 1] = fmaf(__uint_as_float(ws[q] & 0xffff0000u), x, acc[2 * q + 1]);
    }
  }
};

template <>
struct VecOps<false> {
  static constexpr int EPV = 4;  // f32 per 16 bytes
  __device__ __forceinline__ static void fma(float* acc, const uint4& w, float x) {
    acc[0] = fmaf(__uint_as_float(w.x), x, acc[0]);
    acc[1] = fmaf(__uint_as_float(w.y), x, acc[1]);
    acc[2] = fmaf(__uint_as_float(w.z), x, acc[2]);
    acc[3] = fmaf(__uint_as_float(w.w), x, acc[3]);
  }
};

// Thread layout for rows of V 16-byte vectors: the block is split into NG = NT / TPR
// groups of TPR threads; group g takes rows g, g + NG, ...; lane l of a group owns
// vectors l, l + TPR, ..., (VPT of them).
struct RowLayout {
  int V;    // vectors per row
  int TPR;  // threads per row
  int NG;   // row groups
  int VPT;  // vectors per thread
};

template <int NT>
__host__ __device__ inline RowLayout make_row_layout(int64_t m, int epv) {
  RowLayout L;
  L.V = (int)(m / epv);
  int t = 32;
  while (t < L.V && t < NT) t <<= 1;
  L.TPR = t;
  L.NG = NT / t;
  L.VPT = (L.V + t - 1) / t;
  return L;
}

// acc[j][e] += sum over this group's rows r of vals[r] * Wt[rows[r]][(l + j*TPR)*EPV + e].
// rows/vals are the CTA's share in SMEM (nrows entries). U rows are in flight at once
// per thread (U * VPT 16-byte loads).
template <bool BF16, int VPT, int U>
__device__ __forceinline__ void accumulate_rows(const void* __restrict__ Wt, const RowLayout& L,
                                                const int32_t* rows, const float* vals, int nrows,
                                                float (&acc)[VPT][VecOps<BF16>::EPV], uint64_t pol) {
  const int g = threadIdx.x / L.TPR;
  const int l = threadIdx.x % L.TPR;
  const uint4* base = reinterpret_cast<const uint4*>(Wt);
  const int64_t V = L.V;
  int r = g;
  const int step = L.NG;
  for (; r + (U - 1) * step < nrows; r += U * step) {
    uint4 w[U][VPT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint4* rp = base + (int64_t)rows[r + u * step] * V;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = l + j * L.TPR;
        if (v < L.V) w[u][j] = ld_stream_u4(rp + v, pol);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float xv = vals[r + u * step];
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = l + j * L.TPR;
        if (v < L.V) VecOps<BF16>::fma(acc[j], w[u][j], xv);
      }
    }
  }
  for (; r < nrows; r += step) {
    const uint4* rp = base + (int64_t)rows[r] * V;
    const float xv = vals[r];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = l + j * L.TPR;
      if (v < L.V) VecOps<BF16>::fma(acc[j], ld_stream_u4(rp + v, pol), xv);
    }
  }
}

// Sum the NG group accumulators of a CTA and store the CTA's partial row out[0..m)
// (float32, 16-byte aligned). With NG > 1 a row fits in one group (VPT == 1), so `red`
// needs NG * m <= NT * EPV floats of SMEM. Deterministic: groups are added in order.
template <bool BF16, int VPT>
__device__ __forceinline__ void store_partial(float* __restrict__ out, const RowLayout& L,
                                              float (&acc)[VPT][VecOps<BF16>::EPV], float* red) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int g = threadIdx.x / L.TPR;
  const int l = threadIdx.x % L.TPR;
  const int m = L.V * EPV;
  if (L.NG == 1) {
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = l + j * L.TPR;
      if (v < L.V) {
        float4* o = reinterpret_cast<float4*>(out + (int64_t)v * EPV);
#pragma unroll
        for (int q = 0; q < EPV / 4; ++q)
          o[q] = make_float4(acc[j][4 * q], acc[j][4 * q + 1], acc[j][4 * q + 2], acc[j][4 * q + 3]);
      }
    }
    return;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = l + j * L.TPR;
    if (v < L.V) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) red[(int64_t)g * m + v * EPV + e] = acc[j][e];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < m; c += L.NG * L.TPR) {
    float s = 0.f;
    for (int gg = 0; gg < L.NG; ++gg) s += red[(int64_t)gg * m + c];
    out[c] = s;
  }
  __syncthreads();
}

}  // namespace wina
