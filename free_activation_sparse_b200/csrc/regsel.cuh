// Exact top-K selection with the keys held in registers by a CTA of 1024 threads (thread
// t owns channels t, t + 1024, ...): a radix select on the float32 key bits (scores are
// >= 0, so their bit patterns order like the floats), ties to the lower channel, and the
// kept set as channel flags. Used by the single-token FFN kernel and the batched gate.
#pragma once

#include "common.cuh"

namespace wina {

constexpr int kDT = 1024;       // threads per CTA
constexpr int kDW = kDT / 32;   // warps per CTA
constexpr int kDKeys = 16;      // channels per thread at most (vectors of up to 16384)
constexpr int kDMaxN = kDT * kDKeys;

// ------------------------------------------------------------------------------------
// selection with the keys in registers
// ------------------------------------------------------------------------------------

// Bin holding the r-th largest of `nb` counts (nb <= 256), from the top: one warp, each
// lane summing nb/32 consecutive bins. Writes bin, count above, the bin's count.
__device__ __forceinline__ void small_crossing(const uint32_t* h, int nb, uint32_t r, uint32_t* out3) {
  const int lane = threadIdx.x & 31;
  const int per = nb / 32;  // 8 for 256 bins; nb >= 32 and a multiple of 32
  uint32_t v[8], t = 0u;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    v[e] = e < per ? h[nb - 1 - per * lane - e] : 0u;
    t += v[e];
  }
  uint32_t x = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  uint32_t ab = x - t;
  const bool hit = ab < r && ab + t >= r;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if (hit && e < per && ab < r && ab + v[e] >= r) {
      out3[0] = (uint32_t)(nb - 1 - per * lane - e);
      out3[1] = ab;
      out3[2] = v[e];
    }
    ab += v[e];
  }
}

// Exact top-K of the keys held in registers (thread t owns channels t + i * kDT, i < kpt,
// those >= n absent), ties to the lower channel, as a threshold: kept(j) <=> key_j > T or
// (key_j == T and j <= cut). Radix passes on bits 30..19, 18..11, 10..3 and 2..0 of the
// keys, each restricted to the keys that share the prefix found so far, stop as soon as
// every key of the crossing bin is kept. Every thread must call it. hist: SMEM of
// kSelBins + 256 words, zero on entry (see clear_hist).
template <int KMAX>
__device__ __forceinline__ Threshold radix_select_regs(const uint32_t (&key)[KMAX], int kpt, int n, int K,
                                                       uint32_t* hist) {
  __shared__ uint32_t s_x[4];
  __shared__ Threshold s_t;
  __shared__ uint32_t s_cnt[kDW];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (K <= 0) return Threshold{0xffffffffu, -1};
  if (K >= n) return Threshold{0u, n - 1};
  uint32_t r = (uint32_t)K;
  // pass 1: 12-bit digit (bit 31 of a non-negative float is 0); the caller zeroed hist
#pragma unroll
  for (int i = 0; i < KMAX; ++i)
    if (i < kpt && t + i * kDT < n) atomicAdd(&hist[key[i] >> 19], 1u);
  __syncthreads();
  {
    int bin;
    uint32_t above, cnt;
    hist_crossing<kDT>(hist, r, s_cnt, &bin, &above, &cnt);  // ends with __syncthreads
    r -= above;
    uint32_t prefix = (uint32_t)bin;
    int shift = 19;
    if (r == cnt) return Threshold{prefix << shift, n - 1};  // every key of the bin is kept
    // passes 2-4: bits 18..11, 10..3, 2..0
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
      const int w = p < 2 ? 8 : 3;
      const int nb = 1 << w;
      const int nsh = shift - w;
      uint32_t* sub = hist + kSelBins;
      if (p > 0) {  // zeroed by the caller for the first of these passes
        if (t < 256) sub[t] = 0u;
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < KMAX; ++i)
        if (i < kpt && t + i * kDT < n && (key[i] >> shift) == prefix) atomicAdd(&sub[(key[i] >> nsh) & (nb - 1)], 1u);
      __syncthreads();
      if (warp == 0) {
        if (nb >= 32) {
          small_crossing(sub, nb, r, s_x);
        } else {
          // 8 bins: lane l < 8 holds bin 7 - l
          const uint32_t v = lane < nb ? sub[nb - 1 - lane] : 0u;
          uint32_t x = v;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
          const uint32_t ab = x - v;
          if (lane < nb && ab < r && ab + v >= r) {
            s_x[0] = (uint32_t)(nb - 1 - lane);
            s_x[1] = ab;
            s_x[2] = v;
          }
        }
      }
      __syncthreads();
      const uint32_t b2 = s_x[0], ab2 = s_x[1], c2 = s_x[2];
      __syncthreads();
      r -= ab2;
      prefix = (prefix << w) | b2;
      shift = nsh;
      if (r == c2) return Threshold{prefix << shift, n - 1};
    }
    // all 31 bits resolved: the keys equal to T = prefix; keep the r lowest channels
    const uint32_t T = prefix;
    // counts of equal keys per register slot i (channels i*kDT .. i*kDT + kDT - 1)
    int islot = 0;
    uint32_t before = 0u;
#pragma unroll 1
    for (int i = 0; i < kpt; ++i) {
      uint32_t ki = 0u;
#pragma unroll
      for (int q = 0; q < KMAX; ++q)
        if (q == i) ki = key[q];
      const int c = __syncthreads_count(t + i * kDT < n && ki == T);
      if (before + (uint32_t)c >= r) {
        islot = i;
        break;
      }
      before += (uint32_t)c;
    }
    uint32_t ki = 0u;
#pragma unroll
    for (int q = 0; q < KMAX; ++q)
      if (q == islot) ki = key[q];
    const bool eq = t + islot * kDT < n && ki == T;
    const uint32_t m = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_cnt[warp] = (uint32_t)__popc(m);
    __syncthreads();
    if (warp == 0) {
      const uint32_t v = s_cnt[lane];
      uint32_t x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      s_cnt[lane] = x - v;  // equal keys in lower warps
    }
    __syncthreads();
    const uint32_t rr = r - before;  // the rr-th equal key of slot islot (1-based) is the cut
    const uint32_t lower = s_cnt[warp] + (uint32_t)__popc(m & ((1u << lane) - 1u));
    if (eq && lower + 1u == rr) s_t = Threshold{T, t + islot * kDT};
    __syncthreads();
    const Threshold res = s_t;
    __syncthreads();
    return res;
  }
}

__device__ __forceinline__ void clear_hist(uint32_t* hist) {
  for (int i = threadIdx.x; i < kSelBins + 256; i += kDT) hist[i] = 0u;
}

// Flags of a threshold over the register-held keys: bit l of word w = channel 32w + l.
template <int KMAX>
__device__ __forceinline__ void flags_from_keys(const uint32_t (&key)[KMAX], int kpt, int n, Threshold th,
                                                uint32_t* flags) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    if (i < kpt) {
      const int j = t + i * kDT;
      const bool k = j < n && (key[i] > th.T || (key[i] == th.T && j <= th.cut));
      const uint32_t bits = __ballot_sync(0xffffffffu, k);
      const int w = i * kDW + warp;
      if (lane == 0 && w < (n + 31) / 32) flags[w] = bits;
    }
  }
}

// Spark threshold on register-held values: mu + sigma * z, moments in float64
// (Welford per thread, Chan's pairwise merge in a fixed order), strict v > t.

}  // namespace wina
