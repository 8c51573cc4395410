// SwiGLU FFN decode with the gate on every projection ("WAS" article, core innovations:
// weight-aware sparsity per component, gate/up/down among them; "WINA" article,
// section 一: each projection scores with its own column norms and its own K).
//
// One token: a single persistent cooperative kernel, one CTA per SM, 16 consumer warps
// and one producer warp.
//   A  CTAs [0, Gg) work on the gate projection, the rest on up. Each CTA scores x
//      against its projection's c in SMEM, finds the K-th largest score by radix select
//      (or the Spark threshold, or keeps everything) and turns the result into a
//      kept-channel bitmask.
//   B  The producer warp takes units of a few channels from a global counter (dynamic
//      load balance across the CTAs of the projection), and for each kept channel
//      copies the whole input-major weight row HBM -> SMEM with a bulk copy into a ring
//      of stages (full/empty mbarriers). Consumer warps accumulate x_j * row_j in
//      float32 registers and finally store one partial row per CTA.
//      At the end each CTA adds its row sums into g or u (vector float atomics at L2).
//   -- grid barrier --
//   C  Every CTA reads the complete g and u, computes h = silu(g) * u and the down
//      gate's scores |h_j * c_down_j| for all ffn channels, and selects the kept down
//      channels itself (bitmask).
//   E  As B, over the down projection's rows (d wide), all CTAs together; row sums are
//      added into y's accumulator.
//   F  The last CTA to finish (a counter) copies y out and clears the accumulators.
// Every wait (grid barrier, ring stage) is bounded in time; on a timeout the kernel
// records WINA_ERR_TIMEOUT, waits (bounded) for its own copies in flight and returns.
// Several tokens: the batched calls (select, sparse_matvec, silu*mul, select,
// sparse_matvec) in sequence.
#include <math.h>

#include <algorithm>
#include <cmath>

#include "internal.h"
#include "pipeline.cuh"

namespace wina {

constexpr int kCW = 16;                  // consumer warps
constexpr int kCT = kCW * 32;            // consumer threads
constexpr int kFT = kCT + 32;            // threads per CTA (consumers + one producer warp)
constexpr int kMaxStages = 16;           // ring stages at most
constexpr size_t kMaxSmem = 224 * 1024;  // dynamic SMEM per CTA (227 KB per block on sm_100, less static)

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
  int Gg;             // CTAs on the gate projection in phase B
  int uw_b, uw_e;     // channels per work unit in phases B and E
  int S_b, S_e;       // ring stages in phases B and E
  GridBarrier* bar;
  unsigned* ctr;  // [3] unit counters: gate, up, down
  float* h;
  uint8_t* keep_g;
  uint8_t* keep_u;
  uint8_t* keep_d;
  long long* stamps;
  unsigned long long* cta_t;
  unsigned long long* trace;  // CTA 0: phase B [0..63] issued, [64..127] ready; phase E [128..255]
  float* acc_g;     // [2][ffn] float32 sums of the gate rows, one buffer per call parity
  float* acc_u;     // [2][ffn] float32 sums of the up rows, one buffer per call parity
  float* acc_y;     // [d] float32 sums of the down rows (zero between calls)
  unsigned* done;   // CTAs that finished phase E (zero between calls)
  unsigned* epoch;  // calls completed on this workspace (picks the parity)
  int32_t* status;
};

struct SmemLayout {
  uint32_t keys, vals, flags, meta_val, meta_row, bars, ring, hist, cand;
};

// keys | vals | flags | stage metadata | mbarriers | ring. The selection's histogram and
// candidate list overlay the start of the ring, which is idle while a selection runs.
__host__ __device__ inline SmemLayout ffn_smem_layout(int d, int ffn) {
  SmemLayout L;
  const uint32_t nb = (uint32_t)(d > ffn ? d : ffn);
  uint32_t o = 0;
  auto take = [&](uint32_t bytes, uint32_t align) {
    o = (o + align - 1) / align * align;
    const uint32_t at = o;
    o += bytes;
    return at;
  };
  L.keys = take(nb * 4, 16);
  L.vals = take(nb * 4, 16);
  L.flags = take((nb + 31) / 32 * 4, 16);
  L.meta_val = take(kMaxStages * 4, 16);
  L.meta_row = take(kMaxStages * 4, 16);
  L.bars = take(2 * kMaxStages * 8, 16);
  L.ring = take(0, 128);
  L.hist = L.ring;
  L.cand = L.ring + kSelBins * 4;
  return L;
}

// Smallest ring the layout needs (the selection scratch lives in it).
constexpr uint32_t kMinRing = (kSelBins + 2 * kSelCand) * 4;

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// CTA 0 records its SM clock at phase boundaries; every CTA records the global timer at
// the end of its four main phases (diagnostic views of the workspace).
__device__ __forceinline__ void stamp(long long* stamps, int i) {
  if (blockIdx.x == 0 && threadIdx.x == 0) stamps[i] = clock64();
}
__device__ __forceinline__ void cta_time(unsigned long long* t, int i) {
  if (threadIdx.x == 0) t[blockIdx.x * 4 + i] = globaltimer_ns();
}

// ------------------------------------------------------------------------------------
// kept-channel bitmask
// ------------------------------------------------------------------------------------

// flags[w] bit l = channel 32w + l is kept by the top-K threshold.
__device__ void flags_from_topk(const uint32_t* keys, int n, const Threshold& t, uint32_t* flags) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (n + 31) / 32;
  for (int w = warp; w < nw; w += kFT / 32) {
    const int j = w * 32 + lane;
    const bool k = j < n && kept_by(t, keys[j], j);
    const uint32_t bits = __ballot_sync(0xffffffffu, k);
    if (lane == 0) flags[w] = bits;
  }
}

// flags for the Spark threshold: v_j > t (float64 comparison).
__device__ void flags_from_threshold(const float* v, int n, double t, uint32_t* flags) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (n + 31) / 32;
  for (int w = warp; w < nw; w += kFT / 32) {
    const int j = w * 32 + lane;
    const bool k = j < n && (double)v[j] > t;
    const uint32_t bits = __ballot_sync(0xffffffffu, k);
    if (lane == 0) flags[w] = bits;
  }
}

__device__ void flags_all(int n, uint32_t* flags) {
  const int nw = (n + 31) / 32;
  for (int w = threadIdx.x; w < nw; w += kFT) {
    const int rem = n - w * 32;
    flags[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
  }
}

// Byte flags for the workspace's diagnostic view.
__device__ void write_keep_bytes(const uint32_t* flags, int n, uint8_t* out) {
  for (int j = threadIdx.x; j < n; j += kFT) out[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
}

// Spark threshold of v[0..n) in SMEM: mu + sigma * z, moments in float64.
__device__ double spark_threshold(const float* v, int n, double z, double* dred) {
  Moments mo{0.0, 0.0, 0.0};
  for (int i = threadIdx.x; i < n; i += kFT) {
    const double f = (double)v[i];
    mo.n += 1.0;
    const double dl = f - mo.mean;
    mo.mean += dl / mo.n;
    mo.m2 += dl * (f - mo.mean);
  }
  const Moments tot = block_moments<kFT>(mo, dred);
  return tot.mean + sqrt(tot.m2 / (double)n) * z;
}

// ------------------------------------------------------------------------------------
// the row ring: producer and consumers
// ------------------------------------------------------------------------------------

struct Ring {
  char* base;      // SMEM
  uint64_t* full;  // [kMaxStages]
  uint64_t* empty;  // [kMaxStages]
  float* meta_val;  // x_j (or h_j) of the row in each stage
  int* meta_row;    // row index of each stage, -1 = end of phase
};

// Producer state kept across phases (per-stage mbarrier parities).
struct ProdState {
  uint32_t used;       // stage has been filled before
  uint32_t empty_par;  // parity of the next completion to wait for on empty[s]
  uint32_t full_par;   // parity of the next phase on full[s] (last issued = bit ^ 1)
};

// Streams the kept rows of channels [0, n) unit by unit (units of `uw` <= 32 channels
// taken from the global counter `ctr`) into the ring, then an end-of-phase marker. Runs
// on the producer warp. The kept rows of a unit are issued by as many lanes at once (a
// single thread issuing bulk copies one after another is far too slow to fill HBM), in
// rounds of at most S rows so that the stages of a round are distinct. Lane 0 keeps
// kGrab unit requests in flight, each in its own register, so that a request's counter
// round trip is waited on only when that unit is next (a shuffle of a register with a
// load still pending would stall on it). Returns false on a timeout.
constexpr int kGrab = 2;
__device__ bool produce(const Ring& R, int S, uint32_t row_bytes, const char* __restrict__ Wt, int n, int uw,
                        unsigned* ctr, const uint32_t* flags, const float* vals, ProdState& ps, uint64_t pol,
                        unsigned long long* trace = nullptr) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const unsigned nunits = (unsigned)((n + uw - 1) / uw);
  int stage = 0;
  unsigned pend[kGrab];
#pragma unroll
  for (int q = 0; q < kGrab; ++q) pend[q] = lane == 0 ? atomicAdd(ctr, 1u) : 0u;
  uint32_t live = (1u << kGrab) - 1u;
  bool ok = true;
  while (live) {
#pragma unroll
    for (int q = 0; q < kGrab; ++q) {
      if (!((live >> q) & 1u)) continue;  // uniform across the warp
      unsigned unit = lane == 0 ? pend[q] : 0u;
      unit = __shfl_sync(0xffffffffu, unit, 0);
      if (unit >= nunits) {
        live &= ~(1u << q);
        continue;
      }
      if (lane == 0) pend[q] = atomicAdd(ctr, 1u);  // refill this request
      const int j0 = (int)unit * uw;
      const int j = j0 + lane;
      const bool k = lane < uw && j < n && ((flags[j >> 5] >> (j & 31)) & 1u);
      const uint32_t m = __ballot_sync(0xffffffffu, k);
      const int cnt = __popc(m);
      const int pos = __popc(m & lt);
      for (int r0 = 0; r0 < cnt; r0 += S) {
        const int nr = min(S, cnt - r0);
        if (k && pos >= r0 && pos < r0 + nr) {
          const int s = (stage + pos - r0) % S;
          bool mine_ok = true;
          if ((ps.used >> s) & 1u) mine_ok = mbar_wait(&R.empty[s], (ps.empty_par >> s) & 1u);
          if (mine_ok) {
            R.meta_val[s] = vals[j];
            R.meta_row[s] = j;
            mbar_arrive_expect_tx(&R.full[s], row_bytes);
            bulk_copy_g2s(R.base + (size_t)s * row_bytes, Wt + (size_t)j * row_bytes, row_bytes, &R.full[s], pol);
            if (trace && stage + pos - r0 < 64) trace[stage + pos - r0] = globaltimer_ns();
          } else {
            ok = false;
          }
        }
        // the same state update in every lane: nr consecutive stages were filled
        for (int i = 0; i < nr; ++i) {
          const int s = (stage + i) % S;
          if ((ps.used >> s) & 1u) ps.empty_par ^= 1u << s;
          ps.used |= 1u << s;
          ps.full_par ^= 1u << s;
        }
        stage += nr;
        if (__any_sync(0xffffffffu, !ok)) return false;
      }
    }
  }
  // end-of-phase marker: completes a stage with no bytes
  if (lane == 0) {
    const int s = stage % S;
    if ((ps.used >> s) & 1u) {
      if (!mbar_wait(&R.empty[s], (ps.empty_par >> s) & 1u)) ok = false;
    }
    if (ok) {
      R.meta_val[s] = 0.f;
      R.meta_row[s] = -1;
      mbar_arrive(&R.full[s]);
    }
  }
  {
    const int s = stage % S;
    if ((ps.used >> s) & 1u) ps.empty_par ^= 1u << s;
    ps.used |= 1u << s;
    ps.full_par ^= 1u << s;
  }
  return __shfl_sync(0xffffffffu, ok, 0);
}

// Waits (bounded) until every copy the producer issued has landed, so that the CTA may
// exit without bulk copies still writing into its shared memory.
__device__ void drain(const Ring& R, const ProdState& ps) {
  if ((threadIdx.x & 31) != 0) return;
  for (int s = 0; s < kMaxStages; ++s)
    if ((ps.used >> s) & 1u) mbar_wait(&R.full[s], ((ps.full_par >> s) & 1u) ^ 1u);
}

// Consumer warps: take stages in order until the end marker, accumulating
// meta_val * row into acc (thread t owns 16-byte vectors t, t + kCT, ...).
template <bool BF16, int VPT>
__device__ bool consume_t(const Ring& R, int S, uint32_t row_bytes, int V, uint32_t& full_par,
                          float (&acc)[VPT][VecOps<BF16>::EPV], unsigned long long* trace, int& rows) {
  const int t = threadIdx.x, lane = t & 31;
  const uint32_t ring = smem_addr(R.base);
  int stage = 0;
  while (true) {
    const int s = stage % S;
    if (!mbar_wait(&R.full[s], (full_par >> s) & 1u)) return false;
    if (trace && t == 0 && stage < 64) trace[64 + stage] = globaltimer_ns();
    full_par ^= 1u << s;
    const int row = R.meta_row[s];
    if (row >= 0) {
      ++rows;
      const float xv = R.meta_val[s];
      const uint32_t src = ring + (uint32_t)s * row_bytes;
      uint4 w[VPT];
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = t + j * kCT;
        if (v < V) w[j] = ld_shared_u4(src + (uint32_t)v * 16u);
      }
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int v = t + j * kCT;
        if (v < V) VecOps<BF16>::fma(acc[j], w[j], xv);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&R.empty[s]);
    if (row < 0) return true;
    ++stage;
  }
}

__device__ __forceinline__ void red_add_f4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Consume one phase, then add the CTA's float32 row sums into out[0..m) (vector
// atomics at L2; the order of the CTAs' additions is not fixed).
template <bool BF16, int VPT>
__device__ bool consume_store_t(const Ring& R, int S, uint32_t row_bytes, int V, uint32_t& full_par,
                                float* __restrict__ out, unsigned long long* trace) {
  constexpr int EPV = VecOps<BF16>::EPV;
  float acc[VPT][EPV];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[j][e] = 0.f;
  int rows = 0;
  const bool ok = consume_t<BF16, VPT>(R, S, row_bytes, V, full_par, acc, trace, rows);
  if (rows == 0) return ok;  // nothing to add
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = threadIdx.x + j * kCT;
    if (v < V) {
      float* o = out + (int64_t)v * EPV;
#pragma unroll
      for (int q = 0; q < EPV / 4; ++q)
        red_add_f4(o + 4 * q, acc[j][4 * q], acc[j][4 * q + 1], acc[j][4 * q + 2], acc[j][4 * q + 3]);
    }
  }
  __threadfence();  // this thread's additions are ordered before the CTA's next barrier / hand-off
  return ok;
}

// Consume one phase and store the CTA's partial row out[0..m).
template <bool BF16>
__device__ bool consume_store(const Ring& R, int S, uint32_t row_bytes, int m, uint32_t& full_par, float* out,
                              unsigned long long* trace = nullptr) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int V = m / EPV;
  const int vpt = (V + kCT - 1) / kCT;
  switch (vpt) {
    case 1: return consume_store_t<BF16, 1>(R, S, row_bytes, V, full_par, out, trace);
    case 2: return consume_store_t<BF16, 2>(R, S, row_bytes, V, full_par, out, trace);
    case 3: return consume_store_t<BF16, 3>(R, S, row_bytes, V, full_par, out, trace);
    case 4: return consume_store_t<BF16, 4>(R, S, row_bytes, V, full_par, out, trace);
    case 5: return consume_store_t<BF16, 5>(R, S, row_bytes, V, full_par, out, trace);
    case 6: return consume_store_t<BF16, 6>(R, S, row_bytes, V, full_par, out, trace);
    case 7: return consume_store_t<BF16, 7>(R, S, row_bytes, V, full_par, out, trace);
    default: return consume_store_t<BF16, 8>(R, S, row_bytes, V, full_par, out, trace);
  }
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------

template <bool BF16>
__global__ void __launch_bounds__(kFT, 1) k_ffn_fused(FfnParams a) {
  constexpr uint32_t ESZ = BF16 ? 2u : 4u;
  extern __shared__ __align__(128) unsigned char smraw[];
  const int d = a.d, ffn = a.ffn;
  const SmemLayout SL = ffn_smem_layout(d, ffn);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smraw + SL.keys);
  float* vals = reinterpret_cast<float*>(smraw + SL.vals);
  uint32_t* flags = reinterpret_cast<uint32_t*>(smraw + SL.flags);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smraw + SL.hist);
  uint32_t* cand = reinterpret_cast<uint32_t*>(smraw + SL.cand);
  Ring R;
  R.meta_val = reinterpret_cast<float*>(smraw + SL.meta_val);
  R.meta_row = reinterpret_cast<int*>(smraw + SL.meta_row);
  R.full = reinterpret_cast<uint64_t*>(smraw + SL.bars);
  R.empty = R.full + kMaxStages;
  R.base = reinterpret_cast<char*>(smraw + SL.ring);
  __shared__ uint32_t red[2 * kFT / 32 + 8];
  __shared__ double dred[3 * kFT / 32];
  __shared__ int s_abort, s_last;

  const int G = gridDim.x, b = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const bool producer = warp == kCW;
  const uint64_t pol = l2_evict_first_policy();
  stamp(a.stamps, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&R.full[s], 1u);
      mbar_init(&R.empty[s], (uint32_t)kCW);
    }
    mbar_init_fence();
    s_abort = 0;
  }
  ProdState ps{0u, 0u, 0u};
  uint32_t full_par = 0u;

  // this call's g/u sum buffers; the other parity's (last used by the previous call,
  // whose readers have all finished) is cleared here for the next call
  const unsigned par = __ldcg(a.epoch) & 1u;
  float* acc_g = a.acc_g + (size_t)par * ffn;
  float* acc_u = a.acc_u + (size_t)par * ffn;
  {
    float4* cg = reinterpret_cast<float4*>(a.acc_g + (size_t)(par ^ 1u) * ffn);
    float4* cu = reinterpret_cast<float4*>(a.acc_u + (size_t)(par ^ 1u) * ffn);
    const int64_t m4 = ffn / 4;
    for (int64_t q = m4 * b / G + threadIdx.x; q < m4 * (b + 1) / G; q += kFT) {
      __stcg(cg + q, make_float4(0.f, 0.f, 0.f, 0.f));
      __stcg(cu + q, make_float4(0.f, 0.f, 0.f, 0.f));
    }
  }

  // ---------------- A: this CTA's projection, its kept-channel bitmask ----------------
  const bool gate = b < a.Gg;
  const int rank = gate ? b : b - a.Gg;
  const float* cproj = gate ? a.c_gate : a.c_up;
  {
    // all of this thread's loads are issued before any SMEM store (a store through a
    // generic pointer could alias the inputs, which would serialise the round trips)
    constexpr int U = 8;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i0 = threadIdx.x; i0 < d; i0 += U * kFT) {
      float xv[U], cv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kFT;
        xv[u] = i < d ? load_elem(a.x, a.xdt, i) : 0.f;
        cv[u] = (i < d && a.mode == WINA_GATE_TOPK) ? __ldg(cproj + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kFT;
        if (i < d) {
          vals[i] = xv[u];
          if (a.mode == WINA_GATE_TOPK) {
            const uint32_t k = __float_as_uint(fabsf(xv[u] * cv[u]));
            keys[i] = k;
            kmin = min(kmin, k);
            kmax = max(kmax, k);
          }
        }
      }
    }
    if (a.mode == WINA_GATE_TOPK) {
      uint32_t mn, mx;
      block_minmax_u32<kFT>(kmin, kmax, red, mn, mx);  // contains the barrier after the loads
      select_topk_flags<kFT>(keys, d, gate ? a.k_gate : a.k_up, mn, mx, hist, cand, red, flags);
    } else {
      __syncthreads();
      if (a.mode == WINA_GATE_STAT)
        flags_from_threshold(vals, d, spark_threshold(vals, d, a.z, dred), flags);
      else
        flags_all(d, flags);
    }
  }
  __syncthreads();
  if (rank == (gate ? a.Gg : G - a.Gg) - 1) write_keep_bytes(flags, d, gate ? a.keep_g : a.keep_u);
  stamp(a.stamps, 1);
  cta_time(a.cta_t, 0);

  // ---------------- B: stream kept gate / up rows through the ring ----------------
  {
    const uint32_t row_bytes = (uint32_t)ffn * ESZ;
    if (producer) {
      const bool ok = produce(R, a.S_b, row_bytes, reinterpret_cast<const char*>(gate ? a.wt_gate : a.wt_up), d,
                              a.uw_b, a.ctr + (gate ? 0 : 1), flags, vals, ps, pol, b == 0 ? a.trace : nullptr);
      if (!ok && (threadIdx.x & 31) == 0) s_abort = 1;
    } else {
      if (!consume_store<BF16>(R, a.S_b, row_bytes, ffn, full_par, gate ? acc_g : acc_u,
                               b == 0 ? a.trace : nullptr))
        s_abort = 1;
    }
  }
  __syncthreads();
  if (s_abort) {
    record_status(a.status, WINA_ERR_TIMEOUT);
    if (producer) drain(R, ps);
    return;
  }
  stamp(a.stamps, 2);
  cta_time(a.cta_t, 1);
  if (!grid_sync_fixed(a.bar, G, a.status)) return;
  stamp(a.stamps, 3);

  // ---------------- C/D: h for every channel, the down scores, the down bitmask ----------------
  if (b == 0 && threadIdx.x == 0) {
    a.ctr[0] = 0u;  // every CTA is past phase B: the gate/up unit counters can be reset
    a.ctr[1] = 0u;
  }
  {
    constexpr int U = 3;  // float4 columns per thread per round, all loads issued first
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    const int m4 = ffn / 4;
    const bool topk = a.mode == WINA_GATE_TOPK;
    for (int q0 = threadIdx.x; q0 < m4; q0 += U * kFT) {
      float4 g4[U], u4[U], c4[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int q = q0 + u * kFT;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        g4[u] = q < m4 ? __ldcg(reinterpret_cast<const float4*>(acc_g) + q) : z;
        u4[u] = q < m4 ? __ldcg(reinterpret_cast<const float4*>(acc_u) + q) : z;
        c4[u] = (q < m4 && topk) ? __ldg(reinterpret_cast<const float4*>(a.c_down) + q) : z;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int q = q0 + u * kFT;
        if (q >= m4) continue;
        float4 h4;
        h4.x = silu_f(g4[u].x) * u4[u].x;
        h4.y = silu_f(g4[u].y) * u4[u].y;
        h4.z = silu_f(g4[u].z) * u4[u].z;
        h4.w = silu_f(g4[u].w) * u4[u].w;
        reinterpret_cast<float4*>(vals)[q] = h4;
        if (b == G - 1) reinterpret_cast<float4*>(a.h)[q] = h4;
        if (topk) {
          uint4 k4;
          k4.x = __float_as_uint(fabsf(h4.x * c4[u].x));
          k4.y = __float_as_uint(fabsf(h4.y * c4[u].y));
          k4.z = __float_as_uint(fabsf(h4.z * c4[u].z));
          k4.w = __float_as_uint(fabsf(h4.w * c4[u].w));
          reinterpret_cast<uint4*>(keys)[q] = k4;
          kmin = min(min(kmin, min(k4.x, k4.y)), min(k4.z, k4.w));
          kmax = max(max(kmax, max(k4.x, k4.y)), max(k4.z, k4.w));
        }
      }
    }
    stamp(a.stamps, 4);
    if (a.mode == WINA_GATE_TOPK) {
      uint32_t mn, mx;
      block_minmax_u32<kFT>(kmin, kmax, red, mn, mx);
      stamp(a.stamps, 11);
      select_topk_flags<kFT>(keys, ffn, a.k_down, mn, mx, hist, cand, red, flags);
    } else {
      __syncthreads();
      stamp(a.stamps, 11);
      if (a.mode == WINA_GATE_STAT)
        flags_from_threshold(vals, ffn, spark_threshold(vals, ffn, a.z, dred), flags);
      else
        flags_all(ffn, flags);
    }
  }
  __syncthreads();
  stamp(a.stamps, 5);
  stamp(a.stamps, 12);
  if (b == G - 1) write_keep_bytes(flags, ffn, a.keep_d);
  stamp(a.stamps, 6);
  cta_time(a.cta_t, 2);

  // ---------------- E: stream kept down rows through the ring ----------------
  {
    const uint32_t row_bytes = (uint32_t)d * ESZ;
    if (producer) {
      const bool ok = produce(R, a.S_e, row_bytes, reinterpret_cast<const char*>(a.wt_down), ffn, a.uw_e, a.ctr + 2,
                              flags, vals, ps, pol, b == 0 ? a.trace + 128 : nullptr);
      if (!ok && (threadIdx.x & 31) == 0) s_abort = 1;
    } else {
      if (!consume_store<BF16>(R, a.S_e, row_bytes, d, full_par, a.acc_y, b == 0 ? a.trace + 128 : nullptr))
        s_abort = 1;
    }
  }
  __syncthreads();
  if (s_abort) {
    record_status(a.status, WINA_ERR_TIMEOUT);
    if (producer) drain(R, ps);
    return;
  }
  stamp(a.stamps, 7);
  cta_time(a.cta_t, 3);

  // ---------------- F: the last CTA to finish writes y and clears the sums ----------------
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.done, 1u);
    s_last = old == (unsigned)(G - 1);
    __threadfence();
  }
  __syncthreads();
  if (s_last) {
    for (int q = threadIdx.x; q < d / 4; q += kFT) {
      float4* p = reinterpret_cast<float4*>(a.acc_y) + q;
      reinterpret_cast<float4*>(a.y)[q] = __ldcg(p);
      __stcg(p, make_float4(0.f, 0.f, 0.f, 0.f));
    }
    if (threadIdx.x == 0) {
      a.ctr[2] = 0u;
      *a.done = 0u;
      *a.epoch = *a.epoch + 1u;  // the next call uses the other g/u buffers
    }
  }
  stamp(a.stamps, 8);
  stamp(a.stamps, 9);
}

// Byte flags of kept channels from index lists (the multi-token path's diagnostic view).
__global__ void k_keep_bytes(const int32_t* __restrict__ idx, int ld, int k, const int32_t* __restrict__ count, int n,
                             uint8_t* __restrict__ keep) {
  const int b = blockIdx.x;
  uint8_t* row = keep + (int64_t)b * n;
  for (int j = threadIdx.x; j < n; j += blockDim.x) row[j] = 0;
  __syncthreads();
  const int kb = k >= 0 ? k : min(count[b], ld);
  for (int r = threadIdx.x; r < kb; r += blockDim.x) {
    const int j = idx[(int64_t)b * ld + r];
    if (j >= 0 && j < n) row[j] = 1;
  }
}

static wina_status_t launch_keep_bytes(const int32_t* idx, int ld, int k, const int32_t* count, int n, int B,
                                       uint8_t* keep, cudaStream_t s) {
  k_keep_bytes<<<B, 256, 0, s>>>(idx, ld, k, count, n, keep);
  return cuda_status(cudaGetLastError());
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
  uint8_t* keep_g = reinterpret_cast<uint8_t*>(w + L.keep_g);
  uint8_t* keep_u = reinterpret_cast<uint8_t*>(w + L.keep_u);
  uint8_t* keep_d = reinterpret_cast<uint8_t*>(w + L.keep_d);

  if (batch == 1) {
    const bool bf16 = f->wdt == WINA_BF16;
    const uint32_t esz = bf16 ? 2u : 4u;
    const SmemLayout SLay = ffn_smem_layout((int)d, (int)ffn);
    size_t ring = SLay.ring < kMaxSmem ? (kMaxSmem - SLay.ring) / 128 * 128 : 0;
    if (ring < kMinRing) ring = 0;
    const uint32_t rb_b = (uint32_t)ffn * esz, rb_e = (uint32_t)d * esz;
    const int S_b = (int)std::min<size_t>(kMaxStages, ring / rb_b);
    const int S_e = (int)std::min<size_t>(kMaxStages, ring / rb_e);
    const size_t smem = kMaxSmem;
    const int G = bf16 ? max_coresident_grid(k_ffn_fused<true>, kFT, smem)
                       : max_coresident_grid(k_ffn_fused<false>, kFT, smem);
    if (G >= 2 && S_b >= 2 && S_e >= 2) {
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
      // gate/up CTA split in proportion to the kept rows (half each when unknown)
      int Gg = G / 2;
      if (mode == WINA_GATE_TOPK && k_gate + k_up > 0)
        Gg = (int)((G * k_gate + (k_gate + k_up) / 2) / (k_gate + k_up));
      Gg = std::max(1, std::min(G - 1, Gg));
      p.Gg = Gg;
      // channels per work unit: enough to hold ~64 KB of kept rows (at least 4 rows),
      // so that a unit's copies are issued by several lanes at once
      auto unit_width = [](int64_t n, int64_t kept, uint32_t row_bytes) {
        const double keep = kept > 0 ? (double)kept / (double)n : 1.0;
        const double rows = std::max(4.0, 65536.0 / row_bytes);
        const int w = (int)std::ceil(rows / keep);
        int p2 = 1;
        while (p2 < w && p2 < 32) p2 *= 2;
        return p2;
      };
      const int64_t kept_b = mode == WINA_GATE_TOPK ? std::max(k_gate, k_up) : (mode == WINA_GATE_DENSE ? d : (int64_t)(s * d));
      const int64_t kept_e = mode == WINA_GATE_TOPK ? k_down : (mode == WINA_GATE_DENSE ? ffn : (int64_t)(s * ffn));
      p.uw_b = unit_width(d, kept_b, rb_b);
      p.uw_e = unit_width(ffn, kept_e, rb_e);
      p.S_b = S_b;
      p.S_e = S_e;
      p.bar = reinterpret_cast<GridBarrier*>(w + L.bar);
      p.ctr = reinterpret_cast<unsigned*>(w + L.ctr);
      p.h = reinterpret_cast<float*>(w + L.h);
      p.keep_g = keep_g;
      p.keep_u = keep_u;
      p.keep_d = keep_d;
      p.stamps = reinterpret_cast<long long*>(w + L.stamps);
      p.cta_t = reinterpret_cast<unsigned long long*>(w + L.cta_t);
      p.trace = reinterpret_cast<unsigned long long*>(w + L.stamps) + 16;
      p.acc_g = reinterpret_cast<float*>(w + L.acc_g);
      p.acc_u = reinterpret_cast<float*>(w + L.acc_u);
      p.acc_y = reinterpret_cast<float*>(w + L.acc_y);
      p.done = reinterpret_cast<unsigned*>(w + L.ctr) + 3;
      p.epoch = reinterpret_cast<unsigned*>(w + L.ctr) + 4;
      p.status = status_dev;
      cudaError_t e = bf16 ? launch_kernel(k_ffn_fused<true>, dim3(G), dim3(kFT), smem, st, true, p)
                           : launch_kernel(k_ffn_fused<false>, dim3(G), dim3(kFT), smem, st, true, p);
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
    if ((r = launch_keep_bytes(ig, (int)d, -1, cnt, (int)d, B, keep_g, st))) return r;
    if ((r = launch_keep_bytes(iu, (int)d, -1, cnt + B, (int)d, B, keep_u, st))) return r;
    if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, -1, cnt, (int)d, B, g, sw, status_dev, st)))
      return r;
    if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, iu, xu, -1, cnt + B, (int)d, B, u, sw, status_dev, st)))
      return r;
    if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
    if ((r = launch_stat_threshold(h, WINA_F32, (int)ffn, z, B, idn, xd, cnt + 2 * B, nullptr, (int)ffn, status_dev,
                                   st)))
      return r;
    if ((r = launch_keep_bytes(idn, (int)ffn, -1, cnt + 2 * B, (int)ffn, B, keep_d, st))) return r;
    return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, -1, cnt + 2 * B, (int)ffn, B, y, sw, status_dev,
                                st);
  }
  const float* cg = mode == WINA_GATE_TOPK ? f->c_gate : nullptr;
  const float* cu = mode == WINA_GATE_TOPK ? f->c_up : nullptr;
  const float* cd = mode == WINA_GATE_TOPK ? f->c_down : nullptr;
  if ((r = launch_select_topk(x, xdt, cg, (int)d, (int)k_gate, B, ig, xg, (int)d, nullptr, st))) return r;
  if ((r = launch_select_topk(x, xdt, cu, (int)d, (int)k_up, B, iu, xu, (int)d, nullptr, st))) return r;
  if ((r = launch_keep_bytes(ig, (int)d, (int)k_gate, nullptr, (int)d, B, keep_g, st))) return r;
  if ((r = launch_keep_bytes(iu, (int)d, (int)k_up, nullptr, (int)d, B, keep_u, st))) return r;
  if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, (int)k_gate, nullptr, (int)d, B, g, sw,
                                status_dev, st)))
    return r;
  if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, iu, xu, (int)k_up, nullptr, (int)d, B, u, sw, status_dev,
                                st)))
    return r;
  if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
  if ((r = launch_select_topk(h, WINA_F32, cd, (int)ffn, (int)k_down, B, idn, xd, (int)ffn, nullptr, st))) return r;
  if ((r = launch_keep_bytes(idn, (int)ffn, (int)k_down, nullptr, (int)ffn, B, keep_d, st))) return r;
  return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, (int)k_down, nullptr, (int)ffn, B, y, sw,
                              status_dev, st);
}
