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
//   B  The producer warp streams the kept input-major weight rows HBM -> SMEM with bulk
//      copies into a ring of stages (full/empty mbarriers): first the CTA's own block of
//      channels, then units of a few channels from a global counter (dynamic load
//      balance across the CTAs of the projection). Consumer warps accumulate x_j * row_j
//      in float32 registers; at the end each CTA adds its row sums into g or u (vector
//      float atomics at L2).
//   -- grid barrier --
//   C  Every CTA reads the complete g and u, computes h = silu(g) * u and the down
//      gate's scores |h_j * c_down_j| for all ffn channels, and finds the down
//      selection's boundary score bin.
//   D/E The producer warp starts streaming the down rows whose scores lie above that bin
//      (kept whatever the rest of the selection decides) while the consumer warps finish
//      the selection; then the CTA's share of the kept boundary-bin rows follows. Down
//      rows are short, so a stage holds up to four of them in contiguous pieces. Row
//      sums are added straight into y (cleared by the CTAs before the grid barrier).
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
constexpr int kMaxVpt = 4;               // 16-byte row vectors per consumer thread at most
constexpr int kMaxPieces = 4;            // copy pieces (and rows) per ring stage at most
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
  int cs_g, cs_u, cs_e;  // channels in each CTA's own block: gate, up (phase B), down (E)
  int wmin_b, wmin_e;    // shortest dynamic unit (channels) in phases B and E
  int rows_e;            // phase E: rows per ring stage (ring over keys and past them)
  int rows_o;            // the same when phase E overlaps the down selection (smaller ring)
  int smem;              // dynamic SMEM bytes of the launch
  int S_b;               // ring stages in phase B
  int rows_b;            // phase B: rows per ring stage
  GridBarrier* bar;
  unsigned* ctr;  // [3] channel counters of the dynamic units: gate, up, down
  float* h;
  uint8_t* keep_g;
  uint8_t* keep_u;
  uint8_t* keep_d;
  long long* stamps;
  unsigned long long* cta_t;
  unsigned long long* trace;  // CTA 0, phase B: [0..63] stage issued, [64..127] stage taken (ns)
  float* acc_g;     // [2][ffn] float32 sums of the gate rows, one buffer per call parity
  float* acc_u;     // [2][ffn] float32 sums of the up rows, one buffer per call parity
  unsigned* epoch;  // calls completed on this workspace (picks the parity)
  int32_t* status;
};

struct SmemLayout {
  uint32_t vals, flags, meta_np, meta_row, meta_cnt, bars, keys, ring, hist, cand, stage;
};

// vals | flags | stage metadata | mbarriers | keys | ring. The selection's histogram and
// candidate lists, and the input staging buffer, overlay the start of the ring, which is
// idle while a selection runs. Phase E's ring starts past that scratch while it overlaps
// the down selection, or at keys when it runs after a complete selection.
__host__ __device__ inline SmemLayout ffn_smem_layout(int d, int ffn) {
  SmemLayout L;
  // room for max(d, ffn) channels, rounded up to 128 (the selection reads whole
  // 128-channel blocks)
  const uint32_t nb = ((uint32_t)(d > ffn ? d : ffn) + 127u) / 128u * 128u;
  uint32_t o = 0;
  auto take = [&](uint32_t bytes, uint32_t align) {
    o = (o + align - 1) / align * align;
    const uint32_t at = o;
    o += bytes;
    return at;
  };
  L.vals = take(nb * 4, 16);
  L.flags = take((nb + 31) / 32 * 4, 16);
  L.meta_np = take(kMaxStages * 4, 16);
  L.meta_row = take(kMaxStages * kMaxPieces * 4, 16);
  L.meta_cnt = take(kMaxStages * kMaxPieces * 4, 16);
  L.bars = take((2 * kMaxStages + 2) * 8, 16);
  L.keys = take(nb * 4, 128);
  L.ring = take(0, 128);
  L.hist = L.ring;
  L.cand = L.ring + kSelBins * 4;
  L.stage = L.cand + 2 * kSelCand * 4;  // 16-byte aligned input staging
  return L;
}

// Smallest ring the layout needs: the selection scratch and an input staging buffer of
// max(d, ffn) float32 live in it while a selection runs.
__host__ __device__ inline uint32_t ffn_min_ring(int d, int ffn) {
  return (uint32_t)((kSelBins + 2 * kSelCand) * 4) + (uint32_t)(d > ffn ? d : ffn) * 4;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// One L2 prefetch per 2 MB of [p, p + bytes), spread over the CTA's threads.
__device__ __forceinline__ void touch_pages(const void* p, size_t bytes) {
  const char* c = reinterpret_cast<const char*>(p);
  for (size_t o = (size_t)threadIdx.x << 21; o < bytes; o += (size_t)kFT << 21)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(c + o));
}

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
__device__ void write_keep_bytes(const uint32_t* flags, int n, uint8_t* out, int nthreads) {
  for (int j = threadIdx.x; j < n; j += nthreads) out[j] = (uint8_t)((flags[j >> 5] >> (j & 31)) & 1u);
}

// Barrier among the consumer warps only (the producer warp keeps streaming).
struct ConsumerSync {
  __device__ void operator()() const { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }
};

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
// Kept channels that follow one another have adjacent rows in the input-major layout;
// a piece is a run of up to `rmax` such rows, fetched by one bulk copy (bulk copies of
// short rows at scattered addresses stream well below HBM bandwidth, contiguous copies
// of 16 KB and more reach it). A stage holds up to `rmax` rows in one or more pieces:
// its consumers' fixed cost per stage (the barrier hand-offs) is paid once for them all.

struct Ring {
  char* base;       // SMEM
  uint64_t* full;   // [kMaxStages]
  uint64_t* empty;  // [kMaxStages]
  int* meta_np;     // pieces in each stage, -1 = end of phase
  int* meta_row;    // [kMaxStages][kMaxPieces] first row of each piece
  int* meta_cnt;    // [kMaxStages][kMaxPieces] rows in each piece
};

// Producer state kept across phases (per-stage mbarrier parities).
struct ProdState {
  uint32_t used;       // stage has been filled before
  uint32_t empty_par;  // parity of the next completion to wait for on empty[s]
  uint32_t full_par;   // parity of the next phase on full[s] (last issued = bit ^ 1)
};

// Work of one phase for the producer warp: kept rows of channels [0, n), the CTA's own
// block [s0, s1) first, then units over [base, n) taken from the global channel counter
// `ctr` (dynamic load balance). Unit widths are guided: the part of [base, n) not yet
// handed out divided by 2 * `parts` (the CTAs sharing the counter), clamped to
// [wmin, 32], so that units are long while much is left and short at the end.
struct PhaseWork {
  int n, s0, s1, base, parts, wmin;
  unsigned* ctr;
};

// The producer's tail: after its own block and units, the rows listed in list[0..*n)
// (one row each), once `ready` (an mbarrier) has completed its first phase.
struct Tail {
  uint64_t* ready;
  const int* list;
  const int* n;
};

// Streams the phase's kept rows (kept(j) true) into the ring in pieces (see above), then
// an end-of-phase marker. Runs on the producer warp. The pieces of a 32-channel window
// are issued by several lanes at once (a single thread issuing bulk copies one after
// another is far too slow to fill HBM): with one row per stage, each lane issues its
// row as soon as its own stage frees, in rounds of at most half the ring; with several
// rows per stage, the window's pieces are packed into stages, each stage's copies
// issued together once it frees. The first unit is requested halfway through the CTA's
// own block and each next one when a unit starts, so the counter's round trip overlaps
// the copies and no unit is held long. Returns false on a timeout.

template <typename Kept>
__device__ bool produce(const Ring& R, int S, uint32_t row_bytes, uint32_t stage_bytes, int rmax,
                        const char* __restrict__ Wt, const PhaseWork& wk, Kept kept, ProdState& ps, uint64_t pol,
                        unsigned long long* trace = nullptr, Tail tail = Tail{nullptr, nullptr, nullptr}) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u, le = lt | (1u << lane);
  int stage = 0;
  // this lane heads a piece of `len` rows starting at row j (if head): pack the pieces,
  // in lane order, into stages of at most rmax rows and issue them stage by stage
  auto issue_pieces = [&](bool head, int j, int len) {
    const uint32_t heads = __ballot_sync(0xffffffffu, head);
    if (rmax == 1) {
      // one row per stage: rounds of at most half the ring, each lane issuing its row as
      // soon as its own stage is free (the oldest first); the other half of the ring
      // stays in flight while a round waits
      const int np = __popc(heads), pos = __popc(heads & lt);
      const int RS = max(1, S / 2);
      bool ok = true;
      for (int r0 = 0; r0 < np; r0 += RS) {
        const int nr = min(RS, np - r0);
        bool mine = head && pos >= r0 && pos < r0 + nr;
        const int s = (stage + pos - r0) % S;
        const bool was_used = (ps.used >> s) & 1u;
        const uint32_t par = (ps.empty_par >> s) & 1u;
        unsigned long long t0 = 0;
        while (__any_sync(0xffffffffu, mine)) {
          if (!mine) continue;
          if (!was_used || mbar_test_wait(&R.empty[s], par)) {
            R.meta_row[s * kMaxPieces] = j;
            R.meta_cnt[s * kMaxPieces] = 1;
            R.meta_np[s] = 1;
            mbar_arrive_expect_tx(&R.full[s], row_bytes);
            bulk_copy_g2s(R.base + (size_t)s * stage_bytes, Wt + (size_t)j * row_bytes, row_bytes, &R.full[s], pol);
            if (trace && stage + pos - r0 < 64) trace[stage + pos - r0] = globaltimer_ns();
            mine = false;
          } else {
            const unsigned long long now = globaltimer_ns();
            if (t0 == 0) {
              t0 = now;
            } else if (now - t0 > kPipeTimeoutNs) {
              ok = false;
              mine = false;
            }
          }
        }
        for (int i = 0; i < nr; ++i) {  // the same state update in every lane
          const int s2 = (stage + i) % S;
          if ((ps.used >> s2) & 1u) ps.empty_par ^= 1u << s2;
          ps.used |= 1u << s2;
          ps.full_par ^= 1u << s2;
        }
        stage += nr;
        if (__any_sync(0xffffffffu, !ok)) return false;
      }
      return true;
    }
    int my_k = -1, my_off = 0, nst = 0, fill = rmax;
    for (uint32_t hb = heads; hb; hb &= hb - 1u) {
      const int l = __ffs(hb) - 1;
      const int L = __shfl_sync(0xffffffffu, len, l);
      if (fill + L > rmax) {
        ++nst;
        fill = 0;
      }
      if (lane == l) {
        my_k = nst - 1;
        my_off = fill;
      }
      fill += L;
    }
    for (int k = 0; k < nst; ++k) {
      const int s = (stage + k) % S;
      const bool mine = my_k == k;
      const uint32_t pm = __ballot_sync(0xffffffffu, mine);
      const uint32_t rows = __reduce_add_sync(0xffffffffu, mine ? (uint32_t)len : 0u);
      bool ok = true;
      if (lane == 0 && ((ps.used >> s) & 1u)) ok = mbar_wait_poll(&R.empty[s], (ps.empty_par >> s) & 1u);
      if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
      if (mine) {
        const int idx = __popc(pm & lt);
        R.meta_row[s * kMaxPieces + idx] = j;
        R.meta_cnt[s * kMaxPieces + idx] = len;
      }
      if (lane == 0) R.meta_np[s] = __popc(pm);
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&R.full[s], rows * row_bytes);
      __syncwarp();
      if (mine) {
        bulk_copy_g2s(R.base + (size_t)s * stage_bytes + (size_t)my_off * row_bytes, Wt + (size_t)j * row_bytes,
                      (uint32_t)len * row_bytes, &R.full[s], pol);
        if (trace && stage + k < 64) trace[stage + k] = globaltimer_ns();
      }
      if ((ps.used >> s) & 1u) ps.empty_par ^= 1u << s;
      ps.used |= 1u << s;
      ps.full_par ^= 1u << s;
    }
    stage += nst;
    return true;
  };
  // kept rows of channels [j0, j1), j1 - j0 <= 32, in pieces of up to rmax adjacent rows
  auto issue = [&](int j0, int j1) {
    const int j = j0 + lane;
    const bool k = j < j1 && kept(j);
    const uint32_t km = __ballot_sync(0xffffffffu, k);
    const uint32_t runs = km & ~(km << 1);                 // first lanes of runs of kept channels
    const int rs = 31 - __clz(runs & le);                  // start of this lane's run (if kept)
    const bool head = k && ((lane - rs) % rmax == 0);      // first lane of a piece
    const uint32_t heads = __ballot_sync(0xffffffffu, head);
    const uint32_t after = (heads | ~km) & ~le;
    const int len = (after ? __ffs(after) - 1 : 32) - lane;  // rows in the piece headed here
    return issue_pieces(head, j, len);
  };
  bool ok = true;
  const unsigned ndyn = wk.base < wk.n ? (unsigned)(wk.n - wk.base) : 0u;
  auto width = [&](unsigned taken) {
    const unsigned left = taken < ndyn ? ndyn - taken : 0u;
    return (unsigned)min(32, max(wk.wmin, (int)(left / (2u * (unsigned)wk.parts))));
  };
  // the first unit is requested halfway through the CTA's own block, so that its round
  // trip is hidden and it is not held long
  unsigned pw = 0u, pstart = 0u;
  const int half = wk.s0 + (wk.s1 - wk.s0) / 2;
  bool asked = false;
  for (int c = wk.s0; c < wk.s1 && ok; c += 32) {
    if (!asked && c + 32 > half) {
      if (lane == 0 && ndyn) {
        pw = width(0u);
        pstart = atomicAdd(wk.ctr, pw);
      }
      asked = true;
    }
    ok = issue(c, min(wk.s1, c + 32));
  }
  if (ok && ndyn) {
    if (!asked && lane == 0) {
      pw = width(0u);
      pstart = atomicAdd(wk.ctr, pw);
    }
    while (true) {
      const unsigned start = __shfl_sync(0xffffffffu, pstart, 0), w = __shfl_sync(0xffffffffu, pw, 0);
      if (start >= ndyn) break;
      if (lane == 0) {  // the next unit, while this one streams
        pw = width(start + w);
        pstart = atomicAdd(wk.ctr, pw);
      }
      const int j0 = wk.base + (int)start;
      if (!issue(j0, min(wk.n, j0 + (int)w))) {
        ok = false;
        break;
      }
    }
  }
  if (ok && tail.ready) {
    if (lane == 0) ok = mbar_wait(tail.ready, 0u);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    const int nt = ok ? *tail.n : 0;
    for (int c0 = 0; c0 < nt && ok; c0 += 32) {
      const bool v = c0 + lane < nt;
      ok = issue_pieces(v, v ? tail.list[c0 + lane] : 0, 1);
    }
  }
  if (!__all_sync(0xffffffffu, ok)) return false;
  // end-of-phase marker: completes a stage with no bytes
  if (lane == 0) {
    const int s = stage % S;
    if ((ps.used >> s) & 1u) ok = mbar_wait(&R.empty[s], (ps.empty_par >> s) & 1u);
    if (ok) {
      R.meta_np[s] = -1;
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

__device__ __forceinline__ void red_add_f4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Consumer warps: take stages in order until the end marker; for each row r of a stage,
// acc += vals[meta_row + r] * row (thread t owns 16-byte vectors t, t + kCT, ...); then
// add the row sums into out[0..m) (vector float atomics at L2; the order of the CTAs'
// additions is not fixed). Returns false on a timeout.
template <bool BF16, int VPT>
__device__ bool consume_t(const Ring& R, int S, uint32_t row_bytes, uint32_t stage_bytes, int V, uint32_t& full_par,
                          const float* vals, float* __restrict__ out, unsigned long long* trace) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int t = threadIdx.x, lane = t & 31;
  float acc[VPT][EPV];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[j][e] = 0.f;
  const uint32_t ring = smem_addr(R.base);
  int stage = 0, rows = 0;
  bool ok = true;
  while (true) {
    const int s = stage % S;
    if (!mbar_wait(&R.full[s], (full_par >> s) & 1u)) {
      ok = false;
      break;
    }
    if (trace && t == 0 && stage < 64) trace[64 + stage] = globaltimer_ns();
    full_par ^= 1u << s;
    const int np = R.meta_np[s];
    uint32_t src = ring + (uint32_t)s * stage_bytes;
    for (int p = 0; p < np; ++p) {
      const int row = R.meta_row[s * kMaxPieces + p], nr = R.meta_cnt[s * kMaxPieces + p];
      rows += nr;
      // up to RU rows of the piece at a time: all their loads first, then the arithmetic
      constexpr int RU = VPT <= 2 ? 4 : 1;
      for (int r0 = 0; r0 < nr; r0 += RU) {
        float xv[RU];
        uint4 w[RU][VPT];
#pragma unroll
        for (int u = 0; u < RU; ++u) {
          const int r = r0 + u;
          xv[u] = r < nr ? vals[row + r] : 0.f;
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const int v = t + j * kCT;
            if (r < nr && v < V) w[u][j] = ld_shared_u4(src + (uint32_t)r * row_bytes + (uint32_t)v * 16u);
          }
        }
#pragma unroll
        for (int u = 0; u < RU; ++u)
#pragma unroll
          for (int j = 0; j < VPT; ++j)
            if (r0 + u < nr && t + j * kCT < V) VecOps<BF16>::fma(acc[j], w[u][j], xv[u]);
      }
      src += (uint32_t)nr * row_bytes;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&R.empty[s]);
    if (np < 0) break;
    ++stage;
  }
  if (rows == 0) return ok;  // nothing to add
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = t + j * kCT;
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

template <bool BF16, int VF>
__device__ bool consume(const Ring& R, int S, uint32_t row_bytes, uint32_t stage_bytes, int m, uint32_t& full_par,
                        const float* vals, float* out, unsigned long long* trace = nullptr) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int V = m / EPV;
  if constexpr (VF > 0) return consume_t<BF16, VF>(R, S, row_bytes, stage_bytes, V, full_par, vals, out, trace);
  // rows of at most kMaxVpt vectors per consumer thread (the host sends wider shapes to
  // the batched path): the widest case sets the kernel's register budget
  switch ((V + kCT - 1) / kCT) {
    case 1: return consume_t<BF16, 1>(R, S, row_bytes, stage_bytes, V, full_par, vals, out, trace);
    case 2: return consume_t<BF16, 2>(R, S, row_bytes, stage_bytes, V, full_par, vals, out, trace);
    case 3: return consume_t<BF16, 3>(R, S, row_bytes, stage_bytes, V, full_par, vals, out, trace);
    default: return consume_t<BF16, kMaxVpt>(R, S, row_bytes, stage_bytes, V, full_par, vals, out, trace);
  }
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------

// MODE: the gate mode when fixed at compile time, or -1 (read from the parameters).
// VB / VE: 16-byte vectors per consumer thread of a gate/up row and of a down row when
// fixed, or 0 (dispatched at run time). The hot case (bf16, top-K, d <= 4096) gets its
// own instantiations: only the code it runs, so fewer registers and a smaller
// instruction footprint for the streaming loops.
template <bool BF16, int MODE, int VB, int VE>
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
  R.meta_np = reinterpret_cast<int*>(smraw + SL.meta_np);
  R.meta_row = reinterpret_cast<int*>(smraw + SL.meta_row);
  R.meta_cnt = reinterpret_cast<int*>(smraw + SL.meta_cnt);
  R.full = reinterpret_cast<uint64_t*>(smraw + SL.bars);
  R.empty = R.full + kMaxStages;
  R.base = reinterpret_cast<char*>(smraw + SL.ring);
  uint64_t* aux = R.full + 2 * kMaxStages;  // input staging copies; aux + 1: down selection done
  unsigned char* stage_in = smraw + SL.stage;
  __shared__ uint32_t red[2 * kFT / 32 + 8];
  __shared__ double dred[3 * kFT / 32];
  __shared__ int s_abort, s_ntail;

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
    mbar_init(aux, 1u);
    mbar_init(aux + 1, 1u);  // the down selection is finished (overlapped phase E)
    mbar_init_fence();
    s_abort = 0;
  }
  __syncthreads();
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
    // y receives the down rows' sums by atomics after the grid barrier: clear it now
    for (int q = d * b / G + threadIdx.x; q < d * (b + 1) / G; q += kFT) __stcg(a.y + q, 0.f);
    // the previous call has completed: its down-unit counter can start again
    if (b == 0 && threadIdx.x == 0) a.ctr[2] = 0u;
  }

  // ---------------- A: this CTA's projection, its kept-channel bitmask ----------------
  const bool gate = b < a.Gg;
  const int rank = gate ? b : b - a.Gg;
  const float* cproj = gate ? a.c_gate : a.c_up;
  {
    // x and this projection's c arrive by bulk copies (x into the staging buffer, c into
    // the keys buffer, where each score then replaces its c in place); meanwhile the
    // histogram is cleared. An x that is not 16-byte aligned is loaded by the threads.
    const bool topk = MODE >= 0 ? MODE == WINA_GATE_TOPK : a.mode == WINA_GATE_TOPK;
    const uint32_t xbytes = (uint32_t)d * (a.xdt == WINA_BF16 ? 2u : 4u);
    const bool xbulk = ((uintptr_t)a.x & 15u) == 0;
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(aux, (xbulk ? xbytes : 0u) + (topk ? (uint32_t)d * 4u : 0u));
      if (xbulk) bulk_copy_g2s(stage_in, a.x, xbytes, aux, pol);
      if (topk) bulk_copy_g2s(keys, cproj, (uint32_t)d * 4u, aux, pol);
    }
    // touch every 2 MB page of this projection's weights now, so that the address
    // translations are warm when the rows stream (the first rows land later otherwise)
    touch_pages(gate ? a.wt_gate : a.wt_up, (size_t)d * ffn * ESZ);
    for (int i = threadIdx.x; i < kSelBins + 256; i += kFT) hist[i] = 0u;  // and the sub-bin counts
    if (!xbulk)
      for (int i = threadIdx.x; i < d; i += kFT) reinterpret_cast<float*>(stage_in)[i] = load_elem(a.x, a.xdt, i);
    if (!mbar_wait(aux, 0u)) s_abort = 1;
    __syncthreads();
    if (s_abort) {
      record_status(a.status, WINA_ERR_TIMEOUT);
      return;
    }
    stamp(a.stamps, 10);
    const bool xf32 = !xbulk || a.xdt == WINA_F32;
    for (int i = threadIdx.x; i < d; i += kFT) {
      const float xv = xf32 ? reinterpret_cast<const float*>(stage_in)[i]
                            : bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(stage_in)[i]);
      vals[i] = xv;
      if (topk) {
        const uint32_t k = __float_as_uint(fabsf(xv * __uint_as_float(keys[i])));
        keys[i] = k;
        atomicAdd(&hist[k >> 19], 1u);
      }
    }
    stamp(a.stamps, 11);
    if (topk) {
      select_topk_flags_radix<kFT>(keys, d, gate ? a.k_gate : a.k_up, hist, cand, red, flags,
                                   b == 0 ? a.stamps + 12 : nullptr);
    } else if constexpr (MODE != WINA_GATE_TOPK) {
      __syncthreads();
      if (a.mode == WINA_GATE_STAT)
        flags_from_threshold(vals, d, spark_threshold(vals, d, a.z, dred), flags);
      else
        flags_all(d, flags);
    }
  }
  __syncthreads();
  if (rank == (gate ? a.Gg : G - a.Gg) - 1) write_keep_bytes(flags, d, gate ? a.keep_g : a.keep_u, kFT);
  stamp(a.stamps, 1);
  cta_time(a.cta_t, 0);

  // ---------------- B: stream kept gate / up rows through the ring ----------------
  {
    const uint32_t row_bytes = (uint32_t)ffn * ESZ;
    if (producer) {
      // the ring overlays SMEM last written by ordinary stores: order those before the
      // bulk copies
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int cs = gate ? a.cs_g : a.cs_u, np = gate ? a.Gg : G - a.Gg;
      const PhaseWork wk{d, min(d, rank * cs), min(d, (rank + 1) * cs), min(d, np * cs), np, a.wmin_b,
                         a.ctr + (gate ? 0 : 1)};
      auto kept = [&](int j) { return ((flags[j >> 5] >> (j & 31)) & 1u) != 0u; };
      const bool ok = produce(R, a.S_b, row_bytes, (uint32_t)a.rows_b * row_bytes, a.rows_b,
                              reinterpret_cast<const char*>(gate ? a.wt_gate : a.wt_up),
                              wk, kept, ps, pol, b == 0 ? a.trace : nullptr);
      if (!ok && (threadIdx.x & 31) == 0) s_abort = 1;
    } else {
      if (!consume<BF16, VB>(R, a.S_b, row_bytes, (uint32_t)a.rows_b * row_bytes, ffn, full_par, vals, gate ? acc_g : acc_u,
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
  // the ring is drained: fetch c_down into the staging buffer while waiting for the grid
  if (threadIdx.x == 0 && (MODE >= 0 ? MODE == WINA_GATE_TOPK : a.mode == WINA_GATE_TOPK)) {
    mbar_expect_tx(aux, (uint32_t)ffn * 4u);
    bulk_copy_g2s(stage_in, a.c_down, (uint32_t)ffn * 4u, aux, pol);
  }
  if (!grid_sync_fixed(a.bar, G, a.status)) {
    if (threadIdx.x == 0 && (MODE >= 0 ? MODE == WINA_GATE_TOPK : a.mode == WINA_GATE_TOPK)) {  // let the issued copy land before exiting
      mbar_arrive(aux);
      mbar_wait(aux, 1u);
    }
    return;
  }
  stamp(a.stamps, 3);

  // ---------------- C/D: h for every channel, the down scores, the down bitmask ----------------
  touch_pages(a.wt_down, (size_t)d * ffn * ESZ);  // as in phase A, for the down rows
  if (b == 0 && threadIdx.x == 0) {
    a.ctr[0] = 0u;  // every CTA is past phase B: the gate/up unit counters can be reset
    a.ctr[1] = 0u;
    *a.epoch = *a.epoch + 1u;  // every CTA has read it: the next call uses the other g/u buffers
  }
  {
    // g into vals, u into keys (bulk copies); h replaces g and the score replaces u in
    // place; the score histogram is filled on the way
    const bool topk = MODE >= 0 ? MODE == WINA_GATE_TOPK : a.mode == WINA_GATE_TOPK;
    if (threadIdx.x == 0) {
      // the sums were made by other SMs' atomics (generic proxy); order them before the
      // bulk copies (async proxy) that read them
      asm volatile("fence.proxy.async.global;" ::: "memory");
      mbar_arrive_expect_tx(aux, 2u * (uint32_t)ffn * 4u);
      bulk_copy_g2s(vals, acc_g, (uint32_t)ffn * 4u, aux, pol);
      bulk_copy_g2s(keys, acc_u, (uint32_t)ffn * 4u, aux, pol);
    }
    for (int i = threadIdx.x; i < kSelBins + 256; i += kFT) hist[i] = 0u;  // and the sub-bin counts
    if (!mbar_wait(aux, 1u)) s_abort = 1;
    __syncthreads();
    if (s_abort) {
      record_status(a.status, WINA_ERR_TIMEOUT);
      return;
    }
    const float* cdn = reinterpret_cast<const float*>(stage_in);
    for (int q = threadIdx.x; q < ffn / 4; q += kFT) {
      const float4 g4 = reinterpret_cast<const float4*>(vals)[q];
      const float4 u4 = reinterpret_cast<const float4*>(keys)[q];
      float4 h4;
      h4.x = silu_f(g4.x) * u4.x;
      h4.y = silu_f(g4.y) * u4.y;
      h4.z = silu_f(g4.z) * u4.z;
      h4.w = silu_f(g4.w) * u4.w;
      reinterpret_cast<float4*>(vals)[q] = h4;
      if (b == G - 1) reinterpret_cast<float4*>(a.h)[q] = h4;
      if (topk) {
        const float4 c4 = reinterpret_cast<const float4*>(cdn)[q];
        uint4 k4;
        k4.x = __float_as_uint(fabsf(h4.x * c4.x));
        k4.y = __float_as_uint(fabsf(h4.y * c4.y));
        k4.z = __float_as_uint(fabsf(h4.z * c4.z));
        k4.w = __float_as_uint(fabsf(h4.w * c4.w));
        reinterpret_cast<uint4*>(keys)[q] = k4;
        atomicAdd(&hist[k4.x >> 19], 1u);
        atomicAdd(&hist[k4.y >> 19], 1u);
        atomicAdd(&hist[k4.z >> 19], 1u);
        atomicAdd(&hist[k4.w >> 19], 1u);
      }
    }
    stamp(a.stamps, 4);
  }
  // The down selection's boundary bin; with it known, rows surely kept (scores above
  // the bin) can stream while the consumer warps finish the selection.
  const bool topk = MODE >= 0 ? MODE == WINA_GATE_TOPK : a.mode == WINA_GATE_TOPK;
  const bool split = topk && a.k_down > 0 && a.k_down < ffn;
  Crossing cr{0, 0u, 0u};
  if (split) cr = radix_crossing<kFT>(hist, a.k_down, red);
  stamp(a.stamps, 14);
  const bool overlap = split && cr.cnt <= (uint32_t)kSelCand;
  const uint32_t rb_e = (uint32_t)d * ESZ;
  if (!overlap) {
    if (split) {
      select_general_flags<kFT>(keys, ffn, a.k_down, hist, cand, red, flags);
    } else if (topk) {
      select_topk_flags_radix<kFT>(keys, ffn, a.k_down, hist, cand, red, flags);
    } else if constexpr (MODE != WINA_GATE_TOPK) {
      __syncthreads();
      if (a.mode == WINA_GATE_STAT)
        flags_from_threshold(vals, ffn, spark_threshold(vals, ffn, a.z, dred), flags);
      else
        flags_all(ffn, flags);
    }
    __syncthreads();
    stamp(a.stamps, 5);
    if (b == G - 1) write_keep_bytes(flags, ffn, a.keep_d, kFT);
    stamp(a.stamps, 6);
    cta_time(a.cta_t, 2);
    // ---------------- E: stream kept down rows through the ring ----------------
    // the down scores are no longer needed: the ring now starts at keys
    const uint32_t stage_bytes = (uint32_t)a.rows_e * rb_e;
    const int S = min(kMaxStages, (int)(((uint32_t)a.smem - SL.keys) / stage_bytes));
    Ring RE = R;
    RE.base = reinterpret_cast<char*>(smraw + SL.keys);
    if (producer) {
      // the ring overlays SMEM last written by ordinary stores: order those before the
      // bulk copies
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const PhaseWork wk{ffn, min(ffn, b * a.cs_e), min(ffn, (b + 1) * a.cs_e), min(ffn, G * a.cs_e), G, a.wmin_e,
                         a.ctr + 2};
      auto kept = [&](int j) { return ((flags[j >> 5] >> (j & 31)) & 1u) != 0u; };
      if (!produce(RE, S, rb_e, stage_bytes, a.rows_e, reinterpret_cast<const char*>(a.wt_down), wk, kept, ps, pol) &&
          (threadIdx.x & 31) == 0)
        s_abort = 1;
    } else {
      if (!consume<BF16, VE>(RE, S, rb_e, stage_bytes, d, full_par, vals, a.y)) s_abort = 1;
    }
  } else {
    // ---------------- D/E overlapped ----------------
    // The ring lies past the selection's scratch (keys, hist and cand stay intact).
    // Producer: rows whose score bin is above the boundary bin (kept whatever the
    // selection's finish decides), as its own block and units; then, once the
    // consumers have finished the selection, its share (channel mod G == b) of the kept
    // boundary-bin rows. Consumers: finish the selection (named barrier over the 16
    // consumer warps), list that share, then consume the ring.
    const uint32_t stage_bytes = (uint32_t)a.rows_o * rb_e;
    const uint32_t at = SL.stage;
    const int S = min(kMaxStages, (int)(((uint32_t)a.smem - at) / stage_bytes));
    Ring RE = R;
    RE.base = reinterpret_cast<char*>(smraw + at);
    int* tail = reinterpret_cast<int*>(cand);  // written once the finish no longer needs cand
    uint64_t* sel_done = aux + 1;
    if (producer) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const PhaseWork wk{ffn, min(ffn, b * a.cs_e), min(ffn, (b + 1) * a.cs_e), min(ffn, G * a.cs_e), G, a.wmin_e,
                         a.ctr + 2};
      const uint32_t B = (uint32_t)cr.bin;
      auto sure = [&](int j) { return (keys[j] >> 19) > B; };
      if (!produce(RE, S, rb_e, stage_bytes, a.rows_o, reinterpret_cast<const char*>(a.wt_down), wk, sure, ps, pol,
                   nullptr, Tail{sel_done, tail, &s_ntail}) &&
          (threadIdx.x & 31) == 0)
        s_abort = 1;
    } else {
      radix_finish<kCT>(keys, ffn, a.k_down, cr, hist, cand, flags, ConsumerSync{},
                        b == 0 ? a.stamps + 14 : nullptr);
      // this CTA's share of the kept boundary-bin channels
      if (threadIdx.x == 0) s_ntail = 0;
      ConsumerSync{}();
      const uint32_t* lst = hist;  // the bin's (key, channel) pairs, left by the finish
      for (uint32_t e = threadIdx.x; e < cr.cnt; e += kCT) {
        const uint32_t ch = lst[2 * e + 1];
        if ((int)(ch % (uint32_t)G) == b && ((flags[ch >> 5] >> (ch & 31)) & 1u)) tail[atomicAdd(&s_ntail, 1)] = (int)ch;
      }
      ConsumerSync{}();
      if (threadIdx.x == 0) mbar_arrive(sel_done);  // release: the list and its length
      stamp(a.stamps, 5);
      if (b == G - 1) write_keep_bytes(flags, ffn, a.keep_d, kCT);
      stamp(a.stamps, 6);
      cta_time(a.cta_t, 2);
      if (!consume<BF16, VE>(RE, S, rb_e, stage_bytes, d, full_par, vals, a.y)) s_abort = 1;
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
    if (ring < ffn_min_ring((int)d, (int)ffn)) ring = 0;
    const uint32_t rb_b = (uint32_t)ffn * esz;
    // phase B: one row per stage (rows of ffn elements are long enough; more stages keep
    // more bytes in flight while the ring refills)
    const int rows_b = 1;
    const int S_b = (int)std::min<size_t>(kMaxStages, ring / ((size_t)rows_b * rb_b));
    const size_t smem = kMaxSmem;
    // the specialised instantiation for bf16 top-K with one vector per thread of a down
    // row, else the general one
    const int vb = (int)(((int64_t)ffn * esz / 16 + kCT - 1) / kCT), ve = (int)(((int64_t)d * esz / 16 + kCT - 1) / kCT);
    void (*kern)(FfnParams) = bf16 ? k_ffn_fused<true, -1, 0, 0> : k_ffn_fused<false, -1, 0, 0>;
    if (bf16 && mode == WINA_GATE_TOPK && ve == 1) {
      if (vb == 1) kern = k_ffn_fused<true, WINA_GATE_TOPK, 1, 1>;
      else if (vb == 2) kern = k_ffn_fused<true, WINA_GATE_TOPK, 2, 1>;
      else if (vb == 3) kern = k_ffn_fused<true, WINA_GATE_TOPK, 3, 1>;
      else if (vb == 4) kern = k_ffn_fused<true, WINA_GATE_TOPK, 4, 1>;
    }
    const int G = max_coresident_grid(kern, kFT, smem);
    // phase E: rows per stage (pieces of up to that many adjacent rows per bulk copy),
    // at least two stages in the ring, which then starts at keys
    const uint32_t rb_e = (uint32_t)d * esz;
    const int rows_e = SLay.keys < kMaxSmem ? (int)std::min<size_t>(4, (kMaxSmem - SLay.keys) / (2 * (size_t)rb_e)) : 0;
    // overlapped with the down selection, the ring starts past the selection's scratch
    const int rows_o = SLay.stage < kMaxSmem ? (int)std::min<size_t>(4, (kMaxSmem - SLay.stage) / (2 * (size_t)rb_e)) : 0;
    // consumer threads hold at most kMaxVpt 16-byte vectors of a row (ffn and d elements)
    const bool narrow = ((int64_t)ffn * esz / 16 + kCT - 1) / kCT <= kMaxVpt &&
                        ((int64_t)d * esz / 16 + kCT - 1) / kCT <= kMaxVpt;
    if (narrow && G >= 2 && S_b >= 2 && rows_e >= 1 && rows_o >= 1) {
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
      // each CTA first streams its own block of channels (no counter round trip at the
      // start); the counters hand out the rest in guided units, the shortest about one
      // row (gate/up) or two rows (down)
      constexpr double kOwnShare = 0.7;
      p.cs_g = (int)(kOwnShare * (double)d / (double)Gg);
      p.cs_u = (int)(kOwnShare * (double)d / (double)(G - Gg));
      p.cs_e = (int)(kOwnShare * (double)ffn / (double)G);
      const int64_t kept_b = mode == WINA_GATE_TOPK ? std::max(k_gate, k_up) : (mode == WINA_GATE_DENSE ? d : (int64_t)(s * d));
      const int64_t kept_e = mode == WINA_GATE_TOPK ? k_down : (mode == WINA_GATE_DENSE ? ffn : (int64_t)(s * ffn));
      auto min_width = [](int64_t n, int64_t kept, double rows) {
        const double keep = kept > 0 ? std::min(1.0, (double)kept / (double)n) : 1.0;
        return (int)std::max(1.0, std::min(32.0, std::ceil(rows / keep)));
      };
      p.wmin_b = min_width(d, kept_b, 1.0);
      p.wmin_e = min_width(ffn, kept_e, 2.0);
      p.S_b = S_b;
      p.rows_b = rows_b;
      p.rows_e = rows_e;
      p.rows_o = rows_o;
      p.smem = (int)smem;
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
      p.epoch = reinterpret_cast<unsigned*>(w + L.ctr) + 4;
      p.status = status_dev;
      return cuda_status(launch_kernel(kern, dim3(G), dim3(kFT), smem, st, true, p));
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
