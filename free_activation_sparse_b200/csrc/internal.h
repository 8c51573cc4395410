// Host-side helpers shared by the C-ABI entry points (argument checks, device facts,
// launches, workspace layouts). Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "wina.h"

namespace wina {

// Largest grid any kernel here launches; workspaces are sized for it so that their
// size does not depend on the device. (2 CTAs on each of a B200's 148 SMs.)
constexpr int kGridCap = 296;
constexpr int kNT = 512;          // threads per CTA of the selection / product kernels
constexpr int kRowChunk = 1024;   // kept rows staged in SMEM at a time by sparse_matvec
constexpr size_t kAlign = 256;    // alignment of every workspace sub-buffer
constexpr int kFfnStamps = 32;  // phase clock stamps the single-token FFN kernel leaves (16 used)
constexpr int kDecodeRows = 32;  // partial rows of the single-token FFN kernel (its row groups: at most 4 + 16)

inline bool valid_dtype(int dt) { return dt == WINA_F32 || dt == WINA_BF16; }
inline int64_t elem_size(int dt) { return dt == WINA_BF16 ? 2 : 4; }
inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Time limit of the grid-barrier waits of the single-token FFN kernel (wina_set_wait_limit_ns).
unsigned long long wait_limit_ns();

inline wina_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return WINA_OK;
  return WINA_ERR_CUDA;
}

// Streaming multiprocessors of the current device (0 if none). Cached per device.
int device_sm_count();

// Raise a kernel's dynamic SMEM limit to at least `smem` bytes on the current device
// (remembered per device and kernel, so repeated calls cost a table lookup).
cudaError_t ensure_smem_limit(const void* kern, size_t smem);

// Ask for the smallest shared-memory carveout (the rest of the SM's unified L1/SMEM stays
// L1) for `kern` on the current device (remembered per device and kernel).
cudaError_t ensure_prefer_l1(const void* kern);
// Shared-memory carveout preference of a kernel, in percent of the maximum (cached).
cudaError_t ensure_carveout(const void* kern, int pct);

// A second stream of the current device, with two events, for work that can run beside
// the caller's stream (created once per device, non-blocking). Returns false when none is
// available (then everything runs on the caller's stream). `fork` makes the side stream
// wait for the work enqueued so far on `main`; `join` makes `main` wait for the side
// stream's work. Host threads enqueueing fork...join pairs are serialised by `lock`.
struct SideStream {
  cudaStream_t s;
  cudaEvent_t fork_ev, join_ev;
};
bool side_stream(cudaStream_t main, SideStream* out);
std::unique_lock<std::mutex> side_stream_lock();

// Co-resident CTAs per SM of `kern` at this block size and SMEM on the current device
// (cached per device, kernel, block size and SMEM). 0 on error.
int blocks_per_sm(const void* kern, int threads, size_t smem);

// Launch with cudaLaunchKernelEx, optionally as a cooperative launch (all CTAs
// co-resident, required by kernels that use grid_sync).
template <typename... Exp, typename... Act>
cudaError_t launch_kernel(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool coop,
                          Act&&... args) {
  if (smem > 0) {  // any dynamic part: static shared memory comes on top of it
    cudaError_t e = ensure_smem_limit((const void*)kern, smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (coop) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Act&&>(args)...);
}

// Largest co-resident grid for `kern` at this block size and SMEM, capped at kGridCap.
template <typename K>
int max_coresident_grid(K kern, int threads, size_t smem) {
  const int g = blocks_per_sm((const void*)kern, threads, smem) * device_sm_count();
  return g < kGridCap ? g : kGridCap;
}

// ----------------------------------------------------------------------------------
// workspace layouts
// ----------------------------------------------------------------------------------

// sparse_matvec: [GridBarrier][group counters: kGridCap u32][partials: kGridCap x (m + 4)
// float32]. The partial rows are only needed when a token is split over several CTAs
// (batch < kGridCap); the counters serve the single-token column-slice path.
struct SpmvWs {
  size_t bar, counters, partials, total;
};
inline SpmvWs spmv_ws_layout(int64_t m, int64_t batch) {
  SpmvWs w;
  w.bar = 0;
  w.counters = kAlign;
  w.partials = round_up(w.counters + (size_t)kGridCap * 4, kAlign);
  const size_t part = batch < kGridCap ? (size_t)kGridCap * (size_t)(m + 4) * 4 : 0;
  w.total = round_up(w.partials + part, kAlign);
  return w;
}

// The union path of the sparse product (several tokens, bf16 weights): a byte flag per
// channel [n], the chunk list [nblk + 1], the channel of each gather slot [kmax], each
// member's X~ column [n], chunk counts and the number of bf16 parts [4], and X~
// [3 * np][kmax] bf16 (np = tokens per block rounded up to 16, kmax = 64 * (nblk + 1)).
// The flags and X~ are zero between calls (each call clears what it set).
struct UnionWs {
  size_t flag, chunk_row, slot, pos, info, xt, total;
  int64_t kmax, np;
};
UnionWs union_ws_layout(int64_t n, int64_t batch);
// Whether the union path serves this call (bf16 weights, several tokens).
bool union_path_takes(int wdt, int64_t n, int64_t m, int64_t batch);
constexpr int kUnionMinBatch = 4;  // fewer tokens take the per-token product
constexpr int kUnionBlock = 256;   // tokens per union block

// sparse_matvec's workspace: the per-token layout, then the union path's (several tokens)
inline size_t spmv_total_ws(int64_t n, int64_t m, int64_t batch) {
  size_t t = spmv_ws_layout(m, batch).total;
  if (batch >= kUnionMinBatch) t += union_ws_layout(n, batch).total;
  return t;
}

// sparse_ffn_swiglu (d, ffn, batch):
//   bar | groups [2 * kGridCap] | h [B][ffn] | keep_g [B][d] | keep_u [B][d] | keep_d [B][ffn] (bytes)
//   | stamps [kFfnStamps] | cta_t [kGridCap][4]
//   | part [kDecodeRows][pstride] | dkeys [ffn]        (one token: the single-token kernel)
//   | idx_gate, idx_up [B][d] | idx_down [B][ffn] | cnt [3][B] | xs_gate, xs_up [B][d]
//   | xs_down [B][ffn] | g, u [B][ffn] | spmv ws of gate, up, down   (the batched path)
struct FfnWs {
  size_t bar, groups, h, keep_g, keep_u, keep_d, stamps, cta_t, part, pstride, dkeys, idx_gate, idx_up, idx_down, cnt,
      xs_gate, xs_up, xs_down, g, u, spmv, spmv2, spmv3, total;
};
inline FfnWs ffn_ws_layout(int64_t d, int64_t ffn, int64_t B) {
  FfnWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = round_up(o + bytes, kAlign);
    return at;
  };
  const bool one = B == 1;
  w.bar = take(sizeof(GridBarrier));
  // arrival counters of the single-token kernel's column groups (zero between calls)
  w.groups = take((size_t)2 * kGridCap * 4);
  w.h = take((size_t)B * ffn * 4);
  w.keep_g = take((size_t)B * d);
  w.keep_u = take((size_t)B * d);
  w.keep_d = take((size_t)B * ffn);
  w.stamps = take((size_t)kFfnStamps * 8);
  w.cta_t = take((size_t)kGridCap * 4 * 8);
  // partial rows: a multiple of 4 floats plus 4, so that the same column of successive
  // rows (read together when the rows are summed) does not fall on one L2 slice
  w.pstride = (size_t)((ffn > d ? ffn : d) + 3) / 4 * 4 + 4;
  w.part = take(one ? (size_t)kDecodeRows * w.pstride * 4 : 0);
  w.dkeys = take(one ? (size_t)ffn * 4 : 0);
  // the batched path (several tokens, or one token of a shape the single-token kernel
  // does not take)
  w.idx_gate = take((size_t)B * d * 4);
  w.idx_up = take((size_t)B * d * 4);
  w.idx_down = take((size_t)B * ffn * 4);
  w.cnt = take((size_t)3 * B * 4);
  w.xs_gate = take((size_t)B * d * 4);
  w.xs_up = take((size_t)B * d * 4);
  w.xs_down = take((size_t)B * ffn * 4);
  w.g = take((size_t)B * ffn * 4);
  w.u = take((size_t)B * ffn * 4);
  // the products' workspaces: gate, up (its own, so that it can run beside the gate's),
  // down (its own shape: the union path keeps parts of its workspace zero between calls)
  w.spmv = take(spmv_total_ws(d, ffn, B));
  w.spmv2 = take(spmv_total_ws(d, ffn, B));
  w.spmv3 = take(spmv_total_ws(ffn, d, B));
  w.total = o;
  return w;
}

// ----------------------------------------------------------------------------------
// launchers implemented in the kernel files (arguments already checked)
// ----------------------------------------------------------------------------------

// keep (optional): the kept set as bytes [batch][n]; uflag (optional): the union flags of
// the union path, set to 1 at every token's kept channels.
wina_status_t launch_select_topk(const void* x, int xdt, const float* c, int n, int k, int batch, int32_t* idx,
                                 float* xs, int ld, float* scores, cudaStream_t s, uint8_t* keep = nullptr,
                                 uint8_t* uflag = nullptr);
wina_status_t launch_stat_threshold(const void* v, int vdt, int n, double z, int batch, int32_t* idx, float* xs,
                                    int32_t* count, float* t, int cap, int32_t* status_dev, cudaStream_t s,
                                    uint8_t* keep = nullptr, uint8_t* uflag = nullptr);
wina_status_t launch_sparse_matvec(const void* Wt, int wdt, int64_t n, int64_t m, const int32_t* idx,
                                   const float* xs, int k, const int32_t* count, int ld_idx, int batch, float* y,
                                   void* ws, int32_t* status_dev, cudaStream_t s, bool premarked = false);
// The union flags in sparse_matvec's workspace `ws` for this call, when the union path
// serves it with a single token block (so that a gate can mark them); nullptr otherwise.
uint8_t* union_flags_for(void* ws, int wdt, int64_t n, int64_t m, int64_t batch);
wina_status_t launch_silu_mul(const float* g, const float* u, float* h, int64_t count, cudaStream_t s);
// Workspace bytes of spark_ffn_swiglu (spark.cu).
size_t spark_ws_size(int64_t d, int64_t ffn);
size_t dense_ws_size(int64_t d, int64_t ffn);
// The union path (union_gemm.cu); ws is the union region of the workspace. premarked: the
// union flags were already set by the gate that made the lists (launch_select_topk's
// uflag), which serves a single token block (batch <= kUBlock).
wina_status_t launch_union_matvec(const void* Wt, int64_t n, int64_t m, const int32_t* idx, const float* xs, int k,
                                  const int32_t* count, int ld, int batch, float* y, void* ws, int32_t* status,
                                  cudaStream_t s, bool premarked = false);
// The single-token FFN kernel (ffn_decode.cu). Returns WINA_ERR_UNSUPPORTED_DTYPE without
// launching anything when the shape is outside what it takes.
wina_status_t launch_ffn_decode(const wina_ffn_t* f, const void* x, int xdt, int mode, int k_gate, int k_up,
                                int k_down, double z, float* y, const FfnWs& L, char* w, int32_t* status,
                                cudaStream_t st);

}  // namespace wina
