// SwiGLU FFN with the gate on every projection ("WAS" article, core innovations:
// weight-aware sparsity per component, gate/up/down among them; "WINA" article, section
// 一: each projection scores with its own column norms and keeps its own K; "Spark
// Transformer", section 2.2: the statistical threshold variant).
//
// The C-ABI entry point. One token takes the single persistent kernel of ffn_decode.cu;
// several tokens (or shapes that kernel does not take) run as a sequence of batched
// calls: per projection its gate (which also writes the kept-set bytes and, for the union
// path, the union's flags) and its sparse product, with silu(g) * u before the down gate;
// the up projection runs on a side stream beside the gate projection.
#include <math.h>

#include <algorithm>
#include <cmath>

#include "internal.h"

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
    const wina_status_t rd = launch_ffn_decode(f, x, xdt, mode, (int)k_gate, (int)k_up, (int)k_down, z, y, L, w,
                                               status_dev, st);
    if (rd != WINA_ERR_UNSUPPORTED_DTYPE) return rd;
  }
  // Several tokens (or shapes the single-token kernel does not take): batched calls.
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
  void* sw = w + L.spmv;    // gate
  void* sw2 = w + L.spmv2;  // up
  void* sw3 = w + L.spmv3;  // down
  const int B = (int)batch;
  // union flags of each projection's product, set by the gate that makes its lists when
  // the union path serves the call
  uint8_t* uf_g = union_flags_for(sw, f->wdt, d, ffn, B);
  uint8_t* uf_u = union_flags_for(sw2, f->wdt, d, ffn, B);
  uint8_t* uf_d = union_flags_for(sw3, f->wdt, ffn, d, B);
  wina_status_t r;
  // The gate and up projections are independent until silu(g) * u: up runs on a side
  // stream beside gate when one is available (fork after the work enqueued so far, join
  // before silu).
  SideStream ss;
  std::unique_lock<std::mutex> lk = side_stream_lock();
  const bool par = side_stream(st, &ss);
  cudaStream_t su = st;
  if (par) {
    if ((r = cuda_status(cudaEventRecord(ss.fork_ev, st)))) return r;
    if ((r = cuda_status(cudaStreamWaitEvent(ss.s, ss.fork_ev, 0)))) return r;
    su = ss.s;
  }
  auto join = [&]() -> wina_status_t {
    if (!par) return WINA_OK;
    wina_status_t rj = cuda_status(cudaEventRecord(ss.join_ev, su));
    if (rj == WINA_OK) rj = cuda_status(cudaStreamWaitEvent(st, ss.join_ev, 0));
    lk.unlock();
    return rj;
  };
  if (mode == WINA_GATE_STAT) {
    // gate and up threshold the same signed x: one kept set serves both (up reads the
    // lists once they exist, so it waits for the threshold)
    if ((r = launch_stat_threshold(x, xdt, (int)d, z, B, ig, xg, cnt, nullptr, (int)d, status_dev, st, keep_g, uf_g)))
      return r;
    if (par) {
      if ((r = cuda_status(cudaEventRecord(ss.fork_ev, st)))) return r;
      if ((r = cuda_status(cudaStreamWaitEvent(su, ss.fork_ev, 0)))) return r;
    }
    if ((r = cuda_status(cudaMemcpyAsync(keep_u, keep_g, (size_t)B * d, cudaMemcpyDeviceToDevice, su)))) return r;
    if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, ig, xg, -1, cnt, (int)d, B, u, sw2, status_dev, su)))
      return r;
    if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, -1, cnt, (int)d, B, g, sw, status_dev, st,
                                  uf_g != nullptr)))
      return r;
    if ((r = join())) return r;
    if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
    if ((r = launch_stat_threshold(h, WINA_F32, (int)ffn, z, B, idn, xd, cnt + 2 * B, nullptr, (int)ffn, status_dev,
                                   st, keep_d, uf_d)))
      return r;
    return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, -1, cnt + 2 * B, (int)ffn, B, y, sw3, status_dev,
                                st, uf_d != nullptr);
  }
  const float* cg = mode == WINA_GATE_TOPK ? f->c_gate : nullptr;
  const float* cu = mode == WINA_GATE_TOPK ? f->c_up : nullptr;
  const float* cd = mode == WINA_GATE_TOPK ? f->c_down : nullptr;
  if ((r = launch_select_topk(x, xdt, cu, (int)d, (int)k_up, B, iu, xu, (int)d, nullptr, su, keep_u, uf_u))) return r;
  if ((r = launch_sparse_matvec(f->wt_up, f->wdt, d, ffn, iu, xu, (int)k_up, nullptr, (int)d, B, u, sw2, status_dev,
                                su, uf_u != nullptr)))
    return r;
  if ((r = launch_select_topk(x, xdt, cg, (int)d, (int)k_gate, B, ig, xg, (int)d, nullptr, st, keep_g, uf_g)))
    return r;
  if ((r = launch_sparse_matvec(f->wt_gate, f->wdt, d, ffn, ig, xg, (int)k_gate, nullptr, (int)d, B, g, sw,
                                status_dev, st, uf_g != nullptr)))
    return r;
  if ((r = join())) return r;
  if ((r = launch_silu_mul(g, u, h, (int64_t)B * ffn, st))) return r;
  if ((r = launch_select_topk(h, WINA_F32, cd, (int)ffn, (int)k_down, B, idn, xd, (int)ffn, nullptr, st, keep_d,
                              uf_d)))
    return r;
  return launch_sparse_matvec(f->wt_down, f->wdt, ffn, d, idn, xd, (int)k_down, nullptr, (int)ffn, B, y, sw3,
                              status_dev, st, uf_d != nullptr);
}
