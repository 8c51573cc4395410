"""Benchmark: gated SwiGLU FFN decode, Llama-7B shape (d 4096, ffn 11008, bf16), batch 1.

One step = one pass of the whole hot path over L distinct layers (each with its own
packed weight copy and its own resident input): per layer the three gates
(top-K of |x*c|), the three sparse products and the SwiGLU glue, i.e. one
sparse_ffn_swiglu call. The L weight copies (2.2 GB at L = 8) exceed the 126 MB L2,
so every step streams its kept rows from HBM.

Printed (rank 0, one JSON line): effective HBM GB/s on the bytes the kept rows and the
vectors require (value; whole job), us per layer, the roofline of the fused kernel
against the measured HBM copy bandwidth (with the ncu DRAM traffic of one launch when
profiles/ holds it for this kernel source), the dense comparator (a dedicated dense
FFN kernel on the output-major weights), 16 tokens per call on the batched path (against
the union of the kept rows), the other workloads of the scope table, the end-to-end
figure through the C ABI with host buffers, and the CPU oracle's time on a bounded
sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--p 0.5] [--layers 8]
  python bench.py --impl reference ...   # the CPU oracle, timed on the host cores
  python bench.py --profile-case NAME    # one call of a workload three times, for ncu
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "µs/layer & effective HBM GB/s (% of peak), Llama-7B FFN sparse GEMV, bs1"
D, FFN = 4096, 11008


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def layer_bytes(kg: int, ku: int, kd: int, d: int = D, ffn: int = FFN) -> int:
    """Algorithmic HBM bytes of one layer: the kept rows of the three bf16 weights plus
    the vectors that must cross HBM (x bf16, c_gate/c_up/c_down float32, y float32)."""
    rows = (kg + ku) * ffn * 2 + kd * d * 2
    vecs = d * 2 + 2 * d * 4 + ffn * 4 + d * 4
    return rows + vecs


# ------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------


class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------
# the CPU oracle leg (reference arm and cpu_baseline)
# ------------------------------------------------------------------------------------


def oracle_sample(p: float, budget_s: float = 12.0, max_tokens: int = 20, threads: int | None = None) -> dict:
    """Time the CPU oracle's per-token FFN (select + float64 products) on one layer of
    the same workload, as many tokens as fit in about budget_s seconds; with `threads`,
    the BLAS thread pools are limited to that many threads for the run."""
    if threads is not None:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=threads):
            return oracle_sample(p, budget_s, max_tokens)
    import oracle as O

    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        blas_threads = 1
    cfg = synth.make_llama7b_ffn(batch=max_tokens, p=p)
    Wg, Wu, Wd = (O.widen_bf16(cfg[k]) for k in ("Wg", "Wu", "Wd"))
    cg, cu, cd = O.col_norms(Wg), O.col_norms(Wu), O.col_norms(Wd)
    x32 = synth.f32_from_bf16_bits(cfg["x"])
    times = []
    t_all = time.perf_counter()
    for b in range(max_tokens):
        t0 = time.perf_counter()
        O.ffn_swiglu(Wg, Wu, Wd, cg, cu, cd, x32[b], cfg["k_gate"], cfg["k_up"], cfg["k_down"])
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s and len(times) >= 3:
            break
    us = statistics.median(times) * 1e6
    nbytes = layer_bytes(cfg["k_gate"], cfg["k_up"], cfg["k_down"])
    return {"us_per_layer": us, "gbs": nbytes / (us * 1e-6) / 1e9, "tokens": len(times),
            "cores": int(blas_threads), "host_cpus": os.cpu_count()}


def oracle_steps(p: float, steps: int, warmup: int) -> dict:
    """The reference arm: the CPU oracle as it stands, one step = one token through one
    layer of the workload (select + float64 products of the three projections). The
    layer is drawn once (untimed); `warmup` tokens run first, then `steps` tokens are
    timed one by one. Returns the measured time and the throughput on the algorithmic
    bytes of the steps that ran."""
    import oracle as O

    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        blas_threads = 1
    cfg = synth.make_llama7b_ffn(batch=steps + warmup, p=p)
    Wg, Wu, Wd = (O.widen_bf16(cfg[k]) for k in ("Wg", "Wu", "Wd"))
    cg, cu, cd = O.col_norms(Wg), O.col_norms(Wu), O.col_norms(Wd)
    x32 = synth.f32_from_bf16_bits(cfg["x"])

    def run(b):
        O.ffn_swiglu(Wg, Wu, Wd, cg, cu, cd, x32[b], cfg["k_gate"], cfg["k_up"], cfg["k_down"])

    for b in range(warmup):
        run(b)
    t0 = time.perf_counter()
    for b in range(warmup, warmup + steps):
        run(b)
    timed = time.perf_counter() - t0
    nbytes = layer_bytes(cfg["k_gate"], cfg["k_up"], cfg["k_down"])
    return {"steps": steps, "timed_s": timed, "us_per_step": timed / steps * 1e6,
            "gbs": nbytes * steps / timed / 1e9, "cores": int(blas_threads), "host_cpus": os.cpu_count()}


# ------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------


def _events(torch, stream, fn, steps: int) -> float:
    """ms of `steps` calls of fn, CUDA events on `stream` (synchronised on both sides)."""
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def graph_us(torch, fn, steps: int, warm: int = 3) -> float:
    """Microseconds per call of fn(), captured once as a CUDA graph and replayed `steps`
    times between two events on the current stream (synchronised on both sides)."""
    stream = torch.cuda.current_stream()
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        fn()  # warm the library's per-device caches outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.synchronize()
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return ms * 1e3 / steps


def _dev_bf16(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _frac(nbytes: float, us: float, peak: float) -> dict:
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"us": us, "effective_gbs": gbs, "frac_of_measured_hbm": gbs / peak, "bytes": int(nbytes)}


def measure_spark(W, torch, steps: int, peak: float, batches=(1, 2, 4, 8, 16, 32, 64), copies: int = 4) -> dict:
    """Gemma-2-2B FFN (d 2304, ffn 9216, bf16) with the Spark statistical gate (keep
    fraction 0.08) on every projection, `copies` distinct weight copies (4 x 127 MB, above
    L2) called in turn, for several token counts; and, on the stand-alone Gaussian vectors
    of the workload (2304 and 9216 long, 64 tokens), the overlap of the Spark set with the
    exact top-k of the signed values (k = round(s n)), from the GPU's kept sets and a numpy
    sort. Bytes: the kept rows (read back from the call's kept-set views; the union over
    the tokens when several) plus the vectors."""
    cfg = synth.make_gemma2_2b_spark(batch=max(batches))
    d, ffn, s = cfg["d"], cfg["ffn"], cfg["s"]
    fs = []
    for _ in range(copies):
        fs.append(W.ffn_prepare(*(_dev_bf16(torch, cfg[k]) for k in ("Wg", "Wu", "Wd"))))
    xall = _dev_bf16(torch, cfg["x_bf16"])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = {"gate": "Spark statistical top-k, s = 0.08, every projection", "by_batch": {}}
    for B in batches:
        x = xall[:B].contiguous()
        ws = W.Workspace(W.OP_FFN_SWIGLU, d, ffn, 0, B)
        y = torch.empty((B, d), dtype=torch.float32, device="cuda")

        def step():
            for f in fs:
                W.sparse_ffn_swiglu(f, x, W.GATE_STAT, s=s, ws=ws, status=st, y=y)

        us = graph_us(torch, step, steps) / copies
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())}")
        v = W.ffn_ws_view(ws, d, ffn, B)
        kg, ku, kd = (int(v[k].bool().any(0).sum().item()) for k in ("keep_gate", "keep_up", "keep_down"))
        nbytes = (kg + ku) * ffn * 2 + kd * d * 2 + B * (d * 2 + d * 4)
        out["by_batch"][str(B)] = dict(_frac(nbytes, us, peak), us_per_layer=us, union_kept=[kg, ku, kd])
        del ws, y
    # overlap with the exact top-k of the signed values
    ov = {}
    for name, arr in (("x_2304", cfg["x"]), ("v_9216", cfg["v"])):
        n = arr.shape[1]
        k = synth.spark_keep_count(s, n)
        idx, _, cnt, _ = W.stat_topk_threshold(torch.from_numpy(arr).cuda(), s)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        rec, jac = [], []
        for b in range(arr.shape[0]):
            S = set(idx[b, :cnt[b]].tolist())
            T = set(np.argsort(-arr[b], kind="stable")[:k].tolist())
            inter = len(S & T)
            rec.append(inter / k)
            jac.append(inter / max(1, len(S | T)))
        ov[name] = {"k": k, "mean_kept": float(cnt.mean()), "recall_vs_exact_topk": float(np.mean(rec)),
                    "jaccard": float(np.mean(jac)), "tokens": int(arr.shape[0])}
    out["overlap_with_exact_topk"] = ov
    return out


def measure_ultrasparse(W, torch, steps: int, peak: float, copies: int = 2) -> dict:
    """Down projection 14336 -> 4096 (bf16), 256 tokens with 143 nonzero inputs each: the
    nonzero set selected on the GPU and the union-row tensor-core product, per step;
    `copies` distinct weight copies (2 x 117 MB) called in turn, as a CUDA graph. Bytes:
    the union of the tokens' columns (read once) plus the inputs and outputs."""
    cfg = synth.make_ultrasparse_down()
    n, m, nnz = cfg["n"], cfg["m"], cfg["nnz"]
    Wts = [W.pack_in_major(_dev_bf16(torch, cfg["W"])) for _ in range(copies)]
    xb = _dev_bf16(torch, cfg["x"])
    B = xb.shape[0]
    ws = W.Workspace(W.OP_SPARSE_MATVEC, n, m, nnz, B)
    y = torch.empty((B, m), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.empty((B, nnz), dtype=torch.int32, device="cuda")
    xs = torch.empty((B, nnz), dtype=torch.float32, device="cuda")

    def step():
        for Wt in Wts:
            W.lib.wina_select_topk(W._ptr(xb), W.BF16, None, n, nnz, B, W._ptr(idx), W._ptr(xs), None, W._stream())
            W.sparse_matvec(Wt, idx, xs, ws=ws, status=st, y=y)

    us = graph_us(torch, step, steps) / copies
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())}")
    union = int(torch.unique(idx).numel())
    nbytes = union * m * 2 + B * n * 2 + B * m * 4
    mm = graph_us(torch, lambda: [W.sparse_matvec(Wt, idx, xs, ws=ws, status=st, y=y) for Wt in Wts], steps) / copies
    return dict(_frac(nbytes, us, peak), us_per_call=us, union_columns=union, product_only_us=mm,
                useful_gflop=2.0 * m * nnz * B / 1e9, union_mma_gflop=2.0 * m * union * B / 1e9,
                path="wina_select_topk (nonzero set) + sparse_matvec (union of the 256 tokens' rows on tcgen05)")


def measure_ds_decode(W, torch, steps: int, peak: float, batches=(1, 8), copies: int = 3) -> dict:
    """Double Sparsity decode attention on Llama-2-7B attention shapes (32 query and key/
    value heads of 128 channels, 4096 cached tokens, bf16 caches; 16 important channels
    per head, 256 tokens kept = 1/16): per batch size, `copies` distinct caches (above L2
    together) called in turn inside a CUDA graph. Bytes: the label rows of every token,
    the kept tokens' key and value rows, q and the output. Also, for B = 1, the kept sets'
    recall of the exact top-256 by the full q . K (numpy on the synthetic cache) and the
    output's relative L2 distance from full attention over all 4096 tokens."""
    r, k = 16, 256
    out = {"path": "ds_label_build (prefill, untimed) + ds_decode_attention", "r": r, "k": k, "by_batch": {}}
    for B in batches:
        cfg = synth.make_ds_decode(batch=B)
        Hq, Hkv, T, dh = cfg["Hq"], cfg["Hkv"], cfg["Tmax"], cfg["dh"]
        seq = torch.from_numpy(cfg["seq_len"]).cuda()
        C = torch.from_numpy(cfg["outliers"]).cuda()
        sets = []
        for c in range(copies):
            q, K, V = (_dev_bf16(torch, cfg[n]) for n in ("q", "K", "V"))
            if c:
                K = K.roll(c, dims=2).contiguous()  # a distinct cache, same statistics
                V = V.roll(c, dims=2).contiguous()
            sets.append((q, K, V, W.ds_label_build(K, seq, C)))
        o = torch.empty((B, Hq, dh), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")

        def step():
            for (q, K, V, lab) in sets:
                W.ds_decode_attention(q, K, V, lab, C, seq, k, out=o, status=st)

        us = graph_us(torch, step, steps) / copies
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())}")
        nbytes = B * Hkv * T * r * 2 + B * Hq * k * dh * 2 * 2 + B * Hq * dh * (2 + 4)
        line = dict(_frac(nbytes, us, peak), us_per_step=us, heads=Hq, tokens=T, head_dim=dh)
        if B == 1:
            q, K, V, lab = sets[0]
            o1, idx, _ = W.ds_decode_attention(q, K, V, lab, C, seq, k, want_idx=True)
            idx = idx.cpu().numpy()[0]
            qf = synth.f32_from_bf16_bits(cfg["q"])[0].astype(np.float64)
            Kf = synth.f32_from_bf16_bits(cfg["K"])[0].astype(np.float64)
            Vf = synth.f32_from_bf16_bits(cfg["V"])[0].astype(np.float64)
            rec, err = [], []
            full_out = np.zeros((Hq, dh))
            for h in range(Hq):
                sc = Kf[h] @ qf[h]
                top = np.argsort(-sc, kind="stable")[:k]
                rec.append(len(set(top.tolist()) & set(idx[h].tolist())) / k)
                lg = sc / np.sqrt(dh)
                p = np.exp(lg - lg.max())
                full_out[h] = (p / p.sum()) @ Vf[h]
            ds_out = o1.cpu().numpy()[0].astype(np.float64)
            line["recall_vs_exact_topk"] = float(np.mean(rec))
            line["rel_l2_vs_full_attention"] = float(np.linalg.norm(ds_out - full_out) / np.linalg.norm(full_out))
        out["by_batch"][str(B)] = line
        del sets
    return out


def measure_llama3_layer(W, torch, steps: int, peak: float, batches=(1, 4, 16)) -> dict:
    """Llama-3-8B-shaped decoder layer (bf16): Q/K/V/O as gated sparse products (each its
    own top-K of |input * c|; Q, K, V gate the hidden state, O an independent input since
    no attention core is in scope) and the gated SwiGLU FFN (gate/up 4096 -> 14336, down
    14336 -> 4096), per-projection sparsity from the workload's seeded schedule, one layer
    (436 MB of weights, above L2) per step, as a CUDA graph. Bytes: each projection's kept
    rows (their union over the tokens) plus the vectors."""
    cfg = synth.make_llama3_8b_layer(batch=max(batches))
    k = cfg["k"]
    Wt, c = {}, {}
    for name in ("q", "k", "v", "o"):
        Wd = _dev_bf16(torch, cfg["W"][name])
        Wt[name], c[name] = W.pack_in_major(Wd), W.col_norms(Wd)
        del Wd
    f = W.ffn_prepare(*(_dev_bf16(torch, cfg["W"][nm]) for nm in ("gate", "up", "down")))
    del cfg["W"]
    xall = _dev_bf16(torch, cfg["x"])
    oall = _dev_bf16(torch, cfg["o_in"])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = {"k": k, "p": cfg["p"], "by_batch": {}}
    for B in batches:
        x, o_in = xall[:B].contiguous(), oall[:B].contiguous()
        sel = {nm: (torch.empty((B, k[nm]), dtype=torch.int32, device="cuda"),
                    torch.empty((B, k[nm]), dtype=torch.float32, device="cuda")) for nm in ("q", "k", "v", "o")}
        ys = {nm: torch.empty((B, Wt[nm].shape[1]), dtype=torch.float32, device="cuda") for nm in ("q", "k", "v", "o")}
        wss = {nm: W.Workspace(W.OP_SPARSE_MATVEC, 4096, Wt[nm].shape[1], k[nm], B) for nm in ("q", "k", "v", "o")}
        fws = W.Workspace(W.OP_FFN_SWIGLU, 4096, 14336, 0, B)
        yf = torch.empty((B, 4096), dtype=torch.float32, device="cuda")

        def step():
            for nm in ("q", "k", "v", "o"):
                inp = o_in if nm == "o" else x
                idx, xs = sel[nm]
                W.lib.wina_select_topk(W._ptr(inp), W.BF16, W._ptr(c[nm]), 4096, k[nm], B, W._ptr(idx), W._ptr(xs),
                                       None, W._stream())
                W.sparse_matvec(Wt[nm], idx, xs, ws=wss[nm], status=st, y=ys[nm])
            W.sparse_ffn_swiglu(f, x, W.GATE_TOPK, k["gate"], k["up"], k["down"], ws=fws, status=st, y=yf)

        us = graph_us(torch, step, steps)
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())}")
        nbytes = 0
        for nm in ("q", "k", "v", "o"):
            nbytes += int(torch.unique(sel[nm][0]).numel()) * Wt[nm].shape[1] * 2
        v = W.ffn_ws_view(fws, 4096, 14336, B)
        ug, uu, ud = (int(v[kk].bool().any(0).sum().item()) for kk in ("keep_gate", "keep_up", "keep_down"))
        nbytes += (ug + uu) * 14336 * 2 + ud * 4096 * 2 + B * 4096 * 2 * 2
        out["by_batch"][str(B)] = dict(_frac(nbytes, us, peak), us_per_layer=us,
                                       path="per-token kernels (B = 1) / union-row tcgen05 products (B >= 4)")
        del sel, ys, wss, fws, yf
    return out


def reduce_max(v: float, world: int, device: str) -> float:
    """The maximum of v over the ranks of the default process group (every rank must
    call it; a single process returns v). Times are taken as the max over ranks."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())



PROFILE_CASES = ("ffn_decode", "dense_ffn", "union_b256", "batched_b16", "spark_ffn", "ds_decode")


def profile_case(name: str) -> None:
    """One hot-path call of the named workload, three times on one input (the weights once
    on the device, a few hundred MB), for single-kernel ncu captures: no timing, no
    output besides a status line. ffn_decode: the Llama-7B FFN at 50% sparsity, bs1 (the
    single-token kernel); dense_ffn: its dense comparator; union_b256: the ultra-sparse
    down projection, 256 tokens (the tcgen05 union product); batched_b16: the Llama-7B
    FFN at 16 tokens; spark_ffn: the Gemma-2-2B FFN with the Spark gate, bs1; ds_decode:
    Double Sparsity decode attention, Llama-2-7B shapes, 8 sequences."""
    import torch
    import free_activation_sparse_b200 as W

    torch.cuda.set_device(0)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if name in ("ffn_decode", "dense_ffn", "batched_b16"):
        cfg = synth.make_llama7b_ffn(batch=16 if name == "batched_b16" else 1)
        Wg, Wu, Wd = (_dev_bf16(torch, cfg[k]) for k in ("Wg", "Wu", "Wd"))
        x = _dev_bf16(torch, cfg["x"])
        if name == "dense_ffn":
            ws = W.Workspace(W.OP_DENSE_FFN, D, FFN, 0, 1)
            calls = [lambda: W.dense_ffn_swiglu(Wg, Wu, Wd, x[0], ws=ws, status=st)]
        else:
            f = W.ffn_prepare(Wg, Wu, Wd)
            del Wg, Wu, Wd
            B = x.shape[0]
            ws = W.Workspace(W.OP_FFN_SWIGLU, D, FFN, 0, B)
            calls = [lambda: W.sparse_ffn_swiglu(f, x, W.GATE_TOPK, cfg["k_gate"], cfg["k_up"], cfg["k_down"], ws=ws,
                                                 status=st)]
    elif name == "union_b256":
        cfg = synth.make_ultrasparse_down()
        Wt = W.pack_in_major(_dev_bf16(torch, cfg["W"]))
        xb = _dev_bf16(torch, cfg["x"])
        idx, xs = W.select_topk(xb, None, cfg["nnz"])
        ws = W.Workspace(W.OP_SPARSE_MATVEC, cfg["n"], cfg["m"], cfg["nnz"], xb.shape[0])
        calls = [lambda: W.sparse_matvec(Wt, idx, xs, ws=ws, status=st)]
    elif name == "spark_ffn":
        cfg = synth.make_gemma2_2b_spark(batch=1)
        f = W.ffn_prepare(*(_dev_bf16(torch, cfg[k]) for k in ("Wg", "Wu", "Wd")))
        x = _dev_bf16(torch, cfg["x_bf16"][:1])
        ws = W.Workspace(W.OP_FFN_SWIGLU, cfg["d"], cfg["ffn"], 0, 1)
        calls = [lambda: W.sparse_ffn_swiglu(f, x, W.GATE_STAT, s=cfg["s"], ws=ws, status=st)]
    elif name == "ds_decode":
        cfg = synth.make_ds_decode(batch=8)
        q, K, V = (_dev_bf16(torch, cfg[n]) for n in ("q", "K", "V"))
        seq = torch.from_numpy(cfg["seq_len"]).cuda()
        C = torch.from_numpy(cfg["outliers"]).cuda()
        lab = W.ds_label_build(K, seq, C)
        calls = [lambda: W.ds_decode_attention(q, K, V, lab, C, seq, 256, status=st)]
    else:
        raise SystemExit(f"unknown profile case {name}; one of {PROFILE_CASES}")
    for _ in range(3):
        for c in calls:
            c()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise SystemExit(f"{name}: device status {int(st.item())}")
    print(f"ok {name}", flush=True)
    if name == "ffn_decode":
        # the single-token kernel's phase stamps (CTA 0's clock at each phase boundary, read
        # back from the workspace) over 20 more calls, median microseconds per phase
        phases = ["A keys", "A select", "A flags+list", "B loop", "B store", "B group sum", "B tail",
                  "barrier", "C2 keys", "C2 select", "C2 flags+list", "E loop", "E store", "E arrive", "E group sum"]
        mhz = 1965.0  # SM clock under load in the bench's clock samples (the B200's maximum)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        runs = []
        for _ in range(20):
            flush.zero_()
            calls[0]()
            torch.cuda.synchronize()
            sv = W.ffn_ws_view(ws, D, FFN, 1)["stamps"].cpu().numpy()[:16].astype(np.float64)
            runs.append(np.diff(sv) / mhz)
        med = np.median(np.array(runs), axis=0)
        print("phases_us " + json.dumps({n: round(float(v), 2) for n, v in zip(phases, med)}) +
              f" total {float(med.sum()):.1f} (clock {mhz:.0f} MHz)", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--p", type=float, default=0.5, help="dropped fraction per projection")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run one hot-path call of this workload three times (for ncu) and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    kg = synth.keep_count(args.p, D)
    kd = synth.keep_count(args.p, FFN)
    nbytes = layer_bytes(kg, kg, kd)
    config = {"workload": f"llama7b_ffn_4096x11008_bf16 decode bs1, top-K per projection at "
                          f"{int(round(args.p * 100))}% sparsity (K={kg}/{kg}/{kd})",
              "d": D, "ffn": FFN, "batch": 1, "p": args.p, "layers_per_step": args.layers,
              "l2": "inputs larger than L2: distinct weight copies per layer", "parallelism": f"replicas{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        r = oracle_steps(args.p, args.steps, args.warmup)
        line = {"metric": METRIC, "impl": "reference", "value": r["gbs"], "unit": "GB/s",
                "us_per_layer": r["us_per_step"], "n_gpus": args.gpus, "steps": r["steps"], "warmup": args.warmup,
                "ms_per_step": r["us_per_step"] / 1e3, "timed_s": r["timed_s"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": r["gbs"], "unit": "GB/s", "cores": r["cores"], "host_cpus": r["host_cpus"],
                                 "kind": "oracle",
                                 "sample": f"each step: one token through one layer of the workload "
                                           f"({r['steps']} timed steps after {args.warmup} warm-up steps)"},
                "e2e": {"value": r["gbs"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    import free_activation_sparse_b200 as W

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, "cuda")

    # ---- untimed setup: L layers of weights (packed + norms on the GPU), inputs ----
    L = args.layers
    layers, xs, outmajor = [], [], []
    for l in range(L):
        cfg = synth.make_llama7b_ffn(batch=1, p=args.p, layer=l + 1000 * rank)
        up = [torch.from_numpy(cfg[k].view(np.int16)).cuda().view(torch.bfloat16) for k in ("Wg", "Wu", "Wd")]
        layers.append(W.ffn_prepare(*up))
        outmajor.append(up)  # the unpacked weights, for the dense comparator
        xs.append(torch.from_numpy(cfg["x"].view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    ws = W.Workspace(W.OP_FFN_SWIGLU, D, FFN, 0, 1)
    ys = [torch.empty((1, D), dtype=torch.float32, device="cuda") for _ in range(L)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(mode=W.GATE_TOPK, ev=None):
        for l in range(L):
            if ev is not None:
                ev[l][0].record(stream)
            W.sparse_ffn_swiglu(layers[l], xs[l], mode, kg, kg, kd, ws=ws, status=status, y=ys[l])
            if ev is not None:
                ev[l][1].record(stream)

    def capture(mode):
        """The L-layer step as one CUDA graph (launch overhead leaves the timed loop)."""
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(mode)  # warm the library's per-device caches outside capture
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=side):
                step(mode)
        torch.cuda.synchronize()
        return g

    def timed_graph(g, K):
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(K):
            g.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return t0.elapsed_time(t1)

    def timed_eager(mode, K):
        evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(L)]
               for _ in range(K)]
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for k in range(K):
            step(mode, evs[k])
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        per = statistics.mean(e[0].elapsed_time(e[1]) for row in evs for e in row)
        return t0.elapsed_time(t1), per

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    graph = capture(W.GATE_TOPK)
    for _ in range(args.warmup):
        graph.replay()
    clocks = ClockSampler(local)
    clocks.start()
    total_ms = timed_graph(graph, args.steps)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")
    eager_ms, eager_kern_ms = timed_eager(W.GATE_TOPK, max(3, args.steps // 2))
    eager_ms = max_over_ranks(eager_ms)
    eager_kern_ms = max_over_ranks(eager_kern_ms)

    ms_per_step = total_ms / args.steps
    us_layer = ms_per_step * 1e3 / L
    kern_ms = ms_per_step / L  # graph replay: per-launch time including the gap to the next launch
    gbs = world * nbytes * L * args.steps / (total_ms * 1e-3) / 1e9

    peak, peak_kind = _peaks()
    nsteps = max(3, args.steps // 2)

    # dense comparator: the unsparsified FFN on the output-major weights (one cooperative
    # launch streaming the weights as flat slab ranges, no selection)
    dws = W.Workspace(W.OP_DENSE_FFN, D, FFN, 0, 1)
    dst = torch.zeros(1, dtype=torch.int32, device="cuda")

    def dense_step():
        for l in range(L):
            W.dense_ffn_swiglu(outmajor[l][0], outmajor[l][1], outmajor[l][2], xs[l][0], y=ys[l][0], ws=dws,
                               status=dst)

    us_layer_dense = max_over_ranks(graph_us(torch, dense_step, nsteps)) / L
    if int(dst.item()) != 0:
        raise RuntimeError(f"dense comparator: device status {int(dst.item())}")
    dense_bytes = 3 * D * FFN * 2 + D * 2 + D * 4
    # the decode kernel itself with every channel kept (its own dense mode)
    us_layer_dense_mode = max_over_ranks(graph_us(torch, lambda: step(W.GATE_DENSE), nsteps)) / L

    # the headline layer at 65% sparsity (K = 1434 / 1434 / 3853)
    kg65, kd65 = synth.keep_count(0.65, D), synth.keep_count(0.65, FFN)

    def step65():
        for l in range(L):
            W.sparse_ffn_swiglu(layers[l], xs[l], W.GATE_TOPK, kg65, kg65, kd65, ws=ws, status=status, y=ys[l])

    us65 = max_over_ranks(graph_us(torch, step65, nsteps)) / L
    p065 = dict(_frac(layer_bytes(kg65, kg65, kd65), us65, peak), us_per_layer=us65, k=[kg65, kg65, kd65])

    # the sparse product alone at batch 1: the gate projection's kept rows (4096 -> 11008,
    # K = kg) and the down projection's (11008 -> 4096, K = kd, on the h the FFN produced)
    sel_g, sel_d, yg, ydn = [], [], [], []
    mws = W.Workspace(W.OP_SPARSE_MATVEC, FFN, FFN, FFN, 1)
    for l in range(L):
        sel_g.append(W.select_topk(xs[l], layers[l].c_gate, kg))
        W.sparse_ffn_swiglu(layers[l], xs[l], W.GATE_TOPK, kg, kg, kd, ws=ws, status=status, y=ys[l])
        h = W.ffn_ws_view(ws, D, FFN, 1)["h"].clone()
        sel_d.append(W.select_topk(h, layers[l].c_down, kd))
        yg.append(torch.empty((1, FFN), dtype=torch.float32, device="cuda"))
        ydn.append(torch.empty((1, D), dtype=torch.float32, device="cuda"))
    us_mg = max_over_ranks(graph_us(torch, lambda: [W.sparse_matvec(layers[l].wt_gate, *sel_g[l], ws=mws,
                                                                    status=status, y=yg[l]) for l in range(L)],
                                    nsteps)) / L
    us_md = max_over_ranks(graph_us(torch, lambda: [W.sparse_matvec(layers[l].wt_down, *sel_d[l], ws=mws,
                                                                    status=status, y=ydn[l]) for l in range(L)],
                                    nsteps)) / L
    matvec_bs1 = {
        "gate_4096x11008_k%d" % kg: dict(_frac(kg * FFN * 2 + kg * 8 + FFN * 4, us_mg, peak), us_per_call=us_mg),
        "down_11008x4096_k%d" % kd: dict(_frac(kd * D * 2 + kd * 8 + D * 4, us_md, peak), us_per_call=us_md),
        "kernel": "k_spmv_cols (column groups x row groups, the last CTA of a column group sums its partials in order)"}
    del sel_g, sel_d, yg, ydn, mws

    # several tokens (the batched path): 16 tokens per call on the same layers; effective
    # bytes count the union of each projection's kept rows over the tokens
    BT = 16
    xbs, yb = [], torch.empty((BT, D), dtype=torch.float32, device="cuda")
    for l in range(L):
        cfgb = synth.make_llama7b_ffn(batch=BT, p=args.p, layer=l + 1000 * rank)
        xbs.append(torch.from_numpy(cfgb["x"].view(np.int16)).cuda().view(torch.bfloat16))
    wsb = W.Workspace(W.OP_FFN_SWIGLU, D, FFN, 0, BT)

    def batched_step():
        for l in range(L):
            W.sparse_ffn_swiglu(layers[l], xbs[l], W.GATE_TOPK, kg, kg, kd, ws=wsb, status=status, y=yb)

    union_bytes = 0
    for l in range(L):  # the kept sets of every layer (read back from the call's own views)
        W.sparse_ffn_swiglu(layers[l], xbs[l], W.GATE_TOPK, kg, kg, kd, ws=wsb, status=status, y=yb)
        v = W.ffn_ws_view(wsb, D, FFN, BT)
        ug, uu, ud = (int(v[k].bool().any(0).sum().item()) for k in ("keep_gate", "keep_up", "keep_down"))
        union_bytes += (ug + uu) * FFN * 2 + ud * D * 2 + BT * (D * 2 + D * 4) + (2 * D + FFN) * 4
    us_b = max_over_ranks(graph_us(torch, batched_step, nsteps)) / L
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the batched run")
    batched = dict(_frac(union_bytes / L, us_b, peak), batch=BT, us_per_layer=us_b,
                   union_bytes_per_layer=union_bytes // L,
                   path="batched calls: select, union-row tcgen05 product, silu*mul (per projection)")
    del xbs, yb, wsb

    # end to end through the C ABI: host x in pinned memory -> device, the call, y -> host
    hx = [x.cpu().pin_memory() for x in xs]
    hy = [torch.empty((1, D), dtype=torch.float32).pin_memory() for _ in range(L)]
    dx = [torch.empty_like(x) for x in xs]

    def e2e_step():
        for l in range(L):
            dx[l].copy_(hx[l], non_blocking=True)
            W.sparse_ffn_swiglu(layers[l], dx[l], W.GATE_TOPK, kg, kg, kd, ws=ws, status=status, y=ys[l])
            hy[l].copy_(ys[l], non_blocking=True)
        torch.cuda.synchronize()

    for _ in range(3):
        e2e_step()
    barrier()
    t_e0 = torch.cuda.Event(enable_timing=True)
    t_e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t_e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(t_e0.elapsed_time(t_e1))
    e2e_gbs = world * nbytes * L * args.steps / (e2e_ms * 1e-3) / 1e9

    # the other configurations of the scope table, measured on the same GPU (each guarded:
    # a failure is reported in its entry and never affects the headline line)
    extra = {}
    for name, fn in (("spark_ffn_gemma2_2b", lambda: measure_spark(W, torch, nsteps, peak)),
                     ("ultrasparse_down_b256", lambda: measure_ultrasparse(W, torch, nsteps, peak)),
                     ("llama3_8b_layer", lambda: measure_llama3_layer(W, torch, nsteps, peak)),
                     ("double_sparsity_decode_llama2_7b", lambda: measure_ds_decode(W, torch, nsteps, peak))):
        try:
            extra[name] = fn()
        except Exception as e:  # pragma: no cover - reported, not raised
            extra[name] = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.empty_cache()

    achieved = nbytes / (kern_ms * 1e-3) / 1e9
    traffic = None  # ncu dram bytes of one launch, valid only for the kernel it was taken on
    tf = os.path.join(ROOT, "profiles", "ffn_decode_llama7b_traffic.txt")
    if os.path.exists(tf):
        with open(tf) as f:
            tj = dict(line.strip().split("=", 1) for line in f if "=" in line)
        if float(tj.get("p", -1)) == args.p and tj.get("kernel_sha") == _kernel_sha():
            traffic = int(tj["dram_bytes_per_launch"])

    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "us_per_layer": us_layer,
        "pct_of_peak": 100.0 * gbs / world / peak, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 weights, f32 accumulate", "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                     "kernel": "k_ffn_decode (one launch per layer)", "bytes_per_launch": nbytes,
                     "kernel_us": kern_ms * 1e3, "timing": "CUDA graph of the L-layer step, events around K replays"},
        "eager": {"us_per_layer": eager_ms / max(3, args.steps // 2) * 1e3 / L,
                  "kernel_us_events": eager_kern_ms * 1e3},
        "dense": dict(_frac(dense_bytes, us_layer_dense, peak), us_per_layer=us_layer_dense,
                      speedup=us_layer_dense / us_layer, kernel="wina_dense_ffn_swiglu (output-major weights)",
                      decode_kernel_dense_mode_us=us_layer_dense_mode),
        "p065": p065,
        "sparse_matvec_bs1": matvec_bs1,
        "batched": batched,
        "other_configs": extra,
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "us_per_layer": e2e_ms / args.steps * 1e3 / L,
                "h2d_bytes_per_step": L * D * 2, "d2h_bytes_per_step": L * D * 4},
        "gpu_launches": L * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(args.p)
        r1 = oracle_sample(args.p, budget_s=8.0, max_tokens=5, threads=1)
        line["cpu_baseline"] = {"value": r["gbs"], "unit": "GB/s", "us_per_layer": r["us_per_layer"],
                                "cores": r["cores"], "host_cpus": r["host_cpus"], "kind": "oracle",
                                "sample": f"{r['tokens']} tokens through one layer (median per token)",
                                "one_thread": {"value": r1["gbs"], "us_per_layer": r1["us_per_layer"],
                                               "sample": f"{r1['tokens']} tokens, BLAS limited to one thread"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _kernel_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("common.cuh", "regsel.cuh", "colstream.cuh", "ffn_decode.cu"):
        with open(os.path.join(ROOT, "free_activation_sparse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
