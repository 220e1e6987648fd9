"""Benchmark of the Gated DeltaNet hot path on B200.

One step = one pass of the whole layer path over one batch of synthetic input on the
27B-class long-prefill workload (T = 32768, 16 q/k and 32 v heads, d = 128, bf16): chunked
gated delta-rule scan -> gated RMSNorm * SiLU(z) with the fused NVFP4 activation encode ->
NVFP4 W4A4 output projection 4096 -> 2048. The same step on the 1024-wide layer (T = 4096,
16/16 heads, 2048 -> 1024) and on the variable-length batch (8 sequences, 16/32 heads) is
reported under "prefill_1024_wide" and "varlen"; the decode step (B = 256 sequences, fp32
state [256, 32, 128, 128] updated in place) under "decode".

Launch: python bench.py [--gpus N --steps K --warmup W] (N > 1 under torchrun, one rank
per GPU, each rank an independent replica of the workload: weak scaling, no collective
on the data path). `--impl reference` times the CPU oracle on the same workload instead.
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
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "GDN prefill tokens/s & decode GB/s (fraction of B200 roofline), 1 GPU"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def make_l2_flush(torch, dev):
    """L2 flush between timed steps: write a 256 MiB buffer (twice the 126 MB L2), then read a
    second one, so the next step starts with neither its inputs nor dirty lines in L2 (the
    write-back of the flush buffer happens here, outside the timed region)."""
    wbuf = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    rbuf = torch.zeros((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        wbuf.zero_()
        torch.sum(rbuf, dim=0, out=sink)
    return flush
CHUNK = 64
# FP4 (kind::mxf4nvf4) dense rate measured by a tcgen05 probe: 16368 MAC/cycle/SM x 148 SMs x 1965 MHz
FP4_PROBE_TFLOPS = 2.0 * 16368 * 148 * 1.965e9 / 1e12
# DRAM bytes of one fused prefill call (prep + lean + combine + the output pass with the gated
# tail) on the long-prefill workload, from one ncu capture with cold caches, keyed by the digest
# of the scan's source (null in the line once the source has changed)
SCAN_TRAFFIC = {"09b71335661839bc": 4580.83e6}


def source_digest(path: str) -> str:
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def scan_flops(w: workloads.Workload) -> float:
    """Algorithmic FLOPs of the chunked scan (64-token chunks, d = Dk = Dv): per token,
    Hv * (6 d^2 + 6 C d) for the state products, W, U~ and the intra-chunk output, plus
    Hk * 4 C d for K K^T and Q K^T (shared by the value heads of a key head)."""
    d, C = w.D, CHUNK
    return float(w.T) * (w.Hv * (6 * d * d + 6 * C * d) + w.Hk * 4 * C * d)


def fused_bytes(w: workloads.Workload) -> float:
    """Algorithmic HBM bytes of the fused prefill: q, k, v, z read once (bf16), a, b (fp32), the
    NVFP4 activations written (K/2 + K/16 bytes per token), initial/final states when present."""
    K = w.Hv * w.D
    b = w.T * (2 * w.Hk * w.D * 2 + 2 * w.Hv * w.D * 2 + 2 * w.Hv * 4 + K // 2 + K // 16)
    if w.s0_std > 0:
        b += 2 * w.num_seqs * w.Hv * w.D * w.D * 4
    return float(b)


def scan_bytes(w: workloads.Workload, o_bytes=2) -> float:
    """Algorithmic HBM bytes of the scan: q, k, v read once (bf16), a, b (fp32), o written,
    initial/final states when present."""
    b = w.T * (2 * w.Hk * w.D * 2 + w.Hv * w.D * 2 + 2 * w.Hv * 4 + w.Hv * w.D * o_bytes)
    if w.s0_std > 0:
        b += 2 * w.num_seqs * w.Hv * w.D * w.D * 4
    return float(b)


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 0.2 ms through NVML
    while the timed region runs (falls back to an nvidia-smi loop when NVML is missing)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._handle = None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.cuda_index)
        if hasattr(props, "pci_bus_id"):
            bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id, props.pci_device_id)
            self._handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        else:
            self._handle = pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)
        self._nvml = pynvml
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM))

    def _loop(self):
        nv, h = self._nvml, self._handle
        get_reasons = (getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None)
                       or nv.nvmlDeviceGetCurrentClocksThrottleReasons)
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = get_reasons(h)
                self.samples.append((float(mhz), int(reasons)))
            except Exception:  # noqa: BLE001 - a failed sample is skipped
                pass
            time.sleep(0.0002)

    def __enter__(self):
        try:
            self._open()
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()
            t0 = time.time()   # the timed region starts only once sampling runs
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.0005)
            self.samples.clear()
        except Exception:  # noqa: BLE001 - no NVML: report no samples
            self._thread = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=5)

    def summary(self):
        sm = [m for m, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 0.2 ms"}


# ----------------------------------------------------------------- GPU arm ----

def count_kernels(torch, fn):
    """This library's kernels launched by one call of fn (CUPTI kernel records through the
    profiler), and their names; falls back to the step's known launch sequence."""
    try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events()
                 if any(t in e.name for t in ("gdn_", "nvfp4_", "gated_rmsnorm"))]
        if names:
            def short(n):
                n = n.replace("(anonymous namespace)::", "").replace("void ", "")
                return n.split("(")[0].split("::")[-1]
            return len(names), sorted({short(n) for n in names})
    except Exception:  # noqa: BLE001 - no profiler: the static count below
        pass
    return 5, ["gdn_chunk_prep_kernel", "gdn_chunk_lean_kernel", "gdn_segment_combine_kernel",
               "gdn_chunk_chain_kernel<true>", "nvfp4_gemm_kernel"]


def prefill_case(torch, g, w, args, dev, flush, side, with_e2e=False, with_parts=False):
    """One prefill workload end to end: the step (fused prefill = scan + gated RMSNorm + NVFP4
    encode in the output pass, then the NVFP4 W4A4 output projection) captured in a CUDA graph
    and replayed with the L2 flushed before each replay; the fused prefill and the GEMM alone the
    same way. Returns the timings, the inputs (for the oracle baseline) and, when asked, the
    end-to-end timing through the public API from pinned host buffers."""
    x = workloads.generate(w)
    bf, f32 = torch.bfloat16, torch.float32

    def up(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)

    q, k, v, z = up(x["q"], bf), up(x["k"], bf), up(x["v"], bf), up(x["z"], bf)
    a, b = up(x["a"], f32), up(x["b"], f32)
    A_log, dt_bias, nw = up(x["A_log"], f32), up(x["dt_bias"], f32), up(x["norm_weight"], f32)
    cu = up(x["cu_seqlens"], torch.int32) if w.num_seqs > 1 else None
    S0 = None if x["initial_state"] is None else up(x["initial_state"], f32)
    W = up(x["proj_weight"], bf)
    gw = float(448.0 * 6.0 / W.float().abs().max().item())
    wq, ws_w = g.nvfp4_quantize_act(W, gw)         # weights: quantised once, outside timing
    T, Hv, D, K, N = w.T, w.Hv, w.D, w.K, w.n_out
    S = torch.empty((w.num_seqs, Hv, D, D), dtype=f32, device=dev)
    xq = torch.empty((T, K // 2), dtype=torch.uint8, device=dev)
    xs = torch.empty((T, K // 16), dtype=torch.uint8, device=dev)
    Y = torch.empty((T, N), dtype=bf, device=dev)
    ws = torch.empty((g.gdn_prefill_workspace_bytes(T, w.num_seqs, w.Hk, Hv, D, D),), dtype=torch.uint8, device=dev)
    # activation global scale: one calibration pass outside timing
    o = torch.empty((T, Hv, D), dtype=bf, device=dev)
    g.gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0, final_state=S, o=o,
                          workspace=ws)
    y_cal = g.gdn_gated_rmsnorm_silu(o, z, nw, out_dtype=f32)
    gx = float(448.0 * 6.0 / y_cal.abs().max().item())
    alpha = float(np.float32(1.0) / (np.float32(gx) * np.float32(gw)))
    del y_cal
    if not with_parts:
        del o

    def fused():
        g.gdn_prefill_chunked_gated_nvfp4(q, k, v, a, b, A_log, dt_bias, z, nw, gx, cu_seqlens=cu, initial_state=S0,
                                          final_state=S, xq=xq, xs=xs, workspace=ws)

    def gemm():
        g.nvfp4_gemm(xq, xs, wq, ws_w, alpha, y=Y)

    def step():
        fused()
        gemm()

    fns = [("step", step), ("fused", fused), ("gemm", gemm)]
    if with_parts:
        fns += [("scan", lambda: g.gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0,
                                                        final_state=S, o=o, workspace=ws)),
                ("tail", lambda: g.gdn_gated_rmsnorm_silu_nvfp4(o, z, nw, gx, xq=xq, xs=xs))]
    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    graphs = {}
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for name, fn in fns:
            fn()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=side):
                fn()
            graphs[name] = gr
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    res = {"w": w, "x": x, "graphs": graphs}
    if with_e2e:
        hq, hk, hv, hz = (t.cpu().pin_memory() for t in (q, k, v, z))
        ha, hb = a.cpu().pin_memory(), b.cpu().pin_memory()
        hY = [torch.empty((T, N), dtype=bf, pin_memory=True) for _ in range(2)]
        res["h2d"] = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hz, ha, hb))
        res["d2h"] = hY[0].numel() * hY[0].element_size()
        # two device sets of the inputs and of the output: step i uses set i % 2, so that its
        # compute overlaps the host -> device copies of step i + 1 and the device -> host copy of
        # step i - 1 (PCIe carries both directions at once); the workspace and the NVFP4
        # activations are used by the compute stream only and stay single
        ins = [(q, k, v, z, a, b), tuple(torch.empty_like(t) for t in (q, k, v, z, a, b))]
        outs = [Y, torch.empty_like(Y)]
        cs_in, cs_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_run(n):
            """n steps through the public API, every step copying its inputs in from pinned host
            memory and its output Y back; returns ms per step from the first copy in to the last
            copy out."""
            ready = [torch.cuda.Event() for _ in range(2)]
            done = [torch.cuda.Event() for _ in range(2)]
            drained = [torch.cuda.Event() for _ in range(2)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            cs_in.wait_stream(torch.cuda.current_stream())
            t0.record(cs_in)
            for i in range(n):
                j = i % 2
                dq, dk, dv, dz, da, db = ins[j]
                if i >= 2:
                    cs_in.wait_event(done[j])           # step i - 2 has consumed this input set
                with torch.cuda.stream(cs_in):
                    for dst, src in ((dq, hq), (dk, hk), (dv, hv), (dz, hz), (da, ha), (db, hb)):
                        dst.copy_(src, non_blocking=True)
                    ready[j].record(cs_in)
                side.wait_event(ready[j])
                if i >= 2:
                    side.wait_event(drained[j])         # step i - 2's output has reached the host
                with torch.cuda.stream(side):
                    g.gdn_prefill_chunked_gated_nvfp4(dq, dk, dv, da, db, A_log, dt_bias, dz, nw, gx, cu_seqlens=cu,
                                                      initial_state=S0, final_state=S, xq=xq, xs=xs, workspace=ws)
                    g.nvfp4_gemm(xq, xs, wq, ws_w, alpha, y=outs[j])
                    done[j].record(side)
                cs_out.wait_event(done[j])
                with torch.cuda.stream(cs_out):
                    hY[j].copy_(outs[j], non_blocking=True)
                    drained[j].record(cs_out)
            t1.record(cs_out)
            t1.synchronize()
            torch.cuda.current_stream().wait_stream(cs_out)
            return t0.elapsed_time(t1) / n
        res["e2e_run"] = e2e_run
    res["keep"] = (q, k, v, z, a, b, A_log, dt_bias, nw, cu, S0, wq, ws_w, S, xq, xs, Y, ws)
    return res


def timed_graph(torch, stream, flush, gr, n):
    """Mean device time (ms) of n replays, the L2 flushed before each (outside the events)."""
    out = []
    for _ in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gr.replay()
        e1.record(stream)
        out.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def prefill_summary(w, step_ms, fused_ms, gemm_ms, pk, pk_kind):
    fl = scan_flops(w)
    t = statistics.mean(fused_ms) / 1e3
    return {"workload": w.name, "tokens": w.T, "tokens/s": w.T / (statistics.mean(step_ms) / 1e3),
            "ms_per_step": statistics.mean(step_ms), "prefill_fused_ms": statistics.mean(fused_ms),
            "nvfp4_gemm_ms": statistics.mean(gemm_ms),
            "prefill_TFLOP/s": fl / t / 1e12, "prefill_tensor_frac": fl / t / 1e12 / float(pk["bf16_tflops"]),
            "prefill_hbm_frac": fused_bytes(w) / t / 1e9 / float(pk["hbm_gbs"]),
            "gemm_frac_of_fp4_probe": 2.0 * w.T * w.K * w.n_out / (statistics.mean(gemm_ms) / 1e3) / 1e12
            / FP4_PROBE_TFLOPS, "peak_kind": pk_kind}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import gated_deltanet_03_b200 as g

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    bf, f32 = torch.bfloat16, torch.float32

    def up(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)

    flush = make_l2_flush(torch, dev)
    side = torch.cuda.Stream()
    pk, pk_kind = peaks()

    # headline: the 27B-class long prefill (T = 32768, 16/32 heads, out_proj 4096 -> 2048)
    w = workloads.PREFILL_LONG
    main = prefill_case(torch, g, w, args, dev, flush, side, with_e2e=True)
    graphs = main["graphs"]
    T, Hv, D, K, N = w.T, w.Hv, w.D, w.K, w.n_out
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms = timed_graph(torch, stream, flush, graphs["step"], args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    fused_ms = timed_graph(torch, stream, flush, graphs["fused"], args.steps)
    gemm_ms = timed_graph(torch, stream, flush, graphs["gemm"], args.steps)
    launches_per_step, kernel_names = count_kernels(torch, graphs["step"].replay)
    ms = statistics.mean(step_ms)
    ms_max = ms
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    assert g.gdn_get_device_status() == 0
    e2e_run = main["e2e_run"]
    e2e_run(args.warmup)
    torch.cuda.synchronize()
    e2e = e2e_run(args.steps)
    if world > 1:
        t = torch.tensor([e2e], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e = float(t.item())
    h2d, d2h, x_main = main["h2d"], main["d2h"], main["x"]
    del main, graphs, e2e_run
    torch.cuda.empty_cache()

    # the 1024-wide layer's prefill (T = 4096, 16/16 heads) and the variable-length batch
    subs = {}
    for name, wl, parts_too in (("prefill_1024_wide", workloads.PREFILL_1K, True), ("varlen", workloads.VARLEN_8, False)):
        r = prefill_case(torch, g, wl, args, dev, flush, side, with_parts=parts_too)
        n_rep = max(args.steps, 10)
        st_ms = timed_graph(torch, stream, flush, r["graphs"]["step"], n_rep)
        fu_ms = timed_graph(torch, stream, flush, r["graphs"]["fused"], n_rep)
        ge_ms = timed_graph(torch, stream, flush, r["graphs"]["gemm"], n_rep)
        subs[name] = prefill_summary(wl, st_ms, fu_ms, ge_ms, pk, pk_kind)
        if parts_too:
            subs[name]["scan_alone_ms"] = statistics.mean(timed_graph(torch, stream, flush, r["graphs"]["scan"], n_rep))
            subs[name]["gated_norm_nvfp4_alone_ms"] = statistics.mean(
                timed_graph(torch, stream, flush, r["graphs"]["tail"], n_rep))
        assert g.gdn_get_device_status() == 0
        del r
        torch.cuda.empty_cache()

    # the causal short convolution in front of the 1024-wide layer's scan (q|k|v channels,
    # K = 4), timed alone: not part of the step, whose inputs are the scan's
    cw = workloads.PREFILL_1K
    conv_C = 2 * cw.Hk * cw.D + cw.Hv * cw.D
    cx = workloads.conv_inputs(cw.T, conv_C, 4, seed=cw.seed)
    conv_x, conv_w = up(cx["x"], bf), up(cx["weight"], f32)
    conv_y = torch.empty((cw.T * conv_C,), dtype=bf, device=dev)
    conv_parts = (cw.Hk * cw.D, cw.Hk * cw.D, cw.Hv * cw.D)

    def graph_of(fn):
        # device time of one launch, without the host's launch gap between the events
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=side):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        return gr

    conv_graph = graph_of(lambda: g.gdn_short_conv1d_silu(conv_x, conv_w, parts=conv_parts, y=conv_y))
    conv_ms = timed_graph(torch, stream, flush, conv_graph, max(args.steps, 10))
    del conv_graph

    # decode step on the batched-decode workload (L2 flushed before each replay, as for every op)
    dw = workloads.DECODE_B256
    dx = workloads.generate(dw)
    dq, dk, dv = up(dx["q"], bf), up(dx["k"], bf), up(dx["v"], bf)
    da, db = up(dx["a"], f32), up(dx["b"], f32)
    dA, ddt = up(dx["A_log"], f32), up(dx["dt_bias"], f32)
    dstate = up(dx["initial_state"], f32)
    dout = torch.empty((dw.num_seqs, dw.Hv, dw.D), dtype=bf, device=dev)

    dec_graph = graph_of(lambda: g.gdn_decode_step(dq, dk, dv, da, db, dA, ddt, dstate, o=dout))
    for _ in range(max(3, args.warmup)):
        dec_graph.replay()
    torch.cuda.synchronize()
    dec_ms = timed_graph(torch, stream, flush, dec_graph, max(args.steps, 10))
    dec = statistics.mean(dec_ms)
    state_bytes = dstate.numel() * 4
    dec_bytes = 2 * state_bytes + sum(t.numel() * t.element_size() for t in (dq, dk, dv, da, db, dout))
    # the decode step with the gated tail and the NVFP4 encode: fused kernel against the two calls
    dz, dnw = up(dx["z"], bf), up(dx["norm_weight"], f32)
    dxq = torch.empty((dw.num_seqs, dw.Hv * dw.D // 2), dtype=torch.uint8, device=dev)
    dxs = torch.empty((dw.num_seqs, dw.Hv * dw.D // 16), dtype=torch.uint8, device=dev)
    dgs = 448.0 * 6.0 / 4.0
    fdec_graph = graph_of(lambda: g.gdn_decode_step_gated_nvfp4(dq, dk, dv, da, db, dA, ddt, dstate, dz, dnw, dgs,
                                                                xq=dxq, xs=dxs))

    def two_call():
        g.gdn_decode_step(dq, dk, dv, da, db, dA, ddt, dstate, o=dout)
        g.gdn_gated_rmsnorm_silu_nvfp4(dout, dz, dnw, dgs, xq=dxq, xs=dxs)
    tdec_graph = graph_of(two_call)
    fdec = statistics.mean(timed_graph(torch, stream, flush, fdec_graph, max(args.steps, 10)))
    tdec = statistics.mean(timed_graph(torch, stream, flush, tdec_graph, max(args.steps, 10)))
    del fdec_graph, tdec_graph

    # multi-token decode on the batched-decode workload's shape: verify 4 draft tokens per sequence
    # (state read once), then commit a seeded number of accepted tokens (state read and written once)
    mT = 4
    mw = workloads.custom("verify_B%d_T%d" % (dw.num_seqs, mT), (mT,) * dw.num_seqs, dw.Hk, dw.Hv, dw.D,
                          s0_std=0.1, seed=dw.seed)
    mx = workloads.generate(mw)
    mB = dw.num_seqs
    mq = up(mx["q"], bf).view(mB, mT, dw.Hk, dw.D)
    mk = up(mx["k"], bf).view(mB, mT, dw.Hk, dw.D)
    mv = up(mx["v"], bf).view(mB, mT, dw.Hv, dw.D)
    ma, mb = up(mx["a"], f32).view(mB, mT, dw.Hv), up(mx["b"], f32).view(mB, mT, dw.Hv)
    mA, mdt = up(mx["A_log"], f32), up(mx["dt_bias"], f32)
    mstate = up(mx["initial_state"], f32)
    mo = torch.empty((mB, mT, dw.Hv, dw.D), dtype=bf, device=dev)
    macc = torch.from_numpy(np.random.default_rng(dw.seed).integers(0, mT + 1, size=mB).astype(np.int32)).to(dev)
    ver_graph = graph_of(lambda: g.gdn_decode_verify(mq, mk, mv, ma, mb, mA, mdt, mstate, o=mo))
    com_graph = graph_of(lambda: g.gdn_decode_commit(mq, mk, mv, ma, mb, mA, mdt, mstate, macc))
    for _ in range(max(3, args.warmup)):
        ver_graph.replay()
        com_graph.replay()
    torch.cuda.synchronize()
    ver_ms = statistics.mean(timed_graph(torch, stream, flush, ver_graph, max(args.steps, 10)))
    com_ms = statistics.mean(timed_graph(torch, stream, flush, com_graph, max(args.steps, 10)))
    m_tok = sum(t.numel() * t.element_size() for t in (mq, mk, mv, ma, mb))
    ver_bytes = mstate.numel() * 4 + m_tok + mo.numel() * mo.element_size()
    com_bytes = 2 * mstate.numel() * 4 + m_tok
    assert g.gdn_get_device_status() == 0
    del mstate

    # the NVFP4 GEMM at the long-prefill layer's output projection (32768 x 2048 x 4096)
    gM, gN, gK = 32768, 2048, 4096
    ga = g.nvfp4_quantize_act(up(workloads.activations(gM, gK, seed=5, heavy_tail=False), bf), 448.0 * 6.0 / 6.0)
    gw = g.nvfp4_quantize_act(up(workloads.activations(gN, gK, seed=6, heavy_tail=False), bf), 448.0 * 6.0 / 6.0)
    gy = torch.empty((gM, gN), dtype=bf, device=dev)
    big_graph = graph_of(lambda: g.nvfp4_gemm(ga[0], ga[1], gw[0], gw[1], 1.0, y=gy))
    for _ in range(3):
        big_graph.replay()
    big_ms = statistics.mean(timed_graph(torch, stream, flush, big_graph, max(args.steps, 10)))
    del ga, gw, gy, big_graph

    # the Q4_K-weight output projection of the same layer (the tail page's comparison format)
    q4w = up(workloads.q4k_weights(gN, gK, seed=7), torch.uint8)
    q4_ms = {}
    for qm in (gM, dw.num_seqs):
        q4a = up(workloads.activations(qm, gK, seed=8, heavy_tail=False), bf)
        q4y = torch.empty((qm, gN), dtype=bf, device=dev)
        q4_graph = graph_of(lambda: g.q4k_gemm(q4a, q4w, y=q4y))
        q4_ms[qm] = statistics.mean(timed_graph(torch, stream, flush, q4_graph, max(args.steps, 10)))
        del q4a, q4y, q4_graph
    del q4w
    assert g.gdn_get_device_status() == 0

    # short convolution decode on the batched-decode workload's q|k|v channels (state in place)
    dC = 2 * dw.Hk * dw.D + dw.Hv * dw.D
    dcx = workloads.conv_inputs(dw.num_seqs, dC, 4, seed=dw.seed, num_seqs=dw.num_seqs, state=True)
    dconv_x, dconv_w = up(dcx["x"], bf), up(dcx["weight"], f32)
    dconv_s = up(dcx["initial_state"], bf)
    dconv_y = torch.empty((dw.num_seqs * dC,), dtype=bf, device=dev)
    dparts = (dw.Hk * dw.D, dw.Hk * dw.D, dw.Hv * dw.D)
    cdec_graph = graph_of(lambda: g.gdn_short_conv1d_silu_decode(dconv_x, dconv_w, dconv_s, parts=dparts,
                                                                  y=dconv_y))
    for _ in range(max(3, args.warmup)):
        cdec_graph.replay()
    torch.cuda.synchronize()
    cdec = statistics.mean(timed_graph(torch, stream, flush, cdec_graph, max(args.steps, 10)))
    cdec_bytes = 2 * dconv_x.numel() * 2 + 2 * dconv_s.numel() * 2 + dconv_w.numel() * 4
    assert g.gdn_get_device_status() == 0

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    conv_bytes = 2 * cw.T * conv_C * 2 + conv_w.numel() * 4     # x read once, y written once, weights
    conv_mean = statistics.mean(conv_ms)
    scan_s = statistics.mean(fused_ms) / 1e3
    fl = scan_flops(w)
    achieved_tflops = fl / scan_s / 1e12
    peak_tflops = float(pk["bf16_tflops"])
    tokens = T * world
    out = {
        "metric": METRIC,
        "value": tokens / (ms_max / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the pages' 27B-class hybrid layer: 32 x 128 -> 4096 -> 2048)",
        "config": {"workload": w.name, "T": T, "Hk": w.Hk, "Hv": Hv, "d": D, "chunk": CHUNK,
                   "out_proj": "NVFP4 W4A4 %d->%d" % (K, N), "global_batch": 1, "seq_len": T,
                   "parallelism": "replicas x%d" % world,
                   "l2": "flushed between timed steps (256 MiB write, then 256 MiB read)"},
        "breakdown_ms": {"prefill_fused": statistics.mean(fused_ms), "nvfp4_gemm": statistics.mean(gemm_ms),
                         "step": "prefill_fused (scan + gated RMSNorm + NVFP4 encode in the output pass) + nvfp4_gemm",
                         "timing": "CUDA graph replay per op, L2 flushed before each"},
        "roofline": {"kernel": "fused prefill (prep, lean, combine and output-pass kernels of one call)",
                     "bound": "tensor", "achieved": achieved_tflops,
                     "peak": peak_tflops, "unit": "TFLOP/s", "frac": achieved_tflops / peak_tflops,
                     "peak_kind": pk_kind + " (bf16 dense burst; the scan's MMAs are fp16 and bf16)",
                     "algorithmic_flops": fl, "algorithmic_bytes": fused_bytes(w),
                     "hbm_frac": fused_bytes(w) / scan_s / 1e9 / float(pk["hbm_gbs"]),
                     "traffic": SCAN_TRAFFIC.get(source_digest(os.path.join(
                         ROOT, "gated_deltanet_03_b200", "csrc", "chunked.cu"))),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum over the call's four kernels"},
        "e2e": {"value": tokens / (e2e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e,
                "how": "every step copies its inputs in from pinned host memory and its output back; "
                       "copies in, compute and copies out of consecutive steps on three streams "
                       "(double-buffered inputs and outputs), timed from the first copy in to the last "
                       "copy out; inputs larger than L2"},
        "decode": {"workload": dw.name, "ms": dec, "GB/s": dec_bytes / (dec / 1e3) / 1e9,
                   "frac": dec_bytes / (dec / 1e3) / 1e9 / float(pk["hbm_gbs"]),
                   "bytes": dec_bytes, "peak_gbs": float(pk["hbm_gbs"]), "peak_kind": pk_kind,
                   "timing": "CUDA graph replay, L2 flushed before each",
                   "with_gated_nvfp4_tail": {"fused_ms": fdec, "two_calls_ms": tdec,
                                             "what": "decode step + gated RMSNorm + NVFP4 encode: one fused kernel "
                                                     "against gdn_decode_step then gdn_gated_rmsnorm_silu_nvfp4"}},
        "gemm_long_prefill": {"shape": [gM, gN, gK], "ms": big_ms,
                              "TFLOP/s": 2.0 * gM * gN * gK / (big_ms / 1e3) / 1e12,
                              "frac_of_fp4_probe": 2.0 * gM * gN * gK / (big_ms / 1e3) / 1e12 / FP4_PROBE_TFLOPS,
                              "peak_kind": "FP4 tensor rate measured by a tcgen05 probe (16368 MAC/cycle/SM at 1965 MHz)"},
        "q4k_out_proj": {"shape_prefill": [gM, gN, gK], "ms_prefill": q4_ms[gM],
                         "TFLOP/s_prefill": 2.0 * gM * gN * gK / (q4_ms[gM] / 1e3) / 1e12,
                         "tensor_frac_prefill": 2.0 * gM * gN * gK / (q4_ms[gM] / 1e3) / 1e12 / float(pk["bf16_tflops"]),
                         "shape_decode": [dw.num_seqs, gN, gK], "ms_decode": q4_ms[dw.num_seqs],
                         "weight_GB/s_decode": gN * (gK // 256) * 144 / (q4_ms[dw.num_seqs] / 1e3) / 1e9,
                         "what": "Q4_K weights decoded to bf16 in the kernel, bf16 tensor-core MMA"},
        "decode_multi": {"workload": "%s shape, %d draft tokens per sequence" % (dw.name, mT),
                         "verify_ms": ver_ms, "verify_GB/s": ver_bytes / (ver_ms / 1e3) / 1e9,
                         "verify_frac": ver_bytes / (ver_ms / 1e3) / 1e9 / float(pk["hbm_gbs"]),
                         "commit_ms": com_ms, "commit_GB/s": com_bytes / (com_ms / 1e3) / 1e9,
                         "commit_frac": com_bytes / (com_ms / 1e3) / 1e9 / float(pk["hbm_gbs"]),
                         "bytes": {"verify": ver_bytes, "commit": com_bytes},
                         "single_steps_ms": mT * dec,
                         "timing": "CUDA graph replay, L2 flushed before each; commit of a seeded 0..4 accepted tokens"},
        "prefill_1024_wide": subs["prefill_1024_wide"],
        "varlen": subs["varlen"],
        "short_conv": {"workload": "%s q|k|v channels (T = %d, C = %d, K = 4), planes q, k, v" % (cw.name, cw.T, conv_C),
                       "ms": conv_mean,
                       "GB/s": conv_bytes / (conv_mean / 1e3) / 1e9,
                       "frac": conv_bytes / (conv_mean / 1e3) / 1e9 / float(pk["hbm_gbs"]),
                       "bytes": conv_bytes, "bound": "hbm", "peak_kind": pk_kind,
                       "decode": {"workload": "%s q|k|v channels (B = %d, C = %d, K = 4)" % (dw.name, dw.num_seqs, dC),
                                  "ms": cdec, "bytes": cdec_bytes,
                                  "GB/s": cdec_bytes / (cdec / 1e3) / 1e9}},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_kernels_per_step": kernel_names,
        "clocks": clk.summary(),
    }
    if not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(w, x_main)
    print(json.dumps(out))


def run_only(args):
    """One kernel alone, `warmup` + `steps` launches, CUDA-event timed (L2 flushed between)."""
    import torch

    import gated_deltanet_03_b200 as g
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    bf, f32 = torch.bfloat16, torch.float32
    if args.only == "gemm_long":
        return run_gemm_long(args)
    if args.only == "verify":
        return run_verify(args)
    names = {wl.name: wl for wl in workloads.WORKLOADS}
    w = names[args.workload] if args.workload else (workloads.DECODE_B256 if args.only in ("decode", "decode_fused",
                                                                                            "conv_decode")
                                                    else workloads.PREFILL_1K)
    x = workloads.generate(w)

    def up(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)

    q, k, v, z = up(x["q"], bf), up(x["k"], bf), up(x["v"], bf), up(x["z"], bf)
    a, b = up(x["a"], f32), up(x["b"], f32)
    A_log, dt_bias, nw = up(x["A_log"], f32), up(x["dt_bias"], f32), up(x["norm_weight"], f32)
    cu = up(x["cu_seqlens"], torch.int32) if w.num_seqs > 1 else None
    S0 = None if x["initial_state"] is None else up(x["initial_state"], f32)
    o = torch.empty((w.T, w.Hv, w.D), dtype=bf, device=dev)
    S = torch.empty((w.num_seqs, w.Hv, w.D, w.D), dtype=f32, device=dev)
    W = up(x["proj_weight"], bf)
    wq, ws = g.nvfp4_quantize_act(W, 1.0)
    xq = torch.empty((w.T, w.K // 2), dtype=torch.uint8, device=dev)
    xs = torch.empty((w.T, w.K // 16), dtype=torch.uint8, device=dev)
    Y = torch.empty((w.T, w.n_out), dtype=bf, device=dev)
    g.gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0, final_state=S, o=o)
    g.gdn_gated_rmsnorm_silu_nvfp4(o, z, nw, 1.0, xq=xq, xs=xs)
    conv_C = 2 * w.Hk * w.D + w.Hv * w.D
    cx = workloads.conv_inputs(w.T, conv_C, 4, seed=w.seed)
    conv_x, conv_w = up(cx["x"], bf), up(cx["weight"], f32)
    conv_y = torch.empty((w.T * conv_C,), dtype=bf, device=dev)
    dcx = workloads.conv_inputs(w.num_seqs, conv_C, 4, seed=w.seed, num_seqs=w.num_seqs, state=True)
    dconv_x, dconv_s = up(dcx["x"], bf), up(dcx["initial_state"], bf)
    if args.only == "q4k":
        q4a = up(workloads.round_bf16(np.random.default_rng(3).standard_normal((w.T, w.K)).astype(np.float32)), bf)
        q4w = up(workloads.q4k_weights(w.n_out, w.K, seed=7), torch.uint8)
        q4y = torch.empty((w.T, w.n_out), dtype=bf, device=dev)
    fn = {
        "conv_decode": lambda: g.gdn_short_conv1d_silu_decode(dconv_x, conv_w, dconv_s,
                                                              parts=(w.Hk * w.D, w.Hk * w.D, w.Hv * w.D)),
        "conv": lambda: g.gdn_short_conv1d_silu(conv_x, conv_w, parts=(w.Hk * w.D, w.Hk * w.D, w.Hv * w.D),
                                                y=conv_y),
        "scan": lambda: g.gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0,
                                              final_state=S, o=o),
        "tail": lambda: g.gdn_gated_rmsnorm_silu_nvfp4(o, z, nw, 1.0, xq=xq, xs=xs),
        "gemm": lambda: g.nvfp4_gemm(xq, xs, wq, ws, 1.0, y=Y),
        "q4k": lambda: g.q4k_gemm(q4a, q4w, y=q4y),
        "decode": lambda: g.gdn_decode_step(q, k, v, a, b, A_log, dt_bias, S0, o=o),
        "decode_fused": lambda: g.gdn_decode_step_gated_nvfp4(q, k, v, a, b, A_log, dt_bias, S0, z, nw, 1.0,
                                                              xq=xq, xs=xs),
        "fused": lambda: g.gdn_prefill_chunked_gated_nvfp4(q, k, v, a, b, A_log, dt_bias, z, nw, 1.0, cu_seqlens=cu,
                                                           initial_state=S0, final_state=S, xq=xq, xs=xs),
    }[args.only]
    flush = make_l2_flush(torch, dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    assert g.gdn_get_device_status() == 0
    print(json.dumps({"only": args.only, "workload": w.name, "ms_median": statistics.median(times),
                      "ms_mean": statistics.mean(times), "steps": args.steps}))


def run_gemm_long(args):
    """The NVFP4 GEMM alone at the long-prefill layer's output projection (32768 x 2048 x 4096),
    `warmup` + `steps` launches, CUDA-event timed with the L2 flushed between them."""
    import torch

    import gated_deltanet_03_b200 as g
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    gM, gN, gK = 32768, 2048, 4096

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, torch.bfloat16)

    xa = g.nvfp4_quantize_act(up(workloads.activations(gM, gK, seed=5, heavy_tail=False)), 448.0)
    xw = g.nvfp4_quantize_act(up(workloads.activations(gN, gK, seed=6, heavy_tail=False)), 448.0)
    y = torch.empty((gM, gN), dtype=torch.bfloat16, device=dev)
    flush = make_l2_flush(torch, dev)
    for _ in range(args.warmup):
        g.nvfp4_gemm(xa[0], xa[1], xw[0], xw[1], 1.0, y=y)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.nvfp4_gemm(xa[0], xa[1], xw[0], xw[1], 1.0, y=y)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    assert g.gdn_get_device_status() == 0
    ms = statistics.median(times)
    print(json.dumps({"only": "gemm_long", "shape": [gM, gN, gK], "ms_median": ms,
                      "TFLOP/s": 2.0 * gM * gN * gK / (ms / 1e3) / 1e12, "steps": args.steps}))


def run_verify(args):
    """Draft verify alone on the batched-decode shape (256 sequences x 4 draft tokens, 16/32
    heads, d = 128, state read only), `warmup` + `steps` launches, L2 flushed between."""
    import torch

    import gated_deltanet_03_b200 as g
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dw, mT = workloads.DECODE_B256, 4
    mw = workloads.custom("verify_B%d_T%d" % (dw.num_seqs, mT), (mT,) * dw.num_seqs, dw.Hk, dw.Hv, dw.D,
                          s0_std=0.1, seed=dw.seed)
    mx = workloads.generate(mw)
    B, bf, f32 = dw.num_seqs, torch.bfloat16, torch.float32

    def up(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)

    q = up(mx["q"], bf).view(B, mT, dw.Hk, dw.D)
    k = up(mx["k"], bf).view(B, mT, dw.Hk, dw.D)
    v = up(mx["v"], bf).view(B, mT, dw.Hv, dw.D)
    a, b = up(mx["a"], f32).view(B, mT, dw.Hv), up(mx["b"], f32).view(B, mT, dw.Hv)
    A_log, dt_bias, state = up(mx["A_log"], f32), up(mx["dt_bias"], f32), up(mx["initial_state"], f32)
    o = torch.empty((B, mT, dw.Hv, dw.D), dtype=bf, device=dev)
    flush = make_l2_flush(torch, dev)
    for _ in range(args.warmup):
        g.gdn_decode_verify(q, k, v, a, b, A_log, dt_bias, state, o=o)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.gdn_decode_verify(q, k, v, a, b, A_log, dt_bias, state, o=o)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    assert g.gdn_get_device_status() == 0
    print(json.dumps({"only": "verify", "workload": mw.name, "ms_median": statistics.median(times),
                      "steps": args.steps}))


# ----------------------------------------------------------------- CPU arm ----

CPU_SAMPLE_TOKENS = 4096


def token_prefix(w, x, n):
    """The workload cut to its first n tokens (one sequence): the layer on a shorter input."""
    y = dict(x)
    for key in ("q", "k", "v", "z", "a", "b"):
        y[key] = x[key][:n]
    y["cu_seqlens"] = np.array([0, n], np.int32)
    return y


def cpu_pass(w, x, units=None):
    """The oracle over the same workload: scan (threaded over heads), gated tail, NVFP4
    encode and the fp64 GEMM over dequantised operands."""
    import oracle
    o, S = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                           cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"], units=units)
    y = oracle.gated_rmsnorm_silu(workloads.round_bf16(o.astype(np.float32)), x["z"], x["norm_weight"])
    gx = np.float32(448.0 * 6.0 / max(np.abs(y).max(), 1e-30))
    W = x["proj_weight"]
    gw = np.float32(448.0 * 6.0 / np.abs(W).max())
    xq, xs = oracle.nvfp4_quantize(workloads.round_bf16(y.astype(np.float32)), gx)
    wq, ws = oracle.nvfp4_quantize(W, gw)
    return oracle.nvfp4_gemm(xq, xs, gx, wq, ws, gw)


def cpu_baseline(w, x, min_seconds: float = 10.0):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload: whole
    passes of the layer (all heads, all rows) over its first CPU_SAMPLE_TOKENS tokens, repeated
    until about `min_seconds` of CPU work; tokens/s over all passes."""
    import oracle
    n = min(CPU_SAMPLE_TOKENS, w.T)
    xs = token_prefix(w, x, n) if w.num_seqs == 1 else x
    n = n if w.num_seqs == 1 else w.T
    passes = 0
    t0 = time.perf_counter()
    while True:
        cpu_pass(w, xs)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    return {"value": passes * n / dt, "unit": "tokens/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": "the layer (all %d heads, all rows) on the first %d of the %d tokens, %d passes"
                      % (w.Hv, n, w.T, passes), "seconds": dt}


REF_SAMPLE_TOKENS = 2048


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = workloads.PREFILL_LONG
    x = workloads.generate(w)
    n = REF_SAMPLE_TOKENS
    xs = token_prefix(w, x, n)
    for _ in range(args.warmup):
        cpu_pass(w, xs, units=[0])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cpu_pass(w, xs)
        times.append(time.perf_counter() - t0)
    dt = statistics.mean(times)
    val = n / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the pages' 27B-class hybrid layer: 32 x 128 -> 4096 -> 2048)",
        "config": {"workload": w.name, "T": w.T, "Hk": w.Hk, "Hv": w.Hv, "d": w.D},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.default_threads(), "kind": "oracle",
                         "sample": "each step: the layer (all heads, all rows) on the first %d of the %d tokens"
                                   % (n, w.T)},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    p.add_argument("--only", choices=["scan", "tail", "gemm", "gemm_long", "decode", "verify", "fused", "conv",
                                      "conv_decode", "q4k", "decode_fused"],
                   help="time one kernel alone on its workload (for profiling); prints one JSON line")
    p.add_argument("--workload", default=None, help="workload name for --only scan (default: 1024-wide prefill)")
    args = p.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_only(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
