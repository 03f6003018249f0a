"""Benchmark of the whole quantisation path on one layer per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1]

One step = the whole hot path over one seeded synthetic layer, q_proj-like by default (W bf16
[5120, 5120], X bf16 [8192 tokens, 5120] generated as 16 chunks of 512, group 128, damping
0.01 * mean(diag H)):
  H = X^T X (SYRK) -> imatrix -> damping + Cholesky chain -> GPTQ sweep (codes, scales, qerr)
  -> Bf16TrilDiagF32 encode of H -> decode.
Metric: GPTQ-int4 weights/s = N*K / step time (whole job, all ranks).  Inputs are resident in
HBM; L2 is flushed (a 256 MiB write) between timed steps.  `e2e` repeats the measurement through
the same C ABI calls with the inputs in pinned host memory: their H2D copies and the D2H copy of
the results (codes, scales, encoded H, qerr) are inside its timed region, overlapped with the
compute on two copy streams (the encoded H goes back while the factorisation runs).

Under torchrun every rank quantises its own independent layer (weak scaling, no collective in
the data path); times are the max over ranks.  `--impl reference` times the fp64 CPU oracle
on a bounded sample of the same workload instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wl  # noqa: E402

L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.path is None or not os.path.exists(self.path):
            return out
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        busy = [v for v in sm if v > 0]
        out.update(sm_mhz=statistics.median(busy) if busy else None, sm_max_mhz=max(mx) if mx else None,
                   reasons=sorted(reasons), samples=len(rows))
        return out


# ------------------------------------------------------------------------------------ our arm

class Layer:
    """Device buffers of one layer and the calls of one step, all through the C ABI binding."""

    def __init__(self, hq, cfg, device):
        self.hq = hq
        self.cfg = cfg
        self.dev = device
        N, K, G = cfg.N, cfg.K, cfg.group
        self.X = wl.make_activations(cfg, device)
        self.W = wl.make_weights(cfg, device)
        self.H = torch.zeros((K, K), dtype=torch.float32, device=device)
        self.imp = torch.empty(K, dtype=torch.float32, device=device)
        self.codes, self.scales = hq.gptq_outputs(N, K, G, device)
        self.ws = hq.alloc_workspace(hq.hq_gptq_workspace_bytes(N, K, G), device)
        self.tril = torch.empty(hq.hq_bf16tril_bytes(K), dtype=torch.uint8, device=device)
        self.Hfull = torch.empty((K, K), dtype=torch.float32, device=device)
        self.qerr = torch.zeros(1, dtype=torch.float64, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def step(self, X=None, W=None, stage_events=None):
        hq, cfg = self.hq, self.cfg
        X = self.X if X is None else X
        W = self.W if W is None else W
        ev = stage_events
        if ev is not None:
            ev[0].record()
        self.H.zero_()
        hq.hq_hessian_accumulate(self.H, X, dev_status=self.status)
        if ev is not None:
            ev[1].record()
        hq.hq_imatrix(self.H, cfg.T, self.imp)
        hq.hq_gptq_quantize(W, self.H, cfg.group, cfg.damp, self.codes, self.scales, self.ws,
                            imp=self.imp if cfg.use_imatrix else None, want_qerr=False, qerr_dev=self.qerr)
        if ev is not None:
            ev[2].record()
        hq.hq_hessian_pack_bf16tril(self.H, self.tril)
        if ev is not None:
            ev[3].record()
        hq.hq_hessian_unpack_bf16tril(self.tril, cfg.K, self.Hfull)
        if ev is not None:
            ev[4].record()


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (a device time: the job ends with its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, steps: int, total_ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own units each step (weak scaling), and
    the job takes as long as its slowest rank."""
    return units_per_rank * world * steps / (total_ms_max / 1e3)


def run_ours(args, rank, world, local_rank):
    import post_weight_quantization_tcgen05_b200 as hq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = wl.CONFIGS[args.config]
    layer = Layer(hq, cfg, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    for w in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    # the kernel class with the largest share of a step, from one step with every launch timed
    # (outside the timed region), net of the launch processing each launch's event pair holds;
    # its launches are then timed live, inside the timed region when they are few
    overhead_us = launch_overhead_us()
    dominant = dominant_class(kernel_breakdown(hq, layer, flush, steps=1, overhead_us=overhead_us))
    hq.hq_debug_timing_start([dominant])  # creates its events before the timed region
    layer.step()
    torch.cuda.synchronize()
    dom_lps = hq.hq_debug_timing_read(dominant)[2]  # launches in one step
    inline = dom_lps <= MAX_INLINE_TIMED_LAUNCHES

    # ---- timed region: K steps, each bracketed by events, L2 flushed between steps; the library
    #      records events around every launch of the dominant kernel on its own stream
    n_ev = 5
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    launches0 = hq.hq_debug_launch_count()
    _barrier(world)
    torch.cuda.synchronize()
    if inline:
        hq.hq_debug_timing_start([dominant])
    else:
        hq.hq_debug_timing_stop()
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            layer.step(stage_events=evs[k])
        torch.cuda.synchronize()
    hq.hq_debug_timing_stop()
    if inline:
        dom = (dominant,) + tuple(hq.hq_debug_timing_read(dominant))
    else:  # the same steps again, every launch of the dominant class timed
        hq.hq_debug_timing_start([dominant])
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            layer.step()
        torch.cuda.synchronize()
        hq.hq_debug_timing_stop()
        dom = (dominant,) + tuple(hq.hq_debug_timing_read(dominant))
    _barrier(world)
    launches = (hq.hq_debug_launch_count() - launches0) // max(args.steps, 1)
    step_ms = [e[0].elapsed_time(e[4]) for e in evs]
    syrk_ms = [e[0].elapsed_time(e[1]) for e in evs]
    gptq_ms = [e[1].elapsed_time(e[2]) for e in evs]
    enc_ms = [e[2].elapsed_time(e[3]) for e in evs]
    dec_ms = [e[3].elapsed_time(e[4]) for e in evs]
    total_ms = _max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    weights = cfg.N * cfg.K
    value = aggregate_rate(weights, world, args.steps, total_ms)

    # ---- e2e: same calls, inputs from pinned host memory, results copied back
    e2e = None if args.no_e2e else measure_e2e(args, layer, flush, world)
    # ---- per-kernel breakdown (outside the timed region: events around every launch)
    kernels = kernel_breakdown(hq, layer, flush, overhead_us=overhead_us)
    codec = codec_throughput(hq, layer, flush)
    peaks = _peaks()
    dense = measure_dense_peaks(hq, dev)
    peaks["tf32_tflops"] = dense.get("tf32_tflops") or peaks["bf16_tflops"] / 2.0
    peaks["fp64_tflops"] = dense.get("fp64_tflops")
    peaks["int8_tops"] = dense.get("int8_tops")
    syrk_flop = cfg.T * cfg.K * (cfg.K + 1)
    syrk_avg_s = statistics.mean(syrk_ms) / 1e3
    syrk_tflops = syrk_flop / syrk_avg_s / 1e12
    enc_bytes = 2 * cfg.K * (cfg.K + 1) + hq.hq_bf16tril_bytes(cfg.K)   # H lower triangle read + payload
    dec_bytes = hq.hq_bf16tril_bytes(cfg.K) + 4 * cfg.K * cfg.K
    clocks = clk.summary()
    return_line = build_line(args, cfg, world, value, ms_per_step, syrk_ms, gptq_ms, enc_ms, dec_ms, syrk_tflops,
                             enc_bytes, dec_bytes, peaks, e2e, launches, clocks, dom, kernels, dense,
                             inline, overhead_us)
    hbm = peaks["hbm_gbs"]
    return_line["codec_roofline"] = {
        "kernels": "tril_encode_pair_kernel / tril_decode_vec_kernel", "bound": "hbm", "unit": "GB/s",
        "encode": {"achieved": codec["encode_gbs"], "frac": codec["encode_gbs"] / hbm, "us": codec["encode_us"]},
        "decode": {"achieved": codec["decode_gbs"], "frac": codec["decode_gbs"] / hbm, "us": codec["decode_us"]},
        "peak": hbm, "peak_source": f"{peaks['source']} HBM copy",
        "bytes": codec["bytes"],
        "method": "each call alone after an L2 flush (write then read of 256 MiB), events around the call, the GPU rested 0.5 s first"}
    if world == 1 and not args.no_other_configs:
        return_line["hadamard_rotation"] = time_hadamard(hq, layer, flush, peaks)
        return_line["syrk_per_call"] = time_syrk_per_call(hq, layer, flush, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        return_line["cpu_baseline"] = cpu_baseline(cfg, layer)
    if world == 1 and not args.no_other_configs:
        del layer
        torch.cuda.empty_cache()
        return_line["other_configs"] = other_configs(hq, dev, flush, peaks)
    return return_line


def time_hadamard(hq, layer, flush, peaks, block: int = 256):
    """The rotate-then-GPTQ rotation on the layer: W' = W R (bf16 in, fp32 out) and H' = R^T H R
    (columns pass on the lower blocks, then rows pass with the transposed writes), each call timed
    alone after an L2 flush (median of 5); rates are the algorithmic bytes (W: 2 read + 4 written per weight; H: its
    lower triangle read once, K(K+1)/2 x 4, and H' written once, K^2 x 4) over the time, against
    the measured HBM copy rate.  The two-pass Hessian design moves about twice those bytes
    (`design_bytes`)."""
    from post_weight_quantization_tcgen05_b200 import quarot
    N, K = layer.W.shape
    g = torch.Generator(device=layer.W.device)
    g.manual_seed(42)
    s = quarot.random_signs(K, g, device=layer.W.device)
    Wr = torch.empty((N, K), dtype=torch.float32, device=layer.W.device)
    Hr = torch.empty((K, K), dtype=torch.float32, device=layer.W.device)
    out = {}
    for name, fn, nbytes in (("weights", lambda: hq.hq_hadamard_rotate_weights(layer.W, s, block, Wr), 6.0 * N * K),
                             ("hessian", lambda: hq.hq_hadamard_rotate_hessian(layer.H, s, block, Hr),
                              4.0 * K * (K + 1) / 2 + 4.0 * K * K)):
        fn()
        times = []
        for rep in range(5):  # each call after an L2 flush; the median
            flush.fill_(3 + rep)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms": ms, "achieved_gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
    del Wr, Hr
    nb = K // block
    lower = nb * (nb + 1) / 2 * block * block * 4.0
    out["hessian"]["design_bytes"] = 3 * lower + 4.0 * K * K  # pass 1 r+w lower blocks, pass 2 r lower, w all
    out.update({"kernels": "hadamard_rows_warp_kernel (W); hadamard_cols_lower_kernel + hadamard_rows_mirror_kernel (H)",
                "block": block,
                "bound": "hbm", "peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"] + " HBM copy"})
    return out


def time_layer(hq, cfg, dev, flush, steps: int = 2, warmup: int = 1, peaks=None):
    """Whole-path steps on one layer of `cfg` (the main measurement's protocol, fewer steps)."""
    layer = Layer(hq, cfg, dev)
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for k in range(steps):
        flush.fill_(k & 0xFF)
        layer.step(stage_events=evs[k])
    torch.cuda.synchronize()
    step_ms = statistics.mean(e[0].elapsed_time(e[4]) for e in evs)
    syrk_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    gptq_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    out = {"workload": f"{cfg.name}: W bf16 [{cfg.N}, {cfg.K}], X bf16 [{cfg.T}, {cfg.K}], group {cfg.group}"
                       + (", imatrix" if cfg.use_imatrix else ""),
           "steps": steps, "ms_per_step": step_ms, "weights_per_s": cfg.N * cfg.K / (step_ms / 1e3),
           "gptq_quantize_ms": gptq_ms, "gptq_weights_per_s": cfg.N * cfg.K / (gptq_ms / 1e3),
           "syrk_ms": syrk_ms, "xtx_tflops": cfg.T * cfg.K * (cfg.K + 1) / (syrk_ms / 1e3) / 1e12}
    if peaks is not None:  # kernel-level rooflines (one more step, every launch timed)
        kernels = kernel_breakdown(hq, layer, flush, steps=1)
        out["syrk_roofline"] = syrk_line(kernels, out["xtx_tflops"], peaks)
        out["update_roofline"] = update_line(cfg, kernels, peaks)
        out["kernels_ms"] = {k: v["ms_per_step"] for k, v in kernels.items()}
        out["rooflines"] = {k: class_roofline(k, v["ms_total"], v["work_total"], v["launches_total"], 1, peaks, cfg)
                            for k, v in kernels.items()}
    del layer
    torch.cuda.empty_cache()
    return out


def time_hessian_at_scale(hq, cfg, dev, flush, peaks, distinct: int = 8):
    """SYRK over the configuration's 512 chunks of 8192 tokens into one fp32 H (the chunks cycle
    through `distinct` pre-generated ones: the SYRK's cost does not depend on the values;
    generation is outside the timed region), then the codec of that H, each call alone."""
    import post_weight_quantization_tcgen05_b200 as hqm
    K = cfg.K
    scales = wl.channel_scales(cfg)
    chunks = [wl.make_activation_chunk(cfg, c, dev, scales) for c in range(distinct)]
    H = torch.zeros((K, K), dtype=torch.float32, device=dev)
    for c in range(distinct):  # warm-up
        hq.hq_hessian_accumulate(H, chunks[c])
    H.zero_()
    flush.fill_(1)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for c in range(cfg.n_chunks):
        hq.hq_hessian_accumulate(H, chunks[c % distinct])
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)

    class _L:  # what codec_throughput reads
        pass
    lay = _L()
    lay.cfg, lay.H = cfg, H
    lay.tril = torch.empty(hqm.hq_bf16tril_bytes(K), dtype=torch.uint8, device=dev)
    lay.Hfull = torch.empty((K, K), dtype=torch.float32, device=dev)
    burst = codec_throughput(hq, lay, flush, rest_s=0.0)  # right after the SYRK's power-capped burst
    codec = codec_throughput(hq, lay, flush)
    hbm = peaks["hbm_gbs"]
    psd = time_psd_projection(hq, lay.Hfull, peaks)  # the decoded (stored) H, as a reader gets it
    out = {"workload": f"{cfg.name}: {cfg.n_chunks} chunks of X bf16 [{cfg.chunk}, {K}] into one H",
           "syrk_ms": ms, "xtx_tflops": cfg.T * K * (K + 1) / (ms / 1e3) / 1e12,
           "xtx_frac_of_bf16_peak": cfg.T * K * (K + 1) / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
           "codec": {"encode_gbs": codec["encode_gbs"], "encode_frac": codec["encode_gbs"] / hbm,
                     "decode_gbs": codec["decode_gbs"], "decode_frac": codec["decode_gbs"] / hbm,
                     "method": "each call alone after an L2 flush, the GPU rested 0.5 s first",
                     "right_after_syrk_burst": {"encode_frac": burst["encode_gbs"] / hbm,
                                                "decode_frac": burst["decode_gbs"] / hbm}},
           "psd_projection": psd}
    del chunks, H, lay
    torch.cuda.empty_cache()
    return out


def time_psd_projection(hq, Hstored, peaks, steps: int = 40):
    """hq_hessian_project_psd on a copy of a decoded Hessian (one untimed call first): its time
    and its rate against the tensor roofline of its products (three tf32 MMAs per product at the
    tf32 rate measured in this run; half the bf16 burst, NVIDIA's nominal dense ratio, when there
    is none)."""
    K = Hstored.shape[0]
    ws = hq.alloc_workspace(hq.hq_psd_workspace_bytes(K), Hstored.device)
    P = Hstored.clone()
    hq.hq_hessian_project_psd(P, ws, steps=steps)
    P.copy_(Hstored)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    hq.hq_hessian_project_psd(P, ws, steps=steps)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    flops = 4.0 * (steps + 0.5) * float(K) ** 3
    useful = flops / (ms / 1e3) / 1e12
    tf32 = peaks.get("tf32_tflops")
    peak = (tf32 if tf32 else peaks["bf16_tflops"] / 2.0) / 3.0
    moved = float(torch.linalg.norm(P - Hstored) / torch.linalg.norm(Hstored))
    del ws, P
    return {"kernels": "upd_gemm_kernel<BN> (3xTF32 Newton-Schulz products) + elementwise", "K": K,
            "steps": steps, "ms": ms, "achieved_useful_tflops": useful, "peak_useful_tflops": peak,
            "frac": useful / peak, "relative_change": moved,
            "peak_source": ("tf32 dense rate measured in this run" if tf32 else
                            peaks["source"] + " bf16 dense burst / 2 (nominal tf32 ratio)") + " / 3 MMAs per product"}


def other_configs(hq, dev, flush, peaks):
    """The other single-GPU layer configurations (gate_up, down_proj at K = 17408, the Hessian at
    scale), measured after the main line's timed region."""
    out = {}
    for idx in (2, 3):
        cfg = wl.CONFIGS[idx]
        out[cfg.name] = time_layer(hq, cfg, dev, flush, peaks=peaks)
    out["hessian_at_scale"] = time_hessian_at_scale(hq, wl.CONFIGS[4], dev, flush, peaks)
    return out


# Kernel classes the library times (hq_debug_timing_*), with the unit of their algorithmic work.
KERNEL_NAMES = {"f64_gemm_128": ("f64_gemm_kernel<128>", "TFLOP/s"),
                "f64_gemm_64": ("f64_gemm_kernel<64>, <32> (+ split-K reduce)", "TFLOP/s"),
                "i8x_gemm": ("i8x_gemm_kernel (fp64 products from int8 slices on tcgen05 kind::i8)", "TFLOP/s"),
                "i8x_slice": ("i8x_slice_kernel (fp64 operands cut into int8 slices)", "GB/s"),
                "leaf": ("chol_inv_leaf_kernel", "TFLOP/s"),
                "sweep": ("sweep_block_kernel", "GB/s"),
                "tf32_gemm": ("upd_gemm_kernel<BN> (3xTF32 lazy updates)", "TFLOP/s"),
                "syrk": ("syrk_tc_kernel (persistent tcgen05 SYRK)", "TFLOP/s")}
# int8 slice-pair products per fp64 product in the int8-sliced GEMM (7 slices, anti-diagonals 0-6)
I8X_PAIRS = 28
# fp64 tensor-core peak when no fp64 rate was measured: the measured bf16 burst scaled by NVIDIA's
# nominal dense ratio for B200 (fp64 tensor 37 TFLOP/s : bf16 2250 TFLOP/s)
FP64_OVER_BF16 = 37.0 / 2250.0
# committed ncu summaries (DRAM traffic per launch) and the source each was taken from
PROFILES = {"f64_gemm_64": ("f64_gemm_kernel_32_q_proj.md", "gemm_f64.cu"),
            "i8x_gemm": ("i8x_gemm_kernel_q_proj.md", "gemm_i8x.cu"),
            "leaf": ("chol_inv_leaf_kernel_q_proj.md", "factor.cu"),
            "sweep": ("sweep_block_kernel_q_proj.md", "gptq.cu"),
            "tf32_gemm": ("upd_gemm_kernel_q_proj.md", "gemm_upd.cu"),
            "syrk": ("syrk_tc_kernel_q_proj.md", "syrk.cu")}


def dominant_class(kernels) -> str:
    """The timed kernel class with the most device time per step (net of launch processing where
    the breakdown has it)."""
    if not kernels:
        return "f64_gemm_64"
    return max(kernels, key=lambda c: kernels[c].get("ms_net_per_step", kernels[c]["ms_per_step"]))


# A dominant class with more launches per step than this is timed in a second pass of the same
# steps: an event pair around each of its launches would break the chained launches of the
# factorisation and slow the headline steps down.
MAX_INLINE_TIMED_LAUNCHES = 16


def class_roofline(cls: str, ms: float, work: float, launches: int, steps: int, peaks, cfg) -> dict:
    """Roofline of one kernel class from its summed launch time `ms` and algorithmic `work`
    (the library's per-launch figure) over `steps` steps: the bound, achieved rate, peak and
    fraction, in the unit of the bound."""
    s = ms / 1e3
    out = {"kernel": KERNEL_NAMES[cls][0], "class": cls, "launches_per_step": launches / max(steps, 1),
           "ms_per_step": ms / max(steps, 1)}
    fp64 = peaks.get("fp64_tflops") or peaks["bf16_tflops"] * FP64_OVER_BF16
    if cls in ("f64_gemm_128", "f64_gemm_64", "leaf"):
        out.update(bound="tensor", unit="TFLOP/s", achieved=work / s / 1e12 if s > 0 else None, peak=fp64,
                   peak_source="fp64 dense rate measured in this run: the larger of the fp64 torch.matmul (cuBLAS) "
                               "rate and the library's fp64 MMA rate")
    elif cls == "i8x_gemm":
        out.update(bound="tensor", unit="TOP/s", achieved=I8X_PAIRS * work / s / 1e12 if s > 0 else None,
                   peak=peaks.get("int8_tops"), fp64_equivalent_tflops=work / s / 1e12 if s > 0 else None,
                   peak_source="int8 dense rate measured in this run (torch._int_mm); work = 28 exact int8 "
                               "slice-pair products per fp64 multiply-add pair (2 ops each)")
    elif cls in ("sweep", "i8x_slice"):
        out.update(bound="hbm", unit="GB/s", achieved=work / s / 1e9 if s > 0 else None, peak=peaks["hbm_gbs"],
                   peak_source=peaks["source"] + " HBM copy")
    elif cls == "syrk":
        out.update(bound="tensor", unit="TFLOP/s", achieved=work / s / 1e12 if s > 0 else None,
                   peak=peaks["bf16_tflops"], peak_source=peaks["source"] + " bf16 dense burst")
    elif cls == "tf32_gemm":
        roof = update_roofline_ms(cfg, peaks) * max(steps, 1)
        out.update(bound="tensor / hbm per launch", unit="ms", achieved=roof, peak=ms,
                   peak_source="per-launch roofline time (tf32 measured in this run, HBM copy) against the measured "
                               "time: frac = roofline / measured")
    a, p = out.get("achieved"), out.get("peak")
    out["frac"] = (a / p) if (a is not None and p) else None
    return out


def profiled_traffic(cls: str):
    """DRAM bytes per launch of kernel class `cls` from its committed ncu summary, or None when
    there is none or the kernel's source has changed since that capture."""
    import hashlib
    if cls not in PROFILES:
        return None
    summary = os.path.join(ROOT, "profiles", PROFILES[cls][0])
    source = os.path.join(ROOT, "post_weight_quantization_tcgen05_b200", "csrc", PROFILES[cls][1])
    if not os.path.exists(summary):
        return None
    with open(source, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    vals = {}
    with open(summary) as f:
        for line in f:
            if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "source_sha256")):
                k, v = line.strip().split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256") != sha or "traffic_bytes_per_launch" not in vals:
        return None
    return float(vals["traffic_bytes_per_launch"])


def update_roofline_ms(cfg, peaks, tf32_tflops=None) -> float:
    """Sum over the sweep's lazy-update launches of each launch's roofline time: the larger of
    its tensor time (three tf32 MMAs per product at the measured tf32 rate) and its DRAM time at
    the measured HBM rate (C read and written, the split residuals and the split U' block read
    once, 4 bytes each)."""
    N, K = cfg.N, cfg.K
    P = min(512 if cfg.group <= 128 else cfg.group * max(512 // cfg.group, 1), K)
    tf32 = (tf32_tflops or peaks["tf32_tflops"]) * 1e12
    hbm = peaks["hbm_gbs"] * 1e9
    launches = []
    for p0 in range(0, K, P):
        p1 = min(p0 + P, K)
        for j0 in range(p0, p1, 128):
            if j0 + 128 < p1:
                launches.append((p1 - j0 - 128, 128))
        if p1 < K:
            launches.append((K - p1, p1 - p0))
    total = 0.0
    for ncols, kred in launches:
        flops = 3 * 2.0 * N * ncols * kred
        nbytes = 8.0 * N * ncols + 8.0 * N * kred + 8.0 * ncols * kred
        total += max(flops / tf32, nbytes / hbm)
    return total * 1e3


def launch_overhead_us(reps: int = 50) -> float:
    """Median time of an event pair around an empty kernel launched right behind a busy one on
    the same stream (µs): the GPU's processing of a launch, which every per-launch event pair of
    the breakdown also holds.  (In the step itself the chained launches overlap it with their
    predecessor.)"""
    pairs = []
    for _ in range(reps):
        torch.cuda._sleep(200000)  # keeps the GPU busy until the host has queued the pair
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        torch.cuda._sleep(0)
        b.record()
        pairs.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in pairs) * 1e3


def kernel_breakdown(hq, layer, flush, steps: int = 2, overhead_us: float | None = None):
    """Per kernel class: device time and achieved rate over `steps` steps, every launch timed.
    The factorisation's second stream is folded into the caller's stream meanwhile, so that each
    launch's events bracket that launch alone and the shares compare with ncu's serialised
    launch list (the timed region itself keeps both streams).  With `overhead_us` (see
    launch_overhead_us) each class also gets its time net of one launch processing per launch,
    `ms_net_per_step`, the figure that compares with a profiler's kernel durations."""
    hq.hq_debug_timing_serialize(True)
    try:
        hq.hq_debug_timing_start(list(KERNEL_NAMES))
        layer.step()  # creates the events
        torch.cuda.synchronize()
        hq.hq_debug_timing_start(list(KERNEL_NAMES))
        for k in range(steps):
            flush.fill_(k & 0xFF)
            layer.step()
        torch.cuda.synchronize()
        hq.hq_debug_timing_stop()
    finally:
        hq.hq_debug_timing_serialize(False)
    out = {}
    for cls, (name, unit) in KERNEL_NAMES.items():
        ms, work, n = hq.hq_debug_timing_read(cls)
        if n == 0:
            continue
        scale = 1e12 if unit == "TFLOP/s" else 1e9
        out[cls] = {"kernel": name, "ms_per_step": ms / steps, "launches_per_step": n / steps,
                    "achieved": work / (ms / 1e3) / scale, "unit": unit, "ms_total": ms, "work_total": work,
                    "launches_total": n}
        if overhead_us is not None:
            out[cls]["ms_net_per_step"] = max(ms - n * overhead_us / 1e3, 0.0) / steps
    return out


def time_syrk_per_call(hq, layer, flush, peaks, tokens: int = 512, reps: int = 3):
    """The layer's Hessian accumulated call by call as its chunks arrive (16 calls of 512 tokens
    for q_proj) instead of in one call; each pass timed by events after an L2 flush (median of
    `reps`).  Per call the roofline is the larger of its flops at the bf16 burst and the
    read-modify-write of H's lower triangle at the measured HBM rate."""
    try:
        cfg = layer.cfg
        K, T = cfg.K, cfg.T
        calls = T // tokens
        H = torch.zeros((K, K), dtype=torch.float32, device=layer.X.device)
        chunks = [layer.X[c * tokens:(c + 1) * tokens] for c in range(calls)]

        def one_pass():
            for x in chunks:
                hq.hq_hessian_accumulate(H, x)

        one_pass()
        times = []
        for rep in range(reps):
            flush.fill_(7 + rep)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            one_pass()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        del H
        flop_call = tokens * K * (K + 1)
        rmw_call = 2.0 * 4.0 * K * (K + 1) / 2  # H's lower triangle read and written
        roof_us = max(flop_call / (peaks["bf16_tflops"] * 1e12), rmw_call / (peaks["hbm_gbs"] * 1e9)) * 1e6
        per_call_us = ms * 1e3 / calls
        return {"workload": f"{cfg.name}: {calls} calls of X bf16 [{tokens}, {K}] into one H",
                "ms": ms, "us_per_call": per_call_us, "tflops": calls * flop_call / (ms / 1e3) / 1e12,
                "roofline_us_per_call": roof_us, "frac": roof_us / per_call_us,
                "bound": "hbm (H read-modify-write)" if rmw_call / (peaks["hbm_gbs"] * 1e9) >
                flop_call / (peaks["bf16_tflops"] * 1e12) else "tensor",
                "peak_source": peaks["source"] + " bf16 dense burst and HBM copy"}
    except Exception as e:  # a measurement beside the line: never lose the line for it
        return {"error": str(e)}


def codec_throughput(hq, layer, flush, reps: int = 5, rest_s: float = 0.5):
    """Encode and decode of the step's H, each launched right after an L2 flush and timed by
    events around the call alone (in the step, the encode follows hq_gptq_quantize's host
    synchronisation, so its stage time also holds the host's launch latency).  The flush ends
    with a read so that no dirty lines are written back during the timed call.  The GPU first
    idles for `rest_s` seconds: for a few hundred ms after a power-capped burst (the chunked
    SYRK at scale runs at the 1 kW cap) the clocks recover, and in that window a plain fill of
    the same buffer moves about a quarter fewer bytes per second; the rested figure is the
    kernel's, the other the transient's (reported beside it where a burst precedes)."""
    if rest_s > 0:
        torch.cuda.synchronize()
        time.sleep(rest_s)
    K = layer.cfg.K
    enc_ms, dec_ms = [], []
    # a write then a read of buffers larger than L2: the L2 holds clean lines of neither input
    scratch = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=flush.device)

    def clean_flush(r):
        flush.fill_(r & 0xFF)
        scratch.sum()

    for r in range(reps + 1):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        clean_flush(r)
        ev[0].record()
        hq.hq_hessian_pack_bf16tril(layer.H, layer.tril)
        ev[1].record()
        clean_flush(r + 1)
        ev[2].record()
        hq.hq_hessian_unpack_bf16tril(layer.tril, K, layer.Hfull)
        ev[3].record()
        torch.cuda.synchronize()
        if r > 0:  # the first round warms up
            enc_ms.append(ev[0].elapsed_time(ev[1]))
            dec_ms.append(ev[2].elapsed_time(ev[3]))
    enc_bytes = 2 * K * (K + 1) + hq.hq_bf16tril_bytes(K)  # H lower triangle read + payload written
    dec_bytes = hq.hq_bf16tril_bytes(K) + 4 * K * K        # payload read + full H written
    enc_s, dec_s = statistics.median(enc_ms) / 1e3, statistics.median(dec_ms) / 1e3
    return {"encode_gbs": enc_bytes / enc_s / 1e9, "decode_gbs": dec_bytes / dec_s / 1e9,
            "encode_us": enc_s * 1e6, "decode_us": dec_s * 1e6, "bytes": {"encode": enc_bytes, "decode": dec_bytes}}


def fp64_mma_peak(hq):
    """fp64 MMA rate of a kernel doing nothing else (context for the fp64 roofline)."""
    try:
        return hq.hq_debug_fp64_mma_rate()
    except Exception:
        return None


def _best_matmul_rate(fn, flops: float, reps: int) -> float:
    """flops / the shortest of `reps` timed calls of fn (CUDA events, after one warm-up call)."""
    fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        best = min(best, a.elapsed_time(b) / 1e3)
    return flops / best / 1e12


def measure_dense_peaks(hq, dev, n: int = 8192):
    """Dense matrix-product rates of this GPU for the operand types the path uses besides bf16,
    measured the way the bf16 figure of MEASURED_PEAKS.json is (a library GEMM of n^3, the best
    of several calls): tf32 (fp32 torch.matmul with tensor-float-32 allowed), fp64 (fp64
    torch.matmul; the fp64 peak is the larger of that and the library's fp64 MMA rate) and int8
    (torch._int_mm, int32 accumulation)."""
    out = {"method": f"torch.matmul {n}^3 (2 n^3 flops), best of several calls, CUDA events"}
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    flops = 2.0 * n ** 3
    try:
        a = torch.randn((n, n), generator=g, device=dev)
        b = torch.randn((n, n), generator=g, device=dev)
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = True
        try:
            out["tf32_tflops"] = _best_matmul_rate(lambda: a @ b, flops, 10)
        finally:
            torch.backends.cuda.matmul.allow_tf32 = prev
        a64, b64 = a.double(), b.double()
        del a, b
        out["fp64_gemm_tflops"] = _best_matmul_rate(lambda: a64 @ b64, flops, 5)
        del a64, b64
        ai = torch.randint(-128, 128, (n, n), generator=g, device=dev, dtype=torch.int32).to(torch.int8)
        bi = torch.randint(-128, 128, (n, n), generator=g, device=dev, dtype=torch.int32).to(torch.int8)
        out["int8_tops"] = _best_matmul_rate(lambda: torch._int_mm(ai, bi), flops, 10)
        del ai, bi
    except Exception as e:  # a measurement beside the line: never lose the line for it
        out["error"] = str(e)
    torch.cuda.empty_cache()
    out["fp64_mma_rate_tflops"] = fp64_mma_peak(hq)
    rates = [r for r in (out.get("fp64_gemm_tflops"), out["fp64_mma_rate_tflops"]) if r]
    out["fp64_tflops"] = max(rates) if rates else None
    return out


def measure_e2e(args, layer, flush, world):
    cfg = layer.cfg
    weights = cfg.N * cfg.K
    Xh = layer.X.cpu().pin_memory()
    Wh = layer.W.cpu().pin_memory()
    Xd = torch.empty_like(layer.X)
    Wd = torch.empty_like(layer.W)
    codes_h = torch.empty(layer.codes.shape, dtype=layer.codes.dtype).pin_memory()
    scales_h = torch.empty(layer.scales.shape, dtype=layer.scales.dtype).pin_memory()
    tril_h = torch.empty(layer.tril.shape, dtype=layer.tril.dtype).pin_memory()
    qerr_h = torch.empty(1, dtype=torch.float64).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    hq, main = layer.hq, torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined_step():
        """The step's calls with its copies overlapped as a host pipeline would: X then W go up on
        one copy stream; the SYRK starts once X is in; the packed Hessian (which depends on H
        alone) is encoded right after it and copied back on a second copy stream while the
        factorisation runs; the quantisation waits for W."""
        x_in, w_in, tril_out, tril_back = (torch.cuda.Event() for _ in range(4))
        h2d_s.wait_stream(main)
        with torch.cuda.stream(h2d_s):
            Xd.copy_(Xh, non_blocking=True)
            x_in.record()
            Wd.copy_(Wh, non_blocking=True)
            w_in.record()
        main.wait_event(x_in)
        layer.H.zero_()
        hq.hq_hessian_accumulate(layer.H, Xd, dev_status=layer.status)
        hq.hq_imatrix(layer.H, cfg.T, layer.imp)
        hq.hq_hessian_pack_bf16tril(layer.H, layer.tril)
        tril_out.record()
        d2h_s.wait_event(tril_out)
        with torch.cuda.stream(d2h_s):
            tril_h.copy_(layer.tril, non_blocking=True)
            tril_back.record()
        main.wait_event(w_in)
        hq.hq_gptq_quantize(Wd, layer.H, cfg.group, cfg.damp, layer.codes, layer.scales, layer.ws,
                            imp=layer.imp if cfg.use_imatrix else None, want_qerr=False, qerr_dev=layer.qerr)
        hq.hq_hessian_unpack_bf16tril(layer.tril, cfg.K, layer.Hfull)
        codes_h.copy_(layer.codes, non_blocking=True)
        scales_h.copy_(layer.scales, non_blocking=True)
        qerr_h.copy_(layer.qerr, non_blocking=True)
        main.wait_event(tril_back)  # the step ends when every copy has landed

    for _ in range(2):
        pipelined_step()
    torch.cuda.synchronize()
    e_start = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_end = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    _barrier(world)
    for k in range(e2e_steps):
        flush.fill_(k & 0xFF)
        e_start[k].record()
        pipelined_step()
        e_end[k].record()
    torch.cuda.synchronize()
    _barrier(world)
    e2e_ms = _max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_start, e_end)), world) / e2e_steps
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = (codes_h.numel() * codes_h.element_size() + scales_h.numel() * scales_h.element_size() +
           tril_h.numel() * tril_h.element_size() + 8)
    return {"value": weights * world / (e2e_ms / 1e3), "unit": "weights/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def syrk_line(kernels, stage_tflops, peaks):
    """The SYRK kernel against the bf16 peak: `achieved` from the kernel's own launch events,
    `stage_achieved` from the stage events (which also hold the zeroing of H and launch gaps)."""
    k = kernels.get("syrk") if kernels else None
    achieved = k["achieved"] if k else stage_tflops
    sus = peaks.get("bf16_tflops_sustained")
    return {"kernel": "syrk_tc_kernel (X^T X)", "bound": "tensor", "achieved": achieved,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "peak_sustained": sus, "frac_sustained": achieved / sus if sus else None,
            "stage_achieved": stage_tflops, "peak_source": peaks["source"] + " bf16 dense burst (and sustained)"}


def update_line(cfg, kernels, peaks):
    """The lazy updates against their per-launch roofline (update_roofline_ms)."""
    k = kernels.get("tf32_gemm") if kernels else None
    if not k:
        return None
    roof = update_roofline_ms(cfg, peaks)
    sus = peaks.get("bf16_tflops_sustained")
    # sustained tf32: the measured tf32 burst scaled by the bf16 sustained / burst ratio
    tf32_sus = peaks["tf32_tflops"] * sus / peaks["bf16_tflops"] if sus else None
    roof_sus = update_roofline_ms(cfg, peaks, tf32_sus) if sus else None
    return {"kernel": "upd_gemm_kernel<BN> (3xTF32 lazy updates)", "bound": "tensor / hbm per launch",
            "ms_per_step": k["ms_per_step"], "roofline_ms_per_step": roof, "frac": roof / k["ms_per_step"],
            "roofline_ms_per_step_sustained": roof_sus,
            "frac_sustained": roof_sus / k["ms_per_step"] if roof_sus else None,
            "achieved_useful_tflops": k["achieved"], "launches_per_step": k["launches_per_step"],
            "tf32_tflops": peaks["tf32_tflops"],
            "peak_source": ("tf32 dense rate measured in this run (torch.matmul fp32 with TF32, 3 MMAs per "
                            "product); " + peaks["source"] + " HBM copy")}


def build_line(args, cfg, world, value, ms_per_step, syrk_ms, gptq_ms, enc_ms, dec_ms, syrk_tflops, enc_bytes,
               dec_bytes, peaks, e2e, launches, clocks, dom, kernels, dense, inline=True, overhead_us=None):
    cls, dom_ms, dom_work, dom_n = dom
    roofline = class_roofline(cls, dom_ms, dom_work, dom_n, args.steps, peaks, cfg)
    roofline["traffic"] = profiled_traffic(cls)
    where = ("inside the timed region" if inline else
             f"in a second pass of the same {args.steps} steps right after the timed region (more than "
             f"{MAX_INLINE_TIMED_LAUNCHES} launches per step: their event pairs would slow the timed steps)")
    roofline["timing"] = (f"every launch of the class timed by CUDA events on its own stream {where}; the class "
                          "with the largest share of a step, net of the launch processing each launch's event "
                          "pair holds, from a breakdown taken before the timed region")
    roofline["launch_overhead_us"] = overhead_us
    roofline["dense_peaks_measured"] = dense
    line = {
        "metric": "GPTQ-int4 weights/s (whole path: SYRK + factorisation + sweep + codec)",
        "value": value,
        "unit": "weights/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in; bf16 tcgen05 SYRK (fp32 accumulate), fp64 factorisation, fp32 sweep, 3xTF32 updates",
        "data": "synthetic (seeded; shapes and distributions of the q_proj-like layer)",
        "config": {"workload": workload_string(cfg), "layers_per_gpu": 1,
                   "l2": "flushed between timed steps (256 MiB write)"},
        "stages_ms": {"syrk": statistics.mean(syrk_ms), "imatrix+factor+sweep": statistics.mean(gptq_ms),
                      "tril_encode": statistics.mean(enc_ms), "tril_decode": statistics.mean(dec_ms)},
        "xtx_tflops": syrk_tflops,
        "codec_gbs": {"encode": enc_bytes / (statistics.mean(enc_ms) / 1e3) / 1e9,
                      "decode": dec_bytes / (statistics.mean(dec_ms) / 1e3) / 1e9},
        "roofline": roofline,
        "kernels": kernels,
        "rooflines": ({k: class_roofline(k, v["ms_total"], v["work_total"], v["launches_total"],
                                         round(v["launches_total"] / v["launches_per_step"]) if v["launches_per_step"]
                                         else 1, peaks, cfg) for k, v in kernels.items()} if kernels else None),
        "syrk_roofline": syrk_line(kernels, syrk_tflops, peaks),
        "update_roofline": update_line(cfg, kernels, peaks),
        "e2e": e2e,
        "gpu_launches": int(launches) * args.steps,
        "gpu_launches_per_step": int(launches),
        "clocks": clocks,
    }
    return line


# ------------------------------------------------------------------------------------ oracle

def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def workload_string(cfg) -> str:
    """The workload's description, the same in both arms' lines."""
    return (f"{cfg.name}: W bf16 [{cfg.N}, {cfg.K}], X bf16 [{cfg.T}, {cfg.K}] ({cfg.n_chunks} chunks of "
            f"{cfg.chunk}), group {cfg.group}, damp {cfg.damp}")


def oracle_fixed(cfg, X):
    """The oracle's per-layer stages, timed: the fp64 Hessian of all the layer's tokens, damping
    and the factorisation, the codec of H.  Returns (U, seconds per stage)."""
    import oracle
    t0 = time.perf_counter()
    H = oracle.hessian(X)
    t1 = time.perf_counter()
    Hd, _ = oracle.damp_hessian(H, cfg.damp)
    U = oracle.upper_factor_of_inverse(Hd)
    t2 = time.perf_counter()
    buf = oracle.bf16tril_encode(H.astype(np.float32))
    oracle.bf16tril_decode(buf, cfg.K)
    t3 = time.perf_counter()
    return U, {"syrk_s": t1 - t0, "factor_s": t2 - t1, "codec_s": t3 - t2}


def oracle_sweep_rows(cfg, W, U, r0: int, rows: int) -> float:
    """Seconds the oracle's sweep and qerr take on rows r0 .. r0 + rows of W (rows are
    independent given U, so a layer's sweep time is proportional to its rows)."""
    import oracle
    Ws = W[r0:r0 + rows]
    t0 = time.perf_counter()
    codes, scales, _ = oracle.gptq_sweep(Ws, U, cfg.group)
    oracle.qerr(Ws, codes, scales, cfg.group)
    return time.perf_counter() - t0


ORACLE_SAMPLE_ROWS = 512  # rows per timed sweep: enough that the per-column overhead is a few %


def cpu_baseline(cfg, layer=None, rows: int = ORACLE_SAMPLE_ROWS):
    """The oracle on a bounded sample of the layer: its per-layer stages in full, then the sweep
    of `rows` rows, scaled to the layer's rows."""
    if layer is not None:
        X = layer.X.double().cpu().numpy()
        W = layer.W.double().cpu().numpy()
    else:
        X = wl.make_activations(cfg, "cpu").double().numpy()
        W = wl.make_weights(cfg, "cpu").double().numpy()
    U, fixed = oracle_fixed(cfg, X)
    rows = min(rows, cfg.N)
    t_sweep = oracle_sweep_rows(cfg, W, U, 0, rows)
    est = sum(fixed.values()) + t_sweep * cfg.N / rows
    return {"value": cfg.N * cfg.K / est, "unit": "weights/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": (f"{workload_string(cfg)}: the oracle's fp64 Hessian of all {cfg.T} tokens, factorisation "
                       f"and codec in full, and its sweep of {rows} of the {cfg.N} rows, scaled to all rows "
                       f"(rows are independent given U)"),
            "stages_s": dict(fixed, sweep_s=t_sweep, sweep_rows=rows), "host": _host_cpu(),
            "tiny_single_thread": _oracle_tiny_single_thread()}


def _host_cpu():
    """The host's CPU model and logical core count (recorded beside the oracle's timing)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


def _oracle_tiny_single_thread(reps: int = 5):
    """The oracle's whole path on the tiny layer (W [64, 128], X [512, 128], group 32) with the
    BLAS limited to one thread: the median of `reps` runs."""
    import oracle
    cfg = wl.CONFIGS[0]
    X = wl.make_activations(cfg, "cpu").double().numpy()
    W = wl.make_weights(cfg, "cpu").double().numpy()
    try:
        import threadpoolctl
        limit = threadpoolctl.threadpool_limits(1)
    except Exception:
        limit = None
    try:
        times = []
        for _ in range(reps):
            t0 = time.perf_counter()
            H = oracle.hessian(X)
            r = oracle.gptq_quantize(W, H, cfg.group, cfg.damp)
            oracle.qerr(W, r["codes"], r["scales"], cfg.group)
            oracle.bf16tril_decode(oracle.bf16tril_encode(H.astype(np.float32)), cfg.K)
            times.append(time.perf_counter() - t0)
    finally:
        if limit is not None:
            limit.restore_original_limits()
    t = statistics.median(times)
    return {"workload": f"{cfg.name}: W [{cfg.N}, {cfg.K}], X [{cfg.T}, {cfg.K}], group {cfg.group}",
            "threads": 1, "s_per_step": t, "weights_per_s": cfg.N * cfg.K / t}


def run_reference(args, budget_s: float = 150.0):
    """The base contract's reference arm: the fp64 oracle, as it stands, on the host cores.  The
    oracle's per-layer stages (Hessian, factorisation, codec) run once before the timed loop;
    each step then sweeps the next block of rows (up to ORACLE_SAMPLE_ROWS, fewer when
    warm-up + steps would otherwise exceed `budget_s`).  `ms_per_step` is the measured time of a
    step; `value` scales the mean per-row sweep time to the layer and adds the per-layer
    stages."""
    cfg = wl.CONFIGS[args.config]
    X = wl.make_activations(cfg, "cpu").double().numpy()
    W = wl.make_weights(cfg, "cpu").double().numpy()
    U, fixed = oracle_fixed(cfg, X)
    del X
    t_row = oracle_sweep_rows(cfg, W, U, 0, 32) / 32
    n_steps = max(args.warmup + args.steps, 1)
    rows = int(budget_s / n_steps / max(t_row, 1e-9)) // 64 * 64
    rows = max(64, min(ORACLE_SAMPLE_ROWS, rows, cfg.N))
    r0 = 0
    for _ in range(args.warmup):
        oracle_sweep_rows(cfg, W, U, r0, rows)
        r0 = (r0 + rows) % (cfg.N - rows + 1)
    step_s = []
    for _ in range(args.steps):
        step_s.append(oracle_sweep_rows(cfg, W, U, r0, rows))
        r0 = (r0 + rows) % (cfg.N - rows + 1)
    per_row = statistics.mean(step_s) / rows
    est = sum(fixed.values()) + per_row * cfg.N
    value = cfg.N * cfg.K / est
    cores = _blas_threads()
    sample = (f"{workload_string(cfg)}: per step the oracle's sweep (and qerr) of {rows} of the {cfg.N} rows; "
              f"its Hessian of all {cfg.T} tokens, factorisation and codec ({sum(fixed.values()):.1f} s) once "
              f"before the timed steps; value = weights / (those stages + mean per-row sweep time x {cfg.N} rows)")
    return {
        "impl": "reference",
        "metric": "GPTQ-int4 weights/s (whole path: SYRK + factorisation + sweep + codec)",
        "value": value, "unit": "weights/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(step_s) * 1e3 if step_s else None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": workload_string(cfg), "layers_per_gpu": 1},
        "cpu_baseline": {"value": value, "unit": "weights/s", "cores": cores, "kind": "oracle", "sample": sample,
                         "host": _host_cpu(), "stages_s": fixed, "rows_per_step": rows},
        "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the gate_up / down_proj / Hessian-at-scale measurements after the main line")
    ap.add_argument("--profile-case", choices=["step", "rotation"], default=None,
                    help="run one untimed step (or one Hadamard rotation of W and H) of the configuration on "
                         "cuda:0 and exit (for ncu captures)")
    args = ap.parse_args()

    if args.profile_case == "step":
        import post_weight_quantization_tcgen05_b200 as hq
        layer = Layer(hq, wl.CONFIGS[args.config], torch.device("cuda:0"))
        layer.step()
        torch.cuda.synchronize()
        print(f"one step of {wl.CONFIGS[args.config].name} done", flush=True)
        return
    if args.profile_case == "rotation":
        import post_weight_quantization_tcgen05_b200 as hq
        from post_weight_quantization_tcgen05_b200 import quarot
        cfg = wl.CONFIGS[args.config]
        layer = Layer(hq, cfg, torch.device("cuda:0"))
        layer.step()  # the layer's Hessian
        g = torch.Generator(device="cuda:0")
        g.manual_seed(42)
        s = quarot.random_signs(cfg.K, g, device=torch.device("cuda:0"))
        Wr = torch.empty((cfg.N, cfg.K), dtype=torch.float32, device="cuda:0")
        Hr = torch.empty((cfg.K, cfg.K), dtype=torch.float32, device="cuda:0")
        hq.hq_hadamard_rotate_weights(layer.W, s, 256, Wr)
        hq.hq_hadamard_rotate_hessian(layer.H, s, 256, Hr)
        torch.cuda.synchronize()
        print(f"one rotation of {cfg.name} done", flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
