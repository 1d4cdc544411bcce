"""Benchmark: W4A4 Gated DeltaNet layer prefill on B200.

One step = one full layer forward (every hot-path stage: quantize x, fused
q/k/v/a/b NVFP4 GEMM with the gates in its epilogue, chunked delta rule,
quantize o, output NVFP4 GEMM) over the layer workload: B=4 sequences x
T=8192 tokens, d_model=5120, H=32 heads of d=128, synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  N > 1 runs one process per GPU (launched by
torch.distributed.run); every rank runs its own independent batch (weak
scaling, no data-path collective) and the time is the max over ranks.
``--impl reference`` times the CPU oracle (the plain FP64 / FP32 restatement
of the method) on the host cores over a bounded sample of the same workload.
"""
import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN W4A4 layer prefill tokens/s"
UNIT = "tokens/s"
WORKLOAD = dict(B=4, T=8192, d_model=5120, H=32, dk=128, dv=128)
WORKLOAD_NAME = "gdn_w4a4_layer_prefill B=4 T=8192 d_model=5120 H=32 dk=dv=128"
# kernels of ours one layer forward launches: amax(x), quantize(x), q/k/v/a/b GEMM,
# scan, quantize(o) with the scan's amax, output GEMM (the two amax words are
# cleared with cudaMemsetAsync, which launches none of ours)
LAUNCHES_PER_LAYER_STEP = 6
CPU_SAMPLE_T = 256            # tokens of one sequence for the oracle sample


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p = {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
             "bf16_tflops_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]), "source": "measured"}
    return p


# ------------------------------------------------------------ clock sampler --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.skip = 0

    def _lines(self):
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except OSError:
            return 0

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
               "-lms", "20"]
        try:
            # line-buffered, so that every sample reaches the file at once
            self.proc = subprocess.Popen((["stdbuf", "-oL"] if shutil.which("stdbuf") else []) + cmd,
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # nvidia-smi takes a moment to start: wait for its first sample, so that
        # the samples after it fall inside the timed region that follows
        deadline = time.time() + 10
        while self.proc is not None and self.proc.poll() is None and time.time() < deadline:
            n = self._lines()
            if n:
                self.skip = n
                break
            time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        inside = rows[self.skip:]   # the samples taken during the timed region
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        adjacent = not inside
        rows = inside or rows[-1:]   # else the sample taken just before the region began
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s in sm if smax and s > 0.3 * max(smax)] or sm
        out = {"sm_mhz": statistics.median(loaded) if loaded else None,
               "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
               "samples": len(inside)}
        if adjacent:
            out["note"] = "no sample inside the timed region; the one taken just before it"
        return out


# ---------------------------------------------------- multi-rank plumbing --
def replica_seed(rank):
    """Seed of the batch a rank processes: every rank (GPU) runs its own
    independent batch of the layer workload, so the job scales weakly."""
    return 3 + rank


def max_over_ranks(v, world, device):
    """The largest of one float over all ranks (the job's time is its slowest
    rank's)."""
    if world == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(total_ms, steps, tokens_per_rank, world):
    """(whole-job tokens/s, ms per step) from the max-over-ranks time of
    `steps` steps in which every rank processed `tokens_per_rank` tokens."""
    ms_per_step = total_ms / steps
    return tokens_per_rank * world / (ms_per_step / 1e3), ms_per_step


# ---------------------------------------------------------------- our path --
def stage_costs(B, T, d_model, H, dk, dv):
    """Algorithmic bytes (HBM-bound stages) or FLOPs (contractions) of one
    launch of each stage of the layer."""
    M = B * T
    HK, HV = H * dk, H * dv
    N1 = 2 * HK + HV + 2 * H
    return {
        "quant_x": ("hbm", M * d_model * 2 + M * d_model // 2 + M * d_model // 16),
        "gemm_qkvab": ("tensor", 2.0 * M * N1 * d_model),
        "delta_rule": ("hbm", M * (2 * HK + HV) * 2 + 2 * M * H * 4 + M * HV * 2 + B * H * dk * dv * 4),
        "quant_o": ("hbm", M * HV * 2 + M * HV // 2 + M * HV // 16),
        "gemm_out": ("tensor", 2.0 * M * d_model * HV),
    }


def source_digest(files):
    """sha256 (first 16 hex digits) of the kernel sources a profile was taken
    from, concatenated in the given order."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "nvfp4_w4a4_gated_quant_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(stage):
    """DRAM bytes (read + write) per launch of a layer stage from the committed
    ncu summary, if the kernel sources it was taken from are unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(stage)
    if not rec:
        return None
    return rec["bytes_per_launch"] if source_digest(rec["sources"]) == rec["source_sha"] else None


def run_ours(args, rank, world, local_rank):
    import torch
    from nvfp4_w4a4_gated_quant_b200 import _lib, inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    W = dict(WORKLOAD, B=args.layer_B, T=args.layer_T)
    B, T, D, H, dk, dv = W["B"], W["T"], W["d_model"], W["H"], W["dk"], W["dv"]
    M, HK, HV = B * T, H * dk, H * dv
    workload_name = (WORKLOAD_NAME if (B, T) == (WORKLOAD["B"], WORKLOAD["T"]) else
                     f"gdn_w4a4_layer_prefill B={B} T={T} d_model={D} H={H} dk=dv={dk} (reduced: a profiling case)")
    d = inputs.layer_inputs(B, T, D, H, dk, dv, seed=replica_seed(rank))
    stream = torch.cuda.current_stream()
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv, device=dev)
    x_host = torch.from_numpy(d["x"]).to(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    y = torch.empty_like(x)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    y_host = torch.empty(x.shape, dtype=torch.bfloat16).pin_memory()
    cfg = _lib.layer_cfg(B, T, D, H, dk, dv)
    ws = torch.empty(_lib.gdn_layer_workspace_size(cfg), dtype=torch.uint8, device=dev)
    off = _lib.gdn_layer_workspace_offsets(cfg)

    def layer_step():
        _lib.gdn_layer_fwd(lw, x, y=y, S_T=S_T, ws=ws)

    # views of the workspace for the staged run (same calls the layer makes)
    u8 = ws
    NQKV = 2 * HK + HV
    x_codes = u8[off[_lib.WS_X_CODES]:].narrow(0, 0, M * D // 2).view(M, D // 2)
    x_scales = u8[off[_lib.WS_X_SCALES]:].narrow(0, 0, _lib.scales_tiled_bytes(M, D))
    x_g = u8[off[_lib.WS_X_G]:].narrow(0, 0, 4).view(torch.float32)
    qkv = u8[off[_lib.WS_QKV]:].narrow(0, 0, M * NQKV * 2).view(torch.bfloat16).view(M, NQKV)
    la = u8[off[_lib.WS_LOG_ALPHA]:].narrow(0, 0, M * H * 4).view(torch.float32).view(M, H)
    be = u8[off[_lib.WS_BETA]:].narrow(0, 0, M * H * 4).view(torch.float32).view(M, H)
    o = u8[off[_lib.WS_O]:].narrow(0, 0, M * HV * 2).view(torch.bfloat16).view(B, T, H, dv)
    o_codes = u8[off[_lib.WS_O_CODES]:].narrow(0, 0, M * HV // 2).view(M, HV // 2)
    o_scales = u8[off[_lib.WS_O_SCALES]:].narrow(0, 0, _lib.scales_tiled_bytes(M, HV))
    o_g = u8[off[_lib.WS_O_G]:].narrow(0, 0, 4).view(torch.float32)
    qws = u8[off[_lib.WS_QUANT]:].narrow(0, 0, 256)
    segs = [
        {"n_begin": 0, "n_end": HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["q"], "out": qkv, "ld_out": NQKV},
        {"n_begin": HK, "n_end": 2 * HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["k"], "out": qkv, "out_offset": HK,
         "ld_out": NQKV},
        {"n_begin": 2 * HK, "n_end": NQKV, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["v"], "out": qkv,
         "out_offset": 2 * HK, "ld_out": NQKV},
        {"n_begin": NQKV, "n_end": NQKV + H, "kind": _lib.EPI_LOG_ALPHA, "g_b": lw.g["a"], "out": la, "ld_out": H,
         "A_log": lw.A_log, "dt_bias": lw.dt_bias},
        {"n_begin": NQKV + H, "n_end": NQKV + 2 * H, "kind": _lib.EPI_BETA, "g_b": lw.g["b"], "out": be, "ld_out": H},
    ]
    qv = qkv.view(B, T, NQKV)
    stages = [
        ("quant_x", lambda: _lib.gdn_quantize_nvfp4(x.view(M, D), codes=x_codes, scales=x_scales, g_out=x_g, ws=qws)),
        ("gemm_qkvab", lambda: _lib.gdn_gemm_nvfp4(x_codes, x_scales, x_g, lw.codes, lw.scales, M, NQKV + 2 * H, D,
                                                  segs)),
        ("delta_rule", lambda: _lib.gdn_delta_rule_fwd(
            qv[:, :, :HK].view(B, T, H, dk), qv[:, :, HK:2 * HK].view(B, T, H, dk),
            qv[:, :, 2 * HK:].view(B, T, H, dv), la.view(B, T, H), be.view(B, T, H), o=o, S_T=S_T)),
        # the layer quantizes o with the amax the scan recorded (no amax pass)
        ("quant_o", lambda: _lib.gdn_quantize_nvfp4(o.view(M, HV), codes=o_codes, scales=o_scales, g_out=o_g, ws=qws,
                                                    amax=o_amax)),
        ("gemm_out", lambda: _lib.gemm_bf16(o_codes, o_scales, o_g, lw.out_codes, lw.out_scales, lw.g["out"], M, D, HV,
                                            out=y.view(M, D))),
    ]

    def barrier():
        if world > 1:
            torch.distributed.barrier()


    # ---- warm-up
    for _ in range(args.warmup):
        layer_step()
    _lib.stream_check()

    # ---- timed: the product call on device-resident inputs
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            layer_step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
    _lib.stream_check()
    total_ms = ev[0].elapsed_time(ev[-1])
    step_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(total_ms, world, dev)
    value, ms_per_step = aggregate(total_ms, args.steps, M, world)

    # ---- stage breakdown: the same calls one by one, events between them
    o_amax = o.abs().amax().float().reshape(1)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    for _, fn in stages:
        fn()
    torch.cuda.synchronize()
    for i in range(args.steps):
        sev[i][0].record(stream)
        for j, (_, fn) in enumerate(stages):
            fn()
            sev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    _lib.stream_check()
    stage_ms = {name: statistics.mean(sev[i][j].elapsed_time(sev[i][j + 1]) for i in range(args.steps))
                for j, (name, _) in enumerate(stages)}

    # ---- the layer with static, per-module calibrated activation scales: x
    # quantized in one pass (no amax pass), o quantized in the scan's epilogue
    # (no quantizer pass).  Calibrated on this input itself, so the scales are
    # its dynamic ones and the layer's output is the same.
    lw.x_g_enc, lw.o_g_enc = _lib.calibrate_layer(lw, [x])
    for _ in range(args.warmup):
        layer_step()
    ss0, ss1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ss0.record(stream)
    for _ in range(args.steps):
        layer_step()
    ss1.record(stream)
    torch.cuda.synchronize()
    barrier()
    _lib.stream_check()
    lw.x_g_enc = lw.o_g_enc = None
    static_ms = max_over_ranks(ss0.elapsed_time(ss1), world, dev)
    static_value, static_ms_step = aggregate(static_ms, args.steps, M, world)

    # ---- the layer with the rest of a Gated DeltaNet block (outside
    # specification): a sixth W4A4 projection g, the short convolution + SiLU
    # on q, k, v and the gated RMSNorm of o (seeded synthetic weights)
    rng_ext = np.random.default_rng(replica_seed(rank) + 100)
    W_ext = dict(d["W"])
    W_ext["g"] = inputs.weight(rng_ext, HV, D)
    lw_ext = _lib.QuantizedLayerWeights(W_ext, d["A_log"], d["dt_bias"], H, dk, dv, device=dev,
                                        conv_w=rng_ext.uniform(-0.6, 0.6, (2 * HK + HV, 4)).astype(np.float32),
                                        norm_w=rng_ext.uniform(0.5, 1.5, dv).astype(np.float32))
    ws_ext = torch.empty(_lib.gdn_layer_workspace_size(lw_ext.cfg(B, T)), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        _lib.gdn_layer_fwd(lw_ext, x, y=y, S_T=S_T, ws=ws_ext)
    ex0, ex1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ex0.record(stream)
    for _ in range(args.steps):
        _lib.gdn_layer_fwd(lw_ext, x, y=y, S_T=S_T, ws=ws_ext)
    ex1.record(stream)
    torch.cuda.synchronize()
    barrier()
    _lib.stream_check()
    ext_ms = max_over_ranks(ex0.elapsed_time(ex1), world, dev)
    ext_value, ext_ms_step = aggregate(ext_ms, args.steps, M, world)
    del lw_ext, ws_ext

    # ---- end to end through the public call with host buffers: every step
    # copies its input in from pinned host memory and its output back, with
    # two device buffers so that step i+1's copy-in and step i-1's copy-out
    # run on their own streams while step i computes
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    xb, yb = [x, torch.empty_like(x)], [y, torch.empty_like(y)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(args.steps):
        b = i % 2
        if i >= 2:
            s_in.wait_event(ev_cmp[b])            # the step that read xb[b] is done
        with torch.cuda.stream(s_in):
            xb[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])          # yb[b] has been copied out
        _lib.gdn_layer_fwd(lw, xb[b], y=yb[b], S_T=S_T, ws=ws, stream=stream)
        ev_cmp[b].record(stream)
        s_out.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_out):
            y_host.copy_(yb[b], non_blocking=True)
            ev_out[b].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps

    # ---- standalone kernels of the GEMM and scan workloads (context keys)
    kernels = standalone_kernels(args, torch, _lib, inputs, dev, stream) if rank == 0 and not args.skip_kernels else {}

    clk = clocks.summary()
    tokens_per_step = M * world
    pk = peaks()
    # the FP4 denominator: the tensor pipe's own ceiling for this MMA, measured
    # on this GPU in this run; without it, 4x the measured burst bf16 rate (the
    # nominal 9 / 2.25 PFLOP/s ratio)
    fp4_ceiling = kernels.get("fp4_mma_ceiling", {}).get("TFLOPs") if kernels else None
    fp4_peak = fp4_ceiling or 4.0 * pk["bf16_tflops"]
    costs = stage_costs(B, T, D, H, dk, dv)
    stage_out = {}
    for name, ms in stage_ms.items():
        bound, work = costs[name]
        if bound == "hbm":
            ach = work / (ms / 1e3) / 1e9
            stage_out[name] = {"us": round(ms * 1e3, 1), "bound": "hbm", "achieved_GBps": round(ach, 1),
                               "frac": round(ach / pk["hbm_gbs"], 4)}
        else:
            ach = work / (ms / 1e3) / 1e12
            stage_out[name] = {"us": round(ms * 1e3, 1), "bound": "tensor", "achieved_TFLOPs": round(ach, 1),
                               "frac": round(ach / fp4_peak, 4)}
    dom = max(stage_ms, key=stage_ms.get)
    bound, work = costs[dom]
    kname = {"quant_x": "quant_kernel", "quant_o": "quant_kernel", "gemm_qkvab": "gemm_nvfp4_kernel",
             "gemm_out": "gemm_nvfp4_kernel", "delta_rule": "delta_rule_kernel"}[dom]
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": round(work / (stage_ms[dom] / 1e3) / 1e9, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": round(work / (stage_ms[dom] / 1e3) / 1e12, 1), "peak": fp4_peak,
                "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["traffic"] = traffic_from_profiles(dom)
    roof["kernel"] = f"{dom} ({kname})"
    roof["peak_source"] = (f"{pk['source']}: hbm_gbs" if bound == "hbm" else
                           "measured in this run: gdn_fp4_mma_ceiling" if fp4_ceiling else
                           f"{pk['source']}: 4 x bf16_tflops burst (FP4 = 4x bf16 nominal)")
    if bound == "tensor":
        roof["frac_fp4_nominal_9PF"] = round(roof["achieved"] / 9000.0, 4)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3, fp32 acc); scan fp16 mma, fp32 state",
        "data": "synthetic",
        "config": {"workload": workload_name, **W, "tokens_per_step_per_gpu": M,
                   "l2": "inputs exceed L2 (x 335 MB, q/k/v 805 MB per step); no flush",
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "e2e": {"value": round(tokens_per_step / (e2e_ms / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2},
        "gpu_launches": LAUNCHES_PER_LAYER_STEP * args.steps,
        "roofline": roof,
        "stages": stage_out,
        "static_scales": {"value": round(static_value, 1), "unit": UNIT, "ms_per_step": round(static_ms_step, 4),
                          "what": "the same layer with per-module calibrated static activation scales (x and o, "
                                  "calibrated on this input, so equal to its dynamic ones): x quantized in one "
                                  "pass, o quantized in the scan epilogue"},
        "with_conv_and_out_gate": {"value": round(ext_value, 1), "unit": UNIT, "ms_per_step": round(ext_ms_step, 4),
                                   "what": "the layer with a sixth projection g (H*dv more GEMM columns), the short "
                                           "convolution + SiLU on q/k/v and the gated RMSNorm of o"},
        "clocks": clk,
        "step_ms_min_max": [round(min(step_ms), 4), round(max(step_ms), 4)],
    }
    if kernels:
        line["kernels"] = kernels
    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline(seconds_budget=args.cpu_seconds, T_sample=args.sample_tokens)
    return line


def fp4_ceiling_tflops(torch, _lib, stream, iters=40000, reps=3):
    """The FP4 tensor-core ceiling of the GEMM's MMA (gdn_fp4_mma_ceiling:
    one CTA per SM issuing 128 x 256 x 64 block-scaled MMAs back to back from
    resident operands), best of `reps` runs of ~20 ms, in TFLOP/s."""
    best = 0.0
    _lib.fp4_mma_ceiling(1000, stream)
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        flops = _lib.fp4_mma_ceiling(iters, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        best = max(best, flops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    _lib.stream_check()
    return best


def standalone_kernels(args, torch, _lib, inputs, dev, stream, which=None):
    """The GEMM workload (8192 x 12288 x 5120, bf16 out) and the scan workload
    (T=32768, H=16, d=128) timed alone, for their own roofline fractions."""
    out = {}
    pk = peaks()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(args.steps, 10) if which is None else args.steps
    if which == "scan":
        return standalone_scan(args, torch, _lib, dev, stream, out, pk, e0, e1, reps)
    rng = np.random.default_rng(1)
    M, N, K = 8192, 12288, 5120
    x = torch.from_numpy(inputs.activations(rng, (M, K))).to(dev).to(torch.bfloat16)
    w = torch.randn((N, K), generator=torch.Generator().manual_seed(1)).mul_(0.02).to(dev)
    xc, xs, gx = _lib.gdn_quantize_nvfp4(x)
    wc, wsc, gw = _lib.gdn_quantize_nvfp4(w)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for _ in range(args.warmup):
        _lib.gemm_bf16(xc, xs, gx, wc, wsc, gw, M, N, K, out=y)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        _lib.gemm_bf16(xc, xs, gx, wc, wsc, gw, M, N, K, out=y)
    e1.record(stream)
    torch.cuda.synchronize()
    _lib.stream_check()   # a kernel that gave up (bounded waits) raises instead of timing
    ms = e0.elapsed_time(e1) / reps
    tf = 2.0 * M * N * K / (ms / 1e3) / 1e12
    ceil = fp4_ceiling_tflops(torch, _lib, stream)
    out["fp4_mma_ceiling"] = {"TFLOPs": round(ceil, 1), "what": "gdn_fp4_mma_ceiling: 128x256x64 mxf4nvf4 MMAs "
                                                               "back to back from resident operands, one CTA per SM",
                              "frac_fp4_nominal_9PF": round(ceil / 9000.0, 4)}
    out["gemm_8192x12288x5120"] = {"us": round(ms * 1e3, 1), "TFLOPs": round(tf, 1),
                                   "frac_fp4_ceiling": round(tf / ceil, 4),
                                   "frac_fp4_burst": round(tf / (4 * pk["bf16_tflops"]), 4),
                                   "frac_fp4_nominal_9PF": round(tf / 9000.0, 4)}
    del x, w, xc, xs, wc, wsc, y
    if which == "gemm":
        return out
    return standalone_scan(args, torch, _lib, dev, stream, out, pk, e0, e1, reps)


def standalone_scan(args, torch, _lib, dev, stream, out, pk, e0, e1, reps):
    """The scan workload exactly (B=1, T=32768, H=16, d=128, seed 2: q, k, v
    N(0,1) bf16, gates from a, b ~ N(0,1), A_log ~ U(-2,1), dt_bias ~ U(-1,1)),
    gates computed by the library, then the scan timed alone."""
    from nvfp4_w4a4_gated_quant_b200 import inputs
    w = inputs.scan_workload()
    B, T, H, d = w["q"].shape
    q, k, v = (torch.from_numpy(w[n]).to(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    la, be = _lib.gdn_gates(torch.from_numpy(w["a"]).reshape(B * T, H).to(dev),
                            torch.from_numpy(w["b"]).reshape(B * T, H).to(dev),
                            torch.from_numpy(w["A_log"]).to(dev), torch.from_numpy(w["dt_bias"]).to(dev))
    la, be = la.view(B, T, H), be.view(B, T, H)
    g = torch.Generator().manual_seed(2)
    o = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)
    S = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    nbytes = 4 * B * T * H * d * 2 + 2 * B * T * H * 4 + B * H * d * d * 4
    # the default kernel (tcgen05 for this shape) and the mma.sync one
    for key, mma_sync in (("scan_T32768_H16_d128", False), ("scan_T32768_H16_d128_mma_sync", True)):
        for _ in range(args.warmup):
            _lib.gdn_delta_rule_fwd(q, k, v, la, be, o=o, S_T=S, mma_sync=mma_sync)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            _lib.gdn_delta_rule_fwd(q, k, v, la, be, o=o, S_T=S, mma_sync=mma_sync)
        e1.record(stream)
        torch.cuda.synchronize()
        _lib.stream_check()
        ms = e0.elapsed_time(e1) / reps
        gbs = nbytes / (ms / 1e3) / 1e9
        out[key] = {"us": round(ms * 1e3, 1), "GBps": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}
    # one decode step of 64 sequences x 32 heads x d 128 (state updated in
    # place; 134 MB of state, read and written once per step)
    B, T, H = 64, 1, 32
    q = torch.randn((B, T, H, d), generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn((B, T, H, d), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((B, T, H, d), generator=g).to(torch.bfloat16).to(dev)
    la = (-torch.rand((B, T, H), generator=g) * 1.5).to(dev)
    be = torch.rand((B, T, H), generator=g).to(dev)
    S = (torch.randn((B, H, d, d), generator=g) * 0.1).to(dev)
    o = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)
    nbytes = B * H * (2 * d * d * 4 + T * (3 * d * 2 + 8 + d * 2))
    for _ in range(args.warmup):
        _lib.gdn_delta_rule_step(q, k, v, la, be, S=S, S_out=S, o=o)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        _lib.gdn_delta_rule_step(q, k, v, la, be, S=S, S_out=S, o=o)
    e1.record(stream)
    torch.cuda.synchronize()
    _lib.stream_check()
    ms = e0.elapsed_time(e1) / reps
    gbs = nbytes / (ms / 1e3) / 1e9
    out["decode_step_B64_H32_d128"] = {"us": round(ms * 1e3, 1), "GBps": round(gbs, 1),
                                       "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}
    return out


# ------------------------------------------------------------ CPU baseline --
def _all_host_threads():
    """Let the oracle's BLAS use every host core (torch.distributed.run sets
    OMP_NUM_THREADS=1 in each rank; the oracle arm runs on rank 0 alone)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=len(os.sched_getaffinity(0)), user_api="blas")
    except Exception:
        return None


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_sample(T_sample):
    """The oracle layer on the first T_sample tokens of one sequence of the
    layer workload (weights quantized by the oracle once, outside the timing)."""
    from oracle.layer import layer_forward, quantize_weights
    from nvfp4_w4a4_gated_quant_b200 import inputs
    W = WORKLOAD
    rng = np.random.default_rng(3)
    x = inputs.activations(rng, (1, T_sample, W["d_model"]))
    Wd = {n: inputs.weight(rng, r, c) for n, (r, c) in {
        "q": (W["H"] * W["dk"], W["d_model"]), "k": (W["H"] * W["dk"], W["d_model"]),
        "v": (W["H"] * W["dv"], W["d_model"]), "a": (W["H"], W["d_model"]), "b": (W["H"], W["d_model"]),
        "out": (W["d_model"], W["H"] * W["dv"])}.items()}
    A = rng.uniform(-2, 1, W["H"])
    dt = rng.uniform(-1, 1, W["H"])
    Wq = quantize_weights(Wd)
    return lambda: layer_forward(x, Wq, A, dt, W["H"], W["dk"], W["dv"])


def cpu_baseline(seconds_budget=20.0, T_sample=CPU_SAMPLE_T):
    _all_host_threads()
    fn = _oracle_sample(T_sample)
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        if time.perf_counter() - t0 > seconds_budget / 2 or n >= 3:
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": round(T_sample / dt, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": f"{T_sample} tokens of 1 sequence of the layer workload (d_model 5120, H 32, d 128), "
                      f"{n} run(s), mean {dt:.2f} s each; weights quantized outside the timing"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    T_sample = getattr(args, "sample_tokens", CPU_SAMPLE_T)
    _all_host_threads()
    fn = _oracle_sample(T_sample)
    for _ in range(min(args.warmup, 1)):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    dt = (time.perf_counter() - t0) / args.steps
    value = T_sample / dt
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (quantizer f32)", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, **WORKLOAD},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
                         "sample": f"each step: the oracle layer on {T_sample} tokens of 1 sequence"},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------- replay workload --
REPLAY = dict(B=1, T=32768, d_model=5120, H=16, dk=128, dv=128, seed=4, checkpoints=(256, 4096, 32768),
              seeds=tuple(range(1, 12)), t_imp=1024, window=2048, eps=0.01)


def run_replay(args):
    """The replay workload: the oracle's clean trajectory (FP64 projections of
    the bf16 activations, scan in FP64) on the host, and 11 NVFP4
    trajectories (independent d_model permutations) through the library;
    relative state error at the checkpoints, the library's scan on the clean
    inputs (its own error), an impulse of 1% at token 1024 followed through
    the library's decode step, and the gate-error compression (projection
    error on a / b against the error on 1 - alpha and beta)."""
    import torch
    from nvfp4_w4a4_gated_quant_b200 import inputs, replay
    from oracle import replay as oreplay
    R = REPLAY
    T, Dm, H, dk, dv = R["T"], R["d_model"], R["H"], R["dk"], R["dv"]
    t_start = time.perf_counter()
    d = inputs.layer_inputs(R["B"], T, Dm, H, dk, dv, seed=R["seed"])
    x = d["x"].reshape(T, Dm)
    _all_host_threads()
    t0 = time.perf_counter()
    clean_proj = oreplay.clean_projections(x, d["W"])
    clean = oreplay._scan_inputs(clean_proj, 1, T, H, dk, dv, d["A_log"], d["dt_bias"])
    S_clean = oreplay.states_at(*clean, R["checkpoints"])
    oracle_s = time.perf_counter() - t0
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    # the library's own error: its scan on the clean inputs
    cd = (torch.from_numpy(clean[0].astype(np.float32)).to(dev).to(torch.bfloat16),
          torch.from_numpy(clean[1].astype(np.float32)).to(dev).to(torch.bfloat16),
          torch.from_numpy(clean[2].astype(np.float32)).to(dev).to(torch.bfloat16),
          torch.from_numpy(clean[3].astype(np.float32)).to(dev).contiguous(),
          torch.from_numpy(clean[4].astype(np.float32)).to(dev).contiguous())
    eps0 = [oreplay.rel_state_error(a.cpu().numpy(), b) for a, b in zip(replay.states_at(*cd, R["checkpoints"]),
                                                                       S_clean)]
    errs, gate = [], []
    steps_q = None
    for sd in R["seeds"]:
        perm = np.random.default_rng(sd).permutation(Dm)
        qkv, a, b = replay.nvfp4_projections(x, d["W"], H, dk, dv, perm=perm, device=dev)
        sin = replay.scan_inputs(qkv, a, b, d["A_log"], d["dt_bias"], T, H, dk, dv)
        S_q = replay.states_at(*sin, R["checkpoints"])
        errs.append([oreplay.rel_state_error(sq.cpu().numpy(), sc) for sq, sc in zip(S_q, S_clean)])
        g = oreplay.gate_error_compression(clean_proj["a"], clean_proj["b"], a.cpu().numpy().astype(np.float64),
                                           b.cpu().numpy().astype(np.float64), d["A_log"], d["dt_bias"])
        gate.append([g["a"], g["b"], g["one_minus_alpha"], g["beta"]])
        if steps_q is None:
            steps_q = replay.impulse_steps(*sin, R["t_imp"], R["window"], R["eps"], seed=12345)
        del qkv, a, b, sin, S_q
    errs = np.asarray(errs)
    gate = np.asarray(gate)
    # the clean trajectory's impulse (oracle, FP64) and its decay-implied horizon
    steps_c, horizon = oreplay.impulse_response(*clean, R["t_imp"], min(R["window"], 256), R["eps"],
                                                np.random.default_rng(12345))
    return {
        "impl": "ours", "mode": "replay",
        "config": {"workload": f"replay B=1 x 12 trajectories T={T} d_model={Dm} H={H} dk=dv={dk} seed {R['seed']}",
                   "checkpoints": list(R["checkpoints"]), "nvfp4_trajectories": len(R["seeds"]),
                   "impulse": f"S *= 1 + {R['eps']} z at token {R['t_imp']}"},
        "state_error": {"mean": [round(float(v), 4) for v in errs.mean(axis=0)],
                        "max": [round(float(v), 4) for v in errs.max(axis=0)],
                        "per_seed": [[round(float(v), 4) for v in row] for row in errs]},
        "library_scan_error_on_clean_inputs": [float(f"{v:.3e}") for v in eps0],
        "impulse_steps_to_1_over_e": {"nvfp4_library_per_head": steps_q.tolist(),
                                      "clean_oracle_per_head": steps_c[0].tolist(),
                                      "decay_horizon_per_head": horizon[0].tolist(),
                                      "median_nvfp4_library": float(np.median(steps_q))},
        "gate_error_compression": {"projection_a": round(float(gate[:, 0].mean()), 4),
                                   "projection_b": round(float(gate[:, 1].mean()), 4),
                                   "one_minus_alpha": round(float(gate[:, 2].mean()), 4),
                                   "beta": round(float(gate[:, 3].mean()), 4)},
        "oracle_seconds": round(oracle_s, 1), "host_threads": _threads(),
        "wall_seconds": round(time.perf_counter() - t_start, 1),
        "parity": "statistics unpinned (synthetic inputs); the path is pinned by tests/test_gpu_replay.py",
    }


def launch_plan(gpus, env):
    """How to run for ``--gpus`` (None: take the launcher's WORLD_SIZE) given
    the environment: ("run", world) in this process, ("relaunch", n) as n
    processes under torch.distributed.run, or ("error", message)."""
    ws = env.get("WORLD_SIZE")
    if ws is None:
        n = 1 if gpus is None else gpus
        if n < 1:
            return ("error", f"--gpus must be >= 1, got {n}")
        return ("run", 1) if n == 1 else ("relaunch", n)
    ws = int(ws)
    if gpus is not None and gpus != ws:
        return ("error", f"--gpus {gpus} but WORLD_SIZE={ws}: launch with --nproc-per-node {gpus}")
    return ("run", ws)


def relaunch(n, argv):
    """Run this script as ``n`` ranks under torch.distributed.run (one process
    per GPU, rendezvous on 127.0.0.1) and return the launcher's exit code."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    try:
        return subprocess.run(cmd, timeout=3600).returncode
    except subprocess.TimeoutExpired:
        print("bench: the ranks did not finish within an hour", file=sys.stderr)
        return 124


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None,
                    help="GPUs (one process each); default: WORLD_SIZE under a launcher, else 1")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-cpu", action="store_true", help="omit the oracle CPU baseline")
    ap.add_argument("--skip-kernels", action="store_true", help="omit the standalone GEMM / scan timings")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--sample-tokens", type=int, default=CPU_SAMPLE_T,
                    help="tokens of the oracle sample (CPU baseline and --impl reference)")
    ap.add_argument("--only", choices=["gemm", "scan"], default=None,
                    help="time only the standalone GEMM or scan workload (profiling target)")
    ap.add_argument("--layer-B", type=int, default=WORKLOAD["B"],
                    help="sequences of the layer workload (a smaller value gives a profiling case)")
    ap.add_argument("--layer-T", type=int, default=WORKLOAD["T"],
                    help="tokens per sequence of the layer workload (a smaller value gives a profiling case)")
    ap.add_argument("--replay", action="store_true",
                    help="run the replay workload (state error of NVFP4 trajectories, impulse, gate errors)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    plan, n = launch_plan(args.gpus, os.environ)
    if plan == "error":
        print(f"bench: {n}", file=sys.stderr)
        sys.exit(2)
    if plan == "relaunch":
        sys.exit(relaunch(n, sys.argv[1:]))
    world = n
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.replay:
        print(json.dumps(run_replay(args)), flush=True)
        return
    if args.only:
        import torch
        from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
        torch.cuda.set_device(local_rank)
        k = standalone_kernels(args, torch, _lib, inputs, torch.device("cuda", local_rank),
                               torch.cuda.current_stream(), which=args.only)
        print(json.dumps({"only": args.only, "kernels": k}), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    line = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
