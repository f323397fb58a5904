"""Benchmark of the fused MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

One step = one full layer forward (route, align, GEMM1+activation, GEMM2+weight,
combine) over one batch of the workload, inputs resident in HBM. The default workload
is the prefill configuration: bf16 SwiGLU, T=4096 tokens, H=2048, 256 experts, top-8,
I=512, renormalised routing with a per-expert logit bias (skewed expert load).
Synthetic seeded data, random-init weights.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and
cuda.synchronize; each step (the forward captured once as a CUDA graph and replayed,
unless --no-graph) is timed with CUDA events on the launching stream, with L2 flushed (a
512 MB write) before every step outside the events. For N > 1 each rank runs
an independent replica (the layer needs no exchange between replicas) and the time is
the max over ranks. Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle (the plain float64 restatement of the method)
on a bounded sample of the same workload on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_expert_topk_b200.synth import CONFIGS, MoeConfig, make_inputs  # noqa: E402

L2_FLUSH_BYTES = 512 << 20

# DRAM traffic of GEMM1 relative to its algorithmic bytes, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum of the GEMM1 launch on the 64-expert
# prefill case), valid only for the kernel source it was taken on (sha256 prefix of the
# file below); None until such a capture exists for that source.
GEMM1_TRAFFIC = {"source": "gemm_swap.cu", "source_sha256": "1f5867c77b7c", "ratio": 308.59 / 281.02}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def _workload_name(cfg: MoeConfig) -> str:
    act = "SwiGLU" if cfg.gated else "relu2"
    dt = ("NVFP4 E2M1 W4A4 (E4M3 scale per 16, fp32 per tensor)" if cfg.nv else
          ("MXFP8 e4m3 W8A8 (E8M0 scale per 32)" if cfg.mx else
           ("FP8 e4m3 W8A8 per-tensor" if cfg.per_tensor else "FP8 e4m3 W8A8 block-128"))) if cfg.fp8 else "bf16"
    sh = f"+{cfg.num_shared} shared" if cfg.num_shared else ""
    return (f"{cfg.name}: {dt} {act} MoE layer forward, T={cfg.T} H={cfg.H} E={cfg.E}{sh} "
            f"top-{cfg.topk}{sh} I={cfg.I}")


class ClockSampler:
    """SM clock and throttle-reason sampling during the timed region.

    A thread polls NVML (the library nvidia-smi reads) every millisecond for the
    device the bench runs on; the timed regions are tens of milliseconds, too short
    for nvidia-smi's own sampling interval. Falls back to "unsampled" without NVML.
    """

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._nvml = (pynvml, h)
        except Exception:
            self._nvml = None
            return self
        self._stop = threading.Event()

        def run():
            pynvml, h = self._nvml
            while not self._stop.is_set():
                try:
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, const in self.REASONS:
                        if r & getattr(pynvml, const, 0):
                            self.reasons.add(name)
                except Exception:
                    pass
                self._stop.wait(0.001)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if self._nvml is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def _dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def touched_expert_bytes(ids: np.ndarray, cfg: MoeConfig, elt: int):
    touched = np.unique(ids)
    w13 = len(touched) * cfg.N1 * cfg.H * elt
    w2 = len(touched) * cfg.H * cfg.I * elt
    return len(touched), w13, w2


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def run_ours(cfg: MoeConfig, steps: int, warmup: int, world: int, rank: int, local: int, args):
    import mixture_experts_expert_topk_b200 as moe
    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, seed=0)
    I_pad = moe.padded_intermediate(cfg.I, cfg.activation, cfg.fp8)
    # static input scale: the hidden rows' amax / 448 (per-tensor FP8) or / (6 * 448) (NVFP4)
    s_in = (float(inp["hidden"].float().abs().max() / 448) if cfg.per_tensor else
            (float(inp["hidden"].float().abs().max() / 2688) if cfg.nv else 0.0))
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, I_pad, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, fp8=cfg.fp8,
                            input_scale=s_in, activation_scale=cfg.activation_scale)
    pt_kw = dict(input_scale=s_in, activation_scale=cfg.activation_scale) if (cfg.per_tensor or cfg.nv) else {}
    hidden = inp["hidden"].to(dev)
    logits = inp["logits"].to(dev)
    s13 = s2 = None
    w13 = inp["w13"].to(dev)
    w2 = inp["w2"].to(dev)
    g13 = g2 = None
    if cfg.nv:
        w13, s13, g13 = moe.quantize_weights_nvfp4(w13)
        w2, s2, g2 = moe.quantize_weights_nvfp4(w2)
    elif cfg.mx:
        w13, s13 = moe.quantize_weights_mxfp8(w13)
        w2, s2 = moe.quantize_weights_mxfp8(w2)
    elif cfg.per_tensor:
        w13, s13 = moe.quantize_weights_fp8_per_tensor(w13)
        w2, s2 = moe.quantize_weights_fp8_per_tensor(w2)
    elif cfg.fp8:
        w13, s13 = moe.quantize_weights_fp8(w13)
        w2, s2 = moe.quantize_weights_fp8(w2)
    if cfg.mx or cfg.nv:
        # the block scales travel inside the prepared weights; the forward takes none
        # (MXFP8) or the weights' tensor scales (NVFP4)
        w13p, w2p = moe.prepare_weights(prob, w13, w2, cfg.I, w13_scale=s13, w2_scale=s2)
        s13, s2 = g13, g2
    else:
        w13p, w2p = moe.prepare_weights(prob, w13, w2, cfg.I)
    del w13, w2
    ws = moe.new_workspace(prob, dev)
    out = torch.empty_like(hidden)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    def forward():
        moe.moe_forward(hidden, logits, w13p, w2p, cfg.topk, cfg.renormalize, cfg.activation,
                        s13, s2, num_shared=cfg.num_shared, workspace=ws, out=out, **pt_kw)

    for _ in range(warmup):
        flush.zero_()
        forward()
    torch.cuda.synchronize(dev)
    st = moe.device_status(ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after warm-up: {st}")
    step = forward
    if args.graph:
        # the whole forward (all kernels, programmatic dependent launches included) as one
        # CUDA graph, replayed each step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            forward()
        graph.replay()
        torch.cuda.synchronize(dev)
        step = graph.replay

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    clocks = clk.summary()

    # per-kernel breakdown: the same kernels through the per-step entry points, events
    # between the steps on the launching stream, launched without programmatic dependent
    # launch (with it a kernel may start before the previous one ends, across the events), so
    # each step is timed whole and alone
    sprob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, I_pad, renormalize=cfg.renormalize,
                             activation=cfg.activation, num_shared=cfg.num_shared, fp8=cfg.fp8,
                             input_scale=s_in, activation_scale=cfg.activation_scale, pdl=False)
    names = ["route", "align"] + (["quant_act"] if cfg.block128 else []) + ["permute", "gemm1", "gemm2", "combine"]
    per = {n: [] for n in names}

    def stages():
        moe.stage_route(sprob, logits, ws)
        moe.stage_align(sprob, ws)
        if cfg.block128:
            moe.stage_quant_act(sprob, hidden, ws)
        moe.stage_permute(sprob, hidden, ws)
        moe.stage_gemm1(sprob, hidden, w13p, ws, s13)
        moe.stage_gemm2(sprob, w2p, ws, s2)
        moe.stage_combine(sprob, out, ws)

    # one untimed pass first: small batches' forwards fuse routing, align and permute into
    # one kernel, so the separate kernels load (lazily) on their first launch here
    stages()
    torch.cuda.synchronize(dev)
    for _ in range(steps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        evs[0].record(stream)
        k = 0
        moe.stage_route(sprob, logits, ws); k += 1; evs[k].record(stream)
        moe.stage_align(sprob, ws); k += 1; evs[k].record(stream)
        if cfg.block128:
            moe.stage_quant_act(sprob, hidden, ws); k += 1; evs[k].record(stream)
        moe.stage_permute(sprob, hidden, ws); k += 1; evs[k].record(stream)
        moe.stage_gemm1(sprob, hidden, w13p, ws, s13); k += 1; evs[k].record(stream)
        moe.stage_gemm2(sprob, w2p, ws, s2); k += 1; evs[k].record(stream)
        moe.stage_combine(sprob, out, ws); k += 1; evs[k].record(stream)
        torch.cuda.synchronize(dev)
        for i, n in enumerate(names):
            per[n].append(evs[i].elapsed_time(evs[i + 1]))
    kernel_ms = {n: statistics.mean(v) for n, v in per.items()}

    # e2e through the public API with host buffers (pinned), copies inside the timed region
    h_hidden = inp["hidden"].pin_memory()
    h_logits = inp["logits"].pin_memory()
    h_out = torch.empty_like(inp["hidden"]).pin_memory()
    for _ in range(max(1, warmup // 2)):
        moe.moe_forward_host(prob, h_hidden, h_logits, w13p, w2p, h_out, ws, s13, s2)
    barrier(world)
    torch.cuda.synchronize(dev)
    e2e_ms = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        moe.moe_forward_host(prob, h_hidden, h_logits, w13p, w2p, h_out, ws, s13, s2)
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms.append(a.elapsed_time(b))
    barrier(world)
    e2e_total = max_over_ranks(sum(e2e_ms), world)

    # routing statistics for the algorithmic byte counts
    ids = moe.read_workspace(prob, ws)["topk_ids"].cpu().numpy()
    return {
        "total_ms": total_ms, "step_ms": step_ms, "kernel_ms": kernel_ms, "clocks": clocks,
        "e2e_total_ms": e2e_total, "ids": ids, "inp": inp,
        "h2d": h_hidden.numel() * 2 + h_logits.numel() * 4, "d2h": h_out.numel() * 2,
        # one kernel per stage, except align (three kernels above one 2048-pair chunk) and
        # the 8-bit formats' GEMM1 with a separate activation quantisation (block-128 FP8 and
        # MXFP8: the GEMM, then the quantisation)
        "launches_per_step": len(names) + (2 if cfg.T * cfg.k_total > 2048 else 0) +
                             (1 if cfg.block128 or cfg.mx else 0),
    }


def _gemm1_traffic(cfg: MoeConfig, g1_bytes: float):
    """DRAM bytes per GEMM1 launch scaled from the ncu capture, or None if the kernel
    source changed since (or the workload does not run that kernel)."""
    import hashlib
    src = os.path.join(ROOT, "mixture_experts_expert_topk_b200", "csrc", GEMM1_TRAFFIC["source"])
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:12]
    if cfg.fp8 or GEMM1_TRAFFIC["ratio"] is None or sha != GEMM1_TRAFFIC["source_sha256"]:  # bf16 capture
        return None
    return g1_bytes * GEMM1_TRAFFIC["ratio"]


def cpu_baseline(cfg: MoeConfig, inp, budget_s: float, tokens_hint: int):
    """Time the CPU oracle, as it stands, on the first tokens of the workload."""
    from oracle import moe_oracle as O

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    hb, lg = bits(inp["hidden"]), inp["logits"].numpy()
    w13b, w2b = bits(inp["w13"]), bits(inp["w2"])
    n = max(1, min(cfg.T, tokens_hint))
    tok = np.arange(n)
    if cfg.mx or cfg.nv:
        # quantise only the experts the sampled tokens use (the others do not enter the sample)
        ids, _ = O.route(lg[tok], cfg.topk, cfg.renormalize, cfg.num_shared)
        used = sorted(set(int(e) for e in ids.reshape(-1)))
        if cfg.nv:
            fp8w = O.quantize_weights_nvfp4(w13b, w2b, experts=used)
            s_in = np.float32(np.abs(O.bf16_bits_to_f32(hb)).max() / np.float32(2688))
        else:
            fp8w = O.quantize_weights_mxfp8(w13b, w2b, experts=used)
    elif cfg.per_tensor:
        fp8w = O.quantize_weights_fp8_per_tensor(w13b, w2b)
        s_in = np.float32(np.abs(O.bf16_bits_to_f32(hb)).max() / np.float32(448))
    elif cfg.fp8:
        fp8w = O.quantize_weights_fp8(w13b, w2b)
    t0 = time.perf_counter()
    if cfg.nv:
        O.moe_forward_nvfp4(hb, lg, *fp8w, s_in, np.float32(cfg.activation_scale), topk=cfg.topk,
                            renormalize=cfg.renormalize, activation=cfg.activation, num_shared=cfg.num_shared,
                            tokens=tok)
    elif cfg.mx:
        O.moe_forward_mxfp8(hb, lg, *fp8w, topk=cfg.topk, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, tokens=tok)
    elif cfg.per_tensor:
        O.moe_forward_fp8_per_tensor(hb, lg, *fp8w, s_in, cfg.activation_scale, topk=cfg.topk,
                                     renormalize=cfg.renormalize, activation=cfg.activation,
                                     num_shared=cfg.num_shared, tokens=tok)
    elif cfg.fp8:
        O.moe_forward_fp8(hb, lg, *fp8w, topk=cfg.topk, renormalize=cfg.renormalize,
                          activation=cfg.activation, num_shared=cfg.num_shared, tokens=tok)
    else:
        O.moe_forward(hb, lg, w13b, w2b, topk=cfg.topk, renormalize=cfg.renormalize,
                      activation=cfg.activation, num_shared=cfg.num_shared, tokens=tok)
    dt = time.perf_counter() - t0
    flops = cfg.flops() * n / cfg.T
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} of {cfg.T} tokens (routing, both GEMMs, combine), float64 NumPy",
            "seconds": dt}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="prefill", choices=sorted(CONFIGS))
    ap.add_argument("--cpu-tokens", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the kernels from the host each step instead of replaying a CUDA graph")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.impl == "reference":
        # the reference arm runs on rank 0's host cores only; other ranks exit at once
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank, local = int(os.environ.get("RANK", "0")), 0
    else:
        world, rank, local = _dist_setup(args.gpus)
    flops = cfg.flops()
    metric = "fused MoE layer forward throughput (TFLOP/s; us/call in ms_per_step)"
    base = {"metric": metric, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("nvfp4_e2m1" if cfg.nv else ("mxfp8_e4m3" if cfg.mx else "fp8_e4m3")) if cfg.fp8 else "bf16",
            "data": "synthetic"}

    if args.impl == "reference":
        if rank != 0:
            return
        inp = make_inputs(cfg, seed=0)
        times, vals = [], []
        per_step = max(8, args.cpu_tokens // 8)   # a few seconds of host work per step
        for _ in range(args.warmup):
            cpu_baseline(cfg, inp, 0, per_step)
        for _ in range(args.steps):
            r = cpu_baseline(cfg, inp, 0, per_step)
            times.append(r["seconds"])
            vals.append(r["value"])
        v = sum(vals) / len(vals)
        line = dict(base)
        line.update({"impl": "reference", "value": v, "n_gpus": world,
                     "ms_per_step": 1000.0 * sum(times) / len(times),
                     "config": {"workload": _workload_name(cfg),
                                "sample_tokens": per_step, "l2": "n/a (host)"},
                     "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": r["cores"],
                                      "kind": "oracle", "sample": r["sample"]},
                     "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                             "d2h_bytes_per_step": 0},
                     "gpu_launches": 0})
        print(json.dumps(line))
        return

    r = run_ours(cfg, args.steps, args.warmup, world, rank, local, args)
    ms_per_step = r["total_ms"] / args.steps
    value = flops * world / (r["total_ms"] / args.steps / 1e3) / 1e12
    e2e_value = flops * world / (r["e2e_total_ms"] / args.steps / 1e3) / 1e12
    hbm_peak, tc_peak, peak_kind = _peaks()
    elt = 1 if cfg.fp8 else 2
    n_touched, w13_bytes, w2_bytes = touched_expert_bytes(r["ids"], cfg, elt)
    if cfg.mx:  # one E8M0 byte per 32 weights
        w13_bytes, w2_bytes = w13_bytes * 33 // 32, w2_bytes * 33 // 32
    if cfg.nv:  # half a byte per weight plus one E4M3 byte per 16
        w13_bytes, w2_bytes = w13_bytes * 9 // 16, w2_bytes * 9 // 16
    P = cfg.T * cfg.k_total
    # GEMM1 algorithmic bytes per launch: touched w13, hidden rows read once, act written
    act_elt = 2 if (cfg.mx or cfg.nv or cfg.block128) else elt  # GEMM1 writes bf16 before re-quantising
    x_elt = 0.5625 if cfg.nv else elt                            # the GEMM1 input rows read once
    g1_bytes = w13_bytes + cfg.T * cfg.H * x_elt + P * cfg.I * act_elt
    g1_ms = r["kernel_ms"]["gemm1"]
    g1_gbs = g1_bytes / (g1_ms / 1e3) / 1e9
    g1_flops = 2.0 * P * cfg.H * cfg.N1
    g1_tflops = g1_flops / (g1_ms / 1e3) / 1e12
    # the binding roof of GEMM1: tensor cores when its arithmetic intensity exceeds the
    # ridge of the measured peaks (a contraction in 8-bit types takes twice the bf16 peak)
    tc_dtype_peak = tc_peak * (2.0 if cfg.fp8 else 1.0)
    tensor_bound = g1_flops / g1_bytes > tc_dtype_peak * 1e12 / (hbm_peak * 1e9)
    minimal_bytes = w13_bytes + w2_bytes + cfg.T * cfg.H * 2 * 2 + cfg.T * cfg.E * 4
    layer_gbs = minimal_bytes / (ms_per_step / 1e3) / 1e9
    line = dict(base)
    line.update({
        "value": value, "ms_per_step": ms_per_step,
        "us_per_call": ms_per_step * 1e3,
        "config": {"workload": _workload_name(cfg), "T": cfg.T, "H": cfg.H, "E": cfg.E_total,
                   "topk": cfg.k_total, "I": cfg.I,
                   "l2": "flushed before every step (512 MB write, outside the events)",
                   "cuda_graph": bool(args.graph)},
        "clocks": r["clocks"],
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches_per_step"] * args.steps,
        "roofline": ({"bound": "tensor", "kernel": "gemm1 (grouped up-GEMM + activation)",
                      "achieved": g1_tflops, "peak": tc_dtype_peak, "unit": "TFLOP/s",
                      "frac": g1_tflops / tc_dtype_peak, "traffic": _gemm1_traffic(cfg, g1_bytes),
                      "peak_source": f"{peak_kind} bf16_tflops" + (" x 2 (8-bit)" if cfg.fp8 else ""),
                      "algorithmic_flops_per_launch": g1_flops, "algorithmic_bytes_per_launch": g1_bytes,
                      "avg_launch_ms": g1_ms} if tensor_bound else
                     {"bound": "hbm", "kernel": "gemm1 (grouped up-GEMM + activation)",
                      "achieved": g1_gbs, "peak": hbm_peak, "unit": "GB/s",
                      "frac": g1_gbs / hbm_peak, "traffic": _gemm1_traffic(cfg, g1_bytes),
                      "peak_source": f"{peak_kind} hbm_gbs",
                      "algorithmic_bytes_per_launch": g1_bytes, "avg_launch_ms": g1_ms,
                      "gemm1_tflops": g1_tflops}),
        "layer_hbm": {"minimal_bytes": minimal_bytes, "achieved_gbs": layer_gbs,
                      "frac": layer_gbs / hbm_peak, "touched_experts": n_touched},
        "tensor_frac": value / tc_peak,
        "kernel_ms": r["kernel_ms"],
    })
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(cfg, r["inp"], 20.0, args.cpu_tokens)
        cb.pop("seconds")
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
