"""Benchmark of the DeepSeekMoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one whole layer forward (routing, permutation, both grouped GEMMs,
combine) over one batch of T synthetic tokens, through the C ABI
(moe_forward), inputs resident in HBM.  Under torchrun each rank runs its own
replica on its own GPU with its own batch (no collective on the data path:
the layer is data-parallel over tokens), so scaling is weak and the value is
the tokens of all ranks over the slowest rank's time.

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on the host cores instead, on a bounded token sample per step.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_CONFIG = "v3_bf16"

# DRAM traffic per launch of the GEMM1 kernel (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture at full size, summarised under
# profiles/), with the sha256 of the kernel's own sources at the time of the
# capture: once the kernel changes, the number no longer applies.
GEMM1_TRAFFIC = {"v3_bf16": {"bytes": 22114302208,
                             "sources": "010faa1cf13236c0641b9eedc7a0c136dd4ec0d13a452016d05365003a1863fd"}}
GEMM1_SOURCES = ("forward_moe_route_b200/csrc/gemm_gu.cuh", "forward_moe_route_b200/csrc/gemm.cuh",
                 "forward_moe_route_b200/csrc/common.cuh")


def sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in GEMM1_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm1_traffic(cfg):
    rec = GEMM1_TRAFFIC.get(cfg.name)
    if not rec or rec["sources"] != sources_sha():
        return None
    return rec["bytes"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def fp8_gemm_probe():
    """A measured denominator for the FP8 GEMMs beside the nominal 2 x bf16:
    a cuBLAS E4M3 GEMM (torch._scaled_mm, 8192^3, bf16 out) timed as a burst,
    best of 10 with CUDA events.  Returns (TFLOP/s, None) or (None, reason)."""
    import torch
    try:
        n = 8192
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        one = torch.ones((), device="cuda")

        def run():
            return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

        for _ in range(3):
            run()
        torch.cuda.synchronize()
        best = None
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
        del a, b
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12, None
    except Exception as exc:  # the probe is context only; the run goes on without it
        return None, f"{type(exc).__name__}: {exc}"[:200]


def workload_name(cfg):
    gate = "sigmoid+bias" if cfg.bias_half_range is not None else cfg.gate
    return (f"DeepSeekMoE layer forward ({cfg.name}): T={cfg.T} d={cfg.d} "
            f"{cfg.n_shared} shared + {cfg.n_routed} routed SwiGLU experts of width {cfg.inter}, "
            f"top-{cfg.top_k}, {gate}, groups {cfg.n_group}/{cfg.topk_group}, "
            f"{'renorm x' + str(cfg.route_scale) if cfg.renorm else 'no renorm'}, {cfg.dtype}")


def config_dict(cfg, n):
    return {"workload": workload_name(cfg), "T": cfg.T, "d": cfg.d, "n_shared": cfg.n_shared,
            "n_routed": cfg.n_routed, "top_k": cfg.top_k, "inter": cfg.inter, "gate": cfg.gate,
            "n_group": cfg.n_group, "topk_group": cfg.topk_group, "renorm": cfg.renorm,
            "route_scale": cfg.route_scale, "tokens_per_gpu": cfg.T,
            "global_tokens": cfg.T * n,
            "parallelism": f"token batches, one replica per GPU x{n}",
            "l2": "inputs larger than L2 (expert weights and x exceed the 126 MB L2)"}


# ----------------------------------------------------------------------------- ranks
def token_shard(T: int, rank: int, world: int):
    """[lo, hi) of the tokens rank `rank` owns when a batch of T is split over `world`."""
    base, extra = divmod(T, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device) -> float:
    """The maximum of `value` over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks
def visible_gpu(local: int) -> str:
    """nvidia-smi's id of this rank's GPU: entry `local` of CUDA_VISIBLE_DEVICES
    (an index or a UUID, both of which nvidia-smi -i accepts), else `local`."""
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    return vis[local] if local < len(vis) else str(local)


class ClockSampler:
    """nvidia-smi samples of this GPU's clocks while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle leg
class OracleSample:
    """The fp64 oracle on a bounded token sample of the workload (CPU baseline).

    One step routes `S` sampled tokens and evaluates their layer output with
    the oracle as it stands.  Expert weights are regenerated once (synthetic
    input generation, not timed) and kept as stored bf16/fp32 values; the
    oracle's widening to float64 is part of the timed work."""

    def __init__(self, cfg, n_tokens: int, zipf_offsets=None):
        import numpy as np

        from synth import recipes
        self.np = np
        self.cfg = cfg
        T = cfg.T
        self.tokens = [int(i * T // n_tokens) for i in range(n_tokens)]
        self.x = recipes.host_x(cfg, rows=self.tokens)
        self.w_r = recipes.host_router(cfg, zipf_offsets)
        self.bias = recipes.host_bias(cfg)
        # experts the sample touches (by the oracle's own routing), bits kept resident
        from oracle import moe_oracle as mo
        r = mo.route(self.x, self.w_r, self.bias, gate=cfg.gate, top_k=cfg.top_k,
                     n_group=cfg.n_group, topk_group=cfg.topk_group, renorm=cfg.renorm,
                     route_scale=cfg.route_scale)
        need = set(range(cfg.n_shared)) | {cfg.n_shared + int(j) for j in np.unique(r["idx"])}
        self.bits = {e: recipes.host_expert_bits(cfg, e) for e in sorted(need)}

    def _expert(self, e):
        np = self.np
        gu, dn = self.bits[e]
        I = self.cfg.inter
        if gu.dtype == np.uint16:
            from synth import bf16_bits_to_f64
            gu64, dn64 = bf16_bits_to_f64(gu), bf16_bits_to_f64(dn)
        else:
            gu64, dn64 = gu.astype(np.float64), dn.astype(np.float64)
        return gu64[:I], gu64[I:], dn64

    def step(self):
        from oracle import moe_oracle as mo
        c = self.cfg
        t0 = time.perf_counter()
        mo.moe_forward(self.x, self.w_r, self.bias, self._expert, n_shared=c.n_shared,
                       gate=c.gate, top_k=c.top_k, n_group=c.n_group, topk_group=c.topk_group,
                       renorm=c.renorm, route_scale=c.route_scale)
        return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_size(cfg):
    """Tokens per oracle step, sized so a step widens about 1.2e9 stored weight
    elements to float64 (the oracle's dominant cost: every expert a sampled
    token reaches is read whole) -- about 10 s on 16 host cores at the V3
    shape (3 tokens), all 64 experts for the 16B shape (64 tokens)."""
    per_expert = 3 * cfg.d * cfg.inter
    experts = max(1, int(1.2e9 // per_expert))
    if experts >= cfg.n_routed + cfg.n_shared:
        return 64
    return max(1, min(64, (experts - cfg.n_shared) // cfg.top_k))


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    S = oracle_sample_size(cfg)
    samp = OracleSample(cfg, S, load_zipf(cfg))
    for _ in range(args.warmup):
        samp.step()
    times = [samp.step() for _ in range(args.steps)]
    total = sum(times)
    value = S * args.steps / total
    cores = blas_threads()
    line = {"impl": "reference", "metric": "MoE-layer tokens/s", "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{S} tokens per step (strided over T={cfg.T}), "
                                       f"routing + all expert FFNs in fp64"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def load_zipf(cfg):
    if not cfg.zipf:
        return None
    import numpy as np
    path = os.path.join(ROOT, "tests", "golden", f"zipf_offsets_{cfg.name.split('@')[0]}.txt")
    return np.loadtxt(path, dtype=np.float64)


# ----------------------------------------------------------------------------- GPU leg
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    import forward_moe_route_b200 as moe
    from synth import recipes

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    desc = moe.desc_from_config(cfg)
    inp = recipes.device_inputs(cfg, "cuda", load_zipf(cfg))
    if cfg.dtype == "e4m3":
        # offline 128x128 block quantisation of the expert weights (not timed)
        E, I, d = cfg.n_experts, cfg.inter, cfg.d
        gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
        gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
        moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
        inp["w_gu"] = gq
        dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
        ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
        moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
        inp["w_down"] = dq
        inp["w_gu_scale"], inp["w_down_scale"] = gs, ds
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    fp8_probe = fp8_gemm_probe() if cfg.dtype == "e4m3" else (None, None)
    ws = moe.workspace(desc)
    h = torch.empty(cfg.T, cfg.d, dtype=inp["x"].dtype, device="cuda")
    stream = torch.cuda.current_stream()

    def step(x=None):
        moe.moe_forward(desc, inp["x"] if x is None else x, None, inp["w_r"], inp["bias"],
                        inp["w_gu"], inp.get("w_gu_scale"), inp["w_down"],
                        inp.get("w_down_scale"), h, None, None, ws, stream)

    for _ in range(args.warmup):
        step()
    st = moe.moe_last_device_status()
    if st != moe.OK:
        raise SystemExit(f"device status after warm-up: {moe.moe_status_string(st)}")

    # ---- timed region: K steps, events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for row in ev:            # torch creates its events lazily, at the first record
        for e in row:
            e.record(stream)
    clocks = ClockSampler(visible_gpu(local))
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    # ---- stage pass: the same K steps again, with the library's stage events
    # (moe_trace_events) for the per-stage times and the GEMM roofline.  It is
    # kept apart from the timed steps because an event between two launches
    # costs the programmatic overlap at that boundary (0.4 ms of a 13.5 ms V3
    # step, 29 of 76 us on the tiny layer).
    barrier()
    torch.cuda.synchronize()
    t_tr0 = torch.cuda.Event(enable_timing=True)
    t_tr1 = torch.cuda.Event(enable_timing=True)
    t_tr0.record(stream)
    for i in range(args.steps):
        moe.moe_trace_events(ev[i])
        step()
    moe.moe_trace_events(None)
    t_tr1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    st = moe.moe_last_device_status()
    if st != moe.OK:
        raise SystemExit(f"device status after the timed region: {moe.moe_status_string(st)}")
    ms = t_start.elapsed_time(t_end)
    ms_traced = max_over_ranks(t_tr0.elapsed_time(t_tr1), "cuda") / args.steps
    stages = {"route": [], "permute": [], "gemm1_swiglu": [], "gemm2_scatter": [],
              "combine": []}
    for e in ev:
        stages["route"].append(e[0].elapsed_time(e[1]))
        stages["permute"].append(e[1].elapsed_time(e[2]))
        stages["gemm1_swiglu"].append(e[2].elapsed_time(e[3]))
        stages["gemm2_scatter"].append(e[3].elapsed_time(e[4]))
        stages["combine"].append(e[4].elapsed_time(e[5]))
    stage_ms = {k: sum(v) / len(v) for k, v in stages.items()}
    ms = max_over_ranks(ms, "cuda")

    # ---- end to end through the public API: every step copies its x in from
    # pinned host memory and its h back out.  Three streams, two buffers: the
    # copy-in of step i+1 and the copy-out of step i-1 overlap step i's layer.
    x_host = inp["x"].cpu().pin_memory()
    h_hosts = [torch.empty(h.shape, dtype=h.dtype).pin_memory() for _ in range(2)]
    x_devs = [torch.empty_like(inp["x"]) for _ in range(2)]
    h_devs = [torch.empty_like(h) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "done", "out")}

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev["done"][b])        # step i-2 has read x_devs[b]
            x_devs[b].copy_(x_host, non_blocking=True)
            ev["in"][b].record(s_in)
        stream.wait_event(ev["in"][b])
        if i >= 2:
            stream.wait_event(ev["out"][b])           # step i-2's h has left h_devs[b]
        moe.moe_forward(desc, x_devs[b], None, inp["w_r"], inp["bias"], inp["w_gu"],
                        inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"),
                        h_devs[b], None, None, ws, stream)
        ev["done"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["done"][b])
            h_hosts[b].copy_(h_devs[b], non_blocking=True)
            ev["out"][b].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e2e_steps = max(3, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, "cuda")
    x_host_bytes = x_host.numel() * x_host.element_size()
    h_host_bytes = h_hosts[0].numel() * h_hosts[0].element_size()

    ms_step = ms / args.steps
    tokens_s = cfg.T * world / (ms_step * 1e-3)
    pk = peaks()
    gemm_flops = cfg.expert_gemm_flops()
    g1 = stage_ms["gemm1_swiglu"] * 1e-3
    g2 = stage_ms["gemm2_scatter"] * 1e-3
    gemm_tflops = gemm_flops / (g1 + g2) / 1e12
    g1_tflops = gemm_flops * 2 / 3 / g1 / 1e12
    # a contraction takes the peak of its own dtype: measured bf16 x the nominal ratio
    # (fp8 = 2 x bf16, tf32 = 0.5 x bf16)
    ratio = {"bf16": 1.0, "e4m3": 2.0, "f32": 0.5}[cfg.dtype]
    peak = pk["bf16_tflops_sustained"] * ratio
    out = None
    if rank == 0:
        route_bytes = (cfg.T * cfg.d * 2 + cfg.n_routed * cfg.d * 2 + cfg.T * cfg.n_routed * 4 * 2)
        perm_bytes = cfg.T * cfg.d * 2 + cfg.rows_routed * cfg.d * 2
        comb_bytes = cfg.T * (cfg.top_k + cfg.n_shared) * cfg.d * 2 + 2 * cfg.T * cfg.d * 2
        rpc_ms = stage_ms["route"] + stage_ms["permute"] + stage_ms["combine"]
        rpc_gbs = (route_bytes + perm_bytes + comb_bytes) / (rpc_ms * 1e-3) / 1e9
        out = {
            "metric": "MoE-layer tokens/s", "value": tokens_s, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": config_dict(cfg, world),
            "grouped_gemm_tflops": gemm_tflops,
            "grouped_gemm_frac_of_peak": {
                "dtype_peak": cfg.dtype,
                "measured_sustained": gemm_tflops / (pk["bf16_tflops_sustained"] * ratio),
                "measured_burst": gemm_tflops / (pk["bf16_tflops"] * ratio),
                "spec_dense": gemm_tflops / (2250.0 * ratio)},
            "stages_ms": stage_ms,
            "stage_pass_ms_per_step": ms_traced,
            "stage_timing": "stage events (and the GEMM rooflines) from a second pass of the "
                            "same K steps right after the timed steps; the events cost the "
                            "launch overlap at five boundaries, so that pass runs at "
                            "stage_pass_ms_per_step",
            "route_permute_combine_gbs": rpc_gbs,
            "route_permute_combine_frac_of_hbm": rpc_gbs / pk["hbm_gbs"],
            "route_permute_combine_frac_of_8tbs": rpc_gbs / 8000.0,
            "roofline": {"kernel": "grouped GEMM 1 (gate/up + SwiGLU epilogue)",
                         "bound": "tensor", "achieved": g1_tflops, "peak": peak,
                         "unit": "TFLOP/s", "frac": g1_tflops / peak,
                         "traffic": gemm1_traffic(cfg),
                         "peak_source": f"{pk['source']} bf16 sustained x {ratio} "
                                        f"(nominal {cfg.dtype}/bf16 ratio)"},
            "roofline_gemm2": {"kernel": "grouped GEMM 2 (down + weighted scatter)",
                               "bound": "tensor",
                               "achieved": gemm_flops / 3 / g2 / 1e12, "peak": peak,
                               "unit": "TFLOP/s", "frac": gemm_flops / 3 / g2 / 1e12 / peak},
            "e2e": {"value": cfg.T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": x_host_bytes, "d2h_bytes_per_step": h_host_bytes,
                    "overlap": "copy-in of step i+1 and copy-out of step i-1 overlap step i"},
            "gpu_launches": moe.moe_forward_launch_count(desc) * args.steps,
            "clocks": clk,
        }
    if out is not None and cfg.dtype == "e4m3":
        tf, why = fp8_probe
        out["fp8_gemm_probe"] = (
            {"tflops_burst": tf, "how": "cuBLAS E4M3 GEMM, torch._scaled_mm 8192^3, best of 10",
             "grouped_gemm_frac": gemm_tflops / tf} if tf else {"unavailable": why})
    if world > 1:
        dist.destroy_process_group()
    return out


# ----------------------------------------------------------------------------- backward leg
def backward_flops(cfg):
    """FLOPs of the backward's expert GEMMs per step, split into the algorithmic
    part (dz, du, dW_down, dW_gu: 12 d I per active row) and the recomputation
    of the pre-activations a, b (4 d I per active row), plus the router (4 T N d)."""
    rows = cfg.T * (cfg.top_k + cfg.n_shared)
    return {"algorithmic": 12.0 * cfg.d * cfg.inter * rows,
            "recompute": 4.0 * cfg.d * cfg.inter * rows,
            "router": 4.0 * cfg.T * cfg.n_routed * cfg.d}


def run_backward(args, cfg):
    """One layer backward per step (moe_backward: routing, permutation, the
    recomputed pre-activations, dz with the SwiGLU backward, du, the gate and
    affinity backward, dW_down, dW_gu, dW_r), inputs resident in HBM.  With
    --saved the step is moe_backward_saved, which reads the pre-activations
    moe_forward_save kept instead of recomputing them; for an E4M3 layer
    (--config v3_fp8) it is moe_backward_fp8, the backward with FP8 GEMMs."""
    import torch

    import forward_moe_route_b200 as moe
    import synth
    from synth import recipes
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    fp8 = cfg.dtype == "e4m3"
    if cfg.dtype not in ("bf16", "e4m3"):
        raise SystemExit("the backward is built for bf16 and E4M3 layers")
    if fp8 and args.saved:
        raise SystemExit("--saved is for bf16 layers")
    desc = moe.desc_from_config(cfg)
    inp = recipes.device_inputs(cfg, "cuda", load_zipf(cfg))
    dh32 = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    synth.dev_fill_normal(dh32, 1.0, cfg.seed, 6)
    dh = dh32.to(torch.bfloat16)
    del dh32
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    dx = torch.empty(cfg.T, d, dtype=torch.bfloat16, device="cuda")
    gdt = torch.bfloat16 if (args.bf16_grads or fp8) else torch.float32
    dwr = torch.empty(N, d, dtype=gdt, device="cuda")
    dwgu = torch.empty(E, 2 * I, d, dtype=gdt, device="cuda")
    dwd = torch.empty(E, d, I, dtype=gdt, device="cuda")
    ws = moe.backward_fp8_workspace(desc) if fp8 else moe.backward_workspace(desc)
    stream = torch.cuda.current_stream()
    fwd_cost = None
    if fp8:
        # E4M3 codes and 128x128 block scales of the weights and of their
        # transposes (offline, like the forward's weight quantisation)
        W8 = moe.fp8_backward_weights(inp["w_gu"], inp["w_down"])
        del inp["w_gu"], inp["w_down"]
        torch.cuda.empty_cache()

        def step():
            moe.moe_backward_fp8(desc, inp["x"], inp["w_r"], inp["bias"], *W8, dh, dx, dwr, dwgu,
                                 dwd, ws, stream)
    elif args.saved:
        # the forward keeps a | b (moe_forward_save, outside the timed region);
        # its cost over the plain forward is timed alongside
        ab = torch.empty(moe.moe_saved_ab_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
        fws = moe.workspace(desc)
        h = torch.empty(cfg.T, d, dtype=torch.bfloat16, device="cuda")

        def fwd(save):
            if save:
                moe.moe_forward_save(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                                     inp["w_down"], h, None, None, ab, fws, stream)
            else:
                moe.moe_forward(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"], None,
                                inp["w_down"], None, h, None, None, fws, stream)

        # blocks of 5 forwards in the order A B B A A B B A after a warm-up,
        # so that neither form gets the cooler GPU; medians of the blocks
        for _ in range(6):
            fwd(False)
        blocks = {False: [], True: []}
        for save in (False, True, True, False, False, True, True, False):
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(5):
                fwd(save)
            f1.record(stream)
            torch.cuda.synchronize()
            blocks[save].append(f0.elapsed_time(f1) / 5)
        fwd_cost = {"forward_ms": statistics.median(blocks[False]),
                    "forward_save_ms": statistics.median(blocks[True]),
                    "blocks": "median of 4 blocks of 5 steps each, order ABBAABBA"}
        del fws

        def step():
            moe.moe_backward_saved(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"],
                                   inp["w_down"], dh, ab, dx, dwr, dwgu, dwd, ws,
                                   bf16_grads=args.bf16_grads, stream=stream)
    if not fp8 and not args.saved:
        call = moe.moe_backward_bf16_grads if args.bf16_grads else moe.moe_backward

        def step():
            call(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"], inp["w_down"], dh, dx,
                 dwr, dwgu, dwd, ws, stream)

    for _ in range(args.warmup):
        step()
    st = moe.moe_last_device_status()
    if st != moe.OK:
        raise SystemExit(f"device status after warm-up: {moe.moe_status_string(st)}")
    clocks = ClockSampler(visible_gpu(int(os.environ.get("LOCAL_RANK", "0"))))
    torch.cuda.synchronize()
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    st = moe.moe_last_device_status()
    if st != moe.OK:
        raise SystemExit(f"device status after the timed region: {moe.moe_status_string(st)}")
    ms = e0.elapsed_time(e1) / args.steps
    fl = backward_flops(cfg)
    pk = peaks()
    done = fl["algorithmic"] + (0.0 if args.saved else fl["recompute"]) + fl["router"]
    tflops = done / (ms * 1e-3) / 1e12
    # FP8 GEMMs against twice the measured bf16 rate (the sheet's FP8 : bf16 ratio)
    peak = pk["bf16_tflops_sustained"] * (2.0 if fp8 else 1.0)
    return {"metric": "MoE-layer backward tokens/s", "value": cfg.T / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic", "config": config_dict(cfg, 1),
            "weight_gradients": "bf16" if (args.bf16_grads or fp8) else "fp32",
            "gemm_precision": "FP8 E4M3 (gating GEMMs bf16)" if fp8 else "bf16",
            "pre_activations": "saved by the forward" if args.saved else "recomputed",
            "forward_cost": fwd_cost,
            "backward_gemm_tflops": tflops,
            "backward_gemm_frac_of_peak": {
                ("measured_sustained_x2_fp8" if fp8 else "measured_sustained"): tflops / peak,
                "spec_dense": tflops / (4500.0 if fp8 else 2250.0)},
            "backward_flops": fl,
            "algorithmic_tflops": (fl["algorithmic"] + fl["router"]) / (ms * 1e-3) / 1e12,
            "gpu_launches": (moe.moe_backward_fp8_launch_count(desc) if fp8 else
                             moe.moe_backward_launch_count(desc) - (1 if args.saved else 0))
            * args.steps,
            "clocks": clk}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--T", type=int, default=None, help="override the token count")
    ap.add_argument("--n-routed", type=int, default=None,
                    help="override the routed expert count (smaller profiling cases)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer backward (moe_backward) instead of the forward")
    ap.add_argument("--bf16-grads", action="store_true",
                    help="with --backward: weight gradients in bf16 (moe_backward_bf16_grads)")
    ap.add_argument("--saved", action="store_true",
                    help="with --backward: the pre-activations kept by moe_forward_save "
                    "(moe_backward_saved) instead of recomputed")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    from synth import recipes
    cfg = recipes.CONFIGS[args.config]
    if args.T is not None:
        cfg = cfg.with_T(args.T)
    if args.n_routed is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, n_routed=args.n_routed,
                                  name=f"{cfg.name}@N{args.n_routed}")
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.backward:
        print(json.dumps(run_backward(args, cfg)), flush=True)
        return 0
    out = run_ours(args, cfg)
    if out is not None:
        if not args.no_cpu_baseline and args.gpus == 1:
            S = oracle_sample_size(cfg)
            samp = OracleSample(cfg, S, load_zipf(cfg))
            samp.step()
            t = [samp.step() for _ in range(2)]
            v = S * len(t) / sum(t)
            out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": blas_threads(),
                                   "kind": "oracle",
                                   "sample": f"{S} tokens (strided over T={cfg.T}), routing + "
                                             f"all expert FFNs in fp64, 2 timed steps"}
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
