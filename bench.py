#!/usr/bin/env python
"""QLoRA NF4 linear fwd+bwd benchmark on B200: tokens/s and TFLOP/s against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward and one backward pass of every QLoRA linear of the workload over one
batch of synthetic tokens (seeded, resident in HBM before timing):

    XA = X A^T, h = X deq(W0)^T + s XA B^T                (forward)
    dYB = dY B, dX = dY deq(W0) + s dYB A, dB, dA          (backward)

run as the six library stages (lora_down, dequant GEMM, lora_down, dequant GEMM (dX),
lora_grad x 2) with CUDA events between them on the launching stream, so the dominant
kernel's own duration is measured live.  L2 is flushed before every step, outside the events:
a 256 MiB write followed by a read of the same buffer, so no dirty line is left to write back.  One JSON line is printed by rank 0.

Multi-GPU (torchrun): every rank runs an independent replica on its own batch (the layer's
data path has no exchange step in one forward+backward); the step time is the max over ranks.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nf4_base_lora_blockwise_b200 import abi, linear, synth  # noqa: E402

DEFAULT_WORKLOAD = "q_proj_8b"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------------------------
# Work and traffic counts (algorithmic, per launch)
# ----------------------------------------------------------------------------------------------
def weight_stream_bytes(L):
    """HBM bytes of the packed NF4 weight: codes + absmax (fp32 or double-quantised)."""
    nk = L.N * L.K
    if L.double_quant:
        return nk // 2 + nk // 64 + 4 * math.ceil(nk / 64 / 256)
    return nk // 2 + 4 * (nk // 64)


def gemm_work(L, M, trans):
    """(flops, min HBM bytes) of one dequant GEMM launch (forward or dX)."""
    red, rows = (L.N, L.K) if trans else (L.K, L.N)
    flops = 2.0 * M * L.N * L.K + 2.0 * M * rows * L.r
    byts = weight_stream_bytes(L) + 2 * M * red + 2 * M * rows + 2 * M * L.r + 2 * rows * L.r
    return flops, byts


def step_flops(w):
    """Algorithmic flops of one step: fwd 2MNK + 2Mr(K+N), bwd 2MNK + 4Mr(K+N) per linear."""
    M = w.M
    return sum(4.0 * M * L.N * L.K + 6.0 * M * L.r * (L.K + L.N) for L in w.linears)


# ----------------------------------------------------------------------------------------------
# Clocks sampled during the timed region
# ----------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------------------------
class LinearState:
    """Device buffers of one QLoRA linear on M tokens, and its six timed stages."""

    def __init__(self, L, M, X, dY, W0, A, B, dev):
        self.L, self.M = L, M
        self.X, self.dY = X.to(dev), dY.to(dev)
        self.A, self.B = A.to(dev), B.to(dev)
        self.w = linear.nf4_pack(W0.to(dev), double_quant=L.double_quant)
        self.cw = self.w.c_struct()
        self.s = L.alpha / L.r
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.H = torch.empty((M, L.N), **bf)
        self.XA = torch.empty((M, L.r), **bf)
        self.sXA = torch.empty((M, L.r), **bf)
        self.dYB = torch.empty((M, L.r), **bf)
        self.sdYB = torch.empty((M, L.r), **bf)
        self.dX = torch.empty((M, L.K), **bf)
        self.dA = torch.empty((L.r, L.K), dtype=torch.float32, device=dev)
        self.dB = torch.empty((L.N, L.r), dtype=torch.float32, device=dev)
        self.ws = linear.alloc_workspace(M, L.N, L.K, L.r, dev)
        self.stage_names = ("lora_down_fwd", "gemm_fwd", "lora_down_bwd", "gemm_dx",
                            "lora_grad_dB", "lora_grad_dA")

    def stages(self, stream):
        M, L, p = self.M, self.L, lambda t: t.data_ptr()
        ws, wsb = p(self.ws), self.ws.numel()
        return (
            lambda: abi.qlora_lora_down(p(self.X), M, L.K, p(self.A), 1, L.r, self.s, p(self.XA),
                                        p(self.sXA), ws, wsb, stream),
            lambda: abi.qlora_nf4_gemm(p(self.X), self.cw, 0, p(self.B), p(self.sXA), M, L.r,
                                       p(self.H), stream),
            lambda: abi.qlora_lora_down(p(self.dY), M, L.N, p(self.B), 0, L.r, self.s,
                                        p(self.dYB), p(self.sdYB), ws, wsb, stream),
            lambda: abi.qlora_nf4_gemm(p(self.dY), self.cw, 1, p(self.A), p(self.sdYB), M, L.r,
                                       p(self.dX), stream),
            lambda: abi.qlora_lora_grad(p(self.dY), M, L.N, p(self.XA), L.r, self.s, p(self.dB),
                                        0, ws, wsb, stream),
            lambda: abi.qlora_lora_grad(p(self.X), M, L.K, p(self.dYB), L.r, self.s, p(self.dA),
                                        1, ws, wsb, stream),
        )


def build_states(w, dev, seed):
    inp = synth.make_inputs(w, seed=seed)
    if w.mlp:
        raise SystemExit("the MLP workload is benchmarked as its three projections: use "
                         "--workload mlp_8b_proj")
    return [LinearState(L, w.M, d["X"], d["dY"], d["W0"], d["A"], d["B"], dev)
            for L, d in zip(w.linears, inp["linears"])]


def run_steps(states, n, stream, flush, record):
    """Run n steps; per step and per stage, CUDA events on `stream`.  Returns
    (per-step ms list, {stage: [ms...]})."""
    per_step = []
    per_stage = {}
    for _ in range(n):
        # L2 flush: write 256 MiB, then read it back so the evicted lines are clean (the
        # write-back of the flush's own dirty lines must not land on the first timed kernel).
        flush.zero_()
        flush.max()
        evs = []
        calls = []
        for st in states:
            for name, fn in zip(st.stage_names, st.stages(stream.cuda_stream)):
                calls.append((f"{st.L.name}.{name}", fn))
        for name, fn in calls:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            evs.append((name, e))
            fn()
        end = torch.cuda.Event(enable_timing=True)
        end.record(stream)
        evs.append(("end", end))
        if record:
            per_stage.setdefault("_events", []).append(evs)
    torch.cuda.synchronize()
    if record:
        for evs in per_stage.pop("_events"):
            per_step.append(evs[0][1].elapsed_time(evs[-1][1]))
            for (name, a), (_, b) in zip(evs[:-1], evs[1:]):
                per_stage.setdefault(name, []).append(a.elapsed_time(b))
    return per_step, per_stage


def run_e2e(states, steps, dev):
    """The same metric through the public entry points qlora_linear_fwd / qlora_linear_bwd with
    host buffers: each step copies X and dY from pinned host memory, runs the layer, and copies
    h, dX, dA and dB back."""
    host = []
    for st in states:
        host.append({
            "X": st.X.cpu().pin_memory(), "dY": st.dY.cpu().pin_memory(),
            "H": torch.empty_like(st.H, device="cpu").pin_memory(),
            "dX": torch.empty_like(st.dX, device="cpu").pin_memory(),
            "dA": torch.empty_like(st.dA, device="cpu").pin_memory(),
            "dB": torch.empty_like(st.dB, device="cpu").pin_memory(),
        })
    h2d = sum(h["X"].numel() * 2 + h["dY"].numel() * 2 for h in host)
    d2h = sum(h["H"].numel() * 2 + h["dX"].numel() * 2 + h["dA"].numel() * 4 + h["dB"].numel() * 4
              for h in host)

    def one():
        for st, h in zip(states, host):
            st.X.copy_(h["X"], non_blocking=True)
            st.dY.copy_(h["dY"], non_blocking=True)
            linear.forward(st.X, st.w, st.A, st.B, st.L.alpha, H=st.H, XA=st.XA, ws=st.ws)
            linear.backward(st.dY, st.X, st.w, st.A, st.B, st.XA, st.L.alpha, dX=st.dX,
                            dA=st.dA, dB=st.dB, ws=st.ws)
            h["H"].copy_(st.H, non_blocking=True)
            h["dX"].copy_(st.dX, non_blocking=True)
            h["dA"].copy_(st.dA, non_blocking=True)
            h["dB"].copy_(st.dB, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        one()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps, h2d, d2h


def ncu_traffic(workload, stage):
    """DRAM bytes per launch of `stage` from the committed ncu capture (profiles/ncu_traffic.json),
    or None when there is none or the kernel sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(f"{workload}.{stage}")
        if not rec:
            return None
        m = hashlib.sha256()
        for name in rec["source_files"]:
            with open(os.path.join(ROOT, name), "rb") as g:
                m.update(g.read())
        return rec["traffic_bytes"] if m.hexdigest() == rec["source_sha256"] else None
    except (OSError, ValueError, KeyError):
        return None


def roofline(states, per_stage, peaks, workload):
    """Roofline of the dominant kernel (largest total time among the stages)."""
    totals = {k: sum(v) for k, v in per_stage.items()}
    name = max(totals, key=totals.get)
    lin_name, stage = name.split(".", 1)
    st = next(s for s in states if s.L.name == lin_name)
    ms = statistics.mean(per_stage[name])
    if stage.startswith("gemm"):
        flops, byts = gemm_work(st.L, st.M, stage == "gemm_dx")
    elif stage.startswith("lora_down"):
        C = st.L.K if stage.endswith("fwd") else st.L.N
        flops, byts = 2.0 * st.M * C * st.L.r, 2 * st.M * C + 4 * st.M * st.L.r
    else:
        C = st.L.N if stage.endswith("dB") else st.L.K
        flops, byts = 2.0 * st.M * C * st.L.r, 2 * st.M * C + 4 * C * st.L.r
    ai = flops / byts
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if stage.startswith("gemm") and ai >= ridge:
        ach = flops / (ms * 1e-3) / 1e12
        r = {"bound": "tensor", "achieved": round(ach, 2), "peak": peaks["bf16_tflops"],
             "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4)}
    else:
        ach = byts / (ms * 1e-3) / 1e9
        r = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": round(ach / peaks["hbm_gbs"], 4)}
    r.update({"kernel": name, "ms_per_launch": round(ms, 5), "flops_per_launch": flops,
              "bytes_per_launch": byts, "traffic": ncu_traffic(workload, stage),
              "peak_source": peaks["source"]})
    return r


# ----------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ----------------------------------------------------------------------------------------------
def oracle_sample(w, seed, rows_per_linear, threads_note=True):
    """Time the fp64 oracle: dequantise each W0 once (charged per step: once per batch of M
    tokens), then forward + backward on `rows_per_linear` sampled token rows.  Returns
    (seconds for the sample rows, seconds of one dequant per step, description)."""
    from oracle import nf4, qlora  # test infrastructure: only here and in the reference arm
    inp = synth.make_inputs(w, seed=seed)
    t_deq = 0.0
    t_rows = 0.0
    for L, d in zip(w.linears, inp["linears"]):
        Wf = d["W0"].float().numpy()
        t0 = time.perf_counter()
        am = nf4.block_absmax(Wf)
        if L.double_quant:
            q8, sc = nf4.double_quant(am.reshape(-1))
            eff = nf4.dq_effective_absmax(q8, sc).reshape(am.shape)
        else:
            eff = am
        q = nf4.pack_codes(nf4.choose_codes(Wf, eff))
        t1 = time.perf_counter()
        Wd = nf4.dequantize(q, eff, L.N, L.K).astype(np.float64)
        t2 = time.perf_counter()
        t_deq += t2 - t1
        rows = np.arange(min(rows_per_linear, w.M))
        X = d["X"][: len(rows)].float().numpy().astype(np.float64)
        dY = d["dY"][: len(rows)].float().numpy().astype(np.float64)
        A = d["A"].float().numpy().astype(np.float64)
        B = d["B"].float().numpy().astype(np.float64)
        t3 = time.perf_counter()
        qlora.forward(X, Wd, A, B, L.alpha)
        qlora.backward(dY, X, Wd, A, B, L.alpha)
        t_rows += time.perf_counter() - t3
        del t0
    desc = (f"fp64 oracle fwd+bwd on {rows_per_linear} token rows per linear of {w.name} "
            f"(M={w.M}), plus one deq(W0) per step charged per batch of M tokens; "
            f"quantisation not timed")
    return t_rows, t_deq, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, seed=0, rows=32):
    t_rows, t_deq, desc = oracle_sample(w, seed, rows)
    n = min(rows, w.M)
    per_token = t_rows / n + t_deq / w.M
    return {"value": round(1.0 / per_token, 2), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle", "sample": desc}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.workload(args.workload)
    # Calibrate: rows per step so the whole run stays within ~2 minutes.
    t_rows, t_deq, desc = oracle_sample(w, 0, 8)
    budget = 120.0 / max(1, args.steps + args.warmup)
    per_row = t_rows / min(8, w.M)
    rows = int(max(1, min(w.M, (budget - t_deq * 1.0 / max(1, w.M)) / max(per_row, 1e-9))))
    times = []
    for i in range(args.warmup + args.steps):
        tr, td, desc = oracle_sample(w, 0, rows)
        n = min(rows, w.M)
        if i >= args.warmup:
            times.append(tr + td * n / w.M)
    n = min(rows, w.M)
    tot = sum(times)
    value = args.steps * n / tot
    line = {
        "impl": "reference", "metric": "qlora_linear_fwd_bwd_tokens_per_s", "value": round(value, 3),
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * tot / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc.replace("32", str(n))},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w):
    c = {"workload": w.name, "M": w.M,
         "linears": [{"name": L.name, "K": L.K, "N": L.N, "r": L.r, "alpha": L.alpha,
                      "absmax": "double-quant" if L.double_quant else "fp32"} for L in w.linears],
         "l2": "flushed before every step (256 MiB write + read, outside the events)", "parallelism": "replicas"}
    return c


# ----------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    w = synth.workload(args.workload)
    states = build_states(w, dev, seed=rank)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    run_steps(states, args.warmup, stream, flush, record=False)
    if abi.qlora_device_error() != 0:
        raise SystemExit("device error word set during warm-up")

    sampler = ClockSampler(local)
    if not args.no_clocks and rank == 0:
        sampler.start()
        time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = abi.qlora_launch_counter()
    per_step, per_stage = run_steps(states, args.steps, stream, flush, record=True)
    torch.cuda.synchronize()
    launches = abi.qlora_launch_counter() - n0
    if dist:
        dist.barrier()
    clocks = sampler.stop() if (not args.no_clocks and rank == 0) else None
    if abi.qlora_device_error() != 0:
        raise SystemExit("device error word set during the timed region")

    total_ms = sum(per_step)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if dist:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    tokens = world * w.M * args.steps
    value = tokens / (total_ms * 1e-3)
    ms_per_step = total_ms / args.steps

    e2e_ms, h2d, d2h = run_e2e(states, args.e2e_steps, dev)
    te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if dist:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = world * w.M / (float(te.item()) * 1e-3)

    if rank == 0:
        peaks = _peaks()
        tflops = step_flops(w) / (ms_per_step * 1e-3) / 1e12
        line = {
            "metric": "qlora_linear_fwd_bwd_tokens_per_s",
            "value": round(value, 1),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) W0 packed to NF4, random LoRA)",
            "config": workload_config(w),
            "tflops": round(tflops, 2),
            "tflops_frac_of_peak": round(tflops / peaks["bf16_tflops"], 4),
            "stages_ms": {k: round(statistics.mean(v), 5) for k, v in per_stage.items()},
            "roofline": roofline(states, per_stage, peaks, w.name),
            "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
