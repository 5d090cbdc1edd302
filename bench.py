#!/usr/bin/env python
"""QLoRA NF4 linear fwd+bwd benchmark on B200: tokens/s and TFLOP/s against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward and one backward pass of every QLoRA linear of the workload over one
batch of synthetic tokens (seeded, resident in HBM before timing):

    XA = X A^T, h = X deq(W0)^T + s XA B^T                (forward)
    dYB = dY B, dX = dY deq(W0) + s dYB A, dB, dA          (backward)

run as the six library stages (lora_down, dequant GEMM, lora_down, dequant GEMM (dX),
lora_grad x 2; the MLP block adds the SwiGLU glue between its three linears).  The step is
captured once into a CUDA graph with timing events between the stages (recorded by the graph
on its own stream), and each timed step is one replay, so the dominant kernel's own duration
is measured live and host launch cost never appears as idle time (--eager launches every stage
from Python instead).  L2 is flushed before every step, outside the events: a 256 MiB write
followed by a read of the same buffer, so no dirty line is left to write back.  One JSON line
is printed by rank 0.

Multi-GPU (torchrun): every rank runs an independent replica on its own batch (the layer's
data path has no exchange step in one forward+backward); the step time is the max over ranks.
"""

import argparse
import copy
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


def gemm_work(L, M, trans, n_groups=1):
    """(flops, min HBM bytes) of one dequant GEMM launch (forward or dX).  With n adapters
    packed along W0's rows, every output row of the forward takes r extension columns and the
    dX extension runs over all n r."""
    red, rows = (L.N, L.K) if trans else (L.K, L.N)
    r_row = L.r * n_groups if trans else L.r
    flops = 2.0 * M * L.N * L.K + 2.0 * M * rows * r_row
    byts = (weight_stream_bytes(L) + 2 * M * red + 2 * M * rows + 2 * M * L.r * n_groups
            + 2 * rows * r_row)
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
    """Device buffers of one QLoRA linear on M tokens, and its timed stages: forward
    (lora_down, dequant GEMM) and backward (lora_down, dequant GEMM for dX, lora_grad x 2).
    X and dY may be buffers shared with other stages (the MLP block chains them).  With
    `groups` (adapter row counts) the linear is a packed-adapter layer: L.N is the stacked
    weight's rows, L.r each adapter's rank, A [n r, K] and B [N, r] stacked by adapter."""

    def __init__(self, L, M, X, dY, W0, A, B, dev, groups=None):
        self.L, self.M = L, M
        self.groups = list(groups) if groups else None
        self.R = L.r * (len(self.groups) if self.groups else 1)  # packed rank columns
        self.X, self.dY = X.to(dev), dY.to(dev)
        self.A, self.B = A.to(dev), B.to(dev)
        self.w = linear.nf4_pack(W0.to(dev), double_quant=L.double_quant)
        self.cw = self.w.c_struct()
        self.s = L.alpha / L.r
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.H = torch.empty((M, L.N), **bf)
        self.XA = torch.empty((M, self.R), **bf)
        self.sXA = torch.empty((M, self.R), **bf)
        self.dYB = torch.empty((M, self.R), **bf)
        self.sdYB = torch.empty((M, self.R), **bf)
        self.dX = torch.empty((M, L.K), **bf)
        self.dA = torch.empty((self.R, L.K), dtype=torch.float32, device=dev)
        self.dB = torch.empty((L.N, L.r), dtype=torch.float32, device=dev)
        self.ws = linear.alloc_workspace(M, L.N, L.K, self.R, dev)

    def twin(self):
        """The same linear (weights shared) with its own activation, output and scratch
        buffers, so two steps can be in flight at once."""
        t = copy.copy(self)
        for name in ("X", "dY", "H", "XA", "sXA", "dYB", "sdYB", "dX", "dA", "dB", "ws"):
            setattr(t, name, torch.empty_like(getattr(self, name)))
        return t

    def fwd_stages(self, stream):
        M, L, R, g, p = self.M, self.L, self.R, self.groups, lambda t: t.data_ptr()
        ws, wsb = p(self.ws), self.ws.numel()
        n = L.name
        return [
            (f"{n}.lora_down_fwd",
             lambda: abi.qlora_lora_down(p(self.X), M, L.K, p(self.A), 1, R, None, self.s,
                                         p(self.XA), p(self.sXA), ws, wsb, stream)),
            (f"{n}.gemm_fwd",
             lambda: abi.qlora_nf4_gemm(p(self.X), self.cw, 0, p(self.B), p(self.sXA), M, L.r,
                                        g, p(self.H), ws, wsb, stream)),
        ]

    def bwd_stages(self, stream):
        M, L, R, g, p = self.M, self.L, self.R, self.groups, lambda t: t.data_ptr()
        ws, wsb = p(self.ws), self.ws.numel()
        n = L.name
        return [
            (f"{n}.lora_down_bwd",
             lambda: abi.qlora_lora_down(p(self.dY), M, L.N, p(self.B), 0, R, g, self.s,
                                         p(self.dYB), p(self.sdYB), ws, wsb, stream)),
            (f"{n}.gemm_dx",
             lambda: abi.qlora_nf4_gemm(p(self.dY), self.cw, 1, p(self.A), p(self.sdYB), M, R,
                                        None, p(self.dX), ws, wsb, stream)),
            (f"{n}.lora_grad_dB",
             lambda: abi.qlora_lora_grad(p(self.dY), M, L.N, p(self.XA), L.r, g, self.s,
                                         p(self.dB), 0, ws, wsb, stream)),
            (f"{n}.lora_grad_dA",
             lambda: abi.qlora_lora_grad(p(self.X), M, L.K, p(self.dYB), R, None, self.s,
                                         p(self.dA), 1, ws, wsb, stream)),
        ]

    def forward(self):
        """The layer's forward through the public Python entry points."""
        if self.groups:
            linear.grouped_forward(self.X, self.w, self.A, self.B, self.groups, self.L.alpha,
                                   H=self.H, XA=self.XA, ws=self.ws)
        else:
            linear.forward(self.X, self.w, self.A, self.B, self.L.alpha, H=self.H, XA=self.XA,
                           ws=self.ws)

    def backward(self):
        if self.groups:
            linear.grouped_backward(self.dY, self.X, self.w, self.A, self.B, self.XA,
                                    self.groups, self.L.alpha, dX=self.dX, dA=self.dA,
                                    dB=self.dB, ws=self.ws)
        else:
            linear.backward(self.dY, self.X, self.w, self.A, self.B, self.XA, self.L.alpha,
                            dX=self.dX, dA=self.dA, dB=self.dB, ws=self.ws)


class CeState:
    """Device buffers of the LM head + cross-entropy on M tokens, in chunks: per step the label
    count, then for each chunk the forward GEMM into the logits buffer, the cross-entropy rows
    (token losses, gradient in place) and the dX GEMM, then the mean loss."""

    def __init__(self, L, M, X, labels, W0, chunk, dev):
        self.L, self.Mtot = L, M
        self.chunk = min(chunk, M)
        self.M, self.R, self.groups = self.chunk, 0, None  # tokens per GEMM launch
        self.X, self.labels = X.to(dev), labels.to(dev)
        self.w = linear.nf4_pack(W0.to(dev))
        self.cw = self.w.c_struct()
        self.z = torch.empty((self.chunk, L.N), dtype=torch.bfloat16, device=dev)
        self.tl = torch.empty(M, dtype=torch.float32, device=dev)
        self.cnt = torch.empty(64, dtype=torch.int32, device=dev)
        self.loss = torch.empty(1, dtype=torch.float32, device=dev)
        self.dX = torch.empty((M, L.K), dtype=torch.bfloat16, device=dev)
        n = abi.qlora_lm_head_ce_workspace_bytes(M, L.N, L.K, self.chunk)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)

    def twin(self):
        t = copy.copy(self)
        for name in ("X", "labels", "z", "tl", "cnt", "loss", "dX", "ws"):
            setattr(t, name, torch.empty_like(getattr(self, name)))
        return t

    def stages(self, stream):
        L, M, c, p = self.L, self.Mtot, self.chunk, lambda t: t.data_ptr()
        ws, wsb = p(self.ws), self.ws.numel()
        out = [("lm_head.ce_count",
                lambda: abi.qlora_cross_entropy_count(p(self.labels), M, L.N, p(self.cnt), stream))]
        for m0 in range(0, M, c):
            mc = min(c, M - m0)
            out += [
                ("lm_head.gemm_fwd",
                 lambda m0=m0, mc=mc: abi.qlora_nf4_gemm(p(self.X) + 2 * m0 * L.K, self.cw, 0, None,
                                                         None, mc, 0, None, p(self.z), ws, wsb,
                                                         stream)),
                ("lm_head.ce_rows",
                 lambda m0=m0, mc=mc: abi.qlora_cross_entropy_rows(
                     p(self.z), mc, L.N, p(self.labels) + 4 * m0, p(self.cnt), p(self.tl) + 4 * m0,
                     1, stream)),
                ("lm_head.gemm_dx",
                 lambda m0=m0, mc=mc: abi.qlora_nf4_gemm(p(self.z), self.cw, 1, None, None, mc, 0,
                                                         None, p(self.dX) + 2 * m0 * L.K, ws, wsb,
                                                         stream)),
            ]
        out.append(("lm_head.ce_mean",
                    lambda: abi.qlora_cross_entropy_mean(p(self.tl), M, p(self.cnt), p(self.loss),
                                                         stream)))
        return out

    def e2e(self):
        linear.lm_head_ce(self.X, self.w, self.labels, chunk=self.chunk, dX=self.dX,
                          token_loss=self.tl, ws=self.ws)


class Step:
    """One step of a workload: its linears' states and the ordered (name, call) stages."""

    def __init__(self, w, dev, seed, unpacked=False, glu_fused=False):
        self.w = w
        self.glu_fused = glu_fused  # packed MLP: SwiGLU in the gate/up GEMM's epilogue
        self.share_x = False
        self.pglue = None
        self.ce = None
        inp = synth.make_inputs(w, seed=seed)
        bf = dict(dtype=torch.bfloat16, device=dev)
        if w.ce:
            st = CeState(w.linears[0], w.M, inp["X"], inp["labels"], inp["linears"][0]["W0"],
                         synth.CE_CHUNK, dev)
            self.states, self.ce, self.glue = [st], st, None
            self.inputs = [(st, "X"), (st, "labels")]
            return
        if w.grouped:
            # Adapters sharing X: one packed-adapter layer (stacked W0, A, B), or, unpacked,
            # one layer per adapter on the same X with its own column block of dY.
            Ls, lins = w.linears, inp["linears"]
            Ns = [L.N for L in Ls]
            self.glue = None
            if unpacked:
                edges = np.cumsum([0] + Ns)
                self.states = [LinearState(L, w.M, inp["X"],
                                           inp["dY"][:, edges[i]:edges[i + 1]].contiguous(),
                                           d["W0"], d["A"], d["B"], dev)
                               for i, (L, d) in enumerate(zip(Ls, lins))]
                self.share_x = True
                for st in self.states[1:]:
                    st.X = self.states[0].X
            else:
                L0 = Ls[0]
                Lp = synth.LinearShape("+".join(L.name for L in Ls), L0.K, sum(Ns), L0.r,
                                       L0.alpha, L0.w_std, L0.double_quant)
                self.states = [LinearState(Lp, w.M, inp["X"], inp["dY"],
                                           torch.cat([d["W0"] for d in lins]),
                                           torch.cat([d["A"] for d in lins]),
                                           torch.cat([d["B"] for d in lins]), dev, groups=Ns)]
            self.inputs = self._inputs(self.states)
            return
        if not w.mlp:
            self.states = [LinearState(L, w.M, d["X"], d["dY"], d["W0"], d["A"], d["B"], dev)
                           for L, d in zip(w.linears, inp["linears"])]
            self.inputs = [(st, "X") for st in self.states] + [(st, "dY") for st in self.states]
            self.glue = None
            return
        gate, up, down = w.linears
        lg, lu, ld = inp["linears"]
        I = gate.N
        if not unpacked:
            # MLP block with gate and up packed into one layer on the shared X: its output
            # [M, 2I] feeds the packed SwiGLU, whose backward writes the layer's upstream
            # gradient [M, 2I]; the layer's dX is then the block's input gradient (gate's and
            # up's contributions summed by the one dX GEMM).
            Lgu = synth.LinearShape("gate_proj+up_proj", gate.K, 2 * I, gate.r, gate.alpha,
                                    gate.w_std, gate.double_quant)
            self.a = torch.empty((w.M, I), **bf)
            sgu = LinearState(Lgu, w.M, inp["X"], torch.empty((w.M, 2 * I), **bf),
                              torch.cat([lg["W0"], lu["W0"]]), torch.cat([lg["A"], lu["A"]]),
                              torch.cat([lg["B"], lu["B"]]), dev, groups=[I, I])
            sd = LinearState(down, w.M, self.a, inp["dY"], ld["W0"], ld["A"], ld["B"], dev)
            self.states = [sgu, sd]
            self.pglue = (sgu, sd)
            self.glue = None
            self.inputs = [(sgu, "X"), (sd, "dY")]
            return
        # MLP block: gate/up on the shared input X, SwiGLU, down; the backward runs down, the
        # SwiGLU backward, then up and gate on their output gradients dg, du.
        X = inp["X"].to(dev)
        dg = torch.empty((w.M, I), **bf)
        du = torch.empty((w.M, I), **bf)
        self.a = torch.empty((w.M, I), **bf)
        sg = LinearState(gate, w.M, X, dg, lg["W0"], lg["A"], lg["B"], dev)
        su = LinearState(up, w.M, X, du, lu["W0"], lu["A"], lu["B"], dev)
        sd = LinearState(down, w.M, self.a, inp["dY"], ld["W0"], ld["A"], ld["B"], dev)
        su.X = sg.X  # one copy of the block input
        self.states = [sg, su, sd]
        self.glue = (sg, su, sd, dg, du)
        self.inputs = [(sg, "X"), (sd, "dY")]

    def twin(self):
        """A second set of step buffers over the same weights (see LinearState.twin)."""
        t = copy.copy(self)
        if self.ce is not None:
            t.ce = self.ce.twin()
            t.states = [t.ce]
            t.inputs = [(t.ce, "X"), (t.ce, "labels")]
            return t
        if self.pglue is not None:
            sgu, sd = (st.twin() for st in self.pglue)
            t.a = torch.empty_like(self.a)
            sd.X = t.a
            t.states = [sgu, sd]
            t.pglue = (sgu, sd)
            t.inputs = [(sgu, "X"), (sd, "dY")]
            return t
        if self.glue is None:
            t.states = [st.twin() for st in self.states]
            if self.share_x:
                for st in t.states[1:]:
                    st.X = t.states[0].X
            t.inputs = t._inputs(t.states)
            return t
        sg, su, sd, dg, du = (x.twin() if isinstance(x, LinearState) else torch.empty_like(x)
                              for x in self.glue)
        t.a = torch.empty_like(self.a)
        su.X = sg.X
        sg.dY, su.dY, sd.X = dg, du, t.a
        t.states = [sg, su, sd]
        t.glue = (sg, su, sd, dg, du)
        t.inputs = [(sg, "X"), (sd, "dY")]
        return t

    def _inputs(self, states):
        xs = states[:1] if self.share_x else states
        return [(st, "X") for st in xs] + [(st, "dY") for st in states]

    def stages(self, stream):
        p = lambda t: t.data_ptr()
        if self.ce is not None:
            return self.ce.stages(stream)
        if self.pglue is not None:
            sgu, sd = self.pglue
            M, I = self.a.shape
            if self.glu_fused:
                # qlora_grouped_fwd_swiglu as one stage: X A^T, then the GEMM that also writes
                # the SwiGLU output (attributed to the GEMM).
                fused = [(f"{sgu.L.name}.gemm_fwd", lambda: abi.qlora_grouped_fwd_swiglu(
                    p(sgu.X), sgu.cw, p(sgu.A), p(sgu.B), M, sgu.L.r, sgu.L.alpha, p(sgu.H),
                    p(sgu.XA), p(self.a), p(sgu.ws), sgu.ws.numel(), stream))]
                return (fused + sd.fwd_stages(stream) + sd.bwd_stages(stream)
                        + [("swiglu.bwd", lambda: abi.qlora_swiglu_packed_bwd(
                            p(sgu.H), p(sd.dX), p(sgu.dY), M, I, stream))]
                        + sgu.bwd_stages(stream))
            return (sgu.fwd_stages(stream)
                    + [("swiglu.fwd", lambda: abi.qlora_swiglu_packed_fwd(p(sgu.H), p(self.a), M,
                                                                          I, stream))]
                    + sd.fwd_stages(stream) + sd.bwd_stages(stream)
                    + [("swiglu.bwd", lambda: abi.qlora_swiglu_packed_bwd(
                        p(sgu.H), p(sd.dX), p(sgu.dY), M, I, stream))]
                    + sgu.bwd_stages(stream))
        if self.glue is None:
            out = []
            for st in self.states:
                out += st.fwd_stages(stream) + st.bwd_stages(stream)
            return out
        sg, su, sd, dg, du = self.glue
        n = self.a.numel()
        return (sg.fwd_stages(stream) + su.fwd_stages(stream)
                + [("swiglu.fwd", lambda: abi.qlora_swiglu_fwd(p(sg.H), p(su.H), p(self.a), n,
                                                               stream))]
                + sd.fwd_stages(stream) + sd.bwd_stages(stream)
                + [("swiglu.bwd", lambda: abi.qlora_swiglu_bwd(p(sg.H), p(su.H), p(sd.dX), p(dg),
                                                               p(du), n, stream))]
                + su.bwd_stages(stream) + sg.bwd_stages(stream))

    def e2e(self):
        """One step through the public Python entry points (linear.forward / backward and the
        SwiGLU glue), on the device buffers already holding this step's inputs."""
        if self.ce is not None:
            self.ce.e2e()
            return
        if self.pglue is not None:
            sgu, sd = self.pglue
            if self.glu_fused:
                linear.gate_up_swiglu_forward(sgu.X, sgu.w, sgu.A, sgu.B, sgu.L.alpha, GU=sgu.H,
                                              XA=sgu.XA, act=self.a, ws=sgu.ws)
            else:
                sgu.forward()
                linear.swiglu_packed_forward(sgu.H, a=self.a)
            sd.forward()
            sd.backward()
            linear.swiglu_packed_backward(sgu.H, sd.dX, dgu=sgu.dY)
            sgu.backward()
            return
        if self.glue is None:
            for st in self.states:
                st.forward()
                st.backward()
            return
        sg, su, sd, dg, du = self.glue
        for st in (sg, su):
            linear.forward(st.X, st.w, st.A, st.B, st.L.alpha, H=st.H, XA=st.XA, ws=st.ws)
        linear.swiglu_forward(sg.H, su.H, a=self.a)
        linear.forward(sd.X, sd.w, sd.A, sd.B, sd.L.alpha, H=sd.H, XA=sd.XA, ws=sd.ws)
        linear.backward(sd.dY, sd.X, sd.w, sd.A, sd.B, sd.XA, sd.L.alpha, dX=sd.dX, dA=sd.dA,
                        dB=sd.dB, ws=sd.ws)
        linear.swiglu_backward(sg.H, su.H, sd.dX, dg=dg, du=du)
        for st in (su, sg):
            linear.backward(st.dY, st.X, st.w, st.A, st.B, st.XA, st.L.alpha, dX=st.dX,
                            dA=st.dA, dB=st.dB, ws=st.ws)

    def outputs(self):
        """Result tensors a user reads back after a step."""
        if self.ce is not None:
            return [self.ce.loss, self.ce.dX]
        if self.pglue is not None:
            sgu, sd = self.pglue
            return [sd.H, sgu.dX] + [t for st in self.states for t in (st.dA, st.dB)]
        if self.glue is None:
            return [t for st in self.states for t in (st.H, st.dX, st.dA, st.dB)]
        sg, su, sd, _, _ = self.glue
        return [sd.H, sg.dX, su.dX] + [t for st in self.states for t in (st.dA, st.dB)]


def run_steps(step, n, stream, flush, record):
    """Eager mode: run n steps, each stage launched from Python, CUDA events on `stream`
    between the stages.  Returns (per-step ms list, {stage: [ms...]})."""
    per_step = []
    per_stage = {}
    calls = step.stages(stream.cuda_stream)
    events = []
    for _ in range(n):
        # L2 flush: write 256 MiB, then read it back so the evicted lines are clean (the
        # write-back of the flush's own dirty lines must not land on the first timed kernel).
        flush.zero_()
        flush.max()
        evs = []
        for name, fn in calls:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            evs.append((name, e))
            fn()
        end = torch.cuda.Event(enable_timing=True)
        end.record(stream)
        evs.append(("end", end))
        if record:
            events.append(evs)
    torch.cuda.synchronize()
    for evs in events:
        per_step.append(evs[0][1].elapsed_time(evs[-1][1]))
        for (name, a), (_, b) in zip(evs[:-1], evs[1:]):
            per_stage.setdefault(name, []).append(a.elapsed_time(b))
    return per_step, per_stage


class GraphStep:
    """The whole step captured into CUDA graphs, so host-side launch cost never shows up as idle
    time between kernels.  Two captures:
      plain         the layer's public calls (linear.forward / backward, i.e. qlora_linear_fwd /
                    qlora_linear_bwd, and the SwiGLU glue), exactly as a user's step issues them,
                    with no timing nodes inside: each timed step is one replay bracketed by
                    events recorded on the replay stream;
      instrumented  the same work as its stage entry points with an event (recorded by the
                    graph itself) between every two stages, for the per-stage attribution; its
                    event nodes add a little time of their own, so stage times are slight upper
                    bounds.
    Each replay is preceded by the L2 flush (outside the graph) and followed by a synchronize."""

    def __init__(self, step):
        self.side = torch.cuda.Stream()
        calls = step.stages(self.side.cuda_stream)
        self.names = [name for name, _ in calls]
        self.evs = [torch.cuda.Event(enable_timing=True, external=True)
                    for _ in range(len(calls) + 1)]
        self.graph_i = torch.cuda.CUDAGraph()
        n0 = abi.qlora_launch_counter()
        with torch.cuda.graph(self.graph_i, stream=self.side, capture_error_mode="relaxed"):
            for (_, fn), e in zip(calls, self.evs):
                e.record()
                fn()
            self.evs[-1].record()
        self.stage_launches_per_step = abi.qlora_launch_counter() - n0
        self.graph = torch.cuda.CUDAGraph()
        n0 = abi.qlora_launch_counter()
        with torch.cuda.graph(self.graph, stream=self.side, capture_error_mode="relaxed"):
            step.e2e()
        self.launches_per_step = abi.qlora_launch_counter() - n0
        # One linear alone: its public forward and backward also as graphs of their own, so the
        # forward and backward times carry no interior timing nodes either.
        self.graph_f = self.graph_b = None
        if step.ce is None and step.pglue is None and step.glue is None and len(step.states) == 1:
            st = step.states[0]
            self.graph_f, self.graph_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph_f, stream=self.side, capture_error_mode="relaxed"):
                st.forward()
            with torch.cuda.graph(self.graph_b, stream=self.side, capture_error_mode="relaxed"):
                st.backward()

    def run(self, n, flush, record, graph=None):
        """n plain replays (of the step, or of `graph`); per-replay device times (ms)."""
        graph = self.graph if graph is None else graph
        per_step = []
        for _ in range(n):
            flush.zero_()
            flush.max()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize()
            if record:
                per_step.append(a.elapsed_time(b))
        return per_step

    def run_stages(self, n, flush):
        """n instrumented replays: ({stage: [ms...]}, [step ms...] between the first and last
        interior events)."""
        per_stage, per_step = {}, []
        for _ in range(n):
            flush.zero_()
            flush.max()
            self.graph_i.replay()
            torch.cuda.synchronize()
            per_step.append(self.evs[0].elapsed_time(self.evs[-1]))
            for name, a, b in zip(self.names, self.evs[:-1], self.evs[1:]):
                per_stage.setdefault(name, []).append(a.elapsed_time(b))
        return per_stage, per_step


def run_e2e(step, steps):
    """The same metric through the public entry points (qlora_linear_fwd / qlora_linear_bwd, and
    the SwiGLU glue for the MLP block) with host buffers.  Every step copies its inputs from
    pinned host memory, runs the layer(s) and copies every result back.  Two buffer sets and
    three streams (copy in, compute, copy out) overlap one step's transfers with the other
    step's compute, as a training loop feeding the layer from the host would; the time is the
    whole pipeline's, from the first input copy to the last result copy."""
    sets = [step, step.twin()]
    host_in = [getattr(st, attr).cpu().pin_memory() for st, attr in step.inputs]
    host_out = [[torch.empty_like(t, device="cpu").pin_memory() for t in s.outputs()]
                for s in sets]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out[0])
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_comp = [torch.cuda.Event() for _ in sets]
    ev_out = [torch.cuda.Event() for _ in sets]

    def one(i):
        b = i % 2
        S = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])  # step i-2 has finished reading these inputs
            for (st, attr), h in zip(S.inputs, host_in):
                getattr(st, attr).copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])  # step i-2's results have left these buffers
            S.e2e()
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for t, h in zip(S.outputs(), host_out[b]):
                h.copy_(t, non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(3, 3 + steps):
        one(i)
    b.record(s_out)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps, h2d, d2h


def kernel_source_digest(files):
    """sha256 over the kernel's source files with comments and blank space removed, so an edit
    to a comment, or to code no kernel statement changes, does not void a recorded capture."""
    import hashlib
    import re
    m = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, name)) as g:
            txt = g.read()
        txt = re.sub(r"/\*.*?\*/", " ", txt, flags=re.S)
        txt = re.sub(r"//[^\n]*", " ", txt)
        m.update(" ".join(txt.split()).encode())
    return m.hexdigest()


def ncu_traffic(workload, stage):
    """DRAM bytes per launch of `stage` from the committed ncu capture (profiles/ncu_traffic.json),
    or None when there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(f"{workload}.{stage}")
        if not rec:
            return None
        ok = kernel_source_digest(rec["source_files"]) == rec["source_digest"]
        return rec["traffic_bytes"] if ok else None
    except (OSError, ValueError, KeyError):
        return None


def roofline(step, per_stage, peaks, workload):
    """Roofline of the dominant kernel (largest total time among the stages)."""
    totals = {k: sum(v) for k, v in per_stage.items()}
    name = max(totals, key=totals.get)
    lin_name, stage = name.split(".", 1)
    ms = statistics.mean(per_stage[name])
    if lin_name == "swiglu":
        n = step.a.numel()
        flops, byts = 0.0, (3 if stage == "fwd" else 5) * 2 * n
    else:
        st = next(s for s in step.states if s.L.name == lin_name)
        M, L, R = st.M, st.L, st.R  # R: packed rank columns (r for a single adapter)
        if stage.startswith("gemm"):
            flops, byts = gemm_work(L, M, stage == "gemm_dx", R // L.r if L.r else 1)
        elif stage.startswith("ce_"):
            # the rows stage reads the chunk's logits and writes their gradient in place
            flops, byts = 0.0, (4 * M * L.N if stage == "ce_rows" else 4 * st.Mtot)
        elif stage.startswith("lora_down"):
            # X A^T: every input column feeds R outputs; dY B: each feeds its adapter's r.
            C, per = (L.K, R) if stage.endswith("fwd") else (L.N, L.r)
            flops, byts = 2.0 * M * C * per, 2 * M * C + 4 * M * R
        else:
            C, per = (L.N, L.r) if stage.endswith("dB") else (L.K, R)
            flops, byts = 2.0 * M * C * per, 2 * M * C + 2 * M * R + 4 * C * per
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
def oracle_prepare(w, seed):
    """Quantise every W0 with the fp64 oracle (not timed) and dequantise it (timed: the
    dequant is charged once per step, i.e. once per batch of M tokens)."""
    from oracle import nf4  # test infrastructure: only here and in the reference arm
    inp = synth.make_inputs(w, seed=seed)
    t_deq = 0.0
    Wds = []
    for L, d in zip(w.linears, inp["linears"]):
        Wf = d["W0"].float().numpy()
        am = nf4.block_absmax(Wf)
        if L.double_quant:
            q8, sc = nf4.double_quant(am.reshape(-1))
            eff = nf4.dq_effective_absmax(q8, sc).reshape(am.shape)
        else:
            eff = am
        q = np.empty((L.N, L.K // 2), dtype=np.uint8)
        for r0 in range(0, L.N, 8192):  # row chunks bound the host memory of the code choice
            q[r0:r0 + 8192] = nf4.pack_codes(nf4.choose_codes(Wf[r0:r0 + 8192], eff[r0:r0 + 8192]))
        t1 = time.perf_counter()
        Wds.append(nf4.dequantize(q, eff, L.N, L.K).astype(np.float64))
        t_deq += time.perf_counter() - t1
    return inp, Wds, t_deq


def oracle_rows(w, prep, n):
    """Seconds the fp64 oracle takes for forward + backward on the first n token rows of the
    workload (for the MLP block: gate/up, SwiGLU, down, and back; for packed adapters the
    packed layer)."""
    from oracle import qlora  # test infrastructure: only here and in the reference arm
    inp, Wds, _ = prep
    f64 = lambda t: t.float().numpy().astype(np.float64)
    if w.ce:
        from oracle import lm_head  # test infrastructure, as above
        t0 = time.perf_counter()
        lm_head.lm_head_ce(f64(inp["X"][:n]), Wds[0], inp["labels"][:n].numpy())
        return time.perf_counter() - t0
    lora = [(f64(d["A"]), f64(d["B"])) for d in inp["linears"]]
    t0 = time.perf_counter()
    if w.grouped:
        X, dY = f64(inp["X"][:n]), f64(inp["dY"][:n])
        As, Bs = [A for A, _ in lora], [B for _, B in lora]
        qlora.grouped_forward(X, Wds, As, Bs, w.linears[0].alpha)
        qlora.grouped_backward(dY, X, Wds, As, Bs, w.linears[0].alpha)
    elif not w.mlp:
        for L, d, Wd, (A, B) in zip(w.linears, inp["linears"], Wds, lora):
            X, dY = f64(d["X"][:n]), f64(d["dY"][:n])
            qlora.forward(X, Wd, A, B, L.alpha)
            qlora.backward(dY, X, Wd, A, B, L.alpha)
    else:
        (gate, up, down), X, dY = w.linears, f64(inp["X"][:n]), f64(inp["dY"][:n])
        g, _ = qlora.forward(X, Wds[0], *lora[0], gate.alpha)
        u, _ = qlora.forward(X, Wds[1], *lora[1], up.alpha)
        a = qlora.swiglu_forward(g, u)
        qlora.forward(a, Wds[2], *lora[2], down.alpha)
        da = qlora.backward(dY, a, Wds[2], *lora[2], down.alpha)["dX"]
        dg, du = qlora.swiglu_backward(g, u, da)
        qlora.backward(du, X, Wds[1], *lora[1], up.alpha)
        qlora.backward(dg, X, Wds[0], *lora[0], gate.alpha)
    return time.perf_counter() - t0


def oracle_desc(w, n):
    return (f"fp64 oracle fwd+bwd on {n} token rows of {w.name} (M={w.M}), plus one deq(W0) "
            f"per linear per step charged per batch of M tokens; quantisation not timed")


ORACLE_THREADS = 0  # set from --oracle-threads; 0 = all host cores


def blas_threads():
    if ORACLE_THREADS > 0:
        return ORACLE_THREADS
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_rows(w, prep, seconds):
    """Token rows of a sample that keeps the oracle busy about `seconds` (at least 512 rows, or
    all M when fewer), calibrated on 8 rows."""
    per_row = oracle_rows(w, prep, min(8, w.M)) / min(8, w.M)
    n = int(seconds / max(per_row, 1e-9))
    return int(max(min(512, w.M), min(w.M, n)))


def cpu_baseline(w, seed=0, seconds=10.0):
    """The fp64 oracle on the host cores, on a calibrated sample of the workload's token rows
    (about `seconds` of work), plus the single-thread figure of the tiny configuration."""
    prep = oracle_prepare(w, seed)
    n = oracle_sample_rows(w, prep, seconds)
    per_token = oracle_rows(w, prep, n) / n + prep[2] / w.M
    out = {"value": round(1.0 / per_token, 2), "unit": "tokens/s", "cores": blas_threads(),
           "kind": "oracle", "sample": oracle_desc(w, n)}
    try:
        from threadpoolctl import threadpool_limits
        tw = synth.workload("tiny")
        with threadpool_limits(1, user_api="blas"):
            tprep = oracle_prepare(tw, seed)
            oracle_rows(tw, tprep, tw.M)  # warm
            t = min(oracle_rows(tw, tprep, tw.M) for _ in range(5))
        out["single_thread_tiny"] = {"value": round(tw.M / (t + tprep[2]), 1),
                                     "unit": "tokens/s", "cores": 1,
                                     "sample": oracle_desc(tw, tw.M) + ", best of 5"}
    except Exception as exc:  # threadpoolctl missing: leave the figure out, say why
        out["single_thread_tiny"] = {"unavailable": str(exc)}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.workload(args.workload)
    prep = oracle_prepare(w, 0)
    t_deq = prep[2]
    # Calibrate: rows per step so the whole run stays within about two minutes.
    per_row = oracle_rows(w, prep, min(8, w.M)) / min(8, w.M)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(w.M, budget / max(per_row, 1e-9))))
    times = []
    for i in range(args.warmup + args.steps):
        tr = oracle_rows(w, prep, n)
        if i >= args.warmup:
            times.append(tr + t_deq * n / w.M)
    tot = sum(times)
    value = args.steps * n / tot
    line = {
        "impl": "reference", "metric": "qlora_linear_fwd_bwd_tokens_per_s", "value": round(value, 3),
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * tot / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": oracle_desc(w, n)},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# Every other configuration, measured in the same run (one line, key "configs")
# ----------------------------------------------------------------------------------------------
CONFIG_WORKLOADS = ("tiny", "mlp_8b", "proj_70b_dq", "sweep_m1", "sweep_m16", "sweep_m128",
                    "sweep_m1024", "sweep_m16384")
SPEC_HBM_GBS = 8000.0  # the ~8 TB/s HBM3e figure the targets quote, beside the measured copy


def min_bytes(L, M, backward):
    """Minimum HBM bytes of one pass of a linear: the packed weight once, the bf16 activations,
    the LoRA factors (and, backward, their fp32 gradients)."""
    small = 2 * L.r * (L.K + L.N)
    if not backward:
        return weight_stream_bytes(L) + 2 * M * L.K + 2 * M * L.N + 2 * M * L.r + small
    return (weight_stream_bytes(L) + 2 * M * L.N + 4 * M * L.K + 2 * M * L.r + small
            + 4 * L.r * (L.K + L.N))


def is_fwd_stage(name):
    st = name.split(".", 1)[1]
    return st in ("lora_down_fwd", "gemm_fwd", "fwd")


def measure_config(name, dev, steps, warmup, peaks, flush, clocks_on, glu_fused=False):
    """tokens/s, step TFLOP/s, forward and backward times (and, for one linear, their GB/s of
    minimum traffic), the dominant stage's roofline and the clocks, for one workload timed as
    the headline is: CUDA-graph replays with L2 flushed before each."""
    w = synth.workload(name)
    step = Step(w, dev, seed=0, glu_fused=glu_fused)
    stream = torch.cuda.current_stream()
    run_steps(step, warmup, stream, flush, record=False)
    graph = GraphStep(step)
    graph.run(3, flush, record=True)
    sampler = ClockSampler(dev.index or 0)
    if clocks_on:
        sampler.start()
        time.sleep(0.3)
    per_step = graph.run(steps, flush, record=True)
    clocks = sampler.stop() if clocks_on else None
    per_stage, _ = graph.run_stages(max(5, steps), flush)
    if abi.qlora_device_error() != 0:
        raise SystemExit(f"device error word set while timing {name}")
    ms = statistics.mean(per_step)
    means = {k: statistics.mean(v) for k, v in per_stage.items()}
    if graph.graph_f is not None:
        # One linear: its public forward and backward replayed alone, no interior events.
        fwd = statistics.mean(graph.run(max(5, steps), flush, True, graph.graph_f))
        bwd = statistics.mean(graph.run(max(5, steps), flush, True, graph.graph_b))
        fb_note = "plain graph replays of the public forward / backward calls"
    else:
        fwd = sum(v for k, v in means.items() if is_fwd_stage(k))
        bwd = sum(v for k, v in means.items() if not is_fwd_stage(k))
        fb_note = "sums of the instrumented per-stage times"
    if abi.qlora_device_error() != 0:
        raise SystemExit(f"device error word set while timing {name}")
    tflops = step_flops(w) / (ms * 1e-3) / 1e12
    rec = {"M": w.M, "ms_per_step": round(ms, 5), "tokens_per_s": round(w.M / (ms * 1e-3), 1),
           "tflops": round(tflops, 2),
           "tflops_frac_of_peak": round(tflops / peaks["bf16_tflops"], 4),
           "fwd_ms": round(fwd, 5), "bwd_ms": round(bwd, 5), "fwd_bwd_timing": fb_note,
           "stages_ms": {k: round(v, 5) for k, v in means.items()},
           "roofline": roofline(step, per_stage, peaks, name),
           "graph_launches_per_step": graph.launches_per_step, "steps": steps, "clocks": clocks,
           "side_overlap_sms": side_overlap(w)}
    if len(w.linears) == 1 and not w.mlp:
        L = w.linears[0]
        for d, t in (("fwd", fwd), ("bwd", bwd)):
            b = min_bytes(L, w.M, d == "bwd")
            gbs = b / (t * 1e-3) / 1e9
            rec[f"{d}_min_bytes"] = b
            rec[f"{d}_gbs"] = round(gbs, 1)
            rec[f"{d}_hbm_frac"] = {"measured": round(gbs / peaks["hbm_gbs"], 4),
                                    "spec_8000": round(gbs / SPEC_HBM_GBS, 4)}
    del graph, step
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def side_overlap(w, unpacked=False):
    """Linears whose timed backward runs dB and dA beside the dX GEMM (qlora_set_side_overlap,
    the library's current mode), with the SMs they get; the instrumented stage capture calls
    the stage entry points one after another, so there they run after the GEMM."""
    if w.ce:
        return {}
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    groups = [[L] for L in w.linears]
    if w.grouped:
        groups = [list(w.linears)]
    elif w.mlp and not unpacked:
        groups = [list(w.linears[:2]), [w.linears[2]]]
    out = {}
    for g in groups:
        N, K, R = sum(L.N for L in g), g[0].K, sum(L.r for L in g)
        s = abi.qlora_backward_side_sms(w.M, N, K, R, sms, -1)
        if s:
            out["+".join(L.name for L in g)] = s
    return out


def workload_config(w, unpacked=False):
    c = {"workload": w.name, "M": w.M,
         "linears": [{"name": L.name, "K": L.K, "N": L.N, "r": L.r, "alpha": L.alpha,
                      "absmax": "double-quant" if L.double_quant else "fp32"} for L in w.linears],
         "l2": "flushed before every step (256 MiB write + read, outside the events)", "parallelism": "replicas"}
    if w.grouped:
        c["adapters"] = ("unpacked: one layer per adapter on the shared input" if unpacked else
                         "packed: one stacked NF4 weight, adapters along its rows, shared input")
    if w.mlp:
        c["adapters"] = ("unpacked: gate and up as separate layers" if unpacked else
                         "gate and up packed into one layer on the shared input")
    if w.ce:
        c["loss"] = (f"cross-entropy over the {w.linears[0].N}-word vocabulary, uniform labels, "
                     f"chunks of {synth.CE_CHUNK} tokens; frozen NF4 head, no adapter")
    return c


# ----------------------------------------------------------------------------------------------
# Replicas: every rank times its own copy of the step; the job's time is the slowest rank's
# ----------------------------------------------------------------------------------------------
def max_over_ranks(ms, dist, device):
    """The largest of the ranks' device-timed milliseconds (this rank's alone without dist)."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, M, steps, total_ms):
    """Whole-job throughput: every rank processed M tokens per step, in the slowest rank's time."""
    return world * M * steps / (total_ms * 1e-3)


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
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations (the \"configs\" key)")
    ap.add_argument("--config-steps", type=int, default=10,
                    help="timed steps per configuration of the \"configs\" key")
    ap.add_argument("--eager", action="store_true",
                    help="launch every stage from Python instead of replaying a CUDA graph")
    ap.add_argument("--oracle-threads", type=int, default=0,
                    help="BLAS threads for the oracle legs (cpu_baseline, --impl reference); "
                         "0 = all host cores")
    ap.add_argument("--unpacked", action="store_true",
                    help="adapters sharing an input (qkv_8b, mlp_8b's gate/up) run as "
                         "separate layers")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.oracle_threads > 0:
        from threadpoolctl import threadpool_limits
        global ORACLE_THREADS, _ORACLE_LIMITS
        ORACLE_THREADS = args.oracle_threads
        _ORACLE_LIMITS = threadpool_limits(args.oracle_threads, user_api="blas")
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
    step = Step(w, dev, seed=rank, unpacked=args.unpacked)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    run_steps(step, args.warmup, stream, flush, record=False)
    if abi.qlora_device_error() != 0:
        raise SystemExit("device error word set during warm-up")
    graph = None
    if not args.eager:
        try:
            graph = GraphStep(step)
            graph.run(3, flush, record=True)
            graph.run_stages(2, flush)
        except Exception as exc:  # a runtime without timing events in graphs: time eagerly
            print(f"CUDA graph timing unavailable ({exc}); timing eager launches",
                  file=sys.stderr)
            graph = None
            torch.cuda.synchronize()

    sampler = ClockSampler(local)
    if not args.no_clocks and rank == 0:
        sampler.start()
        time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = abi.qlora_launch_counter()
    if graph is not None:
        per_step = graph.run(args.steps, flush, record=True)
        launches = graph.launches_per_step * args.steps
    else:
        per_step, per_stage = run_steps(step, args.steps, stream, flush, record=True)
        torch.cuda.synchronize()
        launches = abi.qlora_launch_counter() - n0
    if dist:
        dist.barrier()
    clocks = sampler.stop() if (not args.no_clocks and rank == 0) else None
    if abi.qlora_device_error() != 0:
        raise SystemExit("device error word set during the timed region")
    instrumented_ms = None
    if graph is not None:  # stage attribution, after (and outside) the timed region
        per_stage, steps_i = graph.run_stages(max(5, min(args.steps, 20)), flush)
        instrumented_ms = statistics.mean(steps_i)

    total_ms = max_over_ranks(sum(per_step), dist, dev)
    value = job_tokens_per_s(world, w.M, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    e2e_ms, h2d, d2h = run_e2e(step, args.e2e_steps)
    e2e_value = job_tokens_per_s(world, w.M, 1, max_over_ranks(e2e_ms, dist, dev))

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
            "config": workload_config(w, args.unpacked),
            "tflops": round(tflops, 2),
            "tflops_frac_of_peak": round(tflops / peaks["bf16_tflops"], 4),
            "stages_ms": {k: round(statistics.mean(v), 5) for k, v in per_stage.items()},
            "stages_note": ("the timed step replays the layer's public calls (qlora_linear_fwd / "
                            "qlora_linear_bwd and the SwiGLU glue) with no interior events; "
                            "per-stage times come from a second capture of the same work as its "
                            "stage entry points with an event between every two stages, replayed "
                            "after the timed region; for the linears in side_overlap_sms the timed "
                            "backward runs lora_grad_dB / lora_grad_dA beside gemm_dx on that many "
                            "SMs (the stage capture runs them after it)"),
            "side_overlap_sms": side_overlap(w, args.unpacked),
            "instrumented_ms_per_step": (round(instrumented_ms, 5) if instrumented_ms else None),
            "roofline": roofline(step, per_stage, peaks, w.name),
            "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "launch_mode": "cuda_graph" if graph is not None else "eager",
            "clocks": clocks,
        }
        if world == 1 and not args.no_configs:
            line["configs"] = {}
            del step
            torch.cuda.empty_cache()
            for name in CONFIG_WORKLOADS:
                if name == w.name:
                    continue
                line["configs"][name] = measure_config(name, dev, args.config_steps,
                                                       args.warmup, peaks, flush,
                                                       not args.no_clocks)
            # The headline workload once more with the rank-r down-projections inside the GEMM
            # launches (qlora_set_rank_fusion; off by default), for the trade-off.
            prev = abi.qlora_set_rank_fusion(True)
            try:
                fused = measure_config(w.name, dev, args.config_steps, args.warmup, peaks, flush,
                                       not args.no_clocks)
            finally:
                abi.qlora_set_rank_fusion(prev)
            fused["rank_fusion"] = True
            line["configs"][w.name + "+rank_fusion"] = fused
            # The MLP block with the SwiGLU in the gate/up GEMM's epilogue
            # (qlora_grouped_fwd_swiglu; the default step runs the packed SwiGLU kernel).
            glu = measure_config("mlp_8b", dev, args.config_steps, args.warmup, peaks, flush,
                                 not args.no_clocks, glu_fused=True)
            glu["swiglu_fusion"] = True
            line["configs"]["mlp_8b+swiglu_fusion"] = glu
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
