"""Seeded synthetic inputs for the QLoRA NF4 linear workloads.

This module only draws random numbers in a fixed order and casts them to bf16; it holds none
of the method's arithmetic (no quantisation, no products).  Both the GPU tests and the CPU
oracle take their inputs from here.

Recipe: one ``torch.Generator`` (CPU) seeded with ``seed`` draws, in this order: for a single
linear (or independent projections, one after the other) X, W0, A, B, dY; for the MLP
workload X, then W0, A, B of gate, up and down, then dY; for a packed-adapter workload (q/k/v
sharing X) X, then W0, A, B of each adapter, then dY over all adapters' outputs.  Values are
drawn in fp32 and cast to bf16 (round to nearest even).  The LM-head workload draws X, the
head W0 and then int32 labels uniform over the vocabulary.  "N(0, s)" means standard deviation s.  The LoRA down-projection A is either uniform
on (-a, a) with a = 1/sqrt(in) ("Kaiming-uniform" with torch's nn.Linear default slope
sqrt(5)), or the explicit bound of the tiny workload.  B is N(0, 0.01) -- non-zero, so the
LoRA path contributes to h and to dX.
"""

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearShape:
    """One QLoRA linear: K = in-features, N = out-features, r = LoRA rank."""
    name: str
    K: int
    N: int
    r: int
    alpha: float
    w_std: float = 0.02
    double_quant: bool = False


@dataclass(frozen=True)
class Workload:
    """A set of linears run on M tokens, with the value distributions of the inputs."""
    name: str
    M: int
    linears: tuple
    x_std: float = 1.0
    dy_std: float = 1e-2
    a_bound: float = 0.0          # 0 -> Kaiming-uniform 1/sqrt(K)
    b_std: float = 0.01
    mlp: bool = False             # gate/up -> SwiGLU -> down
    notes: str = ""
    grouped: bool = False         # the linears share X and run as one packed-adapter layer
    ce: bool = False              # one frozen NF4 LM head (r = 0) + cross-entropy on labels


def _lin(name, K, N, r, alpha, w_std=0.02, dq=False):
    return LinearShape(name, K, N, r, alpha, w_std, dq)


WORKLOADS = {
    # Tiny single layer: in 256, out 512, r 8, alpha 16, 64 tokens; A ~ U(+-1/16), dY ~ N(0,1).
    "tiny": Workload("tiny", 64, (_lin("linear", 256, 512, 8, 16.0),),
                     dy_std=1.0, a_bound=1.0 / 16.0),
    # Llama-3-8B q_proj 4096 -> 4096, r 16, alpha 32, 4096 tokens (2 x 2048).
    "q_proj_8b": Workload("q_proj_8b", 4096, (_lin("q_proj", 4096, 4096, 16, 32.0),)),
    # Llama-3-8B MLP: gate/up 4096 -> 14336, down 14336 -> 4096, r 16, alpha 32, 8192 tokens.
    "mlp_8b": Workload("mlp_8b", 8192, (_lin("gate_proj", 4096, 14336, 16, 32.0),
                                        _lin("up_proj", 4096, 14336, 16, 32.0),
                                        _lin("down_proj", 14336, 4096, 16, 32.0)), mlp=True),
    # Llama-3-70B o_proj 8192 -> 8192 and down 28672 -> 8192, double-quantised absmax,
    # r 64, alpha 16, 4096 tokens, W0 ~ N(0, 0.015).
    "proj_70b_dq": Workload("proj_70b_dq", 4096,
                            (_lin("o_proj", 8192, 8192, 64, 16.0, 0.015, True),
                             _lin("down_proj", 28672, 8192, 64, 16.0, 0.015, True))),
}

# Llama-3-8B attention projections q 4096 -> 4096, k and v 4096 -> 1024 (grouped-query), each
# with its own r 16, alpha 32 adapter, sharing the 4096-token input: one packed-adapter layer.
WORKLOADS["qkv_8b"] = Workload("qkv_8b", 4096, (_lin("q_proj", 4096, 4096, 16, 32.0),
                                                _lin("k_proj", 4096, 1024, 16, 32.0),
                                                _lin("v_proj", 4096, 1024, 16, 32.0)),
                               grouped=True)

# Llama-3-8B LM head 4096 -> 128256 (frozen, no adapter) + cross-entropy on 4096 tokens with
# uniform labels, processed in chunks of 1024 tokens.
WORKLOADS["lm_head_ce_8b"] = Workload("lm_head_ce_8b", 4096,
                                      (_lin("lm_head", 4096, 128256, 0, 0.0),), ce=True)
CE_CHUNK = 1024

# Token-count sweep on 4096 -> 14336, r 16, alpha 32.
SWEEP_M = (1, 16, 128, 1024, 16384)
for _m in SWEEP_M:
    WORKLOADS[f"sweep_m{_m}"] = Workload(f"sweep_m{_m}", _m,
                                         (_lin("up_proj", 4096, 14336, 16, 32.0),))


def workload(name, M=None):
    """Look up a workload, optionally overriding its token count."""
    w = WORKLOADS[name]
    if M is not None and M != w.M:
        w = Workload(w.name, M, w.linears, w.x_std, w.dy_std, w.a_bound, w.b_std, w.mlp,
                     w.notes, w.grouped, w.ce)
    return w


def _normal(gen, shape, std):
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)


def _uniform(gen, shape, bound):
    u = torch.rand(shape, generator=gen, dtype=torch.float32)
    return ((u * 2.0 - 1.0) * bound).to(torch.bfloat16)


def make_inputs(w, seed=0):
    """Draw the inputs of workload ``w`` on the CPU as bf16 tensors.

    MLP workload: X [M, K_gate], then W0, A, B of gate, up and down, then dY [M, N_down] (the
    gradient at the down output).  Packed-adapter workload: X [M, K], then W0, A, B of each
    adapter, then dY [M, sum N] (adapter g's gradient in its own column range).  Other workloads: for each linear, X [M, K], W0, A, B, then
    dY [M, N] -- independent projections, each with its own activations.

    Returns ``{"X", "dY", "linears": [{"W0", "A", "B", "X", "dY"}]}``; the top-level X and dY
    are those of the first linear (MLP: the MLP input and the down-output gradient).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)

    def draw_weights(L):
        W0 = _normal(gen, (L.N, L.K), L.w_std)
        bound = w.a_bound if w.a_bound > 0 else 1.0 / math.sqrt(L.K)
        A = _uniform(gen, (L.r, L.K), bound)
        B = _normal(gen, (L.N, L.r), w.b_std)
        return {"W0": W0, "A": A, "B": B}

    lins = []
    if w.ce:
        L = w.linears[0]
        X = _normal(gen, (w.M, L.K), w.x_std)
        W0 = _normal(gen, (L.N, L.K), L.w_std)
        labels = torch.randint(0, L.N, (w.M,), generator=gen, dtype=torch.int64).to(torch.int32)
        return {"X": X, "linears": [{"W0": W0}], "labels": labels}
    if w.grouped:
        X = _normal(gen, (w.M, w.linears[0].K), w.x_std)
        for L in w.linears:
            lins.append(draw_weights(L))
        dY = _normal(gen, (w.M, sum(L.N for L in w.linears)), w.dy_std)
        return {"X": X, "linears": lins, "dY": dY}
    if w.mlp:
        X = _normal(gen, (w.M, w.linears[0].K), w.x_std)
        for L in w.linears:
            lins.append(draw_weights(L))
        dY = _normal(gen, (w.M, w.linears[-1].N), w.dy_std)
        return {"X": X, "linears": lins, "dY": dY}
    for L in w.linears:
        X = _normal(gen, (w.M, L.K), w.x_std)
        d = draw_weights(L)
        d["X"] = X
        d["dY"] = _normal(gen, (w.M, L.N), w.dy_std)
        lins.append(d)
    return {"X": lins[0]["X"], "linears": lins, "dY": lins[0]["dY"]}


def make_linear(M, K, N, r, alpha=None, seed=0, x_std=1.0, w_std=0.02, a_bound=0.0,
                b_std=0.01, dy_std=1e-2):
    """Inputs of one ad-hoc linear (used by parity tests on ragged / edge shapes)."""
    w = Workload("adhoc", M, (_lin("linear", K, N, r, alpha if alpha else 2.0 * r, w_std),),
                 x_std=x_std, dy_std=dy_std, a_bound=a_bound, b_std=b_std)
    return make_inputs(w, seed)


def make_grouped(M, K, Ns, r, alpha=None, seed=0, x_std=1.0, w_std=0.02, a_bound=0.0,
                 b_std=0.01, dy_std=1e-2):
    """Inputs of an ad-hoc packed-adapter layer: adapters with out-features Ns share X [M, K]."""
    lins = tuple(_lin(f"adapter{i}", K, N, r, alpha if alpha else 2.0 * r, w_std)
                 for i, N in enumerate(Ns))
    w = Workload("adhoc_grouped", M, lins, x_std=x_std, dy_std=dy_std, a_bound=a_bound,
                 b_std=b_std, grouped=True)
    return make_inputs(w, seed)


def make_lm_head(M, K, V, seed=0, ignore_frac=0.0, x_std=1.0, w_std=0.02):
    """Inputs of an ad-hoc LM head + cross-entropy: X [M, K], W0 [V, K], labels [M] int32
    uniform in [0, V), of which a seeded fraction is replaced by -100 (ignored)."""
    w = Workload("adhoc_ce", M, (_lin("lm_head", K, V, 0, 0.0, w_std),), x_std=x_std, ce=True)
    inp = make_inputs(w, seed)
    if ignore_frac > 0:
        gen = torch.Generator(device="cpu")
        gen.manual_seed(seed + 1)
        drop = torch.rand(M, generator=gen) < ignore_frac
        inp["labels"] = torch.where(drop, torch.full_like(inp["labels"], -100), inp["labels"])
    return inp


def sample_rows(M, count=512, seed=1234):
    """Fixed seeded sample of token rows for full-size checks: ``count`` rows plus 0 and M-1."""
    if M <= count + 2:
        return torch.arange(M)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    rows = torch.randperm(M, generator=gen)[:count]
    rows = torch.unique(torch.cat([rows, torch.tensor([0, M - 1])]))
    return rows
