"""Host-side arithmetic of bench.py, on the CPU: the minimum-traffic counts behind the
few-token GB/s figures, the forward/backward split of the stage names, and the digest that
ties a recorded ncu capture to the kernel sources it was taken on."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from nf4_base_lora_blockwise_b200 import synth  # noqa: E402


def test_min_bytes_of_the_sweep_layer():
    """4096 -> 14336, r 16: the packed weight (0.5625 N K bytes) plus activations and factors,
    written out term by term."""
    L = synth.workload("sweep_m16").linears[0]
    NK = L.N * L.K
    w = NK // 2 + 4 * (NK // 64)
    small = 2 * 16 * (4096 + 14336)
    for M in (1, 16):
        fwd = w + M * (2 * 4096 + 2 * 14336 + 2 * 16) + small
        bwd = w + M * (2 * 14336 + 4 * 4096 + 2 * 16) + small + 4 * 16 * (4096 + 14336)
        assert bench.min_bytes(L, M, False) == fwd
        assert bench.min_bytes(L, M, True) == bwd
    # The published shape of these counts: ~33.7 / 34.8 MB at one token.
    assert abs(bench.min_bytes(L, 1, False) / 1e6 - 33.7) < 0.05
    assert abs(bench.min_bytes(L, 1, True) / 1e6 - 34.8) < 0.06


def test_min_bytes_double_quant_weight():
    L = synth.workload("proj_70b_dq").linears[0]
    NK = L.N * L.K
    assert bench.weight_stream_bytes(L) == NK // 2 + NK // 64 + 4 * -(-NK // 64 // 256)


def test_stage_direction():
    assert bench.is_fwd_stage("q_proj.lora_down_fwd")
    assert bench.is_fwd_stage("q_proj.gemm_fwd")
    assert bench.is_fwd_stage("swiglu.fwd")
    for n in ("q_proj.lora_down_bwd", "q_proj.gemm_dx", "q_proj.lora_grad_dB",
              "q_proj.lora_grad_dA", "swiglu.bwd"):
        assert not bench.is_fwd_stage(n)


def test_source_digest_ignores_comments_only(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "k.cu").write_text("int f(int x) {\n  return x + 1;  // add one\n}\n")
    d0 = bench.kernel_source_digest(["k.cu"])
    (tmp_path / "k.cu").write_text("/* header */\nint f(int x) {\n\n  return x + 1;\n}\n")
    assert bench.kernel_source_digest(["k.cu"]) == d0
    (tmp_path / "k.cu").write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.kernel_source_digest(["k.cu"]) != d0
