"""The seeded input generator: deterministic, right shapes, dtypes and spreads."""

import torch

from nf4_base_lora_blockwise_b200 import synth


def test_tiny_inputs_deterministic_and_shaped():
    w = synth.workload("tiny")
    a = synth.make_inputs(w, seed=0)
    b = synth.make_inputs(w, seed=0)
    assert a["X"].shape == (64, 256) and a["X"].dtype == torch.bfloat16
    L = a["linears"][0]
    assert L["W0"].shape == (512, 256) and L["A"].shape == (8, 256) and L["B"].shape == (512, 8)
    assert a["dY"].shape == (64, 512)
    for k in ("X", "dY"):
        assert torch.equal(a[k], b[k])
    assert torch.equal(a["linears"][0]["W0"], b["linears"][0]["W0"])
    assert float(L["A"].float().abs().max()) <= 1.0 / 16
    assert 0.015 < float(L["W0"].float().std()) < 0.025
    assert 0.8 < float(a["dY"].float().std()) < 1.2


def test_workload_table():
    assert synth.workload("q_proj_8b").M == 4096
    mlp = synth.workload("mlp_8b")
    assert mlp.mlp and [L.N for L in mlp.linears] == [14336, 14336, 4096]
    dq = synth.workload("proj_70b_dq")
    assert all(L.double_quant and L.r == 64 and L.alpha == 16.0 for L in dq.linears)
    assert [synth.workload(f"sweep_m{m}").M for m in synth.SWEEP_M] == [1, 16, 128, 1024, 16384]


def test_sample_rows():
    r = synth.sample_rows(4096)
    assert int(r[0]) == 0 and int(r[-1]) == 4095 and 500 <= r.numel() <= 514
    assert torch.equal(synth.sample_rows(100), torch.arange(100))
