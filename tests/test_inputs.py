"""The seeded input recipe shared by the oracle and the CUDA path (CPU only)."""
import pytest
import torch

from linear_attention_layer_gated_b200 import inputs


def test_workload_specs_follow_the_recipe():
    t = inputs.workload("tiny")
    assert (t.seqlens, t.hk, t.hv, t.d, t.io_dtype, t.gate, t.seed) == ([256], 2, 4, 128, torch.float32, "uniform", 0)
    lp = inputs.workload("layer_prefill")
    assert (lp.seqlens, lp.hk, lp.hv, lp.io_dtype, lp.state_std, lp.seed) == ([8192], 16, 32, torch.bfloat16, None, 1)
    vl = inputs.workload("varlen")
    assert (vl.num_seqs, vl.varlen_range, vl.state_std, vl.seed) == (8, (1024, 16384), 0.02, 2)
    d1, d4 = inputs.workload("decode"), inputs.workload("decode_verify")
    assert (d1.num_seqs, d1.ntok, d4.num_seqs, d4.ntok, d1.seed, d4.seed) == (256, 1, 256, 4, 3, 3)
    lg = inputs.workload("long")
    assert (lg.seqlens, lg.seed) == ([262144], 4)
    with pytest.raises(KeyError):
        inputs.workload("nope")


def _check_gates(g, beta, kind):
    assert g.dtype == torch.float32 and beta.dtype == torch.float32
    assert (g <= 0).all()
    if kind == "uniform":
        assert (g >= -0.1).all()
    assert ((beta > 0) & (beta < 1)).all()


def test_tiny_inputs():
    x = inputs.make(inputs.workload("tiny"))
    assert x["q"].shape == (256, 2, 128) and x["v"].shape == (256, 4, 128)
    assert x["q"].dtype == torch.float32
    assert x["initial_state"] is None
    assert x["cu_seqlens"].tolist() == [0, 256] and x["cu_seqlens"].dtype == torch.int32
    _check_gates(x["g"], x["beta"], "uniform")


def test_layer_prefill_inputs():
    x = inputs.make(inputs.workload("layer_prefill"))
    assert x["q"].shape == (8192, 16, 128) and x["k"].shape == (8192, 16, 128)
    assert x["v"].shape == (8192, 32, 128) and x["g"].shape == (8192, 32)
    assert x["q"].dtype == torch.bfloat16
    _check_gates(x["g"], x["beta"], "softplus")
    # q, k, v ~ N(0, 1): moments of a large sample
    assert abs(x["v"].float().mean().item()) < 0.01 and abs(x["v"].float().std().item() - 1) < 0.01


def test_varlen_lengths_and_states():
    # the lengths are the generator's first draw, so fewer heads leave them unchanged
    x = inputs.make(inputs.workload("varlen"), hk=1, hv=1)
    lens = x["seqlens"]
    assert len(lens) == 8 and all(1024 <= n <= 16384 for n in lens)
    cu = x["cu_seqlens"].tolist()
    assert cu[0] == 0 and all(cu[i + 1] - cu[i] == lens[i] for i in range(8))
    assert x["initial_state"].shape == (8, 1, 128, 128)
    assert abs(x["initial_state"].std().item() - 0.02) < 0.001
    full = inputs.make_prefill(None, hk=2, hv=2, seed=2, num_seqs=8, varlen_range=(1024, 16384))
    assert full["seqlens"] == lens


def test_decode_inputs():
    x = inputs.make(inputs.workload("decode_verify"))
    assert x["q"].shape == (256, 4, 16, 128) and x["v"].shape == (256, 4, 32, 128)
    assert x["g"].shape == (256, 4, 32) and x["state"].shape == (256, 32, 128, 128)
    _check_gates(x["g"], x["beta"], "softplus")
    assert abs(x["state"].std().item() - 0.02) < 0.0005


def test_seeded_draws_are_reproducible():
    a = inputs.make_prefill([70, 5], hk=2, hv=4, seed=9)
    b = inputs.make_prefill([70, 5], hk=2, hv=4, seed=9)
    c = inputs.make_prefill([70, 5], hk=2, hv=4, seed=10)
    for key in ("q", "k", "v", "g", "beta"):
        assert torch.equal(a[key], b[key])
    assert not torch.equal(a["q"], c["q"])
