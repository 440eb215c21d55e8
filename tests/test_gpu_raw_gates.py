"""GPU parity of the raw-gate entry points (gates given as projections: g = -a softplus(x + b),
beta = sigmoid(y), per V head, applied inside the kernels) against the fp64 oracle's
activation followed by its recurrence, on the prefill paths, the decode step and the
speculative verify.  Each test also runs once with projections of scale 30, which drive
softplus and sigmoid into saturation (g down to about -12, beta exactly 0 or 1 in fp32).
"""

import pytest
import torch

import oracle
from linear_attention_layer_gated_b200 import gdn, inputs
from parity_util import TOL_BF16, TOL_F32, TOL_ROW_BF16, assert_close, assert_rows_close

pytestmark = pytest.mark.gpu

LENS = [70, 130, 1, 64, 200]  # several chunks and ragged tails
HK, HV = 2, 4


def raw_gates(shape, scale, seed):
    r = inputs.make_raw_gates(shape, HV, scale=scale, seed=seed, device="cuda")
    return r["x"], r["y"], r["a"], r["b"]


@pytest.mark.parametrize("scale", [1.0, 30.0])
@pytest.mark.parametrize("algo,io", [(gdn.GDN_ALGO_TENSOR, torch.bfloat16), (gdn.GDN_ALGO_SIMT, torch.bfloat16),
                                     (gdn.GDN_ALGO_SIMT, torch.float32)])
def test_prefill_raw_gates_match_oracle(algo, io, scale):
    x = inputs.make_prefill(LENS, hk=HK, hv=HV, io_dtype=io, state_std=0.05, seed=500, device="cuda")
    gx, gy, a, b = raw_gates((sum(LENS), HV), scale, seed=501)
    shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo)
    ws = gdn.alloc_workspace(shape, "cuda")
    out = torch.empty_like(x["v"])
    fin = torch.empty(len(LENS), HV, 128, 128, device="cuda")
    gdn.gdn_chunk_prefill_raw_gates(x["q"], x["k"], x["v"], gx, gy, a, b, x["initial_state"], x["cu_seqlens"],
                                    out, fin, workspace=ws, algo=algo)
    torch.cuda.synchronize()
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_OK"
    o_ref, s_ref = oracle.forward_from_projections(x["q"], x["k"], x["v"], gx, gy, a, b, x["cu_seqlens"],
                                                   x["initial_state"])
    tol = TOL_F32 if io == torch.float32 else TOL_BF16
    what = "raw gates prefill algo=%d %s scale=%g" % (algo, str(io).split(".")[-1], scale)
    assert_close(out, o_ref, tol, what + " out")
    assert_close(fin, s_ref, tol, what + " state")
    if io == torch.bfloat16:
        assert_rows_close(out, o_ref, 2, TOL_ROW_BF16, what + " out rows")
        assert_rows_close(fin, s_ref, 2, TOL_ROW_BF16, what + " state rows")


@pytest.mark.parametrize("scale", [1.0, 30.0])
def test_prefill_raw_gates_equal_activated_gates(scale):
    """The fused activation against the same recurrence fed the oracle's activated gates
    (rounded to fp32): the only difference is the fp32 activation, so the results agree far
    inside the bf16 tolerance."""
    x = inputs.make_prefill(LENS, hk=HK, hv=HV, state_std=0.05, seed=510, device="cuda")
    gx, gy, a, b = raw_gates((sum(LENS), HV), scale, seed=511)
    g, beta = oracle.gates_from_projections(gx, gy, a, b)
    g = torch.from_numpy(g).float().cuda()
    beta = torch.from_numpy(beta).float().cuda()
    out_r = torch.empty_like(x["v"])
    fin_r = torch.empty(len(LENS), HV, 128, 128, device="cuda")
    gdn.gdn_chunk_prefill_raw_gates(x["q"], x["k"], x["v"], gx, gy, a, b, x["initial_state"], x["cu_seqlens"],
                                    out_r, fin_r)
    out_a, fin_a = gdn.prefill(x["q"], x["k"], x["v"], g, beta, x["cu_seqlens"], x["initial_state"])
    torch.cuda.synchronize()
    assert_close(out_r, out_a.double().cpu().numpy(), 1e-3, "raw vs activated out scale=%g" % scale)
    assert_close(fin_r, fin_a.double().cpu().numpy(), 1e-4, "raw vs activated state scale=%g" % scale)


@pytest.mark.parametrize("scale", [1.0, 30.0])
@pytest.mark.parametrize("ntok", [1, 2, 3, 4])
@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_decode_and_verify_raw_gates_match_oracle(ntok, io, scale):
    N = 40
    x = inputs.make_decode(N, ntok, hk=HK, hv=HV, io_dtype=io, state_std=0.05, seed=520 + ntok, device="cuda")
    gx, gy, a, b = raw_gates((N, ntok, HV), scale, seed=530 + ntok)
    st = x["state"].clone()
    out = torch.empty_like(x["v"])
    gdn.gdn_decode_step_raw_gates(x["q"], x["k"], x["v"], gx, gy, a, b, st, out)
    out_v = torch.empty_like(x["v"])
    snaps = torch.empty(N, ntok, HV, 128, 128, device="cuda")
    gdn.gdn_decode_verify_raw_gates(x["q"], x["k"], x["v"], gx, gy, a, b, x["state"], out_v, snaps)
    torch.cuda.synchronize()
    assert gdn.STATUS[gdn.gdn_get_decode_device_error()] == "GDN_OK"
    o_ref, s_ref = oracle.decode_from_projections(x["q"], x["k"], x["v"], gx, gy, a, b, x["state"])
    tol = TOL_F32 if io == torch.float32 else TOL_BF16
    what = "raw gates decode ntok=%d %s scale=%g" % (ntok, str(io).split(".")[-1], scale)
    assert_close(out, o_ref, tol, what + " out")
    assert_close(st, s_ref, tol, what + " state")
    assert_close(out_v, o_ref, tol, what + " verify out")
    for t in range(ntok):
        sl = lambda z: z[:, : t + 1].contiguous()  # noqa: E731
        _, s_t = oracle.decode_from_projections(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(gx), sl(gy), a, b,
                                                x["state"])
        assert_close(snaps[:, t], s_t, tol, what + " snapshot %d" % t)
