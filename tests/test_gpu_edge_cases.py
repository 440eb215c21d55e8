"""GPU parity on the degenerate and extreme inputs the gated delta rule allows, the same
special cases that pin the oracle on the CPU, run through both prefill paths, the decode
step and the speculative verify, and compared with the fp64 oracle element by element.

The rule (Gated DeltaNet; Qwen3-Next-80B-A3B model card, "Highlights" and "Model
Overview"): S_t = exp(g_t) S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t.

Cases, each on ragged sequences that span several 64-token chunks:
  beta_zero      b = 0: the state only decays, S_T = exp(sum g) S_0 (closed form checked too)
  unit_keys      g = 0, b = 1, keys distinct standard basis vectors: I + A is furthest from
                 the identity; every step writes v_t into column k_t of S exactly
  repeated_keys  one key for every token of a sequence (per QK head), g = 0, b = 1
  colinear_keys  k_t = c_t k_0 with random sign and scale: normalised keys are +-k_0
  strong_decay   15% of the tokens have g in [-20, -5]: exp(G_r - G_j) and the chunk's
                 cumulative decay underflow inside a chunk
  beta_extremes  b = 1e-4 or 1 - 1e-4 at random
  repeated_b099  repeated keys with g = 0 and b = 0.99: T's entries are not exact in bf16, so any
                 product of T that feeds a cancelling sum must keep more than bf16's 8 bits
  colinear_b097  colinear keys with g = 0 and b = 0.97
"""

import pytest
import torch

import oracle
from linear_attention_layer_gated_b200 import gdn, inputs
from parity_util import TOL_BF16, TOL_F32, TOL_ROW_BF16, assert_close, assert_rows_close

pytestmark = pytest.mark.gpu

CASES = ["beta_zero", "unit_keys", "repeated_keys", "colinear_keys", "strong_decay", "beta_extremes",
         "repeated_b099", "colinear_b097"]
LENS = [70, 130, 1, 64, 200]
HK, HV = 2, 4


def special(x, case, seed):
    """Rewrites the gates and keys of a seeded input dict for one edge case.  Works on
    prefill tensors ([T, H, D] / [T, H]) and decode tensors ([N, m, H, D] / [N, m, H]);
    ``pos`` numbers every token within its sequence and ``first`` gives the flat index of
    its sequence's first token."""
    gen = torch.Generator().manual_seed(seed)
    dev = x["k"].device
    io = x["k"].dtype
    g, b, k = x["g"].cpu(), x["beta"].cpu(), x["k"].cpu().float()
    pos = x["pos"]
    if case == "beta_zero":
        b = torch.zeros_like(b)
    elif case in ("unit_keys", "repeated_keys", "colinear_keys", "repeated_b099", "colinear_b097"):
        g = torch.zeros_like(g)
        b = torch.full_like(b, {"repeated_b099": 0.99, "colinear_b097": 0.97}.get(case, 1.0))
        flat = k.reshape(-1, k.shape[-2], k.shape[-1])
        p = pos  # position of each token within its sequence
        if case == "unit_keys":
            flat.zero_()
            for hq in range(flat.shape[1]):
                col = (p + 37 * hq) % flat.shape[2]
                flat[torch.arange(flat.shape[0]), hq, col] = 2.0
        else:
            first = x["first"]  # index of the first token of each token's sequence
            base = flat[first].clone()
            if case.startswith("repeated"):
                flat.copy_(base)
            else:
                c = (torch.rand(flat.shape[0], flat.shape[1], 1, generator=gen) * 1.5 + 0.5)
                sign = torch.where(torch.rand(flat.shape[0], flat.shape[1], 1, generator=gen) < 0.5, -1.0, 1.0)
                flat.copy_(base * c * sign)
        k = flat.reshape(k.shape)
    elif case == "strong_decay":
        hit = torch.rand(g.shape, generator=gen) < 0.15
        g = torch.where(hit, -5.0 - 15.0 * torch.rand(g.shape, generator=gen), g)
    elif case == "beta_extremes":
        hi = torch.rand(b.shape, generator=gen) < 0.5
        b = torch.where(hi, torch.full_like(b, 1.0 - 1e-4), torch.full_like(b, 1e-4))
    else:
        raise KeyError(case)
    y = dict(x)
    y["g"], y["beta"], y["k"] = g.contiguous().to(dev), b.contiguous().to(dev), k.to(io).contiguous().to(dev)
    return y


def prefill_inputs(case, io, seed):
    x = inputs.make_prefill(LENS, hk=HK, hv=HV, io_dtype=io, state_std=0.05, seed=seed, device="cuda")
    cu = x["cu_seqlens"].cpu().tolist()
    pos = torch.cat([torch.arange(L) for L in LENS])
    first = torch.cat([torch.full((L,), cu[n], dtype=torch.long) for n, L in enumerate(LENS)])
    x["pos"], x["first"] = pos, first
    return special(x, case, seed + 1)


def run_prefill(x, algo):
    ws = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo), "cuda")
    out, fin = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], x["initial_state"],
                           algo=algo, workspace=ws)
    torch.cuda.synchronize()
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_OK"
    return out, fin


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("algo,io", [(gdn.GDN_ALGO_TENSOR, torch.bfloat16), (gdn.GDN_ALGO_SIMT, torch.bfloat16),
                                     (gdn.GDN_ALGO_SIMT, torch.float32)])
def test_prefill_edge_case_matches_oracle(case, algo, io):
    x = prefill_inputs(case, io, seed=200 + CASES.index(case))
    out, fin = run_prefill(x, algo)
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], x["initial_state"])
    tol = TOL_F32 if io == torch.float32 else TOL_BF16
    what = "%s algo=%d %s" % (case, algo, str(io).split(".")[-1])
    assert_close(out, o_ref, tol, what + " out")
    assert_close(fin, s_ref, tol, what + " state")
    if io == torch.bfloat16:
        assert_rows_close(out, o_ref, 2, TOL_ROW_BF16, what + " out rows")
        assert_rows_close(fin, s_ref, 2, TOL_ROW_BF16, what + " state rows")
    if case == "beta_zero":  # the closed form itself: S_T = exp(sum of the sequence's g) S_0
        cu = x["cu_seqlens"].cpu().tolist()
        g = x["g"].double().cpu()
        decay = torch.stack([g[cu[n]:cu[n + 1]].sum(0) for n in range(len(LENS))]).exp()
        closed = decay[:, :, None, None] * x["initial_state"].double().cpu()
        assert_close(fin, closed.numpy(), tol, what + " state vs closed form")


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_decode_and_verify_edge_case_match_oracle(case, io):
    N, ntok = 24, 4
    x = inputs.make_decode(N, ntok, hk=HK, hv=HV, io_dtype=io, state_std=0.05, seed=300 + CASES.index(case),
                           device="cuda")
    x["pos"] = torch.arange(ntok).repeat(N)
    x["first"] = torch.arange(N).repeat_interleave(ntok) * ntok
    x = special(x, case, 301 + CASES.index(case))
    st = x["state"].clone()
    out = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    out_v, snaps = gdn.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    tol = TOL_F32 if io == torch.float32 else TOL_BF16
    what = "decode %s %s" % (case, str(io).split(".")[-1])
    assert_close(out, o_ref, tol, what + " out")
    assert_close(st, s_ref, tol, what + " state")
    assert_close(out_v, o_ref, tol, what + " verify out")
    for t in range(ntok):
        sl = lambda a: a[:, : t + 1].contiguous()  # noqa: E731
        _, s_t = oracle.decode(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]), x["state"])
        assert_close(snaps[:, t], s_t, tol, what + " snapshot %d" % t)
