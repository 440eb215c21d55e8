"""GPU parity: libgdn.so (through its C ABI) against the fp64 oracle on the same
seeded inputs.

Tolerances are relative L2 errors over whole flattened tensors, computed separately
for outputs and states: <= 1e-4 for fp32 I/O (fp32 arithmetic throughout), <= 1e-2 for
bf16 I/O with fp32 state.  Max-abs error is reported in the assertion message.  The
full-size tests also bound every row (token and V head of the output, sequence and V
head of the state) on its own, so that a few wrong rows cannot hide in the norm.
Full-size workloads compare a sample of heads: every (sequence, V head) recurrence is
independent, so the oracle on a subset of QK heads (and the V heads that read them) is
an exact sample of the full result.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_layer_gated_b200 import gdn, inputs
from parity_util import TOL_BF16, TOL_F32, TOL_ROW_BF16, assert_close, assert_rows_close, errs  # noqa: F401

pytestmark = pytest.mark.gpu

ALGOS = [gdn.GDN_ALGO_SIMT, gdn.GDN_ALGO_TENSOR]


def run_prefill(x, algo, want_final=True):
    """Runs the prefill and checks that no bounded device wait gave up."""
    try:
        ws = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo), x["q"].device)
        res = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                          x["initial_state"], want_final, algo=algo, workspace=ws)
    except gdn.GdnError as e:
        if e.code == 9:
            pytest.skip("algorithm not available for these inputs")
        raise
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_OK"
    return res


def to_dev(x, dev="cuda"):
    return {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in x.items()}


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("ntok", [1, 2, 3, 4])
def test_decode_full_batch_matches_oracle(ntok):
    w = inputs.workload("decode")
    x = inputs.make_decode(w.num_seqs, ntok, seed=w.seed, device="cuda")
    s_ref = x["state"].clone()
    o_ref, sn_ref = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], s_ref)
    st = x["state"].clone()
    out = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    torch.cuda.synchronize()
    assert_close(out, o_ref, TOL_BF16, "decode out ntok=%d" % ntok)
    assert_close(st, sn_ref, TOL_BF16, "decode state ntok=%d" % ntok)
    assert_rows_close(out, o_ref, 3, TOL_ROW_BF16, "decode out rows ntok=%d" % ntok)
    assert_rows_close(st, sn_ref, 2, TOL_ROW_BF16, "decode state rows ntok=%d" % ntok)
    assert gdn.STATUS[gdn.gdn_get_decode_device_error()] == "GDN_OK"


def test_decode_fp32_io_tight():
    x = inputs.make_decode(8, 4, hk=4, hv=8, io_dtype=torch.float32, seed=11, device="cuda")
    o_ref, sn_ref = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    st = x["state"].clone()
    out = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    assert_close(out, o_ref, TOL_F32, "decode fp32 out")
    assert_close(st, sn_ref, TOL_F32, "decode fp32 state")


def test_decode_four_tokens_equals_four_single_steps_and_prefill():
    x = inputs.make_decode(16, 4, hk=4, hv=8, io_dtype=torch.float32, seed=12, device="cuda")
    s4 = x["state"].clone()
    o4 = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], s4)
    s1 = x["state"].clone()
    for t in range(4):
        sl = lambda a: a[:, t:t + 1].contiguous()  # noqa: E731
        o1 = gdn.decode(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]), s1)
        assert_close(o1[:, 0], o4[:, t].double().cpu().numpy(), 1e-5, "decode step %d" % t)
    assert_close(s1, s4.double().cpu().numpy(), 1e-5, "decode state 4x1 vs 4")
    N = 16
    cu = torch.arange(0, 4 * N + 1, 4, dtype=torch.int32, device="cuda")
    flat = lambda a: a.reshape(N * 4, *a.shape[2:]).contiguous()  # noqa: E731
    op, sp = gdn.prefill(flat(x["q"]), flat(x["k"]), flat(x["v"]), flat(x["g"]), flat(x["beta"]),
                         cu, x["state"], algo=gdn.GDN_ALGO_SIMT)
    assert_close(op.reshape(N, 4, 8, 128), o4.double().cpu().numpy(), 1e-5, "decode vs prefill out")
    assert_close(sp, s4.double().cpu().numpy(), 1e-5, "decode vs prefill state")


# ------------------------------------------------------------------ speculative verify
@pytest.mark.parametrize("ntok", [1, 2, 3, 4])
def test_verify_snapshots_match_oracle_and_keep_state(ntok):
    x = inputs.make_decode(32, ntok, hk=4, hv=8, seed=40 + ntok, device="cuda")
    st = x["state"].clone()
    out_v, snaps = gdn.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    torch.cuda.synchronize()
    torch.testing.assert_close(st, x["state"], rtol=0, atol=0)  # verify leaves the state alone
    st_d = x["state"].clone()
    out_d = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], st_d)
    if ntok == 1:  # one kernel serves both: the same operations
        torch.testing.assert_close(out_v, out_d, rtol=0, atol=0)
        torch.testing.assert_close(snaps[:, 0], st_d, rtol=0, atol=0)
    else:  # decode has its own kernel for 2..4 tokens: the same values up to fp32 rounding order
        assert_close(out_v, out_d.double().cpu().numpy(), 5e-3, "verify vs decode out ntok=%d" % ntok)
        assert_close(snaps[:, ntok - 1], st_d.double().cpu().numpy(), 1e-5, "last snapshot vs decode state")
    for t in range(ntok):  # snapshot t = the oracle's state after tokens 0..t
        sl = lambda a: a[:, : t + 1].contiguous()  # noqa: E731
        _, s_ref = oracle.decode(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]), x["state"])
        assert_close(snaps[:, t], s_ref, TOL_BF16, "verify snapshot %d of %d" % (t, ntok))
    assert gdn.STATUS[gdn.gdn_get_decode_device_error()] == "GDN_OK"


def test_commit_installs_the_accepted_snapshot():
    ntok = 4
    x = inputs.make_decode(40, ntok, hk=4, hv=8, seed=45, device="cuda")
    st = x["state"].clone()
    _, snaps = gdn.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], st)
    accepted = torch.tensor([i % (ntok + 2) - (1 if i % 7 == 0 else 0) for i in range(40)],
                            dtype=torch.int32, device="cuda")  # 0..ntok, plus -1 and ntok+1
    gdn.gdn_decode_commit(st, snaps, accepted)
    torch.cuda.synchronize()
    for n in range(40):
        a = int(accepted[n])
        want = snaps[n, a - 1] if 1 <= a <= ntok else x["state"][n]
        torch.testing.assert_close(st[n], want, rtol=0, atol=0)


# ------------------------------------------------------------------ state-slot indirection
def _slot_table(n, num_slots, seed):
    """Distinct slots for n sequences from a pool of num_slots (a permutation, so the pool
    order differs from the sequence order); every 5th one is outside [0, num_slots) in one
    of three ways: -1, num_slots itself, or far beyond it."""
    gen = torch.Generator().manual_seed(seed)
    slots = torch.randperm(num_slots, generator=gen)[:n].to(torch.int32)
    bad = [-1, num_slots, num_slots + 1000]
    for i, j in enumerate(range(0, n, 5)):
        slots[j] = bad[i % 3]
    return slots.cuda()


def test_decode_verify_commit_through_slots_match_dense():
    N, ntok, S = 20, 3, 48
    x = inputs.make_decode(N, ntok, hk=4, hv=8, seed=50, device="cuda")
    pool = torch.randn(S, 8, 128, 128, device="cuda") * 0.02
    slots = _slot_table(N, S, 51)
    valid = (slots >= 0) & (slots < S)
    dense = torch.zeros_like(x["state"])
    dense[valid] = pool[slots[valid].long()]
    # decode step in place on the pool
    p1 = pool.clone()
    out_s = torch.full_like(x["v"], float("nan"))
    gdn.gdn_decode_step_slots(x["q"], x["k"], x["v"], x["g"], x["beta"], p1, slots, out_s)
    d1 = dense.clone()
    out_d = gdn.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], d1)
    torch.cuda.synchronize()
    torch.testing.assert_close(out_s[valid], out_d[valid], rtol=0, atol=0)
    assert torch.isnan(out_s[~valid]).all()  # sequences without a slot are skipped
    # against the definition: the oracle run on the states the slot table names
    sel = lambda a: a[valid]  # noqa: E731
    o_ref, s_ref = oracle.decode(sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]), sel(x["beta"]),
                                 pool[slots[valid].long()])
    assert_close(out_s[valid], o_ref, TOL_BF16, "decode through slots out vs oracle")
    assert_close(p1[slots[valid].long()], s_ref, TOL_BF16, "decode through slots state vs oracle")
    torch.testing.assert_close(p1[slots[valid].long()], d1[valid], rtol=0, atol=0)
    untouched = torch.ones(S, dtype=torch.bool, device="cuda")
    untouched[slots[valid].long()] = False
    torch.testing.assert_close(p1[untouched], pool[untouched], rtol=0, atol=0)
    # verify reads the pool, commit writes the accepted snapshot back into it
    p2 = pool.clone()
    out_v = torch.empty_like(x["v"])
    snaps = torch.empty(N, ntok, 8, 128, 128, device="cuda")
    gdn.gdn_decode_verify_slots(x["q"], x["k"], x["v"], x["g"], x["beta"], p2, slots, out_v, snaps)
    torch.testing.assert_close(p2, pool, rtol=0, atol=0)
    # verify's kernel differs from the 3-token decode's: the same values up to fp32 rounding order
    assert_close(out_v[valid], out_d[valid].double().cpu().numpy(), 5e-3, "verify vs decode through slots")
    accepted = torch.tensor([n % (ntok + 1) for n in range(N)], dtype=torch.int32, device="cuda")
    gdn.gdn_decode_commit_slots(p2, slots, snaps, accepted)
    torch.cuda.synchronize()
    for n in range(N):
        a, sl = int(accepted[n]), int(slots[n])
        if not 0 <= sl < S:
            continue
        want = snaps[n, a - 1] if a >= 1 else pool[sl]
        torch.testing.assert_close(p2[sl], want, rtol=0, atol=0)


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_through_slots_matches_dense(algo):
    lens = [70, 0, 130, 64, 1, 200]
    x = inputs.make_prefill(lens, hk=2, hv=4, state_std=0.02, seed=52, device="cuda")
    N, S = len(lens), 16
    pool = torch.randn(S, 4, 128, 128, device="cuda") * 0.02
    slots = _slot_table(N, S, 53)
    valid = (slots >= 0) & (slots < S)
    init = torch.zeros(N, 4, 128, 128, device="cuda")
    init[valid] = pool[slots[valid].long()]
    out_d, fin_d = run_prefill(dict(x, initial_state=init), algo)
    p1 = pool.clone()
    out_s = torch.empty_like(x["v"])
    try:
        gdn.gdn_chunk_prefill_slots(x["q"], x["k"], x["v"], x["g"], x["beta"], p1, slots, x["cu_seqlens"],
                                    out_s, algo=algo)
    except gdn.GdnError as e:
        if e.code == 9:
            pytest.skip("algorithm not available")
        raise
    torch.cuda.synchronize()
    torch.testing.assert_close(out_s, out_d, rtol=0, atol=0)
    torch.testing.assert_close(p1[slots[valid].long()], fin_d[valid], rtol=0, atol=0)
    # against the definition: sequences with a slot start from the pool row it names,
    # the others from zeros
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], init)
    tol = TOL_F32 if x["q"].dtype == torch.float32 else TOL_BF16
    assert_close(out_s, o_ref, tol, "prefill through slots out vs oracle")
    assert_close(p1[slots[valid].long()], s_ref[valid.cpu().numpy()], tol, "prefill through slots state vs oracle")
    untouched = torch.ones(S, dtype=torch.bool, device="cuda")
    untouched[slots[valid].long()] = False
    torch.testing.assert_close(p1[untouched], pool[untouched], rtol=0, atol=0)


# ------------------------------------------------------------------ chunk-boundary states
@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_chunk_states_match_oracle_prefixes(algo):
    lens = [70, 0, 130, 64]
    x = inputs.make_prefill(lens, hk=2, hv=4, state_std=0.02, seed=54, device="cuda")
    nchunks = sum((L + 63) // 64 for L in lens)
    cst = torch.full((nchunks, 4, 128, 128), float("nan"), device="cuda")
    out = torch.empty_like(x["v"])
    fin = torch.empty_like(x["initial_state"])
    try:
        gdn.gdn_chunk_prefill_chunk_states(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"],
                                           x["cu_seqlens"], out, fin, cst, algo=algo)
    except gdn.GdnError as e:
        if e.code == 9:
            pytest.skip("algorithm not available")
        raise
    torch.cuda.synchronize()
    out_ref, _ = run_prefill(x, algo)
    torch.testing.assert_close(out, out_ref, rtol=0, atol=0)  # outputs unchanged by the extra writes
    tol = TOL_F32 if x["q"].dtype == torch.float32 else TOL_BF16
    cu = x["cu_seqlens"].cpu().tolist()
    row = 0
    for n, L in enumerate(lens):
        for c in range((L + 63) // 64):
            end = cu[n] + min(64 * (c + 1), L)
            sl = slice(cu[n], end)
            cu1 = torch.tensor([0, end - cu[n]], dtype=torch.int32)
            _, s_ref = oracle.forward(x["q"][sl], x["k"][sl], x["v"][sl], x["g"][sl], x["beta"][sl], cu1,
                                      x["initial_state"][n:n + 1])
            assert_close(cst[row], s_ref[0], tol, "chunk state %d (sequence %d, chunk %d)" % (row, n, c))
            if 64 * (c + 1) >= L:
                torch.testing.assert_close(cst[row], fin[n], rtol=0, atol=0)
            row += 1
    assert row == nchunks


# ------------------------------------------------------------------ prefill, small
def test_prefill_tiny_fp32_matches_oracle():
    x = inputs.make(inputs.workload("tiny"), device="cuda")
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], None)
    out, fin = run_prefill(x, gdn.GDN_ALGO_AUTO)
    torch.cuda.synchronize()
    assert_close(out, o_ref, TOL_F32, "tiny out")
    assert_close(fin, s_ref, TOL_F32, "tiny final state")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_prefill_ragged_varlen_with_states(algo, io):
    if algo == gdn.GDN_ALGO_TENSOR and io == torch.float32:
        pytest.skip("tensor-core path is bf16 I/O only")
    lens = [1, 63, 64, 65, 0, 200, 129, 7]
    x = inputs.make_prefill(lens, hk=2, hv=4, io_dtype=io, state_std=0.02, seed=21, device="cuda")
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                  x["initial_state"])
    out, fin = run_prefill(x, algo)
    torch.cuda.synchronize()
    tol = TOL_F32 if io == torch.float32 else TOL_BF16
    assert_close(out, o_ref, tol, "ragged out")
    assert_close(fin, s_ref, tol, "ragged final state")
    # an empty sequence hands its initial state through unchanged
    torch.testing.assert_close(fin[4], x["initial_state"][4], rtol=0, atol=0)


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_full_heads_small_T(algo):
    x = inputs.make_prefill([300], seed=22, device="cuda")
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], None)
    out, fin = run_prefill(x, algo)
    assert_close(out, o_ref, TOL_BF16, "16/32 heads out")
    assert_close(fin, s_ref, TOL_BF16, "16/32 heads state")


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_in_place_state_carry(algo):
    x = inputs.make_prefill([70, 130], hk=2, hv=4, state_std=0.02, seed=23, device="cuda")
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                  x["initial_state"])
    st = x["initial_state"].clone()
    out = torch.empty_like(x["v"])
    try:
        gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], st, x["cu_seqlens"], out,
                              st, algo=algo)
    except gdn.GdnError as e:
        if e.code == 9:
            pytest.skip("algorithm not available")
        raise
    assert_close(out, o_ref, TOL_BF16, "in-place out")
    assert_close(st, s_ref, TOL_BF16, "in-place state")


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_paired_heads_identical(algo):
    x = inputs.make_prefill([150], hk=2, hv=4, seed=24, device="cuda")
    for a in ("v", "g", "beta"):
        x[a][:, 1] = x[a][:, 0]
    out, fin = run_prefill(x, algo)
    torch.testing.assert_close(out[:, 1], out[:, 0], rtol=0, atol=0)
    torch.testing.assert_close(fin[:, 1], fin[:, 0], rtol=0, atol=0)


@pytest.mark.parametrize("lens", [[700], [130, 1, 300]])
def test_split_entry_points_match_one_call_and_oracle(lens):
    """gdn_chunk_prefill_prep + gdn_chunk_prefill_state (two launches, a workspace slot per
    chunk) against one gdn_chunk_prefill call (here the one-launch pass with its record ring):
    the same operations, so the same bits; and both against the oracle."""
    x = inputs.make_prefill(lens, hk=4, hv=8, state_std=0.02, seed=60, device="cuda")
    N = len(lens)
    shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"])
    assert gdn.gdn_prefill_phase_workspace_bytes(shape) >= gdn.gdn_prefill_workspace_bytes(shape)
    ws = gdn.alloc_workspace(shape, "cuda", phases=True)
    out_p = torch.full_like(x["v"], float("nan"))
    fin_p = torch.full((N, 8, 128, 128), float("nan"), device="cuda")
    gdn.gdn_chunk_prefill_prep(x["q"], x["k"], x["g"], x["beta"], x["cu_seqlens"], ws, x["v"])
    gdn.gdn_chunk_prefill_state(x["k"], x["v"], x["initial_state"], x["cu_seqlens"], out_p, fin_p, ws)
    out_1, fin_1 = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], x["initial_state"])
    torch.cuda.synchronize()
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_OK"
    torch.testing.assert_close(out_p, out_1, rtol=0, atol=0)
    torch.testing.assert_close(fin_p, fin_1, rtol=0, atol=0)
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], x["initial_state"])
    assert_close(out_p, o_ref, TOL_BF16, "split prefill out")
    assert_close(fin_p, s_ref, TOL_BF16, "split prefill state")


def test_device_error_word_is_clear_after_prefill():
    x = inputs.make_prefill([100], hk=2, hv=4, seed=25, device="cuda")
    ws = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"]), "cuda")
    gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], workspace=ws)
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK


def test_graph_capture_replays_prefill_and_decode():
    x = inputs.make_prefill([64, 100], hk=2, hv=4, state_std=0.02, seed=26, device="cuda")
    out = torch.empty_like(x["v"])
    fin = torch.empty_like(x["initial_state"])
    ws = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"]), "cuda")
    d = inputs.make_decode(4, 2, hk=2, hv=4, seed=27, device="cuda")
    st0 = d["state"].clone()
    st = d["state"].clone()
    dout = torch.empty_like(d["v"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"],
                                  x["cu_seqlens"], out, fin, workspace=ws, stream=s)
            gdn.gdn_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], st, dout, stream=s)
    st.copy_(st0)
    graph.replay()
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                  x["initial_state"])
    assert_close(out, o_ref, TOL_BF16, "graph prefill out")
    assert_close(fin, s_ref, TOL_BF16, "graph prefill state")
    do_ref, ds_ref = oracle.decode(d["q"], d["k"], d["v"], d["g"], d["beta"], st0)
    assert_close(dout, do_ref, TOL_BF16, "graph decode out")
    assert_close(st, ds_ref, TOL_BF16, "graph decode state")
    del graph


# ------------------------------------------------------------------ full-size workloads
@pytest.mark.parametrize("algo", ALGOS)
def test_layer_prefill_8192_sampled_heads(algo):
    w = inputs.workload("layer_prefill")
    x = inputs.make(w, device="cuda")
    out, fin = run_prefill(x, algo)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()
    heads = [0, 7, 15]
    o_ref, s_ref, vh = oracle.forward_heads(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                            x["cu_seqlens"], heads)
    assert_close(out[:, vh], o_ref, TOL_BF16, "T=8192 out (sampled heads)")
    assert_close(fin[:, vh], s_ref, TOL_BF16, "T=8192 state (sampled heads)")
    assert_rows_close(out[:, vh], o_ref, 2, TOL_ROW_BF16, "T=8192 out rows")
    assert_rows_close(fin[:, vh], s_ref, 2, TOL_ROW_BF16, "T=8192 state rows")


@pytest.mark.parametrize("algo", ALGOS)
def test_varlen_8_sequences_sampled_heads(algo):
    w = inputs.workload("varlen")
    x = inputs.make(w, device="cuda")
    out, fin = run_prefill(x, algo)
    torch.cuda.synchronize()
    heads = [3, 12]
    o_ref, s_ref, vh = oracle.forward_heads(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                            x["cu_seqlens"], heads, x["initial_state"])
    assert_close(out[:, vh], o_ref, TOL_BF16, "varlen out (sampled heads)")
    assert_close(fin[:, vh], s_ref, TOL_BF16, "varlen state (sampled heads)")
    assert_rows_close(out[:, vh], o_ref, 2, TOL_ROW_BF16, "varlen out rows")
    assert_rows_close(fin[:, vh], s_ref, 2, TOL_ROW_BF16, "varlen state rows (sequence, head)")


@pytest.mark.parametrize("algo", ALGOS)
def test_long_context_split_carry_and_sampled_heads(algo):
    w = inputs.workload("long")
    x = inputs.make(w, device="cuda")
    out, fin = run_prefill(x, algo)
    torch.cuda.synchronize()
    # 4 segments of 65536 with the state carried in place
    T = x["q"].shape[0]
    seg = T // 4
    st = torch.zeros_like(fin)
    out_s = torch.empty_like(out)
    for s in range(4):
        sl = slice(s * seg, (s + 1) * seg)
        cu = torch.tensor([0, seg], dtype=torch.int32, device="cuda")
        gdn.gdn_chunk_prefill(x["q"][sl], x["k"][sl], x["v"][sl], x["g"][sl], x["beta"][sl],
                              st, cu, out_s[sl], st, algo=algo)
    torch.cuda.synchronize()
    # 65536 is a multiple of the chunk size: every chunk of the split run sees the same tokens
    # and the carried fp32 state, so both paths do the same arithmetic as the whole run
    torch.testing.assert_close(out_s, out, rtol=0, atol=0)
    torch.testing.assert_close(st, fin, rtol=0, atol=0)
    heads = [5]
    o_ref, s_ref, vh = oracle.forward_heads(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                            x["cu_seqlens"], heads)
    assert_close(out[:, vh], o_ref, TOL_BF16, "T=262144 out (sampled heads)")
    assert_close(fin[:, vh], s_ref, TOL_BF16, "T=262144 state (sampled heads)")
    assert_rows_close(out[:, vh], o_ref, 2, TOL_ROW_BF16, "T=262144 out rows")
    assert_rows_close(fin[:, vh], s_ref, 2, TOL_ROW_BF16, "T=262144 state rows")


def test_bounded_wait_expiry_is_reported_and_context_survives():
    """Device waits that nothing completes (an inter-CTA flag, a pair of ring marks and an
    mbarrier phase) give up after their limit, record the timeout in the workspace header
    and return; the next calls still work."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    gdn.gdn_selftest_wait_timeout(ws, limit_us=20000)
    b.record()
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_ERR_DEVICE_TIMEOUT"
    assert a.elapsed_time(b) >= 3 * 20.0 * 0.9  # each of the three waits ran to its 20 ms limit
    x = inputs.make_prefill([80], hk=2, hv=4, seed=28, device="cuda")
    ws2 = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"]), "cuda")
    out, fin = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], workspace=ws2)
    assert gdn.gdn_get_device_error(ws2) == gdn.GDN_OK
    o_ref, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], None)
    assert_close(out, o_ref, TOL_BF16, "prefill after a reported timeout")


# ------------------------------------------------------------------ poisoned buffers
# Outputs and states sit inside NaN-filled buffers with a guard row on each side: every
# element a call owns must be written (finite and matching the oracle) and nothing outside
# it touched.  The prefill workspace starts as 0xFF bytes (NaN in fp32 and bf16), so an
# operand image the kernels forget to write shows up as NaN in the results.
NAN = float("nan")


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_writes_exactly_its_outputs(algo):
    lens = [65, 0, 130, 1, 64]
    hv = 4
    x = inputs.make_prefill(lens, hk=2, hv=hv, state_std=0.02, seed=61, device="cuda")
    T, N = x["q"].shape[0], len(lens)
    out_buf = torch.full((T + 2, hv, 128), NAN, dtype=x["v"].dtype, device="cuda")
    fin_buf = torch.full((N + 2, hv, 128, 128), NAN, device="cuda")
    out, fin = out_buf[1:T + 1], fin_buf[1:N + 1]
    ws = gdn.alloc_workspace(gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo), "cuda")
    ws.fill_(0xFF)
    try:
        gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"],
                              x["cu_seqlens"], out, fin, workspace=ws, algo=algo)
    except gdn.GdnError as e:
        if e.code == 9:
            pytest.skip("algorithm not available for these inputs")
        raise
    torch.cuda.synchronize()
    assert gdn.STATUS[gdn.gdn_get_device_error(ws)] == "GDN_OK"
    for guard in (out_buf[0], out_buf[-1], fin_buf[0], fin_buf[-1]):
        assert torch.isnan(guard).all(), "a write outside the output buffers"
    assert torch.isfinite(out).all() and torch.isfinite(fin).all(), "an output element left unwritten"
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                  x["initial_state"])
    assert_close(out, o_ref, TOL_BF16, "poisoned prefill out")
    assert_close(fin, s_ref, TOL_BF16, "poisoned prefill state")


@pytest.mark.parametrize("ntok", [1, 3, 4])
def test_decode_and_verify_write_exactly_their_outputs(ntok):
    N, hv = 6, 8
    x = inputs.make_decode(N, ntok, hk=4, hv=hv, seed=62 + ntok, device="cuda")
    st_buf = torch.full((N + 2, hv, 128, 128), NAN, device="cuda")
    st_buf[1:N + 1] = x["state"]
    out_buf = torch.full((N + 2, ntok, hv, 128), NAN, dtype=x["v"].dtype, device="cuda")
    st, out = st_buf[1:N + 1], out_buf[1:N + 1]
    gdn.gdn_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], st, out)
    torch.cuda.synchronize()
    for guard in (st_buf[0], st_buf[-1], out_buf[0], out_buf[-1]):
        assert torch.isnan(guard).all(), "a write outside the decode buffers"
    assert torch.isfinite(out).all() and torch.isfinite(st).all()
    o_ref, s_ref = oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    assert_close(out, o_ref, TOL_BF16, "poisoned decode out")
    assert_close(st, s_ref, TOL_BF16, "poisoned decode state")
    # verify: the snapshots too
    snap_buf = torch.full((N + 2, ntok, hv, 128, 128), NAN, device="cuda")
    out_buf.fill_(NAN)
    snaps = snap_buf[1:N + 1]
    gdn.gdn_decode_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"], out, snaps)
    torch.cuda.synchronize()
    for guard in (snap_buf[0], snap_buf[-1], out_buf[0], out_buf[-1]):
        assert torch.isnan(guard).all(), "a write outside the verify buffers"
    assert torch.isfinite(snaps).all() and torch.isfinite(out).all()
    assert_close(snaps[:, ntok - 1], s_ref, TOL_BF16, "poisoned verify last snapshot")


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_more_than_1024_sequences(algo):
    """More sequences than one thread block of the chunk-table scan covers: the scan runs
    in several batches with a carry, and the chunk entries are found in global memory."""
    gen = np.random.default_rng(70)
    lens = [int(x) for x in gen.integers(0, 140, size=1100)]
    lens[5] = 0
    lens[1023] = 64
    x = inputs.make_prefill(lens, hk=2, hv=4, state_std=0.02, seed=71, device="cuda")
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                  x["initial_state"])
    out, fin = run_prefill(x, algo)
    torch.cuda.synchronize()
    assert_close(out, o_ref, TOL_BF16, "1100 sequences out")
    assert_close(fin, s_ref, TOL_BF16, "1100 sequences final state")
    torch.testing.assert_close(fin[5], x["initial_state"][5], rtol=0, atol=0)
