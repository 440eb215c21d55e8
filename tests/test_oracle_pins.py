"""Pins for the fp64 oracle: closed forms, exact identities, invariants and brute
force that the gated delta rule fixes, independent of the oracle's own code.

The rule (Gated DeltaNet, Qwen3-Next-80B-A3B model card, "Highlights" / "Model
Overview"): S_t = exp(g_t) S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t,
with q, k L2-normalised and q scaled by 1/sqrt(d_k).

Every check uses inputs chosen so that the expected value needs none of the
oracle's steps retyped: unit or basis-vector keys and queries (normalisation is
then the identity), b = 0 or b = 1 and g = 0 special cases, and agreement with a
second formulation (numpy chunked closed form, LAPACK triangular solve).
"""

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle.chunked import chunked_forward

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rng(seed):
    return np.random.default_rng(seed)


def unit_rows(r, n, d):
    x = r.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def run1(q, k, v, g, b, s0=None, eps=0.0):
    """Oracle on one sequence, one QK head, one V head. q,k:[T,dk] v:[T,dv] g,b:[T]."""
    T = q.shape[0]
    out, fin = oracle.forward(q[:, None, :], k[:, None, :], v[:, None, :], g[:, None],
                              b[:, None], [0, T], None if s0 is None else s0[None, None],
                              eps=eps)
    return out[:, 0, :], fin[0, 0]


# ---------------------------------------------------------------- I1: beta = 0 closed form
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_beta_zero_only_decays(seed):
    r = rng(seed)
    T, dk, dv = 37, 16, 12
    S0 = r.standard_normal((dv, dk))
    g = -r.uniform(0, 0.3, T)
    cols = r.integers(0, dk, T)
    q = np.zeros((T, dk))
    q[np.arange(T), cols] = r.uniform(0.5, 3.0, T)   # q = c e_col  ->  q_hat = e_col / sqrt(dk)
    k = r.standard_normal((T, dk))
    v = r.standard_normal((T, dv))
    out, fin = run1(q, k, v, g, np.zeros(T), S0)
    G = np.cumsum(g)
    np.testing.assert_allclose(fin, np.exp(G[-1]) * S0, rtol=1e-13, atol=1e-15)
    expect = np.exp(G)[:, None] * S0[:, cols].T / np.sqrt(dk)
    np.testing.assert_allclose(out, expect, rtol=1e-13, atol=1e-15)


# ------------------------------------------------- I2: g = 0, b = 1, unit k -> S_t k_t = v_t
@pytest.mark.parametrize("seed", [0, 1])
def test_unit_key_writes_value_exactly(seed):
    r = rng(seed)
    T, d = 20, 32
    k = unit_rows(r, T, d)
    q = r.standard_normal((T, d))
    v = r.standard_normal((T, d))
    S = r.standard_normal((d, d)) * 0.1
    for t in range(T):
        _, S = run1(q[t:t + 1], k[t:t + 1], v[t:t + 1], np.zeros(1), np.ones(1), S)
        np.testing.assert_allclose(S @ k[t], v[t], rtol=0, atol=1e-12)


# ------------------------------------- I3: orthonormal keys replace columns of S by v_t
def test_basis_keys_replace_columns():
    r = rng(3)
    d, T = 24, 10
    perm = r.permutation(d)[:T]
    k = np.zeros((T, d))
    k[np.arange(T), perm] = r.uniform(0.2, 4.0, T)   # k = c e_perm -> k_hat = e_perm
    m = 5
    q = np.zeros((T, d))
    q[:, m] = 2.0                                    # q_hat = e_m / sqrt(d)
    v = r.standard_normal((T, d))
    S0 = r.standard_normal((d, d))
    out, fin = run1(q, k, v, np.zeros(T), np.ones(T), S0)
    expect = S0.copy()
    for t in range(T):
        expect[:, perm[t]] = v[t]
        np.testing.assert_allclose(out[t], expect[:, m] / np.sqrt(d), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fin, expect, rtol=1e-13, atol=1e-14)


# ------------------------------------------- q scaling and normalisation on a single token
def test_query_scaling_single_token():
    r = rng(4)
    d = 128
    S0 = r.standard_normal((d, d))
    for j in (0, 17, 127):
        q = np.zeros((1, d))
        q[0, j] = 7.5
        out, _ = run1(q, r.standard_normal((1, d)), r.standard_normal((1, d)),
                      np.zeros(1), np.zeros(1), S0)
        np.testing.assert_allclose(out[0], S0[:, j] / np.sqrt(d), rtol=1e-14)


def test_scale_invariance_of_q_and_k():
    r = rng(5)
    T, d = 30, 16
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    g, b = -r.uniform(0, 0.2, T), r.uniform(0.05, 0.95, T)
    o1, s1 = run1(q, k, v, g, b)
    sq, sk = r.uniform(0.1, 10, (T, 1)), r.uniform(0.1, 10, (T, 1))
    o2, s2 = run1(q * sq, k * sk, v, g, b)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s1, rtol=1e-12, atol=1e-13)


# ------------------------------- I4: brute force against the chunked closed form (numpy)
@pytest.mark.parametrize("d", [4, 8, 128])
@pytest.mark.parametrize("chunk", [1, 2, 16, 64, None])
def test_chunked_closed_form_matches_recurrence(d, chunk):
    r = rng(10 + d)
    T = 150 if d < 128 else 131
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    g = -r.uniform(0, 0.5, T)
    b = r.uniform(0.01, 0.99, T)
    S0 = r.standard_normal((d, d)) * 0.1
    o_ref, s_ref = run1(q, k, v, g, b, S0, eps=1e-6)
    o_ch, s_ch = chunked_forward(q, k, v, g, b, S0, chunk=chunk or T, eps=1e-6)
    np.testing.assert_allclose(o_ch, o_ref, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(s_ch, s_ref, rtol=1e-9, atol=1e-11)


def test_single_triangular_solve_zero_state():
    """With S0 = 0 and one chunk spanning the sequence, the outputs are
    (mask * decay * Q K^T) (I + A)^-1 diag(b) V -- one LAPACK triangular solve."""
    r = rng(20)
    T, d = 64, 8
    k = unit_rows(r, T, d)
    q = unit_rows(r, T, d) / np.sqrt(d)     # already the normalised, scaled query
    v = r.standard_normal((T, d))
    g = -r.uniform(0, 0.4, T)
    b = r.uniform(0.05, 0.95, T)
    G = np.cumsum(g)
    decay = np.exp(np.tril(G[:, None] - G[None, :]))
    A = np.tril(b[:, None] * decay * (k @ k.T), -1)
    P = np.tril(decay * (q @ k.T))
    U = scipy.linalg.solve_triangular(np.eye(T) + A, b[:, None] * v, lower=True,
                                      unit_diagonal=True)
    out, _ = run1(q * np.sqrt(d), k, v, g, b)   # oracle re-normalises: q*sqrt(d) has norm sqrt(d)
    np.testing.assert_allclose(out, P @ U, rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------- I5: affine in (S0, V)
def test_affine_in_initial_state():
    r = rng(30)
    T, d = 25, 12
    k = unit_rows(r, T, d)
    q, v = r.standard_normal((T, d)), r.standard_normal((T, d))
    g, b = -r.uniform(0, 0.3, T), r.uniform(0.05, 0.95, T)
    S0 = r.standard_normal((d, d))
    _, s_with = run1(q, k, v, g, b, S0)
    _, s_zero = run1(q, k, v, g, b, np.zeros((d, d)))
    M = np.eye(d)
    for t in range(T):
        M = M @ (np.exp(g[t]) * (np.eye(d) - b[t] * np.outer(k[t], k[t])))
    np.testing.assert_allclose(s_with - s_zero, S0 @ M, rtol=1e-11, atol=1e-12)


def test_linear_in_values_from_zero_state():
    r = rng(31)
    T, d = 40, 10
    q, k = r.standard_normal((T, d)), r.standard_normal((T, d))
    v1, v2 = r.standard_normal((T, d)), r.standard_normal((T, d))
    g, b = -r.uniform(0, 0.3, T), r.uniform(0.05, 0.95, T)
    o1, s1 = run1(q, k, v1, g, b)
    o2, s2 = run1(q, k, v2, g, b)
    o3, s3 = run1(q, k, 2.0 * v1 - 3.0 * v2, g, b)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s3, 2 * s1 - 3 * s2, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------- I6: row independence
def test_value_permutation_permutes_state_rows():
    r = rng(40)
    T, dk, dv = 33, 16, 20
    q, k, v = r.standard_normal((T, dk)), r.standard_normal((T, dk)), r.standard_normal((T, dv))
    g, b = -r.uniform(0, 0.3, T), r.uniform(0.05, 0.95, T)
    S0 = r.standard_normal((dv, dk))
    perm = r.permutation(dv)
    o1, s1 = run1(q, k, v, g, b, S0)
    o2, s2 = run1(q, k, v[:, perm], g, b, S0[perm])
    np.testing.assert_allclose(o2, o1[:, perm], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s2, s1[perm], rtol=1e-13, atol=1e-14)


# -------------------------------------------------------------------- I7: split & carry
def test_split_and_carry_equals_whole():
    r = rng(50)
    T, d = 97, 16
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    g, b = -r.uniform(0, 0.3, T), r.uniform(0.05, 0.95, T)
    S0 = r.standard_normal((d, d)) * 0.1
    o, s = run1(q, k, v, g, b, S0)
    cut = [0, 13, 64, 65, T]
    S = S0
    parts = []
    for a, c in zip(cut[:-1], cut[1:]):
        oo, S = run1(q[a:c], k[a:c], v[a:c], g[a:c], b[a:c], S)
        parts.append(oo)
    np.testing.assert_allclose(np.concatenate(parts), o, rtol=0, atol=0)
    np.testing.assert_allclose(S, s, rtol=0, atol=0)


# -------------------------------------------------------------------------- I8: varlen
def test_varlen_packing_equals_separate_runs():
    r = rng(60)
    lens = [5, 0, 64, 1, 70]
    HK, HV, d = 2, 4, 8
    T = sum(lens)
    q, k = r.standard_normal((T, HK, d)), r.standard_normal((T, HK, d))
    v = r.standard_normal((T, HV, d))
    g, b = -r.uniform(0, 0.3, (T, HV)), r.uniform(0.05, 0.95, (T, HV))
    S0 = r.standard_normal((len(lens), HV, d, d)) * 0.1
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    out, fin = oracle.forward(q, k, v, g, b, cu, S0)
    for n, (a, c) in enumerate(zip(cu[:-1], cu[1:])):
        o1, f1 = oracle.forward(q[a:c], k[a:c], v[a:c], g[a:c], b[a:c], [0, c - a], S0[n:n + 1])
        np.testing.assert_array_equal(out[a:c], o1)
        np.testing.assert_array_equal(fin[n], f1[0])
    # a zero-length sequence leaves its state untouched
    np.testing.assert_array_equal(fin[1], S0[1])


# ------------------------------------------------------------------------- I9: decode
def test_decode_steps_agree_with_prefill():
    r = rng(70)
    N, ntok, HK, HV, d = 3, 4, 2, 4, 16
    q, k = r.standard_normal((N, ntok, HK, d)), r.standard_normal((N, ntok, HK, d))
    v = r.standard_normal((N, ntok, HV, d))
    g, b = -r.uniform(0, 0.3, (N, ntok, HV)), r.uniform(0.05, 0.95, (N, ntok, HV))
    S0 = r.standard_normal((N, HV, d, d)) * 0.1
    o4, s4 = oracle.decode(q, k, v, g, b, S0)
    S = S0
    for t in range(ntok):
        o1, S = oracle.decode(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1],
                              b[:, t:t + 1], S)
        np.testing.assert_allclose(o1[:, 0], o4[:, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S, s4, rtol=1e-13, atol=1e-14)
    for n in range(N):
        op, sp = oracle.forward(q[n], k[n], v[n], g[n], b[n], [0, ntok], S0[n:n + 1])
        np.testing.assert_allclose(op, o4[n], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(sp[0], s4[n], rtol=1e-13, atol=1e-14)


# -------------------------------------------------- I10 / head mapping (V heads 2j, 2j+1)
def test_head_mapping_contiguous_groups():
    r = rng(80)
    T, HK, HV, d = 20, 3, 6, 8
    q, k = r.standard_normal((T, HK, d)), r.standard_normal((T, HK, d))
    v = r.standard_normal((T, HV, d))
    g, b = -r.uniform(0, 0.3, (T, HV)), r.uniform(0.05, 0.95, (T, HV))
    out, fin = oracle.forward(q, k, v, g, b, [0, T])
    for h in range(HV):
        j = h // 2
        o1, f1 = run1(q[:, j], k[:, j], v[:, h], g[:, h], b[:, h], eps=oracle.EPS)
        np.testing.assert_allclose(out[:, h], o1, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(fin[0, h], f1, rtol=1e-14, atol=1e-15)
    # identical v, g, b on the two V heads of a pair give identical outputs
    v[:, 1] = v[:, 0]
    g[:, 1] = g[:, 0]
    b[:, 1] = b[:, 0]
    out, _ = oracle.forward(q, k, v, g, b, [0, T])
    np.testing.assert_array_equal(out[:, 0], out[:, 1])


# -------------------------------------------------------------------- I11: contractivity
def test_state_norm_bound_per_step():
    r = rng(90)
    T, d = 60, 16
    q, k, v = (r.standard_normal((T, d)) for _ in range(3))
    g, b = -r.uniform(0, 0.5, T), r.uniform(0.0, 1.0, T)
    S = r.standard_normal((d, d))
    for t in range(T):
        prev = np.linalg.norm(S)
        _, S = run1(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], b[t:t + 1], S)
        assert np.linalg.norm(S) <= np.exp(g[t]) * prev + b[t] * np.linalg.norm(v[t]) + 1e-12


# --------------------------------------------------- results do not depend on threading
def test_thread_count_does_not_change_result():
    r = rng(100)
    T, HK, HV, d = 50, 2, 4, 16
    args = (r.standard_normal((T, HK, d)), r.standard_normal((T, HK, d)),
            r.standard_normal((T, HV, d)), -r.uniform(0, 0.3, (T, HV)),
            r.uniform(0.05, 0.95, (T, HV)), [0, 17, T])
    o1, f1 = oracle.forward(*args, threads=1)
    o8, f8 = oracle.forward(*args, threads=8)
    np.testing.assert_array_equal(o1, o8)
    np.testing.assert_array_equal(f1, f8)


# ------------------------------------ planted mistakes are caught by the pins above
def _mutant_pre_update_output(q, k, v, g, b, S0):
    """A plausible bug planted on the CPU: output read from the state BEFORE the update."""
    qn = q / np.linalg.norm(q, axis=1, keepdims=True) / np.sqrt(q.shape[1])
    kn = k / np.linalg.norm(k, axis=1, keepdims=True)
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        out.append(S @ qn[t])
        S = np.exp(g[t]) * (S - b[t] * np.outer(S @ kn[t], kn[t])) + b[t] * np.outer(v[t], kn[t])
    return np.array(out), S


def _mutant_missing_alpha_on_correction(q, k, v, g, b, S0):
    """A plausible bug planted on the CPU: the decay is not applied to the delta correction."""
    qn = q / np.linalg.norm(q, axis=1, keepdims=True) / np.sqrt(q.shape[1])
    kn = k / np.linalg.norm(k, axis=1, keepdims=True)
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        S = np.exp(g[t]) * S - b[t] * np.outer(S @ kn[t], kn[t]) + b[t] * np.outer(v[t], kn[t])
        out.append(S @ qn[t])
    return np.array(out), S


def test_pins_reject_planted_mistakes():
    r = rng(110)
    T, d = 16, 8
    k = unit_rows(r, T, d)
    q, v = r.standard_normal((T, d)), r.standard_normal((T, d))
    g, b = -r.uniform(0.05, 0.3, T), r.uniform(0.1, 0.9, T)
    S0 = r.standard_normal((d, d))
    # the pre-update mutant fails the b = 0 closed form (outputs lag one decay step)
    cols = r.integers(0, d, T)
    qb = np.zeros((T, d))
    qb[np.arange(T), cols] = 1.0
    o_mut, _ = _mutant_pre_update_output(qb, k, v, g, np.zeros(T), S0)
    o_ok, _ = run1(qb, k, v, g, np.zeros(T), S0)
    assert np.max(np.abs(o_mut - o_ok)) > 1e-3
    # the missing-alpha mutant fails the affine-in-state pin
    _, s_with = _mutant_missing_alpha_on_correction(q, k, v, g, b, S0)
    _, s_zero = _mutant_missing_alpha_on_correction(q, k, v, g, b, np.zeros((d, d)))
    M = np.eye(d)
    for t in range(T):
        M = M @ (np.exp(g[t]) * (np.eye(d) - b[t] * np.outer(k[t], k[t])))
    assert np.max(np.abs((s_with - s_zero) - S0 @ M)) > 1e-3


# ------------------- the head-subset oracle (checker of the full-size GPU parity tests)
def _forward_heads_wrong_grouping(q, k, v, g, b, cu, qk_heads, s0):
    """A plausible bug planted on the CPU: the V heads of QK head j listed as j + r * HK
    (strided) instead of the contiguous j * group + r."""
    HK, HV = q.shape[1], v.shape[1]
    vh = [j + r * HK for j in qk_heads for r in range(HV // HK)]
    out, fin = oracle.forward(q[:, list(qk_heads)], k[:, list(qk_heads)], v[:, vh], g[:, vh],
                              b[:, vh], cu, s0[:, vh])
    return out, fin, vh


@pytest.mark.parametrize("qk_heads", [[0], [2, 1], [3, 0, 2], [0, 1, 2, 3]])
def test_forward_heads_is_an_exact_sample_of_forward(qk_heads):
    """forward_heads on a subset of QK heads returns exactly the columns of the full
    oracle for the V heads that read those QK heads (contiguous groups, R3), in the
    order of the QK heads given, with their initial and final states."""
    r = rng(120)
    lens = [23, 0, 41, 9]
    T, HK, HV, d = sum(lens), 4, 8, 16
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k = r.standard_normal((T, HK, d)), r.standard_normal((T, HK, d))
    v = r.standard_normal((T, HV, d))
    g, b = -r.uniform(0, 0.3, (T, HV)), r.uniform(0.05, 0.95, (T, HV))
    s0 = r.standard_normal((len(lens), HV, d, d)) * 0.1
    out, fin = oracle.forward(q, k, v, g, b, cu, s0)
    o_s, f_s, vh = oracle.forward_heads(q, k, v, g, b, cu, qk_heads, s0)
    assert vh == [2 * j + rr for j in qk_heads for rr in range(2)]
    np.testing.assert_array_equal(o_s, out[:, vh])
    np.testing.assert_array_equal(f_s, fin[:, vh])
    # the same comparison rejects a strided listing of the V heads
    if qk_heads != [0]:
        o_w, f_w, vh_w = _forward_heads_wrong_grouping(q, k, v, g, b, cu, qk_heads, s0)
        assert np.max(np.abs(o_w - out[:, [2 * j + rr for j in qk_heads for rr in range(2)]])) > 1e-3
