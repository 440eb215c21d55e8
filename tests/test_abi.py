"""C ABI checks that need no GPU: the library loads, exports every function that
include/gdn.h declares, and rejects bad arguments on the host before touching the
device (fake device addresses are never dereferenced on these paths)."""

import ctypes
import os
import re

import pytest

from linear_attention_layer_gated_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

FAKE = 0x7F0000000000  # 16-byte (and 256-byte) aligned, never dereferenced on these paths


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return gdn.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) >= set(gdn.EXPORTED)
    for name in names:
        assert hasattr(L, name), name


def test_abi_version_and_status_strings(L):
    assert gdn.gdn_abi_version() == 2
    for code, name in gdn.STATUS.items():
        assert gdn.gdn_status_string(code).startswith(name)


def shape(**kw):
    base = dict(num_seqs=2, total_tokens=100, num_qk_heads=16, num_v_heads=32, head_dim=128,
                io_dtype=gdn.GDN_BF16, algo=gdn.GDN_ALGO_AUTO, max_seqlen=0)
    base.update(kw)
    return gdn.make_shape(**base)


def prefill_call(L, s, ws_bytes=None, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, s0=None, cu=FAKE, out=FAKE, sT=None,
             ws=FAKE)
    p.update(ptrs)
    if ws_bytes is None:
        ws_bytes = L.gdn_prefill_workspace_bytes(ctypes.byref(s))
    return L.gdn_chunk_prefill(p["q"], p["k"], p["v"], p["g"], p["beta"], p["s0"], p["cu"],
                               p["out"], p["sT"], ctypes.byref(s), p["ws"], ws_bytes, None)


def test_workspace_size_valid_and_invalid(L):
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape())) % 256 == 0
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape())) > 0
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape(head_dim=64))) == 0
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape(num_v_heads=33))) == 0
    assert L.gdn_prefill_workspace_bytes(None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), "GDN_ERR_SHAPE"),
    (dict(num_v_heads=24, num_qk_heads=16), "GDN_ERR_SHAPE"),
    (dict(num_qk_heads=0), "GDN_ERR_SHAPE"),
    (dict(io_dtype=7), "GDN_ERR_DTYPE"),
    (dict(total_tokens=-1), "GDN_ERR_SHAPE"),
    (dict(max_seqlen=101), "GDN_ERR_SHAPE"),
    (dict(algo=9), "GDN_ERR_SHAPE"),
])
def test_prefill_rejects_bad_shapes(L, kw, code):
    assert gdn.STATUS[prefill_call(L, shape(**kw), ws_bytes=1 << 20)] == code


def test_prefill_rejects_null_and_misaligned(L):
    s = shape()
    assert gdn.STATUS[prefill_call(L, s, q=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[prefill_call(L, s, cu=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[prefill_call(L, s, out=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[prefill_call(L, s, v=FAKE + 8)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[prefill_call(L, s, s0=FAKE + 4)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[prefill_call(L, s, ws=FAKE + 16)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[prefill_call(L, s, ws=None)] == "GDN_ERR_WORKSPACE"
    assert gdn.STATUS[prefill_call(L, s, ws_bytes=16)] == "GDN_ERR_WORKSPACE"
    assert L.gdn_chunk_prefill(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, None,
                               FAKE, 1 << 20, None) == 1


def decode_call(L, s, ntok=1, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, st=FAKE, out=FAKE)
    p.update(ptrs)
    return L.gdn_decode_step(p["q"], p["k"], p["v"], p["g"], p["beta"], p["st"], p["out"], ntok,
                             ctypes.byref(s), None)


@pytest.mark.parametrize("ntok", [0, 5, -1, 100])
def test_decode_rejects_num_tokens(L, ntok):
    assert gdn.STATUS[decode_call(L, shape(num_seqs=4), ntok=ntok)] == "GDN_ERR_NUM_TOKENS"


def test_decode_rejects_null_misaligned_and_shape(L):
    s = shape(num_seqs=4)
    assert gdn.STATUS[decode_call(L, s, st=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[decode_call(L, s, out=FAKE + 2)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[decode_call(L, shape(head_dim=256))] == "GDN_ERR_SHAPE"
    assert gdn.STATUS[decode_call(L, shape(io_dtype=3))] == "GDN_ERR_DTYPE"


def test_empty_batches_are_no_ops(L):
    # num_seqs == 0 returns before any device work; no pointer is touched
    assert prefill_call(L, shape(num_seqs=0, total_tokens=0), q=None, k=None, v=None, g=None,
                        beta=None, cu=None, out=None) == 0
    assert decode_call(L, shape(num_seqs=0), q=None) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(4, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn._ptr(q)


def test_selftest_rejects_bad_arguments(L):
    assert gdn.STATUS[L.gdn_selftest_wait_timeout(None, 256, 1000, None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_selftest_wait_timeout(FAKE, 16, 1000, None)] == "GDN_ERR_WORKSPACE"
    assert gdn.STATUS[L.gdn_selftest_wait_timeout(FAKE + 16, 256, 1000, None)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[L.gdn_selftest_wait_timeout(FAKE, 256, 0, None)] == "GDN_ERR_SHAPE"


def test_verify_and_commit_reject_bad_arguments(L):
    s = shape(num_seqs=4)
    verify = lambda ntok=2, **kw: L.gdn_decode_verify(  # noqa: E731
        kw.get("q", FAKE), FAKE, FAKE, FAKE, FAKE, kw.get("st", FAKE), FAKE, kw.get("snap", FAKE), ntok,
        ctypes.byref(s), None)
    assert gdn.STATUS[verify(ntok=0)] == "GDN_ERR_NUM_TOKENS"
    assert gdn.STATUS[verify(ntok=5)] == "GDN_ERR_NUM_TOKENS"
    assert gdn.STATUS[verify(snap=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[verify(st=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[verify(snap=FAKE + 4)] == "GDN_ERR_ALIGN"
    commit = lambda ntok=2, **kw: L.gdn_decode_commit(  # noqa: E731
        kw.get("st", FAKE), kw.get("snap", FAKE), kw.get("acc", FAKE), ntok, ctypes.byref(s), None)
    assert gdn.STATUS[commit(ntok=7)] == "GDN_ERR_NUM_TOKENS"
    assert gdn.STATUS[commit(acc=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[commit(acc=FAKE + 4)] == "GDN_ERR_ALIGN"
    empty = shape(num_seqs=0)
    assert L.gdn_decode_commit(None, None, None, 2, ctypes.byref(empty), None) == 0


def test_slot_entry_points_reject_missing_pool_or_table(L):
    s = shape(num_seqs=4)
    assert gdn.STATUS[L.gdn_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, FAKE, 1,
                                              ctypes.byref(s), None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 8, FAKE, 1,
                                              ctypes.byref(s), None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, FAKE, 1,
                                              ctypes.byref(s), None)] == "GDN_ERR_SHAPE"
    assert gdn.STATUS[L.gdn_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 8, FAKE, 1,
                                              ctypes.byref(s), None)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[L.gdn_decode_verify_slots(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, None, 2,
                                                ctypes.byref(s), None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_decode_commit_slots(FAKE, None, 8, FAKE, FAKE, 2, ctypes.byref(s),
                                                None)] == "GDN_ERR_NULL"
    ps = shape()
    ws_bytes = L.gdn_prefill_workspace_bytes(ctypes.byref(ps))
    assert gdn.STATUS[L.gdn_chunk_prefill_slots(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 8, FAKE, FAKE,
                                                ctypes.byref(ps), FAKE, ws_bytes, None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_chunk_prefill_slots(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -3, FAKE, FAKE,
                                                ctypes.byref(ps), FAKE, ws_bytes, None)] == "GDN_ERR_SHAPE"


def test_chunk_states_prefill_requires_its_buffer(L):
    s = shape()
    ws_bytes = L.gdn_prefill_workspace_bytes(ctypes.byref(s))
    assert gdn.STATUS[L.gdn_chunk_prefill_chunk_states(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None,
                                                       None, ctypes.byref(s), FAKE, ws_bytes,
                                                       None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[L.gdn_chunk_prefill_chunk_states(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None,
                                                       FAKE + 8, ctypes.byref(s), FAKE, ws_bytes,
                                                       None)] == "GDN_ERR_ALIGN"


def test_tensor_path_needs_pairs_of_v_heads_per_qk_head(L):
    """The tensor-core kernels take V heads in pairs that read one QK head: an odd number of
    V heads per QK head is refused on that path (before any device work) and served by the
    fp32 path under GDN_ALGO_AUTO (whose workspace is just the header)."""
    odd = shape(num_qk_heads=8, num_v_heads=8, algo=gdn.GDN_ALGO_TENSOR)
    assert gdn.STATUS[prefill_call(L, odd, ws_bytes=1 << 30)] == "GDN_ERR_UNSUPPORTED"
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape(num_qk_heads=8, num_v_heads=8))) == 256
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape(num_qk_heads=8, num_v_heads=16))) > 256
    assert gdn.STATUS[L.gdn_chunk_prefill_prep(FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(odd), FAKE, 1 << 30,
                                               None)] == "GDN_ERR_UNSUPPORTED"
    assert gdn.STATUS[L.gdn_chunk_prefill_state(FAKE, FAKE, None, FAKE, FAKE, None, ctypes.byref(odd), FAKE,
                                                1 << 30, None)] == "GDN_ERR_UNSUPPORTED"


def test_raw_gate_entry_points_reject_bad_gate_parameters(L):
    s = shape(num_seqs=4)
    dec = lambda a=FAKE, b=FAKE, ntok=2: L.gdn_decode_step_raw_gates(  # noqa: E731
        FAKE, FAKE, FAKE, FAKE, FAKE, a, b, FAKE, FAKE, ntok, ctypes.byref(s), None)
    ver = lambda a=FAKE, b=FAKE, snap=FAKE: L.gdn_decode_verify_raw_gates(  # noqa: E731
        FAKE, FAKE, FAKE, FAKE, FAKE, a, b, FAKE, FAKE, snap, 2, ctypes.byref(s), None)
    for f in (dec, ver):
        assert gdn.STATUS[f(a=None)] == "GDN_ERR_NULL"
        assert gdn.STATUS[f(b=None)] == "GDN_ERR_NULL"
        assert gdn.STATUS[f(a=FAKE + 4)] == "GDN_ERR_ALIGN"
        assert gdn.STATUS[f(b=FAKE + 8)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[ver(snap=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[dec(ntok=5)] == "GDN_ERR_NUM_TOKENS"  # then the decode checks
    ps = shape(num_seqs=1, total_tokens=64)
    pre = lambda a=FAKE, b=FAKE: L.gdn_chunk_prefill_raw_gates(  # noqa: E731
        FAKE, FAKE, FAKE, FAKE, FAKE, a, b, None, FAKE, FAKE, None, ctypes.byref(ps), FAKE, 0, None)
    assert gdn.STATUS[pre(a=None)] == "GDN_ERR_NULL"
    assert gdn.STATUS[pre(b=FAKE + 4)] == "GDN_ERR_ALIGN"
    assert gdn.STATUS[pre()] == "GDN_ERR_WORKSPACE"  # then the prefill checks
