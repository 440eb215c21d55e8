"""The allocation-free prefill entry point, for callers that cannot allocate device
memory where they run (a plugin whose framework owns all device allocations, or a hot
path that must not block on an allocation).  It must give the same results as the
workspace-taking gdn_chunk_prefill, call after call, while reusing the library's one
static scratch array.  This file is collected last so that a failure here comes after
every other test has run."""

import ctypes

import numpy as np
import pytest
import torch

from linear_attention_layer_gated_b200 import build, gdn, inputs

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-2  # relative L2, as for every bf16-I/O comparison in the GPU tests


def rel_l2(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))


def stream_handle():
    return torch.cuda.current_stream().cuda_stream


def run_noalloc(L, x, out, fin):
    shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"])
    stream = torch.cuda.current_stream().cuda_stream
    return L.gdn_chunk_prefill_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(),
        x["beta"].data_ptr(),
        None if x["initial_state"] is None else x["initial_state"].data_ptr(),
        x["cu_seqlens"].data_ptr(), out.data_ptr(), fin.data_ptr(), ctypes.byref(shape), stream)


def test_noalloc_prefill_matches_workspace_prefill_twice_in_a_row():
    build.build()
    L = gdn.lib()
    cases = [inputs.make_prefill([100, 37], state_std=0.02, seed=31, device="cuda"),
             inputs.make_prefill([1, 260, 64, 0, 9], state_std=0.02, seed=32, device="cuda")]
    for x in cases:  # two calls in a row; the second sees the first call's leftovers
        out = torch.full_like(x["v"], float("nan"))
        fin = torch.full_like(x["initial_state"], float("nan"))
        assert run_noalloc(L, x, out, fin) == gdn.GDN_OK
        # no bounded device wait of this call gave up (the word lives in the static scratch)
        assert gdn.STATUS[L.gdn_get_noalloc_device_error(stream_handle())] == "GDN_OK"
        ref_out, ref_fin = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                       x["cu_seqlens"], x["initial_state"])
        torch.cuda.synchronize()
        assert rel_l2(out, ref_out) <= TOL_BF16
        assert rel_l2(fin, ref_fin) <= TOL_BF16


def test_noalloc_prefill_takes_one_long_sequence():
    """One sequence runs in the one-launch pass, whose operands live in a ring of a few
    chunks: the static scratch holds a sequence of any length."""
    L = gdn.lib()
    x = inputs.make_prefill([20000], state_std=0.02, seed=33, device="cuda")
    shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"])
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape)) <= (64 << 20)
    out = torch.full_like(x["v"], float("nan"))
    fin = torch.full_like(x["initial_state"], float("nan"))
    assert run_noalloc(L, x, out, fin) == gdn.GDN_OK
    assert gdn.STATUS[L.gdn_get_noalloc_device_error(stream_handle())] == "GDN_OK"
    ref_out, ref_fin = gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], x["initial_state"])
    torch.cuda.synchronize()
    assert rel_l2(out, ref_out) <= 1e-5 and rel_l2(fin, ref_fin) <= 1e-5  # the same pass, the same scratch layout


def test_noalloc_prefill_rejects_workloads_beyond_its_scratch():
    L = gdn.lib()
    # 8 sequences of 8,192 tokens: too many chains for the one-launch pass, and the operands of
    # every chunk need far more than 64 MiB
    shape = gdn.make_shape(8, 1 << 16, 16, 32)
    assert L.gdn_prefill_workspace_bytes(ctypes.byref(shape)) > (64 << 20)
    rc = L.gdn_chunk_prefill_noalloc(None, None, None, None, None, None, None, None, None,
                                     ctypes.byref(shape), None)
    assert gdn.STATUS[rc] == "GDN_ERR_WORKSPACE"
