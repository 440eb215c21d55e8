"""ctypes binding of libgdn.so (C ABI in include/gdn.h) -- argument marshalling only.

The functions carry the C entry points' names.  Tensors are torch CUDA tensors used
purely as device memory; every step of the layer runs in the library's kernels.
There is no CPU fallback: if the library is missing or a call fails, these raise.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn.so")

GDN_OK = 0
GDN_BF16, GDN_F32 = 0, 1
GDN_ALGO_AUTO, GDN_ALGO_SIMT, GDN_ALGO_TENSOR = 0, 1, 2
STATUS = {0: "GDN_OK", 1: "GDN_ERR_NULL", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_ALIGN",
          4: "GDN_ERR_DTYPE", 5: "GDN_ERR_NUM_TOKENS", 6: "GDN_ERR_WORKSPACE",
          7: "GDN_ERR_CUDA", 8: "GDN_ERR_DEVICE_TIMEOUT", 9: "GDN_ERR_UNSUPPORTED"}
EXPORTED = ["gdn_prefill_workspace_bytes", "gdn_prefill_phase_workspace_bytes", "gdn_chunk_prefill",
            "gdn_chunk_prefill_prep",
            "gdn_chunk_prefill_state", "gdn_decode_step", "gdn_get_device_error",
            "gdn_selftest_wait_timeout", "gdn_status_string", "gdn_abi_version",
            "gdn_chunk_prefill_noalloc", "gdn_decode_verify", "gdn_decode_commit",
            "gdn_chunk_prefill_slots", "gdn_decode_step_slots", "gdn_decode_verify_slots",
            "gdn_decode_commit_slots", "gdn_chunk_prefill_chunk_states",
            "gdn_get_noalloc_device_error", "gdn_get_decode_device_error",
            "gdn_chunk_prefill_raw_gates", "gdn_decode_step_raw_gates", "gdn_decode_verify_raw_gates"]


class GdnShape(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32), ("num_qk_heads", ctypes.c_int32),
                ("num_v_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("io_dtype", ctypes.c_int32), ("algo", ctypes.c_int32)]


class GdnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s" % (what, gdn_status_string(code)))
        self.code = code


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Loads libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libgdn.so is missing at %s; build it with "
                                   "`python -m linear_attention_layer_gated_b200.build`" % LIB_PATH)
            L = ctypes.CDLL(LIB_PATH)
            vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
            sp = ctypes.POINTER(GdnShape)
            L.gdn_prefill_workspace_bytes.restype = ctypes.c_size_t
            L.gdn_prefill_workspace_bytes.argtypes = [sp]
            L.gdn_prefill_phase_workspace_bytes.restype = ctypes.c_size_t
            L.gdn_prefill_phase_workspace_bytes.argtypes = [sp]
            L.gdn_chunk_prefill.restype = ctypes.c_int
            L.gdn_chunk_prefill.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, fp, sp, vp,
                                            ctypes.c_size_t, vp]
            L.gdn_chunk_prefill_prep.restype = ctypes.c_int
            L.gdn_chunk_prefill_prep.argtypes = [vp, vp, fp, fp, ip, sp, vp, ctypes.c_size_t, vp]
            L.gdn_chunk_prefill_state.restype = ctypes.c_int
            L.gdn_chunk_prefill_state.argtypes = [vp, vp, fp, ip, vp, fp, sp, vp, ctypes.c_size_t, vp]
            L.gdn_decode_step.restype = ctypes.c_int
            L.gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, ctypes.c_int32, sp, vp]
            L.gdn_decode_verify.restype = ctypes.c_int
            L.gdn_decode_verify.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ctypes.c_int32, sp, vp]
            L.gdn_decode_commit.restype = ctypes.c_int
            L.gdn_decode_commit.argtypes = [fp, fp, ip, ctypes.c_int32, sp, vp]
            i32 = ctypes.c_int32
            L.gdn_chunk_prefill_slots.restype = ctypes.c_int
            L.gdn_chunk_prefill_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, ip, vp, sp, vp,
                                                  ctypes.c_size_t, vp]
            L.gdn_decode_step_slots.restype = ctypes.c_int
            L.gdn_decode_step_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, vp, i32, sp, vp]
            L.gdn_decode_verify_slots.restype = ctypes.c_int
            L.gdn_decode_verify_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, i32, vp, fp, i32, sp, vp]
            L.gdn_decode_commit_slots.restype = ctypes.c_int
            L.gdn_decode_commit_slots.argtypes = [fp, ip, i32, fp, ip, i32, sp, vp]
            L.gdn_chunk_prefill_chunk_states.restype = ctypes.c_int
            L.gdn_chunk_prefill_chunk_states.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, fp, fp, sp, vp,
                                                         ctypes.c_size_t, vp]
            L.gdn_get_device_error.restype = ctypes.c_int
            L.gdn_get_device_error.argtypes = [vp, vp]
            L.gdn_chunk_prefill_noalloc.restype = ctypes.c_int
            L.gdn_chunk_prefill_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, fp, sp, vp]
            L.gdn_get_noalloc_device_error.restype = ctypes.c_int
            L.gdn_get_noalloc_device_error.argtypes = [vp]
            L.gdn_get_decode_device_error.restype = ctypes.c_int
            L.gdn_get_decode_device_error.argtypes = [vp]
            L.gdn_chunk_prefill_raw_gates.restype = ctypes.c_int
            L.gdn_chunk_prefill_raw_gates.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, ip, vp, fp, sp, vp,
                                                      ctypes.c_size_t, vp]
            L.gdn_decode_step_raw_gates.restype = ctypes.c_int
            L.gdn_decode_step_raw_gates.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, ctypes.c_int32, sp, vp]
            L.gdn_decode_verify_raw_gates.restype = ctypes.c_int
            L.gdn_decode_verify_raw_gates.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, fp, ctypes.c_int32,
                                                      sp, vp]
            L.gdn_selftest_wait_timeout.restype = ctypes.c_int
            L.gdn_selftest_wait_timeout.argtypes = [vp, ctypes.c_size_t, ctypes.c_uint32, vp]
            L.gdn_status_string.restype = ctypes.c_char_p
            L.gdn_status_string.argtypes = [ctypes.c_int]
            L.gdn_abi_version.restype = ctypes.c_int32
            L.gdn_abi_version.argtypes = []
            _lib = L
    return _lib


def gdn_status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def gdn_abi_version() -> int:
    return int(lib().gdn_abi_version())


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError("q/k/v/out must be bfloat16 or float32, got %s" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(num_seqs, total_tokens, num_qk_heads, num_v_heads, head_dim=128,
               io_dtype=GDN_BF16, algo=GDN_ALGO_AUTO, max_seqlen=0) -> GdnShape:
    return GdnShape(int(num_seqs), int(total_tokens), int(max_seqlen), int(num_qk_heads),
                    int(num_v_heads), int(head_dim), int(io_dtype), int(algo))


def gdn_prefill_workspace_bytes(shape: GdnShape) -> int:
    return int(lib().gdn_prefill_workspace_bytes(ctypes.byref(shape)))


def gdn_prefill_phase_workspace_bytes(shape: GdnShape) -> int:
    return int(lib().gdn_prefill_phase_workspace_bytes(ctypes.byref(shape)))


def prefill_shape(q, v, cu_seqlens, algo=GDN_ALGO_AUTO, max_seqlen=0) -> GdnShape:
    T, HK, D = q.shape
    return make_shape(cu_seqlens.numel() - 1, T, HK, v.shape[1], D, _io_dtype(q), algo, max_seqlen)


def alloc_workspace(shape: GdnShape, device, phases=False) -> torch.Tensor:
    """A workspace for gdn_chunk_prefill on `shape` (with phases=True, large enough for the
    two-phase entry points gdn_chunk_prefill_prep / _state as well)."""
    n = gdn_prefill_workspace_bytes(shape)
    if n == 0:
        raise ValueError("invalid prefill shape")
    if phases:
        n = max(n, gdn_prefill_phase_workspace_bytes(shape))
    return torch.empty(n, dtype=torch.uint8, device=device)


def gdn_chunk_prefill(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                      workspace=None, algo=GDN_ALGO_AUTO, max_seqlen=0, stream=None):
    """Calls gdn_chunk_prefill.  Shapes: q, k [T, HK, 128]; v, out [T, HV, 128];
    g, beta [T, HV] fp32; states [N, HV, 128, 128] fp32 or None; cu_seqlens [N+1] int32."""
    if q.dtype != k.dtype or q.dtype != v.dtype or out.dtype != q.dtype:
        raise TypeError("q, k, v and out must share one dtype")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    shape = prefill_shape(q, v, cu_seqlens, algo, max_seqlen)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib().gdn_chunk_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                 _ptr(final_state), ctypes.byref(shape), _ptr(workspace),
                                 workspace.numel(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill")
    return workspace


def gdn_chunk_prefill_prep(q, k, g, beta, cu_seqlens, workspace, v_shape_like, algo=GDN_ALGO_AUTO,
                           stream=None):
    """Calls gdn_chunk_prefill_prep (tensor-core path, phase 1).  ``v_shape_like`` is v (or
    any tensor of v's shape) -- only its head count is used."""
    shape = prefill_shape(q, v_shape_like, cu_seqlens, algo)
    rc = lib().gdn_chunk_prefill_prep(_ptr(q), _ptr(k), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                      ctypes.byref(shape), _ptr(workspace), workspace.numel(),
                                      _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_prep")


def gdn_chunk_prefill_state(k, v, initial_state, cu_seqlens, out, final_state, workspace,
                            algo=GDN_ALGO_AUTO, stream=None):
    """Calls gdn_chunk_prefill_state (tensor-core path, phase 2) on the workspace the prep
    phase of the same shape wrote."""
    shape = prefill_shape(k, v, cu_seqlens, algo)
    rc = lib().gdn_chunk_prefill_state(_ptr(k), _ptr(v), _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                       _ptr(final_state), ctypes.byref(shape), _ptr(workspace),
                                       workspace.numel(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_state")


def gdn_decode_step(q, k, v, g, beta, state_inout, out, num_tokens=None, stream=None):
    """Calls gdn_decode_step.  Shapes: q, k [N, m, HK, 128]; v, out [N, m, HV, 128];
    g, beta [N, m, HV] fp32; state_inout [N, HV, 128, 128] fp32 (updated in place)."""
    N, m, HK, D = q.shape
    if num_tokens is None:
        num_tokens = m
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_inout),
                               _ptr(out), int(num_tokens), ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_step")


def gdn_decode_verify(q, k, v, g, beta, state, out, snapshots, num_tokens=None, stream=None):
    """Calls gdn_decode_verify.  Shapes as gdn_decode_step; state [N, HV, 128, 128] fp32 is
    only read; snapshots [N, m, HV, 128, 128] fp32 receives the state after each token."""
    N, m, HK, D = q.shape
    if num_tokens is None:
        num_tokens = m
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                                 _ptr(snapshots), int(num_tokens), ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_verify")


def gdn_chunk_prefill_raw_gates(q, k, v, x, y, a, b, initial_state, cu_seqlens, out, final_state,
                                workspace=None, algo=GDN_ALGO_AUTO, max_seqlen=0, stream=None):
    """Calls gdn_chunk_prefill_raw_gates: as gdn_chunk_prefill with the gates given as raw
    projections x, y [T, HV] and per-V-head a, b [HV] (all fp32)."""
    if q.dtype != k.dtype or q.dtype != v.dtype or out.dtype != q.dtype:
        raise TypeError("q, k, v and out must share one dtype")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    shape = prefill_shape(q, v, cu_seqlens, algo, max_seqlen)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib().gdn_chunk_prefill_raw_gates(_ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(y), _ptr(a), _ptr(b),
                                           _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                           _ptr(final_state), ctypes.byref(shape), _ptr(workspace),
                                           workspace.numel(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_raw_gates")
    return workspace


def gdn_decode_step_raw_gates(q, k, v, x, y, a, b, state_inout, out, num_tokens=None, stream=None):
    """Calls gdn_decode_step_raw_gates: as gdn_decode_step with raw projections x, y
    [N, m, HV] and per-V-head a, b [HV] (all fp32)."""
    N, m, HK, D = q.shape
    if num_tokens is None:
        num_tokens = m
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_step_raw_gates(_ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(y), _ptr(a), _ptr(b),
                                         _ptr(state_inout), _ptr(out), int(num_tokens), ctypes.byref(shape),
                                         _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_step_raw_gates")


def gdn_decode_verify_raw_gates(q, k, v, x, y, a, b, state, out, snapshots, num_tokens=None, stream=None):
    """Calls gdn_decode_verify_raw_gates: as gdn_decode_verify with raw projections."""
    N, m, HK, D = q.shape
    if num_tokens is None:
        num_tokens = m
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_verify_raw_gates(_ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(y), _ptr(a), _ptr(b),
                                           _ptr(state), _ptr(out), _ptr(snapshots), int(num_tokens),
                                           ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_verify_raw_gates")


def gdn_decode_commit(state, snapshots, accepted, num_tokens=None, stream=None):
    """Calls gdn_decode_commit: state[n] <- snapshots[n, accepted[n] - 1] where
    1 <= accepted[n] <= num_tokens (accepted: [N] int32 on the device)."""
    N, m, HV, D, _ = snapshots.shape
    if num_tokens is None:
        num_tokens = m
    shape = make_shape(N, N * m, 1, HV, D, GDN_BF16)  # the commit reads num_seqs, num_v_heads, head_dim
    rc = lib().gdn_decode_commit(_ptr(state), _ptr(snapshots), _ptr(accepted), int(num_tokens),
                                 ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_commit")


def gdn_chunk_prefill_chunk_states(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                                   chunk_states, workspace=None, algo=GDN_ALGO_AUTO, stream=None):
    """Calls gdn_chunk_prefill_chunk_states: as gdn_chunk_prefill, plus the state after every
    64-token chunk in chunk_states [sum_n ceil(T_n / 64), HV, 128, 128] fp32."""
    shape = prefill_shape(q, v, cu_seqlens, algo)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib().gdn_chunk_prefill_chunk_states(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                              _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                              _ptr(final_state), _ptr(chunk_states), ctypes.byref(shape),
                                              _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_chunk_states")


def gdn_chunk_prefill_slots(q, k, v, g, beta, state_pool, state_slots, cu_seqlens, out,
                            workspace=None, algo=GDN_ALGO_AUTO, stream=None):
    """Calls gdn_chunk_prefill_slots: initial and final states live in state_pool
    [num_slots, HV, 128, 128] fp32 at the rows state_slots [N] (int32, device) names."""
    shape = prefill_shape(q, v, cu_seqlens, algo)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    rc = lib().gdn_chunk_prefill_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                       _ptr(state_slots), int(state_pool.shape[0]), _ptr(cu_seqlens), _ptr(out),
                                       ctypes.byref(shape), _ptr(workspace), workspace.numel(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_slots")


def gdn_decode_step_slots(q, k, v, g, beta, state_pool, state_slots, out, stream=None):
    """Calls gdn_decode_step_slots (the pool rows named by state_slots are updated in place)."""
    N, m, HK, D = q.shape
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                     _ptr(state_slots), int(state_pool.shape[0]), _ptr(out), int(m),
                                     ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_step_slots")


def gdn_decode_verify_slots(q, k, v, g, beta, state_pool, state_slots, out, snapshots, stream=None):
    """Calls gdn_decode_verify_slots (the pool is only read)."""
    N, m, HK, D = q.shape
    shape = make_shape(N, N * m, HK, v.shape[2], D, _io_dtype(q))
    rc = lib().gdn_decode_verify_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                       _ptr(state_slots), int(state_pool.shape[0]), _ptr(out), _ptr(snapshots),
                                       int(m), ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_verify_slots")


def gdn_decode_commit_slots(state_pool, state_slots, snapshots, accepted, stream=None):
    """Calls gdn_decode_commit_slots."""
    N, m, HV, D, _ = snapshots.shape
    shape = make_shape(N, N * m, 1, HV, D, GDN_BF16)
    rc = lib().gdn_decode_commit_slots(_ptr(state_pool), _ptr(state_slots), int(state_pool.shape[0]),
                                       _ptr(snapshots), _ptr(accepted), int(m), ctypes.byref(shape),
                                       _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_commit_slots")


def gdn_chunk_prefill_noalloc(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                              stream=None):
    """Calls gdn_chunk_prefill_noalloc: the tensor-core prefill with the library's own
    static scratch instead of a caller workspace, for callers that cannot allocate."""
    shape = prefill_shape(q, v, cu_seqlens)
    rc = lib().gdn_chunk_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                         _ptr(final_state), ctypes.byref(shape), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_prefill_noalloc")


def gdn_get_decode_device_error(stream=None) -> int:
    """Calls gdn_get_decode_device_error: reads and clears the decode kernels' device error
    word (synchronises the stream).  Returns the gdn_status code."""
    return int(lib().gdn_get_decode_device_error(_stream(stream)))


def gdn_get_noalloc_device_error(stream=None) -> int:
    """Calls gdn_get_noalloc_device_error: the device error word of the static scratch
    the allocation-free prefill uses on the current device."""
    return int(lib().gdn_get_noalloc_device_error(_stream(stream)))


def gdn_selftest_wait_timeout(workspace, limit_us=20000, stream=None):
    """Calls gdn_selftest_wait_timeout (a bounded device wait that must expire)."""
    rc = lib().gdn_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(limit_us),
                                         _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_selftest_wait_timeout")


def gdn_get_device_error(workspace, stream=None) -> int:
    return int(lib().gdn_get_device_error(_ptr(workspace), _stream(stream)))


# ------------------------------------------------------------------ conveniences
def prefill(q, k, v, g, beta, cu_seqlens, initial_state=None, want_final_state=True,
            algo=GDN_ALGO_AUTO, workspace=None, stream=None):
    """Allocates out (and final_state) and runs gdn_chunk_prefill."""
    out = torch.empty_like(v)
    N = cu_seqlens.numel() - 1
    fin = None
    if want_final_state:
        fin = torch.empty((N, v.shape[1], v.shape[2], v.shape[2]), dtype=torch.float32,
                          device=v.device)
    gdn_chunk_prefill(q, k, v, g, beta, initial_state, cu_seqlens, out, fin,
                      workspace=workspace, algo=algo, stream=stream)
    return out, fin


def decode(q, k, v, g, beta, state_inout, stream=None):
    """Allocates out and runs gdn_decode_step (state_inout is updated in place)."""
    out = torch.empty_like(v)
    gdn_decode_step(q, k, v, g, beta, state_inout, out, stream=stream)
    return out


def verify(q, k, v, g, beta, state, stream=None):
    """Allocates out and the snapshots and runs gdn_decode_verify (state is not changed).
    Returns (out, snapshots)."""
    N, m = q.shape[:2]
    HV, D = v.shape[2], v.shape[3]
    out = torch.empty_like(v)
    snaps = torch.empty((N, m, HV, D, D), dtype=torch.float32, device=v.device)
    gdn_decode_verify(q, k, v, g, beta, state, out, snaps, stream=stream)
    return out, snaps
