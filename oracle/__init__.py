"""fp64 CPU oracle for the Gated DeltaNet layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and shares
no code with it; if the CUDA extension is missing the product path raises instead
of falling back here.

Two independent formulations live here:

* :func:`forward` -- the plain token-by-token gated delta rule in fp64, written in
  C (``gdn_ref.c``) and threaded over (sequence, V head).  This is the oracle the
  GPU results are compared with.
* :mod:`oracle.chunked` -- a numpy fp64 chunked closed form (cumulative gates,
  UT/WY triangular system, state carry between chunks), used only to cross-check
  :func:`forward` on small inputs.

:func:`gates_from_projections` (and the ``*_from_projections`` wrappers) derive the
activated gates from raw per-token projections, g = -a softplus(x + b) and
beta = sigmoid(y); that activation is a stated reading, not given by the pages.

The layer is Gated DeltaNet as named in the Qwen3-Next-80B-A3B model card
("Highlights", "Model Overview": 16 QK heads, 32 V heads, head dimension 128); the
recurrence is S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
o_t = S_t q_t, with q and k L2-normalised and q scaled by 1/sqrt(d_k).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_ref.c")
_LIB = os.path.join(_HERE, "libgdn_ref.so")
_lock = threading.Lock()
_lib = None

#: L2-normalisation epsilon: x / sqrt(sum(x^2) + EPS).  The pages do not state one.
EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile ``gdn_ref.c`` with gcc into ``libgdn_ref.so`` (plain -O2, IEEE math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lib.gdn_ref_forward.restype = ctypes.c_int
            lib.gdn_ref_forward.argtypes = [dp, dp, dp, dp, dp, dp, ip,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                            dp, dp, ctypes.c_int32]
            _lib = lib
    return _lib


def host_threads() -> int:
    """Number of host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact widening of bf16/fp32 values
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def forward(q, k, v, g, beta, cu_seqlens, initial_state=None, eps: float = EPS,
            threads: int | None = None):
    """Token-by-token fp64 gated delta rule over a packed (varlen) batch.

    Shapes: q, k ``[T, HK, dk]``; v ``[T, HV, dv]``; g, beta ``[T, HV]``;
    cu_seqlens ``[N+1]`` (int); initial_state ``[N, HV, dv, dk]`` or None (zeros).
    Returns ``(out [T, HV, dv], final_state [N, HV, dv, dk])`` as fp64 numpy arrays.
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    s0 = _f64(initial_state)
    if hasattr(cu_seqlens, "detach"):
        cu_seqlens = cu_seqlens.detach().cpu().numpy()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    T, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    N = cu.shape[0] - 1
    if k.shape != q.shape or v.shape[0] != T or g.shape != (T, HV) or beta.shape != (T, HV):
        raise ValueError("inconsistent shapes")
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the number of packed tokens")
    if s0 is not None and s0.shape != (N, HV, dv, dk):
        raise ValueError("initial_state shape")
    out = np.zeros((T, HV, dv), dtype=np.float64)
    fin = np.zeros((N, HV, dv, dk), dtype=np.float64)
    nthr = threads or host_threads()
    rc = _load().gdn_ref_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
                                 _ptr(cu, ctypes.c_int32), N, HK, HV, dk, dv, float(eps),
                                 _ptr(out), _ptr(fin), int(nthr))
    if rc != 0:
        raise RuntimeError("gdn_ref_forward failed with code %d" % rc)
    return out, fin


def decode(q, k, v, g, beta, state, eps: float = EPS, threads: int | None = None):
    """Decode / multi-token verify: the same recurrence continued from ``state``.

    Shapes: q, k ``[N, ntok, HK, dk]``; v ``[N, ntok, HV, dv]``; g, beta
    ``[N, ntok, HV]``; state ``[N, HV, dv, dk]``.  Returns
    ``(out [N, ntok, HV, dv], new_state [N, HV, dv, dk])``.
    """
    q, k, v, g, beta, state = (_f64(a) for a in (q, k, v, g, beta, state))
    N, ntok, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    cu = np.arange(0, N * ntok + 1, ntok, dtype=np.int32)
    out, fin = forward(q.reshape(N * ntok, HK, dk), k.reshape(N * ntok, HK, dk),
                       v.reshape(N * ntok, HV, dv), g.reshape(N * ntok, HV),
                       beta.reshape(N * ntok, HV), cu, state, eps=eps, threads=threads)
    return out.reshape(N, ntok, HV, dv), fin


def forward_heads(q, k, v, g, beta, cu_seqlens, qk_heads, initial_state=None,
                  eps: float = EPS, threads: int | None = None):
    """Oracle restricted to the V heads that read the given QK heads.

    The (sequence, V head) recurrences are independent, so a subset of heads is an
    exact sample of the full result.  Returns ``(out, final_state, v_heads)`` where
    ``out`` is ``[T, len(v_heads), dv]`` and ``v_heads`` lists the V-head indices
    (in order) that the columns correspond to.
    """
    HK = q.shape[1]
    HV = v.shape[1]
    group = HV // HK
    v_heads = [j * group + r for j in qk_heads for r in range(group)]
    sel = lambda a, idx: a[:, idx]  # noqa: E731
    s0 = None if initial_state is None else initial_state[:, v_heads]
    out, fin = forward(sel(q, list(qk_heads)), sel(k, list(qk_heads)), sel(v, v_heads),
                       sel(g, v_heads), sel(beta, v_heads), cu_seqlens, s0, eps=eps,
                       threads=threads)
    return out, fin, v_heads


# ---------------------------------------------------------------- gates from raw projections
# The pages specify the layer in terms of the activated gates: a decay exp(g_t) in (0, 1] and
# a write strength beta_t in [0, 1].  Serving stacks usually produce both from per-token raw
# projections.  The reading used here (stated, not on the pages): per V head h,
#     g_t    = -a_h * softplus(x_t + b_h),   softplus(z) = log(1 + exp(z)),
#     beta_t = sigmoid(y_t)              = 1 / (1 + exp(-y_t)),
# with x_t, y_t the raw projections [T, HV], a_h > 0 a per-head decay rate [HV] (the positive
# rate itself, not its logarithm) and b_h a per-head bias [HV].

def softplus(z):
    """log(1 + exp(z)) in fp64, written as max(z, 0) + log1p(exp(-|z|)) (the same value,
    without overflow for large z)."""
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sigmoid(y):
    """1 / (1 + exp(-y)) in fp64 (exp overflow for y << 0 gives the limit 0)."""
    y = np.asarray(y, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-y))


def gates_from_projections(x, y, a, b):
    """Activated gates from raw projections: ``(g, beta)``, both ``[T, HV]`` fp64.

    x, y: ``[T, HV]`` raw decay and write-strength projections; a, b: ``[HV]`` per-V-head
    decay rate and bias.  g = -a * softplus(x + b); beta = sigmoid(y)."""
    x, y, a, b = (_f64(t) for t in (x, y, a, b))
    if x.shape != y.shape or x.ndim != 2 or a.shape != (x.shape[1],) or b.shape != (x.shape[1],):
        raise ValueError("x, y must be [T, HV] and a, b [HV]")
    return -a[None, :] * softplus(x + b[None, :]), sigmoid(y)


def forward_from_projections(q, k, v, x, y, a, b, cu_seqlens, initial_state=None,
                             eps: float = EPS, threads: int | None = None):
    """:func:`forward` with the gates taken from raw projections (:func:`gates_from_projections`)."""
    g, beta = gates_from_projections(x, y, a, b)
    return forward(q, k, v, g, beta, cu_seqlens, initial_state, eps=eps, threads=threads)


def decode_from_projections(q, k, v, x, y, a, b, state, eps: float = EPS, threads: int | None = None):
    """:func:`decode` with the gates taken from raw projections; x, y are ``[N, ntok, HV]``."""
    x, y = _f64(x), _f64(y)
    N, ntok, HV = x.shape
    g, beta = gates_from_projections(x.reshape(N * ntok, HV), y.reshape(N * ntok, HV), a, b)
    return decode(q, k, v, g.reshape(N, ntok, HV), beta.reshape(N, ntok, HV), state, eps=eps,
                  threads=threads)
