"""Seeded synthetic inputs for the Gated DeltaNet layer.

This module only draws random tensors; it holds none of the layer's arithmetic
(no normalisation, no gate cumulation), so both the CUDA path and the CPU oracle
can consume exactly the same values.

Head counts and head dimension follow the Qwen3-Next-80B-A3B model card
("Model Overview": Gated DeltaNet with 32 V heads, 16 QK heads, head dim 128).
Gates are drawn already activated: g <= 0 (so alpha = exp(g) is in (0, 1]) and
beta in (0, 1).

Draw order on one ``torch.Generator`` seeded with ``seed``: sequence lengths,
q, k, v, g, beta, then the initial state.  Values are drawn in fp32 on
``device`` and then cast to the I/O dtype; the oracle reads the cast values.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

HK, HV, D = 16, 32, 128


@dataclass
class Workload:
    """Named synthetic workload (sizes and value distributions)."""
    name: str
    kind: str                       # "prefill" or "decode"
    seqlens: list = field(default_factory=list)   # prefill only (drawn lazily if None)
    num_seqs: int = 1
    ntok: int = 1                   # decode only
    hk: int = HK
    hv: int = HV
    d: int = D
    io_dtype: torch.dtype = torch.bfloat16
    gate: str = "softplus"          # "softplus": g = -softplus(N(0,1))*0.1 ; "uniform": U[-0.1, 0]
    state_std: float | None = None  # None: zero initial state
    seed: int = 0
    varlen_range: tuple | None = None


def workload(name: str) -> Workload:
    """The five workloads the layer is tested and measured on."""
    if name == "tiny":
        return Workload("tiny", "prefill", [256], 1, hk=2, hv=4, io_dtype=torch.float32,
                        gate="uniform", seed=0)
    if name == "layer_prefill":
        return Workload("layer_prefill", "prefill", [8192], 1, seed=1)
    if name == "varlen":
        return Workload("varlen", "prefill", None, 8, state_std=0.02, seed=2,
                        varlen_range=(1024, 16384))
    if name == "decode":
        return Workload("decode", "decode", None, 256, ntok=1, state_std=0.02, seed=3)
    if name == "decode_verify":
        return Workload("decode_verify", "decode", None, 256, ntok=4, state_std=0.02, seed=3)
    if name == "long":
        return Workload("long", "prefill", [262144], 1, seed=4)
    raise KeyError(name)


def _gates(gen, shape, kind, device):
    if kind == "uniform":
        g = -0.1 * torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    else:
        g = -torch.nn.functional.softplus(
            torch.randn(shape, generator=gen, device=device, dtype=torch.float32)) * 0.1
    beta = torch.sigmoid(torch.randn(shape, generator=gen, device=device, dtype=torch.float32))
    return g, beta


def make_prefill(seqlens=None, *, hk=HK, hv=HV, d=D, io_dtype=torch.bfloat16,
                 gate="softplus", state_std=None, seed=0, device="cpu",
                 num_seqs=None, varlen_range=None):
    """Packed varlen prefill inputs.

    Returns a dict with q, k ``[T, hk, d]``, v ``[T, hv, d]`` (io_dtype), g, beta
    ``[T, hv]`` (fp32), cu_seqlens ``[N+1]`` (int32), initial_state
    ``[N, hv, d, d]`` (fp32) or None, and ``seqlens`` (python list).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    if seqlens is None:
        lo, hi = varlen_range
        seqlens = torch.randint(lo, hi + 1, (num_seqs,), generator=gen, device=device).tolist()
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    N = len(seqlens)
    q = torch.randn((T, hk, d), generator=gen, device=device, dtype=torch.float32)
    k = torch.randn((T, hk, d), generator=gen, device=device, dtype=torch.float32)
    v = torch.randn((T, hv, d), generator=gen, device=device, dtype=torch.float32)
    g, beta = _gates(gen, (T, hv), gate, device)
    s0 = None
    if state_std is not None:
        s0 = torch.randn((N, hv, d, d), generator=gen, device=device,
                         dtype=torch.float32) * state_std
    cu = torch.zeros(N + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    return dict(q=q.to(io_dtype), k=k.to(io_dtype), v=v.to(io_dtype), g=g, beta=beta,
                cu_seqlens=cu.to(device), initial_state=s0, seqlens=seqlens)


def make_decode(num_seqs, ntok, *, hk=HK, hv=HV, d=D, io_dtype=torch.bfloat16,
                gate="softplus", state_std=0.02, seed=0, device="cpu"):
    """Decode / multi-token-verify inputs: q, k ``[N, ntok, hk, d]``, v
    ``[N, ntok, hv, d]``, g, beta ``[N, ntok, hv]`` and state ``[N, hv, d, d]`` (fp32)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    N = num_seqs
    q = torch.randn((N, ntok, hk, d), generator=gen, device=device, dtype=torch.float32)
    k = torch.randn((N, ntok, hk, d), generator=gen, device=device, dtype=torch.float32)
    v = torch.randn((N, ntok, hv, d), generator=gen, device=device, dtype=torch.float32)
    g, beta = _gates(gen, (N, ntok, hv), gate, device)
    state = torch.randn((N, hv, d, d), generator=gen, device=device,
                        dtype=torch.float32) * state_std
    return dict(q=q.to(io_dtype), k=k.to(io_dtype), v=v.to(io_dtype), g=g, beta=beta,
                state=state)


def make_raw_gates(shape, hv=HV, *, scale=1.0, seed=0, device="cpu"):
    """Raw gate projections for the *_raw_gates entry points: x, y ``shape`` (the token
    layout of g and beta, last axis = V heads) drawn N(0, scale^2), and per V head a decay
    rate a ~ U[0.02, 0.2] and a bias b ~ N(0, 0.5^2), all fp32.  (With these, g = -a
    softplus(x + b) lands mostly in [-0.4, 0]; a large ``scale`` drives both activations
    into saturation.)"""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * scale
    y = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * scale
    a = 0.02 + 0.18 * torch.rand((hv,), generator=gen, device=device, dtype=torch.float32)
    b = 0.5 * torch.randn((hv,), generator=gen, device=device, dtype=torch.float32)
    return dict(x=x, y=y, a=a, b=b)


def make(w: Workload, device="cpu", **overrides):
    """Materialise a named workload on ``device``."""
    if w.kind == "prefill":
        kw = dict(hk=w.hk, hv=w.hv, d=w.d, io_dtype=w.io_dtype, gate=w.gate,
                  state_std=w.state_std, seed=w.seed, device=device,
                  num_seqs=w.num_seqs, varlen_range=w.varlen_range)
        kw.update(overrides)
        return make_prefill(w.seqlens, **kw)
    kw = dict(hk=w.hk, hv=w.hv, d=w.d, io_dtype=w.io_dtype, gate=w.gate,
              state_std=w.state_std if w.state_std is not None else 0.02, seed=w.seed,
              device=device)
    kw.update(overrides)
    return make_decode(w.num_seqs, w.ntok, **kw)
