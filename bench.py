#!/usr/bin/env python3
"""Benchmark of the Gated DeltaNet layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunked prefill of the Qwen3-Next layer workload (B=1, T=8192, 16 QK /
32 V heads, d=128, bf16 I/O, fp32 state) through the C ABI.  The decode step (256
sequences, fp32 state, 1 token and a 4-token verify) is measured alongside and
reported under "decode".  Inputs are seeded synthetic tensors resident in HBM; L2 is
flushed (a 256 MiB write) between timed steps, outside the timed events.

Multi-GPU: every rank runs an independent replica of the same workload (the layer
shards by sequence and head with no exchange); value = all ranks' tokens / the
slowest rank's time ("scaling": "weak").

--impl reference times the fp64 CPU oracle (the only reference this layer has) on a
bounded sample of the same workload, on this host's cores, and prints the same line
with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (% BF16 tensor peak); decode tokens/s (% HBM GB/s)"
UNIT = "tokens/s"
WORKLOAD = "layer_prefill"
HK, HV, D, C = 16, 32, 128, 64

# Algorithmic work per token of prefill (GEMM flops of the chunked form) and bytes.
PREFILL_FLOP_PER_TOKEN = HV * (3 * 2 * C * D + 3 * 2 * D * D) + HK * (2 * 2 * C * D)  # 5,242,880
PREFILL_BYTES_PER_TOKEN = 2 * HK * D * 2 + HV * D * 2 * 2 + HV * 4 * 2                # 24,832
STATE_BYTES = HV * D * D * 4                                                          # per sequence
# Split of the GEMM flops between the two tensor-core phases:
#   prep  = Gram matrices (per QK head) + W and U (per V head)
#   state = [W; Q] S^T, P Delta and the state update (per V head)
PREP_FLOP_PER_TOKEN = HK * (2 * 2 * C * D) + HV * (2 * 2 * C * D)                    # 1,572,864
STATE_FLOP_PER_TOKEN = HV * (2 * C * D + 3 * 2 * D * D)                               # 3,670,016
# Algorithmic HBM bytes per full 64-token chunk of each tensor-core phase (the roofline
# of both phases is the HBM one: their flop/byte ratios, about 30 and 90, are far below
# the B200's bf16 ridge point).
#   prep  reads q, k (bf16, per QK head), v (bf16), g, beta (fp32, per V head) once and
#         writes the chunk's operand images: per V head W~ and U (64 x 128 bf16 each),
#         P and M~ (64 x 64 bf16 each), diag(c) K (64 x 128 bf16) and the gate factors
#         (129 fp32); per QK head the normalised Q (64 x 128 bf16).
#   state reads those images once (Q, W~, M~, P, diag(c) K, U, gate factors) and writes
#         the outputs (64 x 128 bf16 per V head); the state itself enters and leaves once
#         per sequence (fp32, counted separately).
PREP_BYTES_PER_CHUNK = (C * (2 * HK * D * 2 + HV * D * 2 + HV * 4 * 2)
                        + HV * (3 * C * D * 2 + 2 * C * C * 2 + 129 * 4) + HK * C * D * 2)   # 3,440,768
STATE_BYTES_PER_CHUNK = (HK * C * D * 2 + HV * (3 * C * D * 2 + 2 * C * C * 2 + 129 * 4)
                         + HV * C * D * 2)                                                  # 2,900,096


def decode_bytes(num_seqs, ntok):
    """State read + write, q, k, v, out and gates for one decode step."""
    return num_seqs * (STATE_BYTES * 2 + ntok * PREFILL_BYTES_PER_TOKEN)


def source_code_sha256(path):
    """sha256 of a C/CUDA source with its comments removed and its whitespace collapsed, so
    that a record of measured counters stays keyed to the code it was taken on across edits
    of comments and layout only."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()


def load_traffic():
    """DRAM bytes per launch of the prefill kernels from the committed ncu record, or {} if
    the record is missing or was taken on a different version of the kernel code."""
    rec = os.path.join(ROOT, "profiles", "traffic_layer_T8192.txt")
    try:
        lines = open(rec).read().splitlines()
    except OSError:
        return {}
    fields = dict(l.split(": ", 1) for l in lines if ": " in l and not l.startswith("#"))
    try:
        src = os.path.join(ROOT, fields["source"])
        if source_code_sha256(src) != fields["source_code_sha256"]:
            return {}
        out = {}
        for kname in ("chunk_table_kernel", "chunk_prep_kernel", "chunk_state_kernel"):
            parts = fields[kname].split()
            out[kname] = int(parts[1]) + int(parts[3])
        return out
    except (KeyError, OSError, ValueError, IndexError):
        return {}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


# ---------------------------------------------------------------- clocks sampling
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- reference arm
def oracle_tokens_per_s(x, heads_sample, threads=None):
    """Times the fp64 oracle on `heads_sample` QK heads of workload x and scales to the
    whole workload's tokens/s (heads are independent, so cost is linear in heads)."""
    import oracle
    T = x["q"].shape[0]
    hk = x["q"].shape[1]
    t0 = time.perf_counter()
    oracle.forward_heads(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                         list(range(heads_sample)), threads=threads)
    dt = time.perf_counter() - t0
    return T / (dt * hk / heads_sample), dt


def reference_arm(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    from linear_attention_layer_gated_b200 import inputs
    x = inputs.make(inputs.workload(WORKLOAD), device="cpu")
    cores = oracle.host_threads()
    heads_sample = HK
    vals = []
    for _ in range(max(args.warmup, 0)):
        oracle_tokens_per_s(x, heads_sample)
    for _ in range(args.steps):
        v, dt = oracle_tokens_per_s(x, heads_sample)
        vals.append(v)
    value = statistics.mean(vals)
    T = x["q"].shape[0]
    sample = ("fp64 oracle (token recurrence, C, %d threads) on the whole T=%d, 16/32-head "
              "workload, one pass per step" % (cores, T))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": T / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "layer_prefill: B=1, T=8192, 16 QK / 32 V heads, d=128",
                       "sample": "whole workload"},
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": cores,
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def main_ours(args, rank, world, local_rank):
    import torch
    from linear_attention_layer_gated_b200 import build, gdn, inputs, replicas

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    algo = {"auto": gdn.GDN_ALGO_AUTO, "simt": gdn.GDN_ALGO_SIMT,
            "tensor": gdn.GDN_ALGO_TENSOR}[args.algo]

    w = inputs.workload(WORKLOAD)
    if args.tokens:
        w.seqlens = [args.tokens]
    x = inputs.make(w, device=dev)
    T = x["q"].shape[0]
    out = torch.empty_like(x["v"])
    fin = torch.empty((1, HV, D, D), dtype=torch.float32, device=dev)
    shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo)
    ws = gdn.alloc_workspace(shape, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    tensor_path = gdn_launches_per_prefill(algo, x["q"].dtype) == 3
    phase_ev = []

    def prefill_once():
        gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                              out, fin, workspace=ws, algo=algo, stream=stream)

    def prefill_phased():
        # the same two launches gdn_chunk_prefill makes, with events between them
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        gdn.gdn_chunk_prefill_prep(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"],
                                   ws, algo=algo, stream=stream)
        e[1].record(stream)
        gdn.gdn_chunk_prefill_state(None, x["cu_seqlens"], out, fin, ws, x["q"], algo=algo,
                                    stream=stream)
        e[2].record(stream)
        phase_ev.append(e)

    def barrier():
        replicas.barrier(world)
        torch.cuda.synchronize(dev)

    def timed(fn, steps, warmup, flush_between=True):
        for _ in range(warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier()
        for a, b in ev:
            if flush_between:
                flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        barrier()
        return [a.elapsed_time(b) for a, b in ev]

    def max_over_ranks(v):
        return replicas.max_over_ranks(v, world, device=dev)

    # the step as a user runs it: one gdn_chunk_prefill call
    with ClockSampler(local_rank) as clk:
        ms = timed(prefill_once, args.steps, args.warmup)
    clocks = clk.summary()
    if tensor_path:  # the same launches with events between them, for the phase rooflines
        timed(prefill_phased, args.steps, args.warmup)
    ms_step = max_over_ranks(sum(ms) / len(ms))
    value = replicas.job_throughput(T, world, ms_step * 1e-3)

    # ---- dominant kernel roofline, from CUDA events on the launching stream
    launches_per_step = gdn_launches_per_prefill(algo, x["q"].dtype)
    peak = peaks["bf16_tflops"]
    phases = None
    if tensor_path:
        timed_ev = phase_ev[-args.steps:]
        prep_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in timed_ev) / args.steps)
        state_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in timed_ev) / args.steps)
        chunks = T // C  # one sequence of T tokens, T a multiple of the chunk size
        phases = {
            "prep": {"kernels": "chunk_table_kernel + chunk_prep_kernel", "ms": prep_ms,
                     "flop": PREP_FLOP_PER_TOKEN * T, "bytes": PREP_BYTES_PER_CHUNK * chunks},
            "state": {"kernels": "chunk_state_kernel", "ms": state_ms,
                      "flop": STATE_FLOP_PER_TOKEN * T,
                      "bytes": STATE_BYTES_PER_CHUNK * chunks + 2 * STATE_BYTES}}
        for ph in phases.values():
            ph["tflops"] = ph["flop"] / (ph["ms"] * 1e-3) / 1e12
            ph["gbs"] = ph["bytes"] / (ph["ms"] * 1e-3) / 1e9
            ph["frac_hbm"] = ph["gbs"] / peaks["hbm_gbs"]
            ph["frac_tensor"] = ph["tflops"] / peak
        dom = max(phases, key=lambda k2: phases[k2]["ms"])
        d = phases[dom]
        traffic = None
        tr = load_traffic() if T == 8192 and len(x["cu_seqlens"]) == 2 else {}
        if tr:
            traffic = (tr["chunk_table_kernel"] + tr["chunk_prep_kernel"]) if dom == "prep" else tr["chunk_state_kernel"]
        roofline = {"bound": "hbm", "achieved": d["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": d["frac_hbm"], "traffic": traffic,
                    "peak_source": peaks["source"] + " HBM copy",
                    "kernel": d["kernels"], "algorithmic_bytes_per_launch": d["bytes"],
                    "tensor_frac": d["frac_tensor"],
                    "step_frac_tensor": PREFILL_FLOP_PER_TOKEN * T / (ms_step * 1e-3) / 1e12 / peak}
    else:
        flop = PREFILL_FLOP_PER_TOKEN * T
        achieved = flop / (ms_step * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "peak_source": peaks["source"] + " bf16 dense (burst)",
                    "kernel": "prefill_simt_kernel", "algorithmic_flop_per_launch": flop}

    # ---- end to end through the C ABI with pinned host buffers
    host = {k2: x[k2].cpu().pin_memory() for k2 in ("q", "k", "v", "g", "beta", "cu_seqlens")}
    dbuf = {k2: torch.empty_like(x[k2]) for k2 in host}
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_once():
        for k2 in host:
            dbuf[k2].copy_(host[k2], non_blocking=True)
        gdn.gdn_chunk_prefill(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"], None,
                              dbuf["cu_seqlens"], out, fin, workspace=ws, algo=algo, stream=stream)
        hout.copy_(out, non_blocking=True)

    def e2e_pipelined(steps):
        """`steps` prefills back to back, each with its own host->device input copy and
        device->host output copy, pipelined over three streams with double-buffered device
        inputs and outputs: the copies of neighbouring steps overlap each other (PCIe is
        full duplex) and the kernels.  Returns ms per step (device events, whole loop)."""
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        bufs = [{k2: torch.empty_like(x[k2]) for k2 in host} for _ in range(2)]
        outs = [torch.empty_like(out) for _ in range(2)]
        houts = [hout, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
        ev = lambda: torch.cuda.Event()  # noqa: E731
        h2d_done, comp_done, d2h_done = [ev() for _ in range(steps)], [ev() for _ in range(steps)], [ev() for _ in range(steps)]
        torch.cuda.synchronize(dev)
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(steps):
            b2 = i % 2
            if i >= 2:
                s_in.wait_event(comp_done[i - 2])
            with torch.cuda.stream(s_in):
                for k2 in host:
                    bufs[b2][k2].copy_(host[k2], non_blocking=True)
            h2d_done[i].record(s_in)
            stream.wait_event(h2d_done[i])
            if i >= 2:
                stream.wait_event(d2h_done[i - 2])
            gdn.gdn_chunk_prefill(bufs[b2]["q"], bufs[b2]["k"], bufs[b2]["v"], bufs[b2]["g"], bufs[b2]["beta"],
                                  None, bufs[b2]["cu_seqlens"], outs[b2], fin, workspace=ws, algo=algo,
                                  stream=stream)
            comp_done[i].record(stream)
            s_out.wait_event(comp_done[i])
            with torch.cuda.stream(s_out):
                houts[b2].copy_(outs[b2], non_blocking=True)
            d2h_done[i].record(s_out)
        s_out.wait_event(d2h_done[steps - 1])
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        return t0.elapsed_time(t1) / steps

    e2e = None
    if not args.no_e2e:
        e2e_ms = timed(e2e_once, max(3, args.steps // 2), 2)
        serial_step = max_over_ranks(sum(e2e_ms) / len(e2e_ms))
        e2e_pipelined(3)  # warm-up
        e2e_step = max_over_ranks(e2e_pipelined(max(4, args.steps)))
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = hout.numel() * hout.element_size()
        e2e = {"value": world * T / (e2e_step * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_step, "pipelined": True,
               "serial_value": world * T / (serial_step * 1e-3)}

    # ---- decode: 256 sequences, 1 token and 4-token verify
    dec = {}
    for ntok in ((1, 4) if args.only != "prefill" else ()):
        d = inputs.make_decode(256, ntok, seed=3, device=dev)
        dout = torch.empty_like(d["v"])

        def dec_once():
            gdn.gdn_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], dout,
                                stream=stream)

        dms = timed(dec_once, max(args.steps, 10), args.warmup)
        dstep = max_over_ranks(sum(dms) / len(dms))
        nbytes = decode_bytes(256, ntok)
        gbs = nbytes / (dstep * 1e-3) / 1e9
        dec["ntok%d" % ntok] = {
            "tokens_per_s": world * 256 * ntok / (dstep * 1e-3), "ms_per_step": dstep,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "frac_of_8TBs": gbs / 8000.0,
                         "traffic": None, "algorithmic_bytes_per_launch": nbytes}}

    # ---- speculative verify (4 draft tokens, per-token state snapshots) and the commit of
    #      the accepted prefix (2 of 4 accepted everywhere), 256 sequences
    if args.only != "prefill":
        ntok = 4
        d = inputs.make_decode(256, ntok, seed=3, device=dev)
        dout = torch.empty_like(d["v"])
        snaps = torch.empty((256, ntok, HV, D, D), dtype=torch.float32, device=dev)
        acc = torch.full((256,), 2, dtype=torch.int32, device=dev)

        def verify_once():
            gdn.gdn_decode_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], dout, snaps,
                                  stream=stream)

        def commit_once():
            gdn.gdn_decode_commit(d["state"], snaps, acc, stream=stream)

        for name, fn, nbytes in (
                ("verify4_snapshots", verify_once,
                 256 * (STATE_BYTES * (1 + ntok) + ntok * PREFILL_BYTES_PER_TOKEN)),
                ("commit", commit_once, 256 * STATE_BYTES * 2 + 256 * 4)):
            dms = timed(fn, max(args.steps, 10), args.warmup)
            dstep = max_over_ranks(sum(dms) / len(dms))
            gbs = nbytes / (dstep * 1e-3) / 1e9
            dec[name] = {
                "ms_per_step": dstep,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                             "algorithmic_bytes_per_launch": nbytes}}
        dec["verify4_snapshots"]["tokens_per_s"] = world * 256 * ntok / (dec["verify4_snapshots"]["ms_per_step"] * 1e-3)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.tokens:
        import oracle
        xs = {k2: (x[k2].cpu() if hasattr(x[k2], "cpu") else x[k2]) for k2 in x}
        v_cpu, dt = oracle_tokens_per_s(xs, HK)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": oracle.host_threads(), "kind": "oracle",
               "sample": "fp64 oracle (token recurrence) on the whole T=8192, 16/32-head "
                         "workload, one pass, %.1f s" % dt}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "layer_prefill: B=1, T=8192, 16 QK / 32 V heads, d=128, "
                                       "bf16 I/O, fp32 state, chunk 64",
                           "parallelism": "replicas" if world > 1 else "single",
                           "l2": "flushed between timed steps (256 MiB write)",
                           "algo": args.algo},
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "phases": phases,
                "decode": dec, "clocks": clocks, "peaks": peaks}
        print(json.dumps(line), flush=True)
    return 0


def gdn_launches_per_prefill(algo, dtype):
    """Kernels libgdn.so launches per gdn_chunk_prefill call on the chosen path:
    the SIMT path is one kernel; the tensor-core path is chunk table, chunk prep and
    chunk state (the workspace-header memset is not a kernel of ours)."""
    from linear_attention_layer_gated_b200 import gdn
    import torch
    tensor = algo == gdn.GDN_ALGO_TENSOR or (algo == gdn.GDN_ALGO_AUTO and dtype == torch.bfloat16)
    return 3 if tensor else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--only", default="all", choices=["all", "prefill"],
                    help="prefill: skip the decode measurements (profiling runs)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the prefill length (profiling runs; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    from linear_attention_layer_gated_b200 import replicas
    rank, world, local_rank = replicas.rank_info()
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    replicas.init(world, local_rank, "nccl")
    try:
        return main_ours(args, rank, world, local_rank)
    finally:
        replicas.finish(world)


if __name__ == "__main__":
    sys.exit(main())
