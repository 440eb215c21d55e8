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

# Algorithmic work of the method (what any implementation must do; no intermediate of
# ours is counted).  Prefill reads q, k (bf16, per QK head), v (bf16) and g, beta (fp32,
# per V head) once, writes out (bf16) once, and reads / writes each sequence's fp32 state
# once when an initial / final state is given.  GEMM flops are those of the chunked form.
INPUT_BYTES_PER_TOKEN = 2 * HK * D * 2 + HV * D * 2 + 2 * HV * 4                      # 16,640
OUTPUT_BYTES_PER_TOKEN = HV * D * 2                                                   # 8,192
PREFILL_BYTES_PER_TOKEN = INPUT_BYTES_PER_TOKEN + OUTPUT_BYTES_PER_TOKEN              # 24,832
PREFILL_FLOP_PER_TOKEN = HV * (3 * 2 * C * D + 3 * 2 * D * D) + HK * (2 * 2 * C * D)  # 5,242,880
STATE_BYTES = HV * D * D * 4                                                          # per sequence
# The two tensor-core phases split that work:
#   prep  = Gram matrices (per QK head) and W, U (per V head); reads every input
#   state = [W; Q] S^T, P Delta and the state update (per V head); writes every output and
#           reads / writes the states
PREP_FLOP_PER_TOKEN = HK * (2 * 2 * C * D) + HV * (2 * 2 * C * D)                    # 1,572,864
STATE_FLOP_PER_TOKEN = HV * (2 * C * D + 3 * 2 * D * D)                               # 3,670,016


def prefill_work(T, N, with_initial, with_final):
    """Algorithmic (bytes, flop) of one prefill of T packed tokens in N sequences."""
    nbytes = T * PREFILL_BYTES_PER_TOKEN + N * STATE_BYTES * (int(with_initial) + int(with_final))
    return nbytes, T * PREFILL_FLOP_PER_TOKEN


def phase_work(T, N, with_initial, with_final):
    """Algorithmic (bytes, flop) of each tensor-core phase: prep reads the inputs, state
    writes the outputs and moves the states."""
    return {"prep": (T * INPUT_BYTES_PER_TOKEN, T * PREP_FLOP_PER_TOKEN),
            "state": (T * OUTPUT_BYTES_PER_TOKEN + N * STATE_BYTES * (int(with_initial) + int(with_final)),
                      T * STATE_FLOP_PER_TOKEN)}


def roofline_of(nbytes, flop, ms, peaks):
    """Achieved rates of a kernel (or step) against both peaks; its bound is the one its
    arithmetic intensity selects (tensor above the ridge point flop/byte, HBM below)."""
    s = ms * 1e-3
    gbs, tflops = nbytes / s / 1e9, flop / s / 1e12
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if nbytes == 0 or flop / nbytes >= ridge else "hbm"
    r = {"gbs": gbs, "tflops": tflops, "frac_hbm": gbs / peaks["hbm_gbs"],
         "frac_tensor": tflops / peaks["bf16_tflops"], "bound": bound,
         "intensity_flop_per_byte": flop / nbytes if nbytes else None, "ridge_flop_per_byte": ridge}
    return r


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
        for kname in ("chunk_table_kernel", "chunk_prep_kernel", "chunk_state_kernel", "chunk_fused_kernel"):
            if kname in fields:
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

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

    def prefill_step_fn(x, out, fin, ws, with_initial, segments=1):
        """One step: gdn_chunk_prefill over the workload, or over `segments` equal pieces of
        its single sequence with the state carried in place from one call to the next."""
        s0 = x["initial_state"] if with_initial else None
        if segments == 1:
            return lambda: gdn.gdn_chunk_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], s0,
                                                 x["cu_seqlens"], out, fin, workspace=ws, algo=algo,
                                                 stream=stream)
        T = x["q"].shape[0]
        seg = T // segments
        cu = torch.tensor([0, seg], dtype=torch.int32, device=dev)
        views = [{k2: x[k2][i * seg:(i + 1) * seg] for k2 in ("q", "k", "v", "g", "beta")}
                 for i in range(segments)]
        outs = [out[i * seg:(i + 1) * seg] for i in range(segments)]

        def run():
            for i in range(segments):
                v = views[i]
                gdn.gdn_chunk_prefill(v["q"], v["k"], v["v"], v["g"], v["beta"], s0 if i == 0 else fin,
                                      cu, outs[i], fin, workspace=ws, algo=algo, stream=stream)
        return run

    tensor_path = gdn_launches_per_prefill(algo, torch.bfloat16) > 1

    def measure_prefill(w, steps, warmup, with_initial, segments=1, phased=False, clocks=False):
        """Times one prefill workload; returns (record, x, out, fin, ws)."""
        x = inputs.make(w, device=dev)
        T, N = x["q"].shape[0], x["cu_seqlens"].numel() - 1
        out = torch.empty_like(x["v"])
        fin = torch.empty((N, HV, D, D), dtype=torch.float32, device=dev)
        if segments == 1:
            shape = gdn.prefill_shape(x["q"], x["v"], x["cu_seqlens"], algo)
        else:  # every call sees one sequence of T / segments tokens
            shape = gdn.make_shape(1, T // segments, HK, HV, D, gdn.GDN_BF16, algo)
        ws = gdn.alloc_workspace(shape, dev, phases=phased)
        fn = prefill_step_fn(x, out, fin, ws, with_initial, segments)
        clk = ClockSampler(local_rank) if clocks else None
        if clk:
            with clk:
                ms = timed(fn, steps, warmup)
        else:
            ms = timed(fn, steps, warmup)
        ms_step = max_over_ranks(sum(ms) / len(ms))
        nbytes, flop = prefill_work(T, N, with_initial, True)
        rec = {"tokens": T, "sequences": N, "ms_per_step": ms_step,
               "tokens_per_s": replicas.job_throughput(T, world, ms_step * 1e-3),
               "step": roofline_of(nbytes, flop, ms_step, peaks),
               "algorithmic_bytes": nbytes, "algorithmic_flop": flop}
        if segments > 1:
            rec["segments"] = segments
        if clk:
            rec["clocks"] = clk.summary()
        if phased and tensor_path and segments == 1:
            # the same two launches gdn_chunk_prefill makes, with events between them
            evs = []

            def phased_fn():
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                e[0].record(stream)
                gdn.gdn_chunk_prefill_prep(x["q"], x["k"], x["g"], x["beta"], x["cu_seqlens"], ws, x["v"],
                                           algo=algo, stream=stream)
                e[1].record(stream)
                gdn.gdn_chunk_prefill_state(x["k"], x["v"], x["initial_state"] if with_initial else None,
                                            x["cu_seqlens"], out, fin, ws, algo=algo, stream=stream)
                e[2].record(stream)
                evs.append(e)
            timed(phased_fn, steps, warmup)
            tev = evs[-steps:]
            phase_ms = {"prep": max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in tev) / steps),
                        "state": max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in tev) / steps)}
            kernels = {"prep": "chunk_table_kernel + chunk_prep_kernel", "state": "chunk_state_kernel"}
            rec["phases"] = {}
            for ph, (pb, pf) in phase_work(T, N, with_initial, True).items():
                r = roofline_of(pb, pf, phase_ms[ph], peaks)
                r.update(kernels=kernels[ph], ms=phase_ms[ph], algorithmic_bytes=pb, algorithmic_flop=pf)
                rec["phases"][ph] = r
            # the GEMM-phase figure: all GEMM flops over the time of the GEMM phases
            gemm_ms = phase_ms["prep"] + phase_ms["state"]
            rec["gemm_phases_frac_tensor"] = flop / (gemm_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]
        return rec, x, out, fin, ws

    # ---- the headline: the layer workload (B=1, T=8192), one gdn_chunk_prefill call per step
    w = inputs.workload(WORKLOAD)
    if args.tokens:
        w.seqlens = [args.tokens]
    main_rec, x, out, fin, ws = measure_prefill(w, args.steps, args.warmup, False, phased=True, clocks=True)
    T = main_rec["tokens"]
    ms_step = main_rec["ms_per_step"]
    value = main_rec["tokens_per_s"]
    clocks = main_rec.pop("clocks", None)
    launches_per_step = gdn_launches_per_prefill(algo, x["q"].dtype)
    phases = main_rec.get("phases")
    step = main_rec["step"]
    fused = launches_per_step == 2
    if fused:
        # one chunk-table launch and one fused launch per step: the step's events time exactly
        # them, and the whole step's algorithmic work is the fused kernel's
        nbytes, flop = prefill_work(T, 1, False, True)
        tr = load_traffic() if T == 8192 else {}
        traffic = (tr["chunk_table_kernel"] + tr["chunk_fused_kernel"]) if "chunk_fused_kernel" in tr else None
        unit_hbm = step["bound"] == "hbm"
        roofline = {"bound": step["bound"],
                    "achieved": step["gbs"] if unit_hbm else step["tflops"],
                    "peak": peaks["hbm_gbs"] if unit_hbm else peaks["bf16_tflops"],
                    "unit": "GB/s" if unit_hbm else "TFLOP/s",
                    "frac": step["frac_hbm"] if unit_hbm else step["frac_tensor"],
                    "traffic": traffic,
                    "traffic_over_algorithmic_bytes": (traffic / nbytes) if traffic else None,
                    "peak_source": peaks["source"] + (" HBM copy" if unit_hbm else " bf16 dense (burst)"),
                    "kernel": "chunk_table_kernel + chunk_fused_kernel (prep and state passes in one cooperative launch)",
                    "algorithmic_bytes_per_launch": nbytes, "algorithmic_flop_per_launch": flop,
                    "frac_hbm": step["frac_hbm"], "frac_tensor": step["frac_tensor"],
                    "step_frac_tensor": step["frac_tensor"], "step_frac_hbm": step["frac_hbm"],
                    "gemm_phases_frac_tensor": step["frac_tensor"],
                    "two_phase_path_frac_tensor": main_rec.get("gemm_phases_frac_tensor")}
    elif phases:
        dom = max(phases, key=lambda k2: phases[k2]["ms"])
        d = phases[dom]
        traffic = None
        tr = load_traffic() if T == 8192 else {}
        if tr:
            traffic = (tr["chunk_table_kernel"] + tr["chunk_prep_kernel"]) if dom == "prep" else tr["chunk_state_kernel"]
        unit_hbm = d["bound"] == "hbm"
        roofline = {"bound": d["bound"],
                    "achieved": d["gbs"] if unit_hbm else d["tflops"],
                    "peak": peaks["hbm_gbs"] if unit_hbm else peaks["bf16_tflops"],
                    "unit": "GB/s" if unit_hbm else "TFLOP/s",
                    "frac": d["frac_hbm"] if unit_hbm else d["frac_tensor"],
                    "traffic": traffic,
                    "traffic_over_algorithmic_bytes": (traffic / d["algorithmic_bytes"]) if traffic else None,
                    "peak_source": peaks["source"] + (" HBM copy" if unit_hbm else " bf16 dense (burst)"),
                    "kernel": d["kernels"], "algorithmic_bytes_per_launch": d["algorithmic_bytes"],
                    "algorithmic_flop_per_launch": d["algorithmic_flop"],
                    "frac_hbm": d["frac_hbm"], "frac_tensor": d["frac_tensor"],
                    "step_frac_tensor": step["frac_tensor"], "step_frac_hbm": step["frac_hbm"],
                    "gemm_phases_frac_tensor": main_rec["gemm_phases_frac_tensor"]}
    else:
        nbytes, flop = prefill_work(T, 1, False, True)
        roofline = {"bound": "tensor", "achieved": step["tflops"], "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": step["frac_tensor"], "traffic": None,
                    "peak_source": peaks["source"] + " bf16 dense (burst)",
                    "kernel": "prefill_simt_kernel", "algorithmic_flop_per_launch": flop,
                    "step_frac_tensor": step["frac_tensor"], "step_frac_hbm": step["frac_hbm"]}
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

    # ---- the other prefill workloads: varlen (8 sequences with initial and final states) and
    #      long context (T = 262,144 whole, and as 4 segments of 65,536 with the state carried)
    others = {}
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline and not args.tokens
    cpu_samples = {}
    if want_cpu:  # the layer workload's inputs, as the GPU drew them
        cpu_samples["layer"] = {k2: x[k2].cpu() for k2 in ("q", "k", "v", "g", "beta", "cu_seqlens")}
    if not args.tokens and args.only == "all":
        del x, out, fin, ws
        torch.cuda.empty_cache()
        for name, w2, kw in (("varlen", inputs.workload("varlen"), dict(with_initial=True)),
                             ("long", inputs.workload("long"), dict(with_initial=False)),
                             ("long_4x65536_carry", inputs.workload("long"), dict(with_initial=False, segments=4))):
            rec, x2, *_bufs = measure_prefill(w2, max(5, args.steps // 2), args.warmup,
                                              phased=(name != "long_4x65536_carry"), **kw)
            if want_cpu and name == "varlen":  # 4 of the 16 QK heads and the 8 V heads that read them
                cpu_samples[name] = {"q": x2["q"][:, :4].cpu(), "k": x2["k"][:, :4].cpu(), "v": x2["v"][:, :8].cpu(),
                                     "g": x2["g"][:, :8].cpu(), "beta": x2["beta"][:, :8].cpu(),
                                     "cu_seqlens": x2["cu_seqlens"].cpu(),
                                     "initial_state": x2["initial_state"][:, :8].cpu()}
            if want_cpu and name == "long":  # every head of the first 16,384 tokens
                cpu_samples[name] = {k2: x2[k2][:16384].cpu() for k2 in ("q", "k", "v", "g", "beta")}
                cpu_samples[name]["cu_seqlens"] = torch.tensor([0, 16384], dtype=torch.int32)
            del x2, _bufs
            torch.cuda.empty_cache()
            others[name] = rec

    # ---- CPU baseline: the fp64 oracle on bounded samples of the same inputs (rank 0, N=1 only)
    cpu = None
    if want_cpu:
        import oracle
        cores = oracle.host_threads()

        def oracle_rate(xs, with_initial, scale_heads):
            t0 = time.perf_counter()
            oracle.forward(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["cu_seqlens"],
                           xs["initial_state"] if with_initial else None)
            dt = time.perf_counter() - t0
            return xs["q"].shape[0] / (dt * scale_heads), dt

        v_cpu, dt = oracle_rate(cpu_samples["layer"], False, 1)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": "fp64 oracle (token recurrence) on the whole T=8192, 16/32-head "
                         "workload, one pass, %.1f s" % dt}
        if "varlen" in cpu_samples:
            vv, dtv = oracle_rate(cpu_samples["varlen"], True, HK / 4)
            others["varlen"]["cpu_baseline"] = {
                "value": vv, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": "4 of 16 QK heads (8 of 32 V heads) of all %d packed tokens with their "
                          "initial states, %.1f s, scaled to 16 heads" % (cpu_samples["varlen"]["q"].shape[0], dtv)}
        if "long" in cpu_samples:
            vl, dtl = oracle_rate(cpu_samples["long"], False, 1)
            for nm in ("long", "long_4x65536_carry"):
                others[nm]["cpu_baseline"] = {
                    "value": vl, "unit": UNIT, "cores": cores, "kind": "oracle",
                    "sample": "every head of the first 16384 tokens, %.1f s (the recurrence's cost is "
                              "linear in tokens)" % dtl}

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
                "phases_path": "gdn_chunk_prefill_prep and gdn_chunk_prefill_state, the two-kernel path, timed as "
                               "separate launches on the same inputs",
                "gemm_phases_frac_tensor": main_rec.get("gemm_phases_frac_tensor"),
                "configs": others, "decode": dec, "clocks": clocks, "peaks": peaks}
        print(json.dumps(line), flush=True)
    return 0


def fused_prefill_applies(num_seqs, hv):
    """The library's rule for the one-launch tensor-core prefill (prep and state passes in one
    cooperative kernel): the (sequence, V head) chains fill at most half of the SMs."""
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    return 2 * num_seqs * hv <= props.multi_processor_count


def gdn_launches_per_prefill(algo, dtype, num_seqs=1, hv=HV):
    """Kernels libgdn.so launches per gdn_chunk_prefill call on the chosen path:
    the SIMT path is one kernel; the tensor-core path is the chunk table and then either the
    fused kernel or chunk prep and chunk state (the fp32 path's header memset is not a
    kernel of ours)."""
    from linear_attention_layer_gated_b200 import gdn
    import torch
    tensor = algo == gdn.GDN_ALGO_TENSOR or (algo == gdn.GDN_ALGO_AUTO and dtype == torch.bfloat16)
    if not tensor:
        return 1
    return 2 if fused_prefill_applies(num_seqs, hv) else 3


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode"],
                    help="profiling runs: prefill = the layer workload only; decode = the layer "
                         "workload and the decode measurements, without the other prefill configs")
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
