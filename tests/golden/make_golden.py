"""Writes tests/golden/tiny_oracle.json from the fp64 oracle alone.

The pages print no worked example of the Gated DeltaNet recurrence, so the only
stored values are the oracle's own, on the tiny seeded workload (B=1, T=256,
2 QK / 4 V heads, d=128, fp32 inputs, g ~ U[-0.1, 0], beta = sigmoid(N(0,1)),
zero initial state, seed 0).  They pin the oracle against accidental change; the
oracle itself is pinned by closed forms and invariants in test_oracle_pins.py.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from linear_attention_layer_gated_b200 import inputs  # noqa: E402


def sample_index(T, HV, D, n, seed=1234):
    r = np.random.default_rng(seed)
    return np.stack([r.integers(0, T, n), r.integers(0, HV, n), r.integers(0, D, n)], 1)


def main():
    w = inputs.workload("tiny")
    x = inputs.make(w, device="cpu")
    out, fin = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], None)
    idx = sample_index(*out.shape, 64)
    sidx = sample_index(out.shape[2], out.shape[1], out.shape[2], 64, seed=99)
    doc = {
        "workload": "tiny: B=1, T=256, HK=2, HV=4, d=128, fp32, g~U[-0.1,0], beta=sigmoid(N(0,1)), S0=0, seed 0",
        "source": "oracle.forward (fp64 token recurrence); written by tests/golden/make_golden.py",
        "out_fro_norm": float(np.linalg.norm(out)),
        "state_fro_norm": float(np.linalg.norm(fin)),
        "out_samples": [[int(t), int(h), int(i), float(out[t, h, i])] for t, h, i in idx],
        "state_samples": [[int(h), int(i), int(j), float(fin[0, h, i, j])] for i, h, j in sidx],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    text = "{\n"
    for i, (key, val) in enumerate(doc.items()):
        if isinstance(val, list):
            text += ' "%s": [\n' % key + ",\n".join("  " + json.dumps(x) for x in val) + "\n ]"
        else:
            text += ' "%s": %s' % (key, json.dumps(val))
        text += ",\n" if i < len(doc) - 1 else "\n"
    with open(path, "w") as f:
        f.write(text + "}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
