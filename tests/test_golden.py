"""The oracle reproduces its stored values on the tiny seeded workload."""
import json
import os

import numpy as np

import oracle
from linear_attention_layer_gated_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_reproduces_golden_tiny():
    doc = json.load(open(os.path.join(HERE, "golden", "tiny_oracle.json")))
    x = inputs.make(inputs.workload("tiny"), device="cpu")
    out, fin = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu_seqlens"], None)
    np.testing.assert_allclose(np.linalg.norm(out), doc["out_fro_norm"], rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(fin), doc["state_fro_norm"], rtol=1e-12)
    for t, h, i, val in doc["out_samples"]:
        np.testing.assert_allclose(out[t, h, i], val, rtol=1e-12, atol=1e-15)
    for h, i, j, val in doc["state_samples"]:
        np.testing.assert_allclose(fin[0, h, i, j], val, rtol=1e-12, atol=1e-15)
