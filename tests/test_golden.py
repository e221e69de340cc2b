"""The oracle reproduces its frozen output on the stored tiny case (CPU only)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_frozen_fixture():
    with open(os.path.join(HERE, "tiny_forward.json")) as f:
        blob = json.load(f)
    c = {k: np.array(v, np.float32) for k, v in blob["inputs"].items()}
    cfg = oracle.config(**blob["config"])
    pos = np.arange(c["q"].shape[0])
    out = oracle.forward(cfg, c["q"], c["q_idx"], c["w"], pos, c["k_idx"], c["k"], c["v"])
    np.testing.assert_array_equal(out["sel"], np.array(blob["sel"]))
    np.testing.assert_array_equal(out["nsel"], np.array(blob["nsel"]))
    np.testing.assert_allclose(out["o"], np.array(blob["o"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(out["lse"], np.array(blob["lse"]), rtol=1e-13)
