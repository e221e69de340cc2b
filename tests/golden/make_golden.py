"""Write tests/golden/tiny_forward.json from the CPU oracle (calls only oracle/).

The pages print no worked numeric example for QSA, so no stored value here is
the pages'.  This fixture is a regression guard: it freezes the oracle's
output on a tiny seeded case (inputs stored alongside) so that any later
change to the oracle's arithmetic shows up as a diff that must be justified.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_forward.json")
CFG = dict(r=4, budget_tokens=12, n_heads=4, n_groups=2, head_dim=8, idx_heads=4, idx_dim=16,
           rope_dims=4, rope_base=1e7, round_bf16=True)


def case():
    rng = np.random.default_rng(20240601)
    n = 40

    def bf(a):  # inputs are bf16 values held in fp32
        return np.array([oracle.round_bf16(x) for x in a.ravel()], np.float32).reshape(a.shape)
    return dict(q=bf(rng.standard_normal((n, 4, 8))), q_idx=bf(rng.standard_normal((n, 4, 16))),
                w=rng.random((n, 4)).astype(np.float32), k_idx=bf(rng.standard_normal((n, 16))),
                k=bf(rng.standard_normal((2, n, 8))), v=bf(rng.standard_normal((2, n, 8))))


def run(c):
    cfg = oracle.config(**CFG)
    pos = np.arange(c["q"].shape[0])
    return oracle.forward(cfg, c["q"], c["q_idx"], c["w"], pos, c["k_idx"], c["k"], c["v"])


if __name__ == "__main__":
    c = case()
    out = run(c)
    blob = {"config": CFG, "inputs": {k: v.tolist() for k, v in c.items()},
            "sel": out["sel"].tolist(), "nsel": out["nsel"].tolist(),
            "o": out["o"].tolist(), "lse": out["lse"].tolist()}
    with open(OUT, "w") as f:
        json.dump(blob, f)
    print("wrote", OUT)
