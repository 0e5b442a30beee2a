"""Writes tests/golden/tiny_expert_actions.json from the fp64 oracle (and nothing else).

The pages print no worked numerical example, so this file is a regression pin of the oracle
itself: a seeded 2-layer, width-16 expert run through the whole 10-step loop.  Re-running the
script must reproduce the stored numbers exactly; a change to them needs a stated reason.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import model as M  # noqa: E402
from synth import gen  # noqa: E402
from synth import workloads as WL  # noqa: E402


def case():
    cfg = SimpleNamespace(n_layers=2, width=16, mlp_dim=32, n_q_heads=2, n_kv_heads=1, head_dim=8,
                          action_dim=4, n_steps=10, rms_eps=1e-6, rope_theta=10000.0, final_norm=True)
    W = {k: gen.normal(f"golden/{k}", s, 0.1 if k.endswith("_b") else 0.3).astype(np.float64)
         for k, s in WL.expert_weight_shapes(cfg).items()}
    noise = gen.normal("golden/noise", (2, 3, 4), 1.0).astype(np.float64)
    kk = gen.normal("golden/k", (2, 2, 6, 8), 1.0).astype(np.float64)
    vv = gen.normal("golden/v", (2, 2, 6, 8), 1.0).astype(np.float64)
    lv = np.array([4, 6], np.int32)
    return cfg, W, noise, kk, vv, lv


def compute():
    cfg, W, noise, kk, vv, lv = case()
    return M.sample_actions(W, cfg, noise, kk, vv, lv)


if __name__ == "__main__":
    out = compute()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_expert_actions.json")
    with open(path, "w") as f:
        json.dump({"source": "tests/golden/make_golden.py (fp64 oracle, seeded width-16 expert)",
                   "shape": list(out.shape), "actions": [float(x).hex() for x in out.ravel()]}, f, indent=1)
    print("wrote", path)
