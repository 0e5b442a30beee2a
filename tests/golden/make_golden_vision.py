"""Writes tests/golden/tiny_vision_embeddings.json from the fp64 image-encoder oracle (and
nothing else).

The pages print no worked numerical example for the image encoder either, so this file is a
regression pin of oracle/vision.py itself: two seeded 28 x 28 images through a 2-layer,
width-16 tower (4 heads, patch 7, projector to 8).  Re-running the script must reproduce the
stored numbers exactly; a change to them needs a stated reason.
Run: python tests/golden/make_golden_vision.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import vision as V  # noqa: E402
from synth import gen  # noqa: E402
from synth import workloads as WL  # noqa: E402


def case():
    cfg = WL.VisionShape(n_layers=2, width=16, mlp_dim=24, n_heads=4, patch=7, image=28, channels=3,
                         out_width=8)
    W = {}
    for k, s in WL.vision_weight_shapes(cfg).items():
        kind = WL._vision_kind(k)
        x = gen.normal(f"golden-vision/{k}", s, 0.3 if kind == "matrix" else 0.2).astype(np.float64)
        W[k] = 1.0 + x if kind == "ln_gain" else x
    imgs = (2.0 * gen.uniform("golden-vision/images", 2 * 3 * 28 * 28) - 1.0).reshape(2, 3, 28, 28)
    return cfg, W, imgs


def compute():
    cfg, W, imgs = case()
    return V.encode_images(imgs, W, cfg)


if __name__ == "__main__":
    out = compute()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_vision_embeddings.json")
    with open(path, "w") as f:
        json.dump({"source": "tests/golden/make_golden_vision.py (fp64 image-encoder oracle, seeded width-16 tower)",
                   "shape": list(out.shape), "embeddings": [float(x).hex() for x in out.ravel()]}, f, indent=1)
    print("wrote", path)
