"""Pins of the image front-end oracle (oracle/vision.py) to things other than itself (CPU).

Each test checks the oracle against a library routine used as an independent formulation
(torch fp64 conv2d, LayerNorm, MultiheadAttention), brute force on a tiny input, a closed
form or an invariant, so that a transposed patch, a dropped bias, a wrong normalisation or
scale, or a mixed-up token order fails one of them.  The shapes follow the Realtime-VLA
tech blog ("pi0.5 inference flow": SigLIP with 27 layers, 224 x 224 -> 256 tokens, the
1152 -> 2048 projector, embeddings scaled by sqrt(2048)) and readings V1-V8 of the oracle.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vision as V
from synth import gen
from synth import workloads as WL

RNG = np.random.default_rng(4321)
EMB_REL_L2 = 1e-2   # the parity bar of the CUDA path's embeddings (tests/test_gpu_vision.py)


def tiny_vision(n_layers=2):
    return WL.VisionShape(n_layers=n_layers, width=16, mlp_dim=24, n_heads=4, patch=7, image=28,
                          channels=3, out_width=8)


def rand_vision_weights(cfg, std=0.3, rng=RNG):
    out = {}
    for k, s in WL.vision_weight_shapes(cfg).items():
        kind = WL._vision_kind(k)
        if kind == "ln_gain":
            out[k] = 1.0 + rng.normal(0, 0.2, size=s)
        else:
            out[k] = rng.normal(0, std if kind == "matrix" else 0.2, size=s)
    return out


def rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def T(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


# ---------------------------------------------------------------------------------------
# patch embedding (V2)

def test_patch_embed_matches_torch_conv2d():
    img = RNG.uniform(-1, 1, size=(3, 42, 42))
    w = RNG.normal(size=(5, 3, 14, 14))
    b = RNG.normal(size=5)
    out = V.patch_embed(img, w, b, 14)
    ref = F.conv2d(T(img)[None], T(w), T(b), stride=14)[0]          # [5][3][3]
    np.testing.assert_allclose(out, ref.flatten(1).T.numpy(), rtol=1e-12, atol=1e-12)


def test_patch_embed_brute_force_loops():
    img = RNG.uniform(-1, 1, size=(3, 28, 28))
    w = RNG.normal(size=(2, 3, 14, 14))
    b = RNG.normal(size=2)
    out = V.patch_embed(img, w, b, 14)
    for py in range(2):
        for px in range(2):
            for o in range(2):
                s = b[o]
                for c in range(3):
                    for ky in range(14):
                        for kx in range(14):
                            s += w[o, c, ky, kx] * img[c, py * 14 + ky, px * 14 + kx]
                assert abs(out[py * 2 + px, o] - s) < 1e-10


def test_patch_embed_raster_token_order_and_constant_image():
    w = RNG.normal(size=(4, 3, 14, 14))
    b = RNG.normal(size=4)
    img = np.zeros((3, 42, 42))
    img[:, 14:28, 28:42] = 1.0                         # patch row 1, column 2 only
    out = V.patch_embed(img, w, b, 14)
    for t in range(9):
        want = b + (w.reshape(4, -1).sum(1) if t == 1 * 3 + 2 else 0.0)
        np.testing.assert_allclose(out[t], want, rtol=1e-12, atol=1e-12)
    out = V.patch_embed(np.full((3, 28, 28), -0.5), w, b, 14)
    np.testing.assert_allclose(out, np.broadcast_to(b - 0.5 * w.reshape(4, -1).sum(1), (4, 4)), atol=1e-12)


# ---------------------------------------------------------------------------------------
# LayerNorm (V4)

def test_layer_norm_matches_torch_and_closed_forms():
    x = RNG.normal(size=(5, 16)) * 3 + 1
    g = RNG.normal(size=16)
    o = RNG.normal(size=16)
    ref = F.layer_norm(T(x), (16,), T(g), T(o), eps=1e-6).numpy()
    np.testing.assert_allclose(V.layer_norm(x, g, o, 1e-6), ref, rtol=1e-12, atol=1e-12)
    # unit gain, zero offset: zero mean and variance var / (var + eps) per row
    n = V.layer_norm(x, np.ones(16), np.zeros(16), 1e-6)
    np.testing.assert_allclose(n.mean(1), 0, atol=1e-12)
    var = x.var(1)
    np.testing.assert_allclose(n.var(1), var / (var + 1e-6), rtol=1e-12)
    # invariant to adding a constant and (eps = 0) to scaling a row; a constant row gives the offset
    np.testing.assert_allclose(V.layer_norm(x + 7.0, g, o, 1e-6), V.layer_norm(x, g, o, 1e-6), atol=1e-9)
    np.testing.assert_allclose(V.layer_norm(x * 5.0, g, o, 0.0), V.layer_norm(x, g, o, 0.0), atol=1e-12)
    np.testing.assert_allclose(V.layer_norm(np.full((2, 16), 4.0), g, o, 1e-6), np.broadcast_to(o, (2, 16)))


# ---------------------------------------------------------------------------------------
# attention and MLP (V3, V6)

def _layer_weights(cfg):
    W = rand_vision_weights(cfg)
    return {k: v for k, v in W.items()}


def test_self_attention_matches_torch_multihead_attention():
    cfg = tiny_vision(1)
    W = _layer_weights(cfg)
    x = RNG.normal(size=(11, cfg.width))
    mha = torch.nn.MultiheadAttention(cfg.width, cfg.n_heads, bias=True, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(T(np.concatenate([W["vis0.wq"], W["vis0.wk"], W["vis0.wv"]])))
        mha.in_proj_bias.copy_(T(np.concatenate([W["vis0.bq"], W["vis0.bk"], W["vis0.bv"]])))
        mha.out_proj.weight.copy_(T(W["vis0.wo"]))
        mha.out_proj.bias.copy_(T(W["vis0.bo"]))
        ref = mha(T(x)[None], T(x)[None], T(x)[None], need_weights=False)[0][0].numpy()
    np.testing.assert_allclose(V.self_attention(x, W, "vis0.", cfg.n_heads), ref, rtol=1e-10, atol=1e-10)


def test_single_token_attention_returns_its_value_projection():
    cfg = tiny_vision(1)
    W = _layer_weights(cfg)
    x = RNG.normal(size=(1, cfg.width))
    want = (x @ W["vis0.wv"].T + W["vis0.bv"]) @ W["vis0.wo"].T + W["vis0.bo"]
    np.testing.assert_allclose(V.self_attention(x, W, "vis0.", cfg.n_heads), want, rtol=1e-12, atol=1e-12)


def test_attention_scale_two_token_closed_form():
    # one head of width 4: q = k = x (identity projections), v one-hot per token; then the
    # weight of key j for query i is softmax_j(x_i . x_j / sqrt(4))
    cfg = WL.VisionShape(n_layers=1, width=4, mlp_dim=4, n_heads=1, patch=1, image=2, channels=1, out_width=4)
    W = {"vis0.wq": np.eye(4), "vis0.bq": np.zeros(4), "vis0.wk": np.eye(4), "vis0.bk": np.zeros(4),
         "vis0.wv": np.eye(4), "vis0.bv": np.zeros(4), "vis0.wo": np.eye(4), "vis0.bo": np.zeros(4)}
    x = np.array([[3.0, 0, 0, 0], [0, 1.0, 0, 0]])
    out = V.self_attention(x, W, "vis0.", cfg.n_heads)
    a = 9.0 / 2.0                   # x0 . x0 / sqrt(4); x0 . x1 = 0
    p00 = math.exp(a) / (math.exp(a) + 1.0)
    np.testing.assert_allclose(out[0], [3.0 * p00, 1.0 - p00, 0, 0], rtol=1e-12)
    b = 1.0 / 2.0
    p11 = math.exp(b) / (math.exp(b) + 1.0)
    np.testing.assert_allclose(out[1], [3.0 * (1 - p11), p11, 0, 0], rtol=1e-12)


def test_mlp_matches_torch():
    cfg = tiny_vision(1)
    W = _layer_weights(cfg)
    x = RNG.normal(size=(6, cfg.width))
    ref = F.linear(F.gelu(F.linear(T(x), T(W["vis0.fc1_w"]), T(W["vis0.fc1_b"])), approximate="tanh"),
                   T(W["vis0.fc2_w"]), T(W["vis0.fc2_b"])).numpy()
    np.testing.assert_allclose(V.mlp(x, W, "vis0."), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------
# the whole tower (V2-V7)

def _torch_encode(W, cfg, img):
    Tw = {k: T(v) for k, v in W.items()}
    Wd = cfg.width
    h = F.conv2d(T(img)[None], Tw["vis.patch_w"], Tw["vis.patch_b"], stride=cfg.patch)[0].flatten(1).T
    h = h + Tw["vis.pos"]
    for l in range(cfg.n_layers):
        p = f"vis{l}."
        mha = torch.nn.MultiheadAttention(Wd, cfg.n_heads, bias=True, batch_first=True, dtype=torch.float64)
        with torch.no_grad():
            mha.in_proj_weight.copy_(torch.cat([Tw[p + "wq"], Tw[p + "wk"], Tw[p + "wv"]]))
            mha.in_proj_bias.copy_(torch.cat([Tw[p + "bq"], Tw[p + "bk"], Tw[p + "bv"]]))
            mha.out_proj.weight.copy_(Tw[p + "wo"])
            mha.out_proj.bias.copy_(Tw[p + "bo"])
            n = F.layer_norm(h, (Wd,), Tw[p + "ln1_w"], Tw[p + "ln1_b"], eps=cfg.ln_eps)
            h = h + mha(n[None], n[None], n[None], need_weights=False)[0][0]
        n = F.layer_norm(h, (Wd,), Tw[p + "ln2_w"], Tw[p + "ln2_b"], eps=cfg.ln_eps)
        h = h + F.linear(F.gelu(F.linear(n, Tw[p + "fc1_w"], Tw[p + "fc1_b"]), approximate="tanh"),
                         Tw[p + "fc2_w"], Tw[p + "fc2_b"])
    n = F.layer_norm(h, (Wd,), Tw["vis.post_w"], Tw["vis.post_b"], eps=cfg.ln_eps)
    return (F.linear(n, Tw["vis.proj_w"], Tw["vis.proj_b"]) * math.sqrt(cfg.out_width)).numpy()


def test_encoder_matches_independent_torch_formulation():
    cfg = tiny_vision(n_layers=3)
    W = rand_vision_weights(cfg)
    img = RNG.uniform(-1, 1, size=(3, 28, 28))
    np.testing.assert_allclose(V.encode_image(img, W, cfg), _torch_encode(W, cfg, img), rtol=1e-9, atol=1e-9)


def test_tokens_are_permutation_equivariant_without_position_embedding():
    cfg = tiny_vision(n_layers=2)
    W = rand_vision_weights(cfg)
    W["vis.pos"] = np.zeros_like(W["vis.pos"])
    img = RNG.uniform(-1, 1, size=(3, 28, 28))
    g, p = 4, 7
    perm = RNG.permutation(g * g)
    blocks = img.reshape(3, g, p, g, p).transpose(1, 3, 0, 2, 4).reshape(g * g, 3, p, p)
    img2 = blocks[perm].reshape(g, g, 3, p, p).transpose(2, 0, 3, 1, 4).reshape(3, 28, 28)
    np.testing.assert_allclose(V.encode_image(img2, W, cfg), V.encode_image(img, W, cfg)[perm], atol=1e-10)
    # with the position embedding the tokens are no longer exchangeable
    W2 = rand_vision_weights(cfg)
    assert rel_l2(V.encode_image(img2, W2, cfg), V.encode_image(img, W2, cfg)[perm]) > 1e-3


def test_zero_residual_branches_make_layers_identities_and_projector_scale():
    cfg = tiny_vision(n_layers=3)
    W = rand_vision_weights(cfg)
    for l in range(cfg.n_layers):
        for n in ("wo", "bo", "fc2_w", "fc2_b"):
            W[f"vis{l}.{n}"] = np.zeros_like(W[f"vis{l}.{n}"])
    img = RNG.uniform(-1, 1, size=(3, 28, 28))
    tr = []
    out = V.encode_image(img, W, cfg, trace=tr)
    assert len(tr) == cfg.n_layers + 1
    for h in tr[1:]:
        np.testing.assert_array_equal(h, tr[0])
    # projector weight 0, bias c: every embedding is c * sqrt(out_width)
    W["vis.proj_w"] = np.zeros_like(W["vis.proj_w"])
    c = RNG.normal(size=cfg.out_width)
    W["vis.proj_b"] = c
    np.testing.assert_allclose(V.encode_image(img, W, cfg), np.broadcast_to(c * math.sqrt(8.0), (16, 8)), rtol=1e-12)


def test_image_prefix_places_views_in_order_and_keeps_other_rows():
    cfg = tiny_vision(n_layers=1)
    W = rand_vision_weights(cfg)
    imgs = RNG.uniform(-1, 1, size=(4, 3, 28, 28))
    fill = RNG.normal(size=(2, 40, cfg.out_width))
    pre = V.image_prefix(imgs, W, cfg, batch=2, views=2, prefix_len=40, fill=fill)
    for b in range(2):
        for v in range(2):
            np.testing.assert_allclose(pre[b, v * 16:(v + 1) * 16], V.encode_image(imgs[b * 2 + v], W, cfg))
        np.testing.assert_array_equal(pre[b, 32:], fill[b, 32:])


def test_vision_shape_is_the_pages_tower():
    s = WL.VisionShape()
    n = sum(int(np.prod(v)) for v in WL.vision_weight_shapes(s).values())
    assert s.n_layers == 27 and s.width == 1152 and s.out_width == 2048
    assert s.tokens == 256 and s.head_dim * s.n_heads == s.width
    assert 0.38e9 < n < 0.43e9          # "SigLIP (400M)"


# ---------------------------------------------------------------------------------------
# the GPU parity bar has bite: plausible mistakes move the embeddings past it

@pytest.fixture(scope="module")
def real_width_case():
    cfg = WL.VisionShape(n_layers=3)
    W = WL.as_f32(WL.vision_weights(cfg, stressed=True))
    img = WL.images(cfg, 1)[0]
    return cfg, W, img, V.encode_image(img, W, cfg)


def _gelu_erf(x):
    return 0.5 * x * (1.0 + np.vectorize(math.erf)(x / math.sqrt(2.0)))


MUTANTS = {
    "no_position_embedding": lambda mp, W: W.__setitem__("vis.pos", np.zeros_like(W["vis.pos"])),
    "patch_rows_columns_swapped": lambda mp, W: W.__setitem__(
        "vis.patch_w", np.ascontiguousarray(np.asarray(W["vis.patch_w"]).transpose(0, 1, 3, 2))),
    "rms_norm_for_layer_norm": lambda mp, W: mp.setattr(
        V, "layer_norm", lambda x, g, o, eps: x / np.sqrt((x ** 2).mean(-1, keepdims=True) + eps) * g + o),
    "scale_one_over_head_dim": lambda mp, W: mp.setattr(
        V, "attention", (lambda f: lambda q, k, v, m, s: f(q, k, v, m, s * s))(V.attention)),
    "no_value_bias": lambda mp, W: [W.__setitem__(f"vis{l}.bv", np.zeros_like(W[f"vis{l}.bv"])) for l in range(3)],
    "post_norm_without_offset": lambda mp, W: W.__setitem__("vis.post_b", np.zeros_like(W["vis.post_b"])),
    "no_sqrt_width_scale": lambda mp, W: W.__setitem__("vis.proj_w", np.asarray(W["vis.proj_w"]) / math.sqrt(2048)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_vision_mutants_fail_the_parity_bar(real_width_case, monkeypatch, name):
    cfg, W, img, ref = real_width_case
    Wm = dict(W)
    MUTANTS[name](monkeypatch, Wm)
    out = V.encode_image(img, Wm, cfg)
    assert rel_l2(out, ref) > EMB_REL_L2, name


def test_gelu_erf_is_below_the_bar_but_caught_by_the_torch_pin():
    # the exact GELU differs from the tanh form by < 1e-3: the end-to-end bar cannot tell
    # them apart, which is why test_mlp_matches_torch pins the tanh form at 1e-12
    x = np.linspace(-4, 4, 101)
    from oracle.model import gelu_tanh
    assert np.abs(_gelu_erf(x) - gelu_tanh(x)).max() < 1e-3
    assert np.abs(_gelu_erf(x) - gelu_tanh(x)).max() > 1e-5


def test_images_recipe_is_uniform_in_range():
    s = WL.VisionShape()
    im = WL.images(s, 2)
    assert im.shape == (2, 3, 224, 224) and im.dtype == np.float32
    assert im.min() >= -1.0 and im.max() < 1.0 and abs(float(im.mean())) < 5e-3
    np.testing.assert_array_equal(im, WL.images(s, 2))
    w = WL.vision_weights(WL.VisionShape(n_layers=1))
    g = gen.bf16_to_f32(w["vis0.ln1_w"])
    assert abs(float(g.mean()) - 1.0) < 0.02 and 0.05 < float(g.std()) < 0.15


def test_golden_regression_of_the_vision_oracle():
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden_vision", os.path.join(here, "make_golden_vision.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    stored = json.load(open(os.path.join(here, "tiny_vision_embeddings.json")))
    expect = np.array([float.fromhex(x) for x in stored["embeddings"]]).reshape(stored["shape"])
    np.testing.assert_allclose(mg.compute(), expect, rtol=1e-12, atol=1e-12)
