"""The image front-end (SigLIP-shaped tower + multi_modal_projector) through the C ABI against
the fp64 oracle (oracle/vision.py):

  * the full 27-layer tower on 2 views: the residual stream after the embedding and after
    every layer, every layer's update, and the prefix embeddings, on the graph path and on
    the trace path;
  * peaked attention (the stressed weights, W_q and W_k at 3x) on a 4-layer tower;
  * the graph path's row placement for batch x views with the prompt rows left untouched,
    and image counts of 1 and 3 (one and three 256-token tiles);
  * argument errors, checked mode (guard bands around every buffer), the memory cap;
  * images -> rtvla_prefill -> rtvla_sample_actions end to end against the oracle chain.
"""

import numpy as np
import pytest
import torch

import flow_matching_action_expert_b200 as R
from oracle import model as O
from oracle import vision as V
from synth import gen
from synth import workloads as WL

from harness import GpuModel, assert_actions_close, bf16_dev, rel_l2

pytestmark = pytest.mark.gpu

# Plain weights (attention logits of std ~0.5): the hidden-state bar of the contract, relative
# L2 1e-2, for every residual stream, every layer's update and the embeddings; the largest
# |error| within 3% of the largest |embedding| (the output itself is bf16, 0.4% per value).
# Every planted mistake of the oracle's pins moves the 27-layer embeddings by >= 4.7e-2.
EMB_REL_L2 = 1e-2
EMB_MAX_FRAC = 3e-2
# Peaked attention (logits of std ~4): the GEMMs' bf16 operands (LayerNorm output, and Q and K
# themselves) perturb each logit by ~0.3% of its size, which a peaked softmax passes on to the
# attention output: the GPU's rounding points emulated in numpy give 1.5e-2 after 4 layers.
# 3e-2 keeps every planted mistake (>= 4.8e-2 on this tower) outside.
PEAKED_REL_L2 = 3e-2


class GpuVision:
    """One rtvla_vision context built from seeded bf16 weights."""

    def __init__(self, cfg: WL.VisionShape, bits: dict, max_images: int):
        dev = {k: bf16_dev(v) for k, v in bits.items()}
        self.shape = cfg
        self.cfg = R.make_vision_config(n_layers=cfg.n_layers, max_images=max_images, ln_eps=cfg.ln_eps)
        self.ctx = R.rtvla_vision_create(dev, self.cfg)
        del dev
        torch.cuda.synchronize()

    def close(self):
        if self.ctx:
            R.rtvla_vision_destroy(self.ctx)
            self.ctx = 0

    def encode(self, images: np.ndarray, batch: int, views: int, prefix_len: int, fill: torch.Tensor | None = None):
        x = torch.from_numpy(np.ascontiguousarray(images, dtype=np.float32)).cuda()
        out = fill.clone() if fill is not None else torch.zeros((batch, prefix_len, 2048), dtype=torch.bfloat16,
                                                                device="cuda")
        R.rtvla_encode_images(self.ctx, x, batch, views, out, prefix_len)
        st = R.rtvla_vision_sync_status(self.ctx)
        assert st == 0, R.STATUS[st]
        return out

    def trace(self, images: np.ndarray):
        n = images.shape[0]
        x = torch.from_numpy(np.ascontiguousarray(images, dtype=np.float32)).cuda()
        h = torch.empty((self.cfg.n_layers + 1, n * 256, 1152), dtype=torch.float32, device="cuda")
        out = torch.empty((1, n * 256, 2048), dtype=torch.bfloat16, device="cuda")
        R.rtvla_vision_debug_trace(self.ctx, x, n, h, out)
        st = R.rtvla_vision_sync_status(self.ctx)
        assert st == 0, R.STATUS[st]
        return h.cpu().numpy().reshape(self.cfg.n_layers + 1, n, 256, 1152), out.float().cpu().numpy()


def oracle_with_trace(images, W, cfg):
    embs, trs = [], []
    for im in images:
        tr = []
        embs.append(V.encode_image(im, W, cfg, trace=tr))
        trs.append(np.stack(tr))
    return np.stack(embs), np.stack(trs, axis=1)          # [n][256][2048], [L+1][n][256][1152]


def assert_embeddings_close(gpu, ref, tol, what):
    r = rel_l2(gpu, ref)
    frac = float(np.abs(gpu - ref).max() / np.abs(ref).max())
    assert np.isfinite(gpu).all(), f"{what}: non-finite embeddings"
    assert r <= tol and frac <= EMB_MAX_FRAC, f"{what}: rel-L2 {r:.3e}, max-abs / max {frac:.3e}"


def assert_stream_close(gpu_tr, ref_tr, tol, what):
    worst = []
    for i in range(ref_tr.shape[0]):
        r = rel_l2(gpu_tr[i], ref_tr[i])
        u = rel_l2(gpu_tr[i] - gpu_tr[i - 1], ref_tr[i] - ref_tr[i - 1]) if i else 0.0
        worst.append((i, r, u))
        assert r <= tol, f"{what}: residual stream {i} rel-L2 {r:.3e} ({worst})"
        assert u <= tol, f"{what}: layer {i - 1} update rel-L2 {u:.3e} ({worst})"


@pytest.fixture(scope="module")
def full_tower():
    cfg = WL.VisionShape()
    bits = WL.vision_weights(cfg)
    imgs = WL.images(cfg, 2)
    ref, ref_tr = oracle_with_trace(imgs, WL.as_f32(bits), cfg)
    g = GpuVision(cfg, bits, max_images=4)
    yield cfg, g, imgs, ref, ref_tr
    g.close()


def test_full_tower_two_views_per_layer_and_embeddings(full_tower):
    cfg, g, imgs, ref, ref_tr = full_tower
    tr, emb = g.trace(imgs)
    assert_stream_close(tr, ref_tr, EMB_REL_L2, "27-layer tower, trace path")
    assert_embeddings_close(emb.reshape(2, 256, 2048), ref, EMB_REL_L2, "27-layer tower, trace path")
    # the graph path: one sample of two views into a 512-row prefix
    out = g.encode(imgs, 1, 2, 512).float().cpu().numpy()
    assert_embeddings_close(out.reshape(2, 256, 2048), ref, EMB_REL_L2, "27-layer tower, graph path")
    assert R.rtvla_vision_kernels_per_call(g.ctx, 2) == 8 * cfg.n_layers + 5
    assert R.rtvla_vision_kernels_per_call(g.ctx, 3) == -1


def test_peaked_attention_four_layers():
    cfg = WL.VisionShape(n_layers=4)
    bits = WL.vision_weights(cfg, stressed=True)
    imgs = WL.images(cfg, 2, tag="images-peaked")
    ref, ref_tr = oracle_with_trace(imgs, WL.as_f32(bits), cfg)
    g = GpuVision(cfg, bits, max_images=2)
    try:
        tr, emb = g.trace(imgs)
        assert_stream_close(tr, ref_tr, PEAKED_REL_L2, "peaked attention")
        assert_embeddings_close(emb.reshape(2, 256, 2048), ref, PEAKED_REL_L2, "peaked attention")
    finally:
        g.close()


@pytest.fixture(scope="module")
def small_tower():
    cfg = WL.VisionShape(n_layers=2)
    bits = WL.vision_weights(cfg, tag="vision-small")
    g = GpuVision(cfg, bits, max_images=4)
    yield cfg, bits, g
    g.close()


@pytest.mark.parametrize("batch, views", [(1, 1), (3, 1), (2, 2)])
def test_graph_path_rows_and_prompt_rows_untouched(small_tower, batch, views):
    cfg, bits, g = small_tower
    n = batch * views
    imgs = WL.images(cfg, n, tag=f"images-{batch}x{views}")
    P = views * 256 + 32
    fill_bits = gen.normal_bf16(f"prompt/{batch}x{views}", (batch, P, 2048), 45.0)
    fill = bf16_dev(fill_bits)
    out = g.encode(imgs, batch, views, P, fill=fill)
    ref = V.encode_images(imgs, WL.as_f32(bits), cfg)
    got = out.float().cpu().numpy()
    raw = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for b in range(batch):
        for v in range(views):
            assert_embeddings_close(got[b, v * 256:(v + 1) * 256], ref[b * views + v], EMB_REL_L2,
                                    f"{batch}x{views} image ({b}, {v})")
        np.testing.assert_array_equal(raw[b, views * 256:], fill_bits[b, views * 256:])
    assert R.rtvla_vision_kernels_per_call(g.ctx, n) == 8 * cfg.n_layers + 5


def test_argument_errors_are_returned_before_any_launch(small_tower):
    cfg, bits, g = small_tower
    imgs = torch.zeros((4, 3, 224, 224), dtype=torch.float32, device="cuda")
    out = torch.zeros((2, 600, 2048), dtype=torch.bfloat16, device="cuda")

    def code(**kw):
        a = dict(images=imgs.data_ptr(), batch=1, views=1, out=out.data_ptr(), prefix_len=600)
        a.update(kw)
        return R.library().rtvla_encode_images(g.ctx, a["images"], a["batch"], a["views"], a["out"],
                                               a["prefix_len"], None)

    assert code() == 0
    assert R.STATUS[code(batch=5)] == "RTVLA_ERR_SHAPE"              # 5 images > max_images 4
    assert R.STATUS[code(batch=1, views=3, prefix_len=700)] == "RTVLA_ERR_SHAPE"  # 768 rows > 700
    assert R.STATUS[code(views=0)] == "RTVLA_ERR_INVALID_ARG"
    assert R.STATUS[code(images=0)] == "RTVLA_ERR_INVALID_ARG"
    assert R.STATUS[code(images=imgs.data_ptr() + 2)] == "RTVLA_ERR_INVALID_ARG"
    assert R.STATUS[code(out=out.data_ptr() + 8)] == "RTVLA_ERR_INVALID_ARG"
    assert R.rtvla_vision_sync_status(g.ctx) == 0


def test_checked_mode_and_memory_cap(monkeypatch):
    cfg = WL.VisionShape(n_layers=1)
    bits = WL.vision_weights(cfg, tag="vision-checked")
    monkeypatch.setenv("RTVLA_CHECKED", "1")
    g = GpuVision(cfg, bits, max_images=3)
    try:
        imgs = WL.images(cfg, 3, tag="images-checked")
        out = g.encode(imgs, 3, 1, 256)              # sync_status checks every guard band
        ref = V.encode_images(imgs, WL.as_f32(bits), cfg)
        assert_embeddings_close(out.float().cpu().numpy(), ref, EMB_REL_L2, "checked mode")
    finally:
        g.close()
    monkeypatch.delenv("RTVLA_CHECKED")
    monkeypatch.setenv("RTVLA_DEVICE_MEMORY_CAP", str(16 << 20))   # the K = 1152 weight stack alone is 25 MB
    dev = {k: bf16_dev(v) for k, v in bits.items()}
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_vision_create(dev, R.make_vision_config(n_layers=1, max_images=3))
    assert e.value.name == "RTVLA_ERR_OOM"


def test_images_to_actions_end_to_end():
    """Two views -> 512 image embeddings + 32 prompt embeddings -> the Gemma-2B-shaped prefix
    pass -> the π0.5 denoise loop (2-layer expert and prefix pass), against the oracle chain."""
    vcfg = WL.VisionShape(n_layers=2)
    vbits = WL.vision_weights(vcfg, tag="vision-e2e")
    imgs = WL.images(vcfg, 2, tag="images-e2e")
    wl = WL.Workload("images e2e", WL.ExpertShape(n_layers=2), 10, 1, 544, (544,),
                     prefill=WL.PrefillShape(n_layers=2))
    ebits = WL.expert_weights(wl.expert, stressed=True)
    pbits = WL.prefill_weights(wl.prefill)
    prompt_bits, mask = WL.prefill_inputs(wl, tag="prompt-e2e")
    noise = WL.noise(wl)

    gv = GpuVision(vcfg, vbits, max_images=2)
    m = GpuModel(wl, ebits, prefill_bits=pbits)
    try:
        emb = gv.encode(imgs, 1, 2, 544, fill=bf16_dev(prompt_bits))
        k = torch.zeros((2, 1, 544, 256), dtype=torch.bfloat16, device="cuda")
        v = torch.zeros_like(k)
        valid = torch.zeros(1, dtype=torch.int32, device="cuda")
        R.rtvla_prefill(m.ctx, emb, torch.from_numpy(mask).cuda(), 1, 544, R.make_kv(k, v, valid, 1, 544))
        out = m.sample(noise, k, v, valid)
    finally:
        gv.close()
        m.close()
    pre = V.image_prefix(imgs, WL.as_f32(vbits), vcfg, 1, 2, 544, fill=gen.bf16_to_f32(prompt_bits))
    K, Vv, lv = O.prefill(WL.as_f32(pbits), wl.prefill, pre, mask)
    ref = O.sample_actions(WL.as_f32(ebits), wl.expert, noise, K, Vv, lv)
    assert_actions_close(out, ref, "images -> prefill -> denoise")
