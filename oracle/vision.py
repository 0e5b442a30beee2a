"""Plain, slow, fp64 CPU oracle of the image front-end: the SigLIP vision tower and the
multi_modal_projector that turn each camera view into 256 prefix embeddings.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it.  It shares
no code with the CUDA library; weights arrive as the bf16 values the library receives,
upcast to float64.

Sources (cited by page title and section):
  [BLOG]  Realtime-VLA tech blog (blog.w4k4.me), "pi0.5 inference flow": the model
          structure (SigLIP, 400M parameters, 224 x 224 image -> 256 tokens), encoder step 1
          (each view encoded to 256 token embeddings, scaled by sqrt(2048)) and step 3 (image
          tokens, then language tokens, form the prefix); the class hierarchy
          (vision_tower: SiglipVisionTransformer with 27 layers; multi_modal_projector:
          Linear 1152 -> 2048); "Kernel-level optimisation (§4)", Partial Split-k (the
          512 x 1152 x 1152 GEMM: two views of 256 tokens at width 1152).

The pages name the tower but do not spell out its layer.  Readings (each is also listed in
the design notes):
  V1 shape: patch 14 (224 / 14 = 16, 16^2 = 256 tokens), 16 heads x 72, MLP 4304: the public
     SigLIP-So400m/14 configuration, which gives the pages' 27 layers, width 1152 and ~400M
     parameters.
  V2 patch embedding: a convolution 3 -> 1152 with a 14 x 14 kernel, stride 14 and a bias
     over the image as [channel][row][column]; tokens in raster order of the 16 x 16 patch
     grid; then a learned position embedding [256][1152] is added.
  V3 encoder layer (pre-norm): h += o_proj(MHA(LN1(h))); h += fc2(GELU(fc1(LN2(h)))); the
     q, k, v, o, fc1 and fc2 linears carry biases; attention is bidirectional over the 256
     tokens of one image: no mask, no rotary embedding, scale 1/sqrt(72).
  V4 LayerNorm: (x - mean) / sqrt(var + eps) * gain + offset, biased variance, eps 1e-6.
  V5 after the last layer a post-LayerNorm, then the projector Linear(1152 -> 2048) with
     bias, then * sqrt(2048).  The blog's "pooler_output * sqrt(2048)" is read as the
     per-token projector output: the step yields 256 embeddings per view, and the
     end-to-end workload's embeddings are N(0, 1) * sqrt(2048) in scale.
  V6 GELU is the tanh approximation (as R10 of oracle/model.py).
  V7 views are encoded independently (no attention across images); view v of sample b
     fills prefix rows v*256 .. v*256 + 255, views in order, before the prompt tokens.
  V8 pixels are the camera frame after resize and [-1, 1] normalisation (the resize kernel
     of the blog's I/O section is off the GPU path here).
"""
from __future__ import annotations

import numpy as np

from .model import attention, gelu_tanh

F64 = np.float64


def _w(W, name):
    return np.asarray(W[name], dtype=F64)


def patch_embed(img, w, b, patch: int):
    """V2: the stride-`patch` convolution as a sum over each non-overlapping patch.

    img [C][H][H]; w [Wd][C][patch][patch]; b [Wd].  Token t = py * g + px (g = H / patch)
    is b + sum_{c, ky, kx} w[:, c, ky, kx] * img[c, py*patch + ky, px*patch + kx].
    """
    img = np.asarray(img, dtype=F64)
    C, H, _ = img.shape
    g = H // patch
    # blocks[py, px, c, ky, kx] = img[c, py*patch + ky, px*patch + kx]
    blocks = img.reshape(C, g, patch, g, patch).transpose(1, 3, 0, 2, 4).reshape(g * g, C * patch * patch)
    return blocks @ np.asarray(w, dtype=F64).reshape(w.shape[0], -1).T + np.asarray(b, dtype=F64)


def layer_norm(x, gain, offset, eps):
    """V4: per row, (x - mean) / sqrt(mean((x - mean)^2) + eps) * gain + offset."""
    x = np.asarray(x, dtype=F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gain, dtype=F64) + np.asarray(offset, dtype=F64)


def self_attention(x, W, p: str, n_heads: int):
    """V3: multi-head self-attention of one image's tokens x [T][Wd], with biases, no mask."""
    T, Wd = x.shape
    hd = Wd // n_heads
    q = (x @ _w(W, p + "wq").T + _w(W, p + "bq")).reshape(T, n_heads, hd).transpose(1, 0, 2)
    k = (x @ _w(W, p + "wk").T + _w(W, p + "bk")).reshape(T, n_heads, hd).transpose(1, 0, 2)
    v = (x @ _w(W, p + "wv").T + _w(W, p + "bv")).reshape(T, n_heads, hd).transpose(1, 0, 2)
    every = np.ones((T, T), dtype=bool)
    o = attention(q, k, v, every, hd ** -0.5)                      # [heads][T][hd]
    return o.transpose(1, 0, 2).reshape(T, Wd) @ _w(W, p + "wo").T + _w(W, p + "bo")


def mlp(x, W, p: str):
    """V3, V6: fc2(GELU_tanh(fc1(x)))."""
    return gelu_tanh(x @ _w(W, p + "fc1_w").T + _w(W, p + "fc1_b")) @ _w(W, p + "fc2_w").T + _w(W, p + "fc2_b")


def encoder_layer(h, W, l: int, cfg):
    """V3: one pre-norm SigLIP encoder layer on one image's tokens."""
    p = f"vis{l}."
    h = h + self_attention(layer_norm(h, _w(W, p + "ln1_w"), _w(W, p + "ln1_b"), cfg.ln_eps), W, p, cfg.n_heads)
    return h + mlp(layer_norm(h, _w(W, p + "ln2_w"), _w(W, p + "ln2_b"), cfg.ln_eps), W, p)


def encode_image(img, W, cfg, trace=None):
    """One view -> [256][out_width] prefix embeddings (V2-V5).

    trace, when a list, receives the residual stream after the embedding and after each
    layer ([T][width] each).
    """
    h = patch_embed(img, _w(W, "vis.patch_w"), _w(W, "vis.patch_b"), cfg.patch) + _w(W, "vis.pos")
    if trace is not None:
        trace.append(h.copy())
    for l in range(cfg.n_layers):
        h = encoder_layer(h, W, l, cfg)
        if trace is not None:
            trace.append(h.copy())
    n = layer_norm(h, _w(W, "vis.post_w"), _w(W, "vis.post_b"), cfg.ln_eps)
    return (n @ _w(W, "vis.proj_w").T + _w(W, "vis.proj_b")) * np.sqrt(F64(cfg.out_width))


def encode_images(images, W, cfg):
    """[N][C][H][H] -> [N][256][out_width], each image on its own (V7)."""
    return np.stack([encode_image(im, W, cfg) for im in images])


def image_prefix(images, W, cfg, batch: int, views: int, prefix_len: int, fill=None):
    """The prefix embedding tensor [batch][prefix_len][out_width] of V7: image b*views + v
    at rows v*T .. v*T + T - 1 of sample b; other rows from `fill` (default 0)."""
    T = cfg.tokens
    out = np.zeros((batch, prefix_len, cfg.out_width), dtype=F64) if fill is None else np.array(fill, dtype=F64)
    emb = encode_images(images, W, cfg)
    for b in range(batch):
        for v in range(views):
            out[b, v * T:(v + 1) * T] = emb[b * views + v]
    return out
