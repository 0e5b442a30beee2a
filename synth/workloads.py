"""The five synthetic workloads and their seeded tensors.

Shapes follow the pages' π0.5 description (Realtime-VLA tech blog, "pi0.5 inference flow"
and the per-layer op list): action expert width 1024, MLP 4096, 8 query heads x 256,
1 KV head, AdaRMS dense 1024->3072, action dim 32, 10 Euler steps; Gemma-2B-shaped prefix
pass of width 2048, MLP 16384.  No dataset or trained weights are used anywhere: the
real-robot settings of the paper's Table 1 (empty prompt, chunk 63, 1/2/3 camera views)
are stood in for by these seeded tensors.

Recipe (all seeds derive from synth.gen.BASE_SEED and the tensor's name):
  * weights: bf16 N(0, 0.02^2); biases 0 (``bias_std`` > 0 draws them N(0, bias_std^2));
    the "stressed" variant sets every AdaRMS gate bias to 1.0 so residual updates are O(1).
  * prefix KV cache: bf16 N(0, 1), [L][B][P][256] for K (already rotated) and V.
  * valid prefix lengths: per workload below (3-view: 768 + u_b, u_b uniform in {0..48}).
  * noise: float32 N(0, 1), [B][C][32].
  * prefill embeddings: bf16 N(0, 1) * sqrt(2048), [B][P][2048]; pad mask 1 on valid tokens.
  * image front-end (SigLIP-shaped tower, ``VisionShape``): float32 pixels uniform in [-1, 1),
    [N][3][224][224]; weights as ``vision_weights`` states (matrices and biases N(0, 0.02^2),
    LayerNorm gains near 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

from . import gen


@dataclass(frozen=True)
class ExpertShape:
    n_layers: int = 18
    width: int = 1024
    mlp_dim: int = 4096
    n_q_heads: int = 8
    n_kv_heads: int = 1
    head_dim: int = 256
    action_dim: int = 32
    n_steps: int = 10
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    final_norm: bool = True


@dataclass(frozen=True)
class PrefillShape:
    n_layers: int = 18
    width: int = 2048
    mlp_dim: int = 16384
    n_q_heads: int = 8
    n_kv_heads: int = 1
    head_dim: int = 256
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0


@dataclass(frozen=True)
class Workload:
    name: str
    expert: ExpertShape
    chunk: int
    batch: int
    prefix_cap: int
    valid_lens: tuple
    prefill: PrefillShape | None = None
    description: str = ""


def three_view_valid_lens(batch: int) -> tuple:
    u = gen.randint("3view/valid_len_extra", batch, 0, 48)
    return tuple(int(768 + x) for x in u)


def workload(cfg: int, batch: int | None = None) -> Workload:
    """Workloads 1..5 (tiny, 1-view, 2-view, 3-view, end-to-end 2-view)."""
    if cfg == 1:
        return Workload("tiny L2 P272 Lv268 C10 B1", ExpertShape(n_layers=2), 10, 1, 272, (268,),
                        description="2-layer expert, 272 prefix tokens (last 4 padded), chunk 10")
    if cfg == 2:
        return Workload("1-view L18 P288 Lv280 C50 B1", ExpertShape(), 50, 1, 288, (280,),
                        description="256 image + 32 prompt tokens, last 8 padded, chunk 50")
    if cfg == 3:
        return Workload("2-view L18 P512 Lv512 C63 B1", ExpertShape(), 63, 1, 512, (512,),
                        description="512 image tokens, empty prompt, chunk 63")
    if cfg == 4:
        b = 1 if batch is None else batch
        return Workload(f"3-view L18 P816 C63 B{b}", ExpertShape(), 63, b, 816,
                        three_view_valid_lens(b),
                        description="768 image + 48 prompt tokens, per-sample pad, chunk 63")
    if cfg == 5:
        return Workload("e2e 2-view prefill P544 + L18 C63 B1", ExpertShape(), 63, 1, 544, (544,),
                        prefill=PrefillShape(),
                        description="prefill of 512 image + 32 prompt embeddings, then denoise")
    raise ValueError(cfg)


# ----------------------------------------------------------------------------------------
# tensors

def expert_weight_shapes(s: ExpertShape) -> dict:
    D, F, H, hd, A = s.width, s.mlp_dim, s.n_q_heads, s.head_dim, s.action_dim
    kvd = s.n_kv_heads * hd
    shapes = {
        "action_in_w": (D, A), "action_in_b": (D,),
        "action_out_w": (A, D), "action_out_b": (A,),
        "time_in_w": (D, D), "time_in_b": (D,),
        "time_out_w": (D, D), "time_out_b": (D,),
        "ada_final_w": (3 * D, D), "ada_final_b": (3 * D,),
    }
    for l in range(s.n_layers):
        shapes.update({
            f"l{l}.wq": (H * hd, D), f"l{l}.wk": (kvd, D), f"l{l}.wv": (kvd, D),
            f"l{l}.wo": (D, H * hd),
            f"l{l}.wg": (F, D), f"l{l}.wu": (F, D), f"l{l}.wd": (D, F),
            f"l{l}.ada_attn_w": (3 * D, D), f"l{l}.ada_attn_b": (3 * D,),
            f"l{l}.ada_ffn_w": (3 * D, D), f"l{l}.ada_ffn_b": (3 * D,),
        })
    return shapes


def pi0_expert_weight_shapes(s: ExpertShape) -> dict:
    """The π0 action expert: state projection, action-time MLP, plain RMSNorm weights."""
    D, F, H, hd, A = s.width, s.mlp_dim, s.n_q_heads, s.head_dim, s.action_dim
    kvd = s.n_kv_heads * hd
    shapes = {
        "action_in_w": (D, A), "action_in_b": (D,),
        "action_out_w": (A, D), "action_out_b": (A,),
        "state_w": (D, A), "state_b": (D,),
        "action_time_in_w": (D, 2 * D), "action_time_in_b": (D,),
        "action_time_out_w": (D, D), "action_time_out_b": (D,),
        "final_ln": (D,),
    }
    for l in range(s.n_layers):
        shapes.update({
            f"l{l}.wq": (H * hd, D), f"l{l}.wk": (kvd, D), f"l{l}.wv": (kvd, D),
            f"l{l}.wo": (D, H * hd),
            f"l{l}.wg": (F, D), f"l{l}.wu": (F, D), f"l{l}.wd": (D, F),
            f"l{l}.ln1": (D,), f"l{l}.ln2": (D,),
        })
    return shapes


def pi0_expert_weights(s: ExpertShape, std: float = 0.02, bias_std: float = 0.0,
                       tag: str = "pi0") -> dict:
    """bf16 bit patterns of every π0 expert tensor; RMSNorm weights w (scale 1 + w) N(0, std^2)."""
    out = {}
    for name, shape in pi0_expert_weight_shapes(s).items():
        if _is_bias(name) and bias_std <= 0:
            out[name] = np.zeros(shape, dtype=np.uint16)
        else:
            out[name] = gen.normal_bf16(f"{tag}/{name}", shape, bias_std if _is_bias(name) else std)
    return out


def state(w: Workload, tag: str = "state") -> np.ndarray:
    """π0 robot state, float32 N(0, 1) [B][action_dim]."""
    return gen.normal(f"{tag}/{w.batch}", (w.batch, w.expert.action_dim), 1.0)


def prefill_weight_shapes(s: PrefillShape) -> dict:
    D, F, H, hd = s.width, s.mlp_dim, s.n_q_heads, s.head_dim
    kvd = s.n_kv_heads * hd
    shapes = {}
    for l in range(s.n_layers):
        shapes.update({
            f"pf{l}.ln1": (D,), f"pf{l}.wq": (H * hd, D), f"pf{l}.wk": (kvd, D),
            f"pf{l}.wv": (kvd, D), f"pf{l}.wo": (D, H * hd), f"pf{l}.ln2": (D,),
            f"pf{l}.wg": (F, D), f"pf{l}.wu": (F, D), f"pf{l}.wd": (D, F),
        })
    return shapes


def _is_bias(name: str) -> bool:
    return name.endswith("_b")


def expert_weights(s: ExpertShape, std: float = 0.02, bias_std: float = 0.0,
                   stressed: bool = False, tag: str = "expert") -> dict:
    """bf16 bit patterns (uint16) for every expert tensor, in (out, in) Linear layout."""
    out = {}
    D = s.width
    for name, shape in expert_weight_shapes(s).items():
        if _is_bias(name):
            if bias_std > 0:
                out[name] = gen.normal_bf16(f"{tag}/{name}", shape, bias_std)
            else:
                out[name] = np.zeros(shape, dtype=np.uint16)
            if stressed and "ada_" in name:
                b = gen.bf16_to_f32(out[name]).copy()
                b[2 * D:3 * D] = 1.0
                out[name] = gen.bf16_bits(b)
        else:
            out[name] = gen.normal_bf16(f"{tag}/{name}", shape, std)
    return out


def prefill_weights(s: PrefillShape, std: float = 0.02, tag: str = "prefill") -> dict:
    return {name: gen.normal_bf16(f"{tag}/{name}", shape, std)
            for name, shape in prefill_weight_shapes(s).items()}


def kv_cache(w: Workload, tag: str = "kv", pad_fill: float | None = None):
    """(K bits, V bits, valid_len) with K/V bf16 [L][B][P][hd]; pad_fill overwrites slots >= Lv."""
    s = w.expert
    shape = (s.n_layers, w.batch, w.prefix_cap, s.n_kv_heads * s.head_dim)
    k = gen.normal_bf16(f"{tag}/{w.prefix_cap}/k", shape, 1.0)
    v = gen.normal_bf16(f"{tag}/{w.prefix_cap}/v", shape, 1.0)
    valid = np.asarray(w.valid_lens, dtype=np.int32)
    if pad_fill is not None:
        fill = gen.bf16_bits(np.full(1, pad_fill, np.float32))[0]
        for b, lv in enumerate(valid):
            k[:, b, lv:] = fill
            v[:, b, lv:] = fill
    return k, v, valid


def noise(w: Workload, tag: str = "noise") -> np.ndarray:
    s = w.expert
    return gen.normal(f"{tag}/{w.chunk}", (w.batch, w.chunk, s.action_dim), 1.0)


def prefill_inputs(w: Workload, tag: str = "embeds"):
    """(embeds bf16 bits [B][P][2048], pad mask uint8 [B][P])."""
    p = w.prefill
    emb = gen.normal_bf16(f"{tag}/{w.prefix_cap}", (w.batch, w.prefix_cap, p.width),
                          math.sqrt(p.width))
    mask = np.zeros((w.batch, w.prefix_cap), dtype=np.uint8)
    for b, lv in enumerate(w.valid_lens):
        mask[b, :lv] = 1
    return emb, mask


def as_f32(bits_dict: dict) -> dict:
    return {k: gen.bf16_to_f32(v) for k, v in bits_dict.items()}


# ----------------------------------------------------------------------------------------
# image front-end: SigLIP vision tower + multi_modal_projector

@dataclass(frozen=True)
class VisionShape:
    """SigLIP-So400m/14-shaped tower.  The pages give 400M parameters, 27 layers, width 1152,
    224 x 224 images -> 256 tokens and the 1152 -> 2048 projector; patch 14, 16 heads x 72 and
    MLP 4304 are the public So400m/14 values (they give 412M parameters)."""
    n_layers: int = 27
    width: int = 1152
    mlp_dim: int = 4304
    n_heads: int = 16
    patch: int = 14
    image: int = 224
    channels: int = 3
    out_width: int = 2048
    ln_eps: float = 1e-6

    @property
    def head_dim(self) -> int:
        return self.width // self.n_heads

    @property
    def tokens(self) -> int:
        return (self.image // self.patch) ** 2


def vision_weight_shapes(s: VisionShape) -> dict:
    W, Fv, p, c = s.width, s.mlp_dim, s.patch, s.channels
    shapes = {"vis.patch_w": (W, c, p, p), "vis.patch_b": (W,), "vis.pos": (s.tokens, W),
              "vis.post_w": (W,), "vis.post_b": (W,),
              "vis.proj_w": (s.out_width, W), "vis.proj_b": (s.out_width,)}
    for l in range(s.n_layers):
        shapes.update({
            f"vis{l}.ln1_w": (W,), f"vis{l}.ln1_b": (W,),
            f"vis{l}.wq": (W, W), f"vis{l}.bq": (W,), f"vis{l}.wk": (W, W), f"vis{l}.bk": (W,),
            f"vis{l}.wv": (W, W), f"vis{l}.bv": (W,), f"vis{l}.wo": (W, W), f"vis{l}.bo": (W,),
            f"vis{l}.ln2_w": (W,), f"vis{l}.ln2_b": (W,),
            f"vis{l}.fc1_w": (Fv, W), f"vis{l}.fc1_b": (Fv,), f"vis{l}.fc2_w": (W, Fv), f"vis{l}.fc2_b": (W,),
        })
    return shapes


def _vision_kind(name: str) -> str:
    leaf = name.split(".", 1)[1]
    if leaf in ("ln1_w", "ln2_w", "post_w"):
        return "ln_gain"
    if leaf in ("ln1_b", "ln2_b", "post_b"):
        return "ln_bias"
    if leaf == "pos":
        return "pos"
    if leaf in ("patch_b", "bq", "bk", "bv", "bo", "fc1_b", "fc2_b", "proj_b"):
        return "bias"
    return "matrix"


def vision_weights(s: VisionShape, std: float = 0.02, stressed: bool = False, tag: str = "vision") -> dict:
    """bf16 bit patterns of every vision tensor.

    Matrices N(0, std^2) ("stressed": W_q and W_k at 3 std, so attention is peaked rather
    than near-uniform); biases N(0, std^2); position embedding N(0, 0.1^2); LayerNorm
    gains 1 + N(0, 0.1^2) and offsets N(0, 0.05^2), so every affine term is exercised.
    """
    out = {}
    for name, shape in vision_weight_shapes(s).items():
        kind = _vision_kind(name)
        key = f"{tag}/{name}"
        if kind == "ln_gain":
            out[name] = gen.bf16_bits(1.0 + gen.normal(key, shape, 0.1))
        elif kind == "ln_bias":
            out[name] = gen.normal_bf16(key, shape, 0.05)
        elif kind == "pos":
            out[name] = gen.normal_bf16(key, shape, 0.1)
        elif kind == "bias":
            out[name] = gen.normal_bf16(key, shape, std)
        else:
            scale = 3.0 if stressed and name.split(".", 1)[1] in ("wq", "wk") else 1.0
            out[name] = gen.normal_bf16(key, shape, std * scale)
    return out


def images(s: VisionShape, n: int, tag: str = "images") -> np.ndarray:
    """float32 pixels uniform in [-1, 1), [n][channels][image][image]: the camera frames after
    the resize and the [-1, 1] normalisation, which are not part of the path."""
    shape = (n, s.channels, s.image, s.image)
    u = gen.uniform(f"{tag}/{n}", int(np.prod(shape)))
    return (2.0 * u - 1.0).astype(np.float32).reshape(shape)


__all__ = ["ExpertShape", "PrefillShape", "Workload", "workload", "expert_weights",
           "pi0_expert_weight_shapes", "pi0_expert_weights", "state",
           "prefill_weights", "kv_cache", "noise", "prefill_inputs", "as_f32",
           "expert_weight_shapes", "prefill_weight_shapes", "replace", "field",
           "VisionShape", "vision_weight_shapes", "vision_weights", "images"]
