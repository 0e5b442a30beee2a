"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against a closed form, an invariant, brute force on a tiny
input, or an independent formulation built from library routines (torch fp64), chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails one of them.
Sources are the Realtime-VLA tech blog ("pi0.5 inference flow", "Per-layer processing",
"Precompute") and the readings R1-R12 listed in oracle/model.py.
"""
import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import model as M
from synth import gen
from synth import workloads as WL

RNG = np.random.default_rng(1234)


def tiny_expert(n_layers=2, final_norm=True):
    return SimpleNamespace(n_layers=n_layers, width=16, mlp_dim=32, n_q_heads=2, n_kv_heads=1,
                           head_dim=8, action_dim=4, n_steps=10, rms_eps=1e-6,
                           rope_theta=10000.0, final_norm=final_norm)


def tiny_prefill(n_layers=2):
    return SimpleNamespace(n_layers=n_layers, width=16, mlp_dim=32, n_q_heads=2, n_kv_heads=1,
                           head_dim=8, rms_eps=1e-6, rope_theta=10000.0)


def rand_expert_weights(cfg, std=0.3, bias_std=0.1, rng=RNG):
    shapes = WL.expert_weight_shapes(cfg)
    return {k: rng.normal(0, bias_std if k.endswith("_b") else std, size=s) for k, s in shapes.items()}


def rand_prefill_weights(cfg, std=0.3, rng=RNG):
    shapes = WL.prefill_weight_shapes(cfg)
    return {k: rng.normal(0, std, size=s) for k, s in shapes.items()}


def rel_l2(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(np.asarray(b)))


# ---------------------------------------------------------------------------------------
# attention

def test_attention_bruteforce_scalar_loop():
    H, Hkv, Tq, Tk, hd = 4, 2, 3, 7, 5
    q = RNG.normal(size=(H, Tq, hd))
    k = RNG.normal(size=(Hkv, Tk, hd))
    v = RNG.normal(size=(Hkv, Tk, hd))
    mask = RNG.random((Tq, Tk)) < 0.6
    mask[:, 0] = True
    out = M.attention(q, k, v, mask, 0.37)
    ref = np.zeros_like(out)
    for h in range(H):
        g = h // (H // Hkv)                       # head h reads KV group h // (H / Hkv)
        for i in range(Tq):
            logits = [sum(q[h, i, d] * k[g, j, d] for d in range(hd)) * 0.37 if mask[i, j] else None
                      for j in range(Tk)]
            mx = max(x for x in logits if x is not None)
            w = [math.exp(x - mx) if x is not None else 0.0 for x in logits]
            z = sum(w)
            for d in range(hd):
                ref[h, i, d] = sum(w[j] * v[g, j, d] for j in range(Tk)) / z
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_identical_keys_give_mean_of_visible_values():
    H, Tq, Tk, hd = 2, 3, 6, 4
    q = RNG.normal(size=(H, Tq, hd))
    k = np.broadcast_to(RNG.normal(size=(1, 1, hd)), (1, Tk, hd)).copy()
    v = RNG.normal(size=(1, Tk, hd))
    mask = np.zeros((Tq, Tk), bool)
    mask[:, [0, 2, 5]] = True
    out = M.attention(q, k, v, mask, 0.5)
    expect = v[0, [0, 2, 5]].mean(axis=0)
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=1e-12, atol=1e-13)


def test_attention_dominant_key_selects_its_value():
    q = np.zeros((1, 1, 4))
    q[0, 0, 0] = 1.0
    k = np.zeros((1, 3, 4))
    k[0, 1, 0] = 2000.0
    v = RNG.normal(size=(1, 3, 4))
    out = M.attention(q, k, v, np.ones((1, 3), bool), 1.0)
    np.testing.assert_allclose(out[0, 0], v[0, 1], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# RoPE

def test_rope_is_complex_rotation_of_half_pairs():
    hd, T, theta = 16, 5, 10000.0
    x = RNG.normal(size=(3, T, hd))
    pos = np.array([0, 1, 7, 42, 511])
    out = M.rope(x, pos, theta)
    half = hd // 2
    freq = np.array([theta ** (-2.0 * i / hd) for i in range(half)])
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * pos[:, None] * freq[None, :])
    np.testing.assert_allclose(out[..., :half], z.real, atol=1e-12)
    np.testing.assert_allclose(out[..., half:], z.imag, atol=1e-12)


def test_rope_norm_identity_and_relative_position():
    hd = 256
    q = RNG.normal(size=(1, 1, hd))
    k = RNG.normal(size=(1, 1, hd))
    np.testing.assert_allclose(M.rope(q, [0], 1e4), q, atol=0)
    for p in (1, 300, 811):
        np.testing.assert_allclose(np.linalg.norm(M.rope(q, [p], 1e4)), np.linalg.norm(q), rtol=1e-13)
    dots = [float((M.rope(q, [m], 1e4) * M.rope(k, [n], 1e4)).sum()) for m, n in ((9, 4), (105, 100), (605, 600))]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)
    other = float((M.rope(q, [9], 1e4) * M.rope(k, [5], 1e4)).sum())
    assert abs(other - dots[0]) > 1e-3


# ---------------------------------------------------------------------------------------
# norms and activations

def test_rms_normalize_unit_rms_and_scale_invariance():
    x = RNG.normal(size=(5, 1024)) * 3.0
    y = M.rms_normalize(x, 1e-6)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-6)
    np.testing.assert_allclose(M.rms_normalize(7.5 * x, 1e-6), y, rtol=1e-6)
    z = M.rms_normalize(x, 0.0)
    ref = F.rms_norm(torch.from_numpy(x), (1024,), eps=0.0).numpy()
    np.testing.assert_allclose(z, ref, rtol=1e-12)


def test_ada_rms_norm_split_order_scale_shift_gate():
    D = 8
    x = RNG.normal(size=(3, D))
    cond = RNG.normal(size=(D,))
    w = np.zeros((3 * D, D))
    b = np.concatenate([np.full(D, -1.0), np.arange(D, dtype=float), np.full(D, 0.25)])
    out, gate = M.ada_rms_norm(x, cond, w, b, 1e-6)
    np.testing.assert_allclose(out, np.broadcast_to(np.arange(D, dtype=float), (3, D)), atol=0)
    np.testing.assert_allclose(gate, 0.25)
    b2 = np.concatenate([np.full(D, 1.0), np.zeros(D), np.zeros(D)])
    out2, _ = M.ada_rms_norm(x, cond, w, b2, 1e-6)
    np.testing.assert_allclose(out2, 2.0 * M.rms_normalize(x, 1e-6), rtol=1e-14)


def test_activations_match_torch():
    x = np.linspace(-12, 12, 2001)
    np.testing.assert_allclose(M.gelu_tanh(x), F.gelu(torch.from_numpy(x), approximate="tanh").numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(M.silu(x), F.silu(torch.from_numpy(x)).numpy(), rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------------------
# time embedding and time MLP

def test_time_embedding_closed_forms():
    e0 = M.sinusoidal_time_embedding(0.0, 1024)
    np.testing.assert_array_equal(e0[:512], 0.0)
    np.testing.assert_array_equal(e0[512:], 1.0)
    for t in (0.1, 0.5, 1.0):
        e = M.sinusoidal_time_embedding(t, 1024)
        np.testing.assert_allclose(e[:512] ** 2 + e[512:] ** 2, 1.0, rtol=1e-14)
    t = 1e-7
    e = M.sinusoidal_time_embedding(t, 1024)
    omega = np.arcsin(e[:512]) / t                      # = 2 pi / period_i for tiny t
    period = 2 * np.pi / omega
    np.testing.assert_allclose(period[0], 4e-3, rtol=1e-6)
    np.testing.assert_allclose(period[-1], 4.0, rtol=1e-6)
    np.testing.assert_allclose(period[1:] / period[:-1], 1000.0 ** (1 / 511), rtol=1e-6)


def test_time_mlp_identity_weights_reduces_to_silu_silu():
    D = 64
    e = RNG.normal(size=D)
    b1, b2 = RNG.normal(size=D), RNG.normal(size=D)
    out = M.time_mlp(e, np.eye(D), b1, 2.0 * np.eye(D), b2)
    te = torch.from_numpy(e)
    ref = F.silu(2.0 * F.silu(te + torch.from_numpy(b1)) + torch.from_numpy(b2)).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-13)


# ---------------------------------------------------------------------------------------
# expert: structural closed forms

def _tiny_inputs(cfg, B=2, C=3, P=6, lv=(4, 6)):
    noise = RNG.normal(size=(B, C, cfg.action_dim))
    kk = RNG.normal(size=(cfg.n_layers, B, P, cfg.head_dim))
    vv = RNG.normal(size=(cfg.n_layers, B, P, cfg.head_dim))
    return noise, kk, vv, np.array(lv[:B], dtype=np.int32)


def test_zero_adarms_makes_every_layer_the_identity():
    cfg = tiny_expert()
    W = rand_expert_weights(cfg)
    for l in range(cfg.n_layers):
        for nm in ("ada_attn_w", "ada_attn_b", "ada_ffn_w", "ada_ffn_b"):
            W[f"l{l}.{nm}"] = np.zeros_like(W[f"l{l}.{nm}"])
    h = RNG.normal(size=(3, cfg.width))
    cond = RNG.normal(size=cfg.width)
    kp, vp = RNG.normal(size=(6, cfg.head_dim)), RNG.normal(size=(6, cfg.head_dim))
    out = M.expert_layer(h, cond, M.Weights(W), 0, kp, vp, 4, cfg)
    np.testing.assert_array_equal(out, h)


def test_euler_closed_form_zero_out_proj():
    cfg = tiny_expert()
    W = rand_expert_weights(cfg)
    beta = RNG.normal(size=cfg.action_dim)
    W["action_out_w"] = np.zeros_like(W["action_out_w"])
    W["action_out_b"] = beta
    noise, kk, vv, lv = _tiny_inputs(cfg)
    out = M.sample_actions(W, cfg, noise, kk, vv, lv)
    np.testing.assert_allclose(out, noise - beta, rtol=0, atol=1e-12)   # 10 * (-0.1) * beta


def test_linear_closed_form_matrix_power():
    cfg = tiny_expert(final_norm=False)
    W = rand_expert_weights(cfg)
    for l in range(cfg.n_layers):
        for nm in ("ada_attn_w", "ada_attn_b", "ada_ffn_w", "ada_ffn_b"):
            W[f"l{l}.{nm}"] = np.zeros_like(W[f"l{l}.{nm}"])
    noise, kk, vv, lv = _tiny_inputs(cfg)
    out = M.sample_actions(W, cfg, noise, kk, vv, lv)
    dt = -0.1
    Win, bin_, Wout, bout = W["action_in_w"], W["action_in_b"], W["action_out_w"], W["action_out_b"]
    A = np.eye(cfg.action_dim) + dt * Win.T @ Wout.T       # row-vector map x -> x A + c
    c = dt * (bin_ @ Wout.T + bout)
    An = np.linalg.matrix_power(A, 10)
    geo = sum(np.linalg.matrix_power(A, j) for j in range(10))
    expect = noise @ An + c @ geo
    np.testing.assert_allclose(out, expect, rtol=1e-10, atol=1e-10)


def test_padded_prefix_keys_are_ignored_and_prefix_is_a_set():
    cfg = tiny_expert()
    W = M.Weights(rand_expert_weights(cfg))
    h = RNG.normal(size=(3, cfg.width))
    cond = RNG.normal(size=cfg.width)
    kp, vp = RNG.normal(size=(7, cfg.head_dim)), RNG.normal(size=(7, cfg.head_dim))
    base = M.expert_layer(h, cond, W, 1, kp, vp, 5, cfg)
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[5:], vp2[5:] = 1e4, -1e4
    np.testing.assert_array_equal(M.expert_layer(h, cond, W, 1, kp2, vp2, 5, cfg), base)
    perm = np.array([3, 0, 4, 1, 2, 5, 6])
    np.testing.assert_allclose(M.expert_layer(h, cond, W, 1, kp[perm], vp[perm], 5, cfg), base, rtol=1e-12, atol=1e-12)


def test_empty_prefix_equals_suffix_only_attention():
    cfg = tiny_expert()
    W = M.Weights(rand_expert_weights(cfg))
    h = RNG.normal(size=(3, cfg.width))
    cond = RNG.normal(size=cfg.width)
    kp, vp = RNG.normal(size=(5, cfg.head_dim)), RNG.normal(size=(5, cfg.head_dim))
    a = M.expert_layer(h, cond, W, 0, kp, vp, 0, cfg)
    b = M.expert_layer(h, cond, W, 0, kp[:0], vp[:0], 0, cfg)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_samples_are_independent():
    cfg = tiny_expert()
    W = rand_expert_weights(cfg)
    noise, kk, vv, lv = _tiny_inputs(cfg, B=2)
    both = M.sample_actions(W, cfg, noise, kk, vv, lv)
    one = M.sample_actions(W, cfg, noise[1:], kk[:, 1:], vv[:, 1:], lv[1:])
    np.testing.assert_array_equal(both[1:], one)


# ---------------------------------------------------------------------------------------
# independent torch fp64 formulation of the whole expert loop (tiny shapes)

def _torch_rope(x, pos, theta):
    hd = x.shape[-1]
    half = hd // 2
    freq = theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    rot = torch.polar(torch.ones(len(pos), half, dtype=torch.float64),
                      torch.tensor(pos, dtype=torch.float64)[:, None] * freq[None, :])
    z = torch.complex(x[..., :half], x[..., half:]) * rot
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_sample_actions(W, cfg, noise, kk, vv, lv):
    T = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in W.items()}
    D, H, hd = cfg.width, cfg.n_q_heads, cfg.head_dim
    x = torch.from_numpy(noise.astype(np.float64)).clone()
    half = D // 2
    for step in range(cfg.n_steps):
        t = 1.0 - step / cfg.n_steps
        per = 4e-3 * (1000.0 ** (torch.arange(half, dtype=torch.float64) / (half - 1)))
        e = torch.cat([torch.sin(2 * math.pi * t / per), torch.cos(2 * math.pi * t / per)])
        cond = F.silu(F.linear(F.silu(F.linear(e, T["time_in_w"], T["time_in_b"])), T["time_out_w"], T["time_out_b"]))
        for b in range(x.shape[0]):
            C = x.shape[1]
            P = kk.shape[2]
            h = F.linear(x[b], T["action_in_w"], T["action_in_b"])
            for l in range(cfg.n_layers):
                sc, sh, g = F.linear(cond, T[f"l{l}.ada_attn_w"], T[f"l{l}.ada_attn_b"]).chunk(3)
                n = F.rms_norm(h, (D,), eps=cfg.rms_eps) * (1 + sc) + sh
                q = F.linear(n, T[f"l{l}.wq"]).view(C, H, hd).transpose(0, 1)
                k = F.linear(n, T[f"l{l}.wk"]).view(C, 1, hd).transpose(0, 1)
                v = F.linear(n, T[f"l{l}.wv"]).view(C, 1, hd).transpose(0, 1)
                pos = list(range(int(lv[b]), int(lv[b]) + C))
                q, k = _torch_rope(q, pos, cfg.rope_theta), _torch_rope(k, pos, cfg.rope_theta)
                Kall = torch.cat([torch.from_numpy(kk[l, b][None].astype(np.float64)), k], 1).expand(H, P + C, hd)
                Vall = torch.cat([torch.from_numpy(vv[l, b][None].astype(np.float64)), v], 1).expand(H, P + C, hd)
                allowed = torch.cat([torch.arange(P) < int(lv[b]), torch.ones(C, dtype=torch.bool)])
                o = F.scaled_dot_product_attention(q, Kall, Vall, attn_mask=allowed[None, :].expand(C, P + C))
                h = h + F.linear(o.transpose(0, 1).reshape(C, H * hd), T[f"l{l}.wo"]) * g
                sc, sh, g = F.linear(cond, T[f"l{l}.ada_ffn_w"], T[f"l{l}.ada_ffn_b"]).chunk(3)
                n = F.rms_norm(h, (D,), eps=cfg.rms_eps) * (1 + sc) + sh
                m = F.gelu(F.linear(n, T[f"l{l}.wg"]), approximate="tanh") * F.linear(n, T[f"l{l}.wu"])
                h = h + F.linear(m, T[f"l{l}.wd"]) * g
            sc, sh, _ = F.linear(cond, T["ada_final_w"], T["ada_final_b"]).chunk(3)
            n = F.rms_norm(h, (D,), eps=cfg.rms_eps) * (1 + sc) + sh
            x[b] = x[b] - 0.1 * F.linear(n, T["action_out_w"], T["action_out_b"])
    return x.numpy()


def test_expert_loop_matches_independent_torch_formulation():
    cfg = tiny_expert()
    W = rand_expert_weights(cfg)
    noise, kk, vv, lv = _tiny_inputs(cfg, B=2, C=3, P=6, lv=(4, 6))
    out = M.sample_actions(W, cfg, noise, kk, vv, lv)
    ref = _torch_sample_actions(W, cfg, noise, kk, vv, lv)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-10)
    assert rel_l2(out, noise) > 0.05          # the loop really moved x


# ---------------------------------------------------------------------------------------
# prefill

def _torch_prefill(W, cfg, emb, mask):
    T = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in W.items()}
    B, P, D = emb.shape
    H, hd = cfg.n_q_heads, cfg.head_dim
    Ks = np.zeros((cfg.n_layers, B, P, hd))
    Vs = np.zeros_like(Ks)
    for b in range(B):
        x = torch.from_numpy(emb[b].astype(np.float64))
        valid = torch.from_numpy(mask[b].astype(bool))
        pos = (torch.cumsum(valid.long(), 0) - 1).tolist()
        for l in range(cfg.n_layers):
            n = F.rms_norm(x, (D,), eps=cfg.rms_eps) * (1 + T[f"pf{l}.ln1"])
            q = _torch_rope(F.linear(n, T[f"pf{l}.wq"]).view(P, H, hd).transpose(0, 1), pos, cfg.rope_theta)
            k = _torch_rope(F.linear(n, T[f"pf{l}.wk"]).view(P, 1, hd).transpose(0, 1), pos, cfg.rope_theta)
            v = F.linear(n, T[f"pf{l}.wv"]).view(P, 1, hd).transpose(0, 1)
            Ks[l, b], Vs[l, b] = k[0].numpy(), v[0].numpy()
            o = F.scaled_dot_product_attention(q, k.expand(H, P, hd), v.expand(H, P, hd),
                                               attn_mask=valid[None, :].expand(P, P))
            x = x + F.linear(o.transpose(0, 1).reshape(P, H * hd), T[f"pf{l}.wo"])
            n = F.rms_norm(x, (D,), eps=cfg.rms_eps) * (1 + T[f"pf{l}.ln2"])
            x = x + F.linear(F.gelu(F.linear(n, T[f"pf{l}.wg"]), approximate="tanh") * F.linear(n, T[f"pf{l}.wu"]), T[f"pf{l}.wd"])
    return Ks, Vs


def test_prefill_matches_independent_torch_formulation():
    cfg = tiny_prefill(n_layers=3)
    W = rand_prefill_weights(cfg)
    emb = RNG.normal(size=(2, 6, cfg.width)) * 4.0
    mask = np.array([[1, 1, 1, 1, 0, 0], [1, 1, 1, 1, 1, 1]], np.uint8)
    K, V, lv = M.prefill(W, cfg, emb, mask)
    Kr, Vr = _torch_prefill(W, cfg, emb, mask)
    np.testing.assert_array_equal(lv, [4, 6])
    for b, n in enumerate(lv):
        np.testing.assert_allclose(K[:, b, :n], Kr[:, b, :n], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(V[:, b, :n], Vr[:, b, :n], rtol=1e-10, atol=1e-10)


def test_prefill_single_valid_token_closed_form():
    cfg = tiny_prefill(n_layers=2)
    W = rand_prefill_weights(cfg)
    emb = RNG.normal(size=(1, 1, cfg.width))
    K, V, _ = M.prefill(W, cfg, emb, np.ones((1, 1), np.uint8))
    x = emb[0, 0]
    for l in range(cfg.n_layers):
        n = x / np.sqrt((x * x).mean() + cfg.rms_eps) * (1 + W[f"pf{l}.ln1"])
        v = W[f"pf{l}.wv"] @ n
        k = W[f"pf{l}.wk"] @ n                  # position 0: RoPE is the identity
        np.testing.assert_allclose(K[l, 0, 0], k, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(V[l, 0, 0], v, rtol=1e-12, atol=1e-12)
        x = x + W[f"pf{l}.wo"] @ np.tile(v, cfg.n_q_heads)     # softmax over one key = 1
        n = x / np.sqrt((x * x).mean() + cfg.rms_eps) * (1 + W[f"pf{l}.ln2"])
        x = x + W[f"pf{l}.wd"] @ (M.gelu_tanh(W[f"pf{l}.wg"] @ n) * (W[f"pf{l}.wu"] @ n))


def test_prefill_padding_and_layer_dependencies():
    cfg = tiny_prefill(n_layers=3)
    W = rand_prefill_weights(cfg)
    emb = RNG.normal(size=(1, 7, cfg.width))
    mask = np.array([[1, 1, 1, 1, 1, 0, 0]], np.uint8)
    K, V, _ = M.prefill(W, cfg, emb, mask)
    emb2 = emb.copy()
    emb2[0, 5:] = 99.0
    K2, V2, _ = M.prefill(W, cfg, emb2, mask)
    np.testing.assert_array_equal(K2[:, :, :5], K[:, :, :5])
    W3 = dict(W)
    W3["pf2.wd"] = W["pf2.wd"] * 5.0                        # last layer's MLP feeds nothing
    W3["pf2.wo"] = -W["pf2.wo"]
    K3, V3, _ = M.prefill(W3, cfg, emb, mask)
    np.testing.assert_array_equal(K3, K)
    np.testing.assert_array_equal(V3, V)
    W4 = dict(W)
    W4["pf1.wk"] = W["pf1.wk"] * 2.0
    K4, _, _ = M.prefill(W4, cfg, emb, mask)
    np.testing.assert_array_equal(K4[0], K[0])
    assert not np.allclose(K4[1], K[1])


# ---------------------------------------------------------------------------------------
# folding identities the CUDA path relies on (exact in real arithmetic)

def test_folding_identities_fp64():
    D, N = 64, 48
    h = RNG.normal(size=(5, D)) * 3
    s, sh = RNG.normal(size=D) * 0.1, RNG.normal(size=D) * 0.1
    Wt = RNG.normal(size=(N, D))
    r = 1.0 / np.sqrt((h * h).mean(-1, keepdims=True) + 1e-6)
    unfolded = (h * r * (1 + s) + sh) @ Wt.T
    deferred = r * ((h * (1 + s)) @ Wt.T) + sh @ Wt.T       # norm factor applied after the GEMM
    np.testing.assert_allclose(deferred, unfolded, rtol=1e-12, atol=1e-12)
    gamma = RNG.normal(size=D) * 0.02
    np.testing.assert_allclose((M.rms_normalize(h, 1e-6) * (1 + gamma)) @ Wt.T,
                               M.rms_normalize(h, 1e-6) @ (Wt * (1 + gamma)[None, :]).T, rtol=1e-12, atol=1e-12)
    x = RNG.normal(size=(5, 4))
    Wo, bo = RNG.normal(size=(4, D)), RNG.normal(size=4)
    n = RNG.normal(size=(5, D))
    np.testing.assert_allclose(x + (-0.1) * (n @ Wo.T + bo), x + n @ (-0.1 * Wo).T + (-0.1) * bo, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------------------
# mutation tests: the parity tolerances can tell a planted mistake apart (planted in the
# oracle, on the CPU, on the full-width 2-layer workload with gate biases 1.0)

ACT_MAX_ABS, ACT_REL_L2, H_REL_L2 = 3e-2, 1e-2, 1e-2


@pytest.fixture(scope="module")
def stressed_tiny():
    w = WL.workload(1)
    Wt = WL.as_f32(WL.expert_weights(w.expert, stressed=True))
    k, v, lv = WL.kv_cache(w)
    kf, vf = gen.bf16_to_f32(k), gen.bf16_to_f32(v)
    x0 = WL.noise(w)
    ref, tr = M.sample_actions(Wt, w.expert, x0, kf, vf, lv, trace_step=0)
    return w, Wt, kf, vf, lv, x0, ref, tr


def _fails_parity(out, tr, ref, rtr):
    d = np.abs(out - ref).max()
    return (d > ACT_MAX_ABS) or (rel_l2(out, ref) > ACT_REL_L2) or any(
        rel_l2(tr[i] - tr[i - 1], rtr[i] - rtr[i - 1]) > H_REL_L2 for i in range(1, tr.shape[0]))


MUTANTS = {
    "no_rope": lambda mp: mp.setattr(M, "rope", lambda x, pos, theta: x),
    "suffix_pos_from_zero": lambda mp: mp.setattr(
        M, "rope", (lambda f: lambda x, pos, theta: f(x, np.asarray(pos) - np.asarray(pos)[0], theta))(M.rope)),
    "swap_scale_shift": lambda mp: mp.setattr(
        M, "ada_rms_norm", lambda x, c, w, b, eps: (
            M.rms_normalize(x, eps) * (1 + (w @ c + b)[x.shape[-1]:2 * x.shape[-1]]) + (w @ c + b)[:x.shape[-1]],
            (w @ c + b)[2 * x.shape[-1]:])),
    "ignore_suffix_keys": lambda mp: mp.setattr(
        M, "attention", (lambda f: lambda q, k, v, mask, sc: f(q, k, v, np.concatenate(
            [mask[:, :-q.shape[1]], np.zeros_like(mask[:, -q.shape[1]:])], 1), sc))(M.attention)),
    "gelu_dropped": lambda mp: mp.setattr(M, "gelu_tanh", lambda x: x),
}


@pytest.mark.parametrize("name", sorted(MUTANTS) + ["valid_len_plus_one"])
def test_mutants_fail_parity(stressed_tiny, monkeypatch, name):
    w, Wt, kf, vf, lv, x0, ref, rtr = stressed_tiny
    if name == "valid_len_plus_one":
        out, tr = M.sample_actions(Wt, w.expert, x0, kf, vf, lv + 1, trace_step=0)
    else:
        MUTANTS[name](monkeypatch)
        out, tr = M.sample_actions(Wt, w.expert, x0, kf, vf, lv, trace_step=0)
    assert _fails_parity(out, tr, ref, rtr), name


def test_golden_regression_of_the_oracle():
    import json
    import os
    import importlib.util
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(here, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    stored = json.load(open(os.path.join(here, "tiny_expert_actions.json")))
    expect = np.array([float.fromhex(x) for x in stored["actions"]]).reshape(stored["shape"])
    np.testing.assert_allclose(mg.compute(), expect, rtol=1e-12, atol=1e-12)


# The same planted mistakes at full size (18 layers, width 1024, 1-view: chunk 50, 280 of 288
# prefix tokens valid), on plain N(0, 0.02) and on stressed weights, caught by the per-layer
# check the GPU tests apply (every hidden state and every layer's update within the bound of
# PER_LAYER_TOL).  On plain weights a check of the final actions alone misses
# several of them, because each layer's update is small next to h; the per-layer updates do
# not.  Step 0 of the loop is traced (it depends only on t_0 = 1: one Euler step suffices).

@pytest.fixture(scope="module", params=["plain", "stressed"])
def full_size(request):
    from dataclasses import replace
    w = WL.workload(2)
    one = replace(w.expert, n_steps=1)
    Wt = M.Weights(WL.as_f32(WL.expert_weights(w.expert, stressed=request.param == "stressed")))
    k, v, lv = WL.kv_cache(w)
    kf, vf = gen.bf16_to_f32(k), gen.bf16_to_f32(v)
    x0 = WL.noise(w)
    _, tr = M.sample_actions(Wt, one, x0, kf, vf, lv, trace_step=0)
    return request.param, one, Wt, kf, vf, lv, x0, tr


# the per-layer bound of the GPU tests (hidden states and updates): 1e-2 on plain weights;
# 2e-2 where updates are O(1) (stressed weights), there the bf16 floor of the GPU path is ~1e-2
PER_LAYER_TOL = {"plain": 1e-2, "stressed": 2e-2}


def _fails_per_layer(tr, rtr, tol):
    return any(rel_l2(tr[i], rtr[i]) > tol for i in range(tr.shape[0])) or any(
        rel_l2(tr[i] - tr[i - 1], rtr[i] - rtr[i - 1]) > tol for i in range(1, tr.shape[0]))


@pytest.mark.parametrize("name", sorted(MUTANTS) + ["valid_len_plus_one"])
def test_mutants_fail_the_per_layer_check_at_full_size(full_size, monkeypatch, name):
    kind, one, Wt, kf, vf, lv, x0, rtr = full_size
    if name == "valid_len_plus_one":
        _, tr = M.sample_actions(Wt, one, x0, kf, vf, lv + 1, trace_step=0)
    else:
        MUTANTS[name](monkeypatch)
        _, tr = M.sample_actions(Wt, one, x0, kf, vf, lv, trace_step=0)
    assert _fails_per_layer(tr, rtr, PER_LAYER_TOL[kind]), (kind, name)


# ---------------------------------------------------------------------------------------
# the π0 suffix variant (readings P1-P5 in oracle/model.py)

def rand_pi0_weights(cfg, std=0.3, bias_std=0.1, rng=RNG):
    shapes = WL.pi0_expert_weight_shapes(cfg)
    return {k: rng.normal(0, bias_std if k.endswith("_b") else std, size=s) for k, s in shapes.items()}


def _torch_pi0_sample_actions(W, cfg, noise, state, kk, vv, lv):
    """An independent torch fp64 formulation of the π0 loop: F.linear / F.rms_norm / SDPA with a
    boolean mask / complex-rotation RoPE; the suffix built as one [state ; actions] tensor."""
    T = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in W.items()}
    D, H, hd = cfg.width, cfg.n_q_heads, cfg.head_dim
    x = torch.from_numpy(noise.astype(np.float64)).clone()
    st = torch.from_numpy(np.asarray(state, dtype=np.float64))
    half = D // 2
    for step in range(cfg.n_steps):
        t = 1.0 - step / cfg.n_steps
        per = 4e-3 * (1000.0 ** (torch.arange(half, dtype=torch.float64) / (half - 1)))
        e = torch.cat([torch.sin(2 * math.pi * t / per), torch.cos(2 * math.pi * t / per)])
        for b in range(x.shape[0]):
            C = x.shape[1]
            P = kk.shape[2]
            a = F.linear(x[b], T["action_in_w"], T["action_in_b"])
            at = torch.cat([a, e.expand(C, D)], dim=1)
            ha = F.linear(F.silu(F.linear(at, T["action_time_in_w"], T["action_time_in_b"])),
                          T["action_time_out_w"], T["action_time_out_b"])
            h = torch.cat([F.linear(st[b], T["state_w"], T["state_b"])[None], ha], 0)
            Tn = C + 1
            for l in range(cfg.n_layers):
                n = F.rms_norm(h, (D,), weight=1 + T[f"l{l}.ln1"], eps=cfg.rms_eps)
                q = F.linear(n, T[f"l{l}.wq"]).view(Tn, H, hd).transpose(0, 1)
                k = F.linear(n, T[f"l{l}.wk"]).view(Tn, 1, hd).transpose(0, 1)
                v = F.linear(n, T[f"l{l}.wv"]).view(Tn, 1, hd).transpose(0, 1)
                pos = list(range(int(lv[b]), int(lv[b]) + Tn))
                q, k = _torch_rope(q, pos, cfg.rope_theta), _torch_rope(k, pos, cfg.rope_theta)
                Kall = torch.cat([torch.from_numpy(kk[l, b][None].astype(np.float64)), k], 1).expand(H, P + Tn, hd)
                Vall = torch.cat([torch.from_numpy(vv[l, b][None].astype(np.float64)), v], 1).expand(H, P + Tn, hd)
                allowed = torch.cat([torch.arange(P) < int(lv[b]), torch.ones(Tn, dtype=torch.bool)])
                o = F.scaled_dot_product_attention(q, Kall, Vall, attn_mask=allowed[None, :].expand(Tn, P + Tn))
                h = h + F.linear(o.transpose(0, 1).reshape(Tn, H * hd), T[f"l{l}.wo"])
                n = F.rms_norm(h, (D,), weight=1 + T[f"l{l}.ln2"], eps=cfg.rms_eps)
                h = h + F.linear(F.gelu(F.linear(n, T[f"l{l}.wg"]), approximate="tanh") * F.linear(n, T[f"l{l}.wu"]),
                                 T[f"l{l}.wd"])
            n = F.rms_norm(h, (D,), weight=1 + T["final_ln"], eps=cfg.rms_eps)
            x[b] = x[b] - 0.1 * F.linear(n[1:], T["action_out_w"], T["action_out_b"])
    return x.numpy()


def _pi0_inputs(cfg, B=2, C=3, P=6, lv=(4, 6)):
    noise, kk, vv, lvs = _tiny_inputs(cfg, B=B, C=C, P=P, lv=lv)
    return noise, RNG.normal(size=(B, cfg.action_dim)), kk, vv, lvs


def test_pi0_loop_matches_independent_torch_formulation():
    cfg = tiny_expert()
    W = rand_pi0_weights(cfg)
    noise, state, kk, vv, lv = _pi0_inputs(cfg)
    out = M.pi0_sample_actions(W, cfg, noise, state, kk, vv, lv)
    ref = _torch_pi0_sample_actions(W, cfg, noise, state, kk, vv, lv)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-10)
    assert rel_l2(out, noise) > 0.05


def test_pi0_action_time_fold_and_table():
    """The folding the library applies at create time: Linear_in([W_a x + b_a ; e(t)]) =
    (W_in[:, :D] W_a) x + (W_in[:, :D] b_a + W_in[:, D:] e(t) + b_in), one table row per t."""
    cfg = tiny_expert()
    W = rand_pi0_weights(cfg)
    D = cfg.width
    Wi, bi = W["action_time_in_w"], W["action_time_in_b"]
    x = RNG.normal(size=(5, cfg.action_dim))
    fold = Wi[:, :D] @ W["action_in_w"]
    for k in range(cfg.n_steps):
        t = 1.0 - k / cfg.n_steps
        e = M.sinusoidal_time_embedding(t, D)
        direct = np.concatenate([x @ W["action_in_w"].T + W["action_in_b"], np.broadcast_to(e, (5, D))], 1) @ Wi.T + bi
        table = Wi[:, :D] @ W["action_in_b"] + Wi[:, D:] @ e + bi
        np.testing.assert_allclose(x @ fold.T + table, direct, rtol=1e-12, atol=1e-12)


def test_pi0_euler_closed_form_and_state_only_through_attention():
    cfg = tiny_expert()
    W = rand_pi0_weights(cfg)
    noise, state, kk, vv, lv = _pi0_inputs(cfg)
    beta = RNG.normal(size=cfg.action_dim)
    Z = dict(W, action_out_w=np.zeros_like(W["action_out_w"]), action_out_b=beta)
    np.testing.assert_allclose(M.pi0_sample_actions(Z, cfg, noise, state, kk, vv, lv), noise - beta,
                               rtol=0, atol=1e-12)
    # the state token reaches the actions only through attention: with every o_proj zero, the
    # actions ignore the state (and the prefix); with them, they do not
    Wz = dict(W)
    for l in range(cfg.n_layers):
        Wz[f"l{l}.wo"] = np.zeros_like(W[f"l{l}.wo"])
    a = M.pi0_sample_actions(Wz, cfg, noise, state, kk, vv, lv)
    b = M.pi0_sample_actions(Wz, cfg, noise, state + 1.0, kk * -1.0, vv, lv)
    np.testing.assert_array_equal(a, b)
    c = M.pi0_sample_actions(W, cfg, noise, state, kk, vv, lv)
    d = M.pi0_sample_actions(W, cfg, noise, state + 1.0, kk, vv, lv)
    assert np.abs(c - d).max() > 1e-3


def test_pi0_suffix_positions_and_state_row():
    """The suffix is [state ; actions]: the trace has C + 1 rows per step and its first row
    entering layer 0 is the state projection W_s state + b_s (reading P1)."""
    cfg = tiny_expert()
    W = M.Weights(rand_pi0_weights(cfg))
    noise, state, kk, vv, lv = _pi0_inputs(cfg, B=1, lv=(4,))
    _, tr = M.pi0_sample_actions(W, cfg, noise, state, kk, vv, lv, trace_step=0)
    np.testing.assert_allclose(tr[0, 0, 0], W["state_w"] @ state[0] + W["state_b"], rtol=1e-13, atol=1e-13)
    assert tr.shape == (cfg.n_layers + 1, 1, noise.shape[1] + 1, cfg.width)


PI0_MUTANTS = {
    "no_state_token": lambda mp: mp.setattr(
        M, "pi0_suffix", (lambda f: lambda W, x, s, t, cfg: np.concatenate(
            [np.zeros((1, cfg.width)), f(W, x, s, t, cfg)[1:]], 0))(M.pi0_suffix)),
    "time_embedding_dropped": lambda mp: mp.setattr(
        M, "sinusoidal_time_embedding", lambda t, dim, **k: np.zeros(dim)),
    "no_rope": lambda mp: mp.setattr(M, "rope", lambda x, pos, theta: x),
}


@pytest.mark.parametrize("name", sorted(PI0_MUTANTS))
def test_pi0_mutants_fail_parity(monkeypatch, name):
    """On the full-width 2-layer π0 expert with N(0, 0.02) weights, each planted mistake moves
    the actions or a layer's update beyond the parity tolerance."""
    from dataclasses import replace
    w = WL.workload(1)
    Wt = M.Weights(WL.as_f32(WL.pi0_expert_weights(w.expert, bias_std=0.02)))
    k, v, lv = WL.kv_cache(w)
    kf, vf = gen.bf16_to_f32(k), gen.bf16_to_f32(v)
    x0, st = WL.noise(w), WL.state(w)
    ref, rtr = M.pi0_sample_actions(Wt, w.expert, x0, st, kf, vf, lv, trace_step=0)
    PI0_MUTANTS[name](monkeypatch)
    out, tr = M.pi0_sample_actions(Wt, w.expert, x0, st, kf, vf, lv, trace_step=0)
    assert _fails_parity(out, tr, ref, rtr), name
