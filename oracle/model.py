"""Plain, slow, fp64 CPU oracle of the π0.5 action-expert denoise loop and the prefix pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it.  It shares
no code with the CUDA library; its only inputs are numpy arrays (weights given as the same
bf16 values the library receives, upcast to float64).

Sources (cited by page title and section):
  [BLOG]   Realtime-VLA tech blog (blog.w4k4.me), sections "pi0.5 inference flow",
           "Per-layer processing (PiGemmaDecoderLayer.forward)", "Decoder-only path
           (denoise_step)", "Precompute (__init__)".
  [PAPER]  "Running VLAs at Real-time Speed" (arXiv 2510.26742), Sec. 3.2 and Table 1.

It computes the UNFOLDED graph: AdaRMS dense layers evaluated every step, separate Q/K/V
projections, explicit RoPE, an explicit boolean mask matrix, K/V explicitly repeated to
all query heads, an explicit Euler update.  Every array is float64.

Readings where the pages are silent or ambiguous (each is also listed in the design notes):
  R1 time MLP: cond = SiLU(W_out SiLU(W_in e + b_in) + b_out)  [BLOG "Precompute"].
  R2 sinusoidal embedding: 512 sin + 512 cos, periods geometric from 4e-3 to 4.0.
  R3 final expert norm: one more AdaRMS (scale/shift; gate unused) before action_out_proj.
  R4 RoPE pairs (d, d + hd/2) ("rotate half").
  R5 positions: prefix pos = cumsum(mask) - 1; suffix pos = Lv + j.
  R6 suffix tokens see every valid prefix key and all C suffix keys; no causal term.
  R7 masked logits are -inf (the blog's kernel uses -2.38e38; identical after softmax).
  R8 RMS eps 1e-6 inside the rsqrt, mean over the width.
  R9 Gemma RMSNorm multiplies by (1 + w).
  R10 GELU is the tanh approximation.
  R11 attention scaling 1/sqrt(head_dim), no soft-cap.
  R12 t_k = 1 - k/S evaluated exactly (not accumulated), dt = -1/S.

The π0 variant (``pi0_sample_actions``) follows [PAPER-S] ("Running VLAs at Real-time
Speed" summary, section "How": the action time encoder's two linears fold, and its 10
timestep rows become a table in the bias before SiLU; "π0 preliminaries": the state and the
noisy actions are routed to the action expert, a Gemma reduced in width).  Readings:
  P1 suffix = [one state token ; C action tokens]; state token = Linear(32 -> width)(state).
  P2 action token = Linear_out(SiLU(Linear_in([action_in_proj(x) ; SinEmb(t)]))): the time
     embedding (R2) is concatenated to each projected action, then a 2-layer MLP.
  P3 every norm is a plain Gemma RMSNorm, x_hat * (1 + w) (R8, R9); residuals are ungated.
  P4 the C + 1 suffix tokens attend to every valid prefix key and to each other (as R6),
     at positions Lv + i, i = 0 for the state token (as R5).
  P5 a final RMSNorm, then action_out_proj on the C action tokens only; Euler as R12.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------------------
# primitives

def silu(x):
    """SiLU(x) = x * sigmoid(x) (Elfwing et al. 2018)."""
    return x / (1.0 + np.exp(-x))


def gelu_tanh(x):
    """GELU, tanh approximation (Hendrycks & Gimpel 2016); reading R10."""
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def sinusoidal_time_embedding(t: float, dim: int, min_period: float = 4e-3,
                              max_period: float = 4.0) -> np.ndarray:
    """[BLOG "pi0.5 inference flow", decoder step 1]: t -> dim-wide sinusoidal embedding.

    Reading R2: half = dim/2 frequencies; period_i = min_period * (max_period /
    min_period) ** (i / (half - 1)); embedding = [sin(2 pi t / period_i)]_i ++
    [cos(2 pi t / period_i)]_i.
    """
    half = dim // 2
    frac = np.arange(half, dtype=F64) / (half - 1)
    period = min_period * (max_period / min_period) ** frac
    angle = 2.0 * np.pi * F64(t) / period
    return np.concatenate([np.sin(angle), np.cos(angle)])


def time_mlp(e, w_in, b_in, w_out, b_out):
    """[BLOG "Precompute"]: adarms_cond = SiLU(Linear_out(SiLU(Linear_in(e)))) (reading R1)."""
    return silu(w_out @ silu(w_in @ e + b_in) + b_out)


def rms_normalize(x, eps):
    """x / sqrt(mean(x^2) + eps) over the last axis (reading R8)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def ada_rms_norm(x, cond, w, b, eps):
    """[BLOG "Per-layer processing"]: dense(cond) -> (scale, shift, gate);
    returns (x_norm * (1 + scale) + shift, gate)."""
    d = x.shape[-1]
    mod = w @ cond + b
    scale, shift, gate = mod[:d], mod[d:2 * d], mod[2 * d:3 * d]
    return rms_normalize(x, eps) * (1.0 + scale) + shift, gate


def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """[BLOG "Precompute"]: inv_freq_i = 1 / theta^(2i / head_dim), i < head_dim/2."""
    i = np.arange(head_dim // 2, dtype=F64)
    return 1.0 / (F64(theta) ** (2.0 * i / head_dim))


def rope(x, pos, theta):
    """Rotary embedding of x [..., T, hd] at integer positions pos [T] (reading R4).

    Component d and d + hd/2 form one pair, rotated by angle pos * inv_freq_d.
    """
    hd = x.shape[-1]
    half = hd // 2
    ang = np.asarray(pos, dtype=F64)[:, None] * rope_inv_freq(hd, theta)[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def repeat_kv(x, n_rep: int):
    """[BLOG "Per-layer processing"]: repeat_kv expands 1 KV head to all query heads."""
    return np.repeat(x, n_rep, axis=0)


def attention(q, k, v, mask, scaling):
    """softmax(q k^T * scaling + mask) v with an explicit boolean mask.

    q [H, Tq, hd]; k, v [Hkv, Tk, hd]; mask [Tq, Tk] (True = visible).  Masked logits are
    -inf (reading R7); every row must see at least one key.
    """
    rep = q.shape[0] // k.shape[0]
    k = repeat_kv(k, rep)
    v = repeat_kv(v, rep)
    s = (q @ k.transpose(0, 2, 1)) * scaling
    s = np.where(mask[None, :, :], s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v


# ---------------------------------------------------------------------------------------
# weights

class Weights:
    """float64 view of a dict of weight arrays (bf16 values already widened)."""

    def __init__(self, d: dict):
        self._d = d
        self._cache = {}

    def __getitem__(self, name):
        a = self._cache.get(name)
        if a is None:
            a = np.asarray(self._d[name], dtype=F64)
            self._cache[name] = a
        return a

    def __contains__(self, name):
        return name in self._d


def _as_weights(w):
    return w if isinstance(w, Weights) else Weights(w)


# ---------------------------------------------------------------------------------------
# action expert

def expert_layer(h, cond, W, l, k_pref, v_pref, lv, cfg):
    """One action-expert layer for one sample [BLOG "Per-layer processing"].

    h [C, D]; k_pref, v_pref [P, hd] (K already rotated); lv = valid prefix length.
    Order: AdaRMS -> q/k/v proj -> RoPE -> repeat_kv -> masked softmax attention over
    [prefix ; suffix] keys -> o_proj -> gated residual -> AdaRMS -> GELU(gate)*up -> down
    -> gated residual.
    """
    C, D = h.shape
    H, hd, Hkv = cfg.n_q_heads, cfg.head_dim, cfg.n_kv_heads
    P = k_pref.shape[0]
    p = f"l{l}."
    n, gate1 = ada_rms_norm(h, cond, W[p + "ada_attn_w"], W[p + "ada_attn_b"], cfg.rms_eps)
    q = (n @ W[p + "wq"].T).reshape(C, H, hd).transpose(1, 0, 2)
    k = (n @ W[p + "wk"].T).reshape(C, Hkv, hd).transpose(1, 0, 2)
    v = (n @ W[p + "wv"].T).reshape(C, Hkv, hd).transpose(1, 0, 2)
    pos = lv + np.arange(C)                                              # reading R5
    q = rope(q, pos, cfg.rope_theta)
    k = rope(k, pos, cfg.rope_theta)
    K = np.concatenate([np.broadcast_to(k_pref, (Hkv, P, hd)), k], axis=1)
    V = np.concatenate([np.broadcast_to(v_pref, (Hkv, P, hd)), v], axis=1)
    mask = np.zeros((C, P + C), dtype=bool)                              # reading R6
    mask[:, :lv] = True
    mask[:, P:] = True
    o = attention(q, K, V, mask, hd ** -0.5)                             # reading R11
    o = o.transpose(1, 0, 2).reshape(C, H * hd)
    h = h + (o @ W[p + "wo"].T) * gate1
    n2, gate2 = ada_rms_norm(h, cond, W[p + "ada_ffn_w"], W[p + "ada_ffn_b"], cfg.rms_eps)
    m = gelu_tanh(n2 @ W[p + "wg"].T) * (n2 @ W[p + "wu"].T)
    return h + (m @ W[p + "wd"].T) * gate2


def adarms_cond(W, t, cfg):
    e = sinusoidal_time_embedding(t, cfg.width)
    return time_mlp(e, W["time_in_w"], W["time_in_b"], W["time_out_w"], W["time_out_b"])


def velocity(W, x, cond, k_pref, v_pref, lv, cfg, trace=None):
    """v_t for one sample: action_in_proj -> L expert layers -> (final AdaRMS) ->
    action_out_proj [BLOG "pi0.5 inference flow", decoder steps 1-3]."""
    h = x @ W["action_in_w"].T + W["action_in_b"]
    if trace is not None:
        trace.append(h.copy())
    for l in range(cfg.n_layers):
        h = expert_layer(h, cond, W, l, k_pref[l], v_pref[l], lv, cfg)
        if trace is not None:
            trace.append(h.copy())
    if cfg.final_norm:                                                   # reading R3
        n, _ = ada_rms_norm(h, cond, W["ada_final_w"], W["ada_final_b"], cfg.rms_eps)
    else:
        n = h
    return n @ W["action_out_w"].T + W["action_out_b"]


def sample_actions(weights, cfg, noise, kv_k, kv_v, valid_len, trace_step=None,
                   batch_indices=None):
    """The 10-step flow-matching Euler loop [BLOG "pi0.5 inference flow", decoder step 4].

    noise [B, C, A] (t = 1); kv_k, kv_v [L, B, P, hd]; valid_len [B].
    x_{t+dt} = x_t + dt * v_t with dt = -1/S, t_k = 1 - k/S (reading R12).
    Returns actions [B, C, A] (t = 0) and, if trace_step is given, the hidden states
    [L+1, B, C, D] of that step (before layer 0 and after every layer).
    batch_indices restricts the work to those samples (samples are independent).
    """
    W = _as_weights(weights)
    S = cfg.n_steps
    dt = -1.0 / S
    x = np.array(noise, dtype=F64)
    B = x.shape[0]
    idx = range(B) if batch_indices is None else list(batch_indices)
    tr = None
    if trace_step is not None:
        tr = np.zeros((cfg.n_layers + 1, B, x.shape[1], cfg.width), dtype=F64)
    kk = np.asarray(kv_k)
    vv = np.asarray(kv_v)
    for k in range(S):
        t = 1.0 - k / S
        cond = adarms_cond(W, t, cfg)
        for b in idx:
            lst = [] if (trace_step is not None and k == trace_step) else None
            kp = kk[:, b].astype(F64)
            vp = vv[:, b].astype(F64)
            v = velocity(W, x[b], cond, kp, vp, int(valid_len[b]), cfg, lst)
            x[b] = x[b] + dt * v
            if lst is not None:
                tr[:, b] = np.stack(lst)
    return (x, tr) if trace_step is not None else x


# ---------------------------------------------------------------------------------------
# prefix pass (Gemma-2B-shaped VLM layers that fill the KV cache)

def prefill(weights, cfg, embeds, pad_mask):
    """Prefix pass [BLOG "pi0.5 inference flow", encoder steps 3-4].

    embeds [B, P, Dp] (already scaled by sqrt(2048)); pad_mask [B, P] (1 = valid, all
    valid tokens first).  Every layer: x += o_proj(attn(RoPE(q), RoPE(k), v)) over a
    bidirectional mask on valid keys; x += down(GELU(gate) * up) of RMSNorm(x)*(1+w)
    (reading R9).  Returns K (rotated), V as float64 [L, B, P, hd] and valid_len [B].
    All L layers run in full here.
    """
    W = _as_weights(weights)
    B, P, _ = embeds.shape
    L, H, hd, Hkv = cfg.n_layers, cfg.n_q_heads, cfg.head_dim, cfg.n_kv_heads
    K = np.zeros((L, B, P, Hkv * hd), dtype=F64)
    V = np.zeros((L, B, P, Hkv * hd), dtype=F64)
    mask = np.asarray(pad_mask).astype(bool)
    valid_len = mask.sum(axis=1).astype(np.int32)
    for b in range(B):
        x = np.asarray(embeds[b], dtype=F64)
        pos = np.cumsum(mask[b].astype(np.int64)) - 1                    # reading R5
        amask = np.broadcast_to(mask[b][None, :], (P, P))
        for l in range(L):
            p = f"pf{l}."
            n = rms_normalize(x, cfg.rms_eps) * (1.0 + W[p + "ln1"])
            q = (n @ W[p + "wq"].T).reshape(P, H, hd).transpose(1, 0, 2)
            k = (n @ W[p + "wk"].T).reshape(P, Hkv, hd).transpose(1, 0, 2)
            v = (n @ W[p + "wv"].T).reshape(P, Hkv, hd).transpose(1, 0, 2)
            q = rope(q, pos, cfg.rope_theta)
            k = rope(k, pos, cfg.rope_theta)
            K[l, b] = k.transpose(1, 0, 2).reshape(P, Hkv * hd)
            V[l, b] = v.transpose(1, 0, 2).reshape(P, Hkv * hd)
            if valid_len[b] == 0:
                continue
            o = attention(q, k, v, amask, hd ** -0.5)
            x = x + o.transpose(1, 0, 2).reshape(P, H * hd) @ W[p + "wo"].T
            n2 = rms_normalize(x, cfg.rms_eps) * (1.0 + W[p + "ln2"])
            x = x + (gelu_tanh(n2 @ W[p + "wg"].T) * (n2 @ W[p + "wu"].T)) @ W[p + "wd"].T
    return K, V, valid_len


# ---------------------------------------------------------------------------------------
# π0 suffix variant (readings P1-P5 in the header)

def pi0_layer(h, W, l, k_pref, v_pref, lv, cfg):
    """One π0 action-expert layer for one sample: plain RMSNorm (reading P3), attention over
    [valid prefix ; all suffix tokens] (P4), ungated residuals.  h [T, D], T = C + 1."""
    T, D = h.shape
    H, hd, Hkv = cfg.n_q_heads, cfg.head_dim, cfg.n_kv_heads
    P = k_pref.shape[0]
    p = f"l{l}."
    n = rms_normalize(h, cfg.rms_eps) * (1.0 + W[p + "ln1"])
    q = (n @ W[p + "wq"].T).reshape(T, H, hd).transpose(1, 0, 2)
    k = (n @ W[p + "wk"].T).reshape(T, Hkv, hd).transpose(1, 0, 2)
    v = (n @ W[p + "wv"].T).reshape(T, Hkv, hd).transpose(1, 0, 2)
    pos = lv + np.arange(T)
    q = rope(q, pos, cfg.rope_theta)
    k = rope(k, pos, cfg.rope_theta)
    K = np.concatenate([np.broadcast_to(k_pref, (Hkv, P, hd)), k], axis=1)
    V = np.concatenate([np.broadcast_to(v_pref, (Hkv, P, hd)), v], axis=1)
    mask = np.zeros((T, P + T), dtype=bool)
    mask[:, :lv] = True
    mask[:, P:] = True
    o = attention(q, K, V, mask, hd ** -0.5)
    h = h + o.transpose(1, 0, 2).reshape(T, H * hd) @ W[p + "wo"].T
    n2 = rms_normalize(h, cfg.rms_eps) * (1.0 + W[p + "ln2"])
    return h + (gelu_tanh(n2 @ W[p + "wg"].T) * (n2 @ W[p + "wu"].T)) @ W[p + "wd"].T


def pi0_suffix(W, x, state, t, cfg):
    """The π0 suffix tokens [state ; actions] of one sample at time t (readings P1, P2)."""
    a = x @ W["action_in_w"].T + W["action_in_b"]
    e = sinusoidal_time_embedding(t, cfg.width)
    at = np.concatenate([a, np.broadcast_to(e, a.shape)], axis=-1)
    h_a = silu(at @ W["action_time_in_w"].T + W["action_time_in_b"]) @ W["action_time_out_w"].T \
        + W["action_time_out_b"]
    h_s = W["state_w"] @ state + W["state_b"]
    return np.concatenate([h_s[None, :], h_a], axis=0)


def pi0_velocity(W, x, state, t, k_pref, v_pref, lv, cfg, trace=None):
    """v_t of one sample: suffix tokens -> L π0 layers -> final RMSNorm -> action_out_proj on
    the action tokens (reading P5)."""
    h = pi0_suffix(W, x, state, t, cfg)
    if trace is not None:
        trace.append(h.copy())
    for l in range(cfg.n_layers):
        h = pi0_layer(h, W, l, k_pref[l], v_pref[l], lv, cfg)
        if trace is not None:
            trace.append(h.copy())
    n = rms_normalize(h, cfg.rms_eps) * (1.0 + W["final_ln"])
    return n[1:] @ W["action_out_w"].T + W["action_out_b"]


def pi0_sample_actions(weights, cfg, noise, state, kv_k, kv_v, valid_len, trace_step=None):
    """The π0 Euler loop: x_{t+dt} = x_t + dt * v_t, dt = -1/S, t_k = 1 - k/S (R12).

    noise [B, C, A]; state [B, A]; kv_k, kv_v [L, B, P, hd]; valid_len [B].  Returns actions
    [B, C, A] and, if trace_step is given, the hidden states [L+1, B, C+1, D] of that step.
    """
    W = _as_weights(weights)
    S = cfg.n_steps
    x = np.array(noise, dtype=F64)
    st = np.asarray(state, dtype=F64)
    B, C = x.shape[0], x.shape[1]
    tr = None if trace_step is None else np.zeros((cfg.n_layers + 1, B, C + 1, cfg.width), dtype=F64)
    kk, vv = np.asarray(kv_k), np.asarray(kv_v)
    for k in range(S):
        t = 1.0 - k / S
        for b in range(B):
            lst = [] if (trace_step is not None and k == trace_step) else None
            v = pi0_velocity(W, x[b], st[b], t, kk[:, b].astype(F64), vv[:, b].astype(F64),
                             int(valid_len[b]), cfg, lst)
            x[b] = x[b] + (-1.0 / S) * v
            if lst is not None:
                tr[:, b] = np.stack(lst)
    return (x, tr) if trace_step is not None else x
