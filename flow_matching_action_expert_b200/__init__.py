"""Python binding of librtvla.so (argument marshalling only).

Every function here has the name of the C entry point it calls (include/rtvla.h) and does
nothing but convert arguments: torch tensors become device pointers, dicts become the C
structs, status codes become exceptions.  All computation runs in the CUDA library.  If the
library is missing this module raises on first use — there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librtvla.so")

ENGINE_AUTO, ENGINE_LAYERED, ENGINE_PERSISTENT = 0, 1, 2
VARIANT_PI05, VARIANT_PI0 = 0, 1

STATUS = {
    0: "RTVLA_OK", 1: "RTVLA_ERR_INVALID_ARG", 2: "RTVLA_ERR_SHAPE", 3: "RTVLA_ERR_MASK_NOT_PREFIX",
    4: "RTVLA_ERR_OOM", 5: "RTVLA_ERR_CUDA", 6: "RTVLA_ERR_DEVICE_TIMEOUT", 7: "RTVLA_ERR_UNSUPPORTED",
    8: "RTVLA_ERR_DEVICE_BOUNDS", 9: "RTVLA_ERR_GUARD_OVERWRITE",
}

# the symbols include/rtvla.h declares
EXPORTS = (
    "rtvla_create", "rtvla_kv_bytes", "rtvla_prefill", "rtvla_sample_actions", "rtvla_sample_actions_host",
    "rtvla_sample_actions_host_static",
    "rtvla_sync_status", "rtvla_debug_trace", "rtvla_kernels_per_call", "rtvla_set_engine",
    "rtvla_set_wait_timeout_us", "rtvla_destroy", "rtvla_status_string", "rtvla_debug_plant_guard_fault",
    "rtvla_sample_actions_pi0", "rtvla_debug_trace_pi0",
    "rtvla_vision_create", "rtvla_encode_images", "rtvla_vision_debug_trace", "rtvla_vision_sync_status",
    "rtvla_vision_kernels_per_call", "rtvla_vision_destroy",
)


class RtvlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{where}: {self.name} ({_lib().rtvla_status_string(code).decode()})")


class RtvlaConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "n_layers", "width", "mlp_dim", "n_q_heads", "n_kv_heads", "head_dim", "action_dim", "chunk",
        "n_steps", "max_prefix", "max_batch", "final_norm", "has_prefill", "pf_width", "pf_mlp_dim",
        "engine")] + [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float), ("variant", ctypes.c_int)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)

_SINGLE = ("action_in_w", "action_in_b", "action_out_w", "action_out_b", "time_in_w", "time_in_b",
           "time_out_w", "time_out_b")
_LAYER = ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "ada_attn_w", "ada_attn_b", "ada_ffn_w", "ada_ffn_b")
_FINAL = ("ada_final_w", "ada_final_b")
_PF = ("pf_ln1", "pf_wq", "pf_wk", "pf_wv", "pf_wo", "pf_ln2", "pf_wg", "pf_wu", "pf_wd")
_PI0 = ("state_w", "state_b", "action_time_in_w", "action_time_in_b", "action_time_out_w", "action_time_out_b")
_PI0_LAYER = ("ln1", "ln2")


class RtvlaWeights(ctypes.Structure):
    _fields_ = ([(n, _P) for n in _SINGLE] + [(n, _PP) for n in _LAYER] + [(n, _P) for n in _FINAL]
                + [(n, _PP) for n in _PF] + [(n, _P) for n in _PI0] + [(n, _PP) for n in _PI0_LAYER]
                + [("final_ln", _P)])


class RtvlaVisionConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "n_layers", "width", "mlp_dim", "n_heads", "patch", "image", "out_width", "max_images")] + [
        ("ln_eps", ctypes.c_float)]


_VIS_SINGLE = ("patch_w", "patch_b", "pos")
_VIS_LAYER = ("ln1_w", "ln1_b", "wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "ln2_w", "ln2_b",
              "fc1_w", "fc1_b", "fc2_w", "fc2_b")
_VIS_FINAL = ("post_w", "post_b", "proj_w", "proj_b")


class RtvlaVisionWeights(ctypes.Structure):
    _fields_ = [(n, _P) for n in _VIS_SINGLE] + [(n, _PP) for n in _VIS_LAYER] + [(n, _P) for n in _VIS_FINAL]


class RtvlaKV(ctypes.Structure):
    _fields_ = [("k", _P), ("v", _P), ("valid_len", _P), ("batch", ctypes.c_int), ("prefix_cap", ctypes.c_int)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"librtvla.so is not built ({LIB_PATH}); run "
                               "python -m flow_matching_action_expert_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        lib.rtvla_create.argtypes = [ctypes.POINTER(RtvlaWeights), ctypes.POINTER(RtvlaConfig), ctypes.POINTER(_P)]
        lib.rtvla_kv_bytes.argtypes = [ctypes.POINTER(RtvlaConfig), ctypes.c_int, ctypes.c_int]
        lib.rtvla_kv_bytes.restype = ctypes.c_size_t
        lib.rtvla_prefill.argtypes = [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.POINTER(RtvlaKV), _P]
        lib.rtvla_sample_actions.argtypes = [_P, _P, ctypes.POINTER(RtvlaKV), _P, _P]
        lib.rtvla_sample_actions_host.argtypes = [_P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P]
        lib.rtvla_sample_actions_host_static.argtypes = [_P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P]
        lib.rtvla_sample_actions_pi0.argtypes = [_P, _P, _P, ctypes.POINTER(RtvlaKV), _P, _P]
        lib.rtvla_debug_trace_pi0.argtypes = [_P, _P, _P, ctypes.POINTER(RtvlaKV), ctypes.c_int, _P, _P]
        lib.rtvla_sync_status.argtypes = [_P, _P]
        lib.rtvla_debug_trace.argtypes = [_P, _P, ctypes.POINTER(RtvlaKV), ctypes.c_int, _P, _P]
        lib.rtvla_kernels_per_call.argtypes = [_P, ctypes.c_int]
        lib.rtvla_set_engine.argtypes = [_P, ctypes.c_int]
        lib.rtvla_set_wait_timeout_us.argtypes = [_P, ctypes.c_longlong]
        lib.rtvla_debug_plant_guard_fault.argtypes = [_P]
        lib.rtvla_destroy.argtypes = [_P]
        lib.rtvla_destroy.restype = None
        lib.rtvla_vision_create.argtypes = [ctypes.POINTER(RtvlaVisionWeights), ctypes.POINTER(RtvlaVisionConfig),
                                            ctypes.POINTER(_P)]
        lib.rtvla_encode_images.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P]
        lib.rtvla_vision_debug_trace.argtypes = [_P, _P, ctypes.c_int, _P, _P, _P]
        lib.rtvla_vision_sync_status.argtypes = [_P, _P]
        lib.rtvla_vision_kernels_per_call.argtypes = [_P, ctypes.c_int]
        lib.rtvla_vision_destroy.argtypes = [_P]
        lib.rtvla_vision_destroy.restype = None
        lib.rtvla_status_string.argtypes = [ctypes.c_int]
        lib.rtvla_status_string.restype = ctypes.c_char_p
        for n in EXPORTS:
            if n not in ("rtvla_kv_bytes", "rtvla_destroy", "rtvla_status_string", "rtvla_kernels_per_call",
                         "rtvla_vision_destroy", "rtvla_vision_kernels_per_call"):
                getattr(lib, n).restype = ctypes.c_int
        lib.rtvla_kernels_per_call.restype = ctypes.c_int
        lib.rtvla_vision_kernels_per_call.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises if it is not built)."""
    return _lib()


def _check(code: int, where: str):
    if code != 0:
        raise RtvlaError(code, where)


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int:
    if s is None:
        return 0
    if isinstance(s, int):
        return s
    return s.cuda_stream


def make_config(n_layers=18, chunk=63, max_prefix=512, max_batch=1, n_steps=10, final_norm=True,
                has_prefill=False, engine=ENGINE_AUTO, rms_eps=1e-6, rope_theta=10000.0,
                variant=VARIANT_PI05) -> RtvlaConfig:
    """rtvla_config for the π0.5 / π0 shapes (width 1024 / MLP 4096 / 8 x 256 heads / action 32)."""
    return RtvlaConfig(n_layers=n_layers, width=1024, mlp_dim=4096, n_q_heads=8, n_kv_heads=1, head_dim=256,
                       action_dim=32, chunk=chunk, n_steps=n_steps, max_prefix=max_prefix,
                       max_batch=max_batch, final_norm=int(bool(final_norm)),
                       has_prefill=int(bool(has_prefill)), pf_width=2048, pf_mlp_dim=16384,
                       engine=engine, rms_eps=rms_eps, rope_theta=rope_theta, variant=variant)


def make_weights(w: dict, n_layers: int):
    """rtvla_weights from a dict of CUDA bf16 tensors named as in synth.workloads.

    Returns (struct, keepalive); keep both alive until rtvla_create returns.
    """
    keep = []
    ws = RtvlaWeights()
    for n in _SINGLE + _FINAL + _PI0 + ("final_ln",):
        setattr(ws, n, _ptr(w.get(n)))
    for n in _LAYER + _PI0_LAYER:
        if not any(f"l{l}.{n}" in w for l in range(n_layers)):
            continue
        arr = (_P * n_layers)(*[_ptr(w.get(f"l{l}.{n}")) for l in range(n_layers)])
        keep.append(arr)
        setattr(ws, n, ctypes.cast(arr, _PP))
    if all(f"pf0.{n[3:]}" in w for n in _PF):
        for n in _PF:
            arr = (_P * n_layers)(*[_ptr(w[f"pf{l}.{n[3:]}"]) for l in range(n_layers)])
            keep.append(arr)
            setattr(ws, n, ctypes.cast(arr, _PP))
    return ws, keep


def make_vision_config(n_layers=27, max_images=2, ln_eps=1e-6) -> RtvlaVisionConfig:
    """rtvla_vision_config for the SigLIP-So400m/14 shape (width 1152, MLP 4304, 16 heads, patch 14,
    224 x 224 images, projector to 2048)."""
    return RtvlaVisionConfig(n_layers=n_layers, width=1152, mlp_dim=4304, n_heads=16, patch=14, image=224,
                             out_width=2048, max_images=max_images, ln_eps=ln_eps)


def make_vision_weights(w: dict, n_layers: int):
    """rtvla_vision_weights from a dict of CUDA bf16 tensors named as in synth.workloads
    ("vis.patch_w", "vis{l}.wq", ...).  Returns (struct, keepalive)."""
    keep = []
    ws = RtvlaVisionWeights()
    for n in _VIS_SINGLE + _VIS_FINAL:
        setattr(ws, n, _ptr(w.get(f"vis.{n}")))
    for n in _VIS_LAYER:
        if not any(f"vis{l}.{n}" in w for l in range(n_layers)):
            continue
        arr = (_P * n_layers)(*[_ptr(w.get(f"vis{l}.{n}")) for l in range(n_layers)])
        keep.append(arr)
        setattr(ws, n, ctypes.cast(arr, _PP))
    return ws, keep


def make_kv(k, v, valid_len, batch: int, prefix_cap: int) -> RtvlaKV:
    return RtvlaKV(k=_ptr(k), v=_ptr(v), valid_len=_ptr(valid_len), batch=batch, prefix_cap=prefix_cap)


# ---------------------------------------------------------------------------------------
# entry points (same names as the C ABI)

def rtvla_create(weights: dict, cfg: RtvlaConfig) -> int:
    ws, keep = make_weights(weights, cfg.n_layers)
    out = _P()
    _check(_lib().rtvla_create(ctypes.byref(ws), ctypes.byref(cfg), ctypes.byref(out)), "rtvla_create")
    del keep
    return out.value


def rtvla_kv_bytes(cfg: RtvlaConfig, batch: int, prefix_cap: int) -> int:
    return _lib().rtvla_kv_bytes(ctypes.byref(cfg), batch, prefix_cap)


def rtvla_prefill(ctx: int, prefix_embeds, pad_mask, batch: int, prefix_len: int, kv_out: RtvlaKV, stream=None):
    _check(_lib().rtvla_prefill(ctx, _ptr(prefix_embeds), _ptr(pad_mask), batch, prefix_len,
                                ctypes.byref(kv_out), _stream(stream)), "rtvla_prefill")


def rtvla_sample_actions(ctx: int, noise, kv: RtvlaKV, actions_out, stream=None):
    _check(_lib().rtvla_sample_actions(ctx, _ptr(noise), ctypes.byref(kv), _ptr(actions_out), _stream(stream)),
           "rtvla_sample_actions")


def rtvla_sample_actions_host(ctx: int, noise, kv_k, kv_v, valid_len, batch: int, prefix_cap: int, actions_out,
                              stream=None):
    """Host-buffer variant: noise/kv/valid_len/actions are CPU tensors (pinned for full speed)."""
    _check(_lib().rtvla_sample_actions_host(ctx, _ptr(noise), _ptr(kv_k), _ptr(kv_v), _ptr(valid_len), batch,
                                            prefix_cap, _ptr(actions_out), _stream(stream)),
           "rtvla_sample_actions_host")


def rtvla_sample_actions_host_static(ctx: int, noise, kv_k, kv_v, valid_len, batch: int, prefix_cap: int,
                                     actions_out, stream=None):
    """Allocation-free host-buffer call: stages through the library's fixed 32 MiB device array."""
    _check(_lib().rtvla_sample_actions_host_static(ctx, _ptr(noise), _ptr(kv_k), _ptr(kv_v), _ptr(valid_len),
                                                   batch, prefix_cap, _ptr(actions_out), _stream(stream)),
           "rtvla_sample_actions_host_static")


def rtvla_sample_actions_pi0(ctx: int, noise, state, kv: RtvlaKV, actions_out, stream=None):
    _check(_lib().rtvla_sample_actions_pi0(ctx, _ptr(noise), _ptr(state), ctypes.byref(kv), _ptr(actions_out),
                                           _stream(stream)), "rtvla_sample_actions_pi0")


def rtvla_debug_trace_pi0(ctx: int, noise, state, kv: RtvlaKV, step: int, h_layers, stream=None):
    _check(_lib().rtvla_debug_trace_pi0(ctx, _ptr(noise), _ptr(state), ctypes.byref(kv), step, _ptr(h_layers),
                                        _stream(stream)), "rtvla_debug_trace_pi0")


def rtvla_sync_status(ctx: int, stream=None) -> int:
    """Returns the device status code (0 = ok); does not raise."""
    return _lib().rtvla_sync_status(ctx, _stream(stream))


def rtvla_debug_trace(ctx: int, noise, kv: RtvlaKV, step: int, h_layers, stream=None):
    _check(_lib().rtvla_debug_trace(ctx, _ptr(noise), ctypes.byref(kv), step, _ptr(h_layers), _stream(stream)),
           "rtvla_debug_trace")


def rtvla_kernels_per_call(ctx: int, batch: int) -> int:
    return _lib().rtvla_kernels_per_call(ctx, batch)


def rtvla_set_engine(ctx: int, engine: int):
    _check(_lib().rtvla_set_engine(ctx, engine), "rtvla_set_engine")


def rtvla_set_wait_timeout_us(ctx: int, us: int):
    _check(_lib().rtvla_set_wait_timeout_us(ctx, us), "rtvla_set_wait_timeout_us")


def rtvla_debug_plant_guard_fault(ctx: int):
    _check(_lib().rtvla_debug_plant_guard_fault(ctx), "rtvla_debug_plant_guard_fault")


def rtvla_destroy(ctx: int):
    if ctx:
        _lib().rtvla_destroy(ctx)


def rtvla_status_string(code: int) -> str:
    return _lib().rtvla_status_string(code).decode()


# ---------------------------------------------------------------------------------------
# image front-end

def rtvla_vision_create(weights: dict, cfg: RtvlaVisionConfig) -> int:
    ws, keep = make_vision_weights(weights, cfg.n_layers)
    out = _P()
    _check(_lib().rtvla_vision_create(ctypes.byref(ws), ctypes.byref(cfg), ctypes.byref(out)),
           "rtvla_vision_create")
    del keep
    return out.value


def rtvla_encode_images(ctx: int, images, batch: int, views: int, prefix_embeds, prefix_len: int, stream=None):
    _check(_lib().rtvla_encode_images(ctx, _ptr(images), batch, views, _ptr(prefix_embeds), prefix_len,
                                      _stream(stream)), "rtvla_encode_images")


def rtvla_vision_debug_trace(ctx: int, images, n_images: int, h_layers, prefix_embeds, stream=None):
    _check(_lib().rtvla_vision_debug_trace(ctx, _ptr(images), n_images, _ptr(h_layers), _ptr(prefix_embeds),
                                           _stream(stream)), "rtvla_vision_debug_trace")


def rtvla_vision_sync_status(ctx: int, stream=None) -> int:
    """Returns the device status code (0 = ok); does not raise."""
    return _lib().rtvla_vision_sync_status(ctx, _stream(stream))


def rtvla_vision_kernels_per_call(ctx: int, n_images: int) -> int:
    return _lib().rtvla_vision_kernels_per_call(ctx, n_images)


def rtvla_vision_destroy(ctx: int):
    if ctx:
        _lib().rtvla_vision_destroy(ctx)
