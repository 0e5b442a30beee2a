"""fp64 CPU oracle of the π0.5 denoise loop (and its π0 suffix variant), the prefix pass and
the image front-end (SigLIP tower + projector, oracle/vision.py).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline leg, never by the product library.  Shares no code with the CUDA path.
Parity status of each function is stated in the module headers and their pins.
"""
from .model import (  # noqa: F401
    Weights, ada_rms_norm, adarms_cond, attention, expert_layer, gelu_tanh, pi0_layer,
    pi0_sample_actions, pi0_suffix, pi0_velocity, prefill,
    repeat_kv, rms_normalize, rope, rope_inv_freq, sample_actions, silu,
    sinusoidal_time_embedding, time_mlp, velocity,
)
from . import vision  # noqa: F401,E402
