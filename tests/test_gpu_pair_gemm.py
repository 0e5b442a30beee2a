"""The SM-pair GEMM (tcgen05 .cta_group::2, 256 weight rows x 256 tokens per pair of SMs),
which the library uses for token tiles of 256 when RTVLA_PAIR_GEMM=1 is set at
rtvla_create.  It serves every layered GEMM with more than 128 rows: the batch-16 denoise
loop and the 544-token prefix pass, both compared here with the fp64 oracle.
"""
import numpy as np
import pytest

from oracle import model as O
from synth import gen
from synth import workloads as WL

from harness import GpuModel, KV_REL_L2, assert_actions_close, assert_trace_close, device_kv, rel_l2

pytestmark = pytest.mark.gpu


def test_pair_gemm_three_view_batch16(monkeypatch):
    monkeypatch.setenv("RTVLA_PAIR_GEMM", "1")
    wl = WL.workload(4, batch=16)
    bits = WL.expert_weights(wl.expert)
    m = GpuModel(wl, bits)
    monkeypatch.delenv("RTVLA_PAIR_GEMM")
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise = WL.noise(wl)
    ref, rtr = O.sample_actions(WL.as_f32(bits), wl.expert, noise, kf, vf, vnp, trace_step=0)
    out = m.sample(noise, k, v, valid)
    assert_actions_close(out, ref, wl.name + " (SM-pair GEMM)")
    assert_trace_close(m.trace(noise, k, v, valid, 0), rtr, wl.name + " step 0 (SM-pair GEMM)")
    m.close()


def test_pair_gemm_prefill(monkeypatch):
    base = WL.workload(5)
    ebits = WL.expert_weights(base.expert)
    pbits = WL.prefill_weights(base.prefill)
    monkeypatch.setenv("RTVLA_PAIR_GEMM", "1")
    m = GpuModel(base, ebits, prefill_bits=pbits)
    monkeypatch.delenv("RTVLA_PAIR_GEMM")
    emb, mask = WL.prefill_inputs(base)
    Kr, Vr, vr = O.prefill(WL.as_f32(pbits), base.prefill, gen.bf16_to_f32(emb), mask)
    k, v, valid = m.prefill(emb, mask)
    np.testing.assert_array_equal(valid.cpu().numpy(), vr)
    kg, vg = k.float().cpu().numpy(), v.float().cpu().numpy()
    for b, n in enumerate(vr):
        for l in range(base.prefill.n_layers):
            rk = rel_l2(kg[l, b, :n], Kr[l, b, :n])
            rv = rel_l2(vg[l, b, :n], Vr[l, b, :n])
            assert rk <= KV_REL_L2 and rv <= KV_REL_L2, (b, l, rk, rv)
    m.close()
