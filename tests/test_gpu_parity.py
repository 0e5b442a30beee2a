"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded inputs.

Workloads: the tiny 2-layer expert, 1-view, 2-view, 3-view (batch 4 full, batch 64
sampled), the end-to-end prefix pass + denoise, and edge cases (empty / full / ragged
valid lengths, chunk 1 and a chunk spanning two token tiles, garbage in padded cache
slots).  Tolerances are the contract's: actions max-abs 3e-2 and rel-L2 1e-2, per-layer
hidden states and per-layer updates rel-L2 1e-2, prefix KV rel-L2 1e-2 on valid rows.
"""
import numpy as np
import pytest
import torch

import flow_matching_action_expert_b200 as R
from oracle import model as O
from synth import gen
from synth import workloads as WL

from harness import (GpuModel, assert_actions_close, assert_trace_close, bf16_dev, device_kv, rel_l2,
                     KV_REL_L2)

pytestmark = pytest.mark.gpu


def _oracle(wl, wf, kf, vf, valid, noise, trace_step=None, batch_indices=None):
    return O.sample_actions(wf, wl.expert, noise, kf, vf, valid, trace_step=trace_step,
                            batch_indices=batch_indices)


ENGINES = {"layered": R.ENGINE_LAYERED, "persistent": R.ENGINE_PERSISTENT}


@pytest.mark.parametrize("variant", ["plain", "stressed", "biased"])
def test_tiny_expert_actions_and_layers(variant):
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert, stressed=(variant == "stressed"),
                             bias_std=(0.02 if variant == "biased" else 0.0))
    wf = WL.as_f32(bits)
    m = GpuModel(wl, bits)
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise = WL.noise(wl)
    ref, rtr0 = _oracle(wl, wf, kf, vf, vnp, noise, trace_step=0)
    for name, eng in ENGINES.items():
        R.rtvla_set_engine(m.ctx, eng)
        out = m.sample(noise, k, v, valid)
        assert_actions_close(out, ref, f"tiny/{variant}/{name}")
    assert_trace_close(m.trace(noise, k, v, valid, 0), rtr0[:, :], f"tiny/{variant} step 0")
    _, rtr9 = _oracle(wl, wf, kf, vf, vnp, noise, trace_step=9)
    assert_trace_close(m.trace(noise, k, v, valid, 9), rtr9, f"tiny/{variant} step 9")
    m.close()


@pytest.mark.parametrize("engine", sorted(ENGINES))
@pytest.mark.parametrize("cfg", [2, 3])
def test_full_expert_actions(cfg, engine):
    wl = WL.workload(cfg)
    bits = WL.expert_weights(wl.expert)
    wf = WL.as_f32(bits)
    m = GpuModel(wl, bits, engine=ENGINES[engine])
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise = WL.noise(wl)
    ref, rtr = _oracle(wl, wf, kf, vf, vnp, noise, trace_step=4)
    out = m.sample(noise, k, v, valid)
    assert_actions_close(out, ref, wl.name)
    assert_trace_close(m.trace(noise, k, v, valid, 4), rtr, wl.name + " step 4")
    # a second call on the same context agrees with the first and with the oracle (split-K
    # sums are fp32 reductions in varying order, so repeat calls are not bitwise equal)
    out2 = m.sample(noise, k, v, valid)
    assert_actions_close(out2, ref, wl.name + " repeat")
    assert np.abs(out2 - out).max() <= 1e-2
    m.close()


def test_three_view_batch4_full_and_batch64_sampled():
    wl4 = WL.workload(4, batch=4)
    bits = WL.expert_weights(wl4.expert)
    wf = WL.as_f32(bits)
    m = GpuModel(wl4, bits, max_batch=64)
    k, v, valid, kf, vf, vnp = device_kv(wl4)
    noise = WL.noise(wl4)
    ref = _oracle(wl4, wf, kf, vf, vnp, noise)
    out = m.sample(noise, k, v, valid)
    assert_actions_close(out, ref, wl4.name)
    wl64 = WL.workload(4, batch=64)
    k, v, valid, kf, vf, vnp = device_kv(wl64)
    noise = WL.noise(wl64)
    out = m.sample(noise, k, v, valid)
    picks = [0, 37, 63]
    ref = _oracle(wl64, wf, kf, vf, vnp, noise, batch_indices=picks)
    assert_actions_close(out[picks], ref[picks], wl64.name + " sampled")
    m.close()


def test_edge_cases_lengths_chunks_and_padding():
    base = WL.workload(1)
    bits = WL.expert_weights(base.expert, stressed=True)
    wf = WL.as_f32(bits)
    for chunk, lens in ((1, (0, 7, 130)), (65, (130, 1, 0))):
        wl = WL.Workload(f"edge C{chunk}", base.expert, chunk, 3, 130, lens)
        m = GpuModel(wl, bits)
        k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
        noise = WL.noise(wl)
        ref = _oracle(wl, wf, kf, vf, vnp, noise)
        out = m.sample(noise, k, v, valid)
        assert_actions_close(out, ref, wl.name)
        m.close()


def test_persistent_engine_edge_cases():
    base = WL.workload(1)
    bits = WL.expert_weights(base.expert, stressed=True)
    wf = WL.as_f32(bits)
    for chunk, lv in ((1, 0), (64, 130), (37, 1), (64, 0)):
        wl = WL.Workload(f"edge B1 C{chunk} Lv{lv}", base.expert, chunk, 1, 130, (lv,))
        m = GpuModel(wl, bits, engine=R.ENGINE_PERSISTENT)
        k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
        noise = WL.noise(wl)
        ref = _oracle(wl, wf, kf, vf, vnp, noise)
        out = m.sample(noise, k, v, valid)
        assert_actions_close(out, ref, wl.name)
        assert R.rtvla_kernels_per_call(m.ctx, 1) == 1
        m.close()


def test_bounded_waits_report_a_timeout_and_the_context_recovers():
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert)
    wf = WL.as_f32(bits)
    m = GpuModel(wl, bits, engine=R.ENGINE_PERSISTENT)
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise_np = WL.noise(wl)
    noise = torch.from_numpy(noise_np).cuda()
    out = torch.empty_like(noise)
    kv = R.make_kv(k, v, valid, 1, wl.prefix_cap)
    R.rtvla_set_wait_timeout_us(m.ctx, 1)          # every grid barrier gives up after 1 us
    R.rtvla_sample_actions(m.ctx, noise, kv, out)
    assert R.STATUS[R.rtvla_sync_status(m.ctx)] == "RTVLA_ERR_DEVICE_TIMEOUT"
    R.rtvla_set_wait_timeout_us(m.ctx, 2_000_000)
    got = m.sample(noise_np, k, v, valid)
    assert_actions_close(got, _oracle(wl, wf, kf, vf, vnp, noise_np), "after timeout")
    m.close()


def test_host_buffer_entry_point_matches_device_entry_point():
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert, stressed=True)
    m = GpuModel(wl, bits)
    kb, vb, valid = WL.kv_cache(wl)
    noise = WL.noise(wl)
    k, v, vd = bf16_dev(kb), bf16_dev(vb), torch.from_numpy(valid).cuda()
    dev_out = m.sample(noise, k, v, vd)
    hk = torch.from_numpy(kb.view(np.int16)).pin_memory()
    hv = torch.from_numpy(vb.view(np.int16)).pin_memory()
    hl = torch.from_numpy(valid).pin_memory()
    hn = torch.from_numpy(noise).pin_memory()
    ho = torch.empty_like(hn).pin_memory()
    R.rtvla_sample_actions_host(m.ctx, hn, hk, hv, hl, wl.batch, wl.prefix_cap, ho)
    assert R.rtvla_sync_status(m.ctx) == 0
    ref = O.sample_actions(WL.as_f32(bits), wl.expert, noise, gen.bf16_to_f32(kb), gen.bf16_to_f32(vb), valid)
    assert_actions_close(ho.numpy(), ref, "host entry point")
    assert np.abs(ho.numpy() - dev_out).max() <= 1e-2
    m.close()


@pytest.fixture(scope="module")
def e2e():
    wl = WL.workload(5)
    ebits = WL.expert_weights(wl.expert)
    pbits = WL.prefill_weights(wl.prefill)
    m = GpuModel(wl, ebits, prefill_bits=pbits)
    emb, mask = WL.prefill_inputs(wl)
    Kr, Vr, vr = O.prefill(WL.as_f32(pbits), wl.prefill, gen.bf16_to_f32(emb), mask)
    yield wl, m, ebits, emb, mask, Kr, Vr, vr
    m.close()


def test_prefill_kv_parity(e2e):
    wl, m, ebits, emb, mask, Kr, Vr, vr = e2e
    k, v, valid = m.prefill(emb, mask)
    assert R.rtvla_sync_status(m.ctx) == 0
    np.testing.assert_array_equal(valid.cpu().numpy(), vr)
    kg, vg = k.float().cpu().numpy(), v.float().cpu().numpy()
    for b, n in enumerate(vr):
        for l in range(wl.prefill.n_layers):
            rk = rel_l2(kg[l, b, :n], Kr[l, b, :n])
            rv = rel_l2(vg[l, b, :n], Vr[l, b, :n])
            assert rk <= KV_REL_L2 and rv <= KV_REL_L2, (l, rk, rv)


def test_end_to_end_prefill_then_denoise(e2e):
    wl, m, ebits, emb, mask, Kr, Vr, vr = e2e
    k, v, valid = m.prefill(emb, mask)
    noise = WL.noise(wl)
    out = m.sample(noise, k, v, valid)
    ref = O.sample_actions(WL.as_f32(ebits), wl.expert, noise, Kr, Vr, vr)
    assert_actions_close(out, ref, "e2e")


def test_device_errors_are_reported_not_fatal():
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert)
    m = GpuModel(wl, bits)
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise = torch.from_numpy(WL.noise(wl)).cuda()
    out = torch.empty_like(noise)
    bad = torch.tensor([wl.prefix_cap + 5], dtype=torch.int32, device="cuda")
    R.rtvla_sample_actions(m.ctx, noise, R.make_kv(k, v, bad, 1, wl.prefix_cap), out)
    assert R.STATUS[R.rtvla_sync_status(m.ctx)] == "RTVLA_ERR_DEVICE_BOUNDS"
    assert R.rtvla_sync_status(m.ctx) == 0          # cleared, context still usable
    R.rtvla_sample_actions(m.ctx, noise, R.make_kv(k, v, valid, 1, wl.prefix_cap), out)
    assert R.rtvla_sync_status(m.ctx) == 0
    with pytest.raises(R.RtvlaError) as ei:
        R.rtvla_sample_actions(m.ctx, noise, R.make_kv(k, v, valid, 2, wl.prefix_cap), out)
    assert ei.value.name == "RTVLA_ERR_SHAPE"
    m.close()


def test_prefill_rejects_a_mask_that_is_not_a_prefix(e2e):
    wl, m, ebits, emb, mask, Kr, Vr, vr = e2e
    bad = mask.copy()
    bad[0, 3] = 0
    m.prefill(emb, bad)
    assert R.STATUS[R.rtvla_sync_status(m.ctx)] == "RTVLA_ERR_MASK_NOT_PREFIX"
    assert R.rtvla_sync_status(m.ctx) == 0
