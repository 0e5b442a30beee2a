"""Checked mode and the capped allocator, on the GPU.

Checked mode (RTVLA_CHECKED=1 at rtvla_create) places every library buffer between guard
bands and verifies them in rtvla_sync_status; it stands in for an out-of-bounds / race
detector.  The bands must survive every engine (persistent kernel, layered graph at batch 1
and at a ragged batch, the batch-16 kernels: tcgen05 attention and the gated-GELU GEMM, π0 on
both engines) and the prefix pass, and a planted overwrite past the residual-stream buffer
must be reported as RTVLA_ERR_GUARD_OVERWRITE, after which the context still works.

RTVLA_DEVICE_MEMORY_CAP caps the context's device memory: rtvla_create must then return
RTVLA_ERR_OOM and free everything it had allocated.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import flow_matching_action_expert_b200 as R
from oracle import model as O
from synth import gen
from synth import workloads as WL

from harness import GpuModel, assert_actions_close, device_kv

pytestmark = pytest.mark.gpu


def test_guard_bands_hold_on_every_engine_and_catch_a_planted_overwrite(monkeypatch):
    monkeypatch.setenv("RTVLA_CHECKED", "1")
    base = WL.workload(1)
    wl = WL.Workload("checked L2 P272 C10 B2", base.expert, base.chunk, 2, base.prefix_cap, (268, 200),
                     prefill=WL.PrefillShape(n_layers=base.expert.n_layers))
    ebits = WL.expert_weights(wl.expert, stressed=True)
    pbits = WL.prefill_weights(wl.prefill)
    m = GpuModel(wl, ebits, prefill_bits=pbits)
    wf = WL.as_f32(ebits)
    # the prefix pass over a ragged batch
    emb, mask = WL.prefill_inputs(wl)
    k, v, valid = m.prefill(emb, mask)
    assert R.rtvla_sync_status(m.ctx) == 0
    # the denoise loop: ragged batch 2 (layered), then batch 1 on both engines
    noise = WL.noise(wl)
    kn, vn = k.float().cpu().numpy(), v.float().cpu().numpy()
    vnp = valid.cpu().numpy()
    out = m.sample(noise, k, v, valid)
    assert_actions_close(out, O.sample_actions(wf, wl.expert, noise, kn, vn, vnp), "checked B2")
    for eng in (R.ENGINE_PERSISTENT, R.ENGINE_LAYERED):
        R.rtvla_set_engine(m.ctx, eng)
        out1 = m.sample(noise[:1], k[:, :1].contiguous(), v[:, :1].contiguous(), valid[:1].contiguous())
        assert_actions_close(out1, O.sample_actions(wf, wl.expert, noise[:1], kn[:, :1], vn[:, :1], vnp[:1]),
                             f"checked B1 engine {eng}")
    # a planted write past the end of a buffer is reported once, then the bands are whole
    R.rtvla_debug_plant_guard_fault(m.ctx)
    assert R.STATUS[R.rtvla_sync_status(m.ctx)] == "RTVLA_ERR_GUARD_OVERWRITE"
    assert R.rtvla_sync_status(m.ctx) == 0
    out2 = m.sample(noise, k, v, valid)
    assert_actions_close(out2, O.sample_actions(wf, wl.expert, noise, kn, vn, vnp), "checked B2 after the plant")
    m.close()


def test_guard_bands_hold_on_the_batched_layered_kernels(monkeypatch):
    # batch 16 x chunk 63: the tcgen05 attention (64 sample x query-block units) and the
    # gated-GELU gate/up GEMM (K kept whole), over ragged lengths with garbage in the padding
    monkeypatch.setenv("RTVLA_CHECKED", "1")
    base = WL.workload(1)
    lens = (0, 1, 7, 63, 64, 65, 127, 128, 129, 200, 13, 190, 64, 1, 0, 150)
    wl = WL.Workload("checked L2 P200 C63 B16", base.expert, 63, 16, 200, lens)
    bits = WL.expert_weights(wl.expert, stressed=True)
    m = GpuModel(wl, bits)
    k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
    noise = WL.noise(wl)
    out = m.sample(noise, k, v, valid)
    assert R.rtvla_sync_status(m.ctx) == 0
    assert_actions_close(out, O.sample_actions(WL.as_f32(bits), wl.expert, noise, kf, vf, vnp), wl.name)
    m.close()


def test_guard_bands_hold_on_the_pi0_engines(monkeypatch):
    # π0 (state token + action-time output linear) on the persistent kernel and the layered graph
    monkeypatch.setenv("RTVLA_CHECKED", "1")
    wl = WL.workload(1)
    bits = WL.pi0_expert_weights(wl.expert, bias_std=0.02)
    wf = WL.as_f32(bits)
    k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
    noise, state = WL.noise(wl), WL.state(wl)
    ref = O.pi0_sample_actions(wf, wl.expert, noise, state, kf, vf, vnp)
    for eng in (R.ENGINE_PERSISTENT, R.ENGINE_LAYERED):
        m = GpuModel(wl, bits, engine=eng, variant=R.VARIANT_PI0)
        out = m.sample_pi0(noise, state, k, v, valid)
        assert R.rtvla_sync_status(m.ctx) == 0
        assert_actions_close(out, ref, f"checked π0 engine {eng}")
        m.close()


def test_plant_hook_needs_checked_mode(monkeypatch):
    monkeypatch.delenv("RTVLA_CHECKED", raising=False)
    wl = WL.workload(1)
    m = GpuModel(wl, WL.expert_weights(wl.expert))
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_debug_plant_guard_fault(m.ctx)
    assert e.value.name == "RTVLA_ERR_UNSUPPORTED"
    m.close()


def test_device_memory_cap_gives_oom_and_frees_everything(monkeypatch):
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert)
    dev = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in bits.items()}
    cfg = R.make_config(n_layers=wl.expert.n_layers, chunk=wl.chunk, max_prefix=wl.prefix_cap, max_batch=1)
    monkeypatch.delenv("RTVLA_DEVICE_MEMORY_CAP", raising=False)
    R.rtvla_destroy(R.rtvla_create(dev, cfg))     # loads the library's module (static arrays) first
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for cap in (1 << 20, 64 << 20):               # fails at the first buffer / part-way through
        monkeypatch.setenv("RTVLA_DEVICE_MEMORY_CAP", str(cap))
        with pytest.raises(R.RtvlaError) as e:
            R.rtvla_create(dev, cfg)
        assert e.value.name == "RTVLA_ERR_OOM"
        torch.cuda.synchronize()
        assert abs(torch.cuda.mem_get_info()[0] - free0) <= (4 << 20), "memory of the failed create leaked"
    monkeypatch.delenv("RTVLA_DEVICE_MEMORY_CAP")
    ctx = R.rtvla_create(dev, cfg)                # without the cap the same create succeeds
    R.rtvla_destroy(ctx)
