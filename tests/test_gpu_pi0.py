"""Parity of the π0 suffix variant (through the C ABI) with the fp64 oracle.

The π0 expert ("Running VLAs at Real-time Speed" summary, section "How"; readings P1-P5 in
oracle/model.py): the suffix is [state token ; C action tokens], the action tokens come from
the action-time MLP (folded with action_in_proj, its time rows tabulated before SiLU), the
norms are plain RMSNorm and the residuals ungated.  Checked on both engines (the persistent
kernel serves batch 1 with chunk + 1 <= 64): the tiny 2-layer expert with biased weights
(actions and every layer's hidden state and update), the full-size 2-view expert (chunk 63,
so 64 suffix tokens); on the layered engine a ragged batch with empty / short / full
prefixes; and the entry points' variant checks.  Tolerances are those of the π0.5 tests.
"""
import numpy as np
import pytest
import torch

import flow_matching_action_expert_b200 as R
from oracle import model as O
from synth import workloads as WL

from harness import GpuModel, assert_actions_close, assert_trace_close, device_kv, O1_REL_L2

pytestmark = pytest.mark.gpu


def _pi0(wl, bias_std=0.02, **kw):
    bits = WL.pi0_expert_weights(wl.expert, bias_std=bias_std)
    return bits, WL.as_f32(bits), GpuModel(wl, bits, variant=R.VARIANT_PI0, **kw)


ENGINES = {"layered": R.ENGINE_LAYERED, "persistent": R.ENGINE_PERSISTENT}


@pytest.mark.parametrize("engine", ["layered", "persistent"])
def test_tiny_pi0_actions_and_layers(engine):
    wl = WL.workload(1)
    bits, wf, m = _pi0(wl, engine=ENGINES[engine])
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise, state = WL.noise(wl), WL.state(wl)
    for step in (0, 9):
        ref, rtr = O.pi0_sample_actions(wf, wl.expert, noise, state, kf, vf, vnp, trace_step=step)
        assert_trace_close(m.trace_pi0(noise, state, k, v, valid, step), rtr, f"tiny π0 step {step}")
    out = m.sample_pi0(noise, state, k, v, valid)
    d, r = assert_actions_close(out, ref, f"tiny π0 {engine}")
    print(f"tiny π0 {engine}: actions max-abs {d:.2e} rel-L2 {r:.2e}, {R.rtvla_kernels_per_call(m.ctx, 1)} kernels per call")
    m.close()


@pytest.mark.parametrize("engine", ["layered", "persistent"])
def test_full_size_pi0_two_view(engine):
    wl = WL.workload(3)
    bits, wf, m = _pi0(wl, engine=ENGINES[engine])
    k, v, valid, kf, vf, vnp = device_kv(wl)
    noise, state = WL.noise(wl), WL.state(wl)
    ref, rtr = O.pi0_sample_actions(wf, wl.expert, noise, state, kf, vf, vnp, trace_step=0)
    out = m.sample_pi0(noise, state, k, v, valid)
    d, r = assert_actions_close(out, ref, f"2-view π0 {engine}")
    wh, wu = assert_trace_close(m.trace_pi0(noise, state, k, v, valid, 0), rtr, f"2-view π0 {engine} step 0",
                                tol=O1_REL_L2)
    print(f"2-view π0 {engine}: actions max-abs {d:.2e} rel-L2 {r:.2e}; worst per-layer rel-L2 h {wh:.2e} update {wu:.2e}")
    m.close()


def test_pi0_ragged_batch():
    base = WL.workload(1)
    wl = WL.Workload("π0 edge B3", base.expert, base.chunk, 3, 130, (0, 7, 130))
    bits, wf, m = _pi0(wl)
    k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
    noise, state = WL.noise(wl), WL.state(wl)
    out = m.sample_pi0(noise, state, k, v, valid)
    assert_actions_close(out, O.pi0_sample_actions(wf, wl.expert, noise, state, kf, vf, vnp), wl.name)
    m.close()


def test_variant_checks_of_the_entry_points():
    wl = WL.workload(1)
    bits, wf, m = _pi0(wl)
    k, v, valid, kf, vf, vnp = device_kv(wl)
    x = torch.from_numpy(WL.noise(wl)).cuda()
    s = torch.from_numpy(WL.state(wl)).cuda()
    out = torch.empty_like(x)
    kv = R.make_kv(k, v, valid, 1, wl.prefix_cap)
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_sample_actions(m.ctx, x, kv, out)           # π0 needs the state
    assert e.value.name == "RTVLA_ERR_INVALID_ARG"
    hk, hv = k.view(torch.int16).cpu(), v.view(torch.int16).cpu()
    with pytest.raises(R.RtvlaError) as e:                  # host-buffer calls carry no state
        R.rtvla_sample_actions_host_static(m.ctx, x.cpu(), hk, hv, valid.cpu(), 1, wl.prefix_cap, out.cpu())
    assert e.value.name == "RTVLA_ERR_INVALID_ARG"
    m.close()
    # chunk 64 makes 65 suffix tokens: more than the persistent kernel's one token tile
    wl64 = WL.Workload("π0 C64", wl.expert, 64, 1, wl.prefix_cap, wl.valid_lens)
    bits64, wf64, m64 = _pi0(wl64, engine=R.ENGINE_PERSISTENT)
    x64 = torch.from_numpy(WL.noise(wl64)).cuda()
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_sample_actions_pi0(m64.ctx, x64, s, kv, torch.empty_like(x64))
    assert e.value.name == "RTVLA_ERR_UNSUPPORTED"
    m64.close()
    m5 = GpuModel(wl, WL.expert_weights(wl.expert))
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_sample_actions_pi0(m5.ctx, x, s, kv, out)   # a π0.5 context has no state input
    assert e.value.name == "RTVLA_ERR_UNSUPPORTED"
    m5.close()
