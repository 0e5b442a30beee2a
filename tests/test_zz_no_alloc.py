"""The allocation-free host-buffer call, rtvla_sample_actions_host_static.

It exists for callers that must not allocate device memory after start-up: a robot control
loop with a fixed period, where cudaMalloc could block and synchronise the device, and hosts
that fix device-memory budgets up front.  It stages through the library's fixed 32 MiB
device array instead of the buffers rtvla_sample_actions_host allocates on first use.

Checked here through the C ABI, on both engines:
  * AUTO at batch 1 runs the persistent kernel: two static calls in a row agree with the
    existing host-buffer call within the repeat spread and with the fp64 oracle within the
    parity tolerance;
  * LAYERED: the first two static calls run before any graph exists for the shape (direct
    launches); then rtvla_sample_actions captures the graph (rtvla_kernels_per_call > 1),
    and a third static call replays it; all three agree with the existing call and the
    oracle;
  * a request larger than the array is refused with RTVLA_ERR_SHAPE before anything is
    copied.
This file is collected last so that a stop at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import flow_matching_action_expert_b200 as R
from oracle import model as O
from synth import gen
from synth import workloads as WL

from harness import GpuModel, assert_actions_close, bf16_dev

pytestmark = pytest.mark.gpu

# Repeated calls differ only by the fp32 reduction order of split-K partials, which can flip
# a later bf16 rounding; on this stressed 2-layer workload (AdaRMS gates 1) the loop carries
# such flips to a measured max-abs spread of 3.8e-3 on B200, so calls are compared within
# 1e-2, and each also with the oracle.
REPEAT_TOL = 1e-2


def _pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


def _static(m, args, hn):
    o = torch.empty_like(hn).pin_memory()
    R.rtvla_sample_actions_host_static(m.ctx, *args, o)
    return o.numpy().copy()


@pytest.mark.parametrize("engine", ["auto", "layered"])
def test_static_staging_call_matches_existing_call_and_oracle(engine):
    wl = WL.workload(1)
    bits = WL.expert_weights(wl.expert, stressed=True)
    eng = R.ENGINE_AUTO if engine == "auto" else R.ENGINE_LAYERED
    m = GpuModel(wl, bits, max_batch=64, engine=eng)
    kb, vb, valid = WL.kv_cache(wl)
    noise = WL.noise(wl)
    hk, hv = _pinned(kb.view(np.int16)), _pinned(vb.view(np.int16))
    hl, hn = _pinned(valid), _pinned(noise)
    args = (hn, hk, hv, hl, wl.batch, wl.prefix_cap)
    ref = O.sample_actions(WL.as_f32(bits), wl.expert, noise, gen.bf16_to_f32(kb), gen.bf16_to_f32(vb), valid)

    outs = [_static(m, args, hn) for _ in range(2)]           # two calls in a row
    existing = torch.empty_like(hn).pin_memory()
    R.rtvla_sample_actions_host(m.ctx, *args, existing)       # the existing entry point
    existing = existing.numpy()
    if engine == "layered":
        # the device call captures the layered graph for (batch 1, this cache); the next
        # static call replays it
        x = torch.from_numpy(noise).cuda()
        y = torch.empty_like(x)
        kv = R.make_kv(bf16_dev(kb), bf16_dev(vb), torch.from_numpy(valid).cuda(), 1, wl.prefix_cap)
        R.rtvla_sample_actions(m.ctx, x, kv, y)
        assert R.rtvla_sync_status(m.ctx) == 0
        assert R.rtvla_kernels_per_call(m.ctx, 1) > 1
        outs.append(_static(m, args, hn))
    else:
        assert R.rtvla_kernels_per_call(m.ctx, 1) == 1        # the persistent kernel
    assert R.rtvla_sync_status(m.ctx) == 0
    assert np.isfinite(existing).all()
    for i, out in enumerate(outs):
        d = float(np.abs(out - existing).max())
        assert d <= REPEAT_TOL, f"{engine} static call {i}: max-abs {d:.3e} from the existing host call"
        assert_actions_close(out, ref, f"{engine} static call {i} vs oracle")

    # larger than the fixed array (64 samples x 2 layers x 272 tokens x K and V): refused
    big = WL.Workload("big", wl.expert, wl.chunk, 64, wl.prefix_cap, tuple([268] * 64))
    bk, bv, bl = WL.kv_cache(big)
    bn = WL.noise(big)
    bo = np.empty_like(bn)
    with pytest.raises(R.RtvlaError) as e:
        R.rtvla_sample_actions_host_static(m.ctx, torch.from_numpy(bn), torch.from_numpy(bk.view(np.int16)),
                                           torch.from_numpy(bv.view(np.int16)), torch.from_numpy(bl), 64,
                                           wl.prefix_cap, torch.from_numpy(bo))
    assert e.value.name == "RTVLA_ERR_SHAPE"
    m.close()
