"""The tcgen05 attention kernel of the layered engine (k_attn_tc), which serves calls with at
least 64 (sample, 16-query block) units: ragged valid prefix lengths on both sides of every
64-key chunk boundary (0, 1, 63, 64, 65, ..., the whole cache), a suffix of 63 keys (one
chunk) and of 65 keys (a chunk of 64 and a chunk of 1), padded cache slots filled with 3e4,
and the stressed 2-layer expert (AdaRMS gate 1), against the fp64 oracle.
"""
import pytest

from oracle import model as O
from synth import workloads as WL

from harness import GpuModel, assert_actions_close, device_kv

pytestmark = pytest.mark.gpu

LENS_16 = (0, 1, 7, 63, 64, 65, 127, 128, 129, 200, 13, 190, 64, 1, 0, 150)


@pytest.mark.parametrize("chunk, batch", [(63, 16), (65, 13)])
def test_tc_attention_ragged_lengths_and_chunk_edges(chunk, batch):
    base = WL.workload(1)
    bits = WL.expert_weights(base.expert, stressed=True)
    lens = LENS_16[:batch]
    assert batch * ((chunk + 15) // 16) >= 64  # the tcgen05 kernel serves this call
    wl = WL.Workload(f"tc attention C{chunk} B{batch}", base.expert, chunk, batch, 200, lens)
    m = GpuModel(wl, bits, max_batch=batch)
    k, v, valid, kf, vf, vnp = device_kv(wl, pad_fill=3.0e4)
    noise = WL.noise(wl)
    ref = O.sample_actions(WL.as_f32(bits), wl.expert, noise, kf, vf, vnp)
    out = m.sample(noise, k, v, valid)
    assert_actions_close(out, ref, wl.name)
    m.close()
