"""The byte accounting behind every GB/s figure: the algorithmic bytes of each
workload (codes plus fp16 scales, each streamed once) against values worked
out independently from the format -- 0.53125 bytes per int4 weight, 1.03125
per int8 weight -- and the workload shapes."""
import pytest

from weight_only_quantized_g64_b200 import synth


def layer_bytes(wl):
    return sum(synth.algorithmic_weight_bytes(p.N, p.K, wl.bits) for p in wl.projs)


def test_bytes_per_weight():
    assert synth.algorithmic_weight_bytes(64, 64, 4) == 64 * 64 * 0.53125
    assert synth.algorithmic_weight_bytes(64, 64, 8) == 64 * 64 * 1.03125


@pytest.mark.parametrize("wl,per_layer,per_pass", [
    (1, 313_344, 313_344),                       # 768 x 768 int4
    (2, 26_738_688, 641_728_512),                # D = 2048 int4: 12 D^2 weights, 24 layers
    (3, 81_100_800, 2_595_225_600),              # D = 2560 int8: 12 D^2 weights, 32 layers
    (5, 106_954_752, 6_524_239_872),             # D = 4096 int4: 12 D^2 weights, 61 layers
])
def test_workload_bytes(wl, per_layer, per_pass):
    w = synth.WORKLOADS[wl]
    assert layer_bytes(w) == per_layer
    assert w.layers * layer_bytes(w) == per_pass
    # 12 D^2 weights per layer: R, K, V, O (4 D^2) plus the channel-mix key and value (8 D^2)
    if wl != 1:
        D = w.projs[0].N
        bpw = 0.53125 if w.bits == 4 else 1.03125
        assert per_layer == 12 * D * D * bpw
