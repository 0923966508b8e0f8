"""GPU parity of the preset-format quantizers (rq_quantize_p8_g16,
rq_quantize_p4a_g32) against the oracle, through the C ABI: codes, scales,
sub-codes, super-scales, choices and status bit-exact, with and without the
E[x^2]-weighted search, on random shapes, special values and the 1.5B/2.9B
projection shapes (sampled rows at full size)."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_quantized_g64_b200 import build as rq_build
from weight_only_quantized_g64_b200 import rq, synth

pytestmark = pytest.mark.gpu
FACTORS = [1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rq_build.build()
    rq.lib()
    yield
    assert rq.read_device_status(reset=True) == rq.OK


def e2_for(K, seed):
    rng = np.random.default_rng(seed)
    return (10.0 ** rng.uniform(-2.0, 2.0, K)).astype(np.float32)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("search", [False, True])
@pytest.mark.parametrize("N,K", [(1, 64), (37, 640), (300, 2560), (64, 4096)])
def test_p8_bit_exact(search, N, K):
    W = synth.weights(N, K, seed=N + K).numpy()
    e2 = e2_for(K, K) if search else None
    c_ref, s_ref, ch_ref, st_ref = oracle.quantize_sym(W, 8, 16, e2, FACTORS)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c, s, ch = rq.quantize_p8_g16(dev(W), dev(e2) if search else None,
                                  dev(np.array(FACTORS, np.float32)) if search else None, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == st_ref
    assert np.array_equal(c.cpu().numpy(), c_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_ref)
    assert np.array_equal(ch.cpu().numpy(), ch_ref)


@pytest.mark.parametrize("search", [False, True])
@pytest.mark.parametrize("N,K", [(1, 256), (37, 768), (300, 2048), (64, 4096)])
def test_p4a_bit_exact(search, N, K):
    W = synth.weights(N, K, seed=2 * N + K).numpy()
    W[0, :32] = 0.03 + np.abs(W[0, :32])              # a group with no negative weight
    e2 = e2_for(K, K + 1) if search else None
    c_ref, sub_ref, sup_ref, ch_ref, st_ref = oracle.quantize_p4a(W, e2, FACTORS)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c, sub, sup, ch = rq.quantize_p4a_g32(dev(W), dev(e2) if search else None,
                                          dev(np.array(FACTORS, np.float32)) if search else None,
                                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == st_ref
    assert np.array_equal(c.cpu().numpy(), c_ref)
    assert np.array_equal(sub.cpu().numpy(), sub_ref)
    assert np.array_equal(sup.cpu().numpy().view(np.uint16), sup_ref)
    assert np.array_equal(ch.cpu().numpy(), ch_ref)


def test_special_values():
    K = 512
    W = synth.weights(6, K, seed=9).numpy()
    W[0, :64] = 0.0
    W[1, 70] = np.nan
    W[2, 300] = -np.inf
    W[3, 5] = 3e7                  # p8: 3e7/127 overflows fp16; p4a: ds overflows
    W[4, 256:288] = -0.0
    for fn in ("p8", "p4a"):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if fn == "p8":
            ref = oracle.quantize_sym(W, 8, 16)
            got = rq.quantize_p8_g16(dev(W), dev_status=st)
            pairs = [(got[0], ref[0]), (got[1], ref[1]), (got[2], ref[2])]
            st_ref = ref[3]
        else:
            ref = oracle.quantize_p4a(W)
            got = rq.quantize_p4a_g32(dev(W), dev_status=st)
            pairs = [(got[0], ref[0]), (got[1], ref[1]), (got[2], ref[2]), (got[3], ref[3])]
            st_ref = ref[4]
        torch.cuda.synchronize()
        assert int(st.item()) == st_ref == oracle.STATUS_NONFINITE
        for g, r in pairs:
            g = g.cpu().numpy()
            assert np.array_equal(g.view(r.dtype) if g.dtype.itemsize == r.dtype.itemsize else g, r), fn


@pytest.mark.parametrize("fmt,wl", [("p8", 3), ("p4a", 2)])
def test_workload_shapes_sampled(fmt, wl):
    """Every projection shape of the 2.9B (int8 preset) / 1.5B (int4 preset)
    layers at full size, sampled rows checked against the oracle."""
    w = synth.WORKLOADS[wl]
    for pi, pj in enumerate(w.projs):
        W = synth.weights(pj.N, pj.K, seed=synth.seed_for(wl, 0, pi), device="cuda")
        rows = np.unique(np.concatenate([[0, pj.N - 1], np.random.default_rng(pi).integers(0, pj.N, 24)]))
        Wr = W[torch.from_numpy(rows).cuda()].cpu().numpy()
        idx = torch.from_numpy(rows).cuda()
        if fmt == "p8":
            c, s, _ = rq.quantize_p8_g16(W)
            c_ref, s_ref, _, st = oracle.quantize_sym(Wr, 8, 16)
            torch.cuda.synchronize()
            assert st == 0
            assert np.array_equal(c[idx].cpu().numpy(), c_ref)
            assert np.array_equal(s[idx].cpu().numpy().view(np.uint16), s_ref)
        else:
            c, sub, sup, _ = rq.quantize_p4a_g32(W)
            c_ref, sub_ref, sup_ref, _, st = oracle.quantize_p4a(Wr)
            torch.cuda.synchronize()
            assert st == 0
            assert np.array_equal(c[idx].cpu().numpy(), c_ref)
            assert np.array_equal(sub[idx].cpu().numpy(), sub_ref)
            assert np.array_equal(sup[idx].cpu().numpy().view(np.uint16), sup_ref)
