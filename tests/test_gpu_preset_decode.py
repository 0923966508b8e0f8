"""GPU parity of the preset-format decode products (rq_gemv_p8_g16,
rq_gemv_p4a_g32) against the oracle's fp64 products, through the C ABI.

The weights come from the ORACLE's quantizers (so these tests do not depend on
the GPU quantizers); every output, or sampled outputs at the full projection
sizes, must satisfy |y_gpu - y_ref| <= 2e-3 * sum_k |x_k||w_hat_k|, the
tolerance of the group-64 products.  The kernel's own error is far smaller:
each group's sum of x * code is exact up to fp32 rounding of sums of size
~1000 |x| (the biased codes), and the scale and offset are applied in fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_quantized_g64_b200 import build as rq_build
from weight_only_quantized_g64_b200 import rq, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rq_build.build()
    rq.lib()
    rq.set_pdl(False)
    yield
    assert rq.read_device_status(reset=True) == rq.OK


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def quantized(fmt, N, K, seed):
    """Oracle-quantized preset weights of a synthetic W [N, K] (RTN)."""
    W = synth.weights(N, K, seed=seed).numpy()
    if fmt == "p8":
        codes, scales, _, st = oracle.quantize_sym(W, 8, 16)
        assert st == 0
        return codes, (scales,)
    codes, sub, sup, _, st = oracle.quantize_p4a(W)
    assert st == 0
    return codes, (sub, sup)


def run(fmt, x, codes, meta, N):
    if fmt == "p8":
        return rq.gemv_p8_g16(x, dev(codes), dev(meta[0].view(np.int16)), N)
    return rq.gemv_p4a_g32(x, dev(codes), dev(meta[0]), dev(meta[1].view(np.int16)), N)


def reference(fmt, x_np, codes, meta, ms=None, ns=None):
    if fmt == "p8":
        return oracle.matmul_fmt(8, x_np, codes, meta[0], ms=ms, ns=ns)
    return oracle.matmul_fmt(4, x_np, codes, meta[0], meta[1], ms=ms, ns=ns)


def check(y, y_ref, bound, what):
    diff = np.abs(y.astype(np.float64) - y_ref)
    bad = diff > TOL * bound
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs out of tolerance (worst {diff.max():.3e})"


SHAPES = {
    # (N, K): one row; a ragged tail of rows; several slots per row; exactly
    # one m-tile per SM; a ragged N over many blocks
    "p8": [(1, 128), (37, 640), (300, 2560), (2368, 2048), (5000, 1024)],
    "p4a": [(1, 256), (37, 768), (300, 2560), (2368, 2048), (5000, 1024)],
}


@pytest.mark.parametrize("fmt", ["p8", "p4a"])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_all_outputs(fmt, M):
    for i, (N, K) in enumerate(SHAPES[fmt]):
        codes, meta = quantized(fmt, N, K, seed=100 * i + N)
        x = synth.activations(M, K, seed=7 * M + i, device="cuda")
        y = run(fmt, x, codes, meta, N)
        torch.cuda.synchronize()
        y_ref, bound = reference(fmt, x.cpu().numpy(), codes, meta)
        check(y.cpu().numpy(), y_ref, bound, f"{fmt} M={M} {N}x{K}")


@pytest.mark.parametrize("fmt", ["p8", "p4a"])
def test_massive_channel_and_determinism(fmt):
    """One input channel 100x the rest (the 2.9B model's outlier channel):
    still within tolerance, and two launches give identical bits."""
    N, K = 2560, 2560
    codes, meta = quantized(fmt, N, K, seed=31)
    for M in (1, 8, 32):
        x = synth.activations(M, K, seed=M, device="cuda", massive_channel=517)
        y1 = run(fmt, x, codes, meta, N)
        y2 = run(fmt, x, codes, meta, N)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
        y_ref, bound = reference(fmt, x.cpu().numpy(), codes, meta)
        check(y1.cpu().numpy(), y_ref, bound, f"{fmt} massive M={M}")


@pytest.mark.parametrize("fmt,D", [("p8", 2560), ("p4a", 2048)])
def test_layer_shapes_sampled(fmt, D):
    """Every projection shape of the 2.9B (int8 preset) and 1.5B (int4
    preset) layers at full size, and a 16384 x 4096 projection whose CTAs
    each take several row blocks: 256 sampled outputs per shape and M."""
    shapes = [(D, D), (4 * D, D), (D, 4 * D), (16384, 4096)]
    for si, (N, K) in enumerate(shapes):
        codes, meta = quantized(fmt, N, K, seed=1000 + si)
        for M in (1, 16, 32):
            x = synth.activations(M, K, seed=si + M, device="cuda")
            y = run(fmt, x, codes, meta, N)
            torch.cuda.synchronize()
            rng = np.random.default_rng(si * 100 + M)
            ms = np.concatenate([[0, M - 1], rng.integers(0, M, 254)])
            ns = np.concatenate([[0, N - 1], rng.integers(0, N, 254)])
            y_ref, bound = reference(fmt, x.cpu().numpy(), codes, meta, ms=ms, ns=ns)
            check(y.cpu().numpy()[ms, ns], y_ref, bound, f"{fmt} {N}x{K} M={M}")


def test_nonfinite_scale_propagates():
    """A super-block written as non-finite by the quantizer (ds = dm = NaN)
    makes every output of its row NaN; the other rows stay finite."""
    N, K = 40, 512
    W = synth.weights(N, K, seed=5).numpy()
    W[7, 300] = np.nan
    codes, sub, sup, _, st = oracle.quantize_p4a(W)
    assert st == oracle.STATUS_NONFINITE
    x = synth.activations(2, K, seed=3, device="cuda")
    y = rq.gemv_p4a_g32(x, dev(codes), dev(sub), dev(sup.view(np.int16)), N)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    assert np.isnan(y[:, 7]).all()
    assert np.isfinite(np.delete(y, 7, axis=1)).all()
    assert rq.read_device_status(reset=True) == rq.OK
