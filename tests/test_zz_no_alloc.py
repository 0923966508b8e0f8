"""rq_gemv_wq_noalloc: the decode product for callers that cannot have the
library allocate device memory (graph capture, pre-reserved memory budgets,
no implicit synchronisation); its scratch is a fixed array inside librq.

Checked against rq_gemv_wq through the C ABI, within the products' parity
tolerance (|dy| <= 2e-3 * sum_k |x||w_hat|), on two calls in a row -- the
second call finds the first call's leftovers in the shared array.  Kept in a
file that runs last, so a failure here comes after every other test has run.
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
    yield


def _oracle(x, codes, scales, bits):
    """(y, sum_k |x||w_hat|) per output, from the oracle on the host."""
    return oracle.matmul(x.cpu().numpy(), codes.cpu().numpy(),
                         scales.cpu().numpy().view(np.uint16), bits)


@pytest.mark.parametrize("kernel", ["auto", "rowtile", "cluster", "rowblock", "tensor"])
@pytest.mark.parametrize("N,K,M,bits", [(4096, 4096, 1, 4), (2048, 8192, 8, 4),
                                        (300, 640, 17, 4), (2560, 2560, 32, 8),
                                        (129, 128, 3, 8), (4096, 2048, 32, 4)])
def test_noalloc_matches_gemv_two_calls(N, K, M, bits, kernel):
    W = synth.weights(N, K, seed=71 + N + M, device="cuda")
    codes, scales = rq.quantize_g64(W, bits)
    x = synth.activations(M, K, seed=71 + M, device="cuda")
    y1 = torch.full((M, N), float("nan"), device="cuda")
    y2 = torch.full((M, N), float("nan"), device="cuda")
    L = rq.lib()
    s = torch.cuda.current_stream().cuda_stream
    with rq.decode_kernel(kernel):
        y_ref = rq.gemv_wq(x, codes, scales, N, bits)
        for y in (y1, y2):
            st = L.rq_gemv_wq_noalloc(x.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(), N,
                                      bits, y.data_ptr(), s)
            assert st == rq.OK, rq.STATUS[st]
    torch.cuda.synchronize()
    y_or, bound = _oracle(x, codes, scales, bits)
    ref = y_ref.cpu().numpy().astype(np.float64)
    for y in (y1, y2):
        yy = y.cpu().numpy().astype(np.float64)
        d = np.abs(yy - ref)
        assert np.all(d <= TOL * bound), f"vs rq_gemv_wq: max diff {d.max():.3e}"
        d = np.abs(yy - y_or)
        assert np.all(d <= TOL * bound), f"vs oracle: max diff {d.max():.3e}"
    assert rq.read_device_status() == rq.OK


def test_noalloc_rejects_bad_batch():
    """M outside 1..32 is refused before anything is enqueued (the fake
    pointers are never touched).  The scratch bound itself cannot be reached
    on a 148-SM B200: the row-tile kernel needs counters only when it splits
    row tiles across CTAs, which it does only while there are few of them."""
    fake = 1 << 20
    L = rq.lib()
    assert L.rq_gemv_wq_noalloc(fake, 33, 64, fake, fake, 128, 4, fake, None) == rq.ERR_SHAPE
    assert L.rq_gemv_wq_noalloc(fake, 0, 64, fake, fake, 128, 4, fake, None) == rq.ERR_SHAPE


def test_noalloc_tall_projection_on_chip_kernels():
    """N = 262144 + 16 rows at M = 32: the automatic choice runs a kernel that
    keeps its partial sums on chip, so the fixed counters do not limit it;
    checked against rq_gemv_wq and, on sampled outputs, the oracle."""
    N, K, M, bits = 262144 + 16, 64, 32, 4
    W = synth.weights(N, K, seed=91, device="cuda")
    codes, scales = rq.quantize_g64(W, bits)
    x = synth.activations(M, K, seed=91, device="cuda")
    y = torch.full((M, N), float("nan"), device="cuda")
    L = rq.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert rq.decode_kernel_for(M, K, N, bits) != "rowtile"
    st = L.rq_gemv_wq_noalloc(x.data_ptr(), M, K, codes.data_ptr(), scales.data_ptr(), N, bits,
                              y.data_ptr(), s)
    assert st == rq.OK, rq.STATUS[st]
    y_ref = rq.gemv_wq(x, codes, scales, N, bits)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    rng = np.random.default_rng(5)
    ms = rng.integers(0, M, 512)
    ns = np.concatenate([[0, N - 1], rng.integers(0, N, 510)])
    yo, bound = oracle.matmul_sampled(x.cpu().numpy(), codes.cpu().numpy(),
                                      scales.cpu().numpy().view(np.uint16), bits, ms, ns)
    d = np.abs(y.cpu().numpy().astype(np.float64)[ms, ns] - yo)
    assert np.all(d <= TOL * bound)
    assert rq.read_device_status() == rq.OK
