"""GPU parity of the decode variants: fp16 output and the fused squared-ReLU
epilogue (rq_gemv_wq_ex), and R/K/V with one input each (rq_rkv_fused3),
against the oracle through the C ABI.

Budgets: the product keeps |y - y_ref| <= delta = 2e-3 * sum_k |x||w_hat|;
the epilogue max(y, 0)^2 turns that into delta * (2 relu(y_ref) + delta)
(oracle.relu_sq_budget); an fp16 output adds its rounding, 2^-11 of the
value (plus 2^-25 absolute for fp16 subnormals).
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
    assert rq.read_device_status(reset=True) == rq.OK


def case(N, K, bits, M, seed):
    W = synth.weights(N, K, seed=seed)
    x = synth.activations(M, K, seed=seed, device="cuda")
    codes, scales, st = oracle.quantize_g64(W.numpy(), bits)
    assert st == 0
    return x, codes, scales


def up(codes, scales):
    return torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda()


def check(y, ref, budget, half, what):
    y = y.float().cpu().numpy().astype(np.float64)
    lim = budget + (np.abs(ref) + budget) * (2.0 ** -11 if half else 0.0) + (2.0 ** -25 if half else 0.0)
    d = np.abs(y - ref)
    assert np.all(d <= lim), f"{what}: worst {d.max():.3e} (limit {lim.flat[d.argmax()]:.3e})"


@pytest.mark.parametrize("kernel", ["rowblock", "tensor"])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 3, 8, 13, 17, 32])
@pytest.mark.parametrize("N,K", [(300, 640), (256, 2048), (129, 128)])
@pytest.mark.parametrize("out,epi", [(torch.float32, 1), (torch.float16, 0), (torch.float16, 1)])
def test_gemv_ex(kernel, bits, M, N, K, out, epi):
    x, codes, scales = case(N, K, bits, M, seed=4000 + M + N + K)
    cd, sd = up(codes, scales)
    with rq.decode_kernel(kernel):
        y = rq.gemv_wq_ex(x, cd, sd, N, bits, out_dtype=out, epilogue=epi)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul(x.cpu().numpy(), codes, scales, bits)
    delta = TOL * bound
    if epi == rq.EPI_RELU_SQ:
        ref, budget = oracle.relu_sq(y_ref), oracle.relu_sq_budget(y_ref, delta)
        assert np.all(y.float().cpu().numpy() >= 0)
    else:
        ref, budget = y_ref, delta
    check(y, ref, budget, out == torch.float16, f"gemv_ex bits={bits} M={M} N={N} K={K} {out} epi={epi}")


def test_gemv_ex_plain_matches_gemv():
    """No epilogue, fp32 out: the same values as rq_gemv_wq on the row-block kernel."""
    x, codes, scales = case(512, 1024, 4, 8, seed=41)
    cd, sd = up(codes, scales)
    with rq.decode_kernel("rowblock"):
        y1 = rq.gemv_wq_ex(x, cd, sd, 512, 4)
        y2 = rq.gemv_wq(x, cd, sd, 512, 4)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("kernel", ["rowblock", "tensor"])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8, 16, 32])
@pytest.mark.parametrize("out", [torch.float32, torch.float16])
def test_rkv_fused3(kernel, bits, M, out):
    N, K = 200, 512
    cases = [case(N, K, bits, M, seed=5000 + 10 * i + M) for i in range(3)]
    ws = [up(c[1], c[2]) for c in cases]
    with rq.decode_kernel(kernel):
        ys = rq.rkv_fused3(cases[0][0], cases[1][0], cases[2][0], ws[0], ws[1], ws[2], N, bits,
                           out_dtype=out)
    torch.cuda.synchronize()
    for i in range(3):
        y_ref, bound = oracle.matmul(cases[i][0].cpu().numpy(), cases[i][1], cases[i][2], bits)
        check(ys[i], y_ref, TOL * bound, out == torch.float16, f"rkv3[{i}] bits={bits} M={M}")


def test_key_relu_sq_feeds_value():
    """The channel-mix chain of a 1.5B-shaped block: key (2048 -> 8192) with the
    fused squared ReLU and fp16 output feeds the value projection (8192 ->
    2048) directly; checked against the oracle's chain on the GPU's fp16 k."""
    D, M, bits = 2048, 4, 4
    Wk = synth.weights(4 * D, D, seed=61, device="cuda")
    Wv = synth.weights(D, 4 * D, seed=62, device="cuda")
    qk = rq.quantize_g64(Wk, bits)
    qv = rq.quantize_g64(Wv, bits)
    x = synth.activations(M, D, seed=63, device="cuda")
    k = rq.gemv_wq_ex(x, qk[0], qk[1], 4 * D, bits, out_dtype=torch.float16, epilogue=rq.EPI_RELU_SQ)
    v = rq.gemv_wq(k, qv[0], qv[1], D, bits)
    torch.cuda.synchronize()
    ck, sk = qk[0].cpu().numpy(), qk[1].cpu().numpy().view(np.uint16)
    cv, sv = qv[0].cpu().numpy(), qv[1].cpu().numpy().view(np.uint16)
    yk, bk = oracle.matmul(x.cpu().numpy(), ck, sk, bits)
    check(k, oracle.relu_sq(yk), oracle.relu_sq_budget(yk, TOL * bk), True, "key relu^2")
    yv, bv = oracle.matmul(k.cpu().numpy(), cv, sv, bits)
    check(v, yv, TOL * bv, False, "value")
