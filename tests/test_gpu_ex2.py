"""GPU parity of the E[x^2]-weighted scale search (rq_quantize_g64_ex2)
against the oracle, through the C ABI: codes, scales, the chosen candidate and
the device status must be bit-identical (an argmin decides integer codes, so
both sides take the decision in the same fp32 arithmetic)."""
import numpy as np
import pytest
import torch

import oracle
from weight_only_quantized_g64_b200 import build as rq_build
from weight_only_quantized_g64_b200 import rq

pytestmark = pytest.mark.gpu
FACTORS = [1.0, 0.97, 0.94, 0.9, 0.85, 0.8, 0.7]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rq_build.build()
    rq.lib()
    yield


def gpu_ex2(W, e2, bits, factors):
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    ed = torch.from_numpy(np.ascontiguousarray(e2, np.float32)).cuda()
    fd = torch.tensor(factors, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c, s, ch = rq.quantize_g64_ex2(Wd, ed, bits, fd, dev_status=st)
    torch.cuda.synchronize()
    return (c.cpu().numpy(), s.cpu().numpy().view(np.uint16), ch.cpu().numpy(), int(st.item()))


def case(N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0, :64] = 0.0                                       # all-zero group
    if K >= 128:
        W[min(1, N - 1), 64:128] *= 25.0                  # large group
    e2 = rng.gamma(0.7, 1.0, K).astype(np.float32)        # skewed E[x^2]
    e2[5] = 0.0
    W[N - 1, 5] = 0.5                                     # outlier on a zero-weight channel
    return W, e2


def check(W, e2, bits, factors):
    c, s, ch, st = gpu_ex2(W, e2, bits, factors)
    rc, rs, rch, rst = oracle.quantize_g64_ex2(W, e2, bits, factors)
    assert st == rst
    assert np.array_equal(s, rs), "scales differ"
    assert np.array_equal(ch, rch), "choices differ"
    assert np.array_equal(c, rc), "codes differ"
    return ch


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(1, 64), (37, 192), (300, 640), (129, 4096)])
def test_ex2_bit_exact(bits, N, K):
    W, e2 = case(N, K, seed=N + K + bits)
    ch = check(W, e2, bits, FACTORS)
    if N * K >= 64 * 64:
        assert ch.any()


@pytest.mark.parametrize("bits", [4, 8])
def test_ex2_factor_one_is_rtn(bits):
    W, e2 = case(33, 512, seed=5 + bits)
    c, s, ch, st = gpu_ex2(W, e2, bits, [1.0])
    c0, s0 = rq.quantize_g64(torch.from_numpy(W).cuda(), bits)
    torch.cuda.synchronize()
    assert st == 0 and not ch.any()
    assert np.array_equal(c, c0.cpu().numpy())
    assert np.array_equal(s, s0.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("bits", [4, 8])
def test_ex2_special_values(bits):
    W, e2 = case(6, 256, seed=17)
    W[1, 70] = np.nan                       # non-finite group: scale NaN, codes 0, NONFINITE
    W[2, 5] = 1e30                          # huge weight on a zero-weight channel: 0 * inf = NaN errors
    W[3, 128:192] = 0.0
    W[3, 130] = 1e6                         # RTN scale overflows; only small factors stay finite
    check(W, e2, bits, [1.0, 0.9, 0.3, 0.05])
    W2, e22 = case(4, 128, seed=18)
    W2[0, 3] = np.inf
    check(W2, e22, bits, FACTORS)


def test_ex2_hand_group():
    W = np.full((1, 64), 0.36, np.float32)
    W[0, 0] = 0.7
    e2 = np.ones(64, np.float32)
    e2[0] = 0.0
    c, s, ch, st = gpu_ex2(W, e2, 4, [1.0, 0.9])
    assert st == 0 and ch[0, 0] == 1 and s[0, 0] == 0x2DC3
    assert c[0, 0] == 0x47 and np.all(c[0, 1:] == 0x44)
