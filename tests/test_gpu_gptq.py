"""GPU parity of GPTQ on the group-64 grid (rq_gptq_hessian, rq_gptq_factor,
rq_gptq_g64) against the oracle, through the C ABI.

  * hessian: H = (2/T) X^T X against numpy fp64 (relative 1e-12: both are
    fp64 sums of exact products, in different orders);
  * factor: U against the oracle's U (numpy fp64 through the method's own
    steps: Cholesky of H, its inverse, the upper Cholesky factor of H^-1),
    within 1e-6 relative after the fp32 rounding of U; dead inputs equal;
  * column loop: given the same fp32 U, codes, scales, status and the
    compensated weights are bit-exact with the oracle's fp32 loop (the kernel
    takes the oracle's operations in the oracle's order);
  * end to end (GPU factor + GPU loop vs oracle factor + oracle loop): at least
    99.5 % of the codes agree and the layer error ||(W - W_hat) X^T|| is within
    1 % (a one-ulp difference in U can move a code at a rounding boundary,
    after which the row's later codes legitimately differ).
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_quantized_g64_b200 import build as rq_build
from weight_only_quantized_g64_b200 import rq, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    rq_build.build()
    rq.lib()
    yield
    assert rq.read_device_status(reset=True) == rq.OK


def calib(T, K, seed, dead=()):
    rng = np.random.default_rng(seed)
    A = np.eye(K) + 1.6 * rng.standard_normal((K, K)) / np.sqrt(K)
    X = (rng.standard_normal((T, K)) @ A).astype(np.float16)
    X[:, list(dead)] = 0
    return X


def unpack(codes, bits, K):
    if bits == 8:
        return codes.view(np.int8).astype(np.int32)
    lo = (codes & 0xF).astype(np.int32)
    hi = (codes >> 4).astype(np.int32)
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


@pytest.mark.parametrize("T,K", [(300, 192), (64, 512), (1000, 1024)])
def test_hessian_matches(T, K):
    X = calib(T, K, seed=T + K)
    H = rq.gptq_hessian(torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    Xd = X.astype(np.float64)
    ref = (2.0 / T) * (Xd.T @ Xd)
    assert np.allclose(H.cpu().numpy(), ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("K,dead", [(128, ()), (256, (3, 200)), (1024, (0, 511, 1023))])
def test_factor_matches_oracle(K, dead):
    X = calib(max(2 * K, 256), K, seed=K, dead=dead)
    U_or, dead_or = oracle.gptq_prepare(X)
    Xd = X.astype(np.float64)
    H = torch.from_numpy((2.0 / X.shape[0]) * (Xd.T @ Xd)).cuda()
    U, dd = rq.gptq_factor(H, oracle.GPTQ_DAMP)
    torch.cuda.synchronize()
    assert np.array_equal(dd.cpu().numpy(), dead_or)
    Ug = U.cpu().numpy().astype(np.float64)
    assert np.all(np.tril(Ug, -1) == 0)
    err = np.abs(Ug - U_or)
    assert np.all(err <= 1e-6 * np.abs(U_or) + 1e-7 * np.abs(U_or).max()), err.max()


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K,dead", [(64, 256, ()), (33, 640, (5, 130)), (129, 128, ()),
                                      (8, 64, ())])
def test_loop_bit_exact(bits, N, K, dead):
    X = calib(512, K, seed=7 + K, dead=dead)
    U_or, dead_or = oracle.gptq_prepare(X)
    U32 = U_or.astype(np.float32)
    W = synth.weights(N, K, seed=N + K).numpy()
    c_ref, s_ref, W_ref, st_ref = oracle.gptq_g64(W, bits, U32, dead_or)
    Wd = torch.from_numpy(W).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = rq.gptq_g64(Wd, bits, torch.from_numpy(U32).cuda(),
                                torch.from_numpy(dead_or).cuda(), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == st_ref == 0
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(Wd.cpu().numpy(), W_ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_loop_special_values(bits):
    K, N = 256, 6
    X = calib(512, K, seed=99)
    U32 = oracle.gptq_prepare(X)[0].astype(np.float32)
    W = synth.weights(N, K, seed=5).numpy()
    W[1, 70] = np.nan          # NONFINITE in group 1 of row 1
    W[3, 200] = 1e6            # RANGE in group 3 of row 3
    W[4, :64] = 0.0            # an all-zero group at its start
    c_ref, s_ref, W_ref, st_ref = oracle.gptq_g64(W, bits, U32)
    Wd = torch.from_numpy(W).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = rq.gptq_g64(Wd, bits, torch.from_numpy(U32).cuda(), dev_status=status)
    torch.cuda.synchronize()
    assert st_ref == oracle.STATUS_NONFINITE == int(status.item())
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    Wg = Wd.cpu().numpy()
    assert np.array_equal(np.isnan(Wg), np.isnan(W_ref))
    assert np.array_equal(np.nan_to_num(Wg), np.nan_to_num(W_ref))


@pytest.mark.parametrize("bits", [4, 8])
def test_end_to_end_close_to_oracle(bits):
    N, K, T = 256, 512, 1024
    X = calib(T, K, seed=123)
    W = synth.weights(N, K, seed=124).numpy()
    U_or, dead_or = oracle.gptq_prepare(X)
    c_ref, s_ref, _, _ = oracle.gptq_g64(W, bits, U_or, dead_or)
    H = rq.gptq_hessian(torch.from_numpy(X).cuda())
    U, dead = rq.gptq_factor(H, oracle.GPTQ_DAMP)
    Wd = torch.from_numpy(W).cuda()
    codes, scales = rq.gptq_g64(Wd, bits, U, dead)
    torch.cuda.synchronize()
    cg = unpack(codes.cpu().numpy(), bits, K)
    cr = unpack(c_ref, bits, K)
    assert (cg == cr).mean() >= 0.995
    Xd = X.astype(np.float64)

    def layer_err(c, s):
        w_hat = c.astype(np.float64) * np.repeat(s.view(np.float16).astype(np.float64), 64, axis=1)
        return np.linalg.norm((W.astype(np.float64) - w_hat) @ Xd.T)

    e_g = layer_err(cg, scales.cpu().numpy().view(np.uint16))
    e_r = layer_err(cr, s_ref)
    assert abs(e_g - e_r) <= 0.01 * e_r, (e_g, e_r)


def test_workload_shape_sampled_rows():
    """A 4096 x 4096 projection of the 7.2B/13.3B shapes: GPU loop given the
    oracle's U, oracle loop on sampled rows (rows are independent given U)."""
    N = K = 4096
    bits = 4
    X = calib(512, K, seed=4096)
    U32 = oracle.gptq_prepare(X)[0].astype(np.float32)
    W = synth.weights(N, K, seed=synth.seed_for(5, 0, 3), device="cuda")
    rows = np.array([0, 1, 777, 2048, 4095])
    W_rows = W[torch.from_numpy(rows).cuda()].cpu().numpy()
    codes, scales = rq.gptq_g64(W, bits, torch.from_numpy(U32).cuda())
    torch.cuda.synchronize()
    c_ref, s_ref, _, st = oracle.gptq_g64(W_rows, bits, U32)
    assert st == 0
    idx = torch.from_numpy(rows).cuda()
    assert np.array_equal(codes[idx].cpu().numpy(), c_ref)
    assert np.array_equal(scales[idx].cpu().numpy().view(np.uint16), s_ref)
