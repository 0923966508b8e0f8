"""Pins of the oracle's GPTQ on the group-64 grid (oracle.gptq_prepare,
oracle.gptq_g64).

The pages name GPTQ on the same symmetric g64 format ("Hakureirm/rwkv7-sglang-
w4gptq-1.5b" model card, opening summary; "rwkv-quant: uma matriz em bf16
elimina 39% das perdas na quantização do RWKV-7 2.9B", "Vazamento de
calibração e medições honestas") and leave the algorithm to the published
method.  What pins the oracle here, independently of its C code:
  * a diagonal Hessian (inputs with orthogonal columns) leaves nothing to
    spread: GPTQ is then RTN bit for bit, and U is diag(1/sqrt(h_jj + damp));
  * the sequential optimal-brain-surgeon form of the same method (an explicit
    inverse Hessian, downdated after every column: the form GPTQ derives its
    Cholesky formulation from), written here in numpy fp64, gives the same
    codes and scales on random correlated inputs;
  * two hand-worked rows: an error spread within a group flips a later code
    away from RTN's, and an error spread across a group boundary changes the
    next group's scale (found from the updated weights);
  * on correlated inputs the layer-output error ||(W - W_hat) X^T|| is well
    below RTN's;
  * the factor of the prepare step reproduces the damped inverse Hessian, and
    all-zero input columns are marked dead.
"""
import numpy as np
import pytest

import oracle

F32 = np.float32
F16 = np.float16


def unpack(codes, bits, K):
    if bits == 8:
        return codes.view(np.int8).astype(np.int32)
    lo = (codes & 0xF).astype(np.int32)
    hi = (codes >> 4).astype(np.int32)
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def dequant(codes, scales, bits, K):
    c = unpack(codes, bits, K).astype(np.float64)
    s = np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    return c * s


def correlated_inputs(T, K, seed, mix=0.4):
    rng = np.random.default_rng(seed)
    A = np.eye(K) + mix * rng.standard_normal((K, K)) / np.sqrt(K) * 4
    return (rng.standard_normal((T, K)) @ A).astype(F16)


def rtn_scale16(w64, qmax):
    a = F32(np.max(np.abs(w64.astype(F32))))
    return np.array([F32(a / F32(qmax))], F32).astype(F16)[0]


def obs_sequential(W, X, bits, damp=oracle.GPTQ_DAMP):
    """GPTQ in its sequential optimal-brain-surgeon form, numpy fp64: an
    explicit inverse Hessian Hi; column j is quantized on the g64 grid (scale
    from the group's current weights at its first column), its error
    (w_j - q_j) / Hi[j, j] is spread over the remaining columns along row j
    of Hi, and Hi is downdated to remove column j."""
    qmax = 7 if bits == 4 else 127
    Xd = X.astype(np.float64)
    T, K = Xd.shape
    H = (2.0 / T) * (Xd.T @ Xd)
    dead = np.diag(H) == 0
    H[dead, dead] = 1.0
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    N = W.shape[0]
    codes = np.zeros((N, K), np.int32)
    scales = np.zeros((N, K // 64), F16)
    for n in range(N):
        w = W[n].astype(np.float64).copy()
        w[dead] = 0.0
        Hi = np.linalg.inv(H)
        for j in range(K):
            if j % 64 == 0:
                s16 = rtn_scale16(w[j:j + 64], qmax)
                scales[n, j // 64] = s16
                sf = float(s16)
            c = 0 if sf == 0 else int(np.clip(np.rint(F32(w[j]) / F32(sf)), -qmax, qmax))
            codes[n, j] = c
            err = (w[j] - c * sf) / Hi[j, j]
            w[j + 1:] -= err * Hi[j, j + 1:]
            Hi = Hi - np.outer(Hi[:, j], Hi[j, :]) / Hi[j, j]
            w[j] = c * sf
    return codes, scales


@pytest.mark.parametrize("bits", [4, 8])
def test_diagonal_hessian_is_rtn(bits):
    """Orthogonal input columns: H is diagonal, U is diagonal, no error is
    spread, and GPTQ is RTN bit for bit."""
    K, N = 192, 6
    rng = np.random.default_rng(3)
    X = np.zeros((K, K), F16)
    X[np.arange(K), np.arange(K)] = rng.uniform(0.5, 2.0, K).astype(F16)
    U, dead = oracle.gptq_prepare(X)
    assert not dead.any()
    h = 2.0 / K * X.astype(np.float64).diagonal() ** 2
    lam = oracle.GPTQ_DAMP * h.mean()
    assert np.allclose(U, np.diag(1.0 / np.sqrt(h + lam)), rtol=1e-12, atol=0)
    W = (0.02 * rng.standard_normal((N, K))).astype(F32)
    c, s, Wc, st = oracle.gptq_g64(W, bits, U, dead)
    c0, s0, st0 = oracle.quantize_g64(W, bits)
    assert st == st0 == 0
    assert np.array_equal(c, c0) and np.array_equal(s, s0)
    assert np.array_equal(Wc, W)


@pytest.mark.parametrize("bits", [4, 8])
def test_matches_sequential_obs(bits):
    """The Cholesky-factor column loop against the sequential optimal-brain-
    surgeon form of the same method on random correlated inputs."""
    K, N, T = 128, 24, 512
    X = correlated_inputs(T, K, seed=11 + bits)
    W = (0.02 * np.random.default_rng(12).standard_normal((N, K))).astype(F32)
    U, dead = oracle.gptq_prepare(X)
    c, s, _, st = oracle.gptq_g64(W, bits, U, dead)
    assert st == 0
    c_ref, s_ref = obs_sequential(W, X, bits)
    cu = unpack(c, bits, K)
    same = (cu == c_ref).mean()
    assert same >= 0.995, f"only {same:.4f} of the codes agree"
    assert (s.view(F16) == s_ref).mean() >= 0.99
    # and the method really moved codes away from RTN here
    c_rtn, _, _ = oracle.quantize_g64(W, bits)
    assert (unpack(c_rtn, bits, K) != c_ref).mean() > 0.05


def test_hand_worked_rows():
    """Row 0 (one group, int4): columns on the grid of scale 0.25, except
    w0 = 0.3125 and w1 = -1.3125; U = I + 2 e0 e1^T.  Column 0: code
    rint(1.25) = 1, error 0.3125 - 0.25 = 0.0625, so w1 becomes
    -1.3125 - 2 * 0.0625 = -1.4375 and its code rint(-5.75) = -6, where RTN
    gives rint(-5.25) = -5.  Row 1 (two groups): group 0 on the grid of scale
    0.25 except w63 = 0.3125 (code 1, error 0.0625); U[63, 64] = 16 moves
    w64 from -0.375 to -1.375, so group 1 (otherwise on the grid of 0.125,
    amax 0.875) starts with amax 1.375 and scale fp16(fp32(1.375) / 7)."""
    K = 128
    U = np.eye(K, dtype=F32)
    U[0, 1] = 2.0
    U[63, 64] = 16.0
    k = np.arange(K)
    W = np.zeros((2, K), F32)
    W[0, :64] = 0.25 * ((k[:64] % 15) - 7)
    W[0, 0], W[0, 1] = 0.3125, -1.3125
    W[0, 64:] = 0.25 * ((k[64:] % 15) - 7)
    W[1, :64] = 0.25 * ((k[:64] % 15) - 7)
    W[1, 63] = 0.3125
    W[1, 64:] = 0.125 * ((k[64:] % 15) - 7)
    c, s, Wc, st = oracle.gptq_g64(W, 4, U)
    assert st == 0
    cu = unpack(c, 4, K)
    # row 0
    exp0 = (k % 15) - 7
    exp0[0], exp0[1] = 1, -6
    assert np.array_equal(cu[0], exp0)
    assert list(s[0]) == [0x3400, 0x3400]                         # 0.25, 0.25
    assert Wc[0, 1] == F32(-1.4375)
    c_rtn, _, _ = oracle.quantize_g64(W[:1], 4)
    assert unpack(c_rtn, 4, K)[0, 1] == -5
    # row 1
    s1 = np.array([F32(F32(1.375) / F32(7))], F32).astype(F16)[0]
    assert s[1, 0] == 0x3400
    assert s[1, 1] == s1.view(np.uint16)
    assert Wc[1, 64] == F32(-1.375)
    w1 = W[1, 64:].copy()
    w1[0] = F32(-1.375)
    exp1_g1 = np.clip(np.rint(w1 / F32(s1)), -7, 7).astype(np.int32)
    assert np.array_equal(cu[1, 64:], exp1_g1)
    assert cu[1, 63] == 1


@pytest.mark.parametrize("bits", [4, 8])
def test_layer_error_below_rtn(bits):
    K, N, T = 256, 32, 1024
    X = correlated_inputs(T, K, seed=21)
    W = (0.02 * np.random.default_rng(22).standard_normal((N, K))).astype(F32)
    U, dead = oracle.gptq_prepare(X)
    c, s, _, _ = oracle.gptq_g64(W, bits, U, dead)
    c0, s0, _ = oracle.quantize_g64(W, bits)
    Xd = X.astype(np.float64)
    err_g = np.linalg.norm((W - dequant(c, s, bits, K)) @ Xd.T)
    err_r = np.linalg.norm((W - dequant(c0, s0, bits, K)) @ Xd.T)
    assert err_g < 0.9 * err_r, (err_g, err_r)


def test_prepare_factor_and_dead_columns():
    K, T = 128, 300
    X = correlated_inputs(T, K, seed=5)
    X[:, [7, 40]] = 0
    U, dead = oracle.gptq_prepare(X)
    assert list(np.flatnonzero(dead)) == [7, 40]
    assert np.allclose(U, np.triu(U)) and np.all(np.diag(U) > 0)
    Xd = X.astype(np.float64)
    H = (2.0 / T) * (Xd.T @ Xd)
    H[[7, 40], [7, 40]] = 1.0
    H[np.diag_indices(K)] += oracle.GPTQ_DAMP * np.mean(np.diag(H))
    assert np.allclose(U.T @ U @ H, np.eye(K), atol=1e-9)
    # a dead column's weights are zeroed before the loop: code 0
    W = (0.02 * np.random.default_rng(6).standard_normal((3, K))).astype(F32)
    c, _, Wc, _ = oracle.gptq_g64(W, 8, U, dead)
    assert np.all(unpack(c, 8, K)[:, [7, 40]] == 0)
