"""Pins of the oracle's E[x^2]-weighted scale search (oracle.quantize_g64_ex2).

The page ("rwkv-quant: uma matriz em bf16 elimina 39% das perdas na
quantização do RWKV-7 2.9B", "Dois presets e seis tamanhos") says only that a
group's scale is chosen by a search weighted by E[x^2] of the input channel.
The oracle's reading: candidates fp16(fp32(amax * f) / qmax) for caller-given
factors f, RTN codes against each, the candidate whose
sum_k E[x_k^2] (w_k - c_k s16)^2 (fp32, k order) is smallest wins, the earlier
one on a tie.  What pins it here, independently of its C code:
  * with the single factor 1 it is RTN, bit for bit;
  * a numpy float32 restatement written from the reading above, on random
    data, gives the same codes, scales and choices;
  * a hand-worked group (values derived in the comments);
  * all weights E[x^2] = 0 make every candidate tie, so the first one wins;
  * the chosen candidate's weighted error (recomputed in fp64) is never
    above RTN's.
"""
import numpy as np
import pytest

import oracle

F32 = np.float32


def unpack(codes, bits, K):
    if bits == 8:
        return codes.view(np.int8).astype(np.int32)
    lo = (codes & 0xF).astype(np.int32)
    hi = (codes >> 4).astype(np.int32)
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def restated(W, e2, bits, factors):
    """The search written out with numpy float32 scalars, one rounding per
    operation, in the order the reading states."""
    qmax = 7 if bits == 4 else 127
    N, K = W.shape
    G = K // 64
    codes = np.zeros((N, K), np.int32)
    scales = np.zeros((N, G), np.uint16)
    chosen = np.zeros((N, G), np.int32)
    for n in range(N):
        for g in range(G):
            w = W[n, 64 * g:64 * g + 64].astype(F32)
            e = e2[64 * g:64 * g + 64].astype(F32)
            amax = F32(np.max(np.abs(w)))
            best = None
            for j, f in enumerate(factors):
                a32 = F32(amax * F32(f))
                s32 = F32(a32 / F32(qmax))
                s16 = np.array([s32], F32).astype(np.float16)[0]
                if np.isinf(s16):
                    continue
                sf = F32(s16)
                if sf == 0:
                    c = np.zeros(64, np.int32)
                else:
                    c = np.clip(np.rint(w / sf), -qmax, qmax).astype(np.int32)
                err = F32(0)
                for i in range(64):
                    t = F32(F32(c[i]) * sf)
                    d = F32(w[i] - t)
                    err = F32(err + F32(e[i] * F32(d * d)))
                if best is None or err < best[0]:
                    best = (err, j, s16, c)
            _, j, s16, c = best
            codes[n, 64 * g:64 * g + 64] = c
            scales[n, g] = np.array([s16], np.float16).view(np.uint16)[0]
            chosen[n, g] = j
    return codes, scales, chosen


def weighted_err64(W, e2, codes, scales):
    s = np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    d = W.astype(np.float64) - codes.astype(np.float64) * s
    return (d * d * e2.astype(np.float64)[None, :]).reshape(W.shape[0], -1, 64).sum(-1)


def random_case(bits, N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(F32)
    W[0, :64] = 0.0                                    # an all-zero group
    if K >= 128:
        W[min(1, N - 1), 64:128] *= 25.0               # a group with large weights
    e2 = rng.gamma(0.7, 1.0, K).astype(F32)            # E[x^2] per input channel, skewed
    e2[5] = 0.0
    W[N - 1, 5] = 0.5                                  # an outlier on a channel of weight 0:
    return W, e2                                       # a smaller scale serves the rest better


FACTORS = [1.0, 0.97, 0.94, 0.9, 0.85, 0.8, 0.7]


@pytest.mark.parametrize("bits", [4, 8])
def test_single_factor_one_is_rtn(bits):
    W, e2 = random_case(bits, 17, 320, seed=11 + bits)
    c, s, ch, st = oracle.quantize_g64_ex2(W, e2, bits, [1.0])
    c0, s0, st0 = oracle.quantize_g64(W, bits)
    assert st == st0 == 0
    assert np.array_equal(c, c0) and np.array_equal(s, s0)
    assert not ch.any()


@pytest.mark.parametrize("bits,shape", [(4, (3, 192)), (8, (2, 256)), (4, (4, 128))])
def test_matches_numpy_restatement(bits, shape):
    W, e2 = random_case(bits, *shape, seed=101 + shape[0])
    c, s, ch, st = oracle.quantize_g64_ex2(W, e2, bits, FACTORS)
    rc, rs, rch = restated(W, e2, bits, FACTORS)
    assert st == 0
    assert np.array_equal(unpack(c, bits, shape[1]), rc)
    assert np.array_equal(s, rs)
    assert np.array_equal(ch, rch)
    assert ch.any(), "the search should move some group off the RTN scale"


def test_hand_worked_group():
    # w = [0.7, 0.36 x 63], E[x^2] = [0, 1 x 63], factors {1, 0.9}, int4 (qmax 7).
    # f = 1: s32 = 0.7f / 7 -> fp16 1638 * 2^-14 = 0.0999755859375 (0x2E66);
    #        0.36 / s = 3.601 -> 4, d = 0.36 - 0.39990234375 = -0.0399...,
    #        err = 63 * 0.0399^2 ~ 0.1003.
    # f = 0.9: s32 = fp32(0.7f * 0.9f) / 7 ~ 0.0900000 -> fp16 1475 * 2^-14 =
    #        0.09002685546875 (0x2DC3); 0.36 / s = 3.9988 -> 4,
    #        d = 0.36 - 0.360107421875 = -1.07e-4, err ~ 7.3e-7: f = 0.9 wins.
    #        0.7 / s = 7.78 -> clamped to 7 (its weight is 0, so it costs nothing).
    W = np.full((1, 64), 0.36, F32)
    W[0, 0] = 0.7
    e2 = np.ones(64, F32)
    e2[0] = 0.0
    c, s, ch, st = oracle.quantize_g64_ex2(W, e2, 4, [1.0, 0.9])
    assert st == 0 and ch[0, 0] == 1 and s[0, 0] == 0x2DC3
    assert c[0, 0] == 0x47 and np.all(c[0, 1:] == 0x44)     # codes 7, 4, 4, ...
    # weight only k = 0 instead: f = 1 reconstructs 0.7 as 7 * 0.0999756 =
    # 0.69983 (d = 1.7e-4); f = 0.9 gives 7 * 0.0900269 = 0.63019 (d = 0.07): f = 1.
    e2 = np.zeros(64, F32)
    e2[0] = 1.0
    c, s, ch, st = oracle.quantize_g64_ex2(W, e2, 4, [1.0, 0.9])
    assert ch[0, 0] == 0 and s[0, 0] == 0x2E66


@pytest.mark.parametrize("bits", [4, 8])
def test_zero_weights_tie_first_wins(bits):
    W, _ = random_case(bits, 5, 256, seed=7)
    c, s, ch, _ = oracle.quantize_g64_ex2(W, np.zeros(256, F32), bits, FACTORS)
    c0, s0, _ = oracle.quantize_g64(W, bits)
    assert not ch.any()
    assert np.array_equal(c, c0) and np.array_equal(s, s0)


@pytest.mark.parametrize("bits", [4, 8])
def test_never_worse_than_rtn(bits):
    W, e2 = random_case(bits, 64, 512, seed=3 + bits)
    c, s, ch, _ = oracle.quantize_g64_ex2(W, e2, bits, FACTORS)
    c0, s0, _ = oracle.quantize_g64(W, bits)
    K = W.shape[1]
    err = weighted_err64(W, e2, unpack(c, bits, K), s)
    err0 = weighted_err64(W, e2, unpack(c0, bits, K), s0)
    # the choice is made in fp32; fp64 recomputation may differ by rounding
    assert np.all(err <= err0 * (1 + 1e-5) + 1e-12)
    assert (err < err0 * (1 - 1e-3)).any()
