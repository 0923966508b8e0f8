"""Pins of the oracle's preset formats (oracle.quantize_sym, quantize_p4a,
matmul_fmt): "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na
quantização do RWKV-7 2.9B", "Dois presets e seis tamanhos" -- REDUCTION
projections in 8 bits, symmetric, groups of 16; COMPRESSION projections in 4
bits, asymmetric, super-blocks, groups of 32; scales and offsets chosen by an
E[x^2]-weighted search.  The readings are the oracle's (rqo.c, preset
section).  What pins them, independently of the C code:
  * the symmetric path with groups of 64 is the g64 RTN and E[x^2] search bit
    for bit (themselves pinned elsewhere); groups of 16 match a numpy float32
    restatement;
  * the asymmetric super-block path matches a numpy float32 restatement
    (RTN and search) bit for bit;
  * a hand-built super-block whose groups lie on a grid of representable
    scales and offsets is reproduced exactly (codes, sub-codes, fp16
    super-scales);
  * invariants: code ranges, each weight at its nearest grid point;
  * products against numpy fp64 dequantise-then-matmul (non-square).
"""
import numpy as np
import pytest

import oracle

F32, F16 = np.float32, np.float16


def f16(v):
    return np.array([F32(v)], F32).astype(F16)[0]


def unpack_s(codes, bits, K):
    if bits == 8:
        return codes.view(np.int8).astype(np.int32)
    lo = (codes & 0xF).astype(np.int32)
    hi = (codes >> 4).astype(np.int32)
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def unpack_u4(codes, K):
    out = np.empty((codes.shape[0], K), np.int32)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


def rint_clamp(t, lo, hi):
    return int(np.clip(np.rint(F32(t)), lo, hi))


# ------------------------------------------------------------ symmetric ---

def sym_restated(W, bits, G, e2=None, factors=(1.0,)):
    qmax = 7 if bits == 4 else 127
    N, K = W.shape
    codes = np.zeros((N, K), np.int32)
    scales = np.zeros((N, K // G), np.uint16)
    for n in range(N):
        for g in range(K // G):
            w = W[n, G * g:G * g + G].astype(F32)
            amax = F32(np.max(np.abs(w)))
            best = None
            cands = factors if e2 is not None else (1.0,)
            for f in cands:
                a32 = F32(amax * F32(f)) if e2 is not None else amax
                s16 = f16(F32(a32 / F32(qmax)))
                if np.isinf(s16):
                    continue
                sf = F32(s16)
                c = np.zeros(G, np.int32) if sf == 0 else np.clip(np.rint(w / sf), -qmax, qmax).astype(np.int32)
                err = F32(0)
                if e2 is not None:
                    e = e2[G * g:G * g + G].astype(F32)
                    for i in range(G):
                        d = F32(w[i] - F32(F32(c[i]) * sf))
                        err = F32(err + F32(e[i] * F32(d * d)))
                if best is None or err < best[0]:
                    best = (err, s16, c)
            _, s16, c = best
            codes[n, G * g:G * g + G] = c
            scales[n, g] = np.array([s16], F16).view(np.uint16)[0]
    return codes, scales


@pytest.mark.parametrize("bits", [4, 8])
def test_sym_g64_is_the_g64_quantizer(bits):
    rng = np.random.default_rng(1)
    W = (0.02 * rng.standard_normal((6, 512))).astype(F32)
    W[2, 64:128] = 0.0
    c, s, _, st = oracle.quantize_sym(W, bits, 64)
    c0, s0, st0 = oracle.quantize_g64(W, bits)
    assert st == st0 == 0 and np.array_equal(c, c0) and np.array_equal(s, s0)
    e2 = rng.uniform(0.0, 3.0, 512).astype(F32)
    f = [1.0, 0.93, 0.86, 0.8]
    c, s, ch, _ = oracle.quantize_sym(W, bits, 64, e2, f)
    c1, s1, ch1, _ = oracle.quantize_g64_ex2(W, e2, bits, f)
    assert np.array_equal(c, c1) and np.array_equal(s, s1) and np.array_equal(ch, ch1)


@pytest.mark.parametrize("search", [False, True])
def test_sym_g16_matches_restatement(search):
    rng = np.random.default_rng(2)
    W = (0.02 * rng.standard_normal((5, 256))).astype(F32)
    W[1, :16] = 0.0
    W[3, 20] = 0.4                                   # an outlier in one group
    # heavy-tailed E[x^2] (1e-3 .. 1e3): which channels dominate each group's
    # error, and so the chosen scale, depends on that group's own channels
    e2 = (10.0 ** rng.uniform(-3.0, 3.0, 256)).astype(F32) if search else None
    f = [1.0, 0.9, 0.8, 0.7]
    c, s, _, st = oracle.quantize_sym(W, 8, 16, e2, f)
    assert st == 0
    c_ref, s_ref = sym_restated(W, 8, 16, e2, f)
    assert np.array_equal(unpack_s(c, 8, 256), c_ref)
    assert np.array_equal(s, s_ref)


# ----------------------------------------------------------- asymmetric ---

def p4a_restated(W, e2=None, factors=(1.0,)):
    """The asymmetric super-block reading, numpy float32, one rounding per
    operation in the stated order."""
    N, K = W.shape
    codes = np.zeros((N, K), np.int32)
    sub = np.zeros((N, K // 32, 2), np.uint8)
    sup = np.zeros((N, K // 256, 2), np.uint16)
    for n in range(N):
        for sb in range(K // 256):
            w = W[n, 256 * sb:256 * sb + 256].astype(F32)
            s, o = [], []
            for g in range(8):
                wg = w[32 * g:32 * g + 32]
                lo = F32(min(F32(0), np.min(wg)))
                hi = F32(max(F32(0), np.max(wg)))
                best = None
                cands = factors if e2 is not None else (1.0,)
                for fj in cands:
                    loj = F32(lo * F32(fj)) if e2 is not None else lo
                    hij = F32(hi * F32(fj)) if e2 is not None else hi
                    sj = F32(F32(hij - loj) / F32(15))
                    err = F32(0)
                    if e2 is not None:
                        e = e2[256 * sb + 32 * g:256 * sb + 32 * g + 32].astype(F32)
                        for i in range(32):
                            q = 0 if sj == 0 else rint_clamp(F32(F32(wg[i] - loj) / sj), 0, 15)
                            u = F32(F32(F32(q) * sj) + loj)
                            d = F32(wg[i] - u)
                            err = F32(err + F32(e[i] * F32(d * d)))
                    if best is None or err < best[0]:
                        best = (err, sj, loj)
                s.append(best[1])
                o.append(best[2])
            ds = f16(F32(max(s) / F32(63)))
            dm = f16(F32(F32(max(-x for x in o)) / F32(63)))
            sup[n, sb] = np.array([ds, dm], F16).view(np.uint16)
            dsf, dmf = F32(ds), F32(dm)
            for g in range(8):
                a = 0 if dsf == 0 else rint_clamp(F32(s[g] / dsf), 0, 63)
                b = 0 if dmf == 0 else rint_clamp(F32(F32(-o[g]) / dmf), 0, 63)
                sub[n, 8 * sb + g] = (a, b)
                S = F32(dsf * F32(a))
                O = F32(-F32(dmf * F32(b)))
                for i in range(32):
                    wv = w[32 * g + i]
                    codes[n, 256 * sb + 32 * g + i] = 0 if S == 0 else rint_clamp(F32(F32(wv - O) / S), 0, 15)
    return codes, sub, sup


@pytest.mark.parametrize("search", [False, True])
def test_p4a_matches_restatement(search):
    rng = np.random.default_rng(3)
    W = (0.02 * rng.standard_normal((3, 512))).astype(F32)
    W[0, 32:64] = 0.05 + np.abs(W[0, 32:64])        # a group far from zero, no negative weight
    W[1, 300] = -0.3                                 # an outlier
    W[2, 256:288] = 0.0                              # an all-zero group
    e2 = rng.uniform(0.0, 2.0, 512).astype(F32) if search else None
    f = [1.0, 0.9, 0.8, 0.7]
    c, sub, sup, _, st = oracle.quantize_p4a(W, e2, f)
    assert st == 0
    c_ref, sub_ref, sup_ref = p4a_restated(W, e2, f)
    assert np.array_equal(unpack_u4(c, 512), c_ref)
    assert np.array_equal(sub, sub_ref)
    assert np.array_equal(sup, sup_ref)


def test_p4a_hand_built_superblock_reproduced():
    """Groups on the grid of S_g = a_g 2^-12 and O_g = -b_g 2^-10, with a code
    of 0 and of 15 in every group and max a = max b = 63: every step is exact,
    so the quantizer returns ds = 2^-12, dm = 2^-10, the a_g, b_g and codes."""
    a = np.array([63, 20, 41, 33, 55, 27, 48, 60])
    b = np.array([1, 63, 17, 40, 8, 29, 52, 12])
    q = np.tile(np.arange(32) % 16, 1)
    W = np.zeros((1, 256), F32)
    for g in range(8):
        W[0, 32 * g:32 * g + 32] = (a[g] * 2.0 ** -12) * q - b[g] * 2.0 ** -10
    c, sub, sup, _, st = oracle.quantize_p4a(W)
    assert st == 0
    assert sup[0, 0, 0] == 0x0C00 and sup[0, 0, 1] == 0x1400       # 2^-12, 2^-10 in fp16
    assert np.array_equal(sub[0, :, 0], a) and np.array_equal(sub[0, :, 1], b)
    assert np.array_equal(unpack_u4(c, 256)[0], np.tile(q, 8))


def test_p4a_invariants_nearest_grid_point():
    rng = np.random.default_rng(4)
    W = (0.02 * rng.standard_normal((8, 1024))).astype(F32)
    c, sub, sup, _, st = oracle.quantize_p4a(W)
    assert st == 0
    q = unpack_u4(c, 1024)
    assert q.min() >= 0 and q.max() <= 15 and sub.max() <= 63
    ds = sup[:, :, 0].view(F16).astype(np.float64)
    dm = sup[:, :, 1].view(F16).astype(np.float64)
    S = np.repeat(ds, 8, axis=1) * sub[:, :, 0]
    O = -np.repeat(dm, 8, axis=1) * sub[:, :, 1]
    S32, O32 = np.repeat(S, 32, axis=1), np.repeat(O, 32, axis=1)
    err = np.abs(W - (S32 * q + O32))
    for dq in (-1, 1):
        q2 = np.clip(q + dq, 0, 15)
        err2 = np.abs(W - (S32 * q2 + O32))
        assert np.all(err <= err2 + 1e-6 * S32)


@pytest.mark.parametrize("fmt", [8, 4])
def test_preset_products_match_numpy(fmt):
    rng = np.random.default_rng(5)
    N, K, M = 7, 512, 3
    W = (0.02 * rng.standard_normal((N, K))).astype(F32)
    x = rng.standard_normal((M, K)).astype(F16)
    if fmt == 8:
        c, s, _, _ = oracle.quantize_sym(W, 8, 16)
        w_hat = unpack_s(c, 8, K) * np.repeat(s.view(F16).astype(np.float64), 16, axis=1)
        y, bnd = oracle.matmul_fmt(8, x, c, s)
    else:
        c, sub, sup, _, _ = oracle.quantize_p4a(W)
        ds = np.repeat(sup[:, :, 0].view(F16).astype(np.float64), 8, axis=1)
        dm = np.repeat(sup[:, :, 1].view(F16).astype(np.float64), 8, axis=1)
        S = np.repeat(ds * sub[:, :, 0], 32, axis=1)
        O = np.repeat(-dm * sub[:, :, 1], 32, axis=1)
        w_hat = S * unpack_u4(c, K) + O
        y, bnd = oracle.matmul_fmt(4, x, c, sub, sup)
    ref = x.astype(np.float64) @ w_hat.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(bnd, np.abs(x.astype(np.float64)) @ np.abs(w_hat).T, rtol=1e-12)
    # sampled outputs agree with the full product
    ms, ns = np.array([0, 2, 1]), np.array([6, 0, 3])
    ys, _ = oracle.matmul_fmt(fmt, x, c, *( (s,) if fmt == 8 else (sub, sup) ), ms=ms, ns=ns)
    assert np.allclose(ys, y[ms, ns], rtol=0, atol=0)
