"""Pins for the CPU oracle -- checks it against things other than itself.

Definition pinned: "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card, opening
summary and "Format & loading (important)" (symmetric, GROUP = 64, packed
codes + per-group scale, calibration-free round-to-nearest) and its
"Accuracy warning" section (int8 w8g64 tier).

Each pin is chosen so that a plausible mistake fails it:
  * hand-worked values (tests/golden/hand_g64.txt): wrong tie rule, dividing by
    the fp32 instead of the stored fp16 scale, wrong nibble order, wrong group
    index, wrong sign handling;
  * fp16 conversion against numpy's own conversion (ties, subnormals,
    overflow);
  * an independent numpy restatement of the quantizer on random data
    (bit-exact), and the invariants |c| <= qmax, the reconstruction error bound,
    the amax element reaching qmax;
  * exact reconstruction of weights already on the grid;
  * products against numpy fp64 dequantise-then-matmul (library matmul), with
    a non-square shape so a transposed operand fails.
"""
import os
import re

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_g64.txt")


def load_golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = [t.strip() for t in line.split("=", 1)]
            vals = []
            for tok in val.split():
                vals.append(int(tok, 16) if tok.lower().startswith("0x") else
                            (float(tok) if ("." in tok or "e" in tok.lower()) else int(tok)))
            out[key] = vals
    return out


def hand_matrix_int4():
    """The N=3, K=128 int4 example of tests/golden/hand_g64.txt."""
    W = np.zeros((3, 128), dtype=np.float32)
    k = np.arange(64)
    W[0, :64] = 0.25 * ((k % 15) - 7)
    g1 = 0.125 * ((k % 15) - 7)
    g1[1], g1[2], g1[3] = 0.3125, 0.4375, -0.3125
    W[0, 64:] = g1
    W[1, :64] = np.float32(0.3)
    W[1, 0] = np.float32(-0.7)
    W[1, 1] = np.float32(0.25)
    W[2, :64] = (((3 * k) % 15) - 7) * np.float32(0.0087890625)
    W[2, 64:] = (7 - (k % 15)) * np.float32(0.01171875)
    return W


def hand_matrix_int8():
    W = np.zeros((3, 64), dtype=np.float32)
    W[0, :] = np.float32(0.5)
    W[0, 5] = np.float32(1.27)
    W[1] = -W[0]
    s = np.float32(2.0 ** -7)
    W[2, :] = s
    W[2, 0], W[2, 1], W[2, 2], W[2, 3], W[2, 4] = 127 * s, 2.5 * s, 3.5 * s, -0.5 * s, -127 * s
    return W


def unpack(codes, N, K, bits):
    """Independent unpacking (numpy) of the packed code layout."""
    if bits == 8:
        return codes.view(np.int8).astype(np.int64).reshape(N, K)
    lo = (codes & 0xF).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    c = np.empty((N, K), dtype=np.int64)
    c[:, 0::2] = lo
    c[:, 1::2] = hi
    c[c >= 8] -= 16
    return c


def idx(spec):
    m = re.match(r"\[(\d+),(\d+)(?::(\d+))?\]", spec)
    return int(m.group(1)), int(m.group(2)), (int(m.group(3)) if m.group(3) else None)


@pytest.mark.parametrize("bits", [4, 8])
def test_hand_examples(bits):
    gold = load_golden()
    tag = f"int{bits}"
    W = hand_matrix_int4() if bits == 4 else hand_matrix_int8()
    N, K = W.shape
    codes, scales, st = oracle.quantize_g64(W, bits)
    assert st == oracle.STATUS_OK
    c = unpack(codes, N, K, bits)
    for key, vals in gold.items():
        if not key.startswith(tag + ".") or "[" not in key:
            continue
        what, spec = key[len(tag) + 1:].split("[", 1)
        spec = "[" + spec
        if what == "scale":
            n, g, _ = idx(spec)
            assert scales[n, g] == vals[0], key
        elif what == "codes":
            n, k0, k1 = idx(spec)
            assert list(c[n, k0:k1]) == vals, key
        elif what == "packed":
            n, b0, b1 = idx(spec)
            assert list(codes[n, b0:b1]) == vals, key
    x = np.ones((1, K), dtype=np.float16)
    y, b = oracle.matmul(x, codes, scales, bits)
    assert np.array_equal(y[0], np.array(gold[f"{tag}.y_ones"]))
    if bits == 4:
        for j, key in ((0, "int4.y_e0"), (65, "int4.y_e65")):
            e = np.zeros((1, K), dtype=np.float16)
            e[0, j] = 1
            y, _ = oracle.matmul(e, codes, scales, bits)
            assert np.array_equal(y[0], np.array(gold[key])), key


def test_hand_int4_exact_reconstruction_row():
    """Row 2 of the int4 example is on the grid: codes and scales come back."""
    W = hand_matrix_int4()
    codes, scales, _ = oracle.quantize_g64(W, 4)
    c = unpack(codes, 3, 128, 4)
    k = np.arange(64)
    assert np.array_equal(c[2, :64], ((3 * k) % 15) - 7)
    assert np.array_equal(c[2, 64:], 7 - (k % 15))


# ------------------------------------------------------------------ fp16 ---

def _f16_numpy(v):
    return int(np.array([v], dtype=np.float32).astype(np.float16).view(np.uint16)[0])


def test_fp16_conversion_edges():
    edge = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9,
            2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26,
            3 * 2.0 ** -25, 5 * 2.0 ** -25, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
            0.1, 0.01, 1.27 / 127, float("inf"), -float("inf"), 1e-30, 6.0e-8,
            2.0 ** -14 - 2.0 ** -25, 2.0 ** -14 - 2.0 ** -26]
    for v in edge:
        v32 = float(np.float32(v))
        assert oracle.f32_to_f16_bits(v32) == _f16_numpy(v32), v
    assert oracle.f32_to_f16_bits(float("nan")) & 0x7C00 == 0x7C00
    assert oracle.f32_to_f16_bits(float("nan")) & 0x3FF != 0


def test_fp16_conversion_sampled_bit_patterns():
    """Every fp32 bit pattern class in the fp16 range, stepping by sampling."""
    rng = np.random.default_rng(7)
    pats = np.concatenate([
        rng.integers(0x33000000, 0x47800000, size=20000, dtype=np.uint32),  # 2^-25 .. 65536
        rng.integers(0xB3000000, 0xC7800000, size=5000, dtype=np.uint32),
        # exact ties: fp16 grid midpoints in the normal range
        (np.arange(0x38000000, 0x47000000, 0x1000, dtype=np.uint32)),
    ])
    vals = pats.view(np.float32)
    ref = vals.astype(np.float16).view(np.uint16)
    lib = oracle._load()
    mine = np.array([lib.rqo_f32_to_f16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(mine, ref)


def test_fp16_to_f64_all_patterns():
    h = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    lib = oracle._load()
    mine = np.array([lib.rqo_f16_to_f64(int(v)) for v in h[::7]])
    r = ref[::7]
    fin = np.isfinite(r)
    assert np.array_equal(mine[fin], r[fin])
    assert np.array_equal(np.isnan(mine), np.isnan(r))


# ------------------------------------------------------ quantizer (random) ---

def numpy_quantize(W, bits):
    """Independent restatement with numpy fp32 semantics (IEEE division,
    numpy's fp16 rounding, np.rint half-to-even)."""
    qmax = {4: 7, 8: 127}[bits]
    N, K = W.shape
    Wg = W.reshape(N, K // 64, 64).astype(np.float32)
    amax = np.max(np.abs(Wg), axis=2)
    s32 = (amax / np.float32(qmax)).astype(np.float32)
    s16 = s32.astype(np.float16)
    sf = s16.astype(np.float32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        c = np.rint(Wg / sf)
    c = np.where(sf == 0, 0, c)
    c = np.clip(c, -qmax, qmax).astype(np.int64).reshape(N, K)
    return c, s16.view(np.uint16)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("shape,scale", [((37, 192), 0.02), ((5, 768), 1.0), ((64, 64), 3e-3)])
def test_quantizer_matches_numpy_restatement(bits, shape, scale):
    rng = np.random.default_rng(hash((bits, shape)) % 2**32)
    W = (rng.standard_normal(shape) * scale).astype(np.float32)
    # plant exact ties and on-grid values in a few groups
    W[0, :64] = np.float32(0.125) * (np.arange(64) % 15 - 7)
    W[0, 1] = np.float32(0.3125)
    W[1 % shape[0], 64 % shape[1]:64 % shape[1] + 64] = 0.0
    codes, scales, st = oracle.quantize_g64(W, bits)
    assert st == oracle.STATUS_OK
    c_ref, s_ref = numpy_quantize(W, bits)
    assert np.array_equal(scales, s_ref)
    assert np.array_equal(unpack(codes, *shape, bits), c_ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantizer_invariants(bits):
    qmax = oracle.QMAX[bits]
    rng = np.random.default_rng(11 + bits)
    N, K = 64, 1024
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, scales, _ = oracle.quantize_g64(W, bits)
    c = unpack(codes, N, K, bits)
    s = scales.view(np.float16).astype(np.float64)
    assert np.all(np.abs(c) <= qmax)
    sk = np.repeat(s, 64, axis=1)
    err = np.abs(W.astype(np.float64) - c * sk)
    # |w - c*s| <= s/2 + |w| * 2^-24 (one fp32 rounding of w/s before rint)
    assert np.all(err <= sk / 2 + np.abs(W) * 2.0 ** -23)
    # the element attaining amax reaches |c| == qmax (amax/s16 = qmax*(1 +- 2^-11))
    Wg = np.abs(W).reshape(N, K // 64, 64)
    arg = np.argmax(Wg, axis=2)
    cg = np.abs(c.reshape(N, K // 64, 64))
    assert np.all(np.take_along_axis(cg, arg[:, :, None], axis=2) == qmax)


@pytest.mark.parametrize("bits", [4, 8])
def test_exact_reconstruction_on_grid(bits):
    qmax = oracle.QMAX[bits]
    rng = np.random.default_rng(3 + bits)
    N, G = 16, 8
    K = 64 * G
    # fp16-normal scales
    s = (rng.uniform(1e-3, 1.0, size=(N, G))).astype(np.float16)
    c = rng.integers(-qmax, qmax + 1, size=(N, K))
    c[:, ::64] = qmax * np.where(rng.random((N, G)) < 0.5, -1, 1)
    W = (c * np.repeat(s.astype(np.float64), 64, axis=1)).astype(np.float32)
    codes, scales, st = oracle.quantize_g64(W, bits)
    assert st == 0
    assert np.array_equal(scales, s.view(np.uint16))
    assert np.array_equal(unpack(codes, N, K, bits), c)


def test_zero_group_and_statuses():
    W = np.zeros((2, 128), dtype=np.float32)
    W[1, 70] = 1.0
    codes, scales, st = oracle.quantize_g64(W, 4)
    assert st == 0 and scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert np.all(codes[0] == 0)
    W2 = W.copy()
    W2[0, 3] = np.nan
    _, sc, st = oracle.quantize_g64(W2, 8)
    assert st == oracle.STATUS_NONFINITE and sc[0, 0] == 0x7E00
    W3 = W.copy()
    W3[1, 5] = 1e6          # 1e6/7 > 65504 -> fp16 overflow
    c3, sc3, st3 = oracle.quantize_g64(W3, 4)
    assert st3 == oracle.STATUS_RANGE and sc3[1, 0] == 0x7C00
    assert np.all(unpack(c3, 2, 128, 4)[1, :64] == 0)
    W4 = W3.copy()
    W4[0, 0] = np.inf       # NONFINITE wins over RANGE
    _, _, st4 = oracle.quantize_g64(W4, 4)
    assert st4 == oracle.STATUS_NONFINITE


# -------------------------------------------------------------- products ---

@pytest.mark.parametrize("bits", [4, 8])
def test_products_match_numpy_fp64(bits):
    rng = np.random.default_rng(21 + bits)
    M, N, K = 5, 33, 320             # non-square: a transposed operand fails
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float16)
    codes, scales, _ = oracle.quantize_g64(W, bits)
    c = unpack(codes, N, K, bits).astype(np.float64)
    s = np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    what = c * s
    y_np = x.astype(np.float64) @ what.T
    b_np = np.abs(x.astype(np.float64)) @ np.abs(what).T
    y, b = oracle.matmul(x, codes, scales, bits)
    assert np.allclose(y, y_np, rtol=1e-12, atol=1e-12 * np.max(b_np))
    assert np.allclose(b, b_np, rtol=1e-12)
    ms = np.array([0, 4, 2, 4])
    ns = np.array([0, 32, 17, 5])
    ys, bs = oracle.matmul_sampled(x, codes, scales, bits, ms, ns)
    assert np.array_equal(ys, y[ms, ns]) and np.array_equal(bs, b[ms, ns])


def test_unit_vector_picks_column():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((7, 256)) * 0.02).astype(np.float32)
    codes, scales, _ = oracle.quantize_g64(W, 4)
    c = unpack(codes, 7, 256, 4)
    s = scales.view(np.float16).astype(np.float64)
    for j in (0, 63, 64, 200, 255):
        e = np.zeros((1, 256), dtype=np.float16)
        e[0, j] = 1
        y, _ = oracle.matmul(e, codes, scales, 4)
        assert np.array_equal(y[0], c[:, j] * s[:, j // 64])
