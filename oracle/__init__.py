"""CPU oracle for weight-only group-64 symmetric int4/int8 quantized products.

TEST INFRASTRUCTURE ONLY.  The product library never imports, links or calls
anything in this package; only the test suite, the smoke check and the
benchmark's CPU-baseline leg may.  It shares no code, header, table or helper
with the CUDA path; the only thing both sides see is the seeded input
generator module, which holds none of the method's arithmetic.

The arithmetic lives in ``rqo.c`` (plain scalar C, fp32 quantizer exactly as
defined, fp64 products); this module builds it with gcc and wraps it with
ctypes.  What it follows, and every reading taken where the pages are silent,
is written at the top of ``rqo.c``:

  * "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card, opening summary and
    "Format & loading (important)": GROUP = 64, symmetric int4, packed codes
    plus per-group scales, calibration-free round-to-nearest; the kernel output
    equals the product with the offline-dequantised weight.
  * same card, "Accuracy warning": the int8 w8g64 tier.

Parity status: the quantizer is pinned bit-exactly (hand-worked examples,
exact-reconstruction and tie-break cases, an independent numpy restatement,
invariants); the fp16 converter is pinned against numpy's conversion; the
products are pinned against an independent numpy fp64 dequantise-then-matmul
and hand-worked values.  No function is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rqo.c")
_LIB_PATH = os.path.join(_HERE, "_build", "librqo.so")
_lib = None

GROUP = 64
QMAX = {4: 7, 8: 127}
STATUS_OK, STATUS_NONFINITE, STATUS_RANGE = 0, 5, 6


def build(force: bool = False) -> str:
    """Compile rqo.c into oracle/_build/librqo.so (gcc, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-fno-finite-math-only",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.rqo_f32_to_f16.argtypes = [ctypes.c_float]
    lib.rqo_f32_to_f16.restype = ctypes.c_uint16
    lib.rqo_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.rqo_f16_to_f64.restype = ctypes.c_double
    lib.rqo_quantize_g64.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp]
    lib.rqo_quantize_g64.restype = ctypes.c_int
    lib.rqo_quantize_g64_ex2.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp, ctypes.c_int, vp, vp, vp]
    lib.rqo_quantize_g64_ex2.restype = ctypes.c_int
    lib.rqo_matmul.argtypes = [vp, i64, i64, vp, vp, i64, ctypes.c_int, vp, vp]
    lib.rqo_matmul.restype = None
    lib.rqo_matmul_sampled.argtypes = [vp, i64, i64, vp, vp, i64, ctypes.c_int,
                                       i64, vp, vp, vp, vp]
    lib.rqo_matmul_sampled.restype = None
    lib.rqo_get_code.argtypes = [vp, i64, ctypes.c_int, i64, i64]
    lib.rqo_get_code.restype = ctypes.c_int
    lib.rqo_gptq_g64.argtypes = [vp, i64, i64, ctypes.c_int, vp, vp, vp, vp]
    lib.rqo_gptq_g64.restype = ctypes.c_int
    lib.rqo_quantize_sym.argtypes = [vp, i64, i64, ctypes.c_int, ctypes.c_int, vp, vp, ctypes.c_int,
                                     vp, vp, vp]
    lib.rqo_quantize_sym.restype = ctypes.c_int
    lib.rqo_quantize_p4a.argtypes = [vp, i64, i64, vp, vp, ctypes.c_int, vp, vp, vp, vp]
    lib.rqo_quantize_p4a.restype = ctypes.c_int
    lib.rqo_get_ucode4.argtypes = [vp, i64, i64, i64]
    lib.rqo_get_ucode4.restype = ctypes.c_int
    lib.rqo_matmul_fmt.argtypes = [ctypes.c_int, vp, i64, i64, vp, vp, vp, i64, i64, vp, vp, vp, vp]
    lib.rqo_matmul_fmt.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def f32_to_f16_bits(v: float) -> int:
    """Round-to-nearest-even fp32 -> fp16 bit pattern (the oracle's own)."""
    return int(_load().rqo_f32_to_f16(ctypes.c_float(v)))


def f16_bits_to_f64(h: int) -> float:
    return float(_load().rqo_f16_to_f64(ctypes.c_uint16(h)))


def codes_bytes(N: int, K: int, bits: int) -> int:
    return N * K * bits // 8


def quantize_g64(W: np.ndarray, bits: int):
    """RTN group-64 quantization of fp32 W[N, K].

    Returns (codes uint8 [N, K*bits/8], scales uint16 fp16-bits [N, K/64],
    status int)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if bits not in (4, 8) or K % GROUP:
        raise ValueError("bits must be 4 or 8 and K a multiple of 64")
    codes = np.zeros((N, K * bits // 8), dtype=np.uint8)
    scales = np.zeros((N, K // GROUP), dtype=np.uint16)
    st = _load().rqo_quantize_g64(_ptr(W), N, K, bits, _ptr(codes), _ptr(scales))
    return codes, scales, int(st)


def quantize_g64_ex2(W: np.ndarray, e2: np.ndarray, bits: int, factors):
    """E[x^2]-weighted scale search on the symmetric group-64 grid: per group,
    the candidate scale fp16(fp32(amax * f) / qmax), f in `factors`, whose
    codes minimise sum_k e2[k] * (w_k - c_k * s16)^2 (fp32, k order; the
    earlier candidate wins ties).  e2 [K] float32 >= 0, one value per input
    channel.  Returns (codes, scales, chosen int32 [N, K/64], status)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if bits not in (4, 8) or K % GROUP:
        raise ValueError("bits must be 4 or 8 and K a multiple of 64")
    e2 = np.ascontiguousarray(e2, dtype=np.float32)
    f = np.ascontiguousarray(factors, dtype=np.float32)
    if e2.shape != (K,) or f.ndim != 1 or f.size < 1:
        raise ValueError("e2 must have K values and factors at least one")
    codes = np.zeros((N, K * bits // 8), dtype=np.uint8)
    scales = np.zeros((N, K // GROUP), dtype=np.uint16)
    chosen = np.zeros((N, K // GROUP), dtype=np.int32)
    st = _load().rqo_quantize_g64_ex2(_ptr(W), N, K, bits, _ptr(e2), _ptr(f), int(f.size),
                                      _ptr(codes), _ptr(scales), _ptr(chosen))
    return codes, scales, chosen, int(st)


def matmul(x_f16: np.ndarray, codes: np.ndarray, scales: np.ndarray, bits: int,
           with_bound: bool = True):
    """y[M, N] = x @ (c * s16)^T in fp64, plus the budget sum |x||c*s16|.

    x_f16 is float16 (or uint16 fp16 bit patterns) [M, K]."""
    x = np.ascontiguousarray(x_f16).view(np.uint16)
    M, K = x.shape
    N = scales.shape[0]
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales).view(np.uint16)
    y = np.zeros((M, N), dtype=np.float64)
    b = np.zeros((M, N), dtype=np.float64) if with_bound else None
    _load().rqo_matmul(_ptr(x), M, K, _ptr(codes), _ptr(scales), N, bits, _ptr(y),
                       _ptr(b) if b is not None else None)
    return (y, b) if with_bound else y


def matmul_sampled(x_f16: np.ndarray, codes: np.ndarray, scales: np.ndarray,
                   bits: int, ms, ns):
    """y and budget at the sampled outputs (ms[p], ns[p])."""
    x = np.ascontiguousarray(x_f16).view(np.uint16)
    M, K = x.shape
    N = scales.shape[0]
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales).view(np.uint16)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    P = ms.shape[0]
    y = np.zeros(P, dtype=np.float64)
    b = np.zeros(P, dtype=np.float64)
    _load().rqo_matmul_sampled(_ptr(x), M, K, _ptr(codes), _ptr(scales), N, bits, P,
                               _ptr(ms), _ptr(ns), _ptr(y), _ptr(b))
    return y, b


def get_code(codes: np.ndarray, K: int, bits: int, n: int, k: int) -> int:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    return int(_load().rqo_get_code(_ptr(codes), K, bits, n, k))


# ------------------------------------------------------------------ GPTQ ---
# GPTQ on the symmetric group-64 grid ("Hakureirm/rwkv7-sglang-w4gptq-1.5b"
# model card, opening summary: GPTQ-calibrated, symmetric, group 64, same
# format as RTN; "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na
# quantização do RWKV-7 2.9B", "Vazamento de calibração e medições honestas":
# GPTQ on the preset's grid, format and kernels unchanged).  The method is
# the published GPTQ (Frantar et al., arXiv:2210.17323).

GPTQ_DAMP = 0.01


def gptq_prepare(X_f16: np.ndarray, damp: float = GPTQ_DAMP):
    """The inverse-Hessian factor of GPTQ for calibration inputs X (fp16
    [T, K], T tokens), in fp64 with numpy, following the method's steps:
    H = 2 X^T X / T; a column whose input is always zero (H[j, j] == 0) is
    marked dead and gets H[j, j] = 1; H += damp * mean(diag H) * I; then
    H^-1 through the Cholesky factor of H, and U = the upper Cholesky factor
    of H^-1 (H^-1 = U^T U).  Returns (U float64 [K, K], dead uint8 [K])."""
    X = np.ascontiguousarray(X_f16).astype(np.float64)
    T, K = X.shape
    H = (2.0 / T) * (X.T @ X)
    dead = np.diag(H) == 0
    H[dead, dead] = 1.0
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    L = np.linalg.cholesky(H)                       # H = L L^T
    Linv = np.linalg.inv(L)
    Hinv = Linv.T @ Linv                            # H^-1
    U = np.linalg.cholesky(Hinv).T                  # H^-1 = U^T U, U upper
    return np.ascontiguousarray(U), dead.astype(np.uint8)


def gptq_g64(W: np.ndarray, bits: int, U: np.ndarray, dead=None):
    """The GPTQ column loop on the group-64 grid (rqo.c, fp32): W fp32 [N, K],
    U the upper factor (rounded to fp32 here), dead uint8 [K] or None.
    Returns (codes, scales, W_compensated, status)."""
    Wc = np.array(W, dtype=np.float32, order="C", copy=True)
    N, K = Wc.shape
    if bits not in (4, 8) or K % GROUP:
        raise ValueError("bits must be 4 or 8 and K a multiple of 64")
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    if U32.shape != (K, K):
        raise ValueError("U must be K x K")
    d = None if dead is None else np.ascontiguousarray(dead, dtype=np.uint8)
    codes = np.zeros((N, K * bits // 8), dtype=np.uint8)
    scales = np.zeros((N, K // GROUP), dtype=np.uint16)
    st = _load().rqo_gptq_g64(_ptr(Wc), N, K, bits, _ptr(U32), _ptr(d) if d is not None else None,
                              _ptr(codes), _ptr(scales))
    return codes, scales, Wc, int(st)


# ------------------------------------------------ decode epilogues (fused) --
# The squared ReLU that follows the channel-mix key projection of an RWKV-7
# block (k = relu(key(x))^2; the value projection then reads k).

def relu_sq(y: np.ndarray) -> np.ndarray:
    """max(y, 0)^2 in fp64."""
    r = np.maximum(np.asarray(y, dtype=np.float64), 0.0)
    return r * r


def relu_sq_budget(y_ref: np.ndarray, delta: np.ndarray) -> np.ndarray:
    """Error budget of relu(a)^2 when |a - y_ref| <= delta:
    |relu(a)^2 - relu(b)^2| <= |a - b| (relu(a) + relu(b)) <= delta (2 relu(b) + delta)."""
    return delta * (2.0 * np.maximum(y_ref, 0.0) + delta)


# ------------------------------------------- preset formats ("rwkv-quant") --
# "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na quantização do
# RWKV-7 2.9B", "Dois presets e seis tamanhos": REDUCTION projections in 8
# bits, symmetric, groups of 16; COMPRESSION projections in 4 bits,
# asymmetric, super-blocks, groups of 32; scales and offsets chosen by a
# search weighted by E[x^2].  The readings are written at the top of the
# preset section of rqo.c.


def _search_args(e2, factors, K):
    if e2 is None:
        return None, np.ones(1, np.float32), 1
    e2 = np.ascontiguousarray(e2, dtype=np.float32)
    f = np.ascontiguousarray(factors if factors is not None else [1.0], dtype=np.float32)
    if e2.shape != (K,) or f.ndim != 1 or f.size < 1:
        raise ValueError("e2 must have K values and factors at least one")
    return e2, f, int(f.size)


def quantize_sym(W: np.ndarray, bits: int, G: int, e2=None, factors=None):
    """Symmetric group-G quantization (RTN when e2 is None, else the
    E[x^2]-weighted scale search over `factors`).  Returns (codes, scales
    uint16 [N, K/G], chosen int32 [N, K/G], status)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if bits not in (4, 8) or G not in (16, 32, 64) or K % G:
        raise ValueError("bits 4/8, G in {16, 32, 64}, K a multiple of G")
    e2a, f, nf = _search_args(e2, factors, K)
    codes = np.zeros((N, K * bits // 8), dtype=np.uint8)
    scales = np.zeros((N, K // G), dtype=np.uint16)
    chosen = np.zeros((N, K // G), dtype=np.int32)
    st = _load().rqo_quantize_sym(_ptr(W), N, K, bits, G, _ptr(e2a) if e2a is not None else None,
                                  _ptr(f), nf, _ptr(codes), _ptr(scales), _ptr(chosen))
    return codes, scales, chosen, int(st)


def quantize_p4a(W: np.ndarray, e2=None, factors=None):
    """Asymmetric int4, groups of 32 in super-blocks of 8 groups.  Returns
    (codes uint8 [N, K/2], sub uint8 [N, K/32, 2] = (a, b), sup uint16
    [N, K/256, 2] = (ds, dm) fp16 bits, chosen int32 [N, K/32], status)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if K % 256:
        raise ValueError("K must be a multiple of 256")
    e2a, f, nf = _search_args(e2, factors, K)
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    sub = np.zeros((N, K // 32, 2), dtype=np.uint8)
    sup = np.zeros((N, K // 256, 2), dtype=np.uint16)
    chosen = np.zeros((N, K // 32), dtype=np.int32)
    st = _load().rqo_quantize_p4a(_ptr(W), N, K, _ptr(e2a) if e2a is not None else None, _ptr(f), nf,
                                  _ptr(codes), _ptr(sub), _ptr(sup), _ptr(chosen))
    return codes, sub, sup, chosen, int(st)


def matmul_fmt(fmt: int, x_f16: np.ndarray, codes, meta0, meta1=None, ms=None, ns=None):
    """Products of the preset formats in fp64 with the budget sum |x||w_hat|:
    fmt 8 = int8 g16 symmetric (meta0 = scales [N, K/16]); fmt 4 = int4 g32
    asymmetric super-blocks (meta0 = sub, meta1 = sup).  Every output, or the
    sampled pairs (ms[p], ns[p])."""
    x = np.ascontiguousarray(x_f16).view(np.uint16)
    M, K = x.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    m0 = np.ascontiguousarray(meta0)
    m1 = None if meta1 is None else np.ascontiguousarray(meta1)
    N = m0.shape[0]
    if ms is None:
        P = M * N
        y = np.zeros(P, np.float64)
        b = np.zeros(P, np.float64)
        _load().rqo_matmul_fmt(fmt, _ptr(x), M, K, _ptr(codes), _ptr(m0),
                               _ptr(m1) if m1 is not None else None, N, P, None, None, _ptr(y), _ptr(b))
        return y.reshape(M, N), b.reshape(M, N)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    P = ms.shape[0]
    y = np.zeros(P, np.float64)
    b = np.zeros(P, np.float64)
    _load().rqo_matmul_fmt(fmt, _ptr(x), M, K, _ptr(codes), _ptr(m0), _ptr(m1) if m1 is not None else None,
                           N, P, _ptr(ms), _ptr(ns), _ptr(y), _ptr(b))
    return y, b
