"""Thin Python binding of librq (include/rq.h): argument marshalling only.

Every step of every call runs in librq's sm_100a kernels; torch is used for
device memory, streams and output allocation.  There is no fallback: if
librq.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librq.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "rq.h")

GROUP = 64
MAX_DECODE_M = 32

STATUS = {0: "RQ_OK", 1: "RQ_ERR_NULL", 2: "RQ_ERR_BITS", 3: "RQ_ERR_SHAPE", 4: "RQ_ERR_ALIGN",
          5: "RQ_ERR_NONFINITE", 6: "RQ_ERR_RANGE", 7: "RQ_ERR_TIMEOUT", 8: "RQ_ERR_CUDA"}
OK, ERR_NULL, ERR_BITS, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_RANGE, ERR_TIMEOUT, ERR_CUDA = range(9)
DECODE_KERNELS = {"auto": 0, "rowtile": 1, "cluster": 2, "rowblock": 3, "tensor": 4}

_lib = None


class RQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {STATUS.get(status, status)}"
        if status == ERR_CUDA and _lib is not None:
            msg += f" ({_lib.rq_last_cuda_error().decode()})"
        super().__init__(msg)


def lib():
    """Load librq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"librq.so not built at {LIB_PATH}: run "
                           "`python -m weight_only_quantized_g64_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i64, vp, i32, u64 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
    L.rq_codes_bytes.argtypes = [i64, i64, i32]
    L.rq_codes_bytes.restype = ctypes.c_size_t
    L.rq_scales_bytes.argtypes = [i64, i64]
    L.rq_scales_bytes.restype = ctypes.c_size_t
    L.rq_quantize_g64.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
    L.rq_quantize_g64.restype = i32
    L.rq_quantize_g64_ex2.argtypes = [vp, i64, i64, i32, vp, vp, i32, vp, vp, vp, vp, vp]
    L.rq_quantize_g64_ex2.restype = i32
    L.rq_gemv_wq.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, vp]
    L.rq_gemv_wq.restype = i32
    L.rq_gemm_wq.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, vp]
    L.rq_gemm_wq.restype = i32
    L.rq_gemv_wq_noalloc.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, vp]
    L.rq_gemv_wq_noalloc.restype = i32
    L.rq_rkv_fused.argtypes = [vp, i64, i64, i64, i32] + [vp] * 9 + [vp]
    L.rq_rkv_fused.restype = i32
    L.rq_gptq_hessian.argtypes = [vp, i64, i64, vp, vp]
    L.rq_gptq_hessian.restype = i32
    L.rq_gptq_factor.argtypes = [vp, i64, ctypes.c_double, vp, vp, vp, vp]
    L.rq_gptq_factor.restype = i32
    L.rq_gptq_g64.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp]
    L.rq_gptq_g64.restype = i32
    L.rq_gemv_wq_ex.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, i32, i32, vp]
    L.rq_gemv_wq_ex.restype = i32
    L.rq_rkv_fused3.argtypes = [vp, vp, vp, i64, i64, i64, i32] + [vp] * 9 + [i32, vp]
    L.rq_rkv_fused3.restype = i32
    L.rq_quantize_p8_g16.argtypes = [vp, i64, i64, vp, vp, i32, vp, vp, vp, vp, vp]
    L.rq_quantize_p8_g16.restype = i32
    L.rq_quantize_p4a_g32.argtypes = [vp, i64, i64, vp, vp, i32, vp, vp, vp, vp, vp, vp]
    L.rq_quantize_p4a_g32.restype = i32
    L.rq_gemv_p8_g16.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp]
    L.rq_gemv_p8_g16.restype = i32
    L.rq_gemv_p4a_g32.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
    L.rq_gemv_p4a_g32.restype = i32
    L.rq_set_pdl.argtypes = [i32]
    L.rq_set_pdl.restype = i32
    L.rq_set_decode_kernel.argtypes = [i32]
    L.rq_set_decode_kernel.restype = i32
    L.rq_decode_kernel_for.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_int)]
    L.rq_decode_kernel_for.restype = i32
    L.rq_set_wait_limit_ns.argtypes = [u64]
    L.rq_set_wait_limit_ns.restype = i32
    L.rq_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), i32]
    L.rq_read_device_status.restype = i32
    L.rq_selftest_bounded_wait.argtypes = [u64, vp]
    L.rq_selftest_bounded_wait.restype = i32
    L.rq_status_string.argtypes = [i32]
    L.rq_status_string.restype = ctypes.c_char_p
    L.rq_last_cuda_error.argtypes = []
    L.rq_last_cuda_error.restype = ctypes.c_char_p
    L.rq_version.argtypes = []
    L.rq_version.restype = ctypes.c_char_p
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of every function include/rq.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(rq_[a-z0-9_]+)\s*\(",
                                 text, flags=re.M)))


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _p(t):
    return None if t is None else t.data_ptr()


def _check(st: int, what: str):
    if st != OK:
        raise RQError(st, what)


def codes_bytes(N: int, K: int, bits: int) -> int:
    return int(lib().rq_codes_bytes(N, K, bits))


def scales_bytes(N: int, K: int) -> int:
    return int(lib().rq_scales_bytes(N, K))


def empty_weights(N: int, K: int, bits: int, device="cuda"):
    """Allocate (codes uint8 [N, K*bits/8], scales int16 [N, K/64]) for N x K."""
    codes = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=device)
    scales = torch.empty((N, K // GROUP), dtype=torch.int16, device=device)
    return codes, scales


def quantize_g64(W: torch.Tensor, bits: int, codes=None, scales=None, dev_status=None,
                 stream=None):
    """RTN group-64 quantization of fp32 W[N, K] on the GPU -> (codes, scales)."""
    N, K = W.shape
    if codes is None:
        codes, scales = empty_weights(N, K, bits, W.device)
    _check(lib().rq_quantize_g64(_p(W), N, K, bits, _p(codes), _p(scales), _p(dev_status),
                                 _stream(stream)), "rq_quantize_g64")
    return codes, scales


def quantize_g64_ex2(W: torch.Tensor, e2: torch.Tensor, bits: int, factors: torch.Tensor,
                     codes=None, scales=None, chosen=None, dev_status=None, stream=None):
    """Group-64 quantization of fp32 W[N, K] with each group's scale chosen by
    an E[x^2]-weighted search over `factors` (fp32 device, 1..16 values);
    e2: fp32 [K] device.  Returns (codes, scales, chosen int32 [N, K/64])."""
    N, K = W.shape
    if codes is None:
        codes, scales = empty_weights(N, K, bits, W.device)
    if chosen is None:
        chosen = torch.empty((N, K // GROUP), dtype=torch.int32, device=W.device)
    _check(lib().rq_quantize_g64_ex2(_p(W), N, K, bits, _p(e2), _p(factors), int(factors.numel()),
                                     _p(codes), _p(scales), _p(chosen), _p(dev_status),
                                     _stream(stream)), "rq_quantize_g64_ex2")
    return codes, scales, chosen


def quantize_p8_g16(W: torch.Tensor, e2=None, factors=None, dev_status=None, stream=None):
    """Preset int8 symmetric groups of 16 -> (codes int8-as-uint8 [N, K],
    scales int16 [N, K/16], chosen int32 [N, K/16])."""
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // 16), dtype=torch.int16, device=W.device)
    chosen = torch.empty((N, K // 16), dtype=torch.int32, device=W.device)
    nf = 0 if factors is None else int(factors.numel())
    _check(lib().rq_quantize_p8_g16(_p(W), N, K, _p(e2), _p(factors), nf, _p(codes), _p(scales),
                                    _p(chosen), _p(dev_status), _stream(stream)), "rq_quantize_p8_g16")
    return codes, scales, chosen


def quantize_p4a_g32(W: torch.Tensor, e2=None, factors=None, dev_status=None, stream=None):
    """Preset int4 asymmetric groups of 32 in super-blocks -> (codes uint8
    [N, K/2], sub uint8 [N, K/32, 2], sup int16 [N, K/256, 2], chosen int32 [N, K/32])."""
    N, K = W.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    sub = torch.empty((N, K // 32, 2), dtype=torch.uint8, device=W.device)
    sup = torch.empty((N, K // 256, 2), dtype=torch.int16, device=W.device)
    chosen = torch.empty((N, K // 32), dtype=torch.int32, device=W.device)
    nf = 0 if factors is None else int(factors.numel())
    _check(lib().rq_quantize_p4a_g32(_p(W), N, K, _p(e2), _p(factors), nf, _p(codes), _p(sub), _p(sup),
                                     _p(chosen), _p(dev_status), _stream(stream)), "rq_quantize_p4a_g32")
    return codes, sub, sup, chosen


def gptq_hessian(X: torch.Tensor, H=None, stream=None):
    """H = (2/T) X^T X (fp64 [K, K]) of calibration inputs X fp16 [T, K]."""
    T, K = X.shape
    if H is None:
        H = torch.empty((K, K), dtype=torch.float64, device=X.device)
    _check(lib().rq_gptq_hessian(_p(X), T, K, _p(H), _stream(stream)), "rq_gptq_hessian")
    return H


def gptq_factor(H: torch.Tensor, damp: float = 0.01, stream=None):
    """(U fp32 [K, K], dead uint8 [K]) from H (consumed)."""
    K = H.shape[0]
    U = torch.empty((K, K), dtype=torch.float32, device=H.device)
    dead = torch.empty((K,), dtype=torch.uint8, device=H.device)
    work = torch.empty((K * K + K,), dtype=torch.float64, device=H.device)
    _check(lib().rq_gptq_factor(_p(H), K, float(damp), _p(U), _p(dead), _p(work), _stream(stream)),
           "rq_gptq_factor")
    return U, dead


def gptq_g64(W: torch.Tensor, bits: int, U: torch.Tensor, dead=None, codes=None, scales=None,
             dev_status=None, stream=None):
    """GPTQ column loop on the group-64 grid; W fp32 [N, K] is overwritten with
    the compensated weights.  Returns (codes, scales)."""
    N, K = W.shape
    if codes is None:
        codes, scales = empty_weights(N, K, bits, W.device)
    work = torch.empty((N, 128), dtype=torch.float32, device=W.device)
    _check(lib().rq_gptq_g64(_p(W), N, K, bits, _p(U), _p(dead), _p(codes), _p(scales), _p(work),
                             _p(dev_status), _stream(stream)), "rq_gptq_g64")
    return codes, scales


def gemv_wq(x: torch.Tensor, codes, scales, N: int, bits: int, y=None, stream=None):
    """Decode product y[M, N] = x[M, K] @ w_hat^T, 1 <= M <= 32."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().rq_gemv_wq(_p(x), M, K, _p(codes), _p(scales), N, bits, _p(y), _stream(stream)),
           "rq_gemv_wq")
    return y


def gemv_p8_g16(x: torch.Tensor, codes, scales, N: int, y=None, stream=None):
    """Decode product of the int8 preset (codes [N, K], scales fp16 [N, K/16])."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().rq_gemv_p8_g16(_p(x), M, K, _p(codes), _p(scales), N, _p(y), _stream(stream)),
           "rq_gemv_p8_g16")
    return y


def gemv_p4a_g32(x: torch.Tensor, codes, sub, sup, N: int, y=None, stream=None):
    """Decode product of the int4 asymmetric preset (codes [N, K/2], sub
    [N, K/32, 2], sup fp16 [N, K/256, 2])."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().rq_gemv_p4a_g32(_p(x), M, K, _p(codes), _p(sub), _p(sup), N, _p(y),
                                 _stream(stream)), "rq_gemv_p4a_g32")
    return y


def gemv_wq_noalloc(x: torch.Tensor, codes, scales, N: int, bits: int, y=None, stream=None):
    """Decode product with the library's fixed scratch array: the library
    allocates no device memory (y is allocated here only when not given)."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().rq_gemv_wq_noalloc(_p(x), M, K, _p(codes), _p(scales), N, bits, _p(y),
                                    _stream(stream)), "rq_gemv_wq_noalloc")
    return y


OUT_F32, OUT_F16 = 0, 1
EPI_NONE, EPI_RELU_SQ = 0, 1


def gemv_wq_ex(x: torch.Tensor, codes, scales, N: int, bits: int, out_dtype=torch.float32,
               epilogue: int = EPI_NONE, y=None, stream=None):
    """Decode product with the output stored as fp32 or fp16 and an optional
    fused epilogue (EPI_RELU_SQ: max(y, 0)^2)."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    od = OUT_F16 if y.dtype == torch.float16 else OUT_F32
    _check(lib().rq_gemv_wq_ex(_p(x), M, K, _p(codes), _p(scales), N, bits, _p(y), od, epilogue,
                               _stream(stream)), "rq_gemv_wq_ex")
    return y


def rkv_fused3(xr: torch.Tensor, xk: torch.Tensor, xv: torch.Tensor, wr, wk, wv, N: int, bits: int,
               out_dtype=torch.float32, ys=None, stream=None):
    """R/K/V projections, each with its own input, in one launch."""
    M, K = xr.shape
    if ys is None:
        ys = tuple(torch.empty((M, N), dtype=out_dtype, device=xr.device) for _ in range(3))
    od = OUT_F16 if ys[0].dtype == torch.float16 else OUT_F32
    _check(lib().rq_rkv_fused3(_p(xr), _p(xk), _p(xv), M, K, N, bits, _p(wr[0]), _p(wr[1]),
                               _p(wk[0]), _p(wk[1]), _p(wv[0]), _p(wv[1]), _p(ys[0]), _p(ys[1]),
                               _p(ys[2]), od, _stream(stream)), "rq_rkv_fused3")
    return ys


def gemm_wq(x: torch.Tensor, codes, scales, N: int, bits: int, y=None, stream=None):
    """Prefill product y[M, N] = x[M, K] @ w_hat^T on the tcgen05 tensor cores."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().rq_gemm_wq(_p(x), M, K, _p(codes), _p(scales), N, bits, _p(y), _stream(stream)),
           "rq_gemm_wq")
    return y


def rkv_fused(x: torch.Tensor, wr, wk, wv, N: int, bits: int, ys=None, stream=None):
    """Three projections of one shared x in one launch; w* = (codes, scales)."""
    M, K = x.shape
    if ys is None:
        ys = tuple(torch.empty((M, N), dtype=torch.float32, device=x.device) for _ in range(3))
    _check(lib().rq_rkv_fused(_p(x), M, K, N, bits, _p(wr[0]), _p(wr[1]), _p(wk[0]), _p(wk[1]),
                              _p(wv[0]), _p(wv[1]), _p(ys[0]), _p(ys[1]), _p(ys[2]),
                              _stream(stream)), "rq_rkv_fused")
    return ys


def set_pdl(enable: bool):
    _check(lib().rq_set_pdl(1 if enable else 0), "rq_set_pdl")


def set_decode_kernel(kind: str):
    """Decode kernel for later products: "auto", "rowtile", "cluster" or "rowblock"."""
    _check(lib().rq_set_decode_kernel(DECODE_KERNELS[kind]), "rq_set_decode_kernel")


def decode_kernel_for(M: int, K: int, N: int, bits: int, nmat: int = 1) -> str:
    """The decode kernel ("rowtile", "cluster", "rowblock" or "tensor") a product of this shape runs on."""
    out = ctypes.c_int(-1)
    _check(lib().rq_decode_kernel_for(M, K, N, bits, nmat, ctypes.byref(out)), "rq_decode_kernel_for")
    return {v: k for k, v in DECODE_KERNELS.items()}[out.value]


class decode_kernel:
    """Context manager: run the enclosed decode products on one kernel."""

    def __init__(self, kind: str):
        self.kind = kind

    def __enter__(self):
        set_decode_kernel(self.kind)
        return self

    def __exit__(self, *exc):
        set_decode_kernel("auto")
        return False


def set_wait_limit_ns(ns: int):
    _check(lib().rq_set_wait_limit_ns(ns), "rq_set_wait_limit_ns")


def read_device_status(reset: bool = False) -> int:
    out = ctypes.c_int(-1)
    _check(lib().rq_read_device_status(ctypes.byref(out), 1 if reset else 0),
           "rq_read_device_status")
    return out.value


def selftest_bounded_wait(limit_ns: int, stream=None):
    _check(lib().rq_selftest_bounded_wait(limit_ns, _stream(stream)), "rq_selftest_bounded_wait")
