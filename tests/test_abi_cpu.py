"""librq's C ABI on a machine without a GPU: it loads, exports every function
include/rq.h declares, sizes come out right, and argument errors are returned
synchronously before any CUDA call (so these tests launch nothing)."""
import ctypes
import subprocess

import pytest

from weight_only_quantized_g64_b200 import build as rq_build
from weight_only_quantized_g64_b200 import rq


@pytest.fixture(scope="module")
def L():
    rq_build.build()
    return rq.lib()


def test_exports_every_header_function(L):
    names = rq.header_functions()
    assert len(names) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", rq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert getattr(L, n) is not None


def test_sizes(L):
    assert L.rq_codes_bytes(768, 768, 4) == 768 * 384
    assert L.rq_codes_bytes(2560, 10240, 8) == 2560 * 10240
    assert L.rq_scales_bytes(4096, 16384) == 4096 * 256 * 2
    assert L.rq_codes_bytes(10, 100, 4) == 0       # K % 64 != 0
    assert L.rq_codes_bytes(10, 128, 3) == 0       # bad bits
    assert L.rq_codes_bytes(0, 128, 4) == 0


FAKE = 1 << 20          # aligned, non-null; never dereferenced because validation fails first


@pytest.mark.parametrize("fn", ["rq_gemv_wq", "rq_gemm_wq"])
def test_product_argument_errors(L, fn):
    f = getattr(L, fn)
    assert f(FAKE, 1, 768, FAKE, FAKE, 768, 3, FAKE, None) == rq.ERR_BITS
    assert f(FAKE, 1, 100, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_SHAPE
    assert f(FAKE, 1, 0, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_SHAPE
    assert f(FAKE, 1, 768, FAKE, FAKE, 0, 4, FAKE, None) == rq.ERR_SHAPE
    assert f(FAKE, 0, 768, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_SHAPE
    assert f(None, 1, 768, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_NULL
    assert f(FAKE, 1, 768, None, FAKE, 768, 4, FAKE, None) == rq.ERR_NULL
    assert f(FAKE, 1, 768, FAKE, None, 768, 4, FAKE, None) == rq.ERR_NULL
    assert f(FAKE, 1, 768, FAKE, FAKE, 768, 4, None, None) == rq.ERR_NULL
    assert f(FAKE + 2, 1, 768, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_ALIGN
    assert f(FAKE, 1, 768, FAKE + 8, FAKE, 768, 4, FAKE, None) == rq.ERR_ALIGN
    assert f(FAKE, 1, 768, FAKE, FAKE + 2, 768, 4, FAKE, None) == rq.ERR_ALIGN
    assert f(FAKE, 1, 768, FAKE, FAKE, 768, 4, FAKE + 4, None) == rq.ERR_ALIGN


def test_gemv_m_range(L):
    assert L.rq_gemv_wq(FAKE, 33, 768, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_SHAPE
    assert L.rq_gemv_wq(FAKE, -1, 768, FAKE, FAKE, 768, 4, FAKE, None) == rq.ERR_SHAPE


def test_fused_argument_errors(L):
    ok = [FAKE] * 9
    assert L.rq_rkv_fused(FAKE, 1, 768, 768, 5, *ok, None) == rq.ERR_BITS
    assert L.rq_rkv_fused(FAKE, 40, 768, 768, 4, *ok, None) == rq.ERR_SHAPE
    for i in range(9):
        bad = list(ok)
        bad[i] = None
        assert L.rq_rkv_fused(FAKE, 1, 768, 768, 4, *bad, None) == rq.ERR_NULL, i
        bad[i] = FAKE + 4
        assert L.rq_rkv_fused(FAKE, 1, 768, 768, 4, *bad, None) == rq.ERR_ALIGN, i


def test_quantize_argument_errors(L):
    q = L.rq_quantize_g64
    assert q(FAKE, 16, 768, 6, FAKE, FAKE, None, None) == rq.ERR_BITS
    assert q(FAKE, 16, 65, 4, FAKE, FAKE, None, None) == rq.ERR_SHAPE
    assert q(None, 16, 768, 4, FAKE, FAKE, None, None) == rq.ERR_NULL
    assert q(FAKE, 16, 768, 4, None, FAKE, None, None) == rq.ERR_NULL
    assert q(FAKE + 4, 16, 768, 4, FAKE, FAKE, None, None) == rq.ERR_ALIGN
    assert q(FAKE, 16, 768, 4, FAKE, FAKE, FAKE + 2, None) == rq.ERR_ALIGN


def test_control_calls(L):
    assert L.rq_set_wait_limit_ns(0) == rq.ERR_RANGE
    assert L.rq_set_wait_limit_ns(10**9) == rq.OK
    assert L.rq_set_pdl(0) == rq.OK
    # decode kernel selection: 0 automatic, 1 row tiles, 2 cluster split-K, 3 row
    # blocks, 4 tensor cores
    for bad in (-1, 5, 1 << 20):
        assert L.rq_set_decode_kernel(bad) == rq.ERR_RANGE
    for kind, code in rq.DECODE_KERNELS.items():
        assert L.rq_set_decode_kernel(code) == rq.OK
        with rq.decode_kernel(kind):
            pass
    assert L.rq_set_decode_kernel(0) == rq.OK
    assert L.rq_selftest_bounded_wait(0, None) == rq.ERR_RANGE
    assert L.rq_read_device_status(None, 0) == rq.ERR_NULL
    for s in range(9):
        assert L.rq_status_string(s)
    assert L.rq_version() == b"0.1.0"


def test_decode_kernel_choice(L):
    """The automatic choice between the decode kernels (host logic, no GPU,
    so the SM count is taken as 148).  Launches with at least one 16-row
    m-tile per SM (the fused R/K/V and the channel-mix key of the 1.5B-shaped
    layer, every projection of the 13.3B-shaped one): the row-block kernel,
    except M > 16 on rows of >= 16384 k or launches of >= 16384 rows (the
    tensor-core kernel).  Fewer
    m-tiles: row tiles for M <= 8, row blocks for M 9..16 and for M > 16 on
    rows of <= 4096 k, the cluster kernel for M > 16 on longer rows."""
    D = 2048
    layer = {"rkv": (D, D, 3), "o": (D, D, 1), "key": (4 * D, D, 1), "value": (D, 4 * D, 1)}
    for M in (1, 4, 8, 9, 16, 17, 24, 32):
        for name in ("rkv", "key"):
            N, K, nmat = layer[name]
            assert rq.decode_kernel_for(M, K, N, 4, nmat) == "rowblock", (M, name)
            assert rq.decode_kernel_for(M, K, N, 8, nmat) == "rowblock", (M, name)
        small = "rowtile" if M <= 8 else "rowblock"
        assert rq.decode_kernel_for(M, D, D, 4, 1) == small, M                          # o
        assert rq.decode_kernel_for(M, 4 * D, D, 4, 1) == (
            small if M <= 16 else "cluster"), M                                          # value
    # the 13.3B-shaped layer (D = 4096): row blocks, the key and value
    # projections (16384 rows, 16384-long rows) at M > 16 on tensor cores
    for M in (1, 8, 16, 17, 32):
        for N, K, nmat in ((4096, 4096, 3), (4096, 4096, 1)):
            assert rq.decode_kernel_for(M, K, N, 4, nmat) == "rowblock", (M, N, K)
        big = "tensor" if M > 16 else "rowblock"
        assert rq.decode_kernel_for(M, 16384, 4096, 4, 1) == big
        assert rq.decode_kernel_for(M, 4096, 16384, 4, 1) == big
    # the boundary: 148 m-tiles (2368 rows) in the launch
    assert rq.decode_kernel_for(1, D, 2368, 4, 1) == "rowblock"
    assert rq.decode_kernel_for(1, D, 2352, 4, 1) == "rowtile"
    # a selection overrides the automatic choice
    for kind in ("rowtile", "cluster"):
        with rq.decode_kernel(kind):
            for M in (1, 16, 32):
                assert rq.decode_kernel_for(M, D, D, 8, 1) == kind
    assert rq.decode_kernel_for(1, D, D, 4, 1) == "rowtile"
    # forced row-block and tensor-core selections take every decode batch size
    for kind in ("rowblock", "tensor"):
        with rq.decode_kernel(kind):
            for M in (1, 9, 16, 17, 32):
                assert rq.decode_kernel_for(M, D, D, 4, 3) == kind
    # argument checks
    out = ctypes.c_int()
    assert L.rq_decode_kernel_for(0, D, D, 4, 1, ctypes.byref(out)) == rq.ERR_SHAPE
    assert L.rq_decode_kernel_for(33, D, D, 4, 1, ctypes.byref(out)) == rq.ERR_SHAPE
    assert L.rq_decode_kernel_for(1, 100, D, 4, 1, ctypes.byref(out)) == rq.ERR_SHAPE
    assert L.rq_decode_kernel_for(1, D, D, 4, 2, ctypes.byref(out)) == rq.ERR_SHAPE
    assert L.rq_decode_kernel_for(1, D, D, 5, 1, ctypes.byref(out)) == rq.ERR_BITS
    assert L.rq_decode_kernel_for(1, D, D, 4, 1, None) == rq.ERR_NULL


def test_quantize_ex2_argument_errors(L):
    """rq_quantize_g64_ex2 rejects bad arguments before any CUDA call."""
    p = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
    q = rq.lib().rq_quantize_g64_ex2
    assert q(p, 4, 128, 4, p, p, 0, p, p, None, None, None) == rq.ERR_RANGE     # nf = 0
    assert q(p, 4, 128, 4, p, p, 17, p, p, None, None, None) == rq.ERR_RANGE    # nf > 16
    assert q(p, 4, 128, 5, p, p, 4, p, p, None, None, None) == rq.ERR_BITS
    assert q(p, 4, 100, 4, p, p, 4, p, p, None, None, None) == rq.ERR_SHAPE
    assert q(p, 0, 128, 4, p, p, 4, p, p, None, None, None) == rq.ERR_SHAPE
    assert q(None, 4, 128, 4, p, p, 4, p, p, None, None, None) == rq.ERR_NULL
    assert q(p, 4, 128, 4, None, p, 4, p, p, None, None, None) == rq.ERR_NULL
    assert q(p, 4, 128, 4, p, None, 4, p, p, None, None, None) == rq.ERR_NULL
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert q(p, 4, 128, 4, odd, p, 4, p, p, None, None, None) == rq.ERR_ALIGN   # e2 not 16-B
    assert q(p, 4, 128, 4, p, ctypes.c_void_p((1 << 20) + 2), 4, p, p, None, None, None) == rq.ERR_ALIGN


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(rq, "_lib", None)
    monkeypatch.setattr(rq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        rq.lib()


def test_decode_variant_argument_errors(L):
    """rq_gemv_wq_ex and rq_rkv_fused3 reject bad arguments before any launch."""
    p = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 8)
    g = L.rq_gemv_wq_ex
    assert g(p, 1, 128, p, p, 64, 4, p, 2, 0, None) == rq.ERR_RANGE        # out dtype
    assert g(p, 1, 128, p, p, 64, 4, p, 0, 7, None) == rq.ERR_RANGE        # epilogue
    assert g(p, 33, 128, p, p, 64, 4, p, 0, 0, None) == rq.ERR_SHAPE       # M > 32
    assert g(p, 1, 100, p, p, 64, 4, p, 0, 0, None) == rq.ERR_SHAPE
    assert g(p, 1, 128, p, p, 64, 5, p, 0, 0, None) == rq.ERR_BITS
    assert g(None, 1, 128, p, p, 64, 4, p, 0, 0, None) == rq.ERR_NULL
    assert g(p, 1, 128, p, p, 64, 4, None, 0, 0, None) == rq.ERR_NULL
    assert g(p, 1, 128, p, p, 64, 4, odd, 1, 1, None) == rq.ERR_ALIGN
    f = L.rq_rkv_fused3
    assert f(p, p, p, 1, 128, 64, 4, p, p, p, p, p, p, p, p, p, 3, None) == rq.ERR_RANGE
    assert f(p, None, p, 1, 128, 64, 4, p, p, p, p, p, p, p, p, p, 0, None) == rq.ERR_NULL
    assert f(p, p, odd, 1, 128, 64, 4, p, p, p, p, p, p, p, p, p, 0, None) == rq.ERR_ALIGN
    assert f(p, p, p, 0, 128, 64, 4, p, p, p, p, p, p, p, p, p, 0, None) == rq.ERR_SHAPE
    assert f(p, p, p, 1, 128, 64, 4, p, p, p, p, p, None, p, p, p, 0, None) == rq.ERR_NULL


def test_preset_decode_argument_errors(L):
    """rq_gemv_p8_g16 / rq_gemv_p4a_g32 reject bad arguments before any launch."""
    p = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 8)
    g8 = L.rq_gemv_p8_g16
    assert g8(p, 1, 192, p, p, 64, p, None) == rq.ERR_SHAPE        # K % 128
    assert g8(p, 0, 128, p, p, 64, p, None) == rq.ERR_SHAPE
    assert g8(p, 33, 128, p, p, 64, p, None) == rq.ERR_SHAPE
    assert g8(p, 1, 128, p, p, 0, p, None) == rq.ERR_SHAPE
    assert g8(None, 1, 128, p, p, 64, p, None) == rq.ERR_NULL
    assert g8(p, 1, 128, p, None, 64, p, None) == rq.ERR_NULL
    assert g8(p, 1, 128, p, p, 64, None, None) == rq.ERR_NULL
    assert g8(odd, 1, 128, p, p, 64, p, None) == rq.ERR_ALIGN
    assert g8(p, 1, 128, odd, p, 64, p, None) == rq.ERR_ALIGN
    g4 = L.rq_gemv_p4a_g32
    assert g4(p, 1, 128, p, p, p, 64, p, None) == rq.ERR_SHAPE     # K % 256
    assert g4(p, 33, 256, p, p, p, 64, p, None) == rq.ERR_SHAPE
    assert g4(p, 1, 256, p, None, p, 64, p, None) == rq.ERR_NULL
    assert g4(p, 1, 256, p, p, None, 64, p, None) == rq.ERR_NULL
    assert g4(p, 1, 256, p, p, odd, 64, p, None) == rq.ERR_ALIGN
    assert g4(p, 1, 256, p, odd, p, 64, p, None) == rq.ERR_ALIGN


def test_gptq_argument_errors(L):
    p = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.rq_gptq_hessian(p, 10, 100, p, None) == rq.ERR_SHAPE
    assert L.rq_gptq_hessian(p, 0, 128, p, None) == rq.ERR_SHAPE
    assert L.rq_gptq_hessian(None, 10, 128, p, None) == rq.ERR_NULL
    assert L.rq_gptq_hessian(odd, 10, 128, p, None) == rq.ERR_ALIGN
    assert L.rq_gptq_factor(p, 128, -1.0, p, p, p, None) == rq.ERR_RANGE
    assert L.rq_gptq_factor(p, 100, 0.01, p, p, p, None) == rq.ERR_SHAPE
    assert L.rq_gptq_factor(p, 128, 0.01, p, None, p, None) == rq.ERR_NULL
    assert L.rq_gptq_g64(p, 4, 128, 5, p, None, p, p, p, None, None) == rq.ERR_BITS
    assert L.rq_gptq_g64(p, 4, 100, 4, p, None, p, p, p, None, None) == rq.ERR_SHAPE
    assert L.rq_gptq_g64(p, 4, 128, 4, None, None, p, p, p, None, None) == rq.ERR_NULL
    assert L.rq_gptq_g64(p, 4, 128, 4, p, None, p, p, odd, None, None) == rq.ERR_ALIGN
