"""GPU parity: librq's sm_100a kernels against the CPU oracle, through the C ABI.

Quantizer: codes and scales bit-exact (and the device status).  Products:
|y_gpu - y_ref| <= 2e-3 * sum_k |x||w_hat| per output, the tolerance the
format's accuracy claim is held to here (fp16 rounding of code*scale, at most
2^-11 relative, plus fp32 accumulation).  Product tests feed the ORACLE's
codes to the GPU so they do not depend on the GPU quantizer.
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
    rq.set_pdl(False)
    yield
    assert rq.read_device_status(reset=True) == rq.OK


def to_host(t):
    return t.detach().cpu().numpy()


def oracle_weights(W_dev, bits):
    codes, scales, st = oracle.quantize_g64(to_host(W_dev), bits)
    assert st == 0
    return codes, scales


def upload(codes, scales):
    return (torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda())


def check_close(y_gpu, y_ref, bound, what):
    diff = np.abs(y_gpu.astype(np.float64) - y_ref)
    lim = TOL * bound
    bad = diff > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} outputs out of tolerance; worst "
                           f"diff {diff.max():.3e} vs limit {lim[np.unravel_index(diff.argmax(), diff.shape)]:.3e}")


# ------------------------------------------------------------- quantizer ---

@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(1, 64), (3, 128), (300, 640), (768, 768), (129, 4096)])
def test_quantizer_bit_exact(bits, N, K):
    W = synth.weights(N, K, seed=synth.seed_for(0, N, K % 7), device="cuda")
    codes, scales = rq.quantize_g64(W, bits)
    c_ref, s_ref, st = oracle.quantize_g64(to_host(W), bits)
    assert st == 0
    torch.cuda.synchronize()
    assert np.array_equal(to_host(scales).view(np.uint16), s_ref)
    assert np.array_equal(to_host(codes), c_ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantizer_special_values(bits):
    N, K = 8, 256
    W = synth.weights(N, K, seed=77, device="cpu")
    W[0, :64] = 0.0                                            # all-zero group
    W[1, :64] = 0.125 * (torch.arange(64) % 15 - 7).float()    # on grid, with ties below
    W[1, 1], W[1, 2], W[1, 3] = 0.3125, 0.4375, -0.3125
    W[2, 64:128] = 1e-9                                        # scale underflows to fp16 subnormal/0
    W[3, 5] = 1e6                                              # fp16 scale overflow -> RANGE
    W[4, 70] = float("nan")                                    # NONFINITE
    W[5, 200] = -float("inf")                                  # NONFINITE
    W[6, 128:192] = torch.linspace(-3e-5, 3e-5, 64)            # subnormal fp16 scales
    Wd = W.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = rq.quantize_g64(Wd, bits, dev_status=status)
    c_ref, s_ref, st = oracle.quantize_g64(W.numpy(), bits)
    torch.cuda.synchronize()
    assert int(status.item()) == st == oracle.STATUS_NONFINITE
    assert np.array_equal(to_host(scales).view(np.uint16), s_ref)
    assert np.array_equal(to_host(codes), c_ref)
    # RANGE alone
    W2 = synth.weights(4, 128, seed=78)
    W2[2, 100] = 3e7                                          # 3e7/127 > 65504 too
    status.zero_()
    codes2, scales2 = rq.quantize_g64(W2.cuda(), bits, dev_status=status)
    c2, s2, st2 = oracle.quantize_g64(W2.numpy(), bits)
    torch.cuda.synchronize()
    assert int(status.item()) == st2 == oracle.STATUS_RANGE
    assert np.array_equal(to_host(scales2).view(np.uint16), s2)
    assert np.array_equal(to_host(codes2), c2)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantizer_near_ties(bits):
    """Weights at and a few ulps around half-integer multiples of the scale,
    where w * (1/s) and the IEEE quotient w / s can round to different
    integers: exact scales (powers of two) and inexact ones, on both sides of
    every half-integer of the code range."""
    qmax = 7 if bits == 4 else 127
    rng = np.random.default_rng(91)
    groups = []
    for gi in range(512):
        # group max q_max * s sets the scale; exact for the first half
        s = np.float32(2.0 ** -rng.integers(2, 9)) if gi < 256 else np.float32(rng.uniform(1e-3, 0.2))
        g = np.empty(64, np.float32)
        g[0] = np.float32(qmax) * s * (1 if gi % 2 else -1)
        k = rng.integers(-qmax, qmax, size=63).astype(np.float32) + np.float32(0.5)
        base = (k * s).astype(np.float32)
        ulps = rng.integers(-6, 7, size=63)
        v = base.copy()
        for u in range(1, 7):       # move |ulps| steps towards +inf or -inf
            up = ulps >= u
            dn = ulps <= -u
            v[up] = np.nextafter(v[up], np.float32(np.inf))
            v[dn] = np.nextafter(v[dn], np.float32(-np.inf))
        g[1:] = v
        groups.append(g)
    W = np.stack(groups).reshape(16, 32 * 64)
    codes, scales = rq.quantize_g64(torch.from_numpy(W).cuda(), bits)
    c_ref, s_ref, st = oracle.quantize_g64(W, bits)
    torch.cuda.synchronize()
    assert st == 0
    assert np.array_equal(to_host(scales).view(np.uint16), s_ref)
    assert np.array_equal(to_host(codes), c_ref)


# -------------------------------------------------------------- products ---

def product_case(N, K, bits, M, seed, massive=None):
    W = synth.weights(N, K, seed=seed, device="cuda")
    x = synth.activations(M, K, seed=seed, device="cuda", massive_channel=massive)
    codes, scales = oracle_weights(W, bits)
    return x, codes, scales


DECODE_KERNELS = ["rowtile", "cluster", "rowblock", "tensor"]


def takes(kernel, M):
    """Whether a decode kernel takes batch M (all take 1 <= M <= 32)."""
    return 1 <= M <= 32


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 31, 32])
@pytest.mark.parametrize("N,K", [(300, 640), (1, 64), (129, 128), (256, 2048), (390, 1792), (256, 16384)])
def test_gemv_parity(kernel, bits, M, N, K):
    if not takes(kernel, M):
        pytest.skip("the row-block kernel takes M <= 16")
    x, codes, scales = product_case(N, K, bits, M, seed=1000 + M + N + K)
    cd, sd = upload(codes, scales)
    with rq.decode_kernel(kernel):
        y = rq.gemv_wq(x, cd, sd, N, bits)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul(to_host(x), codes, scales, bits)
    check_close(to_host(y), y_ref, bound, f"gemv {kernel} bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 3, 8, 16, 32])
@pytest.mark.parametrize("N,K", [(2400, 512), (5000, 256), (7500, 192), (16400, 128)])
def test_rowblock_tall_blocks(bits, M, N, K):
    """Every output of launches whose row blocks hold 2, 3, 4 and 7 m-tiles
    (the row-block kernel splits them over two halves of 16 warps at M <= 8,
    an odd count leaving the second half one short), ragged N included."""
    x, codes, scales = product_case(N, K, bits, M, seed=3000 + M + N)
    cd, sd = upload(codes, scales)
    with rq.decode_kernel("rowblock"):
        y = rq.gemv_wq(x, cd, sd, N, bits)
        y2 = rq.gemv_wq(x, cd, sd, N, bits)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    y_ref, bound = oracle.matmul(to_host(x), codes, scales, bits)
    check_close(to_host(y), y_ref, bound, f"rowblock bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8, 13, 32])
@pytest.mark.parametrize("N,K", [(200, 512), (256, 2048)])
def test_rkv_fused_parity(kernel, bits, M, N, K):
    if not takes(kernel, M):
        pytest.skip("the row-block kernel takes M <= 16")
    cases = [product_case(N, K, bits, M, seed=2000 + i) for i in range(3)]
    x = cases[0][0]
    ws = [upload(c[1], c[2]) for c in cases]
    with rq.decode_kernel(kernel):
        ys = rq.rkv_fused(x, ws[0], ws[1], ws[2], N, bits)
    torch.cuda.synchronize()
    for i in range(3):
        y_ref, bound = oracle.matmul(to_host(x), cases[i][1], cases[i][2], bits)
        check_close(to_host(ys[i]), y_ref, bound, f"rkv[{i}] {kernel} bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 64, 100, 256, 300])
def test_gemm_parity(bits, M):
    N, K = 384, 512
    x, codes, scales = product_case(N, K, bits, M, seed=3000 + M)
    cd, sd = upload(codes, scales)
    y = rq.gemm_wq(x, cd, sd, N, bits)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul(to_host(x), codes, scales, bits)
    check_close(to_host(y), y_ref, bound, f"gemm bits={bits} M={M}")


# Ragged shapes of the tensor-core product on full outputs: N not a multiple
# of the 128-row MMA tile (1, 129, 257, 300), a single k-block (K = 64), three
# (K = 192), a k-block count that no cluster split divides evenly (K = 64*37),
# and token counts that leave a partial token tile (65, 130, 2047).
GEMM_RAGGED = [
    (65, 1, 64), (65, 129, 192), (64, 300, 64 * 37), (130, 300, 64), (2047, 129, 512),
    (256, 129, 4096), (300, 257, 64 * 37), (1, 129, 192), (100, 1, 64 * 37), (2047, 1, 192),
]


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", GEMM_RAGGED)
def test_gemm_parity_ragged(bits, M, N, K):
    x, codes, scales = product_case(N, K, bits, M, seed=3100 + M + N + K)
    cd, sd = upload(codes, scales)
    y = rq.gemm_wq(x, cd, sd, N, bits)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul(to_host(x), codes, scales, bits)
    check_close(to_host(y), y_ref, bound, f"gemm ragged bits={bits} M={M} N={N} K={K}")


def test_unit_vectors_pick_columns():
    """x = e_j returns column j of the dequantised weight (exact up to fp32)."""
    N, K, bits = 130, 192, 4
    W = synth.weights(N, K, seed=9, device="cuda")
    codes, scales = oracle_weights(W, bits)
    cd, sd = upload(codes, scales)
    js = [0, 1, 63, 64, 127, 191]
    x = torch.zeros((len(js), K), dtype=torch.float16, device="cuda")
    for i, j in enumerate(js):
        x[i, j] = 1.0
    y = to_host(rq.gemv_wq(x, cd, sd, N, bits))
    s = scales.view(np.float16).astype(np.float64)
    for i, j in enumerate(js):
        col = np.array([oracle.get_code(codes, K, bits, n, j) for n in range(N)]) * s[:, j // 64]
        # fp16(code*s) is what the tensor core sees: within 2^-11 relative of code*s
        assert np.all(np.abs(y[i] - col) <= np.abs(col) * 2.0 ** -11 + 1e-12)


def test_quantize_then_product_chain():
    """GPU quantizer feeding GPU products on the same stream."""
    N, K, bits, M = 512, 1024, 4, 5
    W = synth.weights(N, K, seed=11, device="cuda")
    x = synth.activations(M, K, seed=11, device="cuda")
    codes, scales = rq.quantize_g64(W, bits)
    y = rq.gemv_wq(x, codes, scales, N, bits)
    torch.cuda.synchronize()
    c_ref, s_ref, _ = oracle.quantize_g64(to_host(W), bits)
    y_ref, bound = oracle.matmul(to_host(x), c_ref, s_ref, bits)
    check_close(to_host(y), y_ref, bound, "quantize->gemv")


# ------------------------------------------ configuration shapes, sampled ---

def sampled_check(y, x, codes_dev, scales_dev, N, K, bits, n_samples=512, seed=0, rows=None):
    """Compare sampled outputs; rows of the weight are pulled to the host only
    for the sampled n."""
    M = x.shape[0]
    rng = np.random.default_rng(seed)
    ns = rng.integers(0, N, size=n_samples)
    ns[:4] = [0, N - 1, N // 2, 127 % N]
    ms = rng.integers(0, M, size=n_samples)
    ms[:2] = [0, M - 1]
    uniq = np.unique(ns)
    sub_c = to_host(codes_dev[torch.from_numpy(uniq).cuda()])
    sub_s = to_host(scales_dev[torch.from_numpy(uniq).cuda()]).view(np.uint16)
    remap = {int(n): i for i, n in enumerate(uniq)}
    ns_local = np.array([remap[int(n)] for n in ns])
    y_ref, bound = oracle.matmul_sampled(to_host(x), sub_c, sub_s, bits, ms, ns_local)
    yg = to_host(y)[ms, ns]
    check_close(yg, y_ref, bound, f"sampled N={N} K={K} bits={bits} M={M}")


def quantize_checked(W, bits, sample_rows=64, seed=0):
    """GPU quantizer, with a bit-exact oracle check on sampled rows."""
    codes, scales = rq.quantize_g64(W, bits)
    N = W.shape[0]
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, size=sample_rows)]))
    Wr = to_host(W[torch.from_numpy(rows).cuda()])
    c_ref, s_ref, st = oracle.quantize_g64(Wr, bits)
    assert st == 0
    idx = torch.from_numpy(rows).cuda()
    assert np.array_equal(to_host(codes[idx]), c_ref)
    assert np.array_equal(to_host(scales[idx]).view(np.uint16), s_ref)
    return codes, scales


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
@pytest.mark.parametrize("wl", [1, 2, 3, 5])
def test_decode_workload_shapes(kernel, wl):
    w = synth.WORKLOADS[wl]
    for pi, pj in enumerate(w.projs):
        W = synth.weights(pj.N, pj.K, seed=synth.seed_for(wl, 0, pi), device="cuda")
        codes, scales = quantize_checked(W, w.bits, seed=pi)
        del W
        for M in w.Ms:
            if not takes(kernel, M):
                continue
            x = synth.activations(M, pj.K, seed=synth.seed_for(wl, 0, pi) + M, device="cuda",
                                  massive_channel=w.massive_channel)
            with rq.decode_kernel(kernel):
                y = rq.gemv_wq(x, codes, scales, pj.N, w.bits)
            torch.cuda.synchronize()
            sampled_check(y, x, codes, scales, pj.N, pj.K, w.bits, seed=M)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_decode_workload_rkv_fused(kernel):
    for wl in (2, 3, 5):
        w = synth.WORKLOADS[wl]
        D = w.projs[0].N
        ws = []
        for pi in range(3):
            W = synth.weights(D, D, seed=synth.seed_for(wl, 1, pi), device="cuda")
            ws.append(rq.quantize_g64(W, w.bits))
            del W
        for M in (w.Ms[0], w.Ms[-1]):
            if not takes(kernel, M):
                M = 16
            x = synth.activations(M, D, seed=M, device="cuda", massive_channel=w.massive_channel)
            with rq.decode_kernel(kernel):
                ys = rq.rkv_fused(x, ws[0], ws[1], ws[2], D, w.bits)
            torch.cuda.synchronize()
            for i in range(3):
                sampled_check(ys[i], x, ws[i][0], ws[i][1], D, D, w.bits, n_samples=256, seed=i)


def test_prefill_workload_shapes():
    w = synth.WORKLOADS[4]
    for pi, pj in enumerate(w.projs):
        W = synth.weights(pj.N, pj.K, seed=synth.seed_for(4, 0, pi), device="cuda")
        codes, scales = quantize_checked(W, w.bits, seed=pi)
        del W
        for M in w.Ms:
            x = synth.activations(M, pj.K, seed=M + pi, device="cuda")
            y = rq.gemm_wq(x, codes, scales, pj.N, w.bits)
            torch.cuda.synchronize()
            sampled_check(y, x, codes, scales, pj.N, pj.K, w.bits, n_samples=384, seed=M)


# ------------------------------------------------------------ robustness ---

def test_bounded_wait_times_out_cleanly():
    """A wait nothing completes gives up, reports RQ_ERR_TIMEOUT, and the
    context stays usable."""
    assert rq.read_device_status(reset=True) == rq.OK
    rq.selftest_bounded_wait(50_000_000)        # 50 ms
    torch.cuda.synchronize()
    assert rq.read_device_status(reset=True) == rq.ERR_TIMEOUT
    # the context still works
    x, codes, scales = product_case(128, 128, 4, 1, seed=5)
    cd, sd = upload(codes, scales)
    y = rq.gemv_wq(x, cd, sd, 128, 4)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul(to_host(x), codes, scales, 4)
    check_close(to_host(y), y_ref, bound, "after timeout")
    assert rq.read_device_status() == rq.OK


@pytest.mark.parametrize("kernel,M", [("rowtile", 4), ("cluster", 4), ("cluster", 24),
                                      ("rowblock", 4), ("rowblock", 13), ("tensor", 4),
                                      ("tensor", 24)])
def test_pdl_chain_matches(kernel, M):
    """With programmatic dependent launch on, a chain of dependent products
    (each reading the previous output as its input) still matches."""
    N = K = 512
    bits = 4
    W = [synth.weights(N, K, seed=40 + i, device="cuda") for i in range(3)]
    qs = [rq.quantize_g64(w, bits) for w in W]
    torch.cuda.synchronize()
    x0 = synth.activations(M, K, seed=40, device="cuda")
    rq.set_pdl(True)
    try:
        with rq.decode_kernel(kernel):
            x = x0
            outs = []
            for c, s in qs:
                y = rq.gemv_wq(x, c, s, N, bits)
                x = (y * 0.05).to(torch.float16)   # torch op between: still ordered
                outs.append(y)
        torch.cuda.synchronize()
    finally:
        rq.set_pdl(False)
    xh = to_host(x0)
    for i, (c, s) in enumerate(qs):
        ch, sh = to_host(c), to_host(s).view(np.uint16)
        y_ref, bound = oracle.matmul(xh, ch, sh, bits)
        check_close(to_host(outs[i]), y_ref, bound, f"pdl chain {i}")
        xh = (to_host(outs[i]) * 0.05).astype(np.float16)


# ------------------------------------------------------------ repeatability ---

@pytest.mark.parametrize("path", ["gemv", "gemv-cluster", "gemv-cluster-m32", "gemv-rowblock",
                                  "gemv-rowblock-m16", "gemv-tensor", "gemv-tensor-m32",
                                  "gemv-tensor-fused", "gemm"])
def test_repeat_runs_bit_identical(path):
    """Every kernel sums in a fixed order, so repeated runs must agree bit for
    bit; a pipeline race (a stage read before or after its data) shows up here
    even when it stays within tolerance."""
    kernel = ("cluster" if path.startswith("gemv-cluster") else
              "rowblock" if path.startswith("gemv-rowblock") else
              "tensor" if path.startswith("gemv-tensor") else "rowtile")
    if path == "gemv-tensor-fused":
        # three matrices, partial row blocks across CTAs and matrices
        N, K, M, bits = 2048, 2048, 24, 4
        qs = [rq.quantize_g64(synth.weights(N, K, seed=33 + i, device="cuda"), bits) for i in range(3)]
        x = synth.activations(M, K, seed=33, device="cuda")
        with rq.decode_kernel(kernel):
            ref = rq.rkv_fused(x, *qs, N, bits)
            torch.cuda.synchronize()
            for _ in range(20):
                ys = rq.rkv_fused(x, *qs, N, bits)
                torch.cuda.synchronize()
                for a, b in zip(ys, ref):
                    assert torch.equal(a.view(torch.int32), b.view(torch.int32)), path
        return
    if path == "gemm":
        N, K, M, bits = 1024, 8192, 512, 4
    elif path == "gemv-cluster-m32":
        N, K, M, bits = 2048, 8192, 32, 4
    elif path == "gemv-rowblock-m16":
        N, K, M, bits = 16384, 4096, 16, 4
    elif path == "gemv-tensor-m32":
        N, K, M, bits = 16384, 4096, 32, 4
    else:
        N, K, M, bits = 4096, 4096, 5, 4
    W = synth.weights(N, K, seed=31, device="cuda")
    codes, scales = rq.quantize_g64(W, bits)
    x = synth.activations(M, K, seed=31, device="cuda")
    fn = rq.gemm_wq if path == "gemm" else rq.gemv_wq
    with rq.decode_kernel(kernel):
        ref = fn(x, codes, scales, N, bits)
        torch.cuda.synchronize()
        for _ in range(20):
            y = fn(x, codes, scales, N, bits)
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
