"""GPU parity of the bf16-activation NVFP4 linear (the pages' f16a_nvfp4weight_scaled_mm in
its compiled form): the activation's amax, global scale and alpha and its quantized bytes
bit-exact against the oracle, the output within the GEMM tolerance of the oracle's fp64
reference, and the call equal to nvfp4_global_scale_quantize + nvfp4_gemm.  With a static
(calibrated) activation scale, in both forms (two launches, and the one GEMM launch that
quantizes the activation itself): the quantized activation bit-exact against the oracle, the
output within the tolerance (and a faithful rounding at every tile for the large case), and
the two forms equal to nvfp4_quantize + nvfp4_gemm byte for byte on repeated calls."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import (assert_gemm_close, bf16_to_f64, check_full_size, dev_bf16, dev_f32, dev_u8, first_diff, host,
                           tile_positions)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    yield
    assert nv.nvfp4_device_status(clear=True) == 0


def _weight(oracle, n, k, seed):
    w = S.normal_bf16((n, k), 0.02, seed, S.TID["w"])
    amax_w, gsf_w = oracle.global_scale(w)
    qw, sfw = oracle.quantize(w, gsf_w)
    return amax_w, qw, sfw


@pytest.mark.parametrize("m,n,k,bias", [(1, 256, 64, False), (130, 384, 512, True), (300, 264, 1024, False),
                                         (1024, 1024, 2048, True)])
def test_bf16a_linear_matches_oracle(oracle, m, n, k, bias):
    x = S.normal_with_outliers_bf16((m, k), 0.01, 50.0, seed=m + n + k)
    amax_w, qw, sfw = _weight(oracle, n, k, m)
    b = S.normal_bf16((n,), 0.1, m, S.TID["bias"]) if bias else None
    out, aq, asf, sc = nv.nvfp4_gemm_bf16a(dev_bf16(x), dev_u8(qw), dev_u8(sfw), dev_f32(amax_w),
                                           dev_bf16(b) if bias else None)
    torch.cuda.synchronize()
    amax_x, gsf_x = oracle.global_scale(x)
    alpha = np.float32(oracle.alpha(float(amax_x), float(amax_w)))
    s = host(sc)
    assert s[0] == amax_x and s[1] == gsf_x and s[2] == alpha
    qx, sfx = oracle.quantize(x, gsf_x)
    assert first_diff(host(aq), qx) is None and first_diff(host(asf), sfx) is None
    ref = oracle.gemm_ref(qx, qw, sfx, sfw, alpha, m, n, k, bias=b)
    assert_gemm_close(bf16_to_f64(out), ref, f"bf16a {m}x{n}x{k}")


def test_bf16a_equals_the_two_calls(oracle):
    m, n, k = 513, 640, 768
    x = dev_bf16(S.normal_bf16((m, k), 2.0, 5, S.TID["x"]))
    amax_w, qw, sfw = _weight(oracle, n, k, 5)
    aw = dev_f32(amax_w)
    out, _, _, _ = nv.nvfp4_gemm_bf16a(x, dev_u8(qw), dev_u8(sfw), aw)
    _, _, alpha, q, sf = nv.nvfp4_global_scale_quantize(x, other_amax=aw)
    out2 = nv.nvfp4_gemm(q, dev_u8(qw), sf, dev_u8(sfw), alpha)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_bf16a_invalid_arguments_write_nothing(oracle):
    m, n, k = 128, 100, 256                         # n % 8 != 0: rejected before any launch
    x = dev_bf16(S.normal_bf16((m, k), 1.0, 6, S.TID["x"]))
    qw = torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda")
    sfw = torch.zeros(nv.nvfp4_scale_bytes(n, k), dtype=torch.uint8, device="cuda")
    aq = torch.full((m, k // 2), 7, dtype=torch.uint8, device="cuda")
    sc = torch.full((3,), -1.0, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_gemm_bf16a(x, qw, sfw, dev_f32(1.0), a_q_ws=aq, scalars_ws=sc)
    assert (host(aq) == 7).all() and (host(sc) == -1.0).all()


# ---- a static activation scale ------------------------------------------------------------------
# The activation's global scale is calibrated (448*6 / amax of a calibration batch).  In the
# one-launch form the GEMM kernel's epilogue warps quantize the activation into the workspace
# before draining any accumulator, and its producers load each K chunk once every slab's chunk
# is counted.

def _static_case(oracle, m, n, k, seed, calib_factor=1.25):
    x = S.normal_with_outliers_bf16((m, k), 0.01, 50.0, seed=seed)
    amax_w, qw, sfw = _weight(oracle, n, k, seed)
    amax_x, _ = oracle.global_scale(x)
    amax_c = np.float32(amax_x * np.float32(calib_factor))      # a calibrated amax (not this batch's)
    gsf = np.float32(np.float32(2688.0) / amax_c)
    alpha = np.float32(oracle.alpha(float(amax_c), float(amax_w)))
    return x, qw, sfw, gsf, alpha


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("m,n,k,bias", [(1, 256, 64, False), (130, 384, 512, True), (300, 264, 1024, False),
                                         (257, 520, 320, True), (1024, 1024, 2048, False), (2048, 4864, 6144, True)])
def test_bf16a_static_matches_oracle(oracle, m, n, k, bias, one_launch):
    x, qw, sfw, gsf, alpha = _static_case(oracle, m, n, k, seed=m + n + k)
    b = S.normal_bf16((n,), 0.1, m, S.TID["bias"]) if bias else None
    out, aq, asf = nv.nvfp4_gemm_bf16a_static(dev_bf16(x), dev_u8(qw), dev_u8(sfw), dev_f32(gsf), dev_f32(alpha),
                                              dev_bf16(b) if bias else None, one_launch=one_launch)
    torch.cuda.synchronize()
    # the quantized activation: every byte, the padding rows' zero scales included
    qx, sfx = oracle.quantize(x, gsf)
    assert first_diff(host(aq), qx) is None and first_diff(host(asf), sfx) is None
    if m * n <= 1 << 20:
        ref = oracle.gemm_ref(qx, qw, sfx, sfw, alpha, m, n, k, bias=b)
        assert_gemm_close(bf16_to_f64(out), ref, f"bf16a static {m}x{n}x{k}")
    else:
        ii, jj = tile_positions(m, n, 256, 256, seed=k)
        check_full_size(oracle, host(out), qx, sfx, qw, sfw, alpha, k, ii, jj, f"bf16a static {m}x{n}x{k}", bias=b)


@pytest.mark.parametrize("m,n,k", [(1000, 2048, 5120), (8192, 2048, 16384)])
def test_bf16a_static_forms_equal_quantize_then_gemm(oracle, m, n, k):
    # both forms give the bytes of nvfp4_quantize + nvfp4_gemm, on three calls in a row (the
    # one-launch kernel's chunk counters must be back at zero after every call); k = 16384 is
    # the one-launch form's largest (64 chunk counters)
    for call in range(3):
        x = S.normal_bf16((m, k), 1.0 + call, seed=40 + call)
        amax_w, qw, sfw = _weight(oracle, n, k, call)
        gsf, alpha = np.float32(2688.0 / (3.0 + call)), np.float32(1e-4)
        xd, wq, wsf, g, al = dev_bf16(x), dev_u8(qw), dev_u8(sfw), dev_f32(gsf), dev_f32(alpha)
        q2, sf2 = nv.nvfp4_quantize(xd, g)
        out2 = nv.nvfp4_gemm(q2, wq, sf2, wsf, al)
        for one_launch in (True, False):
            out, aq, asf = nv.nvfp4_gemm_bf16a_static(xd, wq, wsf, g, al, one_launch=one_launch)
            torch.cuda.synchronize()
            assert torch.equal(aq, q2) and torch.equal(asf, sf2) and torch.equal(out, out2), (call, one_launch)
        assert nv.nvfp4_device_status(clear=True) == 0


def test_bf16a_static_limits(oracle):
    # k > 16384: the one-launch form rejects it before anything is written
    m, k = 128, 64 * 257
    x = dev_bf16(S.normal_bf16((m, k), 1.0, 7, S.TID["x"]))
    qw = torch.zeros((128, k // 2), dtype=torch.uint8, device="cuda")
    sfw = torch.zeros(nv.nvfp4_scale_bytes(128, k), dtype=torch.uint8, device="cuda")
    aq = torch.full((m, k // 2), 7, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_gemm_bf16a_static(x, qw, sfw, dev_f32(1.0), dev_f32(1.0), a_q_ws=aq, one_launch=True)
    assert (host(aq) == 7).all()
    # n % 8 != 0: both forms reject it before anything is written
    for one_launch in (False, True):
        with pytest.raises(nv.NVFP4Error):
            nv.nvfp4_gemm_bf16a_static(x[:, :256].contiguous(), qw[:100, :128].contiguous(), sfw, dev_f32(1.0),
                                       dev_f32(1.0), a_q_ws=aq[:, :128].contiguous(), one_launch=one_launch)
    # n = 0: only the quantized activation is written
    x, qw, sfw, gsf, alpha = _static_case(oracle, 200, 8, 256, seed=8)
    for one_launch in (False, True):
        out, aq, asf = nv.nvfp4_gemm_bf16a_static(dev_bf16(x), dev_u8(qw[:0]), dev_u8(sfw[:0]), dev_f32(gsf),
                                                  dev_f32(alpha), one_launch=one_launch)
        qx, sfx = oracle.quantize(x, gsf)
        assert out.shape == (200, 0) and (host(aq) == qx).all() and (host(asf) == sfx).all()
