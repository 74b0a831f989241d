"""GPU parity of the bf16-activation NVFP4 linear (the pages' f16a_nvfp4weight_scaled_mm in
its compiled form): the activation's amax, global scale and alpha and its quantized bytes
bit-exact against the oracle, the output within the GEMM tolerance of the oracle's fp64
reference, and the call equal to nvfp4_global_scale_quantize + nvfp4_gemm."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import assert_gemm_close, bf16_to_f64, dev_bf16, dev_f32, dev_u8, first_diff, host

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
