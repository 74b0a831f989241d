"""GPU parity at the limits the entry points accept: the largest expert count of the
grouped GEMM (1024) with empty, partial and full experts, a grouped call whose every mask
is 0, the largest batch of the per-item global scale (4096 items), a very long K (32768)
and very wide quantizer rows (k = 65536)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import assert_gemm_close, bf16_to_f64, dev_bf16, dev_f32, dev_i32, dev_u8, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    yield


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert nv.nvfp4_device_status(clear=True) == 0, "a device-side wait timed out"


def test_grouped_gemm_1024_experts(oracle):
    E, mmax, n, k = 1024, 128, 64, 64
    a = S.normal_bf16((E, mmax, k), 1.0, 41, S.TID["x"])
    w = S.normal_bf16((E, n, k), 0.05, 41, S.TID["w"])
    mask = S.rng(41, S.TID["mask"]).integers(0, mmax + 1, E).astype(np.int32)
    mask[:3] = [0, mmax, 1]
    _, ga = oracle.global_scale_batched(a, mask)
    _, gw = oracle.global_scale_batched(w, None)
    qa, sfa = oracle.quantize_masked_batched(a, ga, mask)
    qw, sfw = oracle.quantize_masked_batched(w, gw, None)
    alphas = S.rng(41, S.TID["sample"]).uniform(0.5, 2.0, E).astype(np.float32)
    out = torch.full((E, mmax, n), -5.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(dev_u8(qa), dev_u8(qw), dev_u8(sfa), dev_u8(sfw), dev_i32(mask), dev_f32(alphas),
                                 out)
    ref = oracle.grouped_gemm_ref(qa, qw, sfa, sfw, mask, alphas, E, mmax, n, k)
    o = bf16_to_f64(out)
    for e in (0, 1, 2, 511, 1023):
        v = int(mask[e])
        assert_gemm_close(o[e, :v], ref[e, :v], f"expert {e}")
        assert (o[e, v:] == -5.0).all()
    valid = ~np.isnan(ref)
    assert_gemm_close(o[valid], ref[valid], "all experts")
    assert (o[~valid] == -5.0).all()


def test_grouped_gemm_all_masks_zero():
    E, mmax, n, k = 8, 256, 256, 128
    qa = torch.zeros((E, mmax, k // 2), dtype=torch.uint8, device="cuda")
    qw = torch.zeros((E, n, k // 2), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((E, nv.nvfp4_scale_bytes(mmax, k)), dtype=torch.uint8, device="cuda")
    sfw = torch.zeros((E, nv.nvfp4_scale_bytes(n, k)), dtype=torch.uint8, device="cuda")
    out = torch.full((E, mmax, n), 9.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(qa, qw, sfa, sfw, dev_i32(np.zeros(E, np.int32)), dev_f32(np.ones(E)), out)
    assert (out == 9.0).all()


def test_global_scale_4096_items(oracle):
    b, m, k = 4096, 5, 32
    x = S.normal_bf16((b, m, k), 1.0, 43, S.TID["x"])
    mask = S.rng(43, S.TID["mask"]).integers(0, m + 1, b).astype(np.int32)
    amax, gsf = nv.nvfp4_global_scale_batched(dev_bf16(x), dev_i32(mask))
    amax_ref, gsf_ref = oracle.global_scale_batched(x, mask)
    assert (host(amax) == amax_ref).all() and (host(gsf) == gsf_ref).all()


def test_gemm_long_k(oracle):
    m, n, k = 256, 256, 32768
    xa = S.normal_bf16((m, k), 1.0, 44, S.TID["x"])
    xb = S.normal_bf16((n, k), 0.02, 44, S.TID["w"])
    am_a, ga = oracle.global_scale(xa)
    am_b, gb = oracle.global_scale(xb)
    qa, sfa = oracle.quantize(xa, ga)
    qb, sfb = oracle.quantize(xb, gb)
    alpha = np.float32(oracle.alpha(float(am_a), float(am_b)))
    out = nv.nvfp4_gemm(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha))
    assert_gemm_close(bf16_to_f64(out), oracle.gemm_ref(qa, qb, sfa, sfb, alpha, m, n, k), "k=32768")


def test_quantize_wide_rows(oracle):
    m, k = 3, 65536
    x = S.normal_with_outliers_bf16((m, k), 0.001, 50.0, 45, S.TID["x"])
    _, gsf = oracle.global_scale(x)
    q, sf = nv.nvfp4_quantize(dev_bf16(x), dev_f32(gsf))
    q_ref, sf_ref = oracle.quantize(x, gsf)
    assert (host(q) == q_ref).all() and (host(sf) == sf_ref).all()


@pytest.mark.parametrize("silu", [False, True])
def test_masked_quantize_1024_items(oracle, silu):
    # 1024 items of 5 rows: one chunk per item, so the persistent grid changes item (and
    # rebuilds its table of inverse scales) on almost every chunk; masks 0..5
    b, m, k = 1024, 5, 32
    x = S.normal_with_outliers_bf16((b, m, 2 * k if silu else k), 0.01, 50.0, 46, S.TID["x"])
    mask = S.rng(46, S.TID["mask"]).integers(0, m + 1, b).astype(np.int32)
    mask[:2] = [0, m]
    _, gsf = oracle.global_scale_batched(x, mask, silu_mul=silu)
    q = torch.full((b, m, k // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((b, nv.nvfp4_scale_bytes(m, k)), 0x5A, dtype=torch.uint8, device="cuda")
    fn = nv.nvfp4_silu_mul_quantize_batched if silu else nv.nvfp4_quantize_masked_batched
    fn(dev_bf16(x), dev_f32(gsf), dev_i32(mask), q, sf)
    q_ref, sf_ref = (oracle.silu_mul_quantize_batched if silu else oracle.quantize_masked_batched)(
        x, gsf, mask, q_fill=0xA5, sf_fill=0x5A)
    assert (host(q) == q_ref).all() and (host(sf) == sf_ref).all()
