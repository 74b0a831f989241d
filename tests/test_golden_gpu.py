"""The CUDA path against the hand-worked example in tests/golden/nvfp4_worked_example.txt.

The fixture was derived by hand from the format definitions and the pages' formulas, so
these tests hold the kernels to values no program produced: the fused global-scale
quantizer, the dense quantizer with a given global scale (every packed byte and every
scale byte, padding included), the block-scaled FP4 GEMM (exact bf16 outputs, since the
fixture's sums lie far from any bf16 rounding midpoint), and the SiLU-and-mul, masked,
smooth, low-rank, masked grouped, fused gate/up SiLU-and-mul, LoRA-down, bf16-activation
and SiLU-and-mul-only variants on inputs whose results follow from the example by hand."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
from tests.helpers import (assert_gemm_close, bf16_to_f64, dev_bf16, dev_f32, dev_i32, grouped_expectation, host,
                           load_worked_example, lora_expectation, lowrank_expectation, masked_expectations, ones_rows,
                           swiglu_expectation, swiglu_grouped_expectation, worked_variants)

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


@pytest.fixture(scope="module")
def ex():
    return load_worked_example()


def test_global_scale_quantize(ex):
    amax, gsf, alpha, q, sf = nv.nvfp4_global_scale_quantize(dev_bf16(ex["x"]), other_amax=dev_f32(ex["amax"]))
    assert host(amax)[0] == ex["amax"] and host(gsf)[0] == ex["gsf"]
    assert host(alpha)[0] == np.float32(1.0)
    assert np.array_equal(host(q), ex["q"])
    assert np.array_equal(host(sf), ex["sf"])


def test_global_scale(ex):
    amax, gsf, alpha = nv.nvfp4_global_scale(dev_bf16(ex["x"]), other_amax=dev_f32(ex["ones_amax"]))
    assert host(amax)[0] == ex["amax"] and host(gsf)[0] == ex["gsf"]
    assert host(alpha)[0] == np.float32(1.0 / 2688.0)
    # batched over two items with masks 34 and 33: the second item's valid rows end just
    # before the worked row, so it sees only zeros and its amax is clamped to 1e-12
    amax, gsf = nv.nvfp4_global_scale_batched(dev_bf16(np.stack([ex["x"], ex["x"]])), mask=dev_i32([34, 33]))
    assert list(host(amax)) == [np.float32(ex["amax"]), np.float32(1e-12)]
    assert list(host(gsf)) == [np.float32(ex["gsf"]), np.float32(2688.0) / np.float32(1e-12)]


def test_quantize(ex):
    q = torch.full((ex["rows"], ex["k"] // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((ex["sf"].size,), 0xAA, dtype=torch.uint8, device="cuda")
    nv.nvfp4_quantize(dev_bf16(ex["x"]), dev_f32(ex["gsf"]), q, sf)
    assert np.array_equal(host(q), ex["q"])
    assert np.array_equal(host(sf), ex["sf"])


def test_gemm(ex):
    rows, k, row = ex["rows"], ex["k"], ex["row"]
    qa, sfa = nv.nvfp4_quantize(dev_bf16(ex["x"]), dev_f32(ex["gsf"]))
    out = nv.nvfp4_gemm(qa, qa, sfa, sfa, dev_f32(1.0))
    want = np.zeros((rows, rows))
    want[row, row] = ex["gemm_self_bf16"]
    assert np.array_equal(bf16_to_f64(out), want)

    ones = dev_bf16(ones_rows(8, k))
    amax_b, gsf_b, alpha, qb, sfb = nv.nvfp4_global_scale_quantize(ones, other_amax=dev_f32(ex["amax"]))
    assert host(amax_b)[0] == ex["ones_amax"] and host(gsf_b)[0] == ex["ones_gsf"]
    assert np.all(host(qb) == ex["ones_code"] * 0x11)
    assert host(alpha)[0] == np.float32(1.0 / 2688.0)
    out = bf16_to_f64(nv.nvfp4_gemm(qa, qb, sfa, sfb, alpha))
    want = np.zeros((rows, 8))
    want[row, :] = ex["gemm_ones_bf16"]
    assert np.array_equal(out, want)
    ref = np.zeros((rows, 8))
    ref[row, :] = ex["gemm_ones"]
    assert_gemm_close(out, ref, "worked example, ones operand")


def test_silu_mul_variant(ex):
    v = worked_variants(ex)
    x = dev_bf16(v["silu_x"])
    amax, gsf = nv.nvfp4_global_scale_batched(x, silu_mul=True)
    assert host(amax)[0] == ex["amax"] and host(gsf)[0] == ex["gsf"]
    q = torch.full((1, ex["rows"], ex["k"] // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((1, ex["sf"].size), 0xAA, dtype=torch.uint8, device="cuda")
    nv.nvfp4_silu_mul_quantize_batched(x, gsf, q_out=q, sf_out=sf)
    assert np.array_equal(host(q)[0], ex["q"]) and np.array_equal(host(sf)[0], ex["sf"])


def test_masked_variant(ex):
    q = torch.full((1, ex["rows"], ex["k"] // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((1, ex["sf"].size), 0xAA, dtype=torch.uint8, device="cuda")
    nv.nvfp4_quantize_masked_batched(dev_bf16(ex["x"][None]), dev_f32(ex["gsf"]), mask=dev_i32([ex["mask"]]),
                                     q_out=q, sf_out=sf)
    q_want, sf_want = masked_expectations(ex, 0xAA)
    assert np.array_equal(host(q)[0], q_want) and np.array_equal(host(sf)[0], sf_want)


def test_smooth_variant(ex):
    v = worked_variants(ex)
    q, sf = nv.nvfp4_quantize_smooth(dev_bf16(v["smooth_x"]), dev_bf16(v["pqs"]), dev_f32(ex["gsf"]))
    assert np.array_equal(host(q), ex["q"]) and np.array_equal(host(sf), ex["sf"])


def test_lowrank_variant(ex):
    v = worked_variants(ex)
    qa, sfa = nv.nvfp4_quantize(dev_bf16(ex["x"]), dev_f32(ex["gsf"]))
    out = nv.nvfp4_gemm_lowrank_bias(qa, qa, sfa, sfa, dev_f32(1.0), dev_bf16(v["d"]), dev_bf16(v["l1"]),
                                     dev_bf16(v["bias"]))
    assert np.array_equal(bf16_to_f64(out), lowrank_expectation(ex, exact=False))


def _ones_operand(ex, n):
    _, _, alpha, qb, sfb = nv.nvfp4_global_scale_quantize(dev_bf16(ones_rows(n, ex["k"])),
                                                          other_amax=dev_f32(ex["amax"]))
    return qb, sfb, host(alpha)[0]


def test_grouped_variant(ex):
    rows = ex["rows"]
    qa, sfa = nv.nvfp4_quantize(dev_bf16(ex["x"]), dev_f32(ex["gsf"]))
    qb, sfb, _ = _ones_operand(ex, 8)
    alphas = np.float32([m / 2688.0 for m in ex["grouped_alpha_mult"]])
    out = torch.full((2, rows, 8), -1.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(torch.stack([qa, qa]), torch.stack([qb, qb]), torch.stack([sfa, sfa]),
                                 torch.stack([sfb, sfb]), dev_i32(ex["grouped_mask"]), dev_f32(alphas), out=out)
    assert np.array_equal(bf16_to_f64(out), grouped_expectation(ex, -1.0))


def test_swiglu_variant(ex):
    rows, n = ex["rows"], ex["swiglu_n"]
    qa, sfa = nv.nvfp4_quantize(dev_bf16(ex["x"]), dev_f32(ex["gsf"]))
    qb, sfb, alpha_g = _ones_operand(ex, n)
    alpha_u = np.float32(alpha_g / np.float32(ex["swiglu_up_div"]))
    gsf_h = np.float32(np.float32(2688.0) / np.float32(ex["swiglu_h"]))
    q = torch.full((rows, n // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((ex["swiglu_sf_bytes"],), 0xAA, dtype=torch.uint8, device="cuda")
    nv.nvfp4_gemm_silu_mul_quantize(qa, qb, qb, sfa, sfb, sfb, dev_f32(alpha_g), dev_f32(alpha_u), dev_f32(gsf_h),
                                    q_out=q, sf_out=sf)
    q_want, sf_want = swiglu_expectation(ex)
    assert np.array_equal(host(q), q_want) and np.array_equal(host(sf), sf_want)

    two = lambda t: torch.stack([t, t])
    q = torch.full((2, rows, n // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((2, ex["swiglu_sf_bytes"]), 0xAA, dtype=torch.uint8, device="cuda")
    nv.nvfp4_grouped_gemm_silu_mul_quantize_masked(two(qa), two(qb), two(qb), two(sfa), two(sfb), two(sfb),
                                                   dev_i32(ex["swiglu_grouped_mask"]), dev_f32([alpha_g] * 2),
                                                   dev_f32([alpha_u] * 2), dev_f32([gsf_h] * 2), q_out=q, sf_out=sf)
    q_want, sf_want = swiglu_grouped_expectation(ex, 0xAA)
    assert np.array_equal(host(q), q_want) and np.array_equal(host(sf), sf_want)


def test_lora_down_variant(ex):
    v = worked_variants(ex)
    want = lora_expectation(ex, ex["row_sum_bf16"])
    d = nv.nvfp4_lora_down(dev_bf16(ex["x"]), dev_bf16(v["lora_w"]))
    assert np.array_equal(bf16_to_f64(d), want)
    q, sf, d = nv.nvfp4_quantize_smooth_lora_down(dev_bf16(v["smooth_x"]), dev_bf16(v["pqs"]), dev_f32(ex["gsf"]),
                                                  dev_bf16(v["lora_w_scaled"]))
    assert np.array_equal(host(q), ex["q"]) and np.array_equal(host(sf), ex["sf"])
    assert np.array_equal(bf16_to_f64(d), want)


def test_bf16a_variant(ex):
    qb, sfb, _ = _ones_operand(ex, 8)
    out, a_q, a_sf, scalars = nv.nvfp4_gemm_bf16a(dev_bf16(ex["x"]), qb, sfb, dev_f32(ex["ones_amax"]))
    assert list(host(scalars)) == [np.float32(ex["amax"]), np.float32(ex["gsf"]), np.float32(1.0 / 2688.0)]
    assert np.array_equal(host(a_q), ex["q"]) and np.array_equal(host(a_sf), ex["sf"])
    want = np.zeros((ex["rows"], 8))
    want[ex["row"], :] = ex["gemm_ones_bf16"]
    assert np.array_equal(bf16_to_f64(out), want)


def test_silu_and_mul_variant(ex):
    v = worked_variants(ex)
    h = nv.nvfp4_silu_and_mul(dev_bf16(v["silu_x"][0]))
    assert np.array_equal(host(h), ex["x"])
