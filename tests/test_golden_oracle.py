"""The oracle against the hand-worked example in tests/golden/nvfp4_worked_example.txt.

The fixture's values were derived with pencil and paper from the format definitions and
the pages' formulas (its header gives the sources and each step), not by a program, so
these tests pin the oracle's global scale, quantizer, scale layout, dequantization and
GEMM reference to something other than the oracle, and its SiLU-and-mul, masked, smooth,
low-rank, masked grouped, fused gate/up SiLU-and-mul and LoRA-down variants to inputs built so that
their results follow from the example by hand.  The first
test checks the fixture against itself (codes x scales = dequantized values, the padded
scale size, the sums)."""
import numpy as np
import pytest
import torch

from tests.helpers import (E2M1, e4m3_values, grouped_expectation, load_worked_example, lora_expectation,
                           lowrank_expectation, masked_expectations, ones_rows, swiglu_expectation, swiglu_grouped_expectation,
                           worked_variants)


@pytest.fixture(scope="module")
def ex():
    return load_worked_example()


def test_fixture_is_consistent(ex):
    k = ex["k"]
    s = np.repeat(e4m3_values(ex["scales"]), 16)
    assert np.array_equal(E2M1[ex["codes"]] * s, ex["dq"])
    # padded scale size pad_up(rows, 128) * pad_up(k/16, 4)
    assert ex["sf"].size == (-(-ex["rows"] // 128) * 128) * (-(-(k // 16) // 4) * 4)
    assert ex["amax"] == np.abs(ex["x_values"]).max()
    assert ex["gsf"] == 448.0 * 6.0 / ex["amax"]
    assert ex["gemm_self"] == float(np.dot(ex["dq"], ex["dq"]))
    assert ex["gemm_ones"] == float(ex["dq"].sum())
    for exact, rounded in [(ex["gemm_self"], ex["gemm_self_bf16"]), (ex["gemm_ones"], ex["gemm_ones_bf16"])]:
        assert torch.tensor(exact, dtype=torch.float64).to(torch.bfloat16).item() == rounded


def test_oracle_global_scale(oracle, ex):
    amax, gsf = oracle.global_scale(ex["x"])
    assert float(amax) == ex["amax"] and float(gsf) == ex["gsf"]
    ones = np.full((8, ex["k"]), 0x3F80, np.uint16)        # bf16 1.0
    amax_b, gsf_b = oracle.global_scale(ones)
    assert float(amax_b) == ex["ones_amax"] and float(gsf_b) == ex["ones_gsf"]
    # two items with masks 34 and 33: the second sees only zero rows, amax clamps to 1e-12
    # (the clamp the FastVideo review thread's global-scale helper applies)
    amax2, gsf2 = oracle.global_scale_batched(np.stack([ex["x"], ex["x"]]), np.int32([34, 33]))
    assert list(amax2) == [np.float32(ex["amax"]), np.float32(1e-12)]
    assert list(gsf2) == [np.float32(ex["gsf"]), np.float32(2688.0) / np.float32(1e-12)]
    assert np.float32(oracle.alpha(ex["amax"], ex["amax"])) == np.float32(1.0)
    assert np.float32(oracle.alpha(ex["amax"], ex["ones_amax"])) == np.float32(1.0 / 2688.0)


def test_oracle_quantize(oracle, ex):
    q, sf = oracle.quantize(ex["x"], ex["gsf"], sf_fill=0xAA)
    assert np.array_equal(q, ex["q"])
    assert np.array_equal(sf, ex["sf"])


def test_oracle_dequantize(oracle, ex):
    q, sf = oracle.quantize(ex["x"], ex["gsf"])
    dq = oracle.dequantize_logical(q, sf, ex["rows"], ex["k"])
    assert np.array_equal(dq[ex["row"]], ex["dq"])
    assert not np.any(np.delete(dq, ex["row"], axis=0))


def test_oracle_gemm(oracle, ex):
    rows, k, row = ex["rows"], ex["k"], ex["row"]
    q, sf = oracle.quantize(ex["x"], ex["gsf"])
    out = oracle.gemm_ref(q, q, sf, sf, oracle.alpha(ex["amax"], ex["amax"]), rows, rows, k)
    want = np.zeros((rows, rows))
    want[row, row] = ex["gemm_self"]
    assert np.array_equal(out, want)
    bits = torch.tensor([ex["gemm_self_bf16"]], dtype=torch.bfloat16).view(torch.int16).item() & 0xFFFF
    assert oracle.f64_to_bf16(ex["gemm_self"]) == bits

    ones = np.full((8, k), 0x3F80, np.uint16)
    qb, sfb = oracle.quantize(ones, ex["ones_gsf"])
    assert np.all(qb == ex["ones_code"] * 0x11)
    assert np.all(sfb.reshape(-1)[[r * 16 + c for r in range(8) for c in range(4)]] == ex["ones_scale"])
    alpha = np.float32(oracle.alpha(ex["amax"], ex["ones_amax"]))
    out = oracle.gemm_ref(q, qb, sf, sfb, alpha, rows, 8, k)
    # alpha is 1/2688 rounded to fp32; every other factor is exact
    assert np.allclose(out[row], ex["gemm_ones"], rtol=2.0 ** -23, atol=0)
    assert not np.any(np.delete(out, row, axis=0))


def test_oracle_silu_mul_variant(oracle, ex):
    v = worked_variants(ex)
    amax, gsf = oracle.global_scale_batched(v["silu_x"], None, silu_mul=True)
    assert float(amax[0]) == ex["amax"] and float(gsf[0]) == ex["gsf"]
    q, sf = oracle.silu_mul_quantize_batched(v["silu_x"], gsf, q_fill=0xAA, sf_fill=0xAA)
    assert np.array_equal(q[0], ex["q"]) and np.array_equal(sf[0], ex["sf"])


def test_oracle_masked_variant(oracle, ex):
    q, sf = oracle.quantize_masked_batched(ex["x"][None], np.float32([ex["gsf"]]),
                                           mask=np.int32([ex["mask"]]), q_fill=0xAA, sf_fill=0xAA)
    q_want, sf_want = masked_expectations(ex, 0xAA)
    assert np.array_equal(q[0], q_want) and np.array_equal(sf[0], sf_want)


def test_oracle_smooth_variant(oracle, ex):
    v = worked_variants(ex)
    q, sf = oracle.quantize_smooth(v["smooth_x"], v["pqs"], ex["gsf"], sf_fill=0xAA)
    assert np.array_equal(q, ex["q"]) and np.array_equal(sf, ex["sf"])


def test_oracle_lowrank_variant(oracle, ex):
    v = worked_variants(ex)
    rows, k = ex["rows"], ex["k"]
    q, sf = oracle.quantize(ex["x"], ex["gsf"])
    out = oracle.gemm_ref(q, q, sf, sf, 1.0, rows, rows, k, d=v["d"], l1=v["l1"], bias=v["bias"])
    assert np.array_equal(out, lowrank_expectation(ex))


def bf16_value(bits):
    return torch.from_numpy(np.array([bits], np.uint16).view(np.int16)).view(torch.bfloat16).item()


def _ones_operand(oracle, n, k):
    amax, gsf = oracle.global_scale(ones_rows(n, k))
    q, sf = oracle.quantize(ones_rows(n, k), gsf)
    return q, sf, float(amax)


def test_oracle_grouped_variant(oracle, ex):
    rows, k = ex["rows"], ex["k"]
    q, sf = oracle.quantize(ex["x"], ex["gsf"])
    qb, sfb, _ = _ones_operand(oracle, 8, k)
    alphas = np.float32([m / 2688.0 for m in ex["grouped_alpha_mult"]])
    out = oracle.grouped_gemm_ref(np.stack([q, q]), np.stack([qb, qb]), np.stack([sf, sf]), np.stack([sfb, sfb]),
                                  ex["grouped_mask"], alphas, 2, rows, 8, k)
    want = grouped_expectation(ex, np.nan)
    # the kernel writes bf16: round the fp64 reference once, as the oracle rounds it
    bf = np.vectorize(lambda v: v if np.isnan(v) else bf16_value(oracle.f64_to_bf16(v)))(out)
    assert np.array_equal(bf, want, equal_nan=True)


def _swiglu_operands(oracle, ex):
    q, sf = oracle.quantize(ex["x"], ex["gsf"])
    qb, sfb, amax_b = _ones_operand(oracle, ex["swiglu_n"], ex["k"])
    alpha_g = np.float32(oracle.alpha(ex["amax"], amax_b))
    alpha_u = np.float32(alpha_g / np.float32(ex["swiglu_up_div"]))
    gsf_h = np.float32(np.float32(2688.0) / np.float32(ex["swiglu_h"]))
    return q, sf, qb, sfb, alpha_g, alpha_u, gsf_h


def test_oracle_swiglu_variant(oracle, ex):
    rows, k, n, row = ex["rows"], ex["k"], ex["swiglu_n"], ex["row"]
    q, sf, qb, sfb, ag, au, gsf_h = _swiglu_operands(oracle, ex)
    gu = oracle.gemm_gate_up_bf16(q, qb, qb, sf, sfb, sfb, ag, au, n, k, [row, 0])
    vals = torch.from_numpy(gu.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.all(vals[0, :n] == ex["swiglu_g"]) and np.all(vals[0, n:] == ex["swiglu_u"])
    assert not np.any(vals[1])
    h = oracle.silu_mul(gu[:1])
    assert np.all(torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).double().numpy() == ex["swiglu_h"])
    q_want, sf_want = swiglu_expectation(ex)
    qh, sfh = oracle.gemm_silu_mul_quantize(q, qb, qb, sf, sfb, sfb, ag, au, gsf_h, rows, n, k, sf_fill=0xAA)
    assert np.array_equal(qh, q_want) and np.array_equal(sfh, sf_want)
    two = lambda t: np.stack([t, t])
    qg, sfg = oracle.grouped_gemm_silu_mul_quantize(two(q), two(qb), two(qb), two(sf), two(sfb), two(sfb),
                                                    ex["swiglu_grouped_mask"], [ag, ag], [au, au], [gsf_h, gsf_h],
                                                    2, rows, n, k, q_fill=0xAA, sf_fill=0xAA)
    q_want, sf_want = swiglu_grouped_expectation(ex, 0xAA)
    assert np.array_equal(qg, q_want) and np.array_equal(sfg, sf_want)


def test_oracle_lora_down_variant(oracle, ex):
    v = worked_variants(ex)
    d = oracle.lora_down(ex["x"], v["lora_w"])
    assert np.array_equal(d, lora_expectation(ex, ex["row_sum"]))
    assert bf16_value(oracle.f64_to_bf16(ex["row_sum"])) == ex["row_sum_bf16"]
    # the unsmoothed x/2 against the scaled weight: the same products
    assert np.array_equal(oracle.lora_down(v["smooth_x"], v["lora_w_scaled"]), d)


def test_oracle_silu_and_mul_variant(oracle, ex):
    v = worked_variants(ex)
    assert np.array_equal(oracle.silu_mul(v["silu_x"][0]), ex["x"])
