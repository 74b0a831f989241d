"""GPU parity of the tcgen05 block-scaled FP4 GEMMs against the oracle's fp64 reference
on the dequantized operands, within |out - ref| <= 1e-2*|ref| + 1e-3*max|ref|.

Operands are quantized by the oracle, so these tests pin the GEMM alone: the packing
(low nibble = lower K index), the 128x4 scale layout read straight into tensor memory,
the accumulator layout and the epilogue.  Sizes span several 128 x 256 tiles with ragged
M, N and K tails.  The full-size cases check the four corners and two interior points of
every 256 x 256 output tile (every expert tile of the grouped GEMM): within the tolerance,
and, more strictly, each bf16 output is a faithful rounding of the exact value (nearest, or
the other neighbour where the exact value lies within the fp32 accumulation bound of a
tie)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import (assert_gemm_close, bf16_to_f64, check_full_size, dev_bf16, dev_f32, dev_i32, dev_u8, host,
                           tile_positions)

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


def quantized(oracle, x):
    amax, gsf = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gsf)
    return q, sf, amax


def operands(oracle, m, n, k, seed=0, std_b=0.02):
    xa = S.normal_bf16((m, k), 1.0, seed, S.TID["x"])
    xb = S.normal_bf16((n, k), std_b, seed, S.TID["w"])
    qa, sfa, amax_a = quantized(oracle, xa)
    qb, sfb, amax_b = quantized(oracle, xb)
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    return qa, sfa, qb, sfb, alpha


def run_gemm(qa, sfa, qb, sfb, alpha, bias=None):
    return nv.nvfp4_gemm(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                         None if bias is None else dev_bf16(bias))


def test_unit_scales_integer_codes_bit_exact(oracle):
    # All scales 1.0 and alpha 1: every product is a multiple of 1/4 with |sum| small, so
    # the fp32 accumulation is exact and the bf16 output must equal the exact result
    # rounded once.
    for m, n, k in [(128, 256, 256), (128, 256, 64), (256, 512, 128)]:
        g = np.random.default_rng(m + n + k)
        ca = g.integers(0, 16, size=(m, k)).astype(np.uint8)
        cb = g.integers(0, 16, size=(n, k)).astype(np.uint8)
        qa = (ca[:, 0::2] | (ca[:, 1::2] << 4)).astype(np.uint8)
        qb = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
        sfa = np.full(nv.nvfp4_scale_bytes(m, k), 0x38, np.uint8)
        sfb = np.full(nv.nvfp4_scale_bytes(n, k), 0x38, np.uint8)
        ref = oracle.gemm_ref(qa, qb, sfa, sfb, 1.0, m, n, k)
        out = run_gemm(qa, sfa, qb, sfb, np.float32(1.0))
        expect = S.f32_to_bf16_bits(ref.astype(np.float32))
        assert (host(out) == expect).all(), np.argwhere(host(out) != expect)[:5]


@pytest.mark.parametrize("m,n,k", [(128, 576, 128), (300, 392, 256), (256, 968, 64), (130, 200, 192)])
def test_per_row_scales_bit_exact(oracle, m, n, k):
    # Power-of-two scales of A and B that change every 32 rows and every block: a scale read
    # from the wrong 32-row group, chunk or K step multiplies a row or column by another
    # scale.  Codes of at most 6 and scales of at most 2 keep every fp32 sum exact, so the
    # output equals the exact result rounded to bf16 once.
    g = np.random.default_rng(m * n + k)
    ca = g.integers(0, 16, size=(m, k)).astype(np.uint8)
    cb = g.integers(0, 16, size=(n, k)).astype(np.uint8)
    qa = (ca[:, 0::2] | (ca[:, 1::2] << 4)).astype(np.uint8)
    qb = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
    sfa = np.zeros(nv.nvfp4_scale_bytes(m, k), np.uint8)
    sfb = np.zeros(nv.nvfp4_scale_bytes(n, k), np.uint8)
    codes = (0x30, 0x38, 0x40)                                  # 0.5, 1, 2
    for r in range(m):
        for c in range(k // 16):
            sfa[oracle.sf_offset(r, c, k)] = codes[(r // 32 + 2 * c + 1) % 3]
    for r in range(n):
        for c in range(k // 16):
            sfb[oracle.sf_offset(r, c, k)] = codes[(r // 32 + c) % 3]
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, 1.0, m, n, k)
    out = host(run_gemm(qa, sfa, qb, sfb, np.float32(1.0)))
    expect = S.f32_to_bf16_bits(ref.astype(np.float32))
    assert (out == expect).all(), np.argwhere(out != expect)[:5]


def test_pr1_linear(oracle):
    d = S.pr1_linear()
    qa, sfa, amax_a = quantized(oracle, d["x"])
    qb, sfb, amax_b = quantized(oracle, d["w"])
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    out = run_gemm(qa, sfa, qb, sfb, alpha)
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, alpha, 128, 256, 256)
    assert_gemm_close(bf16_to_f64(out), ref, "pr1 linear 128x256x256")


@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (200, 264, 320), (300, 520, 1024), (1, 8, 64),
                                   (129, 256, 64), (384, 768, 576)])
def test_gemm_ragged(oracle, m, n, k):
    qa, sfa, qb, sfb, alpha = operands(oracle, m, n, k, seed=m + n + k)
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, alpha, m, n, k)
    out = run_gemm(qa, sfa, qb, sfb, alpha)
    assert_gemm_close(bf16_to_f64(out), ref, f"gemm {m}x{n}x{k}")


def test_gemm_bias_and_output_bounds(oracle):
    m, n, k = 200, 264, 320
    qa, sfa, qb, sfb, alpha = operands(oracle, m, n, k, seed=5)
    bias = S.normal_bf16((n,), 0.1, 5, S.TID["bias"])
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, alpha, m, n, k, bias=bias)
    # write into the middle of a larger sentinel buffer: nothing outside [m, n] may change
    big = torch.full((m * n + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[32:32 + m * n].view(m, n)
    nv.nvfp4_gemm(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha), dev_bf16(bias), out)
    assert_gemm_close(bf16_to_f64(out), ref, "gemm + bias")
    assert (big[:32] == 7.0).all() and (big[32 + m * n:] == 7.0).all()


@pytest.mark.parametrize("r", [32, 64, 96, 128])
def test_lowrank_bias(oracle, r):
    m, n, k = 200, 264, 320
    qa, sfa, qb, sfb, alpha = operands(oracle, m, n, k, seed=r)
    d = S.normal_bf16((m, r), 1.0, r, S.TID["d"])
    l1 = S.f32_to_bf16_bits(S.rng(r, S.TID["l1"]).standard_normal((n, r), dtype=np.float32)
                            * np.float32(0.01) / alpha)
    bias = S.normal_bf16((n,), 0.1, r, S.TID["bias"])
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, alpha, m, n, k, d=d, l1=l1, bias=bias)
    out = nv.nvfp4_gemm_lowrank_bias(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                                     dev_bf16(d), dev_bf16(l1), dev_bf16(bias))
    assert_gemm_close(bf16_to_f64(out), ref, f"lowrank r={r}")


def test_lowrank_special_cases(oracle):
    m, n, k, r = 128, 256, 256, 64
    qa, sfa, qb, sfb, alpha = operands(oracle, m, n, k, seed=9)
    d = S.normal_bf16((m, r), 1.0, 9, S.TID["d"])
    l1 = S.normal_bf16((n, r), 0.5, 9, S.TID["l1"])
    bias = S.normal_bf16((n,), 0.1, 9, S.TID["bias"])
    # a == 0: only the bf16 low-rank product and the bias remain
    qz = np.zeros_like(qa)
    ref = oracle.gemm_ref(qz, qb, sfa, sfb, alpha, m, n, k, d=d, l1=l1, bias=bias)
    out = nv.nvfp4_gemm_lowrank_bias(dev_u8(qz), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                                     dev_bf16(d), dev_bf16(l1), dev_bf16(bias))
    assert_gemm_close(bf16_to_f64(out), ref, "lowrank with a = 0")
    # d == 0: identical to the plain GEMM with bias
    dz = np.zeros_like(d)
    out_lr = nv.nvfp4_gemm_lowrank_bias(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                                        dev_bf16(dz), dev_bf16(l1), dev_bf16(bias))
    out_plain = run_gemm(qa, sfa, qb, sfb, alpha, bias)
    assert (host(out_lr) == host(out_plain)).all()


@pytest.mark.parametrize("E,mmax,n,k,mask", [
    (4, 300, 264, 320, [0, 300, 77, 129]),
    (3, 128, 256, 256, [128, 1, 0]),
    (2, 64, 512, 128, [64, 64]),
])
def test_grouped_masked(oracle, E, mmax, n, k, mask):
    mask = np.array(mask, np.int32)
    a = S.normal_bf16((E, mmax, k), 1.0, E, S.TID["x"])
    w = S.normal_bf16((E, n, k), 0.02, E, S.TID["w"])
    amax_a, ga = oracle.global_scale_batched(a, mask)
    amax_w, gw = oracle.global_scale_batched(w, None)
    qa, sfa = oracle.quantize_masked_batched(a, ga, mask)
    qw, sfw = oracle.quantize_masked_batched(w, gw, None)
    alphas = np.array([oracle.alpha(float(x), float(y)) for x, y in zip(amax_a, amax_w)], np.float32)
    ref = oracle.grouped_gemm_ref(qa, qw, sfa, sfw, mask, alphas, E, mmax, n, k)
    out = torch.full((E, mmax, n), -3.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(dev_u8(qa), dev_u8(qw), dev_u8(sfa), dev_u8(sfw), dev_i32(mask),
                                 dev_f32(alphas), out)
    o = bf16_to_f64(out)
    for e in range(E):
        v = int(mask[e])
        if v:
            assert_gemm_close(o[e, :v], ref[e, :v], f"expert {e}")
        assert (o[e, v:] == -3.0).all(), f"expert {e}: rows beyond the mask were written"


# ---- full sizes, every output tile ------------------------------------------------------------

def test_swiglu_gate_up_full_size_every_tile(oracle):
    # [8192 x 5120] @ [16384 x 5120]^T, the large dense GEMM of the SwiGLU block
    m, n, k = 8192, 16384, 5120
    qa, sfa, qb, sfb, alpha = operands(oracle, m, n, k, seed=0)
    out = host(run_gemm(qa, sfa, qb, sfb, alpha))
    ii, jj = tile_positions(m, n, 256, 256, seed=1)
    check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, "gate/up 8192x16384x5120 (every tile)")


def test_swiglu_down_full_size_every_tile(oracle):
    # the down projection at its configuration size: [8192 x 8192] @ [5120 x 8192]^T (K = 8192,
    # one epilogue warp per lane quarter with two staging tiles)
    m, n, k = 8192, 5120, 8192
    xa = S.normal_bf16((m, k), 1.0, 0, S.TID["x"])
    xb = S.swiglu_block()["w_down"]
    qa, sfa, amax_a = quantized(oracle, xa)
    qb, sfb, amax_b = quantized(oracle, xb)
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    out = host(run_gemm(qa, sfa, qb, sfb, alpha))
    ii, jj = tile_positions(m, n, 256, 256, seed=2)
    check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, "down 8192x5120x8192 (every tile)")


@pytest.mark.parametrize("r", [32, 64, 128])
def test_lowrank_full_size(oracle, r):
    d = S.lowrank(r=r)
    m, k, n = 4096, 3072, 3072
    qa, sfa, amax_a = quantized(oracle, d["x"])
    qb, sfb, amax_b = quantized(oracle, d["w"])
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    l1 = S.f32_to_bf16_bits(d["l1_f32"] / alpha)
    out = host(nv.nvfp4_gemm_lowrank_bias(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                                          dev_bf16(d["d"]), dev_bf16(l1), dev_bf16(d["bias"])))
    ii, jj = tile_positions(m, n, 256, 256, seed=r)
    check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, f"lowrank full r={r} (every tile)", d=d["d"],
                    l1=l1, bias=d["bias"])


@pytest.mark.parametrize("m,n,k,r", [(4096, 2560, 4096, 64), (2048, 4864, 6144, 0)])
def test_long_k_gemms_take_the_one_warp_epilogue(oracle, m, n, k, r):
    # K >= 4096 and at least one tile per SM: the launcher picks the kernel with one epilogue
    # warp per TMEM lane quarter and two staging tiles; low-rank (r > 0) and plain (r = 0)
    xa = S.normal_bf16((m, k), 1.0, 47 + r, S.TID["x"])
    xb = S.normal_bf16((n, k), 0.02, 47 + r, S.TID["w"])
    qa, sfa, amax_a = quantized(oracle, xa)
    qb, sfb, amax_b = quantized(oracle, xb)
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    ii, jj = tile_positions(m, n, 256, 256, seed=r + 1)
    if r:
        dd = S.normal_bf16((m, r), 1.0, 47, S.TID["d"])
        l1 = S.f32_to_bf16_bits(S.rng(47, S.TID["l1"]).standard_normal((n, r), dtype=np.float32) * np.float32(0.01)
                                / alpha)
        bias = S.normal_bf16((n,), 0.1, 47, S.TID["bias"])
        out = host(nv.nvfp4_gemm_lowrank_bias(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha),
                                              dev_bf16(dd), dev_bf16(l1), dev_bf16(bias)))
        check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, f"{m}x{n}x{k} r={r}", d=dd, l1=l1,
                        bias=bias)
    else:
        out = host(nv.nvfp4_gemm(dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha)))
        check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, f"{m}x{n}x{k}")


def test_grouped_full_size_every_expert_tile(oracle):
    d = S.grouped_moe()
    E, mmax, k, n = 16, 2048, 5120, 8192
    mask = d["mask"]
    amax_a, ga = oracle.global_scale_batched(d["a"], mask)
    amax_w, gw = oracle.global_scale_batched(d["w"], None)
    qa, sfa = oracle.quantize_masked_batched(d["a"], ga, mask)
    qw, sfw = oracle.quantize_masked_batched(d["w"], gw, None)
    alphas = np.array([oracle.alpha(float(x), float(y)) for x, y in zip(amax_a, amax_w)], np.float32)
    out = torch.full((E, mmax, n), -3.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(dev_u8(qa), dev_u8(qw), dev_u8(sfa), dev_u8(sfw), dev_i32(mask),
                                 dev_f32(alphas), out)
    o = host(out)
    for e in range(E):
        v = int(mask[e])
        if v:
            ii, jj = tile_positions(v, n, 256, 256, seed=e)
            check_full_size(oracle, o[e], qa[e], sfa[e], qw[e], sfw[e], alphas[e], k, ii, jj,
                            f"expert {e} ({v} rows, every tile)")
        if v < mmax:
            tail = o[e, v:]
            assert (tail == S.f32_to_bf16_bits(np.float32([-3.0]))[0]).all()
