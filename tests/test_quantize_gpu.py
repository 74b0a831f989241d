"""GPU parity of the global-scale reductions and the NVFP4 quantizers: bit-exact against
the CPU oracle on the same seeded inputs, from tiny ragged shapes up to the full
quantize-sweep sizes ([8192, 8192] with outliers, masked [8, 4096, 7168] and the
SiLU-and-mul variant on [8, 4096, 2*7168])."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import bf16_value, dev_bf16, dev_f32, dev_i32, dev_u8, first_diff, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    yield
    assert nv.nvfp4_device_status(clear=True) == 0


# ---- global scale ------------------------------------------------------------------------

@pytest.mark.parametrize("numel", [0, 1, 7, 8, 8003, 1 << 20])
def test_global_scale_matches_oracle(oracle, numel):
    x = S.normal_with_outliers_bf16((numel,), 0.01, 50.0, seed=numel)
    amax_o, gsf_o = oracle.global_scale(x)
    other = np.float32(3.25)
    amax, gsf, alpha = nv.nvfp4_global_scale(dev_bf16(x), other_amax=dev_f32(other))
    torch.cuda.synchronize()
    assert host(amax)[0] == amax_o and host(gsf)[0] == gsf_o
    assert host(alpha)[0] == np.float32(oracle.alpha(float(amax_o), float(other)))


def test_global_scale_special_values(oracle):
    vals = np.array([0.0, -3.0, np.nan, 2.0], np.float32)
    x = S.f32_to_bf16_bits(vals)
    amax, gsf, _ = nv.nvfp4_global_scale(dev_bf16(x))
    a_o, g_o = oracle.global_scale(x)
    assert host(amax)[0] == a_o == 3.0 and host(gsf)[0] == g_o
    x = S.f32_to_bf16_bits(np.array([1.0, -np.inf], np.float32))
    amax, gsf, _ = nv.nvfp4_global_scale(dev_bf16(x))
    a_o, g_o = oracle.global_scale(x)
    assert host(amax)[0] == a_o and host(gsf)[0] == g_o
    x = np.zeros(64, np.uint16)
    amax, gsf, _ = nv.nvfp4_global_scale(dev_bf16(x))
    a_o, g_o = oracle.global_scale(x)
    assert host(amax)[0] == a_o == np.float32(1e-12) and host(gsf)[0] == g_o


def test_global_scale_repeated_calls_reuse_workspace(oracle):
    for seed in range(3):
        x = S.normal_bf16((4099,), 1.0 + seed, seed=seed)
        _, g_o = oracle.global_scale(x)
        _, gsf, _ = nv.nvfp4_global_scale(dev_bf16(x))
        assert host(gsf)[0] == g_o


@pytest.mark.parametrize("silu", [False, True])
def test_global_scale_batched(oracle, silu):
    b, m, k = 5, 70, 48
    w = 2 * k if silu else k
    x = S.normal_bf16((b, m, w), 1.0, seed=21)
    mask = np.array([0, 70, 1, 33, 69], np.int32)
    a_o, g_o = oracle.global_scale_batched(x, mask, silu_mul=silu)
    amax, gsf = nv.nvfp4_global_scale_batched(dev_bf16(x), dev_i32(mask), silu_mul=silu)
    assert (host(amax) == a_o).all() and (host(gsf) == g_o).all()
    a_o, g_o = oracle.global_scale_batched(x, None, silu_mul=silu)
    amax, gsf = nv.nvfp4_global_scale_batched(dev_bf16(x), None, silu_mul=silu)
    assert (host(amax) == a_o).all() and (host(gsf) == g_o).all()


# ---- dense quantize ----------------------------------------------------------------------

def check_dense(oracle, x, gsf=None):
    if gsf is None:
        _, gsf = oracle.global_scale(x)
    q_o, sf_o = oracle.quantize(x, gsf)
    m, k = x.shape
    q = torch.full((m, k // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((nv.nvfp4_scale_bytes(m, k),), 0x5A, dtype=torch.uint8, device="cuda")
    nv.nvfp4_quantize(dev_bf16(x), dev_f32(gsf), q, sf)
    assert first_diff(host(q), q_o) is None, first_diff(host(q), q_o)
    assert first_diff(host(sf), sf_o) is None, first_diff(host(sf), sf_o)


@pytest.mark.parametrize("m,k", [(1, 16), (3, 48), (130, 80), (128, 256), (256, 256), (257, 512), (64, 4096)])
def test_quantize_matches_oracle(oracle, m, k):
    check_dense(oracle, S.normal_with_outliers_bf16((m, k), 0.01, 50.0, seed=m * 7 + k))


def test_quantize_signed_zeros_and_tiny_values(oracle):
    # Negative values that round to zero, exact zeros of both signs, subnormal scales.
    vals = np.array([1000.0, -0.0, 0.0, -1e-3, 1e-3, -0.01, 5e-3, -2.0] * 4, np.float32).reshape(2, 16)
    check_dense(oracle, S.f32_to_bf16_bits(vals))
    tiny = (np.arange(64, dtype=np.float32).reshape(4, 16) - 32) * np.float32(1e-6)
    tiny[0, 0] = 100.0
    check_dense(oracle, S.f32_to_bf16_bits(tiny))


def test_quantize_constant_and_zero_tensors(oracle):
    check_dense(oracle, np.full((128, 64), S.f32_to_bf16_bits(np.float32([-2.5]))[0], np.uint16))
    check_dense(oracle, np.zeros((5, 32), np.uint16), gsf=np.float32(2688.0 / 1e-12))


def every_bf16_block_maximum():
    """One 16-value block per non-negative finite bf16 value v (0x0000..0x7F7F): v at a seeded
    position, the other 15 values seeded fractions of +-v rounded to bf16 (never above v), so
    v is the block maximum; returns (blocks [n, 16] bf16 bits, v)."""
    v_bits = np.arange(0, 0x7F80, dtype=np.uint16)
    v = bf16_value(v_bits)
    g = np.random.default_rng([5, 16])
    frac = g.uniform(-1.0, 1.0, (v.size, 15))
    others = S.f32_to_bf16_bits((frac * v[:, None]).astype(np.float32))
    x = np.concatenate([v_bits[:, None], others], axis=1)
    perm = np.argsort(g.random((v.size, 16)), axis=1)
    return np.take_along_axis(x, perm, axis=1), v


def test_quantize_every_bf16_block_maximum(oracle):
    # The block scale is (vmax / 6) * gsf; the kernels form vmax / 6 as a product with fp32(1/6)
    # and one correction step, which must equal the IEEE quotient for every bf16 vmax.  Every
    # non-negative finite bf16 value is a block maximum here, each block with its own global
    # scale, a power of two that puts (vmax / 6) * gsf in the e4m3 range (so the product is
    # exact and the scale byte shows the quotient's rounding, ties included), and once more
    # with gsf = 1 through the dense quantizer.
    x, v = every_bf16_block_maximum()
    n = v.size
    j = np.where(v > 0, np.clip(np.round(np.log2(288.0 / np.maximum(v, 1e-300))), -126, 100), 0)
    gsf = (2.0 ** j).astype(np.float32)
    xb = np.ascontiguousarray(x.reshape(n, 1, 16))
    for mask in (None, np.ones(n, np.int32)):       # grid over items, and the persistent masked quantizer
        q = torch.full((n, 1, 8), 0xAB, dtype=torch.uint8, device="cuda")
        sf = torch.full((n, nv.nvfp4_scale_bytes(1, 16)), 0xCD, dtype=torch.uint8, device="cuda")
        nv.nvfp4_quantize_masked_batched(dev_bf16(xb), dev_f32(gsf), None if mask is None else dev_i32(mask), q, sf)
        q_ref, sf_ref = oracle.quantize_masked_batched(xb, gsf, mask, q_fill=0xAB, sf_fill=0xCD)
        assert first_diff(host(q), q_ref) is None, first_diff(host(q), q_ref)
        assert first_diff(host(sf), sf_ref) is None, first_diff(host(sf), sf_ref)
    one = np.float32([1.0])
    q, sf = nv.nvfp4_quantize(dev_bf16(x), dev_f32(one))
    q_ref, sf_ref = oracle.quantize(x, one[0])
    assert first_diff(host(q), q_ref) is None and first_diff(host(sf), sf_ref) is None


def test_quantize_full_size_with_outliers(oracle):
    x = S.quant_dense()["x"]                      # [8192, 8192], 0.1% outliers x50
    check_dense(oracle, x)


# ---- global scale and quantize in one launch ------------------------------------------------

def check_global_scale_quantize(oracle, x, other=np.float32(0.75)):
    """amax, gsf, alpha, codes and scales bit-exact against the oracle's global scale and
    quantizer (the fused launch must equal the two-call definition)."""
    m, k = x.shape
    amax_o, gsf_o = oracle.global_scale(x)
    q = torch.full((m, k // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((nv.nvfp4_scale_bytes(m, k),), 0x5A, dtype=torch.uint8, device="cuda")
    amax, gsf, alpha, _, _ = nv.nvfp4_global_scale_quantize(dev_bf16(x), other_amax=dev_f32(other), q_out=q,
                                                             sf_out=sf)
    torch.cuda.synchronize()
    assert host(amax)[0] == amax_o and host(gsf)[0] == gsf_o
    assert host(alpha)[0] == np.float32(oracle.alpha(float(amax_o), float(other)))
    if m:
        q_o, sf_o = oracle.quantize(x, gsf_o)
        assert first_diff(host(q), q_o) is None, first_diff(host(q), q_o)
        assert first_diff(host(sf), sf_o) is None, first_diff(host(sf), sf_o)


@pytest.mark.parametrize("m,k", [(1, 16), (3, 48), (130, 80), (300, 272), (257, 512), (64, 4096), (2048, 5120)])
def test_global_scale_quantize_matches_oracle(oracle, m, k):
    check_global_scale_quantize(oracle, S.normal_with_outliers_bf16((m, k), 0.01, 50.0, seed=m * 11 + k))


def test_global_scale_quantize_full_size(oracle):
    # the activation of the SwiGLU block: x [8192, 5120] ~ N(0, 1)
    check_global_scale_quantize(oracle, S.normal_bf16((8192, 5120), 1.0, 0, S.TID["x"]))


def test_global_scale_quantize_empty_rows_and_zeros(oracle):
    check_global_scale_quantize(oracle, np.zeros((0, 64), np.uint16))          # scalars only: amax = 1e-12
    check_global_scale_quantize(oracle, np.zeros((5, 32), np.uint16))


def test_global_scale_quantize_equals_two_calls_and_reuses_its_workspace():
    # repeated calls on one stream with different maxima (a workspace left set would leak
    # the previous maximum), NaN and inf included: the fused launch equals
    # nvfp4_global_scale followed by nvfp4_quantize
    for seed, scale in ((0, 8.0), (1, 0.5), (2, 3.0)):
        x = S.normal_bf16((700, 1024), scale, seed=seed)
        if seed == 2:
            x[3, 5] = 0x7FC0                      # NaN (counted as 0 by the amax)
            x[9, 100] = 0xFF80                    # -inf
        xd = dev_bf16(x)
        a1, g1, _ = nv.nvfp4_global_scale(xd)
        q1, s1 = nv.nvfp4_quantize(xd, g1)
        a2, g2, _, q2, s2 = nv.nvfp4_global_scale_quantize(xd)
        torch.cuda.synchronize()
        assert torch.equal(a1, a2) and torch.equal(g1, g2)
        assert torch.equal(q1, q2) and torch.equal(s1, s2)


def test_quantize_empty_and_invalid():
    x = torch.zeros((0, 32), dtype=torch.bfloat16, device="cuda")
    q, sf = nv.nvfp4_quantize(x, torch.ones(1, device="cuda"))
    assert q.numel() == 0 and sf.numel() == 0
    # an invalid call writes nothing
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    q = torch.full((4, 12), 7, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_quantize(x, torch.ones(1, device="cuda"), q, torch.zeros(512, dtype=torch.uint8, device="cuda"))
    assert (q == 7).all()


# ---- masked batched ------------------------------------------------------------------------

def check_masked(oracle, x, mask, silu):
    b, m, w = x.shape
    k = w // 2 if silu else w
    _, gsf = oracle.global_scale_batched(x, mask, silu_mul=silu)
    fn_o = oracle.silu_mul_quantize_batched if silu else oracle.quantize_masked_batched
    q_o, sf_o = fn_o(x, gsf, mask, q_fill=0xA5, sf_fill=0x5A)
    q = torch.full((b, m, k // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((b, nv.nvfp4_scale_bytes(m, k)), 0x5A, dtype=torch.uint8, device="cuda")
    fn = nv.nvfp4_silu_mul_quantize_batched if silu else nv.nvfp4_quantize_masked_batched
    fn(dev_bf16(x), dev_f32(gsf), None if mask is None else dev_i32(mask), q, sf)
    # the oracle leaves the same sentinels in rows >= mask, so whole buffers must agree
    assert first_diff(host(q), q_o) is None, first_diff(host(q), q_o)
    assert first_diff(host(sf), sf_o) is None, first_diff(host(sf), sf_o)


@pytest.mark.parametrize("silu", [False, True])
@pytest.mark.parametrize("b,m,k,mask", [
    (4, 200, 96, [0, 200, 77, 129]),
    (3, 128, 64, [128, 1, 0]),
    (2, 300, 512, None),
    (1, 5, 16, [3]),
])
def test_masked_batched_matches_oracle(oracle, silu, b, m, k, mask):
    w = 2 * k if silu else k
    x = S.normal_bf16((b, m, w), 1.0, seed=b * 100 + m)
    check_masked(oracle, x, None if mask is None else np.array(mask, np.int32), silu)


def test_masked_batched_equals_dense_per_item(oracle):
    b, m, k = 3, 160, 128
    x = S.normal_bf16((b, m, k), 1.0, seed=77)
    mask = np.array([160, 5, 131], np.int32)
    _, gsf = oracle.global_scale_batched(x, mask)
    qb, sfb = nv.nvfp4_quantize_masked_batched(dev_bf16(x), dev_f32(gsf), dev_i32(mask))
    for i in range(b):
        v = int(mask[i])
        q, sf = nv.nvfp4_quantize(dev_bf16(x[i, :v]), dev_f32(gsf[i]))
        assert (host(qb[i, :v]) == host(q)).all()
        sb = nv.nvfp4_scale_bytes(v, k)
        # the valid rows' chunks coincide (row tiles of 128 rows, same k)
        full_tiles = v // 128
        n = full_tiles * 128 * (k // 16)
        assert (host(sfb[i, :n]) == host(sf[:n])).all() and sb >= n


@pytest.mark.parametrize("silu", [False, True])
def test_masked_full_size(oracle, silu):
    d = S.quant_silu() if silu else S.quant_masked()    # [8, 4096, 7168] (x2 for SiLU), masks U[0, 4096]
    check_masked(oracle, d["x"], d["mask"], silu)


def test_silu_zero_up_and_zero_gate(oracle):
    b, m, k = 1, 8, 32
    g = S.normal_bf16((b, m, k), 1.0, seed=4)
    x = np.concatenate([g, np.zeros_like(g)], axis=-1)
    check_masked(oracle, x, None, True)
    x = np.concatenate([np.zeros_like(g), g], axis=-1)      # silu(0) = 0
    check_masked(oracle, x, None, True)


@pytest.mark.parametrize("u_kind", ["one", "negative", "random"])
def test_silu_and_mul_every_bf16_gate_bit_exact(oracle, u_kind):
    # every finite bf16 value as the gate (both signs, subnormals, |g| up to 3.4e38: the
    # exponential's clamps at -104 / 89 and its 2^n scaling outside [-125, 127] are reached)
    pats = np.arange(65536, dtype=np.uint32)
    finite = ((pats >> 7) & 0xFF) != 0xFF
    g = pats[finite].astype(np.uint16)
    k = 256
    g = np.concatenate([g, np.zeros((-len(g)) % k, np.uint16)]).reshape(-1, k)
    if u_kind == "one":
        u = np.full_like(g, 0x3F80)
    elif u_kind == "negative":
        u = np.full_like(g, S.f32_to_bf16_bits(np.float32([-3.5]))[0])
    else:
        u = S.normal_bf16(g.shape, 1.0, 5, S.TID["x"])
    x = np.concatenate([g, u], axis=1)
    h = nv.nvfp4_silu_and_mul(dev_bf16(x))
    want = oracle.silu_mul(x)
    got = host(h)
    assert (got == want).all(), np.argwhere(got != want)[:5]
