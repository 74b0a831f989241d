"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: the e2m1 grid the
pages give, the 448*6/amax and alpha formulas, the padded scale-buffer size, an
independent tensor-permutation construction of the 128x4 swizzle, PyTorch's fp8 e4m3
cast, exact dequantize-requantize round trips, closed-form constant tensors, error
bounds, and brute-force integer matmuls.  All run on the CPU.
"""
import math
import struct

import numpy as np
import pytest
import torch

import nvfp4_synth as S

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # e2m1 magnitudes (the method's value grid)


def f32(x):
    return struct.unpack("f", struct.pack("f", x))[0]


def torch_e4m3_value(code):
    return torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()


def py_e2m1_value(code):
    v = GRID[code & 7]
    return -v if code & 8 else v


def unpack_codes(q):
    q = np.asarray(q, np.uint8)
    lo = q & 15
    hi = q >> 4
    return np.stack([lo, hi], axis=-1).reshape(q.shape[:-1] + (q.shape[-1] * 2,))


E2M1_VALUES = np.array([py_e2m1_value(c) for c in range(16)])
E4M3_VALUES = np.array([torch_e4m3_value(c) for c in range(256)])


def py_sf_index_perm(rows, k):
    """Swizzled order of the padded logical scale matrix, built by a tensor permutation:
    [rp/128, 4, 32, cp/4, 4] -> [rp/128, cp/4, 32, 4, 4] (row = 128a + 32b + c, col = 4d + e)."""
    rp = -(-rows // 128) * 128
    cp = -(-(k // 16) // 4) * 4
    ids = np.arange(rp * cp).reshape(rp, cp)
    sw = ids.reshape(rp // 128, 4, 32, cp // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    off = np.empty(rp * cp, np.int64)
    off[sw] = np.arange(rp * cp)
    return off.reshape(rp, cp)      # off[r, c] = byte offset of logical (r, c)


def py_logical_scales(sf, rows, k):
    off = py_sf_index_perm(rows, k)
    return E4M3_VALUES[np.asarray(sf, np.uint8)[off[:rows, :k // 16]]]


def py_dequant_logical(q, sf, rows, k):
    codes = unpack_codes(np.asarray(q).reshape(rows, k // 2))
    s = np.repeat(py_logical_scales(sf, rows, k), 16, axis=1)
    return E2M1_VALUES[codes] * s


# --------------------------------------------------------------------------------------
# P1: scale-buffer size, closed form
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,k,expect", [
    (128, 256, 2048), (256, 256, 4096), (8192, 8192, 4194304), (8192, 5120, 2621440),
    (4096, 7168, 1835008), (16384, 5120, 5242880), (5120, 8192, 2621440),
    (1, 16, 512), (129, 16, 1024), (200, 80, 2048), (0, 64, 0), (130, 112, 2048),
])
def test_scale_bytes_closed_form(oracle, rows, k, expect):
    assert oracle.scale_bytes(rows, k) == expect
    assert expect == math.ceil(rows / 128) * 128 * math.ceil(k / 64) * 4


def test_scale_bytes_matches_unpadded_batched_shape(oracle):
    # The masked quantizer's [b, m*k/16] scale shape equals the padded per-item size
    # whenever m % 128 == 0 and k % 64 == 0.
    for m, k in [(4096, 7168), (128, 64), (256, 8192)]:
        assert oracle.scale_bytes(m, k) == m * k // 16


# --------------------------------------------------------------------------------------
# R6: swizzle offsets vs an independent permutation construction
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,k", [(128, 64), (256, 256), (130, 80), (300, 208), (1, 16)])
def test_sf_offset_matches_permutation(oracle, rows, k):
    off = py_sf_index_perm(rows, k)
    rp, cp = off.shape
    for r in range(rp):
        for c in range(cp):
            assert oracle.sf_offset(r, c, k) == off[r, c]


def test_sf_chunks_are_contiguous_512B(oracle):
    # one 128-row x 4-column tile occupies exactly one 512-byte chunk
    k = 512
    for rt in range(2):
        for cg in range(k // 64):
            offs = {oracle.sf_offset(128 * rt + r, 4 * cg + c, k) for r in range(128) for c in range(4)}
            base = min(offs)
            assert base % 512 == 0 and offs == set(range(base, base + 512))


# --------------------------------------------------------------------------------------
# P2: e2m1 codec (the grid) and e4m3 codec (PyTorch's float8_e4m3fn)
# --------------------------------------------------------------------------------------

def test_e2m1_decode_is_the_grid(oracle):
    for c in range(16):
        assert oracle.e2m1_value(c) == py_e2m1_value(c)


@pytest.mark.parametrize("v,code", [
    (0.0, 0), (0.5, 1), (1.0, 2), (1.5, 3), (2.0, 4), (3.0, 5), (4.0, 6), (6.0, 7),
    # ties go to the even code
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    # just off the ties
    (0.2500001, 1), (0.7499999, 1), (1.2500001, 3), (4.9999995, 6), (5.0000005, 7),
    # saturation
    (6.5, 7), (100.0, 7), (3.0e38, 7),
    # signs: a negative value that rounds to zero keeps its sign bit
    (-0.0, 8), (-0.1, 8), (-0.25, 8), (-0.3, 9), (-6.0, 15), (-1e9, 15), (-2.5, 12),
])
def test_e2m1_encode_table(oracle, v, code):
    assert oracle.e2m1_encode(f32(v)) == code


def test_e2m1_encode_is_nearest_on_random_values(oracle):
    g = np.random.default_rng(1234)
    vals = np.concatenate([g.uniform(-7, 7, 4000), g.normal(0, 2, 2000)]).astype(np.float32)
    grid = np.array(GRID)
    for v in vals:
        c = oracle.e2m1_encode(float(v))
        err = np.abs(abs(float(v)) - grid)
        best = np.flatnonzero(err == err.min())
        assert (c & 7) in best
        if len(best) == 2:
            assert (c & 7) % 2 == 0
        assert (c >> 3) == (1 if math.copysign(1.0, float(v)) < 0 else 0)


def test_e4m3_decode_matches_torch(oracle):
    for c in range(256):
        ref = torch_e4m3_value(c)
        got = oracle.e4m3_value(c)
        if math.isnan(ref):
            assert math.isnan(got)
        else:
            assert got == ref


def _e4m3_test_points():
    vals = sorted({torch_e4m3_value(c) for c in range(0x7F)})
    pts = set()
    for a, b in zip(vals, vals[1:]):
        mid = f32((a + b) / 2)
        pts.update([a, b, mid, np.nextafter(np.float32(mid), np.float32(0)).item(),
                    np.nextafter(np.float32(mid), np.float32(1e9)).item()])
    g = np.random.default_rng(7)
    pts.update(np.exp2(g.uniform(-12, 8.8, 20000)).astype(np.float32).tolist())
    return sorted(p for p in pts if p <= 448.0)


def test_ue4m3_encode_matches_torch_cast(oracle):
    pts = np.array(_e4m3_test_points(), np.float32)
    ref = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.ue4m3_encode(float(p)) for p in pts], np.uint8)
    bad = np.flatnonzero(ref != got)
    assert bad.size == 0, (pts[bad[:5]], ref[bad[:5]], got[bad[:5]])


@pytest.mark.parametrize("s,code", [
    (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (1e30, 0x7E),   # satfinite
    (2.0 ** -9, 0x01), (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (0.0, 0x00),
    (1.0, 0x38), (1.0625, 0x38), (1.1875, 0x3A),
])
def test_ue4m3_encode_special(oracle, s, code):
    assert oracle.ue4m3_encode(f32(s)) == code


# --------------------------------------------------------------------------------------
# global scale: 448*6/amax with nan_to_num and clamp(min=1e-12); alpha
# --------------------------------------------------------------------------------------

def bits(vals):
    return S.f32_to_bf16_bits(np.array(vals, np.float32))


def test_global_scale_closed_forms(oracle):
    amax, gsf = oracle.global_scale(bits([0.0, 3.0, -5.0, 1.0]))
    assert amax == 5.0 and gsf == np.float32(2688.0 / 5.0)
    amax, gsf = oracle.global_scale(bits([0.5, -0.25]))
    assert amax == 0.5 and gsf == np.float32(5376.0)
    # NaN counts as 0
    amax, gsf = oracle.global_scale(bits([np.nan, 2.0, -1.0]))
    assert amax == 2.0 and gsf == np.float32(1344.0)
    # +-Inf counts as FLT_MAX
    amax, gsf = oracle.global_scale(bits([-np.inf, 1.0]))
    assert amax == np.finfo(np.float32).max
    assert gsf == np.float32(2688.0) / np.finfo(np.float32).max
    # an all-zero tensor clamps to 1e-12
    amax, gsf = oracle.global_scale(bits([0.0, -0.0]))
    assert amax == np.float32(1e-12) and gsf == np.float32(2688.0) / np.float32(1e-12)
    amax, gsf = oracle.global_scale(np.zeros(0, np.uint16))
    assert amax == np.float32(1e-12)


def test_alpha_is_inverse_of_global_scales(oracle):
    g = np.random.default_rng(3)
    for _ in range(200):
        a, b = np.float32(g.uniform(0.01, 300)), np.float32(g.uniform(0.001, 5))
        al = oracle.alpha(float(a), float(b))
        assert al == np.float32(np.float32(a * b) / np.float32(2688.0 * 2688.0))
        ga, gb = 2688.0 / float(a), 2688.0 / float(b)
        assert abs(al * ga * gb - 1.0) < 4e-7


# --------------------------------------------------------------------------------------
# specified exp and SiLU (reading R8)
# --------------------------------------------------------------------------------------

def ulp32(x):
    x = abs(np.float32(x))
    return float(np.nextafter(x, np.float32(np.inf)) - x)


def test_exp_spec_within_2ulp(oracle):
    g = np.random.default_rng(11)
    xs = np.concatenate([np.linspace(-87, 88, 20001), g.uniform(-10, 10, 20000),
                         g.uniform(-1e-3, 1e-3, 2000)]).astype(np.float32)
    for x in xs:
        got = oracle.exp_spec(float(x))
        ref = math.exp(float(x))
        assert abs(got - ref) <= 2 * ulp32(ref), (x, got, ref)
    assert oracle.exp_spec(0.0) == 1.0
    assert oracle.exp_spec(100.0) == math.inf
    assert oracle.exp_spec(-200.0) == 0.0


def test_silu_mul_close_to_fp64(oracle):
    g = np.random.default_rng(5)
    gv = S.f32_to_bf16_bits(g.normal(0, 3, 3000).astype(np.float32))
    uv = S.f32_to_bf16_bits(g.normal(0, 1, 3000).astype(np.float32))
    for a, b in zip(gv, uv):
        h = oracle.silu_mul_bf16(int(a), int(b))
        ga = float(S.bf16_bits_to_f32(np.array([a]))[0])
        ub = float(S.bf16_bits_to_f32(np.array([b]))[0])
        ref = ga / (1 + math.exp(-ga)) * ub
        got = float(S.bf16_bits_to_f32(np.array([h], np.uint16))[0])
        # one bf16 rounding of a value carrying a few fp32 ulps of error
        assert abs(got - ref) <= 2 ** -7 * abs(ref) + 1e-30


def test_silu_special_cases(oracle):
    zero = int(bits([0.0])[0])
    for gval in [0.0, 1.0, -3.0, 10.0]:
        gb = int(bits([gval])[0])
        h = oracle.silu_mul_bf16(gb, zero)
        assert h in (0x0000, 0x8000)
    one = int(bits([1.0])[0])
    assert oracle.silu_mul_bf16(zero, one) == 0x0000


# --------------------------------------------------------------------------------------
# P3: constant tensors
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("c", [1.0, 0.3, -2.5, 1e-3, 300.0])
@pytest.mark.parametrize("m,k", [(4, 32), (130, 80)])
def test_constant_tensor(oracle, c, m, k):
    x = np.full((m, k), bits([c])[0], np.uint16)
    cb = float(S.bf16_bits_to_f32(bits([c]))[0])
    amax, gsf = oracle.global_scale(x)
    assert amax == np.float32(abs(cb)) and gsf == np.float32(2688.0) / np.float32(abs(cb))
    q, sf = oracle.quantize(x, gsf)
    logical = py_sf_index_perm(m, k)[:m, :k // 16]
    assert (sf[logical] == 0x7E).all()                       # every scale is 448
    expect = 0xFF if cb < 0 else 0x77                        # every code is +-6
    assert (q == expect).all()
    # padding entries are zero
    mask = np.ones(sf.size, bool)
    mask[logical.ravel()] = False
    assert (sf[mask] == 0).all()


# --------------------------------------------------------------------------------------
# P4: exact dequantize -> requantize round trip for values already on the grid
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("j", [0, 3, -2, 7])
@pytest.mark.parametrize("m,k", [(8, 64), (130, 96)])
def test_round_trip(oracle, j, m, k):
    g = np.random.default_rng(100 + j)
    nb = k // 16
    codes = g.integers(0, 16, size=(m, k)).astype(np.uint8)
    # every block holds a +-6
    pos = g.integers(0, 16, size=(m, nb))
    for r in range(m):
        for b in range(nb):
            codes[r, 16 * b + pos[r, b]] = 7 | (8 * int(g.integers(0, 2)))
    scales = g.integers(1, 0x7E, size=(m, nb)).astype(np.uint8)      # any finite non-zero scale
    scales[0, 0] = 0x7E                                              # one block reaches 448
    gsf = 2.0 ** j
    xs = E2M1_VALUES[codes] * np.repeat(E4M3_VALUES[scales], 16, axis=1) / gsf
    x = S.f32_to_bf16_bits(xs.astype(np.float32))
    assert (S.bf16_bits_to_f32(x).astype(np.float64) == xs).all()   # exact in bf16
    amax, gsf_o = oracle.global_scale(x)
    assert gsf_o == np.float32(gsf)
    q, sf = oracle.quantize(x, gsf_o)
    q_expect = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    assert (q == q_expect).all()
    off = py_sf_index_perm(m, k)[:m, :nb]
    assert (sf[off] == scales).all()


# --------------------------------------------------------------------------------------
# quantizer error bounds on random data (per element and per scale)
# --------------------------------------------------------------------------------------

def half_gap(mag):
    return np.where(mag < 2.0, 0.25, np.where(mag < 4.0, 0.5, 1.0))


def test_quantize_error_bounds(oracle):
    x = S.normal_with_outliers_bf16((256, 512), 0.01, 50.0, seed=3)
    amax, gsf = oracle.global_scale(x)
    q, sf = oracle.quantize(x, gsf)
    xf = S.bf16_bits_to_f32(x).astype(np.float64)
    scales = py_logical_scales(sf, 256, 512)
    blocks = np.abs(xf).reshape(256, 32, 16).max(-1)
    s_exact = blocks / 6.0 * float(gsf)
    # the scale is the e4m3 value nearest (vmax/6)*gsf: within half an e4m3 step (+ rounding)
    step = np.where(s_exact >= 2 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(s_exact, 1e-30))) - 3), 2.0 ** -9)
    assert (np.abs(scales - s_exact) <= step / 2 * (1 + 1e-6) + 1e-12).all()
    # each element lies within half a grid gap of its code (scaled), except saturation
    deq = py_dequant_logical(q, sf, 256, 512)
    v = xf * float(gsf) / np.repeat(scales, 16, axis=1)
    mag = np.abs(deq / np.repeat(scales, 16, axis=1))
    ok = (np.abs(v - deq / np.repeat(scales, 16, axis=1)) <= half_gap(mag) * (1 + 1e-5)) | (np.abs(v) > 6)
    assert ok.all()
    # and the largest element of every block maps to the top code
    codes = unpack_codes(q).reshape(256, 32, 16)
    top = np.take_along_axis(codes, np.abs(xf).reshape(256, 32, 16).argmax(-1)[..., None], -1)
    assert ((top & 7) == 7).all()


# --------------------------------------------------------------------------------------
# P9: masked batched quantize = dense quantize on each item's valid rows
# --------------------------------------------------------------------------------------

def test_masked_batched_equals_dense_slices(oracle):
    b, m, k = 4, 200, 96
    x = S.normal_bf16((b, m, k), 1.0, seed=9)
    mask = np.array([0, 200, 77, 129], np.int32)
    amax, gsf = oracle.global_scale_batched(x, mask)
    q, sf = oracle.quantize_masked_batched(x, gsf, mask, q_fill=0xA5, sf_fill=0x5A)
    sb = oracle.scale_bytes(m, k)
    assert sf.shape == (b, sb)
    for i in range(b):
        v = int(mask[i])
        if v:
            a_i, g_i = oracle.global_scale(x[i, :v])
            assert g_i == gsf[i] and a_i == amax[i]
            qd, sfd = oracle.quantize(x[i, :v], gsf[i])
            assert (q[i, :v] == qd).all()
            off = py_sf_index_perm(m, k)
            offd = py_sf_index_perm(v, k)
            assert (sf[i][off[:v, :k // 16]] == sfd[offd[:v, :k // 16]]).all()
        assert (q[i, v:] == 0xA5).all()                      # masked rows untouched
        off = py_sf_index_perm(m, k)
        assert (sf[i][off[v:, :]] == 0x5A).all()
    _, gsf_all = oracle.global_scale_batched(x, None)
    q2, sf2 = oracle.quantize_masked_batched(x, gsf_all, None)
    for i in range(b):
        qd, sfd = oracle.quantize(x[i], gsf_all[i])
        assert (q2[i] == qd).all() and (sf2[i] == sfd).all()


def test_silu_mul_quantize_equals_unfused(oracle):
    b, m, k = 3, 70, 64
    x = S.normal_bf16((b, m, 2 * k), 1.0, seed=4)
    mask = np.array([70, 0, 33], np.int32)
    _, gsf = oracle.global_scale_batched(x, mask, silu_mul=True)
    q, sf = oracle.silu_mul_quantize_batched(x, gsf, mask, q_fill=0x11, sf_fill=0x22)
    h = oracle.silu_mul(x)
    _, gsf_h = oracle.global_scale_batched(h, mask)
    assert (gsf_h == gsf).all()
    qh, sfh = oracle.quantize_masked_batched(h, gsf, mask, q_fill=0x11, sf_fill=0x22)
    assert (q == qh).all() and (sf == sfh).all()


def test_silu_mul_zero_up_gives_zero_codes(oracle):
    b, m, k = 1, 16, 32
    g = S.normal_bf16((b, m, k), 1.0, seed=2)
    x = np.concatenate([g, np.zeros((b, m, k), np.uint16)], axis=-1)
    q, sf = oracle.silu_mul_quantize_batched(x, np.array([100.0], np.float32))
    assert ((q & 0x77) == 0).all() and (sf == 0).all()


# --------------------------------------------------------------------------------------
# P5/P6: the GEMM reference against numpy matmuls of independently decoded operands
# --------------------------------------------------------------------------------------

def test_gemm_ref_matches_numpy_on_decoded(oracle):
    m, n, k, r = 40, 24, 128, 32
    xa = S.normal_bf16((m, k), 1.0, seed=1)
    xb = S.normal_bf16((n, k), 0.02, seed=2, tensor_id=2)
    amax_a, gsf_a = oracle.global_scale(xa)
    amax_b, gsf_b = oracle.global_scale(xb)
    qa, sfa = oracle.quantize(xa, gsf_a)
    qb, sfb = oracle.quantize(xb, gsf_b)
    al = oracle.alpha(float(amax_a), float(amax_b))
    d = S.normal_bf16((m, r), 1.0, seed=5, tensor_id=6)
    l1 = S.normal_bf16((n, r), 0.01, seed=5, tensor_id=7)
    bias = S.normal_bf16((n,), 0.1, seed=5, tensor_id=8)
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, al, m, n, k, d=d, l1=l1, bias=bias)
    A = py_dequant_logical(qa, sfa, m, k)
    B = py_dequant_logical(qb, sfb, n, k)
    D = S.bf16_bits_to_f32(d).astype(np.float64)
    L = S.bf16_bits_to_f32(l1).astype(np.float64)
    bb = S.bf16_bits_to_f32(bias).astype(np.float64)
    expect = float(al) * (A @ B.T + D @ L.T) + bb
    assert np.allclose(ref, expect, rtol=1e-12, atol=1e-12)
    # P5: alpha * sum(qa sfa)(qb sfb) equals the dot of the dequantized tensors x^ = E*S/gsf
    xa_hat, xb_hat = A / float(gsf_a), B / float(gsf_b)
    plain = oracle.gemm_ref(qa, qb, sfa, sfb, al, m, n, k)
    assert np.allclose(plain, xa_hat @ xb_hat.T, rtol=1e-6, atol=1e-9)
    # sampled positions agree with the full reference
    ii = np.array([0, 5, 39, 17]); jj = np.array([0, 23, 1, 12])
    smp = oracle.gemm_ref_sampled(qa, qb, sfa, sfb, al, k, ii, jj, d=d, l1=l1, bias=bias)
    assert (smp == ref[ii, jj]).all()


def test_gemm_ref_unit_scales_is_integer_matmul(oracle):
    m, n, k = 16, 8, 64
    g = np.random.default_rng(0)
    ca = g.integers(0, 16, size=(m, k)).astype(np.uint8)
    cb = g.integers(0, 16, size=(n, k)).astype(np.uint8)
    qa = (ca[:, 0::2] | (ca[:, 1::2] << 4)).astype(np.uint8)
    qb = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
    sfa = np.full(oracle.scale_bytes(m, k), 0x38, np.uint8)       # every scale 1.0
    sfb = np.full(oracle.scale_bytes(n, k), 0x38, np.uint8)
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, 1.0, m, n, k)
    ia = (2 * E2M1_VALUES[ca]).astype(np.int64)
    ib = (2 * E2M1_VALUES[cb]).astype(np.int64)
    assert (ref * 4 == ia @ ib.T).all()


def test_grouped_ref_equals_per_expert(oracle):
    E, mmax, n, k = 3, 140, 32, 64
    a = S.normal_bf16((E, mmax, k), 1.0, seed=8)
    w = S.normal_bf16((E, n, k), 0.02, seed=8, tensor_id=2)
    mask = np.array([0, 140, 61], np.int32)
    _, ga = oracle.global_scale_batched(a, mask)
    aw, gw = oracle.global_scale_batched(w, None)
    qa, sfa = oracle.quantize_masked_batched(a, ga, mask)
    qw, sfw = oracle.quantize_masked_batched(w, gw, None)
    alphas = np.array([1.5, 0.25, 2.0], np.float32)
    out = oracle.grouped_gemm_ref(qa, qw, sfa, sfw, mask, alphas, E, mmax, n, k)
    for e in range(E):
        v = int(mask[e])
        assert np.isnan(out[e, v:]).all()
        if v:
            ref = oracle.gemm_ref(qa[e], qw[e], sfa[e], sfw[e], alphas[e], mmax, n, k)[:v]
            assert (out[e, :v] == ref).all()


# --------------------------------------------------------------------------------------
# SwiGLU first half: gate/up projections, SiLU-and-mul quantization of h
# --------------------------------------------------------------------------------------

def _bf16_value(bits):
    """Exact value of one bf16 bit pattern (reinterpretation of the upper half of an fp32)."""
    w = np.array([int(bits) << 16], np.uint32)
    return float(w.view(np.float32)[0])


def test_f64_to_bf16_is_nearest_ties_even(oracle):
    # brute force on the definition: of the two bf16 neighbours (by bit pattern) of v, the
    # nearer one; on a tie the one with the even bit pattern
    g = np.random.default_rng(3)
    vals = list(g.standard_normal(3000) * 10.0 ** g.integers(-30, 30, 3000))
    # exact midpoints between neighbours, and points just beside them
    for bits in g.integers(0x0080, 0x7F00, 400):
        lo, hi = _bf16_value(bits), _bf16_value(bits + 1)
        mid = (lo + hi) / 2
        vals += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf), -mid]
    vals += [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 1e39,
             float.fromhex("0x1.FEp127"), float.fromhex("0x1.FFp127")]
    for v in vals:
        got = oracle.f64_to_bf16(v)
        a = abs(v)
        sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
        if a >= float.fromhex("0x1.FFp127"):     # at or past the overflow midpoint: infinity
            assert got == sign | 0x7F80, v
            continue
        t = int(np.array([a], np.float32).view(np.uint32)[0] >> 16)   # neighbour by truncation
        cands = [c for c in (t - 1, t, t + 1) if 0 <= c <= 0x7F7F]
        dist = [abs(_bf16_value(c) - a) for c in cands]
        best = min(dist)
        near = [c for c, d in zip(cands, dist) if d == best]
        want = near[0] if len(near) == 1 else [c for c in near if c % 2 == 0][0]
        assert got == sign | want, (v, hex(got), hex(sign | want))


def _pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def test_gemm_silu_mul_closed_form(oracle):
    # A = 1 everywhere, gate weight = 1, up weight = +-1 per output column (unit scales):
    # acc_g = k, acc_u = +-k.  With alpha_gate = 1, alpha_up = 1/64 and k = 128: g = 128
    # (silu(128) = 128 exactly in fp32), u = +-2, h = +-256, and gsf_h = 2688/256 makes
    # every block scale 448 (0x7E) and every code +-6 (0x7 / 0xF).  Swapping gate and up,
    # or their alphas, changes h.
    m, n, k = 130, 256, 128
    sign = np.random.default_rng(5).integers(0, 2, n).astype(np.uint8)   # 1: negative up row
    a = _pack(np.full((m, k), 0x2, np.uint8))
    bg = _pack(np.full((n, k), 0x2, np.uint8))
    bu = _pack(np.where(sign[:, None] == 1, 0xA, 0x2).astype(np.uint8) * np.ones((1, k), np.uint8))
    sa = np.full(oracle.scale_bytes(m, k), 0x38, np.uint8)
    sb = np.full(oracle.scale_bytes(n, k), 0x38, np.uint8)
    q, sf = oracle.gemm_silu_mul_quantize(a, bg, bu, sa, sb, sb, 1.0, 1.0 / 64, 2688.0 / 256, m, n, k)
    want_codes = np.where(sign == 1, 0xF, 0x7).astype(np.uint8)
    assert (unpack_codes(q) == want_codes[None, :]).all()
    for r in range(-(-m // 128) * 128):
        for c in range(n // 16):
            want = 0x7E if r < m else 0x00          # padding rows of the dense output are 0
            assert sf[oracle.sf_offset(r, c, n)] == want
    # swapped roles give something else
    q2, _ = oracle.gemm_silu_mul_quantize(a, bu, bg, sa, sb, sb, 1.0, 1.0 / 64, 2688.0 / 256, m, n, k)
    assert (q2 != q).any()
    _, sf3 = oracle.gemm_silu_mul_quantize(a, bg, bu, sa, sb, sb, 1.0 / 64, 1.0, 2688.0 / 256, m, n, k)
    assert (sf3 != sf).any()          # h = silu(2) * 128: the codes saturate alike, the scales differ


def test_gemm_silu_mul_zero_up_weight_gives_zero(oracle):
    m, n, k = 40, 128, 64
    xa = S.normal_bf16((m, k), 1.0, seed=11)
    xg = S.normal_bf16((n, k), 0.02, seed=11, tensor_id=2)
    _, ga = oracle.global_scale(xa)
    _, gg = oracle.global_scale(xg)
    qa, sa = oracle.quantize(xa, ga)
    qg, sg = oracle.quantize(xg, gg)
    qu = np.zeros_like(qg)
    su = np.zeros_like(sg)
    q, sf = oracle.gemm_silu_mul_quantize(qa, qg, qu, sa, sg, su, 0.5, 0.5, 100.0, m, n, k)
    assert ((q & 0x77) == 0).all() and (sf == 0).all()


def test_gemm_silu_mul_rows_and_grouped_agree_with_dense(oracle):
    # invariants: a row of the result depends only on that row of A; a masked expert equals
    # the dense result on its valid rows and leaves the other rows untouched
    E, mmax, n, k = 3, 150, 128, 128
    xa = S.normal_bf16((E, mmax, k), 1.0, seed=12)
    xg = S.normal_bf16((E, n, k), 0.02, seed=12, tensor_id=2)
    xu = S.normal_bf16((E, n, k), 0.02, seed=12, tensor_id=3)
    mask = np.array([150, 0, 77], np.int32)
    _, ga = oracle.global_scale_batched(xa, None)
    _, gg = oracle.global_scale_batched(xg, None)
    _, gu = oracle.global_scale_batched(xu, None)
    qa, sa = oracle.quantize_masked_batched(xa, ga)
    qg, sg = oracle.quantize_masked_batched(xg, gg)
    qu, su = oracle.quantize_masked_batched(xu, gu)
    al_g = np.array([0.7, 0.9, 1.1], np.float32)
    al_u = np.array([1.3, 0.6, 0.8], np.float32)
    gsf = np.array([40.0, 50.0, 60.0], np.float32)
    qG, sG = oracle.grouped_gemm_silu_mul_quantize(qa, qg, qu, sa, sg, su, mask, al_g, al_u, gsf, E, mmax, n, k,
                                                   q_fill=0xAB, sf_fill=0xCD)
    for e in range(E):
        v = int(mask[e])
        qd, sd = oracle.gemm_silu_mul_quantize(qa[e], qg[e], qu[e], sa[e], sg[e], su[e], al_g[e], al_u[e], gsf[e],
                                               mmax, n, k)
        assert (qG[e, :v] == qd[:v]).all() and (qG[e, v:] == 0xAB).all()
        for r in range(-(-mmax // 128) * 128):
            offs = [oracle.sf_offset(r, c, n) for c in range(n // 16)]
            if r < v:
                assert (sG[e, offs] == sd[offs]).all()
            else:
                assert (sG[e, offs] == 0xCD).all()
        rows = np.array([0, 3, mmax - 1])
        qr, sr = oracle.gemm_silu_mul_quantize_rows(qa[e], qg[e], qu[e], sa[e], sg[e], su[e], al_g[e], al_u[e],
                                                    gsf[e], n, k, rows)
        assert (qr == qd[rows]).all()
        for i, r in enumerate(rows):
            assert (sr[i] == sd[[oracle.sf_offset(r, c, n) for c in range(n // 16)]]).all()


# --------------------------------------------------------------------------------------
# SVDQuant input stage: smooth quantize and LoRA-down
# --------------------------------------------------------------------------------------

BF16_ONE = 0x3F80


def test_quantize_smooth_unit_scale_is_quantize(oracle):
    x = S.normal_bf16((70, 96), 1.0, seed=21)
    _, gsf = oracle.global_scale(x)
    q1, s1 = oracle.quantize_smooth(x, np.full(96, BF16_ONE, np.uint16), gsf)
    q2, s2 = oracle.quantize(x, gsf)
    assert (q1 == q2).all() and (s1 == s2).all()


def test_quantize_smooth_power_of_two_scales_are_exact(oracle):
    # pqs[c] = 2^e[c]: x * pqs is exact in bf16 (no overflow / underflow at these sizes), so
    # the smoothed tensor is x with e[c] added to every exponent of column c
    m, k = 40, 64
    x = S.normal_bf16((m, k), 1.0, seed=22)
    e = np.random.default_rng(3).integers(-3, 4, k)
    pqs = ((127 + e).astype(np.uint16) << 7).astype(np.uint16)             # bf16 2^e
    xs = x.astype(np.int32)
    expo = (xs >> 7) & 0xFF
    nz = expo != 0
    xs = np.where(nz, (xs & ~(0xFF << 7)) | ((expo + e[None, :]) << 7), xs).astype(np.uint16)
    _, gsf = oracle.global_scale(xs)
    q1, s1 = oracle.quantize_smooth(x, pqs, gsf)
    q2, s2 = oracle.quantize(xs, gsf)
    assert (q1 == q2).all() and (s1 == s2).all()


def test_quantize_smooth_matches_numpy_rounding(oracle):
    m, k = 33, 128
    x = S.normal_bf16((m, k), 1.0, seed=23)
    pqs = S.f32_to_bf16_bits(np.random.default_rng(4).uniform(0.25, 4.0, k).astype(np.float32))
    xh = S.f32_to_bf16_bits(S.bf16_bits_to_f32(x) * S.bf16_bits_to_f32(pqs)[None, :])
    _, gsf = oracle.global_scale(xh)
    q1, s1 = oracle.quantize_smooth(x, pqs, gsf)
    q2, s2 = oracle.quantize(xh, gsf)
    assert (q1 == q2).all() and (s1 == s2).all()


def test_lora_down_matches_numpy_and_identity(oracle):
    m, k, r = 50, 96, 32
    x = S.normal_bf16((m, k), 1.0, seed=24)
    w = S.normal_bf16((r, k), 0.05, seed=24, tensor_id=2)
    d = oracle.lora_down(x, w)
    ref = S.bf16_bits_to_f32(x).astype(np.float64) @ S.bf16_bits_to_f32(w).astype(np.float64).T
    assert np.allclose(d, ref, rtol=1e-12, atol=1e-12)
    eye = np.zeros((r, k), np.uint16)
    eye[np.arange(r), np.arange(r)] = BF16_ONE
    assert (oracle.lora_down(x, eye) == S.bf16_bits_to_f32(x[:, :r]).astype(np.float64)).all()


def test_gemm_gate_up_bf16_rows(oracle):
    # the [g | u] rows are the gate and up references rounded once to bf16; in the closed
    # form of test_gemm_silu_mul_closed_form they are exactly 128 and +-2
    m, n, k = 20, 64, 128
    xa = S.normal_bf16((m, k), 1.0, seed=25)
    xg = S.normal_bf16((n, k), 0.05, seed=25, tensor_id=2)
    xu = S.normal_bf16((n, k), 0.05, seed=25, tensor_id=3)
    ops = []
    for x in (xa, xg, xu):
        _, g = oracle.global_scale(x)
        ops.append(oracle.quantize(x, g))
    (qa, sa), (qg, sg), (qu, su) = ops
    rows = np.array([0, 7, 19])
    x = oracle.gemm_gate_up_bf16(qa, qg, qu, sa, sg, su, 0.75, 1.25, n, k, rows)
    rg = oracle.gemm_ref(qa, qg, sa, sg, 0.75, m, n, k)[rows]
    ru = oracle.gemm_ref(qa, qu, sa, su, 1.25, m, n, k)[rows]
    to_bf16 = np.vectorize(oracle.f64_to_bf16, otypes=[np.uint16])
    assert (x[:, :n] == to_bf16(rg)).all() and (x[:, n:] == to_bf16(ru)).all()
    a = _pack(np.full((4, k), 0x2, np.uint8))
    bg = _pack(np.full((n, k), 0x2, np.uint8))
    bu = _pack(np.full((n, k), 0xA, np.uint8))
    sa1 = np.full(oracle.scale_bytes(4, k), 0x38, np.uint8)
    sb1 = np.full(oracle.scale_bytes(n, k), 0x38, np.uint8)
    x = oracle.gemm_gate_up_bf16(a, bg, bu, sa1, sb1, sb1, 1.0, 1.0 / 64, n, k, np.arange(4))
    assert (x[:, :n] == 0x4300).all() and (x[:, n:] == 0xC000).all()      # bf16 128 and -2
