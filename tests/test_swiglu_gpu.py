"""GPU parity of the gate/up GEMM whose epilogue emits SiLU(g) * u as NVFP4
(nvfp4_gemm_silu_mul_quantize and its masked grouped form).

Comparisons:
  * unit scales and integer-friendly codes with power-of-two alphas, where the fp32
    accumulation is exact, so g, u, h and the quantized output must equal the oracle's
    composition bit for bit (codes of valid rows and the whole scale buffer);
  * random operands, complete and bit-exact: the library's own bf16 projections g and u
    (nvfp4_gemm) are fed to the oracle's SiLU-and-mul quantizer with the same gsf_h, and
    the fused kernel's codes and scales must equal the oracle's bit for bit (every row,
    the padding rows' zero scales included); the fused kernel also equals the unfused GPU
    sequence bit for bit;
  * the library's g and u against the exact fp64 projections: each is the exact value
    rounded to nearest, or, where the exact value lies within the fp32 accumulation bound
    of a bf16 tie, the neighbour on the other side (a faithful rounding);
  * against the oracle's fp64 composition (projections rounded once): a 16-value block of
    the output may differ only where one of its g or u values is such a near-tie rounding;
  * masked grouped: rows at or beyond mask[e] (codes and scale entries) stay untouched.
Sizes span several 256 x 128 output tiles with ragged M; the full-size case checks every
row of the 8192 x 8192 (hidden 5120) SwiGLU block bit for bit, the projections at points
of every output tile, and eight whole rows against the fp64 composition."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import (check_explained_vs_composition, check_projections_faithful, dev_f32, dev_i32, dev_u8, host,
                           sf_logical, tile_positions)

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


def _pack(codes):
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def integer_operands(shape_a, shape_w, seed):
    """Random e2m1 codes with every block scale 1.0 (0x38)."""
    g = np.random.default_rng(seed)
    ops = []
    for shape in (shape_a, shape_w, shape_w):
        codes = g.integers(0, 16, size=shape).astype(np.uint8)
        rows, k = shape[-2], shape[-1]
        lead = shape[:-2]
        sf = np.full(lead + (nv.nvfp4_scale_bytes(rows, k),), 0x38, np.uint8)
        ops.append((_pack(codes), sf))
    return ops


# Operand tuples follow the oracle's argument order:
#   (a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up[, gsf_h])

def real_operands(oracle, m, n, k, seed, std=0.05):
    """Quantized normal activations and gate/up weights with their alphas, plus gsf_h
    calibrated on the oracle's h (448*6 / amax(h))."""
    xs = [S.normal_bf16((m, k), 1.0, seed, S.TID["x"]),
          S.normal_bf16((n, k), std, seed, S.TID["w_gate_up"]),
          S.normal_bf16((n, k), std, seed, S.TID["w_down"])]
    ops, amax = [], []
    for x in xs:
        am, g = oracle.global_scale(x)
        ops.append(oracle.quantize(x, g))
        amax.append(float(am))
    al_g = np.float32(oracle.alpha(amax[0], amax[1]))
    al_u = np.float32(oracle.alpha(amax[0], amax[2]))
    (qa, sa), (qg, sg), (qu, su) = ops
    x = oracle.gemm_gate_up_bf16(qa, qg, qu, sa, sg, su, al_g, al_u, n, k, np.arange(m))
    _, gsf = oracle.global_scale_batched(x[None], None, silu_mul=True)
    return qa, qg, qu, sa, sg, su, al_g, al_u, np.float32(gsf[0])


def run_fused(qa, qg, qu, sa, sg, su, al_g, al_u, gsf):
    q, sf = nv.nvfp4_gemm_silu_mul_quantize(dev_u8(qa), dev_u8(qg), dev_u8(qu), dev_u8(sa), dev_u8(sg),
                                            dev_u8(su), dev_f32(al_g), dev_f32(al_u), dev_f32(gsf))
    return host(q), host(sf)


def run_unfused(qa, qg, qu, sa, sg, su, al_g, al_u, gsf):
    g = nv.nvfp4_gemm(dev_u8(qa), dev_u8(qg), dev_u8(sa), dev_u8(sg), dev_f32(al_g))
    u = nv.nvfp4_gemm(dev_u8(qa), dev_u8(qu), dev_u8(sa), dev_u8(su), dev_f32(al_u))
    x = torch.cat([g, u], dim=-1).unsqueeze(0).contiguous()
    q, sf = nv.nvfp4_silu_mul_quantize_batched(x, dev_f32(gsf))
    return host(q)[0], host(sf).reshape(-1)


@pytest.mark.parametrize("m,n,k", [(300, 384, 256), (128, 128, 64), (1, 128, 128), (513, 256, 512)])
def test_unit_scales_bit_exact_vs_oracle(oracle, m, n, k):
    (qa, sa), (qg, sg), (qu, su) = integer_operands((m, k), (n, k), seed=m + n + k)
    al_g, al_u = np.float32(2.0 ** -5), np.float32(2.0 ** -4)
    x = oracle.gemm_gate_up_bf16(qa, qg, qu, sa, sg, su, al_g, al_u, n, k, np.arange(m))
    _, gsf = oracle.global_scale_batched(x[None], None, silu_mul=True)
    q_ref, sf_ref = oracle.gemm_silu_mul_quantize(qa, qg, qu, sa, sg, su, al_g, al_u, gsf[0], m, n, k)
    q, sf = run_fused(qa, qg, qu, sa, sg, su, al_g, al_u, gsf[0])
    assert (q == q_ref).all(), np.argwhere(q != q_ref)[:5]
    assert (sf == sf_ref).all(), np.argwhere(sf != sf_ref)[:5]     # including zeroed padding rows


def library_gate_up(ops):
    """[g | u] bf16 [m, 2n] from the library's plain GEMM (bf16(alpha * acc), the rounding the
    fused epilogue applies before SiLU), on the device."""
    qa, qg, qu, sa, sg, su, al_g, al_u = ops[:8]
    g = nv.nvfp4_gemm(dev_u8(qa), dev_u8(qg), dev_u8(sa), dev_u8(sg), dev_f32(al_g))
    u = nv.nvfp4_gemm(dev_u8(qa), dev_u8(qu), dev_u8(sa), dev_u8(su), dev_f32(al_u))
    return torch.cat([g, u], dim=-1).contiguous()


@pytest.mark.parametrize("m,n,k", [(300, 384, 320), (256, 256, 5120), (129, 640, 1024)])
def test_random_bit_exact_vs_oracle_quantizer_on_library_projections(oracle, m, n, k):
    ops = real_operands(oracle, m, n, k, seed=m + k)
    gsf = ops[-1]
    q, sf = run_fused(*ops)
    gu = library_gate_up(ops)
    q_u, sf_u = run_unfused(*ops)
    assert (q == q_u).all(), np.argwhere(q != q_u)[:5]
    assert (sf == sf_u).all(), np.argwhere(sf != sf_u)[:5]
    gu_h = host(gu)
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h[None], np.float32([gsf]))
    assert (q == q_ref[0]).all(), np.argwhere(q != q_ref[0])[:5]
    assert (sf == sf_ref[0]).all(), np.argwhere(sf != sf_ref[0])[:5]     # padding rows' zero scales included
    rows = np.arange(m)
    ii, jj = np.repeat(rows, n), np.tile(np.arange(n), m)
    check_projections_faithful(oracle, ops, gu_h, ii, jj, n, k, f"swiglu {m}x{n}x{k}")
    check_explained_vs_composition(oracle, ops, gsf, q, sf_logical(sf, m, n), gu_h, rows, n, k,
                                   f"swiglu {m}x{n}x{k}")


def test_concatenated_gate_up_weight(oracle):
    # one [2n, k] weight quantized as one tensor: b_up and its scales are views into it
    m, n, k = 200, 256, 256
    xa = S.normal_bf16((m, k), 1.0, 3, S.TID["x"])
    xw = S.normal_bf16((2 * n, k), 0.05, 3, S.TID["w_gate_up"])
    am_a, ga = oracle.global_scale(xa)
    am_w, gw = oracle.global_scale(xw)
    qa, sa = oracle.quantize(xa, ga)
    qw, sw = oracle.quantize(xw, gw)
    al = np.float32(oracle.alpha(float(am_a), float(am_w)))
    half = nv.nvfp4_scale_bytes(n, k)
    ops = (qa, qw[:n], qw[n:], sa, sw[:half], sw[half:], al, al)
    x = oracle.gemm_gate_up_bf16(*ops, n, k, np.arange(m))
    _, gsf = oracle.global_scale_batched(x[None], None, silu_mul=True)
    wq, wsf = dev_u8(qw), dev_u8(sw)
    q, sf = nv.nvfp4_gemm_silu_mul_quantize(dev_u8(qa), wq[:n], wq[n:], dev_u8(sa), wsf[:half], wsf[half:],
                                            dev_f32(al), dev_f32(al), dev_f32(gsf[0]))
    gu_h = host(library_gate_up(ops))
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h[None], gsf)
    assert (host(q) == q_ref[0]).all() and (host(sf) == sf_ref[0]).all()
    check_explained_vs_composition(oracle, ops, gsf[0], host(q), sf_logical(host(sf), m, n), gu_h, np.arange(m), n,
                                   k, "concat")


def test_output_bounds(oracle):
    # codes and scales land inside [m, n/2] and the scale buffer; nothing around them changes
    m, n, k = 130, 256, 128
    ops = real_operands(oracle, m, n, k, seed=7)
    qn, sn = m * n // 2, nv.nvfp4_scale_bytes(m, n)
    qbig = torch.full((qn + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    sbig = torch.full((sn + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    qa, qg, qu, sa, sg, su, al_g, al_u, gsf = ops
    nv.nvfp4_gemm_silu_mul_quantize(dev_u8(qa), dev_u8(qg), dev_u8(qu), dev_u8(sa), dev_u8(sg), dev_u8(su),
                                    dev_f32(al_g), dev_f32(al_u), dev_f32(gsf), qbig[32:32 + qn].view(m, n // 2),
                                    sbig[32:32 + sn])
    qh, sh = host(qbig), host(sbig)
    assert (qh[:32] == 0x5A).all() and (qh[32 + qn:] == 0x5A).all()
    assert (sh[:32] == 0xA5).all() and (sh[32 + sn:] == 0xA5).all()
    q_u, sf_u = run_unfused(*ops)
    assert (qh[32:32 + qn].reshape(m, n // 2) == q_u).all() and (sh[32:32 + sn] == sf_u).all()


# ---- masked grouped --------------------------------------------------------------------------

def grouped_real(oracle, E, mmax, n, k, mask, seed):
    xa = S.normal_bf16((E, mmax, k), 1.0, seed, S.TID["x"])
    xg = S.normal_bf16((E, n, k), 0.05, seed, S.TID["w_gate_up"])
    xu = S.normal_bf16((E, n, k), 0.05, seed, S.TID["w_down"])
    am_a, ga = oracle.global_scale_batched(xa, mask)
    am_g, gg = oracle.global_scale_batched(xg, None)
    am_u, gu = oracle.global_scale_batched(xu, None)
    qa, sa = oracle.quantize_masked_batched(xa, ga, mask)
    qg, sg = oracle.quantize_masked_batched(xg, gg, None)
    qu, su = oracle.quantize_masked_batched(xu, gu, None)
    al_g = np.array([oracle.alpha(float(a), float(b)) for a, b in zip(am_a, am_g)], np.float32)
    al_u = np.array([oracle.alpha(float(a), float(b)) for a, b in zip(am_a, am_u)], np.float32)
    gsf = np.zeros(E, np.float32)
    for e in range(E):
        v = int(mask[e])
        if v:
            x = oracle.gemm_gate_up_bf16(qa[e], qg[e], qu[e], sa[e], sg[e], su[e], al_g[e], al_u[e], n, k,
                                         np.arange(v))
            gsf[e] = oracle.global_scale_batched(x[None], None, silu_mul=True)[1][0]
        else:
            gsf[e] = 1.0
    return qa, qg, qu, sa, sg, su, al_g, al_u, gsf


def run_grouped_fused(ops, mask, E, mmax, n, qfill=0xAB, sffill=0xCD):
    qa, qg, qu, sa, sg, su, al_g, al_u, gsf = ops
    q = torch.full((E, mmax, n // 2), qfill, dtype=torch.uint8, device="cuda")
    sf = torch.full((E, nv.nvfp4_scale_bytes(mmax, n)), sffill, dtype=torch.uint8, device="cuda")
    nv.nvfp4_grouped_gemm_silu_mul_quantize_masked(dev_u8(qa), dev_u8(qg), dev_u8(qu), dev_u8(sa), dev_u8(sg),
                                                   dev_u8(su), dev_i32(mask), dev_f32(al_g), dev_f32(al_u),
                                                   dev_f32(gsf), q, sf)
    return host(q), host(sf)


def test_grouped_unit_scales_bit_exact_vs_oracle(oracle):
    E, mmax, n, k = 4, 300, 256, 256
    mask = np.array([300, 0, 1, 129], np.int32)
    (qa, sa), (qg, sg), (qu, su) = integer_operands((E, mmax, k), (E, n, k), seed=11)
    al_g = np.float32([2.0 ** -5, 2.0 ** -6, 2.0 ** -4, 2.0 ** -5])
    al_u = np.float32([2.0 ** -4, 2.0 ** -5, 2.0 ** -5, 2.0 ** -6])
    gsf = np.float32([30.0, 1.0, 40.0, 50.0])
    ops = (qa, qg, qu, sa, sg, su, al_g, al_u, gsf)
    q, sf = run_grouped_fused(ops, mask, E, mmax, n)
    q_ref, sf_ref = oracle.grouped_gemm_silu_mul_quantize(qa, qg, qu, sa, sg, su, mask, al_g, al_u, gsf, E, mmax,
                                                          n, k, q_fill=0xAB, sf_fill=0xCD)
    assert (q == q_ref).all(), np.argwhere(q != q_ref)[:5]
    assert (sf == sf_ref).all(), np.argwhere(sf != sf_ref)[:5]      # rows >= mask keep 0xCD


def test_grouped_random_bit_exact_vs_oracle_quantizer_on_library_projections(oracle):
    E, mmax, n, k = 5, 384, 256, 512
    mask = np.array([384, 0, 257, 1, 128], np.int32)
    ops = grouped_real(oracle, E, mmax, n, k, mask, seed=13)
    q, sf = run_grouped_fused(ops, mask, E, mmax, n)
    qa, qg, qu, sa, sg, su, al_g, al_u, gsf = ops
    # unfused GPU sequence: two grouped GEMMs, then the masked SiLU-and-mul quantizer
    g = nv.nvfp4_grouped_gemm_masked(dev_u8(qa), dev_u8(qg), dev_u8(sa), dev_u8(sg), dev_i32(mask), dev_f32(al_g))
    u = nv.nvfp4_grouped_gemm_masked(dev_u8(qa), dev_u8(qu), dev_u8(sa), dev_u8(su), dev_i32(mask), dev_f32(al_u))
    x = torch.cat([g, u], dim=-1).contiguous()
    qx = torch.full((E, mmax, n // 2), 0xAB, dtype=torch.uint8, device="cuda")
    sx = torch.full((E, nv.nvfp4_scale_bytes(mmax, n)), 0xCD, dtype=torch.uint8, device="cuda")
    nv.nvfp4_silu_mul_quantize_batched(x, dev_f32(gsf), mask=dev_i32(mask), q_out=qx, sf_out=sx)
    assert (q == host(qx)).all() and (sf == host(sx)).all()
    # the oracle's quantizer on the library's projections, every valid row, bit for bit
    gu_h = host(x)
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h, gsf, mask, q_fill=0xAB, sf_fill=0xCD)
    assert (q == q_ref).all(), np.argwhere(q != q_ref)[:5]
    assert (sf == sf_ref).all(), np.argwhere(sf != sf_ref)[:5]
    for e in range(E):
        v = int(mask[e])
        assert (q[e, v:] == 0xAB).all(), f"expert {e}: rows beyond the mask were written"
        rows_pad = -(-mmax // 128) * 128
        assert (sf_logical(sf[e], rows_pad, n)[v:] == 0xCD).all(), f"expert {e}: scales beyond the mask written"
        if v:
            ops_e = (qa[e], qg[e], qu[e], sa[e], sg[e], su[e], al_g[e], al_u[e])
            rows = np.arange(v)
            check_explained_vs_composition(oracle, ops_e, gsf[e], q[e, :v], sf_logical(sf[e], v, n), gu_h[e, :v],
                                           rows, n, k, f"expert {e}")


# ---- full size, sampled rows ---------------------------------------------------------------------

def test_swiglu_block_full_size_every_row(oracle):
    # x [8192, 5120]; W_gate_up [16384, 5120] as one tensor: gate = rows [0, 8192), up = the rest
    m, k, n = 8192, 5120, 8192
    d = S.swiglu_block()
    am_a, ga = oracle.global_scale(d["x"])
    am_w, gw = oracle.global_scale(d["w_gate_up"])
    qa, sa = oracle.quantize(d["x"], ga)
    qw, sw = oracle.quantize(d["w_gate_up"], gw)
    al = np.float32(oracle.alpha(float(am_a), float(am_w)))
    half = nv.nvfp4_scale_bytes(n, k)
    ops = (qa, qw[:n], qw[n:], sa, sw[:half], sw[half:], al, al)
    gu = library_gate_up(ops)
    gu_h = host(gu)
    del gu
    # the static scale of h, calibrated on the whole h of the library's projections
    gsf = np.float32(oracle.global_scale_batched(gu_h[None], None, silu_mul=True)[1][0])
    q, sf = run_fused(*ops, gsf)
    # every row of the output, bit for bit, against the oracle's quantizer on the same projections
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h[None], np.float32([gsf]))
    assert (q == q_ref[0]).all(), np.argwhere(q != q_ref[0])[:5]
    assert (sf == sf_ref[0]).all(), np.argwhere(sf != sf_ref[0])[:5]
    # the projections at the corners and two interior points of every 256 x 128 output tile
    ii, jj = tile_positions(m, n, 256, 128, seed=3)
    check_projections_faithful(oracle, ops, gu_h, ii, jj, n, k, "swiglu 8192x8192x5120 (every tile)")
    # eight whole rows (both CTAs of a pair, the first and the last tile rows) against the fp64 composition
    rows = np.array([0, 1, 127, 128, 4095, 5000, 8190, 8191])
    check_explained_vs_composition(oracle, ops, gsf, q[rows], sf_logical(sf, m, n)[rows], gu_h[rows], rows, n, k,
                                   "swiglu 8192x8192x5120 (rows)")
