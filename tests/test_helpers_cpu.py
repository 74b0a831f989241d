"""CPU checks of the comparison helpers the GPU parity tests rely on: the vectorised
scale-layout reader against the oracle's per-entry offset, the per-tile sampler, the
faithful-rounding check, and the SiLU * up epilogue's checks against planted mistakes
(made in the oracle's inputs or in a copy of its outputs, on the CPU)."""
import numpy as np
import pytest

import nvfp4_synth as S
from tests.helpers import (assert_bf16_faithful, check_explained_vs_composition, check_projections_faithful,
                           f64_to_bf16_bits, sf_logical, tile_positions, unpack_codes)


@pytest.mark.parametrize("rows,k", [(1, 16), (130, 80), (300, 256), (256, 1024)])
def test_sf_logical_matches_oracle_offsets(oracle, rows, k):
    sf = np.random.default_rng(rows + k).integers(0, 256, oracle.scale_bytes(rows, k)).astype(np.uint8)
    got = sf_logical(sf, rows, k)
    want = np.array([[sf[oracle.sf_offset(r, c, k)] for c in range(k // 16)] for r in range(rows)])
    assert (got == want).all()


def test_unpack_codes_low_nibble_first():
    assert unpack_codes(np.array([[0x21, 0xF0]], np.uint8)).tolist() == [[1, 2, 0, 15]]


@pytest.mark.parametrize("m,n,tm,tn", [(300, 520, 256, 256), (8192, 8192, 256, 128), (1, 8, 256, 256)])
def test_tile_positions_cover_every_tile(m, n, tm, tn):
    ii, jj = tile_positions(m, n, tm, tn, seed=1)
    assert ((0 <= ii) & (ii < m) & (0 <= jj) & (jj < n)).all()
    tiles = set(zip((ii // tm).tolist(), (jj // tn).tolist()))
    assert tiles == {(a, b) for a in range(-(-m // tm)) for b in range(-(-n // tn))}
    pts = set(zip(ii.tolist(), jj.tolist()))
    for r0 in range(0, m, tm):
        for c0 in range(0, n, tn):
            r1, c1 = min(m, r0 + tm) - 1, min(n, c0 + tn) - 1
            assert {(r0, c0), (r0, c1), (r1, c0), (r1, c1)} <= pts


def test_bf16_faithful_check():
    one, next_up = 0x3F80, 0x3F81           # 1.0 and 1 + 2^-7
    tie = 1.0 + 2.0 ** -8
    # nearest: accepted with no difference
    assert assert_bf16_faithful([one], [one], [1.0], [0.0]) == (0, 0.0)
    # the other neighbour of an exact value within the bound of the tie: accepted
    assert assert_bf16_faithful([next_up], [one], [tie - 2.0 ** -20], [2.0 ** -18])[0] == 1
    # ... but not when the exact value is farther from the tie than the bound
    with pytest.raises(AssertionError):
        assert_bf16_faithful([next_up], [one], [tie - 2.0 ** -12], [2.0 ** -18])
    # two steps away is never a faithful rounding
    with pytest.raises(AssertionError):
        assert_bf16_faithful([0x3F82], [one], [tie], [1.0])
    # signed zeros are the same value
    assert assert_bf16_faithful([0x8000], [0x0000], [0.0], [0.0]) == (0, 0.0)
    # adjacency across zero: the smallest subnormals of either sign
    assert assert_bf16_faithful([0x8001], [0x0000], [-(2.0 ** -134)], [2.0 ** -140])[0] == 1


def _silu_ops(oracle, seed, m=64, n=128, k=256):
    """Quantized operands (oracle argument order) with their real alphas and an
    oracle-calibrated gsf_h, and the oracle's own bf16 projections [g | u]."""
    xa = S.normal_bf16((m, k), 1.0, seed)
    xg = S.normal_bf16((n, k), 0.05, seed, 2)
    xu = S.normal_bf16((n, k), 0.05, seed, 3)
    outs, amax = [], []
    for x in (xa, xg, xu):
        am, g = oracle.global_scale(x)
        outs.append(oracle.quantize(x, g))
        amax.append(float(am))
    (qa, sa), (qg, sg), (qu, su) = outs
    al_g = np.float32(oracle.alpha(amax[0], amax[1]))
    al_u = np.float32(oracle.alpha(amax[0], amax[2]))
    ops = (qa, qg, qu, sa, sg, su, al_g, al_u)
    gu = oracle.gemm_gate_up_bf16(*ops, n, k, np.arange(m))
    gsf = oracle.global_scale_batched(gu[None], None, silu_mul=True)[1][0]
    return ops, np.float32(gsf), gu


def _quantized(oracle, gu, gsf, m, n):
    q, sf = oracle.silu_mul_quantize_batched(gu[None], np.float32([gsf]))
    return q[0], sf_logical(sf[0], m, n)


def test_epilogue_checks_accept_the_oracle_and_reject_planted_mistakes(oracle):
    m, n, k = 64, 128, 256
    ops, gsf, gu = _silu_ops(oracle, 1)
    rows = np.arange(m)
    q, s = _quantized(oracle, gu, gsf, m, n)
    check_explained_vs_composition(oracle, ops, gsf, q, s, gu, rows, n, k, "identical")
    ii, jj = np.repeat(rows, n), np.tile(np.arange(n), m)
    assert [st[0] for st in check_projections_faithful(oracle, ops, gu, ii, jj, n, k, "identical")] == [0, 0]
    # gate and up swapped: the projections are wrong, so the faithful check fails ...
    ops_sw = (ops[0], ops[2], ops[1], ops[3], ops[5], ops[4], ops[6], ops[7])
    gu_sw = oracle.gemm_gate_up_bf16(*ops_sw, n, k, rows)
    with pytest.raises(AssertionError):
        check_projections_faithful(oracle, ops, gu_sw, ii, jj, n, k, "swapped")
    # ... and so is the composition check on the swapped projections' output
    q_sw, s_sw = _quantized(oracle, gu_sw, gsf, m, n)
    with pytest.raises(AssertionError):
        check_explained_vs_composition(oracle, ops, gsf, q_sw, s_sw, gu_sw, rows, n, k, "swapped")
    # alpha of the gate projection off by 25%
    ops_al = ops[:6] + (np.float32(ops[6] * 1.25), ops[7])
    gu_al = oracle.gemm_gate_up_bf16(*ops_al, n, k, rows)
    q_al, s_al = _quantized(oracle, gu_al, gsf, m, n)
    with pytest.raises(AssertionError):
        check_explained_vs_composition(oracle, ops, gsf, q_al, s_al, gu_al, rows, n, k, "alpha")
    # one projection one bf16 step off where the exact value is far from a tie
    exact = oracle.gemm_ref_sampled(ops[0], ops[1], ops[3], ops[4], ops[6], k, np.array([5]), np.array([7]))
    assert f64_to_bf16_bits(oracle, exact)[0] == gu[5, 7]
    gu_1 = gu.copy()
    gu_1[5, 7] += 1
    q_1, s_1 = _quantized(oracle, gu_1, gsf, m, n)
    with pytest.raises(AssertionError):
        check_explained_vs_composition(oracle, ops, gsf, q_1, s_1, gu_1, rows, n, k, "one step")
    # an output block changed while every projection is exact
    q_b = q.copy()
    q_b[9, 3] ^= 0x01
    with pytest.raises(AssertionError):
        check_explained_vs_composition(oracle, ops, gsf, q_b, s, gu, rows, n, k, "planted code")


def test_synth_leading_items_match_whole_tensor(monkeypatch):
    # small chunks so the test stays small: items of 1200 values, item 1 straddles the
    # 2048-value chunk boundary
    monkeypatch.setattr(S, "CHUNK", 1 << 11)
    whole = S.normal_bf16((3, 40, 30), 0.02, 4, 11)
    for items in (1, 2):
        part = S.normal_bf16((3, 40, 30), 0.02, 4, 11, items=items)
        assert part.shape == (items, 40, 30)
        assert (part == whole[:items]).all()
