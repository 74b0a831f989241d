"""CPU checks of the comparison helpers the GPU parity tests rely on: the vectorised
scale-layout reader against the oracle's per-entry offset, and the NVFP4 closeness check
against planted mistakes (made in the oracle's inputs, on the CPU)."""
import numpy as np
import pytest

import nvfp4_synth as S
from tests.helpers import assert_nvfp4_close, sf_logical, unpack_codes


@pytest.mark.parametrize("rows,k", [(1, 16), (130, 80), (300, 256), (256, 1024)])
def test_sf_logical_matches_oracle_offsets(oracle, rows, k):
    sf = np.random.default_rng(rows + k).integers(0, 256, oracle.scale_bytes(rows, k)).astype(np.uint8)
    got = sf_logical(sf, rows, k)
    want = np.array([[sf[oracle.sf_offset(r, c, k)] for c in range(k // 16)] for r in range(rows)])
    assert (got == want).all()


def test_unpack_codes_low_nibble_first():
    assert unpack_codes(np.array([[0x21, 0xF0]], np.uint8)).tolist() == [[1, 2, 0, 15]]


def _silu_case(oracle, seed, swap=False, alpha_scale=1.0):
    """Quantized operands with their real alphas and an oracle-calibrated gsf_h."""
    m, n, k = 64, 128, 256
    xa = S.normal_bf16((m, k), 1.0, seed)
    xg = S.normal_bf16((n, k), 0.05, seed, 2)
    xu = S.normal_bf16((n, k), 0.05, seed, 3)
    outs, amax = [], []
    for x in (xa, xg, xu):
        am, g = oracle.global_scale(x)
        outs.append(oracle.quantize(x, g))
        amax.append(float(am))
    (qa, sa), (qg, sg), (qu, su) = outs
    al_g, al_u = oracle.alpha(amax[0], amax[1]), oracle.alpha(amax[0], amax[2])
    x = oracle.gemm_gate_up_bf16(qa, qg, qu, sa, sg, su, al_g, al_u, n, k, np.arange(m))
    _, gsf = oracle.global_scale_batched(x[None], None, silu_mul=True)
    if swap:
        qg, sg, qu, su = qu, su, qg, sg
    q, sf = oracle.gemm_silu_mul_quantize(qa, qg, qu, sa, sg, su, al_g * alpha_scale, al_u, gsf[0], m, n, k)
    return q, sf_logical(sf, m, n), gsf[0]


def test_nvfp4_close_accepts_identical_and_rejects_planted_mistakes(oracle):
    q, s, gsf = _silu_case(oracle, 1)
    assert assert_nvfp4_close(q, s, q, s, gsf) == (0.0, 0.0)
    for kw in ({"swap": True}, {"alpha_scale": 1.25}):
        q2, s2, _ = _silu_case(oracle, 1, **kw)
        with pytest.raises(AssertionError):
            assert_nvfp4_close(q2, s2, q, s, gsf)


def test_synth_leading_items_match_whole_tensor(monkeypatch):
    # small chunks so the test stays small: items of 1200 values, item 1 straddles the
    # 2048-value chunk boundary
    monkeypatch.setattr(S, "CHUNK", 1 << 11)
    whole = S.normal_bf16((3, 40, 30), 0.02, 4, 11)
    for items in (1, 2):
        part = S.normal_bf16((3, 40, 30), 0.02, 4, 11, items=items)
        assert part.shape == (items, 40, 30)
        assert (part == whole[:items]).all()
