"""Full-size end-to-end parity of the two SwiGLU blocks, x -> y through the exact sequence of
library calls the benchmark times [NVIDIA/Fuser PR #5737, module tree: NVFP4InferenceSwiGLU
(gate_proj, up_proj, down_proj) and NVFP4InferenceGroupedSwiGLU for the routed experts;
flashinfer PR #1774: the masked quantizer and the silu_and_mul quantizer of the gate/up
output].

Dense block (tokens 8192, hidden 5120, intermediate 8192):
    nvfp4_global_scale_quantize(x) -> nvfp4_gemm_silu_mul_quantize (gate/up, SiLU * up and
    NVFP4 quantization of h in the epilogue) -> nvfp4_gemm (down).
Routed experts (E = 16, Mmax = 2048, valid rows min(Poisson(512), 2048)):
    nvfp4_quantize_masked_batched(x) -> nvfp4_grouped_gemm_silu_mul_quantize_masked ->
    nvfp4_grouped_gemm_masked (down).

Every intermediate is checked against the oracle: the activation's scalars and NVFP4 bytes
bit for bit (whole tensors); h bit for bit against the oracle's SiLU-and-mul quantizer on
the library's own bf16 projections (every valid row); y at 64 rows (two in every 256-row
tile) against the oracle's down GEMM of the path's own h (the tolerance and faithful
rounding); and y against the oracle's whole composition at the same rows (its own
projections rounded once, its own h), where a difference beyond the tolerance is allowed
only by the exact effect of the h blocks that differ, and those differ only at near-tie
projections (the projections' own check).  Weights are quantized by the oracle (offline
weight quantization)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import (GEMM_ATOL_OF_MAX, GEMM_RTOL, bf16_value, check_explained_vs_composition, check_full_size,
                           dev_bf16, dev_f32, dev_i32, dev_u8, host, sf_logical)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


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


def rows_per_tile(valid, seed, per_tile=2, tile=256):
    """`per_tile` seeded rows of every `tile`-row tile below `valid`, plus the first and the
    last valid row (sorted, distinct)."""
    g = np.random.default_rng([seed, 4242])
    rows = {0, valid - 1}
    for r0 in range(0, valid, tile):
        r1 = min(valid, r0 + tile)
        rows.update(g.choice(np.arange(r0, r1), size=min(per_tile, r1 - r0), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


def check_y(oracle, y_rows, hq, hsf, qwd, swd, alpha_d, hq_ref, hsf_ref, rows, H, I, what):
    """y at `rows` (bf16 bits [len, H]): against the oracle's down GEMM of the path's own h
    (hq, hsf: the whole [M, I/2] codes and swizzled scales), within the tolerance and as a
    faithful rounding; then against the oracle's composition (hq_ref, hsf_ref: the oracle's
    own h for `rows`, [len, I/2] and a swizzled buffer for len rows), whose difference may
    exceed the tolerance only by the exact difference the differing h blocks make."""
    ii, jj = np.repeat(rows, H), np.tile(np.arange(H), len(rows))
    y_full = np.zeros((int(rows.max()) + 1, H), np.uint16)
    y_full[rows] = y_rows
    check_full_size(oracle, y_full, hq, hsf, qwd, swd, alpha_d, I, ii, jj, f"{what}: y vs down(h of the path)")
    y_path = oracle.gemm_ref_sampled(hq, qwd, hsf, swd, alpha_d, I, ii, jj).reshape(len(rows), H)
    y_comp = oracle.gemm_ref(hq_ref, qwd, hsf_ref, swd, alpha_d, len(rows), H, I)
    got = bf16_value(y_rows)
    tol = GEMM_RTOL * np.abs(y_comp) + GEMM_ATOL_OF_MAX * np.abs(y_comp).max() + np.abs(y_path - y_comp)
    bad = np.abs(got - y_comp) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} y values beyond the tolerance of the composition"
    print(f"{what}: y at {len(rows)} rows within tolerance of the oracle composition; the path's h moves "
          f"{int((y_path != y_comp).any(axis=1).sum())} of these rows")


def test_dense_swiglu_block_full_size_x_to_y(oracle):
    M, H, I = 8192, 5120, 8192
    d = S.swiglu_block()
    am_wgu, g_wgu = oracle.global_scale(d["w_gate_up"])
    qwgu, swgu = oracle.quantize(d["w_gate_up"], g_wgu)
    am_wd, g_wd = oracle.global_scale(d["w_down"])
    qwd, swd = oracle.quantize(d["w_down"], g_wd)
    half = nv.nvfp4_scale_bytes(I, H)
    wgu_q, wgu_sf = dev_u8(qwgu), dev_u8(swgu)
    # 1. amax, global scale, gate/up alpha and the quantized x in one launch
    amax_x, gsf_x, alpha1, xq, xsf = nv.nvfp4_global_scale_quantize(dev_bf16(d["x"]), other_amax=dev_f32(am_wgu))
    am_o, g_o = oracle.global_scale(d["x"])
    al1 = np.float32(oracle.alpha(float(am_o), float(am_wgu)))
    qx_o, sx_o = oracle.quantize(d["x"], g_o)
    assert host(amax_x)[0] == am_o and host(gsf_x)[0] == g_o and host(alpha1)[0] == al1
    assert (host(xq) == qx_o).all() and (host(xsf) == sx_o).all()
    # the library's bf16 projections calibrate the static scale of h, as a deployed layer would
    g = nv.nvfp4_gemm(xq, wgu_q[:I], xsf, wgu_sf[:half], alpha1)
    u = nv.nvfp4_gemm(xq, wgu_q[I:], xsf, wgu_sf[half:], alpha1)
    gu_h = host(torch.cat([g, u], dim=-1))
    del g, u
    amax_h, gsf_h = oracle.global_scale_batched(gu_h[None], None, silu_mul=True)
    # 2. gate/up with the SiLU * up NVFP4 epilogue
    hq, hsf = nv.nvfp4_gemm_silu_mul_quantize(xq, wgu_q[:I], wgu_q[I:], xsf, wgu_sf[:half], wgu_sf[half:], alpha1,
                                              alpha1, dev_f32(gsf_h[0]))
    hq_h, hsf_h = host(hq), host(hsf)
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h[None], gsf_h)
    assert (hq_h == q_ref[0]).all(), np.argwhere(hq_h != q_ref[0])[:5]
    assert (hsf_h == sf_ref[0]).all(), np.argwhere(hsf_h != sf_ref[0])[:5]
    # 3. down projection
    al2 = np.float32(oracle.alpha(float(amax_h[0]), float(am_wd)))
    y = nv.nvfp4_gemm(hq, dev_u8(qwd), hsf, dev_u8(swd), dev_f32(al2))
    rows = rows_per_tile(M, seed=1)
    y_rows = host(y)[rows]
    # the oracle's own composition at these rows: projections rounded once, its own h
    ops = (qx_o, qwgu[:I], qwgu[I:], sx_o, swgu[:half], swgu[half:], al1, al1)
    gu_ref = oracle.gemm_gate_up_bf16(*ops, I, H, rows)
    check_explained_vs_composition(oracle, ops, gsf_h[0], hq_h[rows], sf_logical(hsf_h, M, I)[rows], gu_h[rows],
                                   rows, I, H, "dense block h", gu_ref=gu_ref)
    hq_ref, hsf_ref = oracle.silu_mul_quantize_batched(gu_ref[None], gsf_h)
    check_y(oracle, y_rows, hq_h, hsf_h, qwd, swd, al2, hq_ref[0], hsf_ref[0], rows, H, I, "dense block")


def test_routed_expert_swiglu_block_full_size_x_to_y(oracle):
    E, mmax, H, I = 16, 2048, 5120, 8192
    d = S.grouped_swiglu(E, mmax, H, I, 512, 0)
    mask = d["mask"]
    qw, sw, amw = {}, {}, {}
    for name in ("w_gate", "w_up", "w_down"):
        amw[name], gw = oracle.global_scale_batched(d[name], None)
        qw[name], sw[name] = oracle.quantize_masked_batched(d[name], gw, None)
        del d[name]
    # static per-expert activation scales (calibration over each expert's valid rows)
    amax_x, gsf_x = oracle.global_scale_batched(d["x"], mask)
    al_g = np.float32([oracle.alpha(float(a), float(b)) for a, b in zip(amax_x, amw["w_gate"])])
    al_u = np.float32([oracle.alpha(float(a), float(b)) for a, b in zip(amax_x, amw["w_up"])])
    mask_d = dev_i32(mask)
    # 1. masked quantize of every expert's tokens
    xq = torch.full((E, mmax, H // 2), 0x5A, dtype=torch.uint8, device="cuda")
    xsf = torch.full((E, nv.nvfp4_scale_bytes(mmax, H)), 0x5A, dtype=torch.uint8, device="cuda")
    nv.nvfp4_quantize_masked_batched(dev_bf16(d["x"]), dev_f32(gsf_x), mask_d, xq, xsf)
    qx_o, sx_o = oracle.quantize_masked_batched(d["x"], gsf_x, mask, q_fill=0x5A, sf_fill=0x5A)
    assert (host(xq) == qx_o).all() and (host(xsf) == sx_o).all()
    del d["x"]
    wg_q, wg_sf, wu_q, wu_sf = (dev_u8(a) for a in (qw["w_gate"], sw["w_gate"], qw["w_up"], sw["w_up"]))
    # library projections per expert calibrate the static scales of h
    g = nv.nvfp4_grouped_gemm_masked(xq, wg_q, xsf, wg_sf, mask_d, dev_f32(al_g))
    u = nv.nvfp4_grouped_gemm_masked(xq, wu_q, xsf, wu_sf, mask_d, dev_f32(al_u))
    gu_h = host(torch.cat([g, u], dim=-1))
    del g, u
    amax_h, gsf_h = oracle.global_scale_batched(gu_h, mask, silu_mul=True)
    # 2. grouped gate/up with the SiLU * up NVFP4 epilogue
    hq = torch.full((E, mmax, I // 2), 0xAB, dtype=torch.uint8, device="cuda")
    hsf = torch.full((E, nv.nvfp4_scale_bytes(mmax, I)), 0xCD, dtype=torch.uint8, device="cuda")
    nv.nvfp4_grouped_gemm_silu_mul_quantize_masked(xq, wg_q, wu_q, xsf, wg_sf, wu_sf, mask_d, dev_f32(al_g),
                                                   dev_f32(al_u), dev_f32(gsf_h), hq, hsf)
    del wg_q, wg_sf, wu_q, wu_sf
    hq_h, hsf_h = host(hq), host(hsf)
    q_ref, sf_ref = oracle.silu_mul_quantize_batched(gu_h, gsf_h, mask, q_fill=0xAB, sf_fill=0xCD)
    assert (hq_h == q_ref).all(), np.argwhere(hq_h != q_ref)[:5]       # rows beyond each mask keep 0xAB
    assert (hsf_h == sf_ref).all(), np.argwhere(hsf_h != sf_ref)[:5]   # their scale entries keep 0xCD
    # 3. grouped down projection; rows beyond each mask stay untouched
    al_d = np.float32([oracle.alpha(float(a), float(b)) for a, b in zip(amax_h, amw["w_down"])])
    y = torch.full((E, mmax, H), -3.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_grouped_gemm_masked(hq, dev_u8(qw["w_down"]), hsf, dev_u8(sw["w_down"]), mask_d, dev_f32(al_d), y)
    y_h = host(y)
    minus3 = S.f32_to_bf16_bits(np.float32([-3.0]))[0]
    checked = 0
    for e in range(E):
        v = int(mask[e])
        assert (y_h[e, v:] == minus3).all(), f"expert {e}: rows beyond the mask were written"
        if not v:
            continue
        rows = rows_per_tile(v, seed=e)            # two per 256-row tile and the mask edge: 64+ rows in all
        ops = (qx_o[e], qw["w_gate"][e], qw["w_up"][e], sx_o[e], sw["w_gate"][e], sw["w_up"][e], al_g[e], al_u[e])
        gu_ref = oracle.gemm_gate_up_bf16(*ops, I, H, rows)
        check_explained_vs_composition(oracle, ops, gsf_h[e], hq_h[e, rows], sf_logical(hsf_h[e], mmax, I)[rows],
                                       gu_h[e, rows], rows, I, H, f"expert {e} h", gu_ref=gu_ref)
        hq_ref, hsf_ref = oracle.silu_mul_quantize_batched(gu_ref[None], gsf_h[e:e + 1])
        check_y(oracle, y_h[e, rows], hq_h[e], hsf_h[e], qw["w_down"][e], sw["w_down"][e], al_d[e], hq_ref[0],
                hsf_ref[0], rows, H, I, f"expert {e}")
        checked += len(rows)
    assert checked >= 64
