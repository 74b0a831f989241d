"""Programmatic dependent launch changes only when a kernel may start, never what it
computes [flashinfer docs mm_nvfp4_svdquant, Parameters: enable_pdl].  Each kernel of the
library waits for its predecessor before its first global access, so every byte of every
output must be the same with nvfp4_set_pdl(1) and nvfp4_set_pdl(0): checked on the dense
SwiGLU step, the routed-expert step and the SVDQuant layer, run back to back on one stream
exactly as the benchmark chains them."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import dev_bf16, dev_f32, dev_i32, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    yield
    assert nv.nvfp4_device_status(clear=True) == 0


def weight(bits):
    amax, gsf, _ = nv.nvfp4_global_scale(dev_bf16(bits))
    q, sf = nv.nvfp4_quantize(dev_bf16(bits), gsf)
    return q, sf, amax


def dense_step(M=1024, H=1024, I=768):
    x = dev_bf16(S.normal_bf16((M, H), 1.0, 3, S.TID["x"]))
    wgu_q, wgu_sf, am_wgu = weight(S.normal_bf16((2 * I, H), 0.02, 3, S.TID["w_gate_up"]))
    wd_q, wd_sf, _ = weight(S.normal_bf16((H, I), 0.02, 3, S.TID["w_down"]))
    half = nv.nvfp4_scale_bytes(I, H)
    gsf_h = dev_f32(np.float32(2688.0 / 3.0))
    alpha2 = dev_f32(np.float32(1e-5))

    def run():
        amax, gsf, alpha1, xq, xsf = nv.nvfp4_global_scale_quantize(x, other_amax=am_wgu)
        hq, hsf = nv.nvfp4_gemm_silu_mul_quantize(xq, wgu_q[:I], wgu_q[I:], xsf, wgu_sf[:half], wgu_sf[half:], alpha1,
                                                  alpha1, gsf_h)
        y = nv.nvfp4_gemm(hq, wd_q, hsf, wd_sf, alpha2)
        return [amax, gsf, alpha1, xq, xsf, hq, hsf, y]
    return run


def routed_step(E=4, mmax=384, H=512, I=256):
    mask = dev_i32(np.array([384, 0, 129, 300], np.int32))
    x = dev_bf16(S.normal_bf16((E, mmax, H), 1.0, 4, S.TID["x"]))
    ws = {}
    for name, shape in (("g", (E, I, H)), ("u", (E, I, H)), ("d", (E, H, I))):
        bits = dev_bf16(S.normal_bf16(shape, 0.02, 4, S.TID["w_" + {"g": "gate", "u": "up", "d": "down"}[name]]))
        _, gw = nv.nvfp4_global_scale_batched(bits, None)
        ws[name] = nv.nvfp4_quantize_masked_batched(bits, gw, None)
    _, gsf_x = nv.nvfp4_global_scale_batched(x, mask)
    al = dev_f32(np.full(E, 1e-4, np.float32))
    gsf_h = dev_f32(np.full(E, 500.0, np.float32))

    def run():
        xq = torch.zeros((E, mmax, H // 2), dtype=torch.uint8, device="cuda")
        xsf = torch.zeros((E, nv.nvfp4_scale_bytes(mmax, H)), dtype=torch.uint8, device="cuda")
        hq = torch.zeros((E, mmax, I // 2), dtype=torch.uint8, device="cuda")
        hsf = torch.zeros((E, nv.nvfp4_scale_bytes(mmax, I)), dtype=torch.uint8, device="cuda")
        y = torch.zeros((E, mmax, H), dtype=torch.bfloat16, device="cuda")
        nv.nvfp4_quantize_masked_batched(x, gsf_x, mask, xq, xsf)
        nv.nvfp4_grouped_gemm_silu_mul_quantize_masked(xq, ws["g"][0], ws["u"][0], xsf, ws["g"][1], ws["u"][1], mask,
                                                       al, al, gsf_h, hq, hsf)
        nv.nvfp4_grouped_gemm_masked(hq, ws["d"][0], hsf, ws["d"][1], mask, al, y)
        return [xq, xsf, hq, hsf, y]
    return run


def svdquant_step(m=512, k=1024, n=768, r=64):
    d = S.svdquant_linear(m, k, n, r, 5)
    x, pqs, w_down = dev_bf16(d["x"]), dev_bf16(d["pqs"]), dev_bf16(d["w_down"])
    wq, wsf, _ = weight(d["w"])
    gsf = dev_f32(np.float32(100.0))
    alpha = dev_f32(np.float32(1e-4))
    l1 = dev_bf16(S.f32_to_bf16_bits(d["l1_f32"]))
    bias = dev_bf16(d["bias"])

    def run():
        xq, xsf, dd = nv.nvfp4_quantize_smooth_lora_down(x, pqs, gsf, w_down)
        out = nv.nvfp4_gemm_lowrank_bias(xq, wq, xsf, wsf, alpha, dd, l1, bias)
        return [xq, xsf, dd, out]
    return run


@pytest.mark.parametrize("make", [dense_step, routed_step, svdquant_step])
def test_pdl_on_and_off_give_identical_bytes(make):
    run = make()
    before = nv.nvfp4_get_pdl()
    try:
        results = []
        for pdl in (True, False, True):
            nv.nvfp4_set_pdl(pdl)
            results.append([host(t) for t in run()])
            torch.cuda.synchronize()
    finally:
        nv.nvfp4_set_pdl(before)
    for other in results[1:]:
        for a, b in zip(results[0], other):
            assert a.shape == b.shape and (a == b).all()
