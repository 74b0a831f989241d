"""GPU parity of the SVDQuant input stage: the smooth quantizer (bit-exact against the
oracle), the LoRA-down product d = x @ w^T (within the GEMM tolerance of the oracle's fp64
dot products), and the fused op that produces both in one pass over x (bit-identical to
the two separate calls).  Sizes span ragged M, K split unevenly over the 4 CTAs of a
cluster (including a CTA with no K chunk), ranks 32 to 256, and the full 4096 x 3072
layer with r in {32, 64, 128}; the last test runs the whole SVDQuant linear layer."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import assert_gemm_close, bf16_to_f64, dev_bf16, dev_f32, dev_u8, host

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


def smooth_inputs(oracle, m, k, r, seed):
    """x ~ N(0,1), pre_quant_scale ~ U[0.25, 4], w ~ N(0, 0.05) (bf16 bits), and gsf of x_hat
    from the oracle (448*6 / amax(bf16(x * pqs)))."""
    x = S.normal_bf16((m, k), 1.0, seed, S.TID["x"])
    pqs = S.f32_to_bf16_bits(S.rng(seed, S.TID["bias"]).uniform(0.25, 4.0, k).astype(np.float32))
    w = S.normal_bf16((r, k), 0.05, seed, S.TID["d"]) if r else None
    xh = S.f32_to_bf16_bits(S.bf16_bits_to_f32(x) * S.bf16_bits_to_f32(pqs)[None, :])
    _, gsf = oracle.global_scale(xh)
    return x, pqs, w, np.float32(gsf)


@pytest.mark.parametrize("m,k", [(1, 16), (130, 80), (300, 208), (257, 3072)])
def test_quantize_smooth_bit_exact(oracle, m, k):
    x, pqs, _, gsf = smooth_inputs(oracle, m, k, 0, seed=m + k)
    q, sf = nv.nvfp4_quantize_smooth(dev_bf16(x), dev_bf16(pqs), dev_f32(gsf))
    q_ref, sf_ref = oracle.quantize_smooth(x, pqs, gsf)
    assert (host(q) == q_ref).all(), np.argwhere(host(q) != q_ref)[:5]
    assert (host(sf) == sf_ref).all(), np.argwhere(host(sf) != sf_ref)[:5]


@pytest.mark.parametrize("m,k,r", [(128, 64, 32), (300, 320, 64), (1, 256, 128), (513, 1024, 96), (200, 3072, 256)])
def test_lora_down(oracle, m, k, r):
    x, _, w, _ = smooth_inputs(oracle, m, k, r, seed=m + k + r)
    d = nv.nvfp4_lora_down(dev_bf16(x), dev_bf16(w))
    assert_gemm_close(bf16_to_f64(d), oracle.lora_down(x, w), f"lora-down {m}x{k} r={r}")


@pytest.mark.parametrize("m,k,r", [(300, 320, 64), (129, 256, 32), (513, 1024, 128), (64, 3072, 256)])
def test_fused_equals_separate_calls(oracle, m, k, r):
    x, pqs, w, gsf = smooth_inputs(oracle, m, k, r, seed=7 * m + k)
    xd, pd, wd, gd = dev_bf16(x), dev_bf16(pqs), dev_bf16(w), dev_f32(gsf)
    # outputs in the middle of sentinel-filled buffers: nothing around them may change
    qn, sn, dn = m * k // 2, nv.nvfp4_scale_bytes(m, k), m * r
    qbig = torch.full((qn + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    sbig = torch.full((sn + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    dbig = torch.full((dn + 64,), 3.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_quantize_smooth_lora_down(xd, pd, gd, wd, qbig[32:32 + qn].view(m, k // 2), sbig[32:32 + sn],
                                       dbig[32:32 + dn].view(m, r))
    qh, sh = host(qbig), host(sbig)
    assert (qh[:32] == 0x5A).all() and (qh[32 + qn:] == 0x5A).all()
    assert (sh[:32] == 0xA5).all() and (sh[32 + sn:] == 0xA5).all()
    assert (dbig[:32] == 3.0).all() and (dbig[32 + dn:] == 3.0).all()
    q_s, sf_s = nv.nvfp4_quantize_smooth(xd, pd, gd)
    d_s = nv.nvfp4_lora_down(xd, wd)
    assert (qh[32:32 + qn] == host(q_s).reshape(-1)).all()
    assert (sh[32:32 + sn] == host(sf_s)).all()
    assert (host(dbig[32:32 + dn]) == host(d_s).reshape(-1)).all()
    q_ref, sf_ref = oracle.quantize_smooth(x, pqs, gsf)
    assert (qh[32:32 + qn] == q_ref.reshape(-1)).all() and (sh[32:32 + sn] == sf_ref).all()


@pytest.mark.parametrize("r", [32, 64, 128])
def test_full_size_layer_input(oracle, r):
    m, k = 4096, 3072
    x, pqs, w, gsf = smooth_inputs(oracle, m, k, r, seed=r)
    q, sf, d = nv.nvfp4_quantize_smooth_lora_down(dev_bf16(x), dev_bf16(pqs), dev_f32(gsf), dev_bf16(w))
    q_ref, sf_ref = oracle.quantize_smooth(x, pqs, gsf)
    assert (host(q) == q_ref).all() and (host(sf) == sf_ref).all()
    assert_gemm_close(bf16_to_f64(d), oracle.lora_down(x, w), f"lora-down full r={r}")


def test_svdquant_linear_end_to_end(oracle):
    # x -> (smooth quantize, LoRA-down) -> residual FP4 GEMM + rank-r correction + bias
    m, k, n, r = 300, 512, 384, 64
    x, pqs, w, gsf = smooth_inputs(oracle, m, k, r, seed=31)
    wres = S.normal_bf16((n, k), 0.02, 31, S.TID["w"])
    amax_w, gw = oracle.global_scale(wres)
    qw, sfw = oracle.quantize(wres, gw)
    alpha = np.float32(oracle.alpha(float(2688.0 / gsf), float(amax_w)))
    l1 = S.f32_to_bf16_bits(S.rng(31, S.TID["l1"]).standard_normal((n, r), dtype=np.float32) * np.float32(0.01) / alpha)
    bias = S.normal_bf16((n,), 0.1, 31, S.TID["bias"])
    q, sf, d = nv.nvfp4_quantize_smooth_lora_down(dev_bf16(x), dev_bf16(pqs), dev_f32(gsf), dev_bf16(w))
    out = nv.nvfp4_gemm_lowrank_bias(q, dev_u8(qw), sf, dev_u8(sfw), dev_f32(alpha), d, dev_bf16(l1), dev_bf16(bias))
    # the oracle's composition: its own quantized x and its own d (fp64 rounded once to bf16)
    q_ref, sf_ref = oracle.quantize_smooth(x, pqs, gsf)
    d_ref = np.vectorize(oracle.f64_to_bf16, otypes=[np.uint16])(oracle.lora_down(x, w))
    ref = oracle.gemm_ref(q_ref, qw, sf_ref, sfw, alpha, m, n, k, d=d_ref, l1=l1, bias=bias)
    assert_gemm_close(bf16_to_f64(out), ref, "svdquant linear")
