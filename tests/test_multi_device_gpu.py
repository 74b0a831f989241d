"""The library keeps its launch set-up per device (the dynamic shared-memory opt-in and the
persistent grid size are properties of the current device): a process that uses two GPUs
must get the same results on both.  Runs when two or more GPUs are visible, skips
otherwise."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two visible GPUs")
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    yield


def on_device(dev):
    """The kernels whose launch set-up is per device: the GEMMs (plain, low-rank, SiLU * up),
    the one-launch global scale and quantize, and the SVDQuant input stage."""
    with torch.cuda.device(dev):
        def bf16(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
        x = bf16(S.normal_bf16((384, 512), 1.0, 8, S.TID["x"]))
        w = bf16(S.normal_bf16((512, 512), 0.02, 8, S.TID["w"]))
        amax_w, gsf_w, _ = nv.nvfp4_global_scale(w)
        wq, wsf = nv.nvfp4_quantize(w, gsf_w)
        amax, gsf, alpha, xq, xsf = nv.nvfp4_global_scale_quantize(x, other_amax=amax_w)
        out = nv.nvfp4_gemm(xq, wq, xsf, wsf, alpha)
        d = bf16(S.normal_bf16((384, 64), 1.0, 8, S.TID["d"]))
        l1 = bf16(S.normal_bf16((512, 64), 0.01, 8, S.TID["l1"]))
        out_lr = nv.nvfp4_gemm_lowrank_bias(xq, wq, xsf, wsf, alpha, d, l1)
        hq, hsf = nv.nvfp4_gemm_silu_mul_quantize(xq, wq[:256], wq[256:], xsf, wsf[:nv.nvfp4_scale_bytes(256, 512)],
                                                  wsf[nv.nvfp4_scale_bytes(256, 512):], alpha, alpha, gsf)
        pqs = bf16(np.full(512, 0x3F80, np.uint16))
        wd = bf16(S.normal_bf16((64, 512), 0.05, 8, S.TID["lora_down"]))
        sq, ssf, dd = nv.nvfp4_quantize_smooth_lora_down(x, pqs, gsf, wd)
        torch.cuda.synchronize()
        assert nv.nvfp4_device_status(clear=True) == 0
        return [host(t) for t in (amax, gsf, alpha, xq, xsf, out, out_lr, hq, hsf, sq, ssf, dd)]


def test_same_results_on_two_devices():
    r0 = on_device(0)
    r1 = on_device(1)
    for a, b in zip(r0, r1):
        assert (a == b).all()
