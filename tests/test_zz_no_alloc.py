"""The non-allocating batched global scale, called through the C ABI.

Some callers cannot let the library allocate device memory: hosts whose device memory
belongs to their own allocator or is a fixed budget set at start-up, and paths that must
not risk the implicit synchronization of cudaMalloc.  nvfp4_global_scale_batched_noalloc
takes its reduction scratch from a fixed array inside the library instead; these checks
compare it with the allocating entry point and with the oracle on two calls in a row (the
array is reused and must be cleared by each call), and check its size limit.  The file name sorts last so a
run that stops at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S

pytestmark = pytest.mark.gpu

INVALID = 1


@pytest.fixture(scope="module")
def lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    return nv.load_library()


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def call_noalloc(lib, x, mask, silu, amax, gsf):
    b, m, w = x.shape
    k = w // 2 if silu else w
    st = lib.nvfp4_global_scale_batched_noalloc(
        ctypes.c_void_p(x.data_ptr()), b, m, k, None if mask is None else ctypes.c_void_p(mask.data_ptr()),
        int(silu), ctypes.c_void_p(amax.data_ptr()), ctypes.c_void_p(gsf.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("silu", [False, True])
def test_noalloc_matches_allocating_entry_point(lib, oracle, silu):
    b, m, k = 6, 90, 64
    for call, seed in enumerate((31, 32)):                  # two calls in a row, different data
        w = 2 * k if silu else k
        x = to_dev(S.normal_bf16((b, m, w), 1.0 + call, seed=seed))
        mask = torch.tensor([0, 90, 1, 33, 89, 45], dtype=torch.int32, device="cuda")
        ref_amax, ref_gsf = nv.nvfp4_global_scale_batched(x, mask, silu_mul=silu)
        amax = torch.full((b,), -1.0, dtype=torch.float32, device="cuda")
        gsf = torch.full((b,), -1.0, dtype=torch.float32, device="cuda")
        assert call_noalloc(lib, x, mask, silu, amax, gsf) == 0
        torch.cuda.synchronize()
        # the reduction is a max, so the result is exact: the tolerance is zero
        assert torch.equal(amax, ref_amax) and torch.equal(gsf, ref_gsf), (call, amax, ref_amax)
        # and both equal the oracle's per-item global scale over the valid rows
        o_amax, o_gsf = oracle.global_scale_batched(S.normal_bf16((b, m, w), 1.0 + call, seed=seed),
                                                    mask.cpu().numpy(), silu_mul=silu)
        assert (amax.cpu().numpy() == o_amax).all() and (gsf.cpu().numpy() == o_gsf).all()


def test_noalloc_without_mask_and_size_limit(lib, oracle):
    x_bits = S.normal_bf16((3, 17, 48), 2.0, seed=5)
    x = to_dev(x_bits)
    ref_amax, ref_gsf = nv.nvfp4_global_scale_batched(x, None)
    o_amax, o_gsf = oracle.global_scale_batched(x_bits, None)
    assert (ref_amax.cpu().numpy() == o_amax).all() and (ref_gsf.cpu().numpy() == o_gsf).all()
    amax = torch.empty(3, dtype=torch.float32, device="cuda")
    gsf = torch.empty(3, dtype=torch.float32, device="cuda")
    for _ in range(2):
        assert call_noalloc(lib, x, None, False, amax, gsf) == 0
        torch.cuda.synchronize()
        assert torch.equal(amax, ref_amax) and torch.equal(gsf, ref_gsf)
    # more items than the fixed scratch holds: rejected before anything is launched
    big = torch.zeros((1025, 1, 8), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(1025, dtype=torch.float32, device="cuda")
    assert call_noalloc(lib, big, None, False, out, out) == INVALID
    assert nv.nvfp4_device_status(clear=True) == 0
