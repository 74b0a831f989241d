"""Host-only checks of the C-ABI library: it builds, loads, exports every symbol that
include/nvfp4.h declares, and rejects invalid arguments before touching the GPU.
None of these call a kernel."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_16_b200 as nv
from nvfp4_block_scaled_16_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INVALID = 1


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"^NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    return nv.load_library()


def test_library_exports_every_declared_symbol(lib):
    decl = declared_symbols()
    assert decl, "no declarations found"
    assert decl == set(binding.EXPORTED_SYMBOLS) | (decl - set(binding.EXPORTED_SYMBOLS))
    handle = ctypes.CDLL(nv.library_path())
    for name in sorted(decl):
        assert hasattr(handle, name), f"{name} declared in include/ but not exported"
    for name in binding.EXPORTED_SYMBOLS:
        assert name in decl, f"{name} bound in Python but not declared in include/"


@pytest.mark.parametrize("rows,k,expect", [(128, 256, 2048), (8192, 8192, 4194304), (129, 16, 1024),
                                           (0, 64, 0), (200, 80, 2048), (5, 8, -1), (-1, 16, -1)])
def test_scale_bytes(lib, rows, k, expect):
    assert nv.nvfp4_scale_bytes(rows, k) == expect


def test_status_strings(lib):
    assert nv.nvfp4_status_string(0) == "NVFP4_OK"
    assert nv.nvfp4_status_string(1) == "NVFP4_ERR_INVALID_ARGUMENT"
    assert nv.nvfp4_status_string(4) == "NVFP4_ERR_DEVICE_TIMEOUT"
    assert nv.nvfp4_status_string(6) == "NVFP4_ERR_INDEX"
    assert nv.nvfp4_status_string(99) == "NVFP4_ERR_UNKNOWN"


def test_release_library_has_no_index_checks(lib):
    # the default library is the release build; the debug build reports its checks
    assert nv.nvfp4_debug_index_checks() is (nv.library_path().endswith("_debug.so"))


P = ctypes.c_void_p
A16 = P(1 << 20)      # 16-byte aligned fake address, never dereferenced by validation
A1 = P((1 << 20) + 1)  # misaligned


@pytest.mark.parametrize("args", [
    (A16, 4, 32, P(0), A16, A16, None),      # null gsf
    (A1, 4, 32, A16, A16, A16, None),        # misaligned x
    (A16, 4, 24, A16, A16, A16, None),       # k % 16 != 0
    (A16, -1, 32, A16, A16, A16, None),      # negative m
])
def test_quantize_rejects_invalid(lib, args):
    assert lib.nvfp4_quantize(*args) == INVALID


def test_quantize_empty_is_noop(lib):
    # m == 0 or k == 0: nothing to do, no device needed
    assert lib.nvfp4_quantize(None, 0, 32, None, None, None, None) == 0
    assert lib.nvfp4_quantize_masked_batched(None, 0, 4, 32, None, None, None, None, None) == 0


def test_silu_rejects_odd_width(lib):
    assert lib.nvfp4_silu_mul_quantize_batched(A16, 1, 4, 40, None, A16, A16, A16, None) == INVALID


@pytest.mark.parametrize("m,n,k", [(128, 256, 96), (128, 250, 256), (128, 256, 0)])
def test_gemm_rejects_bad_shapes(lib, m, n, k):
    assert lib.nvfp4_gemm(A16, A16, A16, A16, A16, None, A16, m, n, k, None) == INVALID


def test_gemm_rejects_null_and_misaligned(lib):
    assert lib.nvfp4_gemm(A16, P(0), A16, A16, A16, None, A16, 128, 256, 256, None) == INVALID
    assert lib.nvfp4_gemm(A16, A16, A1, A16, A16, None, A16, 128, 256, 256, None) == INVALID
    assert lib.nvfp4_gemm(A16, A16, A16, A16, A16, A1, A16, 128, 256, 256, None) == INVALID


@pytest.mark.parametrize("r", [0, 16, 48, 288, -32])
def test_lowrank_rejects_bad_rank(lib, r):
    assert lib.nvfp4_gemm_lowrank_bias(A16, A16, A16, A16, A16, A16, A16, r, None, A16, 128, 256, 256, None) == INVALID


def test_grouped_requires_mask(lib):
    assert lib.nvfp4_grouped_gemm_masked(A16, A16, A16, A16, None, A16, A16, 2, 128, 256, 256, None) == INVALID
    assert lib.nvfp4_grouped_gemm_masked(A16, A16, A16, A16, A16, A16, A16, 2000, 128, 256, 256, None) == INVALID


def test_global_scale_argument_checks(lib):
    assert lib.nvfp4_global_scale(A16, 16, None, None, None, None, None) == INVALID          # gsf required
    assert lib.nvfp4_global_scale(A16, 16, None, A16, A16, None, None) == INVALID           # alpha_out required
    assert lib.nvfp4_global_scale(A1, 16, None, A16, None, None, None) == INVALID            # misaligned
    assert lib.nvfp4_global_scale_batched(A16, 5000, 4, 16, None, 0, None, A16, None) == INVALID


def test_valid_call_without_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments reach the device query, which must report an error (no fallback)
    st = lib.nvfp4_quantize(A16, 4, 32, A16, A16, A16, None)
    assert st != 0


@pytest.mark.parametrize("n", [0 + 64, 200, 136])
def test_silu_mul_gemm_rejects_width_not_multiple_of_128(lib, n):
    args = [A16] * 11
    assert lib.nvfp4_gemm_silu_mul_quantize(*args, 256, n, 256, None) == INVALID


def test_silu_mul_gemm_rejects_null_and_misaligned(lib):
    for i in range(11):                     # every pointer argument is required
        args = [A16] * 11
        args[i] = None
        assert lib.nvfp4_gemm_silu_mul_quantize(*args, 256, 256, 256, None) == INVALID, i
    args = [A16] * 11
    args[2] = A1                            # b_up misaligned
    assert lib.nvfp4_gemm_silu_mul_quantize(*args, 256, 256, 256, None) == INVALID
    assert lib.nvfp4_gemm_silu_mul_quantize(*([A16] * 11), 256, 256, 96, None) == INVALID    # k % 64


def test_grouped_silu_mul_gemm_argument_checks(lib):
    args = [A16] * 12
    assert lib.nvfp4_grouped_gemm_silu_mul_quantize_masked(*args, 2000, 128, 256, 256, None) == INVALID
    args[6] = None                          # mask required
    assert lib.nvfp4_grouped_gemm_silu_mul_quantize_masked(*args, 2, 128, 256, 256, None) == INVALID
    assert lib.nvfp4_grouped_gemm_silu_mul_quantize_masked(*([A16] * 12), 0, 128, 256, 256, None) == 0  # empty


def test_pdl_switch(lib):
    import nvfp4_block_scaled_16_b200 as nv
    assert nv.nvfp4_get_pdl() is True              # on by default
    nv.nvfp4_set_pdl(False)
    assert nv.nvfp4_get_pdl() is False
    nv.nvfp4_set_pdl(True)
    assert nv.nvfp4_get_pdl() is True


def test_svdquant_input_argument_checks(lib):
    # k % 64, rank in [32, 256] and a multiple of 32, required pointers
    assert lib.nvfp4_lora_down(A16, 128, 96, A16, 64, A16, None) == INVALID
    for r in (0, 16, 48, 288):
        assert lib.nvfp4_lora_down(A16, 128, 128, A16, r, A16, None) == INVALID
    assert lib.nvfp4_lora_down(A16, 128, 128, None, 64, A16, None) == INVALID
    assert lib.nvfp4_lora_down(A16, 0, 128, A16, 64, A16, None) == 0                      # empty
    args = [A16, 128, 128, A16, A16, A16, 64, A16, A16, A16, None]
    for i in (3, 4, 7, 8):                                                                 # pqs, gsf, q, sf
        bad = list(args)
        bad[i] = None
        assert lib.nvfp4_quantize_smooth_lora_down(*bad) == INVALID, i
    assert lib.nvfp4_quantize_smooth(A16, 4, 32, None, A16, A16, A16, None) == INVALID       # pqs required
    assert lib.nvfp4_quantize_smooth(A16, 4, 32, A1, A16, A16, A16, None) == INVALID         # misaligned pqs


def test_global_scale_quantize_argument_checks(lib):
    # (x, m, k, amax, gsf, other_amax, alpha, q, sf, stream)
    assert lib.nvfp4_global_scale_quantize(A16, 4, 24, None, A16, None, None, A16, A16, None) == INVALID   # k % 16
    assert lib.nvfp4_global_scale_quantize(A16, 4, 32, None, None, None, None, A16, A16, None) == INVALID  # gsf
    assert lib.nvfp4_global_scale_quantize(A16, 4, 32, None, A16, A16, None, A16, A16, None) == INVALID    # alpha
    assert lib.nvfp4_global_scale_quantize(A16, 4, 32, None, A16, None, None, None, A16, None) == INVALID  # q
    assert lib.nvfp4_global_scale_quantize(A1, 4, 32, None, A16, None, None, A16, A16, None) == INVALID    # x
    assert lib.nvfp4_selftest_grid_barrier(A16, 4, 24, A16, A16, A16, None) == INVALID


def test_bf16a_argument_checks(lib):
    # (a, b, b_sf, b_amax, bias, out, a_q_ws, a_sf_ws, scalars_ws, m, n, k, stream)
    args = [A16] * 9
    assert lib.nvfp4_gemm_bf16a(*args, 128, 256, 96, None) == INVALID          # k % 64
    assert lib.nvfp4_gemm_bf16a(*args, 128, 100, 256, None) == INVALID         # n % 8
    for i in (0, 1, 2, 3, 5, 6, 7, 8):                                          # required pointers (bias is optional)
        bad = list(args)
        bad[i] = None
        assert lib.nvfp4_gemm_bf16a(*bad, 128, 256, 256, None) == INVALID, i
    for i in (0, 1, 2, 4, 5, 6, 7):                                             # 16-byte alignment
        bad = list(args)
        bad[i] = A1
        assert lib.nvfp4_gemm_bf16a(*bad, 128, 256, 256, None) == INVALID, i


def test_empty_gemms_are_noops(lib):
    # m, n or E == 0 (with valid k): nothing to compute, no pointer read, no device needed
    N7 = [None] * 7
    assert lib.nvfp4_gemm(*N7, 0, 256, 256, None) == 0
    assert lib.nvfp4_gemm(*N7, 128, 0, 256, None) == 0
    assert lib.nvfp4_gemm_lowrank_bias(*N7, 32, None, None, 0, 256, 256, None) == 0
    assert lib.nvfp4_grouped_gemm_masked(*N7, 0, 128, 256, 256, None) == 0
    assert lib.nvfp4_grouped_gemm_masked(*N7, 4, 0, 256, 256, None) == 0
    assert lib.nvfp4_gemm_silu_mul_quantize(*([None] * 11), 0, 256, 256, None) == 0
    # an empty shape is still checked: k must be a positive multiple of 64
    assert lib.nvfp4_gemm(*N7, 0, 256, 96, None) == INVALID


def test_plain_c_client(lib, tmp_path):
    # the C ABI from C99 alone: include/nvfp4.h, link libnvfp4.so, host-only calls
    import subprocess
    from nvfp4_block_scaled_16_b200 import build
    exe = str(tmp_path / "c_abi_check")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe, "-L", build.PKG, "-lnvfp4",
                    "-Wl,-rpath," + build.PKG], check=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stderr
