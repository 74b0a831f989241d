"""Failure detection on the GPU without a fault: a bounded wait that nothing completes must
give up (about one second), record NVFP4_ERR_DEVICE_TIMEOUT in the device status word,
and leave the context usable; a GEMM whose first K stage is withheld must unwind the same
way, after which the same GEMM runs correctly; a global-scale quantize whose grid barrier
waits for an arrival that never comes must give up, write nothing, and — once the status
is cleared — leave its stream's workspace clean for the next call."""
import numpy as np
import pytest

import nvfp4_block_scaled_16_b200 as nv
import nvfp4_synth as S
from tests.helpers import assert_gemm_close, bf16_to_f64, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu

NVFP4_ERR_DEVICE_TIMEOUT = 4
NVFP4_ERR_INDEX = 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_block_scaled_16_b200 import build
    build.build()
    nv.load_library()
    nv.nvfp4_device_status(clear=True)
    yield
    nv.nvfp4_device_status(clear=True)


def test_bounded_wait_reports_timeout():
    assert nv.nvfp4_device_status(clear=True) == 0
    nv.nvfp4_selftest_bounded_wait()
    assert nv.nvfp4_device_status(clear=True) == NVFP4_ERR_DEVICE_TIMEOUT
    assert nv.nvfp4_device_status(clear=True) == 0            # cleared


def test_gemm_stall_unwinds_and_the_device_stays_usable(oracle):
    m, n, k = 256, 512, 512
    xa = S.normal_bf16((m, k), 1.0, 3, S.TID["x"])
    xb = S.normal_bf16((n, k), 0.02, 3, S.TID["w"])
    amax_a, ga = oracle.global_scale(xa)
    amax_b, gb = oracle.global_scale(xb)
    qa, sfa = oracle.quantize(xa, ga)
    qb, sfb = oracle.quantize(xb, gb)
    alpha = np.float32(oracle.alpha(float(amax_a), float(amax_b)))
    args = (dev_u8(qa), dev_u8(qb), dev_u8(sfa), dev_u8(sfb), dev_f32(alpha))
    assert nv.nvfp4_device_status(clear=True) == 0
    nv.nvfp4_selftest_gemm_stall(*args)
    assert nv.nvfp4_device_status(clear=True) == NVFP4_ERR_DEVICE_TIMEOUT
    out = nv.nvfp4_gemm(*args)                                 # the same GEMM, nothing withheld
    assert nv.nvfp4_device_status(clear=True) == 0
    ref = oracle.gemm_ref(qa, qb, sfa, sfb, alpha, m, n, k)
    assert_gemm_close(bf16_to_f64(out), ref, "gemm after a stalled launch")


def test_grid_barrier_timeout_writes_nothing_and_recovers(oracle):
    x = S.normal_bf16((512, 1024), 4.0, 9, S.TID["x"])
    xd = dev_bf16(x)
    assert nv.nvfp4_device_status(clear=True) == 0
    gsf, q, sf = nv.nvfp4_selftest_grid_barrier(xd)
    assert nv.nvfp4_device_status(clear=True) == NVFP4_ERR_DEVICE_TIMEOUT    # clearing re-zeroes the workspace
    assert host(gsf)[0] == -1.0 and not host(q).any() and not host(sf).any()
    _, gsf_o = oracle.global_scale(x)
    q_o, sf_o = oracle.quantize(x, gsf_o)
    _, g2, _, q2, s2 = nv.nvfp4_global_scale_quantize(xd)
    assert nv.nvfp4_device_status(clear=True) == 0
    assert host(g2)[0] == gsf_o
    assert (host(q2) == q_o).all() and (host(s2) == sf_o).all()


def test_index_check_records_an_error_in_debug_builds_only():
    # One index equal to its extent goes through the check (nothing is accessed): the debug
    # build (NVFP4_LIBRARY=debug) records NVFP4_ERR_INDEX, the release build compiles the
    # check away and records nothing.
    assert nv.nvfp4_device_status(clear=True) == 0
    nv.nvfp4_selftest_index_check()
    want = NVFP4_ERR_INDEX if nv.nvfp4_debug_index_checks() else 0
    assert nv.nvfp4_device_status(clear=True) == want
