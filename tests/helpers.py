"""Shared helpers of the GPU parity tests (placement and comparison only)."""
import numpy as np
import torch

# GEMM tolerance: |out - ref| <= 1e-2*|ref| + 1e-3*max|ref|, ref in fp64 from the
# dequantized operands.
GEMM_RTOL = 1e-2
GEMM_ATOL_OF_MAX = 1e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns (host) -> bf16 CUDA tensor."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.atleast_1d(a), dtype=np.float32)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_gemm_close(out: np.ndarray, ref: np.ndarray, what: str = ""):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape
    tol = GEMM_RTOL * np.abs(ref) + GEMM_ATOL_OF_MAX * (np.abs(ref).max() if ref.size else 0.0)
    err = np.abs(out - ref)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first {idx.tolist()}: "
                             f"out={out[tuple(idx[0])]} ref={ref[tuple(idx[0])]}")


def first_diff(a: np.ndarray, b: np.ndarray):
    d = np.argwhere(np.asarray(a) != np.asarray(b))
    return None if d.size == 0 else (d.shape[0], d[:5].tolist())
