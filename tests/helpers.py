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


def sf_logical(sf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Scale codes of rows [0, rows) in logical order [rows, k/16], read from a 128x4-swizzled
    buffer: chunk (r // 128, c // 4) of 512 bytes, byte (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4."""
    sf = np.asarray(sf, np.uint8).reshape(-1)
    groups = -(-(k // 16) // 4)
    r = np.arange(rows)[:, None]
    c = np.arange(k // 16)[None, :]
    off = ((r // 128) * groups + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return sf[off]


def unpack_codes(q: np.ndarray) -> np.ndarray:
    """[..., k/2] packed bytes -> [..., k] e2m1 codes (low nibble first)."""
    q = np.asarray(q, np.uint8)
    return np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[:-1] + (q.shape[-1] * 2,))


E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def assert_nvfp4_close(q, s, q_ref, s_ref, gsf, what="", max_frac=1e-2):
    """NVFP4 outputs of the same h computed along two fp32 accumulation orders: codes and
    scale codes may differ where h crossed a rounding boundary.  Requires at most
    `max_frac` of scales and of codes to differ, and every dequantized value within
    2 * max(scale) / gsf (two e2m1 steps of the larger block scale) plus 1% of the value.
    q [rows, k/2] packed codes; s [rows, k/16] logical scale codes."""
    c, cr = unpack_codes(q), unpack_codes(q_ref)
    s, s_ref = np.asarray(s, np.uint8), np.asarray(s_ref, np.uint8)
    scale_frac = float(np.mean(s != s_ref)) if s.size else 0.0
    code_frac = float(np.mean(c != cr)) if c.size else 0.0
    assert scale_frac <= max_frac, f"{what}: {scale_frac:.2e} of the block scales differ"
    assert code_frac <= max_frac, f"{what}: {code_frac:.2e} of the codes differ"
    sv = np.repeat(e4m3_values(s), 16, axis=-1)
    svr = np.repeat(e4m3_values(s_ref), 16, axis=-1)
    v = E2M1[c] * sv / float(gsf)
    vr = E2M1[cr] * svr / float(gsf)
    bound = 2.0 * np.maximum(sv, svr) / float(gsf) + 1e-2 * np.abs(vr)
    bad = np.abs(v - vr) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} values beyond two e2m1 steps; first {np.argwhere(bad)[:3].tolist()}"
    return scale_frac, code_frac
