"""NumPy front end of the plain-C NVFP4 oracle (``nvfp4_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path (the C-ABI library and its
Python binding) never does, and fails loudly when its CUDA extension is missing.

Every function here only marshals NumPy arrays into the C oracle; the arithmetic is
in ``nvfp4_oracle.c``.  bf16 tensors travel as ``uint16`` bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        sig = {
            "nvo_set_threads": (None, [ctypes.c_int]),
            "nvo_get_threads": (ctypes.c_int, []),
            "nvo_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
            "nvo_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
            "nvo_e2m1_value": (ctypes.c_double, [ctypes.c_uint8]),
            "nvo_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "nvo_e4m3_value": (ctypes.c_double, [ctypes.c_uint8]),
            "nvo_ue4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "nvo_scale_bytes": (_i64, [_i64, _i64]),
            "nvo_sf_offset": (_i64, [_i64, _i64, _i64]),
            "nvo_global_scale": (None, [_u16p, _i64, _f32p, _f32p]),
            "nvo_alpha": (ctypes.c_float, [ctypes.c_float, ctypes.c_float]),
            "nvo_exp_spec": (ctypes.c_float, [ctypes.c_float]),
            "nvo_silu_mul_bf16": (ctypes.c_uint16, [ctypes.c_uint16, ctypes.c_uint16]),
            "nvo_quantize": (None, [_u16p, _i64, _i64, ctypes.c_float, _u8p, _u8p]),
            "nvo_quantize_masked_batched": (None, [_u16p, _i64, _i64, _i64, _i32p, _f32p, _u8p, _u8p]),
            "nvo_silu_mul_quantize_batched": (None, [_u16p, _i64, _i64, _i64, _i32p, _f32p, _u8p, _u8p]),
            "nvo_silu_mul": (None, [_u16p, _i64, _i64, _u16p]),
            "nvo_global_scale_batched": (None, [_u16p, _i64, _i64, _i64, _i32p, ctypes.c_int, _f32p, _f32p]),
            "nvo_dequantize_logical": (None, [_u8p, _u8p, _i64, _i64, _f64p]),
            "nvo_gemm_ref": (None, [_u8p, _u8p, _u8p, _u8p, ctypes.c_float, _u16p, _u16p, _i64, _u16p,
                                    _i64, _i64, _i64, _f64p]),
            "nvo_gemm_ref_sampled": (None, [_u8p, _u8p, _u8p, _u8p, ctypes.c_float, _u16p, _u16p, _i64,
                                            _u16p, _i64, _i64p, _i64p, _i64, _f64p]),
            "nvo_grouped_gemm_ref": (None, [_u8p, _u8p, _u8p, _u8p, _i32p, _f32p, _i64, _i64, _i64, _i64,
                                            _f64p]),
            "nvo_f64_to_bf16": (ctypes.c_uint16, [ctypes.c_double]),
            "nvo_quantize_smooth": (None, [_u16p, _i64, _i64, _u16p, ctypes.c_float, _u8p, _u8p]),
            "nvo_lora_down": (None, [_u16p, _i64, _i64, _u16p, _i64, _f64p]),
            "nvo_gemm_silu_mul_quantize": (None, [_u8p] * 6 + [ctypes.c_float] * 3 + [_i64, _i64, _i64,
                                                                                      _u8p, _u8p]),
            "nvo_grouped_gemm_silu_mul_quantize": (None, [_u8p] * 6 + [_i32p, _f32p, _f32p, _f32p, _i64, _i64,
                                                                       _i64, _i64, _u8p, _u8p]),
            "nvo_gemm_gate_up_bf16": (None, [_u8p] * 6 + [ctypes.c_float] * 2 + [_i64, _i64, _i64p, _i64, _u16p]),
            "nvo_gemm_silu_mul_quantize_rows": (None, [_u8p] * 6 + [ctypes.c_float] * 3 + [_i64, _i64, _i64p,
                                                                                           _i64, _u8p, _u8p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        L.nvo_set_threads(int(os.environ.get("NVFP4_ORACLE_THREADS", os.cpu_count() or 1)))
        _lib = L
    return _lib


def _p(a, t):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(t)


def set_threads(n: int) -> None:
    lib().nvo_set_threads(int(n))


def get_threads() -> int:
    return lib().nvo_get_threads()


# ---- scalar definitions -----------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().nvo_e2m1_value(code)


def e2m1_encode(v: float) -> int:
    return lib().nvo_e2m1_encode(v)


def e4m3_value(code: int) -> float:
    return lib().nvo_e4m3_value(code)


def ue4m3_encode(s: float) -> int:
    return lib().nvo_ue4m3_encode(s)


def exp_spec(x: float) -> float:
    return lib().nvo_exp_spec(x)


def silu_mul_bf16(g_bits: int, u_bits: int) -> int:
    return lib().nvo_silu_mul_bf16(g_bits, u_bits)


def f32_to_bf16(f: float) -> int:
    return lib().nvo_f32_to_bf16(f)


def alpha(amax_a: float, amax_b: float) -> float:
    return lib().nvo_alpha(amax_a, amax_b)


def scale_bytes(rows: int, k: int) -> int:
    return lib().nvo_scale_bytes(rows, k)


def sf_offset(r: int, c: int, k: int) -> int:
    return lib().nvo_sf_offset(r, c, k)


# ---- tensor operations -------------------------------------------------------------

def global_scale(x):
    """amax (clamped) and gsf = 2688/amax of a bf16 tensor given as uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    amax = ctypes.c_float()
    gsf = ctypes.c_float()
    lib().nvo_global_scale(_p(x, _u16p), x.size, ctypes.byref(amax), ctypes.byref(gsf))
    return np.float32(amax.value), np.float32(gsf.value)


def global_scale_batched(x, mask=None, silu_mul=False):
    """Per-item amax/gsf over valid rows of x [b, m, k] (or [b, m, 2k] with silu_mul)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    b, m, w = x.shape
    k = w // 2 if silu_mul else w
    amax = np.zeros(b, np.float32)
    gsf = np.zeros(b, np.float32)
    mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.int32)
    lib().nvo_global_scale_batched(_p(x, _u16p), b, m, k, _p(mk, _i32p), int(bool(silu_mul)),
                                   _p(amax, _f32p), _p(gsf, _f32p))
    return amax, gsf


def quantize(x, gsf, sf_fill=0):
    """Dense quantize of x [m, k] -> (q [m, k/2] uint8, sf [scale_bytes] uint8)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    m, k = x.shape
    q = np.zeros((m, k // 2), np.uint8)
    sf = np.full(scale_bytes(m, k), sf_fill, np.uint8)
    lib().nvo_quantize(_p(x, _u16p), m, k, float(np.float32(gsf)), _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def quantize_masked_batched(x, gsf, mask=None, q_fill=0, sf_fill=0):
    """Masked batched quantize of x [b, m, k] with per-item gsf [b]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    b, m, k = x.shape
    g = np.ascontiguousarray(gsf, dtype=np.float32).reshape(b)
    q = np.full((b, m, k // 2), q_fill, np.uint8)
    sf = np.full((b, scale_bytes(m, k)), sf_fill, np.uint8)
    mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.int32)
    lib().nvo_quantize_masked_batched(_p(x, _u16p), b, m, k, _p(mk, _i32p), _p(g, _f32p),
                                      _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def silu_mul_quantize_batched(x, gsf, mask=None, q_fill=0, sf_fill=0):
    """SiLU-and-mul fused quantize of x [b, m, 2k] with per-item gsf [b]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    b, m, w = x.shape
    k = w // 2
    g = np.ascontiguousarray(gsf, dtype=np.float32).reshape(b)
    q = np.full((b, m, k // 2), q_fill, np.uint8)
    sf = np.full((b, scale_bytes(m, k)), sf_fill, np.uint8)
    mk = None if mask is None else np.ascontiguousarray(mask, dtype=np.int32)
    lib().nvo_silu_mul_quantize_batched(_p(x, _u16p), b, m, k, _p(mk, _i32p), _p(g, _f32p),
                                        _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def silu_mul(x):
    """h = bf16(silu(gate) * up) for x [rows, 2k] -> [rows, k] uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, w = x.reshape(-1, x.shape[-1]).shape
    k = w // 2
    h = np.zeros((rows, k), np.uint16)
    lib().nvo_silu_mul(_p(x, _u16p), rows, k, _p(h, _u16p))
    return h.reshape(x.shape[:-1] + (k,))


def dequantize_logical(q, sf, rows, k):
    """value(code) * value(scale) for every element, fp64 [rows, k] (gsf not applied)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    out = np.zeros((rows, k), np.float64)
    lib().nvo_dequantize_logical(_p(q, _u8p), _p(sf, _u8p), rows, k, _p(out, _f64p))
    return out


def _opt_u16(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.uint16)


def gemm_ref(a, b, a_sf, b_sf, alpha_v, m, n, k, d=None, l1=None, bias=None):
    """fp64 reference alpha*(A.B^T + d.l1^T) + bias on the logical operand values."""
    a, b = np.ascontiguousarray(a, np.uint8), np.ascontiguousarray(b, np.uint8)
    a_sf, b_sf = np.ascontiguousarray(a_sf, np.uint8), np.ascontiguousarray(b_sf, np.uint8)
    d, l1, bias = _opt_u16(d), _opt_u16(l1), _opt_u16(bias)
    r = 0 if d is None else d.shape[-1]
    out = np.zeros((m, n), np.float64)
    lib().nvo_gemm_ref(_p(a, _u8p), _p(b, _u8p), _p(a_sf, _u8p), _p(b_sf, _u8p),
                       float(np.float32(alpha_v)), _p(d, _u16p), _p(l1, _u16p), r, _p(bias, _u16p),
                       m, n, k, _p(out, _f64p))
    return out


def gemm_ref_sampled(a, b, a_sf, b_sf, alpha_v, k, ii, jj, d=None, l1=None, bias=None):
    """The same reference at positions (ii[s], jj[s]) only."""
    a, b = np.ascontiguousarray(a, np.uint8), np.ascontiguousarray(b, np.uint8)
    a_sf, b_sf = np.ascontiguousarray(a_sf, np.uint8), np.ascontiguousarray(b_sf, np.uint8)
    d, l1, bias = _opt_u16(d), _opt_u16(l1), _opt_u16(bias)
    r = 0 if d is None else d.shape[-1]
    ii = np.ascontiguousarray(ii, np.int64)
    jj = np.ascontiguousarray(jj, np.int64)
    out = np.zeros(ii.size, np.float64)
    lib().nvo_gemm_ref_sampled(_p(a, _u8p), _p(b, _u8p), _p(a_sf, _u8p), _p(b_sf, _u8p),
                               float(np.float32(alpha_v)), _p(d, _u16p), _p(l1, _u16p), r,
                               _p(bias, _u16p), k, _p(ii, _i64p), _p(jj, _i64p), ii.size, _p(out, _f64p))
    return out


def grouped_gemm_ref(a, b, a_sf, b_sf, mask, alphas, E, mmax, n, k):
    """Masked grouped reference; rows >= mask[e] of the result are NaN (not computed)."""
    a, b = np.ascontiguousarray(a, np.uint8), np.ascontiguousarray(b, np.uint8)
    a_sf, b_sf = np.ascontiguousarray(a_sf, np.uint8), np.ascontiguousarray(b_sf, np.uint8)
    mk = np.ascontiguousarray(mask, np.int32)
    al = np.ascontiguousarray(alphas, np.float32)
    out = np.full((E, mmax, n), np.nan, np.float64)
    lib().nvo_grouped_gemm_ref(_p(a, _u8p), _p(b, _u8p), _p(a_sf, _u8p), _p(b_sf, _u8p), _p(mk, _i32p),
                               _p(al, _f32p), E, mmax, n, k, _p(out, _f64p))
    return out


def f64_to_bf16(v: float) -> int:
    """bf16 bits nearest to the double v (ties to even)."""
    return int(lib().nvo_f64_to_bf16(float(v)))


def _u8(*arrs):
    return [np.ascontiguousarray(x, np.uint8) for x in arrs]


def gemm_silu_mul_quantize(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, gsf_h, m, n, k,
                           sf_fill=0):
    """Gate/up projections, h = bf16(silu(g) * u), NVFP4 quantization of h with gsf_h.

    Returns (q [m, n/2] uint8, sf [scale_bytes(m, n)] uint8)."""
    a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf = _u8(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf)
    q = np.zeros((m, n // 2), np.uint8)
    sf = np.full(scale_bytes(m, n), sf_fill, np.uint8)
    lib().nvo_gemm_silu_mul_quantize(_p(a, _u8p), _p(b_gate, _u8p), _p(b_up, _u8p), _p(a_sf, _u8p),
                                     _p(b_gate_sf, _u8p), _p(b_up_sf, _u8p), float(np.float32(alpha_gate)),
                                     float(np.float32(alpha_up)), float(np.float32(gsf_h)), m, n, k,
                                     _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def grouped_gemm_silu_mul_quantize(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, mask, alpha_gate, alpha_up, gsf_h,
                                   E, mmax, n, k, q_fill=0, sf_fill=0):
    """Masked grouped form; rows >= mask[e] keep q_fill / sf_fill.

    Returns (q [E, mmax, n/2], sf [E, scale_bytes(mmax, n)])."""
    a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf = _u8(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf)
    mk = np.ascontiguousarray(mask, np.int32)
    ag, au, g = (np.ascontiguousarray(v, np.float32).reshape(E) for v in (alpha_gate, alpha_up, gsf_h))
    q = np.full((E, mmax, n // 2), q_fill, np.uint8)
    sf = np.full((E, scale_bytes(mmax, n)), sf_fill, np.uint8)
    lib().nvo_grouped_gemm_silu_mul_quantize(_p(a, _u8p), _p(b_gate, _u8p), _p(b_up, _u8p), _p(a_sf, _u8p),
                                             _p(b_gate_sf, _u8p), _p(b_up_sf, _u8p), _p(mk, _i32p),
                                             _p(ag, _f32p), _p(au, _f32p), _p(g, _f32p), E, mmax, n, k,
                                             _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def gemm_silu_mul_quantize_rows(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, gsf_h, n, k,
                                rows):
    """The dense result at the listed rows only: (q_rows [len, n/2], scale codes [len, n/16] in
    logical order)."""
    a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf = _u8(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf)
    ii = np.ascontiguousarray(rows, np.int64)
    q = np.zeros((len(ii), n // 2), np.uint8)
    s = np.zeros((len(ii), n // 16), np.uint8)
    lib().nvo_gemm_silu_mul_quantize_rows(_p(a, _u8p), _p(b_gate, _u8p), _p(b_up, _u8p), _p(a_sf, _u8p),
                                          _p(b_gate_sf, _u8p), _p(b_up_sf, _u8p), float(np.float32(alpha_gate)),
                                          float(np.float32(alpha_up)), float(np.float32(gsf_h)), n, k,
                                          _p(ii, _i64p), len(ii), _p(q, _u8p), _p(s, _u8p))
    return q, s


def gemm_gate_up_bf16(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, n, k, rows):
    """[g | u] = [bf16(alpha_gate A.Bg^T) | bf16(alpha_up A.Bu^T)] at the listed rows -> uint16 [len, 2n]."""
    a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf = _u8(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf)
    ii = np.ascontiguousarray(rows, np.int64)
    x = np.zeros((len(ii), 2 * n), np.uint16)
    lib().nvo_gemm_gate_up_bf16(_p(a, _u8p), _p(b_gate, _u8p), _p(b_up, _u8p), _p(a_sf, _u8p),
                                _p(b_gate_sf, _u8p), _p(b_up_sf, _u8p), float(np.float32(alpha_gate)),
                                float(np.float32(alpha_up)), n, k, _p(ii, _i64p), len(ii), _p(x, _u16p))
    return x


def quantize_smooth(x, pqs, gsf, sf_fill=0):
    """Smooth quantize: NVFP4 quantization of x_hat = bf16(x * pqs) -> (q [m, k/2], sf)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    pq = np.ascontiguousarray(pqs, dtype=np.uint16)
    m, k = x.shape
    q = np.zeros((m, k // 2), np.uint8)
    sf = np.full(scale_bytes(m, k), sf_fill, np.uint8)
    lib().nvo_quantize_smooth(_p(x, _u16p), m, k, _p(pq, _u16p), float(np.float32(gsf)), _p(q, _u8p), _p(sf, _u8p))
    return q, sf


def lora_down(x, w):
    """d = x @ w^T in fp64 for bf16 bits x [m, k], w [r, k] -> [m, r]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    m, k = x.shape
    r = w.shape[0]
    out = np.zeros((m, r), np.float64)
    lib().nvo_lora_down(_p(x, _u16p), m, k, _p(w, _u16p), r, _p(out, _f64p))
    return out
