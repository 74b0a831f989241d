"""ctypes binding of libnvfp4.so (argument marshalling only).

Every function takes PyTorch CUDA tensors (or None for nullable arguments), passes their
device pointers and the current stream to the C entry point of the same name, and raises
:class:`NVFP4Error` on a non-zero status.  Outputs the caller does not provide are
allocated with ``torch.empty`` on the input's device.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

EXPORTED_SYMBOLS = (
    "nvfp4_status_string",
    "nvfp4_scale_bytes",
    "nvfp4_global_scale",
    "nvfp4_global_scale_batched",
    "nvfp4_global_scale_batched_noalloc",
    "nvfp4_quantize",
    "nvfp4_global_scale_quantize",
    "nvfp4_quantize_masked_batched",
    "nvfp4_silu_mul_quantize_batched",
    "nvfp4_gemm",
    "nvfp4_gemm_bf16a",
    "nvfp4_gemm_bf16a_static",
    "nvfp4_grouped_gemm_masked",
    "nvfp4_gemm_lowrank_bias",
    "nvfp4_gemm_silu_mul_quantize",
    "nvfp4_grouped_gemm_silu_mul_quantize_masked",
    "nvfp4_silu_and_mul",
    "nvfp4_quantize_smooth",
    "nvfp4_lora_down",
    "nvfp4_quantize_smooth_lora_down",
    "nvfp4_set_pdl",
    "nvfp4_get_pdl",
    "nvfp4_selftest_bounded_wait",
    "nvfp4_selftest_gemm_stall",
    "nvfp4_selftest_grid_barrier",
    "nvfp4_debug_index_checks",
    "nvfp4_selftest_index_check",
    "nvfp4_device_status",
)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

_SIGNATURES = {
    "nvfp4_status_string": (ctypes.c_char_p, [_INT]),
    "nvfp4_scale_bytes": (_I64, [_I64, _I64]),
    "nvfp4_global_scale": (_INT, [_P, _I64, _P, _P, _P, _P, _P]),
    "nvfp4_global_scale_batched": (_INT, [_P, _I64, _I64, _I64, _P, _INT, _P, _P, _P]),
    "nvfp4_global_scale_batched_noalloc": (_INT, [_P, _I64, _I64, _I64, _P, _INT, _P, _P, _P]),
    "nvfp4_quantize": (_INT, [_P, _I64, _I64, _P, _P, _P, _P]),
    "nvfp4_global_scale_quantize": (_INT, [_P, _I64, _I64, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_quantize_masked_batched": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "nvfp4_silu_mul_quantize_batched": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "nvfp4_gemm": (_INT, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "nvfp4_gemm_bf16a": (_INT, [_P] * 9 + [_I64, _I64, _I64, _P]),
    "nvfp4_gemm_bf16a_static": (_INT, [_P] * 9 + [_I64, _I64, _I64, _INT, _P]),
    "nvfp4_grouped_gemm_masked": (_INT, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]),
    "nvfp4_gemm_lowrank_bias": (_INT, [_P, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _I64, _I64, _I64, _P]),
    "nvfp4_gemm_silu_mul_quantize": (_INT, [_P] * 11 + [_I64, _I64, _I64, _P]),
    "nvfp4_grouped_gemm_silu_mul_quantize_masked": (_INT, [_P] * 12 + [_I64, _I64, _I64, _I64, _P]),
    "nvfp4_silu_and_mul": (_INT, [_P, _I64, _I64, _P, _P]),
    "nvfp4_quantize_smooth": (_INT, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "nvfp4_lora_down": (_INT, [_P, _I64, _I64, _P, _I64, _P, _P]),
    "nvfp4_quantize_smooth_lora_down": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _P]),
    "nvfp4_set_pdl": (_INT, [_INT]),
    "nvfp4_get_pdl": (_INT, []),
    "nvfp4_selftest_bounded_wait": (_INT, [_P]),
    "nvfp4_selftest_gemm_stall": (_INT, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "nvfp4_selftest_grid_barrier": (_INT, [_P, _I64, _I64, _P, _P, _P, _P]),
    "nvfp4_debug_index_checks": (_INT, []),
    "nvfp4_selftest_index_check": (_INT, [_P]),
    "nvfp4_device_status": (_INT, [ctypes.POINTER(_INT), _INT]),
}


class NVFP4Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {nvfp4_status_string(status)} ({status})")


def library_path() -> str:
    """libnvfp4.so, or with NVFP4_LIBRARY=debug the index-checking libnvfp4_debug.so."""
    name = "libnvfp4_debug.so" if os.environ.get("NVFP4_LIBRARY") == "debug" else "libnvfp4.so"
    return os.path.join(_HERE, name)


def load_library():
    """Load libnvfp4.so (built in-tree by ``python -m nvfp4_block_scaled_16_b200.build``)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with `python -m nvfp4_block_scaled_16_b200.build`"
                              + (" --debug" if path.endswith("_debug.so") else ""))
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a torch.Tensor, got {type(t)}")
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise NVFP4Error(fn, status)


def _device_of(*ts):
    for t in ts:
        if isinstance(t, torch.Tensor):
            return t.device
    return torch.device("cuda", torch.cuda.current_device())


def nvfp4_status_string(status: int) -> str:
    return load_library().nvfp4_status_string(int(status)).decode()


def nvfp4_scale_bytes(rows: int, k: int) -> int:
    return int(load_library().nvfp4_scale_bytes(int(rows), int(k)))


def nvfp4_global_scale(x, amax_out=None, gsf_out=None, other_amax=None, alpha_out=None, stream=None):
    """amax/gsf (and alpha when ``other_amax`` is given) of a bf16 tensor; fp32 [1] outputs."""
    dev = x.device
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    gsf_out = torch.empty(1, dtype=torch.float32, device=dev) if gsf_out is None else gsf_out
    if other_amax is not None and alpha_out is None:
        alpha_out = torch.empty(1, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = load_library().nvfp4_global_scale(_ptr(x), x.numel(), _ptr(amax_out), _ptr(gsf_out),
                                               _ptr(other_amax), _ptr(alpha_out), _stream(stream))
    _check("nvfp4_global_scale", st)
    return amax_out, gsf_out, alpha_out


def nvfp4_global_scale_batched(x, mask=None, silu_mul=False, amax_out=None, gsf_out=None, stream=None):
    """Per-item amax/gsf over valid rows of x [b, m, k] (or [b, m, 2k] with silu_mul)."""
    b, m, w = x.shape
    k = w // 2 if silu_mul else w
    amax_out = torch.empty(b, dtype=torch.float32, device=x.device) if amax_out is None else amax_out
    gsf_out = torch.empty(b, dtype=torch.float32, device=x.device) if gsf_out is None else gsf_out
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_global_scale_batched(_ptr(x), b, m, k, _ptr(mask), int(bool(silu_mul)),
                                                       _ptr(amax_out), _ptr(gsf_out), _stream(stream))
    _check("nvfp4_global_scale_batched", st)
    return amax_out, gsf_out


def nvfp4_global_scale_batched_noalloc(x, mask, silu_mul, amax_out, gsf_out, stream=None):
    """nvfp4_global_scale_batched with library-internal fixed scratch: nothing is allocated,
    so the outputs must be passed in (fp32 [b] each; amax_out may be None)."""
    b, m, w = x.shape
    k = w // 2 if silu_mul else w
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_global_scale_batched_noalloc(_ptr(x), b, m, k, _ptr(mask), int(bool(silu_mul)),
                                                               _ptr(amax_out), _ptr(gsf_out), _stream(stream))
    _check("nvfp4_global_scale_batched_noalloc", st)
    return amax_out, gsf_out


def nvfp4_quantize(x, gsf, q_out=None, sf_out=None, stream=None):
    """x [m, k] bf16 -> (q [m, k/2] uint8, sf [scale_bytes(m, k)] uint8)."""
    m, k = x.shape
    q_out = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device) if q_out is None else q_out
    if sf_out is None:
        sf_out = torch.empty(max(nvfp4_scale_bytes(m, k), 0), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_quantize(_ptr(x), m, k, _ptr(gsf), _ptr(q_out), _ptr(sf_out), _stream(stream))
    _check("nvfp4_quantize", st)
    return q_out, sf_out


def nvfp4_global_scale_quantize(x, other_amax=None, amax_out=None, gsf_out=None, alpha_out=None, q_out=None,
                                sf_out=None, stream=None):
    """x [m, k] bf16 -> (amax [1], gsf [1], alpha [1] or None, q [m, k/2] uint8, sf [scale_bytes(m, k)] uint8):
    nvfp4_global_scale and nvfp4_quantize in one launch."""
    m, k = x.shape
    dev = x.device
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    gsf_out = torch.empty(1, dtype=torch.float32, device=dev) if gsf_out is None else gsf_out
    if other_amax is not None and alpha_out is None:
        alpha_out = torch.empty(1, dtype=torch.float32, device=dev)
    q_out = torch.empty((m, k // 2), dtype=torch.uint8, device=dev) if q_out is None else q_out
    if sf_out is None:
        sf_out = torch.empty(max(nvfp4_scale_bytes(m, k), 0), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = load_library().nvfp4_global_scale_quantize(_ptr(x), m, k, _ptr(amax_out), _ptr(gsf_out),
                                                        _ptr(other_amax), _ptr(alpha_out), _ptr(q_out),
                                                        _ptr(sf_out), _stream(stream))
    _check("nvfp4_global_scale_quantize", st)
    return amax_out, gsf_out, alpha_out, q_out, sf_out


def _batched_outputs(x, b, m, k, q_out, sf_out):
    q_out = torch.empty((b, m, k // 2), dtype=torch.uint8, device=x.device) if q_out is None else q_out
    if sf_out is None:
        sf_out = torch.empty((b, max(nvfp4_scale_bytes(m, k), 0)), dtype=torch.uint8, device=x.device)
    return q_out, sf_out


def nvfp4_quantize_masked_batched(x, gsf, mask=None, q_out=None, sf_out=None, stream=None):
    """x [b, m, k] bf16, gsf [b], mask [b] int32 or None -> (q [b, m, k/2], sf [b, scale_bytes(m, k)])."""
    b, m, k = x.shape
    q_out, sf_out = _batched_outputs(x, b, m, k, q_out, sf_out)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_quantize_masked_batched(_ptr(x), b, m, k, _ptr(mask), _ptr(gsf), _ptr(q_out),
                                                          _ptr(sf_out), _stream(stream))
    _check("nvfp4_quantize_masked_batched", st)
    return q_out, sf_out


def nvfp4_silu_mul_quantize_batched(x, gsf, mask=None, q_out=None, sf_out=None, stream=None):
    """x [b, m, 2k] bf16 (gate | up) -> quantized h = bf16(silu(gate) * up): (q [b, m, k/2], sf)."""
    b, m, w = x.shape
    k = w // 2
    q_out, sf_out = _batched_outputs(x, b, m, k, q_out, sf_out)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_silu_mul_quantize_batched(_ptr(x), b, m, k, _ptr(mask), _ptr(gsf), _ptr(q_out),
                                                            _ptr(sf_out), _stream(stream))
    _check("nvfp4_silu_mul_quantize_batched", st)
    return q_out, sf_out


def nvfp4_gemm(a, b, a_sf, b_sf, alpha, bias=None, out=None, stream=None):
    """a [m, k/2], b [n, k/2] packed e2m1 -> out [m, n] bf16 = alpha * a @ b^T (+ bias)."""
    m, kh = a.shape
    n = b.shape[0]
    out = torch.empty((m, n), dtype=torch.bfloat16, device=a.device) if out is None else out
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_gemm(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(alpha), _ptr(bias), _ptr(out),
                                       m, n, 2 * kh, _stream(stream))
    _check("nvfp4_gemm", st)
    return out


def nvfp4_gemm_bf16a(a, b, b_sf, b_amax, bias=None, out=None, a_q_ws=None, a_sf_ws=None, scalars_ws=None,
                     stream=None):
    """bf16 activation a [m, k] x NVFP4 weight b [n, k/2] -> (out [m, n] bf16, a_q [m, k/2], a_sf, scalars [3]):
    the activation's dynamic global scale and quantization, then the FP4 GEMM."""
    m, k = a.shape
    n = b.shape[0]
    dev = a.device
    out = torch.empty((m, n), dtype=torch.bfloat16, device=dev) if out is None else out
    a_q_ws = torch.empty((m, k // 2), dtype=torch.uint8, device=dev) if a_q_ws is None else a_q_ws
    if a_sf_ws is None:
        a_sf_ws = torch.empty(max(nvfp4_scale_bytes(m, k), 0), dtype=torch.uint8, device=dev)
    scalars_ws = torch.empty(3, dtype=torch.float32, device=dev) if scalars_ws is None else scalars_ws
    with torch.cuda.device(dev):
        st = load_library().nvfp4_gemm_bf16a(_ptr(a), _ptr(b), _ptr(b_sf), _ptr(b_amax), _ptr(bias), _ptr(out),
                                             _ptr(a_q_ws), _ptr(a_sf_ws), _ptr(scalars_ws), m, n, k, _stream(stream))
    _check("nvfp4_gemm_bf16a", st)
    return out, a_q_ws, a_sf_ws, scalars_ws


def nvfp4_gemm_bf16a_static(a, b, b_sf, a_gsf, alpha, bias=None, out=None, a_q_ws=None, a_sf_ws=None, one_launch=False,
                            stream=None):
    """bf16 activation a [m, k] x NVFP4 weight b [n, k/2] with a static activation scale a_gsf [1]
    -> (out [m, n] bf16, a_q [m, k/2], a_sf); one_launch picks the fused single-kernel form."""
    m, k = a.shape
    n = b.shape[0]
    dev = a.device
    out = torch.empty((m, n), dtype=torch.bfloat16, device=dev) if out is None else out
    a_q_ws = torch.empty((m, k // 2), dtype=torch.uint8, device=dev) if a_q_ws is None else a_q_ws
    if a_sf_ws is None:
        a_sf_ws = torch.empty(max(nvfp4_scale_bytes(m, k), 0), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = load_library().nvfp4_gemm_bf16a_static(_ptr(a), _ptr(b), _ptr(b_sf), _ptr(a_gsf), _ptr(alpha), _ptr(bias),
                                                    _ptr(out), _ptr(a_q_ws), _ptr(a_sf_ws), m, n, k, int(one_launch),
                                                    _stream(stream))
    _check("nvfp4_gemm_bf16a_static", st)
    return out, a_q_ws, a_sf_ws


def nvfp4_grouped_gemm_masked(a, b, a_sf, b_sf, mask, alpha, out=None, stream=None):
    """a [E, mmax, k/2], b [E, n, k/2] -> out [E, mmax, n] bf16 (rows >= mask[e] not written)."""
    E, mmax, kh = a.shape
    n = b.shape[1]
    out = torch.empty((E, mmax, n), dtype=torch.bfloat16, device=a.device) if out is None else out
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_grouped_gemm_masked(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(mask),
                                                      _ptr(alpha), _ptr(out), E, mmax, n, 2 * kh, _stream(stream))
    _check("nvfp4_grouped_gemm_masked", st)
    return out


def nvfp4_gemm_lowrank_bias(a, b, a_sf, b_sf, alpha, d, l1, bias=None, out=None, stream=None):
    """out [m, n] bf16 = alpha * (a @ b^T + d @ l1^T) (+ bias); d [m, r], l1 [n, r] bf16."""
    m, kh = a.shape
    n = b.shape[0]
    r = d.shape[1]
    out = torch.empty((m, n), dtype=torch.bfloat16, device=a.device) if out is None else out
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_gemm_lowrank_bias(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(alpha), _ptr(d),
                                                    _ptr(l1), r, _ptr(bias), _ptr(out), m, n, 2 * kh,
                                                    _stream(stream))
    _check("nvfp4_gemm_lowrank_bias", st)
    return out


def nvfp4_gemm_silu_mul_quantize(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, gsf_h,
                                 q_out=None, sf_out=None, stream=None):
    """h = bf16(silu(bf16(alpha_gate * a @ b_gate^T)) * bf16(alpha_up * a @ b_up^T)) quantized with gsf_h.

    a [m, k/2], b_gate / b_up [n, k/2] -> (q_out [m, n/2] uint8, sf_out [nvfp4_scale_bytes(m, n)] uint8).
    """
    m, kh = a.shape
    n = b_gate.shape[0]
    if q_out is None:
        q_out = torch.empty((m, n // 2), dtype=torch.uint8, device=a.device)
    if sf_out is None:
        sf_out = torch.empty((nvfp4_scale_bytes(m, n),), dtype=torch.uint8, device=a.device)
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_gemm_silu_mul_quantize(
            _ptr(a), _ptr(b_gate), _ptr(b_up), _ptr(a_sf), _ptr(b_gate_sf), _ptr(b_up_sf), _ptr(alpha_gate),
            _ptr(alpha_up), _ptr(gsf_h), _ptr(q_out), _ptr(sf_out), m, n, 2 * kh, _stream(stream))
    _check("nvfp4_gemm_silu_mul_quantize", st)
    return q_out, sf_out


def nvfp4_grouped_gemm_silu_mul_quantize_masked(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, mask, alpha_gate,
                                                alpha_up, gsf_h, q_out=None, sf_out=None, stream=None):
    """Per expert e, rows < mask[e]: nvfp4_gemm_silu_mul_quantize of a[e] with b_gate[e], b_up[e].

    a [E, mmax, k/2], b_gate / b_up [E, n, k/2] -> (q_out [E, mmax, n/2], sf_out [E, nvfp4_scale_bytes(mmax, n)]).
    """
    E, mmax, kh = a.shape
    n = b_gate.shape[1]
    if q_out is None:
        q_out = torch.empty((E, mmax, n // 2), dtype=torch.uint8, device=a.device)
    if sf_out is None:
        sf_out = torch.empty((E, nvfp4_scale_bytes(mmax, n)), dtype=torch.uint8, device=a.device)
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_grouped_gemm_silu_mul_quantize_masked(
            _ptr(a), _ptr(b_gate), _ptr(b_up), _ptr(a_sf), _ptr(b_gate_sf), _ptr(b_up_sf), _ptr(mask),
            _ptr(alpha_gate), _ptr(alpha_up), _ptr(gsf_h), _ptr(q_out), _ptr(sf_out), E, mmax, n, 2 * kh,
            _stream(stream))
    _check("nvfp4_grouped_gemm_silu_mul_quantize_masked", st)
    return q_out, sf_out


def nvfp4_silu_and_mul(x, h_out=None, stream=None):
    """x [rows, 2k] bf16 (gate | up) -> h [rows, k] bf16 = bf16(silu(gate) * up)."""
    rows, w = x.shape
    k = w // 2
    if h_out is None:
        h_out = torch.empty((rows, k), dtype=torch.bfloat16, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_silu_and_mul(_ptr(x), rows, k, _ptr(h_out), _stream(stream))
    _check("nvfp4_silu_and_mul", st)
    return h_out


def nvfp4_quantize_smooth(x, pre_quant_scale, gsf, q_out=None, sf_out=None, stream=None):
    """x [m, k] bf16, pre_quant_scale [k] bf16 -> NVFP4 of bf16(x * pre_quant_scale): (q [m, k/2], sf)."""
    m, k = x.shape
    if q_out is None:
        q_out = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device)
    if sf_out is None:
        sf_out = torch.empty((nvfp4_scale_bytes(m, k),), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_quantize_smooth(_ptr(x), m, k, _ptr(pre_quant_scale), _ptr(gsf), _ptr(q_out),
                                                  _ptr(sf_out), _stream(stream))
    _check("nvfp4_quantize_smooth", st)
    return q_out, sf_out


def nvfp4_lora_down(x, w, d_out=None, stream=None):
    """d [m, r] bf16 = x [m, k] @ w [r, k]^T (w: the pre-quantization-scaled LoRA-down weight)."""
    m, k = x.shape
    r = w.shape[0]
    if d_out is None:
        d_out = torch.empty((m, r), dtype=torch.bfloat16, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_lora_down(_ptr(x), m, k, _ptr(w), r, _ptr(d_out), _stream(stream))
    _check("nvfp4_lora_down", st)
    return d_out


def nvfp4_quantize_smooth_lora_down(x, pre_quant_scale, gsf, w, q_out=None, sf_out=None, d_out=None, stream=None):
    """Both in one pass over x: (q [m, k/2], sf, d [m, r])."""
    m, k = x.shape
    r = w.shape[0]
    if q_out is None:
        q_out = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device)
    if sf_out is None:
        sf_out = torch.empty((nvfp4_scale_bytes(m, k),), dtype=torch.uint8, device=x.device)
    if d_out is None:
        d_out = torch.empty((m, r), dtype=torch.bfloat16, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_quantize_smooth_lora_down(_ptr(x), m, k, _ptr(pre_quant_scale), _ptr(gsf),
                                                            _ptr(w), r, _ptr(q_out), _ptr(sf_out), _ptr(d_out),
                                                            _stream(stream))
    _check("nvfp4_quantize_smooth_lora_down", st)
    return q_out, sf_out, d_out


def nvfp4_set_pdl(enable: bool) -> None:
    """Launch subsequent kernels with (True) or without programmatic dependent launch."""
    _check("nvfp4_set_pdl", load_library().nvfp4_set_pdl(1 if enable else 0))


def nvfp4_get_pdl() -> bool:
    return bool(load_library().nvfp4_get_pdl())


def nvfp4_selftest_bounded_wait(stream=None):
    """Launch a wait that nothing completes; its bounded wait records NVFP4_ERR_DEVICE_TIMEOUT."""
    with torch.cuda.device(torch.cuda.current_device()):
        _check("nvfp4_selftest_bounded_wait", load_library().nvfp4_selftest_bounded_wait(_stream(stream)))


def nvfp4_selftest_gemm_stall(a, b, a_sf, b_sf, alpha, out=None, stream=None):
    """nvfp4_gemm with the first K stage's loads withheld: the MMA wait runs out and the kernel unwinds."""
    m, kh = a.shape
    n = b.shape[0]
    out = torch.empty((m, n), dtype=torch.bfloat16, device=a.device) if out is None else out
    with torch.cuda.device(a.device):
        st = load_library().nvfp4_selftest_gemm_stall(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(alpha),
                                                      _ptr(out), m, n, 2 * kh, _stream(stream))
    _check("nvfp4_selftest_gemm_stall", st)
    return out


def nvfp4_selftest_grid_barrier(x, stream=None):
    """nvfp4_global_scale_quantize whose grid barrier waits for one arrival too many: every
    CTA's wait runs out, NVFP4_ERR_DEVICE_TIMEOUT is recorded and nothing is written."""
    m, k = x.shape
    gsf = torch.full((1,), -1.0, dtype=torch.float32, device=x.device)
    q = torch.zeros((m, k // 2), dtype=torch.uint8, device=x.device)
    sf = torch.zeros(max(nvfp4_scale_bytes(m, k), 0), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        st = load_library().nvfp4_selftest_grid_barrier(_ptr(x), m, k, _ptr(gsf), _ptr(q), _ptr(sf), _stream(stream))
    _check("nvfp4_selftest_grid_barrier", st)
    return gsf, q, sf


def nvfp4_debug_index_checks() -> bool:
    """Whether the loaded library checks kernel indices (the debug build)."""
    return bool(load_library().nvfp4_debug_index_checks())


def nvfp4_selftest_index_check(stream=None):
    """Submit one out-of-range index to the debug-build check (nothing is accessed)."""
    _check("nvfp4_selftest_index_check", load_library().nvfp4_selftest_index_check(_stream(stream)))


def nvfp4_device_status(clear: bool = True) -> int:
    """Synchronize the device and return (optionally clearing) its status word."""
    v = _INT(0)
    st = load_library().nvfp4_device_status(ctypes.byref(v), int(bool(clear)))
    _check("nvfp4_device_status", st)
    return v.value
