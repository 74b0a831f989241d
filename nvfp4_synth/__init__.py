"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds only random-number recipes and the bf16 rounding of the drawn
values; it contains none of the quantization or GEMM arithmetic, and it imports
neither the oracle nor the CUDA library.

Recipe: a tensor is drawn in chunks of 2^24 values, chunk c from its own stream
``numpy.random.default_rng([seed, tensor_id, c])`` (chunks are generated in parallel
threads); values are drawn in fp32 and rounded to bf16 with round-to-nearest-even; bf16
tensors are returned as ``uint16`` bit patterns.  Small per-tensor draws (masks, l1) use
``default_rng([seed, tensor_id])``.  Seed 0 everywhere unless a caller says otherwise.

Workload shapes (NVFP4 linear-layer inference):
  * pr1_linear      x [128, 256] ~ N(0,1), W [256, 256] ~ N(0, 0.02)
  * quant_dense     x [8192, 8192] ~ N(0,1) with 0.1% of entries (Bernoulli) times 50
  * quant_masked    x [8, 4096, 7168] ~ N(0,1), valid rows per item uniform in [0, 4096]
  * quant_silu      x [8, 4096, 2*7168] ~ N(0,1), the same masks
  * swiglu_block    x [8192, 5120] ~ N(0,1), W_gate_up [16384, 5120], W_down [5120, 8192]
                    ~ N(0, 0.02)
  * grouped_moe     A [16, 2048, 5120] ~ N(0,1), W [16, 8192, 5120] ~ N(0, 0.02), valid
                    rows per expert min(Poisson(512), 2048)
  * lowrank         x [4096, 3072] ~ N(0,1), W [3072, 3072] ~ N(0, 0.02), d [4096, r] ~
                    N(0,1), l1 [3072, r] ~ N(0, 0.01) (divided by alpha by the caller),
                    bias [3072] ~ N(0, 0.1)
"""
import numpy as np

# Tensor ids: one independent stream per tensor of a workload.
TID = {
    "x": 1, "w": 2, "w_gate_up": 3, "w_down": 4, "mask": 5, "d": 6, "l1": 7, "bias": 8,
    "outlier": 9, "sample": 10, "w_gate": 11, "w_up": 12, "pqs": 13, "lora_down": 14,
}


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # uint32 arithmetic: only NaN bit patterns can wrap around, and they are replaced below
    t = (u >> np.uint32(16)) & np.uint32(1)
    t += np.uint32(0x7FFF)
    t += u
    t >>= np.uint32(16)
    r = t.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(u) -> np.ndarray:
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


CHUNK = 1 << 24


def _chunked(shape, fill, items=None):
    """Fill a flat uint16 array chunk by chunk; chunk c gets its own generator.  With
    `items`, only the leading `items` entries of dimension 0 are produced (the same values
    as in the whole tensor)."""
    if items is not None:
        shape = (int(items),) + tuple(shape[1:])
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)
    starts = list(range(0, n, CHUNK))
    if len(starts) <= 1:
        for c, s in enumerate(starts):
            fill(c, out[s:min(n, s + CHUNK)])
    else:
        from concurrent.futures import ThreadPoolExecutor
        import os
        with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(lambda cs: fill(cs[0], out[cs[1]:min(n, cs[1] + CHUNK)]), enumerate(starts)))
    return out.reshape(shape)


def normal_bf16(shape, std=1.0, seed=0, tensor_id=TID["x"], items=None) -> np.ndarray:
    """N(0, std^2) drawn in fp32 and rounded to bf16 (optionally only the leading `items`
    entries of dimension 0)."""
    def fill(c, dst):
        v = np.random.default_rng([int(seed), int(tensor_id), c]).standard_normal(dst.size, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        dst[:] = f32_to_bf16_bits(v)
    return _chunked(shape, fill, items)


def normal_with_outliers_bf16(shape, p=0.001, factor=50.0, seed=0, tensor_id=TID["x"]) -> np.ndarray:
    """N(0,1) with Bernoulli(p) positions multiplied by ``factor`` before bf16 rounding."""
    def fill(c, dst):
        v = np.random.default_rng([int(seed), int(tensor_id), c]).standard_normal(dst.size, dtype=np.float32)
        hit = np.random.default_rng([int(seed), TID["outlier"], c]).random(dst.size, dtype=np.float32) < np.float32(p)
        v[hit] *= np.float32(factor)
        dst[:] = f32_to_bf16_bits(v)
    return _chunked(shape, fill)


def masks_uniform(count, mmax, seed=0, tensor_id=TID["mask"]) -> np.ndarray:
    """Valid rows per item, uniform on the integers 0..mmax (both ends included)."""
    return rng(seed, tensor_id).integers(0, mmax + 1, size=count).astype(np.int32)


def masks_poisson(count, mean, cap, seed=0, tensor_id=TID["mask"]) -> np.ndarray:
    """Valid rows per expert, min(Poisson(mean), cap)."""
    v = rng(seed, tensor_id).poisson(mean, size=count)
    return np.minimum(v, cap).astype(np.int32)


# ---- the workloads -------------------------------------------------------------------

def pr1_linear(seed=0):
    return {"x": normal_bf16((128, 256), 1.0, seed, TID["x"]),
            "w": normal_bf16((256, 256), 0.02, seed, TID["w"])}


def quant_dense(m=8192, k=8192, seed=0):
    return {"x": normal_with_outliers_bf16((m, k), 0.001, 50.0, seed, TID["x"])}


def quant_masked(b=8, m=4096, k=7168, seed=0):
    return {"x": normal_bf16((b, m, k), 1.0, seed, TID["x"]),
            "mask": masks_uniform(b, m, seed)}


def quant_silu(b=8, m=4096, k=7168, seed=0):
    return {"x": normal_bf16((b, m, 2 * k), 1.0, seed, TID["x"]),
            "mask": masks_uniform(b, m, seed)}


def swiglu_block(m=8192, hidden=5120, inter=8192, seed=0):
    return {"x": normal_bf16((m, hidden), 1.0, seed, TID["x"]),
            "w_gate_up": normal_bf16((2 * inter, hidden), 0.02, seed, TID["w_gate_up"]),
            "w_down": normal_bf16((hidden, inter), 0.02, seed, TID["w_down"])}


def grouped_moe(E=16, mmax=2048, k=5120, n=8192, mean=512, seed=0):
    return {"a": normal_bf16((E, mmax, k), 1.0, seed, TID["x"]),
            "w": normal_bf16((E, n, k), 0.02, seed, TID["w"]),
            "mask": masks_poisson(E, mean, mmax, seed)}


def grouped_swiglu(E=16, mmax=2048, hidden=5120, inter=8192, mean=512, seed=0, experts=None):
    """Routed experts: tokens per expert min(Poisson(mean), mmax); per-expert gate, up and
    down weights.  With `experts`, only the leading experts' tensors are produced."""
    return {"x": normal_bf16((E, mmax, hidden), 1.0, seed, TID["x"], experts),
            "w_gate": normal_bf16((E, inter, hidden), 0.02, seed, TID["w_gate"], experts),
            "w_up": normal_bf16((E, inter, hidden), 0.02, seed, TID["w_up"], experts),
            "w_down": normal_bf16((E, hidden, inter), 0.02, seed, TID["w_down"], experts),
            "mask": masks_poisson(E, mean, mmax, seed)}


def svdquant_linear(m=4096, k=3072, n=3072, r=64, seed=0):
    """SVDQuant layer: activations, pre-quantization scale U[0.25, 4] (per input channel),
    the pre-scaled LoRA-down weight [r, k] ~ N(0, 0.05), residual weight ~ N(0, 0.02), LoRA-up
    draws N(0, 0.01) (fp32; the caller divides by alpha and rounds), bias ~ N(0, 0.1)."""
    return {"x": normal_bf16((m, k), 1.0, seed, TID["x"]),
            "pqs": f32_to_bf16_bits(rng(seed, TID["pqs"]).uniform(0.25, 4.0, k).astype(np.float32)),
            "w_down": normal_bf16((r, k), 0.05, seed, TID["lora_down"]),
            "w": normal_bf16((n, k), 0.02, seed, TID["w"]),
            "l1_f32": rng(seed, TID["l1"]).standard_normal((n, r), dtype=np.float32) * np.float32(0.01),
            "bias": normal_bf16((n,), 0.1, seed, TID["bias"])}


def lowrank(m=4096, k=3072, n=3072, r=64, seed=0):
    """l1 is returned as fp32 N(0, 0.01) draws; the caller divides by alpha and rounds."""
    return {"x": normal_bf16((m, k), 1.0, seed, TID["x"]),
            "w": normal_bf16((n, k), 0.02, seed, TID["w"]),
            "d": normal_bf16((m, r), 1.0, seed, TID["d"]),
            "l1_f32": rng(seed, TID["l1"]).standard_normal((n, r), dtype=np.float32) * np.float32(0.01),
            "bias": normal_bf16((n,), 0.1, seed, TID["bias"])}
