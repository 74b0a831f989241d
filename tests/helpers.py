"""Shared helpers of the parity tests (placement, comparison and fixture loading only)."""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

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


def load_worked_example():
    """The hand-worked example of tests/golden/nvfp4_worked_example.txt as arrays.

    Returns a dict: rows, k, row, amax, gsf; x (uint16 bf16 bits [rows, k], zero except
    the worked row) and x_values (that row's values, fp64); codes [k] and dq [k] (fp64)
    of that row; scales [k/16] (codes); q ([rows, k/2] packed bytes, low nibble first) and
    sf ([sf_bytes], the row's scales at sf_offsets, every other byte 0) as the quantizer
    must write them; gemm_self, gemm_ones and their bf16 roundings gemm_self_bf16,
    gemm_ones_bf16; ones_amax, ones_gsf, ones_scale, ones_code of the all-ones operand;
    the variants' inputs silu_gate, mask, pre_quant_scale, lowrank_r, lowrank_l1, bias and
    the low-rank GEMM's outputs lowrank_row (row 33 off the diagonal), lowrank_other; the
    grouped GEMM's grouped_mask, grouped_alpha_mult (alpha[e] = mult/2688) and grouped_row;
    the fused gate/up SiLU-and-mul quantize case (swiglu_*); the LoRA-down case's rank
    lora_r and row 33's input sum row_sum with its bf16 rounding row_sum_bf16."""
    kv = {}
    with open(os.path.join(GOLDEN, "nvfp4_worked_example.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                kv[line[0]] = line[1:]
    rows, k, row = int(kv["rows"][0]), int(kv["k"][0]), int(kv["row"][0])
    nb = k // 16
    xs = np.concatenate([np.array(kv[f"x{j}"], np.float64) for j in range(nb)])
    x32 = torch.from_numpy(xs.astype(np.float32))
    bits = x32.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if not np.array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy(), xs):
        raise ValueError("worked example: an input value is not a bf16 number")
    x = np.zeros((rows, k), np.uint16)
    x[row] = bits
    codes = np.concatenate([np.array([int(c, 16) for c in kv[f"codes{j}"]], np.uint8) for j in range(nb)])
    scales = np.array([int(kv[f"scale{j}"][0], 16) for j in range(nb)], np.uint8)
    q = np.zeros((rows, k // 2), np.uint8)
    q[row] = codes[0::2] | (codes[1::2] << 4)
    sf = np.zeros(int(kv["sf_bytes"][0]), np.uint8)
    sf[np.array(kv["sf_offsets"], np.int64)] = scales
    return {
        "rows": rows, "k": k, "row": row, "amax": float(kv["amax"][0]), "gsf": float(kv["gsf"][0]),
        "x": x, "x_values": xs, "codes": codes, "scales": scales, "q": q, "sf": sf,
        "sf_offsets": np.array(kv["sf_offsets"], np.int64),
        "dq": np.concatenate([np.array(kv[f"dq{j}"], np.float64) for j in range(nb)]),
        "gemm_self": float(kv["gemm_self"][0]), "gemm_ones": float(kv["gemm_ones"][0]),
        "gemm_self_bf16": float(kv["gemm_self_bf16"][0]), "gemm_ones_bf16": float(kv["gemm_ones_bf16"][0]),
        "ones_amax": float(kv["ones_amax"][0]), "ones_gsf": float(kv["ones_gsf"][0]),
        "ones_scale": int(kv["ones_scale"][0], 16), "ones_code": int(kv["ones_code"][0]),
        "silu_gate": float(kv["silu_gate"][0]), "mask": int(kv["mask"][0]),
        "pre_quant_scale": float(kv["pre_quant_scale"][0]), "lowrank_r": int(kv["lowrank_r"][0]),
        "lowrank_l1": float(kv["lowrank_l1"][0]), "bias": float(kv["bias"][0]),
        "lowrank_row": float(kv["lowrank_row"][0]), "lowrank_other": float(kv["lowrank_other"][0]),
        "grouped_mask": [int(v) for v in kv["grouped_mask"]],
        "grouped_alpha_mult": [float(v) for v in kv["grouped_alpha_mult"]],
        "grouped_row": [float(v) for v in kv["grouped_row"]],
        "swiglu_n": int(kv["swiglu_n"][0]), "swiglu_up_div": float(kv["swiglu_up_div"][0]),
        "swiglu_g": float(kv["swiglu_g"][0]), "swiglu_u": float(kv["swiglu_u"][0]),
        "swiglu_h": float(kv["swiglu_h"][0]), "swiglu_byte": int(kv["swiglu_byte"][0], 16),
        "swiglu_scale": int(kv["swiglu_scale"][0], 16), "swiglu_sf_bytes": int(kv["swiglu_sf_bytes"][0]),
        "swiglu_sf_offsets": np.array(kv["swiglu_sf_offsets"], np.int64),
        "swiglu_grouped_mask": [int(v) for v in kv["swiglu_grouped_mask"]],
        "lora_r": int(kv["lora_r"][0]), "row_sum": float(kv["row_sum"][0]),
        "row_sum_bf16": float(kv["row_sum_bf16"][0]),
    }


def bf16_bits(values) -> np.ndarray:
    """fp64 values that are bf16 numbers -> their uint16 bit patterns (raises otherwise)."""
    v = np.asarray(values, np.float64)
    bits = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    if not np.array_equal(back, v):
        raise ValueError("not a bf16 number")
    return bits


def worked_variants(ex):
    """Inputs of the worked example's variants as uint16 bf16 bits: the LoRA-down weight
    [lora_r, k] and its pre_quant_scale-scaled form, the SiLU-and-mul input [1, rows, 2k],
    the smooth-quantize input x/2 and its pre_quant_scale [k], and the low-rank GEMM's
    d [rows, r], l1 [rows, r] and bias [rows]."""
    rows, k, row = ex["rows"], ex["k"], ex["row"]
    xv = np.zeros((rows, k))
    xv[row] = ex["x_values"]
    gu = np.zeros((1, rows, 2 * k))
    gu[0, row, :k] = ex["silu_gate"]
    gu[0, row, k:] = ex["x_values"] / ex["silu_gate"]
    r = ex["lowrank_r"]
    d = np.zeros((rows, r))
    d[row, 0] = 1.0
    l1 = np.zeros((rows, r))
    l1[:, 0] = ex["lowrank_l1"]
    w = np.zeros((ex["lora_r"], k))
    w[0, :] = 1.0
    w[1, 0] = 1.0
    return {
        "lora_w": bf16_bits(w), "lora_w_scaled": bf16_bits(w * ex["pre_quant_scale"]),
        "silu_x": bf16_bits(gu), "smooth_x": bf16_bits(xv / ex["pre_quant_scale"]),
        "pqs": bf16_bits(np.full(k, ex["pre_quant_scale"])), "d": bf16_bits(d), "l1": bf16_bits(l1),
        "bias": bf16_bits(np.full(rows, ex["bias"])),
    }


def masked_expectations(ex, fill):
    """q and sf of the masked variant: the worked bytes on rows below the mask, the
    sentinel on the rest (row r's scales at (r%32)*16 + (r//32)*4 + c for 40 rows, k = 64)."""
    q = np.full_like(ex["q"], fill)
    q[:ex["mask"]] = ex["q"][:ex["mask"]]
    sf = np.full_like(ex["sf"], fill)
    for r in range(ex["mask"]):
        for c in range(ex["k"] // 16):
            sf[(r % 32) * 16 + (r // 32) * 4 + c] = ex["sf"][(r % 32) * 16 + (r // 32) * 4 + c]
    return q, sf


def lowrank_expectation(ex, exact=True):
    rows, row = ex["rows"], ex["row"]
    out = np.full((rows, rows), ex["lowrank_other"])
    out[row, :] = ex["lowrank_row"]
    out[row, row] = (ex["gemm_self"] + ex["lowrank_row"]) if exact else ex["gemm_self_bf16"]
    return out


def grouped_expectation(ex, fill):
    """out [2, rows, 8] of the grouped variant: 0 on rows below each expert's mask, the
    expert's row value on row 33 when the mask covers it, `fill` on unwritten rows."""
    rows, row = ex["rows"], ex["row"]
    out = np.full((2, rows, 8), fill, np.float64)
    for e, m in enumerate(ex["grouped_mask"]):
        out[e, :m] = 0.0
        if row < m:
            out[e, row] = ex["grouped_row"][e]
    return out


def swiglu_expectation(ex):
    """(q [rows, n/2], sf [swiglu_sf_bytes]) of the fused gate/up SiLU-and-mul quantize case."""
    q = np.zeros((ex["rows"], ex["swiglu_n"] // 2), np.uint8)
    q[ex["row"]] = ex["swiglu_byte"]
    sf = np.zeros(ex["swiglu_sf_bytes"], np.uint8)
    sf[ex["swiglu_sf_offsets"]] = ex["swiglu_scale"]
    return q, sf


def swiglu_grouped_expectation(ex, fill):
    """The grouped form [2, ...]: the dense result on rows below each expert's mask, `fill`
    on the rest and on their scale entries (row r, block c at
    (c//4)*512 + (r%32)*16 + (r//32)*4 + c%4 for these 40 rows)."""
    q1, sf1 = swiglu_expectation(ex)
    q = np.full((2,) + q1.shape, fill, np.uint8)
    sf = np.full((2, sf1.size), fill, np.uint8)
    for e, m in enumerate(ex["swiglu_grouped_mask"]):
        q[e, :m] = q1[:m]
        for r in range(m):
            for c in range(ex["swiglu_n"] // 16):
                o = (c // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + c % 4
                sf[e, o] = sf1[o]
    return q, sf


def ones_rows(n, k) -> np.ndarray:
    """bf16 bits of an [n, k] tensor of ones."""
    return np.full((n, k), 0x3F80, np.uint16)


def lora_expectation(ex, value):
    """d [rows, lora_r] of the LoRA-down case with `value` (exact or bf16) at (row, 0)."""
    d = np.zeros((ex["rows"], ex["lora_r"]))
    d[ex["row"], 0] = value
    d[ex["row"], 1] = ex["x_values"][0]
    return d



# ---- full-size coverage and faithful bf16 rounding ------------------------------------------

def tile_positions(m, n, tile_m, tile_n, seed, interior=2):
    """Output positions (ii, jj) covering every tile_m x tile_n tile of an [m, n] output: the
    tile's four corners (clipped to the output, so ragged edge tiles get their last row and
    column) and `interior` seeded random points inside it."""
    g = np.random.default_rng([int(seed), 977])
    ii, jj = [], []
    for r0 in range(0, m, tile_m):
        r1 = min(m, r0 + tile_m) - 1
        for c0 in range(0, n, tile_n):
            c1 = min(n, c0 + tile_n) - 1
            ii += [r0, r0, r1, r1]
            jj += [c0, c1, c0, c1]
            ii += list(g.integers(r0, r1 + 1, interior))
            jj += list(g.integers(c0, c1 + 1, interior))
    return np.array(ii, np.int64), np.array(jj, np.int64)


def bf16_value(bits) -> np.ndarray:
    u = np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _bf16_order(bits) -> np.ndarray:
    """Monotone integer key of bf16 bit patterns (adjacent finite values differ by 1; +0 and
    -0 share the key 0)."""
    b = np.asarray(bits, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def fp32_accumulation_bound(k, alpha, sum_abs):
    """Bound on |alpha * (fp32 sum of k products) - alpha * (exact sum)| for the tensor cores'
    accumulation: one fp32 rounding (relative 2^-24) per 64-wide MMA K-step of the running sum,
    whose magnitude never exceeds the sum of |products|, plus the alpha product, times a
    safety factor of 4."""
    return 4.0 * (k / 64.0 + 2.0) * 2.0 ** -24 * abs(float(alpha)) * np.asarray(sum_abs, np.float64)


def assert_bf16_faithful(got_bits, ref_bits, exact, bound, what=""):
    """bf16 results of a GEMM whose exact value is known: each must be `ref_bits` (the exact
    value rounded to nearest, ties to even) or, where the exact value lies within `bound` of
    the midpoint between `ref_bits` and an adjacent bf16 value, that adjacent value (the fp32
    accumulation landed on the other side of the tie).  Returns (number of such differences,
    largest |exact - midpoint| / bound among them)."""
    got_bits = np.asarray(got_bits, np.uint16).reshape(-1)
    ref_bits = np.asarray(ref_bits, np.uint16).reshape(-1)
    exact = np.asarray(exact, np.float64).reshape(-1)
    bound = np.broadcast_to(np.asarray(bound, np.float64), exact.shape)
    vg, vr = bf16_value(got_bits), bf16_value(ref_bits)
    diff = vg != vr
    if not diff.any():
        return 0, 0.0
    adjacent = np.abs(_bf16_order(got_bits) - _bf16_order(ref_bits)) == 1
    mid = 0.5 * (vg + vr)
    ratio = np.abs(exact - mid) / np.maximum(bound, 1e-300)
    bad = diff & ~(adjacent & (ratio <= 1.0))
    if bad.any():
        i = int(np.argwhere(bad)[0][0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {exact.size} bf16 results are not a faithful rounding; "
                             f"first at {i}: got {vg[i]!r} ref {vr[i]!r} exact {exact[i]!r} bound {bound[i]!r}")
    return int(diff.sum()), float(ratio[diff].max())


def abs_codes(q) -> np.ndarray:
    """Packed e2m1 bytes with both sign bits cleared: the GEMM of these operands (scales are
    unsigned) is the sum of |products|."""
    return (np.asarray(q, np.uint8) & np.uint8(0x77)).astype(np.uint8)


def check_full_size(oracle, out, qa, sfa, qb, sfb, alpha, k, ii, jj, what, d=None, l1=None, bias=None):
    """out (bf16 bits) at (ii, jj) against the oracle: the tolerance, and faithful rounding of
    the exact value (the bias, when given, is added exactly by the epilogue's fma)."""
    ref = oracle.gemm_ref_sampled(qa, qb, sfa, sfb, alpha, k, ii, jj, d=d, l1=l1, bias=bias)
    got_bits = out[ii, jj]
    assert_gemm_close(bf16_value(got_bits), ref, what)
    r = 0 if d is None else d.shape[-1]
    sum_abs = oracle.gemm_ref_sampled(abs_codes(qa), abs_codes(qb), sfa, sfb, alpha, k, ii, jj,
                                      d=None if d is None else d & np.uint16(0x7FFF),
                                      l1=None if l1 is None else l1 & np.uint16(0x7FFF))
    bound = fp32_accumulation_bound(k + 4 * r, 1.0, sum_abs) + (2.0 ** -24 * np.abs(ref) if bias is not None else 0.0)
    stats = assert_bf16_faithful(got_bits, f64_to_bf16_bits(oracle, ref), ref, bound, what)
    print(f"{what}: {len(ii)} outputs, {stats[0]} at the other side of a near tie (worst |exact-tie|/bound "
          f"{stats[1]:.3f})")


# ---- the SiLU * up epilogue against the oracle ---------------------------------------------

def f64_to_bf16_bits(oracle, v):
    return np.array([oracle.f64_to_bf16(float(x)) for x in np.asarray(v).reshape(-1)], np.uint16)


def check_projections_faithful(oracle, ops, gu_lib, ii, jj, n, k, what):
    """g and u of the library at output positions (ii, jj): faithful roundings of the exact
    fp64 projections (nearest, or the other side of a tie within the accumulation bound)."""
    qa, qg, qu, sa, sg, su, al_g, al_u = ops[:8]
    stats = []
    for half, (qb, sb, al) in enumerate(((qg, sg, al_g), (qu, su, al_u))):
        exact = oracle.gemm_ref_sampled(qa, qb, sa, sb, al, k, ii, jj)
        sum_abs = oracle.gemm_ref_sampled(abs_codes(qa), abs_codes(qb), sa, sb, al, k, ii, jj)
        got = gu_lib[ii, half * n + jj]
        stats.append(assert_bf16_faithful(got, f64_to_bf16_bits(oracle, exact), exact,
                                          fp32_accumulation_bound(k, 1.0, sum_abs), f"{what} {'gu'[half]}"))
    print(f"{what}: projections differing from round-to-nearest (count, worst |exact-tie|/bound): {stats}")
    return stats


def check_explained_vs_composition(oracle, ops, gsf, q_rows, s_rows, gu_rows, rows, n, k, what, gu_ref=None):
    """The fused output at `rows` (q_rows [len, n/2], logical scales s_rows [len, n/16]) against the
    oracle's fp64 composition: every 16-value block that differs must hold a g or u value that
    differs from the exact projection rounded to nearest, and every such value must be a
    faithful rounding of the exact value.  `gu_ref`, when given, is the oracle's [g | u] at `rows`
    (oracle.gemm_gate_up_bf16), which is then not recomputed."""
    if gu_ref is None:
        gu_ref = oracle.gemm_gate_up_bf16(*ops[:8], n, k, rows)
    q_ref = np.zeros((len(rows), n // 2), np.uint8)
    s_ref = np.zeros((len(rows), n // 16), np.uint8)
    for i in range(len(rows)):
        qi, sfi = oracle.silu_mul_quantize_batched(gu_ref[i][None, None], np.float32([gsf]))
        q_ref[i] = qi[0, 0]
        s_ref[i] = sf_logical(sfi[0], 1, n)[0]
    diff = gu_rows != gu_ref
    ri, ci = np.nonzero(diff)
    qa, qg, qu, sa, sg, su, al_g, al_u = ops[:8]
    for half, (qb, sb, al) in enumerate(((qg, sg, al_g), (qu, su, al_u))):
        sel = (ci >= n) if half else (ci < n)
        if not sel.any():
            continue
        ii, jj = np.asarray(rows)[ri[sel]], ci[sel] - half * n
        exact = oracle.gemm_ref_sampled(qa, qb, sa, sb, al, k, ii, jj)
        sum_abs = oracle.gemm_ref_sampled(abs_codes(qa), abs_codes(qb), sa, sb, al, k, ii, jj)
        assert_bf16_faithful(gu_rows[ri[sel], ci[sel]], gu_ref[ri[sel], ci[sel]], exact,
                             fp32_accumulation_bound(k, 1.0, sum_abs), f"{what} {'gu'[half]}")
    nb = n // 16
    blk = (unpack_codes(q_rows) != unpack_codes(q_ref)).reshape(len(rows), nb, 16).any(-1) | (s_rows != s_ref)
    explained = diff[:, :n].reshape(len(rows), nb, 16).any(-1) | diff[:, n:].reshape(len(rows), nb, 16).any(-1)
    unexplained = blk & ~explained
    assert not unexplained.any(), f"{what}: blocks differ from the fp64 composition with every g and u exact: " \
                                  f"{np.argwhere(unexplained)[:5].tolist()}"
    print(f"{what}: {int(diff.sum())} of {diff.size} projections and {int(blk.sum())} of {blk.size} blocks differ "
          f"from the fp64 composition, all at near-tie roundings")
