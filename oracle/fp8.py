"""CPU oracle of the fine-grained FP8 quantization of the expert GEMMs.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module.  The GPU path never calls it and shares no code with it.

What it computes
----------------
DeepSeek-V3 technical report summary, section 3.3 "FP8 Training": most GEMMs
run in FP8, with fine-grained scaling to cover FP8's narrow dynamic range,
high-precision accumulation, and power-of-two scaling factors for the
activations.  Appendix B.2 "Discussion About Block-Wise Quantization": in the
forward pass activations are grouped 1 x 128 (one token, 128 consecutive
channels), as opposed to the plain 128 x 128 block-wise grouping, which is the
weights'.  The pages name no FP8 format and give no formula; the readings
taken here:

Q1 format    E4M3 with no infinities ("fn"): 1 sign, 4 exponent bits (bias 7),
             3 mantissa bits; largest finite value 448, smallest normal 2^-6,
             subnormal step 2^-9; codes 0x7F / 0xFF are NaN.
Q2 scale     per group, s = 2^e with e the smallest integer such that
             amax <= 448 * 2^e (amax = largest |value| in the group), clamped
             to [-127, 127] (the range of an 8-bit power-of-two exponent); an
             all-zero group therefore takes e = -127.  The largest element
             then lands in (224, 448].
Q3 rounding  code = E4M3(x / s), round to nearest, ties to the even code, on
             the exact quotient (s is a power of two); the code keeps the sign
             of x, so a negative value that rounds to zero is -0 (0x80).
Q4 groups    activations (the rows entering a GEMM): 1 x 128 along the
             reduction dimension; weights: 128 x 128 blocks of each [out, in]
             matrix; in the backward pass, activations that a weight-gradient
             GEMM contracts over tokens: 128 x 1.  A ragged last group is a
             shorter group.
Q5 value     dequantized = decode(code) * s; the GEMMs accumulate in float64
             here (high-precision accumulation).
Q6 layer     the router stays in high precision (section 3.3 keeps selected
             operations out of FP8); both expert GEMMs take FP8 operands: x
             and the SwiGLU product H are quantized 1 x 128, W_gate, W_up and
             W_down 128 x 128.  The residual is the unquantized input.

Parity pins (``tests/test_oracle_fp8.py``): the code table and the rounding
against torch's own float8_e4m3fn conversion, the scale rule by brute force,
exactness on representable inputs, the error bound of a half step, the group
geometry by perturbation, and the layer against the plain oracle on lossless
inputs.
"""
from __future__ import annotations

import math

import numpy as np

from . import moe_oracle as M

E4M3_MAX = 448.0
GROUP = 128
EXP_MIN, EXP_MAX = -127, 127


def e4m3_decode(codes) -> np.ndarray:
    """Value of each 8-bit E4M3 code (float64; NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    mag = np.where(ex == 0, man * 2.0 ** -9, (1.0 + man / 8.0) * np.exp2(ex - 7.0))
    mag = np.where((ex == 15) & (man == 7), np.nan, mag)
    return sign * mag


# the 127 non-negative finite values, ascending with their codes 0x00..0x7E
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = e4m3_decode(_POS_CODES)


def e4m3_encode(v) -> np.ndarray:
    """Round float64 values with |v| <= 448 to the nearest E4M3 code (ties to even), sign kept."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    if np.any(~np.isfinite(a)) or np.any(a > E4M3_MAX):
        raise ValueError("e4m3_encode: values must be finite and within +-448")
    hi = np.clip(np.searchsorted(_POS_VALUES, a, side="left"), 0, 126)  # first table value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(np.signbit(v), code | 0x80, code)
    return code.astype(np.uint8)


def scale_exponent(amax) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-127, 127] (reading Q2)."""
    a = np.asarray(amax, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.int64)
    for i, x in np.ndenumerate(a):
        if x == 0.0:
            e = EXP_MIN
        else:
            m, ex = math.frexp(x / E4M3_MAX)    # x / 448 = m * 2^ex, m in [0.5, 1)
            e = ex - 1 if m == 0.5 else ex      # ceil(log2(x / 448))
        out[i] = min(max(e, EXP_MIN), EXP_MAX)
    return out


def quantize_groups(a, group_rows: int, group_cols: int):
    """Quantize a 2-D array in [group_rows x group_cols] groups -> (codes uint8, exponents int64).

    exponents[i, j] is the scale exponent of the group of rows
    [i*group_rows, ...) and columns [j*group_cols, ...).
    """
    x = M.f64(a)
    R, C = x.shape
    gr, gc = -(-R // group_rows), -(-C // group_cols)
    codes = np.empty((R, C), dtype=np.uint8)
    exps = np.empty((gr, gc), dtype=np.int64)
    for i in range(gr):
        for j in range(gc):
            blk = x[i * group_rows:(i + 1) * group_rows, j * group_cols:(j + 1) * group_cols]
            e = int(scale_exponent(np.abs(blk).max() if blk.size else 0.0))
            exps[i, j] = e
            codes[i * group_rows:(i + 1) * group_rows, j * group_cols:(j + 1) * group_cols] = \
                e4m3_encode(blk * 2.0 ** -e)
    return codes, exps


def dequantize_groups(codes, exps, group_rows: int, group_cols: int) -> np.ndarray:
    """decode(code) * 2^e of each element's group."""
    v = e4m3_decode(codes)
    s = np.repeat(np.repeat(np.exp2(np.asarray(exps, dtype=np.float64)), group_rows, axis=0),
                  group_cols, axis=1)
    return v * s[:v.shape[0], :v.shape[1]]


def quantize_rows(x):
    """Activations: 1 x 128 groups along the last dimension (reading Q4)."""
    return quantize_groups(x, 1, GROUP)


def quantize_cols(x):
    """Activations in the backward pass, where the weight-gradient GEMM contracts over tokens:
    128 x 1 groups (128 consecutive rows of one column; Appendix B.2)."""
    return quantize_groups(x, GROUP, 1)


def quantize_blocks(w):
    """A weight matrix [out, in] (or a stack [n, out, in]): 128 x 128 blocks (reading Q4)."""
    w = M.f64(w)
    if w.ndim == 2:
        return quantize_groups(w, GROUP, GROUP)
    pairs = [quantize_groups(m, GROUP, GROUP) for m in w]
    return np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs])


def qdq_rows(x) -> np.ndarray:
    return dequantize_groups(*quantize_rows(x), 1, GROUP)


def qdq_blocks(w) -> np.ndarray:
    w = M.f64(w)
    if w.ndim == 2:
        return dequantize_groups(*quantize_groups(w, GROUP, GROUP), GROUP, GROUP)
    return np.stack([qdq_blocks(m) for m in w])


def swiglu_ffn_fp8(u, w_gate, w_up, w_down) -> np.ndarray:
    """FFN(u) with FP8 operands (reading Q6): both GEMMs see quantized-dequantized inputs."""
    uq = qdq_rows(u)
    a = uq @ qdq_blocks(w_gate).T
    b = uq @ qdq_blocks(w_up).T
    hq = qdq_rows(M.silu(a) * b)
    return hq @ qdq_blocks(w_down).T


def moe_forward_fp8(u, router_w, K: int, experts, shared=None, **kw):
    """The layer of ``moe_oracle.moe_forward`` with FP8 expert GEMMs (routing in high precision)."""
    return M.moe_forward(u, router_w, K, experts, shared, ffn=swiglu_ffn_fp8, **kw)
