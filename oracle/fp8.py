"""fp64 reference of the fp8 backbone variant (an optional serving precision for W_base).

TEST INFRASTRUCTURE ONLY (see the package docstring): the product never imports this file.

The pages fix no backbone precision beyond serving the backbone shared by every tenant; this
variant stores W_base in 8-bit floating point to halve its bytes (decode) and double the tensor
rate (prefill), with the delta path unchanged.  It is an option next to the bf16 backbone, and its
own oracle is this file.

Format: E4M3 of the OCP 8-bit floating point specification ("OCP 8-bit Floating Point
Specification (OFP8)", revision 1.0, 2023): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits; exponent field 0 holds the subnormals m * 2^-9; no infinities; S.1111.111 is NaN, so the
largest finite magnitude is 448.

Readings (stated where used):
F1  Weights are quantised per output row: s_row = max|w_row| / 448 computed in fp32 (1 if the row
    is zero), code = E4M3 round-to-nearest-even of the fp32 quotient w / s_row, saturating at 448.
F2  Activations are quantised per token the same way with the token's max|x| (fp32 arithmetic).
F3  y = sum_j (code_w * s_row) (code_x * s_tok) + the token's delta, the backbone part exact in
    fp64 from the quantised values.

Parity: the E4M3 rounding is pinned against a brute-force nearest search over the 254 finite
values, ties, subnormals and saturation, and the backbone against the plain product on inputs the
quantisation represents exactly (tests/test_oracle_fp8.py).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code, from the format's definition (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)])


def e4m3_round(x) -> np.ndarray:
    """Codes (uint8) of the nearest E4M3 values to x (float32 input), ties to the even code,
    magnitudes beyond 448 saturated to 448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    pos_codes = np.arange(0, 0x7F)            # 0x00 .. 0x7E: the non-negative finite values
    pos_vals = E4M3_TABLE[pos_codes]           # increasing
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(pos_vals, a, side="left"), 0, len(pos_vals) - 1)
    lo = np.clip(hi - 1, 0, len(pos_vals) - 1)
    dlo = np.abs(a - pos_vals[lo])
    dhi = np.abs(pos_vals[hi] - a)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (pos_codes[hi] % 2 == 0))
    code = np.where(pick_hi, pos_codes[hi], pos_codes[lo]).astype(np.uint8)
    neg = (x < 0) & (code != 0)
    return np.where(neg, code | 0x80, code).astype(np.uint8)


def quantize_rows(w: np.ndarray):
    """F1/F2: per-row scale and codes.  w: float32 [rows, cols].  Returns (codes uint8, scales
    float32)."""
    w = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w), axis=1).astype(np.float32)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(scale == 0, np.float32(1.0), scale).astype(np.float32)
    q = (w / scale[:, None]).astype(np.float32)
    return e4m3_round(q), scale


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.int64)] * np.asarray(scales, dtype=np.float64)[:, None]


def backbone(w_codes: np.ndarray, w_scales: np.ndarray, x: np.ndarray, rows=None) -> np.ndarray:
    """F3: W_hat x_hat for every token (rows of x, float32 values), exact in fp64."""
    xc, xs = quantize_rows(np.asarray(x, dtype=np.float32))
    Xh = dequantize_rows(xc, xs)
    Wh = dequantize_rows(w_codes, w_scales)
    if rows is not None:
        Wh = Wh[np.asarray(rows)]
    return Xh @ Wh.T
