"""Plain CPU definition of the FP8 (E4M3) variant of the prefill linear layer.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): imported by the
tests and the CPU legs of the benchmark, never by the library.  It shares no
code, table or constant with the CUDA path.

Source: DynaQuant (zingnex forum thread), "Custom kernel architecture": for
5-7-bit codes the packed data is expanded to FP8 E4M3 and fed to FP8 tensor
cores.  E4M3 holds every integer of magnitude up to 16 exactly (3 mantissa
bits) and 17 no longer, so codes of b <= 5 bits (|q| <= 15) are exact and
this variant is defined for b <= 5 only; 6- and 7-bit codes would be rounded.

An FP8 tensor-core product needs both operands in FP8, so the activations are
quantized too.  The pages do not say how; the reading taken here is the
symmetric per-channel formula of the quantization tutorial ("How
quantization works") applied to each token of x, with E4M3's largest finite
value in place of max_int:

* sx_m = fl32(max_k |x_mk| / 448), an IEEE fp32 division; a zero token takes
  fl32(1 / 448);
* xq_mk = E4M3_rn(fl32(x_mk / sx_m)): the fp32 quotient rounded to the
  nearest E4M3 value, ties to the even mantissa, saturating at +-448;
* y_mn = bf16(s_n * sx_m * sum_k xq_mk * q_nk), accumulated in fp32.

E4M3 (the OCP 8-bit format): sign, 4 exponent bits with bias 7, 3 mantissa
bits; exponent field 0 encodes subnormals m * 2^-9; no infinities; the
largest finite magnitude is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import numpy as np

from .quant import QLINEAR_ABS_TOL, QLINEAR_REL_TOL

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6      # smallest normal value 2^-6
E4M3_MANT_BITS = 3
FP8_MAX_BITS = 5              # widest code that E4M3 holds exactly


def e4m3_round(v) -> np.ndarray:
    """float32 array of the E4M3 values nearest to v (ties to the even
    mantissa), saturated to +-448.  v must be finite."""
    v = np.asarray(v, dtype=np.float32)
    if not np.all(np.isfinite(v)):
        raise ValueError("non-finite value")
    a = np.abs(v.astype(np.float64))
    _, e = np.frexp(a)                      # a = f * 2^e with f in [0.5, 1)
    lead = e - 1                             # 2^lead <= a < 2^(lead + 1)
    lead = np.maximum(lead, E4M3_MIN_NORMAL_EXP)   # subnormals share the quantum of 2^-6
    quantum = np.ldexp(1.0, lead - E4M3_MANT_BITS)
    r = np.rint(a / quantum) * quantum       # exact scalings by powers of two; rint ties to even
    r = np.minimum(r, E4M3_MAX)
    return (np.sign(v.astype(np.float64)) * r).astype(np.float32)


def quantize_x_fp8(x):
    """(xq float32 [M, K] of E4M3 values, sx float32 [M]) for bf16-valued x."""
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise TypeError("x must be 2-D")
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    fmax = np.float32(E4M3_MAX)
    with np.errstate(under="ignore"):
        sx = np.where(amax == 0, np.float32(1.0) / fmax, amax / fmax).astype(np.float32)
    t = (x / sx[:, None]).astype(np.float32)     # IEEE fp32 division
    return e4m3_round(t), sx


def check_bits(b: int) -> None:
    if not 4 <= int(b) <= FP8_MAX_BITS:
        raise ValueError(f"the E4M3 path holds codes of 4..{FP8_MAX_BITS} bits exactly, not {b}")


def qlinear_fp8_ref(x, q: np.ndarray, s: np.ndarray):
    """(y_ref, bound) in fp64 for the E4M3 path: y = sx * (xq @ (q * s)^T),
    accepted within 8e-3 * (|sx xq| @ |w_hat|^T) + 1e-6 (fp32 accumulation and
    the bf16 output; the rounding of x is part of the definition)."""
    q = np.asarray(q)
    xq, sx = quantize_x_fp8(x)
    xs = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    w_hat = q.astype(np.float64) * np.asarray(s, np.float64)[:, None]
    y = xs @ w_hat.T
    bound = QLINEAR_REL_TOL * (np.abs(xs) @ np.abs(w_hat).T) + QLINEAR_ABS_TOL
    return y, bound


def fp8_input_error_bound(x, q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Bound on |y_fp8 - x @ w_hat^T| that the rounding of x alone causes:
    each |x - sx * xq| is at most half an E4M3 step of the quotient, 2^-4 |x|
    in the normal range and 2^-10 sx below it, plus 2^-22 |x| for the fp32
    quotient itself (which also covers the rounding at the saturation point
    448), summed against |w_hat|."""
    x = np.asarray(x, np.float64)
    _, sx = quantize_x_fp8(x.astype(np.float32))
    half_step = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * sx.astype(np.float64)[:, None]) + \
        2.0 ** -22 * np.abs(x)
    w_hat = np.asarray(q, np.float64) * np.asarray(s, np.float64)[:, None]
    return half_step @ np.abs(w_hat).T
