"""Plain CPU definition of per-row symmetric INT-b quantization, bit packing and
the dequantize-then-multiply linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
it.  It shares no code, table or constant with the CUDA path.

Sources (page title, section):

* Quantization tutorial (aiknowledge.cn, "量化"), "How quantization works":
  scale = max|t| / max_int, q = round(t / scale), reconstruction q * scale,
  rounding error at most scale/2, one scale per output channel.
* Same page, "Step 1: symmetric quantization": the numpy reading of the same
  formulas -- qmax = 2^(b-1) - 1, np.round (round half to even), a zero channel
  takes the scale 1.0 / qmax, codes clipped to the integer range.
* DynaQuant (zingnex forum thread), "Step 3: apply the recipe" and "Custom kernel
  architecture": one bit width per matrix, packed N-bit storage, expanded to the
  hardware format and multiplied on tensor cores; "Status": bit pack / unpack.
* Quantization tutorial, exercises, item 1: group-wise scales (one per 128
  weights; 32, 64, 128 and 256 compared) -- ``quantize_groups`` and friends,
  groups of g consecutive weights along K, the last one shorter when g does
  not divide K.  No kernel reads this variant yet.

Readings taken where the pages are silent (each also listed in the design
notes):

* Scale axis: one fp32 scale per output row n of W[N, K], reduced over K.
* s_n = fl32(m_n / Q) with m_n = max_k |w_nk| (exact) and Q = 2^(b-1) - 1, an
  IEEE fp32 division.  A zero row takes s_n = fl32(1 / Q) and all-zero codes.
* q = clamp(rint_half_even(fl32(w / s_n)), -Q, Q) with an IEEE fp32 division.
  For a normal s_n the clamp is never active; it is active for subnormal
  scales.  If fl32(m_n / Q) underflows to zero the quotient is +-inf (clamped
  to +-Q) or, for w = 0, NaN, which is taken as code 0.
* Packing: u = q mod 2^b (two's complement), written LSB-first into a bit
  stream along K (code k occupies bits [k*b, k*b+b) of the row read as a
  little-endian integer); each row is padded with zero bits to
  16 * ceil(K*b/128) bytes.
* Linear layer: y[m, n] = s_n * sum_k x[m, k] * q[n, k]; the reference value is
  computed in fp64 from the exact w_hat = q * s, and an output is accepted when
  |y - y_ref| <= 8e-3 * sum_k |x[m, k] * w_hat[n, k]| + 1e-6.
* Non-finite weights are outside the method's domain: the oracle raises.
* Recipe data flow (no page gives one): a linear flagged to read the
  normalised input computes y = s_n * r_m * sum_k x[m, k] q[n, k] with
  r_m = 1 / sqrt(mean_k x[m, k]^2 + 1e-6).
"""
from __future__ import annotations

import numpy as np

MIN_BITS = 4
MAX_BITS = 15

# Acceptance bound for the fused linear layer (decode and prefill alike).
QLINEAR_REL_TOL = 8e-3
QLINEAR_ABS_TOL = 1e-6


def _check_bits(b: int) -> None:
    if not (MIN_BITS <= int(b) <= MAX_BITS):
        raise ValueError(f"bit width {b} outside {MIN_BITS}..{MAX_BITS}")


def qmax(b: int) -> int:
    """Largest code magnitude Q = 2^(b-1) - 1 (tutorial, "Step 1")."""
    _check_bits(b)
    return (1 << (b - 1)) - 1


def packed_row_bytes(K: int, b: int) -> int:
    """Bytes per packed row: ceil(K*b/8) rounded up to a multiple of 16."""
    _check_bits(b)
    return 16 * ((K * b + 127) // 128)


def unpadded_row_bytes(K: int, b: int) -> int:
    """ceil(K*b/8): the bytes a row needs before padding."""
    return (K * b + 7) // 8


# ----------------------------------------------------------------------------
# a1: row scales
# ----------------------------------------------------------------------------

def row_scales(W: np.ndarray, b: int) -> np.ndarray:
    """s_n = fl32(max_k |w_nk| / Q); zero rows take fl32(1/Q).

    Tutorial, "How quantization works" (scale = max(abs) / max_int) and
    "Step 1" (per-channel abs max; zero channel -> 1.0 / qmax).
    """
    W = np.asarray(W)
    if W.dtype != np.float32 or W.ndim != 2:
        raise TypeError("W must be a 2-D float32 array")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    Q = np.float32(qmax(b))
    m = np.max(np.abs(W), axis=1) if W.shape[1] > 0 else np.zeros(W.shape[0], np.float32)
    m = m.astype(np.float32)
    one = np.float32(1.0)
    with np.errstate(under="ignore"):
        s = np.where(m == 0, one / Q, m / Q).astype(np.float32)
    return s


# ----------------------------------------------------------------------------
# a2: codes
# ----------------------------------------------------------------------------

def quantize(W: np.ndarray, b: int):
    """(q int32[N, K], s float32[N]): q = clamp(rint(fl32(w / s)), -Q, Q).

    Tutorial, "How quantization works" (q = round(t / scale)) and "Step 1"
    (np.round, i.e. round half to even, then clip to the integer range).
    """
    s = row_scales(W, b)
    Q = qmax(b)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        t = W / s[:, None]                      # fp32 / fp32: IEEE quotient
    r = np.rint(t)                              # half to even
    r = np.where(np.isnan(r), np.float32(0), r)  # 0 / 0 when s underflowed
    q = np.clip(r, -Q, Q).astype(np.int32)
    return q, s


# ----------------------------------------------------------------------------
# a3 / a4: bit packing
# ----------------------------------------------------------------------------

def pack(q: np.ndarray, b: int) -> np.ndarray:
    """uint8[N, packed_row_bytes(K, b)]: LSB-first b-bit two's-complement stream.

    DynaQuant, "Status" (bit pack / unpack tools) and "Custom kernel
    architecture" (packed N-bit storage); bit order and padding per the
    canonical format above.
    """
    q = np.asarray(q)
    N, K = q.shape
    Q = qmax(b)
    if np.any(np.abs(q) > Q):
        raise ValueError("code outside +-Q")
    rb = packed_row_bytes(K, b)
    u = (q.astype(np.int64) & ((1 << b) - 1)).astype(np.uint32)
    bits = ((u[:, :, None] >> np.arange(b, dtype=np.uint32)) & 1).astype(np.uint8)
    bits = bits.reshape(N, K * b)
    padded = np.zeros((N, rb * 8), dtype=np.uint8)
    padded[:, : K * b] = bits
    return np.packbits(padded, axis=1, bitorder="little")


def unpack(packed: np.ndarray, K: int, b: int) -> np.ndarray:
    """int32[N, K]: the inverse of :func:`pack`, sign-extended."""
    packed = np.asarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    if packed.shape[1] != packed_row_bytes(K, b):
        raise ValueError("row stride does not match K and b")
    bits = np.unpackbits(packed, axis=1, bitorder="little")[:, : K * b]
    bits = bits.reshape(N, K, b).astype(np.int64)
    u = (bits << np.arange(b, dtype=np.int64)).sum(axis=2)
    q = np.where(u >= (1 << (b - 1)), u - (1 << b), u)
    return q.astype(np.int32)


# ----------------------------------------------------------------------------
# Paired-halves layout: a kernel-private re-ordering of the same bits.  No page
# defines it; the decode kernels read it because a 32-bit word then holds two
# codes 16 bits apart, the form in which they become one bf16x2 operand.
# ----------------------------------------------------------------------------

PAIR_GROUP = 32  # codes per group; K must be a multiple


def _paired_check(K: int, b: int) -> None:
    _check_bits(b)
    if K < 1 or K % PAIR_GROUP != 0:
        raise ValueError("the paired layout needs K to be a positive multiple of 32")


def pack_paired(q: np.ndarray, b: int) -> np.ndarray:
    """uint8[N, packed_row_bytes(K, b)] in the paired-halves layout.

    Row n is cut into groups of 32 codes.  In group g the even codes
    q[32g + 2i] (i = 0..15) form the stream E and the odd codes q[32g + 2i + 1]
    the stream O; in each stream code i occupies bits [i*b, i*b + b), LSB
    first, as b-bit two's complement, so each stream is b half-words of 16
    bits.  Little-endian 32-bit word g*b + h of the row holds half-word h of E
    in its low 16 bits and half-word h of O in its high 16 bits.  The bytes
    after the last group are zero.  The row stride is the canonical one, and
    the layout holds exactly the canonical bits, re-ordered.
    """
    q = np.asarray(q)
    N, K = q.shape
    _paired_check(K, b)
    if np.any(np.abs(q) > qmax(b)):
        raise ValueError("code outside +-Q")
    G = K // PAIR_GROUP
    u = (q.astype(np.int64) & ((1 << b) - 1)).astype(np.uint32).reshape(N, G, 16, 2)
    # bits[n, g, stream, i*b + t] = bit t of code i of the stream
    bits = ((u[..., None] >> np.arange(b, dtype=np.uint32)) & 1).astype(np.uint8)  # [N,G,16,2,b]
    streams = bits.transpose(0, 1, 3, 2, 4).reshape(N, G, 2, b, 16)  # [N,G,stream,half-word,bit]
    words = np.concatenate([streams[:, :, 0], streams[:, :, 1]], axis=3)  # [N,G,b,32]: E low, O high
    out = np.zeros((N, packed_row_bytes(K, b) * 8), dtype=np.uint8)
    out[:, : G * b * 32] = words.reshape(N, G * b * 32)
    return np.packbits(out, axis=1, bitorder="little")


def unpack_paired(packed: np.ndarray, K: int, b: int) -> np.ndarray:
    """int32[N, K]: the codes held by a paired-halves row (inverse of
    :func:`pack_paired`), sign-extended."""
    packed = np.asarray(packed, dtype=np.uint8)
    _paired_check(K, b)
    N = packed.shape[0]
    if packed.shape[1] != packed_row_bytes(K, b):
        raise ValueError("row stride does not match K and b")
    G = K // PAIR_GROUP
    bits = np.unpackbits(packed, axis=1, bitorder="little")[:, : G * b * 32]
    words = bits.reshape(N, G, b, 32)
    streams = np.stack([words[..., :16], words[..., 16:]], axis=2)  # [N,G,stream,b,16]
    codes_bits = streams.reshape(N, G, 2, 16, b).astype(np.int64)  # [N,G,stream,i,t]
    u = (codes_bits << np.arange(b, dtype=np.int64)).sum(axis=4)  # [N,G,stream,i]
    q = np.where(u >= (1 << (b - 1)), u - (1 << b), u)
    return q.transpose(0, 1, 3, 2).reshape(N, K).astype(np.int32)


def pair_halves(packed: np.ndarray, K: int, b: int) -> np.ndarray:
    """Canonical packed rows re-ordered into the paired-halves layout."""
    return pack_paired(unpack(packed, K, b), b)


def quantize_pack(W: np.ndarray, b: int):
    """(packed uint8[N, rb], s float32[N]) -- the whole quantizer."""
    q, s = quantize(W, b)
    return pack(q, b), s


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """float32[N, K]: fl32(q * s) (tutorial, reconstruction = quantized * scale)."""
    return (np.asarray(q).astype(np.float32) * np.asarray(s, np.float32)[:, None]).astype(np.float32)


# ----------------------------------------------------------------------------
# a5 / a6: fused linear layer
# ----------------------------------------------------------------------------

def qlinear_ref(x, q: np.ndarray, s: np.ndarray):
    """(y_ref, bound) in fp64 for y = x @ (q * s)^T.

    x: [M, K] values that are exactly bf16 (any float dtype holding them).
    Returns y_ref[M, N] and the per-element acceptance bound
    8e-3 * (|x| @ |w_hat|^T) + 1e-6.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w_hat = np.asarray(q).astype(np.float64) * np.asarray(s).astype(np.float64)[:, None]
    y = x64 @ w_hat.T
    bound = QLINEAR_REL_TOL * (np.abs(x64) @ np.abs(w_hat).T) + QLINEAR_ABS_TOL
    return y, bound


def qlinear_rows_ref(x, W_rows: np.ndarray, b: int):
    """Quantize only the given rows of W and return (y_ref, bound) for them.

    Row-wise quantization makes each output column depend on one row of W,
    so full-size cases can be checked on a sample of rows.
    """
    q, s = quantize(W_rows, b)
    return qlinear_ref(x, q, s)


def check_qlinear(y_gpu, y_ref, bound):
    """Boolean mask of accepted outputs."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    return np.abs(y_gpu - y_ref) <= bound


# ----------------------------------------------------------------------------
# a7: recipe decode pass helpers
# ----------------------------------------------------------------------------

RMS_EPS = 1e-6


def rms_scale(v) -> np.ndarray:
    """r_m = 1 / sqrt(mean_k(v[m, k]^2) + 1e-6) per row of v, in fp64.

    The pages give no data flow between the linears of the recipe stack; a
    linear that "reads rms(x)" computes y = s_n * r_m * sum_k x[m, k] q[n, k],
    i.e. the normalisation is a per-token scale applied to the product (see
    the design notes).  Returns shape [M, 1].
    """
    v = np.asarray(v, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(v ** 2, axis=-1, keepdims=True) + RMS_EPS)


def qlinear_rms_ref(x, q: np.ndarray, s: np.ndarray):
    """(y_ref, bound) for the linear of the rms-scaled input r_m * x[m, :]."""
    x64 = np.asarray(x, dtype=np.float64) * rms_scale(x)
    return qlinear_ref(x64, q, s)


# ----------------------------------------------------------------------------
# quality diagnostics (tutorial, "Step 2: quality metrics") -- not parity
# ----------------------------------------------------------------------------

# ----------------------------------------------------------------------------
# group-wise scales (a format variant; the oracle comes before any kernel)
# ----------------------------------------------------------------------------

def group_count(K: int, g: int) -> int:
    """Number of groups of g consecutive weights along a row of K."""
    if g < 1:
        raise ValueError("group size must be positive")
    return -(-int(K) // int(g))


def group_scales(W: np.ndarray, b: int, g: int) -> np.ndarray:
    """s[n, j] = fl32(max |w_nk| / Q) over group j = weights k in
    [j*g, min((j+1)*g, K)) of row n; a zero group takes fl32(1/Q).

    Tutorial, exercise 1 ("one scale per 128 weights instead of per channel",
    group sizes 32, 64, 128, 256 compared); the formula per group is the one
    of "How quantization works".
    """
    W = np.asarray(W)
    if W.dtype != np.float32 or W.ndim != 2:
        raise TypeError("W must be a 2-D float32 array")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    N, K = W.shape
    Q = np.float32(qmax(b))
    one = np.float32(1.0)
    s = np.empty((N, group_count(K, g)), np.float32)
    for j in range(s.shape[1]):
        m = np.max(np.abs(W[:, j * g:(j + 1) * g]), axis=1).astype(np.float32)
        with np.errstate(under="ignore"):
            s[:, j] = np.where(m == 0, one / Q, m / Q).astype(np.float32)
    return s


def group_scale_of_weight(s: np.ndarray, K: int, g: int) -> np.ndarray:
    """[N, K] array holding each weight's group scale."""
    return np.repeat(np.asarray(s, np.float32), g, axis=1)[:, :K]


def quantize_groups(W: np.ndarray, b: int, g: int):
    """(q int32[N, K], s float32[N, ceil(K/g)]): every weight is coded with its
    group's scale, q = clamp(rint(fl32(w / s_group)), -Q, Q)."""
    s = group_scales(W, b, g)
    sw = group_scale_of_weight(s, W.shape[1], g)
    Q = qmax(b)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        t = W / sw
    r = np.rint(t)
    r = np.where(np.isnan(r), np.float32(0), r)
    return np.clip(r, -Q, Q).astype(np.int32), s


def dequantize_groups(q: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """float32[N, K]: fl32(q * s_group)."""
    q = np.asarray(q)
    return (q.astype(np.float32) * group_scale_of_weight(s, q.shape[1], g)).astype(np.float32)


def qlinear_groups_ref(x, q: np.ndarray, s: np.ndarray, g: int):
    """(y_ref, bound) in fp64 for y = x @ w_hat^T with w_hat = q * s_group,
    accepted within 8e-3 * (|x| @ |w_hat|^T) + 1e-6 as for per-row scales."""
    q = np.asarray(q)
    x64 = np.asarray(x, dtype=np.float64)
    w_hat = q.astype(np.float64) * group_scale_of_weight(s, q.shape[1], g).astype(np.float64)
    y = x64 @ w_hat.T
    bound = QLINEAR_REL_TOL * (np.abs(x64) @ np.abs(w_hat).T) + QLINEAR_ABS_TOL
    return y, bound


def quality(original: np.ndarray, reconstructed: np.ndarray) -> dict:
    o = np.asarray(original, np.float64).ravel()
    r = np.asarray(reconstructed, np.float64).ravel()
    mse = float(np.mean((o - r) ** 2))
    snr = 10.0 * np.log10(np.mean(o ** 2) / max(mse, 1e-300))
    cos = float(np.dot(o, r) / (np.linalg.norm(o) * np.linalg.norm(r)))
    return {"mse": mse, "snr_db": float(snr), "cosine_similarity": cos}
