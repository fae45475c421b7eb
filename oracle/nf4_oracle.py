"""Plain CPU definitions of every step of the QLoRA NF4 linear layer.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

Sources, cited by page title and section:

* [UL] "QLoRA" -- Ultralytics glossary.  Section "How QLoRA works": the NF4 bullet
  (4-bit code per weight into 16 normal-quantile levels, one absmax scale per
  block of 64), the double-quantisation bullet (scales quantised to 8 bits in
  blocks of 256, overhead 0.5 -> about 0.127 bit/param), the paragraph on the
  forward/backward rule (dequantise to bfloat16 right before the matmul, add the
  LoRA path; gradients flow through the dequantised weights; only the two LoRA
  matrices are updated), and the snippet that builds the levels and quantises
  N(0, 0.02) blocks of 64 (printed MSE 3.395e-06 vs 4.053e-06).
* [VN] "Grokking QLoRA" -- vnread.  Section "Double Quantization": the
  per-block constants are compressed to FP8.
* [IBM] "What is LoRA?" -- IBM.  Low-rank matrices A, B of rank r; lora_alpha is
  the LoRA scaling factor; merging the update into the weights.
* [EZ] "Mastering model fine-tuning" -- ezsol.ir.  Section "Low-Rank Adaptation
  (LoRA)": Delta W = B A.

Readings where the pages are silent or loose:

* The level table is built in exact arithmetic (float64, Wichura's AS241 for the
  normal quantile) and rounded to float32 once; the offset is the printed
  decimal 0.9677083.
* Code assignment follows the snippet's float32 arithmetic: x = fl32(w / S),
  distance fl32(|fl32(x - L_j)|), first (lowest) j on ties, as torch.argmin does.
* An all-zero block gets S = 0 and code 7 (the exact-zero level).
* The 8-bit second-level format is OCP FP8 E4M3 (the only 8-bit format a page
  names): per group of 256 consecutive blocks c2 = fl32(max S / 448) and
  q = E4M3_rne_satfinite(fl32(S / c2)); an all-zero group has c2 = 0, q = 0.
  Two other readings of "8 bits in blocks of 256" are selectable with the same
  structure, the group maximum mapping to the format's largest value: OCP FP8
  E5M2 (c2 = fl32(max S / 57344), q = E5M2_rne_satfinite(fl32(S / c2))) and a
  linear unsigned byte (c2 = fl32(max S / 255), q = rne(fl32(S / c2)) clamped
  to 0..255, decoded value q).
* Codes are computed from the float32 S; double quantisation is applied to the
  scales afterwards.
* Dequantised weight: w' = bf16_rne(fl32(L[c] * fl32(dec(q) * c2))).
* Blocks are 64 consecutive elements of row-major W (cols % 64 == 0); groups of
  256 blocks run over the flat block index and may span rows; packed byte i holds
  element 2i in its low nibble and element 2i+1 in its high nibble.
* LoRA scale s = fl32(alpha) / fl32(r); y = X W'^T + s (X A^T) B^T.
* Merged export: the 16-bit weight a page says merging needs is bf16, the
  round-to-nearest-even of the exact W' + s B A (one rounding).
* LoRA dropout acts on the adapter branch's input only: D(X) = X * keep / (1-p)
  with a drawn keep mask passed in (bit j % 8 of byte j // 8 of each row).
* Adapter optimiser: the pages name Adam's per-parameter momentum and variance
  but give no update rule; the step is decoupled-weight-decay Adam (AdamW,
  Loshchilov and Hutter) with bias correction, the form torch.optim.AdamW uses.

What pins each function to something other than itself (tests/test_oracle_pins.py;
no function here is left unpinned):

* norm_ppf: statistics.NormalDist and scipy's ndtri; the erf-based CDF inverts it.
* nf4_levels: structure (sorted, exact 0 and +-1) and the snippet's float32 build.
* assign_codes / quantize: the page's worked example (printed MSEs, codes equal to
  torch's argmin), an exact-rational brute force, constructed ties, exact levels,
  all-zero blocks and groups, the ~16% MSE gain over evenly spaced levels.
* pack_codes / unpack_codes: the byte layout.
* e4m3_encode / e4m3_decode: the format's spec points, torch's float8 cast.
* double_quantize / dequantize: the scale error bound, requantise idempotence,
  one rounding of level times scale, the storage-overhead closed form.
* linear_fwd / linear_bwd: brute-force loops, central finite differences, B = 0,
  W = 0, the merged form.
* merged_weight / merge_export: B = 0 gives the dequantised weight bit for bit,
  W = 0 gives one bf16 rounding of the update, the layer's forward.
* adamw_step: torch.optim.AdamW over several steps, closed forms, a planted error.
* linear_fwd_multi: reduces to linear_fwd per token, adapters kept apart.
* unpack_keep / linear_fwd_dropout / linear_bwd_dropout: the mask layout, p = 0
  and everything dropped, central finite differences.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # weights per first-level absmax block [UL, NF4 bullet]
GROUP = 256         # first-level scales per second-level group [UL, double-quant bullet]
E4M3_MAX = 448.0    # largest finite OCP FP8 E4M3 value, 1.75 * 2**8
E5M2_MAX = 57344.0  # largest finite OCP FP8 E5M2 value, 1.75 * 2**15
U8_MAX = 255.0      # largest linear unsigned byte
SCALE_FORMATS = ("e4m3", "e5m2", "u8")
NF4_OFFSET = 0.9677083  # quantile offset exactly as printed in the [UL] snippet

_F32 = np.float32


# ---------------------------------------------------------------------------
# Normal quantile: Wichura, "Algorithm AS 241: The Percentage Points of the
# Normal Distribution", Applied Statistics 37 (1988) 477-484 (PPND16).
# ---------------------------------------------------------------------------
_AS241_A = (3.3871328727963666080e0, 1.3314166789178437745e2, 1.9715909503065514427e3,
            1.3731693765509461125e4, 4.5921953931549871457e4, 6.7265770927008700853e4,
            3.3430575583588128105e4, 2.5090809287301226727e3)
_AS241_B = (1.0, 4.2313330701600911252e1, 6.8718700749205790830e2, 5.3941960214247511077e3,
            2.1213794301586595867e4, 3.9307895800092710610e4, 2.8729085735721942674e4,
            5.2264952788528545610e3)
_AS241_C = (1.42343711074968357734e0, 4.63033784615654529590e0, 5.76949722146069140550e0,
            3.64784832476320460504e0, 1.27045825245236838258e0, 2.41780725177450611770e-1,
            2.27238449892691845833e-2, 7.74545014278341407640e-4)
_AS241_D = (1.0, 2.05319162663775882187e0, 1.67638483018380384940e0, 6.89767334985100004550e-1,
            1.48103976427480074590e-1, 1.51986665636164571966e-2, 5.47593808499534494600e-4,
            1.05075007164441684324e-9)
_AS241_E = (6.65790464350110377720e0, 5.46378491116411436990e0, 1.78482653991729133580e0,
            2.96560571828504891230e-1, 2.65321895265761230930e-2, 1.24266094738807843860e-3,
            2.71155556874348757815e-5, 2.01033439929228813265e-7)
_AS241_F = (1.0, 5.99832206555887937690e-1, 1.36929880922735805310e-1, 1.48753612908506148525e-2,
            7.86869131145613259100e-4, 1.84631831751005468180e-5, 1.42151175831644588870e-7,
            2.04426310338993978564e-15)


def _poly(coeffs, x):
    """c0 + c1 x + ... + c7 x^7 by Horner's rule (float64)."""
    acc = 0.0
    for c in reversed(coeffs):
        acc = acc * x + c
    return acc


def norm_ppf(p: float) -> float:
    """Standard normal quantile Phi^{-1}(p), 0 < p < 1, by AS241 (float64).

    Central region |p - 1/2| <= 0.425: rational function in (0.180625 - q^2).
    Tails: rational function in sqrt(-log(min(p, 1-p))) shifted by 1.6 (up to
    5) or by 5 beyond.
    """
    if not (0.0 < p < 1.0):
        raise ValueError("norm_ppf needs 0 < p < 1")
    q = p - 0.5
    if abs(q) <= 0.425:
        r = 0.180625 - q * q
        return q * _poly(_AS241_A, r) / _poly(_AS241_B, r)
    r = p if q < 0 else 1.0 - p
    r = math.sqrt(-math.log(r))
    if r <= 5.0:
        r -= 1.6
        val = _poly(_AS241_C, r) / _poly(_AS241_D, r)
    else:
        r -= 5.0
        val = _poly(_AS241_E, r) / _poly(_AS241_F, r)
    return -val if q < 0 else val


# ---------------------------------------------------------------------------
# Level tables
# ---------------------------------------------------------------------------
def nf4_levels() -> np.ndarray:
    """The 16 NF4 levels [UL, "How QLoRA works", snippet].

    Positive side: Phi^{-1} at the 9 evenly spaced points from the offset down to
    1/2, the last (1/2) dropped -> 8 values.  Negative side: -Phi^{-1} at the 8
    evenly spaced points from the offset down to 1/2, last dropped -> 7 values.
    Add an exact zero, sort ascending, divide by the largest.  Exact arithmetic
    (float64) rounded once to float32.
    """
    off = NF4_OFFSET
    pos = [norm_ppf(off + k * (0.5 - off) / 8.0) for k in range(8)]
    neg = [-norm_ppf(off + k * (0.5 - off) / 7.0) for k in range(7)]
    vals = sorted(neg + [0.0] + pos)
    top = max(vals)
    return np.array([v / top for v in vals], dtype=np.float64).astype(_F32)


def uniform4_levels() -> np.ndarray:
    """16 evenly spaced levels on [-1, 1], the snippet's comparison table
    [UL, "How QLoRA works", snippet], each fl32(-1 + 2k/15)."""
    return np.array([-1.0 + 2.0 * k / 15.0 for k in range(16)], dtype=np.float64).astype(_F32)


# ---------------------------------------------------------------------------
# First-level quantisation [UL, "How QLoRA works", NF4 bullet and snippet]
# ---------------------------------------------------------------------------
def block_absmax(w: np.ndarray) -> np.ndarray:
    """S[b] = max |w| over the b-th run of 64 consecutive (row-major) weights."""
    w = np.asarray(w, dtype=_F32).reshape(-1, BLOCK)
    return np.abs(w).max(axis=1)


def assign_codes(w: np.ndarray, absmax: np.ndarray, levels: np.ndarray,
                 chunk: int = 1 << 18) -> np.ndarray:
    """Code per weight: argmin_j fl32(|fl32(fl32(w / S) - L_j)|), lowest j on ties.

    Float32 throughout, as in the snippet.  A block with S == 0 gets the index of
    the exact-zero level (7 for NF4).
    """
    w = np.asarray(w, dtype=_F32).reshape(-1, BLOCK)
    absmax = np.asarray(absmax, dtype=_F32).reshape(-1)
    levels = np.asarray(levels, dtype=_F32)
    zero_code = int(np.flatnonzero(levels == 0)[0]) if np.any(levels == 0) else 0
    out = np.empty(w.shape, dtype=np.uint8)
    for b0 in range(0, w.shape[0], chunk):
        wb = w[b0:b0 + chunk]
        sb = absmax[b0:b0 + chunk]
        nz = sb != 0
        with np.errstate(invalid="ignore", divide="ignore"):
            x = wb / sb[:, None]                                  # fl32(w / S)
        dist = np.abs(x[..., None] - levels)                      # fl32(|fl32(x - L_j)|)
        codes = dist.argmin(axis=-1).astype(np.uint8)             # first minimum
        codes[~nz] = zero_code
        out[b0:b0 + chunk] = codes
    return out.reshape(-1)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: byte i = code[2i] | code[2i+1] << 4."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes."""
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


# ---------------------------------------------------------------------------
# OCP FP8 E4M3 ("fn": no infinities, max finite 448), written from the OCP
# 8-bit floating point specification: 1 sign, 4 exponent (bias 7), 3 mantissa
# bits; exponent field 0 is subnormal m * 2^-9; 0x7F/0xFF are NaN.
# ---------------------------------------------------------------------------
def e4m3_decode(code) -> np.ndarray:
    """Value (float64) of each E4M3 byte; NaN for 0x7F / 0xFF."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.power(2.0, e - 10))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(0x7F))  # codes 0x00..0x7E, strictly increasing


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code of each non-negative finite x: round to nearest, ties to the
    code with an even last mantissa bit, saturating to 448 (0x7E)."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(~np.isfinite(x)) or np.any(x < 0):
        raise ValueError("e4m3_encode takes finite non-negative values")
    xs = np.minimum(x, E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, xs, side="left")       # first value >= x
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E4M3_POS[hi] - xs                               # exact in float64
    d_lo = xs - _E4M3_POS[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & ((lo & 1) == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(_E4M3_POS[hi] == xs, hi, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# OCP FP8 E5M2 (IEEE-like: infinities and NaNs kept, max finite 57344), from the
# OCP 8-bit floating point specification: 1 sign, 5 exponent (bias 15), 2
# mantissa bits; exponent field 0 is subnormal m * 2^-16; exponent field 31 is
# infinity (m = 0) or NaN.
# ---------------------------------------------------------------------------
def e5m2_decode(code) -> np.ndarray:
    """Value (float64) of each E5M2 byte; +-inf for 0x7C / 0xFC, NaN for the rest
    of exponent field 31."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 2) & 0x1F
    m = c & 0x3
    with np.errstate(over="ignore"):
        mag = np.where(e == 0, m * 2.0 ** -16, (4 + m) * np.power(2.0, e - 17))
    mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    return sign * mag


_E5M2_POS = e5m2_decode(np.arange(0x7C))  # codes 0x00..0x7B, strictly increasing


def _encode_rne(x, table, top):
    """Index of the nearest table value to each x in [0, table[top]] (ties to the
    even index, which for these formats is the even last mantissa bit); values
    above table[top] saturate to top."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(~np.isfinite(x)) or np.any(x < 0):
        raise ValueError("scale codes take finite non-negative values")
    xs = np.minimum(x, table[top])
    hi = np.minimum(np.searchsorted(table, xs, side="left"), top)  # first value >= x
    lo = np.maximum(hi - 1, 0)
    d_hi = table[hi] - xs                                           # exact in float64
    d_lo = xs - table[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & ((lo & 1) == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(table[hi] == xs, hi, code)
    return code.astype(np.uint8)


def e5m2_encode(x) -> np.ndarray:
    """E5M2 code of each non-negative finite x: round to nearest, ties to even,
    saturating to 57344 (0x7B)."""
    return _encode_rne(x, _E5M2_POS, 0x7B)


def u8_encode(x) -> np.ndarray:
    """Linear byte of each non-negative finite x: round to nearest, ties to
    even, clamped to 255."""
    return _encode_rne(x, np.arange(256, dtype=np.float64), 255)


def scale_format_max(fmt: str) -> float:
    """The value the largest scale of a group maps to."""
    return {"e4m3": E4M3_MAX, "e5m2": E5M2_MAX, "u8": U8_MAX}[fmt]


def scale_decode(code, fmt: str = "e4m3") -> np.ndarray:
    """Value (float64, exact) of each 8-bit scale code in format fmt."""
    if fmt == "e4m3":
        return e4m3_decode(code)
    if fmt == "e5m2":
        return e5m2_decode(code)
    if fmt == "u8":
        return np.asarray(code, dtype=np.int64).astype(np.float64)
    raise ValueError(fmt)


def scale_encode(x, fmt: str = "e4m3") -> np.ndarray:
    if fmt == "e4m3":
        return e4m3_encode(x)
    if fmt == "e5m2":
        return e5m2_encode(x)
    if fmt == "u8":
        return u8_encode(x)
    raise ValueError(fmt)


# ---------------------------------------------------------------------------
# Second-level ("double") quantisation [UL, double-quant bullet; VN, "Double
# Quantization"]
# ---------------------------------------------------------------------------
def double_quantize(absmax: np.ndarray, fmt: str = "e4m3"):
    """Per group of 256 consecutive first-level scales (last group may be short):
    c2 = fl32(max S / F) and q[b] = enc(fl32(S[b] / c2)), with F and enc the
    format's largest value and encoder (E4M3: 448; E5M2: 57344; linear byte:
    255); an all-zero group has c2 = 0 and q = 0.  Returns (q uint8[nb], c2
    float32[ng])."""
    s = np.asarray(absmax, dtype=_F32).reshape(-1)
    nb = s.size
    ng = (nb + GROUP - 1) // GROUP
    q = np.zeros(nb, dtype=np.uint8)
    c2 = np.zeros(ng, dtype=_F32)
    fmax = _F32(scale_format_max(fmt))
    for g in range(ng):
        sg = s[g * GROUP:(g + 1) * GROUP]
        m = sg.max()
        if m == 0:
            continue
        c2[g] = _F32(m) / fmax                                  # fl32(m / F)
        q[g * GROUP:g * GROUP + sg.size] = scale_encode((sg / c2[g]).astype(_F32), fmt)
    return q, c2


def quantize(w: np.ndarray, rows: int, cols: int, levels: np.ndarray | None = None, scale_format: str = "e4m3"):
    """Whole quantiser: absmax per 64-block, NF4 codes, packing, double quant.

    ``w`` holds the rows x cols weights (float32, or bfloat16 values widened
    exactly).  Returns a dict with packed ``codes`` (rows*cols/2 bytes),
    ``scale_codes`` (8-bit codes in ``scale_format``, one per block), ``c2``
    (float32 per group) and the first-level ``absmax`` (float32 per block, for
    tests).
    """
    if cols % BLOCK:
        raise ValueError("cols must be a multiple of 64")
    if levels is None:
        levels = nf4_levels()
    w = np.asarray(w, dtype=_F32).reshape(rows * cols)
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weights")
    s = block_absmax(w)
    codes = assign_codes(w, s, levels)
    q, c2 = double_quantize(s, scale_format)
    return {"codes": pack_codes(codes), "scale_codes": q, "c2": c2, "absmax": s, "scale_format": scale_format}


# ---------------------------------------------------------------------------
# Dequantisation [UL, forward rule: NF4 -> bfloat16 right before the matmul]
# ---------------------------------------------------------------------------
def dequantize_scales(scale_codes: np.ndarray, c2: np.ndarray, fmt: str = "e4m3") -> np.ndarray:
    """S'[b] = fl32(dec(q[b]) * c2[b // 256])."""
    q = np.asarray(scale_codes, dtype=np.uint8).reshape(-1)
    g = np.arange(q.size) // GROUP
    dec = scale_decode(q, fmt).astype(_F32)                     # exact in float32
    return (dec * np.asarray(c2, dtype=_F32)[g]).astype(_F32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16
    bit patterns.  Finite inputs only."""
    b = np.ascontiguousarray(np.asarray(x, dtype=_F32)).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    return ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 value of bf16_rne(x)."""
    bits = bf16_bits(x).astype(np.uint32) << 16
    return bits.view(_F32)


def dequantize(codes: np.ndarray, scale_codes: np.ndarray, c2: np.ndarray,
               rows: int, cols: int, levels: np.ndarray | None = None, scale_format: str = "e4m3") -> np.ndarray:
    """W'[i] = bf16_rne(fl32(L[c_i] * S'[i // 64])), returned as float32 values
    (each exactly a bfloat16), shape (rows, cols)."""
    if levels is None:
        levels = nf4_levels()
    c = unpack_codes(codes)
    sp = dequantize_scales(scale_codes, c2, scale_format)
    prod = (levels[c].reshape(-1, BLOCK) * sp[:, None]).astype(_F32)   # fl32(L * S')
    return bf16_round(prod.reshape(-1)).reshape(rows, cols)


def storage_bytes(rows: int, cols: int):
    """Bytes of the quantised tensor: (codes, scale codes, c2 constants)."""
    n = rows * cols
    nb = n // BLOCK
    ng = (nb + GROUP - 1) // GROUP
    return n // 2, nb, 4 * ng


# ---------------------------------------------------------------------------
# Frozen linear layer with LoRA [UL, forward/backward paragraph; IBM; EZ]
# ---------------------------------------------------------------------------
def lora_scale(alpha: float, r: int) -> float:
    """s = fl32(alpha) / fl32(r), computed in float32."""
    return float(_F32(alpha) / _F32(r))


def linear_fwd(w_dq: np.ndarray, a: np.ndarray, b: np.ndarray, x: np.ndarray,
               alpha: float, r: int):
    """y = X W'^T + s (X A^T) B^T; returns (y, T) with T = X A^T, float64.

    Shapes: W' [N, K], A [r, K], B [N, r], X [M, K].
    """
    s = lora_scale(alpha, r)
    x64 = np.asarray(x, dtype=np.float64)
    t = x64 @ np.asarray(a, dtype=np.float64).T
    y = x64 @ np.asarray(w_dq, dtype=np.float64).T + s * (t @ np.asarray(b, dtype=np.float64).T)
    return y, t


def linear_bwd(w_dq: np.ndarray, a: np.ndarray, b: np.ndarray, x: np.ndarray,
               dy: np.ndarray, alpha: float, r: int, t: np.ndarray | None = None):
    """Gradients of the layer for upstream gradient dY [M, N], float64.

    U = dY B;  dX = dY W' + s U A;  dA = s U^T X;  dB = s dY^T T.
    The frozen W' gets no gradient; only A and B are trained.
    """
    s = lora_scale(alpha, r)
    x64 = np.asarray(x, dtype=np.float64)
    dy64 = np.asarray(dy, dtype=np.float64)
    a64 = np.asarray(a, dtype=np.float64)
    b64 = np.asarray(b, dtype=np.float64)
    if t is None:
        t = x64 @ a64.T
    u = dy64 @ b64
    dx = dy64 @ np.asarray(w_dq, dtype=np.float64) + s * (u @ a64)
    da = s * (u.T @ x64)
    db = s * (dy64.T @ np.asarray(t, dtype=np.float64))
    return dx, da, db


def unpack_keep(keep_bits: np.ndarray, m: int, k: int) -> np.ndarray:
    """Keep mask [m, k] (bool) from its packed form: bit (j % 8) of byte j // 8 of row i."""
    bits = np.asarray(keep_bits, np.uint8).reshape(m, k // 8)
    return ((bits[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).reshape(m, k).astype(bool)


def linear_fwd_dropout(w_dq: np.ndarray, a: np.ndarray, b: np.ndarray, x: np.ndarray, keep: np.ndarray,
                       p: float, alpha: float, r: int):
    """Forward with dropout on the LoRA input (lora_dropout):
    y = X W'^T + s (D(X) A^T) B^T,  D(X) = X * keep / (1 - p).  Returns (y, T = D(X) A^T).

    [EZ] "Low-Rank Adaptation (LoRA)": the LoRA configuration of its example sets
    lora_dropout; the dropped input feeds only the adapter branch.  keep is the
    drawn mask (passed in; 1 keeps an element).
    """
    s = lora_scale(alpha, r)
    x64 = np.asarray(x, np.float64)
    xd = x64 * np.asarray(keep, np.float64) / (1.0 - p)
    t = xd @ np.asarray(a, np.float64).T
    y = x64 @ np.asarray(w_dq, np.float64).T + s * (t @ np.asarray(b, np.float64).T)
    return y, t


def linear_bwd_dropout(w_dq: np.ndarray, a: np.ndarray, b: np.ndarray, x: np.ndarray, dy: np.ndarray,
                       keep: np.ndarray, p: float, alpha: float, r: int):
    """Gradients of linear_fwd_dropout for upstream dY, float64:
    U = dY B;  dX = dY W' + s (U A) * keep / (1 - p);  dA = s U^T D(X);  dB = s dY^T D(X) A^T."""
    s = lora_scale(alpha, r)
    x64 = np.asarray(x, np.float64)
    dy64 = np.asarray(dy, np.float64)
    a64 = np.asarray(a, np.float64)
    b64 = np.asarray(b, np.float64)
    kp = np.asarray(keep, np.float64) / (1.0 - p)
    xd = x64 * kp
    u = dy64 @ b64
    dx = dy64 @ np.asarray(w_dq, np.float64) + s * (u @ a64) * kp
    da = s * (u.T @ xd)
    db = s * (dy64.T @ (xd @ a64.T))
    return dx, da, db


def linear_fwd_multi(w_dq: np.ndarray, adapters, adapter_of_token, x: np.ndarray):
    """Forward of one frozen base serving several adapters: token t uses adapter
    adapters[adapter_of_token[t]] = (A, B, alpha, r), y_t = W' x_t + s_t (x_t A^T) B^T.

    [IBM] (one shared base model, many small LoRA modules swapped per task);
    [UL] "Trade-offs" (adapters small enough to store and swap per task).
    Returns y [M, N] float64.
    """
    x = np.asarray(x)
    out = []
    for t in range(x.shape[0]):
        a, b, alpha, r = adapters[adapter_of_token[t]]
        y, _ = linear_fwd(w_dq, a, b, x[t:t + 1], alpha, r)
        out.append(y[0])
    return np.stack(out)


def merged_weight(w_dq: np.ndarray, a: np.ndarray, b: np.ndarray, alpha: float, r: int):
    """W' + s B A (float64): the merged deployment form [IBM; EZ, Delta W = B A]."""
    s = lora_scale(alpha, r)
    return np.asarray(w_dq, np.float64) + s * (np.asarray(b, np.float64) @ np.asarray(a, np.float64))


def merge_export(codes: np.ndarray, scale_codes: np.ndarray, c2: np.ndarray, rows: int, cols: int,
                 a: np.ndarray, b: np.ndarray, alpha: float, r: int, scale_format: str = "e4m3") -> np.ndarray:
    """The merged 16-bit weight, as float32 values of bf16: bf16_rne(W' + s B A).

    [UL] "Trade-offs": merging the adapters into the base model first needs the
    base dequantised to 16 bit; [IBM]: the trained low-rank update is merged into
    the frozen weights for deployment.  W' + s B A is summed exactly (float64)
    and rounded to bf16 once.
    """
    wd = dequantize(codes, scale_codes, c2, rows, cols, scale_format=scale_format)
    return bf16_round(merged_weight(wd, a, b, alpha, r))


def adamw_step(p: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, step: int, lr: float,
               beta1: float, beta2: float, eps: float, weight_decay: float):
    """One AdamW step on float64 copies; returns (p, m, v) after step number `step` (1-based).

    m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2;
    p = p (1 - lr wd) - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps).
    [UL] "How QLoRA works": only the LoRA matrices are updated; [VN] "Paged
    Optimizers": Adam keeps momentum and variance for every trained parameter.
    """
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    p = p * (1.0 - lr * weight_decay) - (lr / bc1) * m / (np.sqrt(v) / math.sqrt(bc2) + eps)
    return p, m, v
