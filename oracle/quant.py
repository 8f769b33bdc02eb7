"""MXFP8 and NVFP4 weight formats: decoders and max-scaling quantisers.

TEST INFRASTRUCTURE (see package docstring).

The pages fix the formats only by name: MXFP8 W8A16 with group size 32
(MXFP8 explainer page, deployment section) and NVFP4 as E2M1 values with
E4M3 scale factors (paper summary, 前置知识 / NVFP4).  The element encodings
below follow the public OCP Microscaling (MX) format definitions and NVIDIA's
NVFP4 description.  The quantisers use maximum scaling (paperlayer §5.2:
MXFP8 uses standard max scaling), and quant_nvfp4_mse the dynamic MSE block
scale selection that the same section names for NVFP4 (its search range is
a reading, stated there).  Both sides decode the same bytes, so the choice
of quantiser changes accuracy, not parity.

Layouts (row-major, K = input/contraction axis):
  MXFP8: q uint8 [N, K] (E4M3 codes), e uint8 [N, K/32] (E8M0 codes).
         w = e4m3(q) * 2^(e - 127).
  NVFP4: q uint8 [N, K/2] (two E2M1 codes: element 2j in bits 0-3, element
         2j+1 in bits 4-7), sb uint8 [N, K/16] (E4M3 codes), S float32.
         w = e2m1(q) * e4m3(sb) * S; S is applied after the contraction.
"""
import numpy as np


def e4m3_decode(code):
    """OCP E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinity;
    S.1111.111 is NaN; largest finite 448; subnormals m * 2^-9."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e8m0_decode(code):
    """OCP E8M0 scale: 2^(code - 127); 0xFF is NaN."""
    c = np.asarray(code, dtype=np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 127))


def e2m1_decode(code):
    """E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; values
    0, 0.5, 1, 1.5, 2, 3, 4, 6 with sign; no NaN or infinity."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * 2.0 ** (e - 1.0))
    return sign * mag


def _round_to_codes(x, pos_codes, decode, sign_bit):
    """Round to the nearest representable value, ties to the even code;
    magnitudes beyond the largest finite value saturate to it."""
    vals = decode(pos_codes)
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo = hi - 1
    dlo, dhi = a - vals[lo], vals[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((pos_codes[hi] & 1) == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a >= vals[-1], len(vals) - 1, idx)
    code = pos_codes[idx]
    return np.where(np.signbit(x), code | sign_bit, code).astype(np.uint8)


_E4M3_POS = np.arange(0x00, 0x7F, dtype=np.int64)      # 0x7F is NaN
_E2M1_POS = np.arange(0, 8, dtype=np.int64)


def round_e4m3(x):
    return _round_to_codes(x, _E4M3_POS, e4m3_decode, 0x80)


def round_e2m1(x):
    return _round_to_codes(x, _E2M1_POS, e2m1_decode, 0x8)


def quant_mxfp8(w):
    """Max scaling per 32 consecutive weights along K: the shared exponent is
    floor(log2(amax)) - 8 (8 = exponent of E4M3's largest power of two),
    clamped to [-127, 127]; an all-zero group gets code 0."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    g = w.reshape(N, K // 32, 32)
    amax = np.abs(g).max(axis=-1)
    _, ex = np.frexp(amax)                  # amax = f * 2^ex, f in [0.5, 1)
    e = np.clip(ex - 1 - 8, -127, 127)
    ecode = np.where(amax > 0, e + 127, 0).astype(np.uint8)
    scale = np.ldexp(1.0, ecode.astype(np.int64) - 127)
    q = round_e4m3(g / scale[..., None]).reshape(N, K)
    return q, ecode


def dequant_mxfp8(q, ecode):
    N, K = q.shape
    v = e4m3_decode(q).reshape(N, K // 32, 32)
    return (v * e8m0_decode(ecode)[..., None]).reshape(N, K)


def quant_nvfp4(w):
    """Two-level max scaling: tensor scale S = amax/(6*448); per 16 weights
    along K a block scale sb = E4M3(amax_blk / (6 S)); values
    E2M1(w / (sb S)) saturating at +-6."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    amax_t = float(np.abs(w).max())
    S = np.float32(amax_t / (6.0 * 448.0)) if amax_t > 0 else np.float32(1.0)
    g = w.reshape(N, K // 16, 16)
    sb = round_e4m3(np.abs(g).max(axis=-1) / (6.0 * float(S)))
    den = e4m3_decode(sb) * float(S)
    safe = np.where(den > 0, den, 1.0)
    codes = np.where(den[..., None] > 0, round_e2m1(g / safe[..., None]), 0)
    codes = codes.reshape(N, K).astype(np.uint8)
    packed = (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)
    return packed.astype(np.uint8), sb, S


def quant_nvfp4_mse(w, below=8, above=1):
    """NVFP4 with dynamic MSE block-scale selection (paperlayer summary §5.2:
    NVFP4 uses dynamic MSE scale selection, MXFP8 and the other formats max
    scaling).  The pages give no search range; the reading taken here: the
    tensor scale S stays the max-scaling one, and for every 16-weight block
    the E4M3 scale code is the one, among the max-scaling code c and the
    codes c - below .. c + above (within the finite positive codes 1..126;
    `below` = 8 spans one binade), whose decoded block has the smallest sum
    of squared errors; ties go to the larger code.  All-zero blocks keep
    code 0.  Values are rounded as in quant_nvfp4."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    amax_t = float(np.abs(w).max())
    S = np.float32(amax_t / (6.0 * 448.0)) if amax_t > 0 else np.float32(1.0)
    g = w.reshape(N, K // 16, 16)
    c_max = round_e4m3(np.abs(g).max(axis=-1) / (6.0 * float(S))).astype(np.int64)
    best_c = c_max.copy()
    best_err = np.full(c_max.shape, np.inf)
    for off in range(above, -below - 1, -1):            # larger codes first
        c = np.clip(c_max + off, 1, 126)
        den = e4m3_decode(c) * float(S)
        codes = round_e2m1(g / den[..., None])
        err = np.sum((g - e2m1_decode(codes) * den[..., None]) ** 2, axis=-1)
        better = err < best_err
        best_err = np.where(better, err, best_err)
        best_c = np.where(better, c, best_c)
    sb = np.where(c_max > 0, best_c, 0).astype(np.uint8)
    den = e4m3_decode(sb) * float(S)
    safe = np.where(den > 0, den, 1.0)
    codes = np.where(den[..., None] > 0, round_e2m1(g / safe[..., None]), 0)
    codes = codes.reshape(N, K).astype(np.uint8)
    packed = (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)
    return packed.astype(np.uint8), sb, S


def unpack_nvfp4(packed):
    N, Kh = packed.shape
    out = np.empty((N, 2 * Kh), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def dequant_nvfp4(packed, sb, S=None):
    """Weights before the tensor scale (e2m1 * e4m3); times S if given."""
    codes = unpack_nvfp4(packed)
    N, K = codes.shape
    v = e2m1_decode(codes).reshape(N, K // 16, 16)
    w = (v * e4m3_decode(sb)[..., None]).reshape(N, K)
    return w if S is None else w * float(S)
