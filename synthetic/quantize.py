"""Weight-format encoding of the seeded BF16 weights into the quantised
checkpoint formats the Dory pages name: MXFP8 W8A16 (E4M3 values, E8M0 scale
per 32 weights; MXFP8 explainer page, deployment section) and NVFP4 W4A16
(E2M1 values, E4M3 scale per 16 weights, f32 tensor scale; paper summary,
前置知识 / NVFP4).  Maximum scaling, and for NVFP4 also the dynamic MSE
block-scale selection (paperlayer §5.2).  This is input
preparation only; a test checks that it produces exactly the bytes of the
oracle's own quantiser.

Only the block projections are quantised; embeddings and the LM head stay
BF16 (paperlayer §5.2).  A quantised matrix `name` becomes
  name.q  uint8 codes  (MXFP8 [N, K]; NVFP4 [N, K/2], element 2j in the low
                        nibble)
  name.s  uint8 scales (MXFP8 E8M0 [N, K/32]; NVFP4 E4M3 [N, K/16])
  name.t  float32 [1]  (NVFP4 tensor scale)
"""
import numpy as np

from .gen import bf16_bits_to_f32

QUANT_LEAVES = ("w_qkvg", "w_o", "w_gu", "w_down")


def _e4m3_values():
    c = np.arange(0x7F)
    e, m = (c >> 3) & 0xF, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7.0))


def _e2m1_values():
    return np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _nearest(x, vals):
    """Code of the nearest value (ties to the even code), with sign bit as
    the top bit of the format; magnitudes beyond the table saturate."""
    a = np.abs(x)
    hi = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo = hi - 1
    up = (vals[hi] - a < a - vals[lo]) | ((vals[hi] - a == a - vals[lo]) &
                                          (hi % 2 == 0))
    return np.where(a >= vals[-1], len(vals) - 1, np.where(up, hi, lo))


def encode_mxfp8(w):
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    g = w.reshape(N, K // 32, 32)
    amax = np.abs(g).max(-1)
    _, ex = np.frexp(amax)
    e = np.clip(ex - 9, -127, 127)
    ecode = np.where(amax > 0, e + 127, 0).astype(np.uint8)
    scale = np.ldexp(1.0, ecode.astype(np.int64) - 127)
    y = g / scale[..., None]
    code = _nearest(y, _e4m3_values()) | np.where(np.signbit(y), 0x80, 0)
    return code.reshape(N, K).astype(np.uint8), ecode


def encode_nvfp4(w):
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    amax = float(np.abs(w).max())
    S = np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)
    g = w.reshape(N, K // 16, 16)
    e4 = _e4m3_values()
    sb = _nearest(np.abs(g).max(-1) / (6.0 * float(S)), e4).astype(np.uint8)
    den = e4[sb] * float(S)
    y = g / np.where(den > 0, den, 1.0)[..., None]
    c = _nearest(y, _e2m1_values()) | np.where(np.signbit(y), 0x8, 0)
    c = np.where(den[..., None] > 0, c, 0).reshape(N, K).astype(np.uint8)
    packed = (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)
    return packed.astype(np.uint8), sb, np.array([S], dtype=np.float32)


def _nvfp4_block_codes(g, S, e4, below=8, above=1):
    """E4M3 block-scale codes of 16-weight blocks g [n, K/16, 16] chosen by
    minimum squared error among the max-scaling code c and c - below ..
    c + above (finite positive codes only; ties to the larger code; all-zero
    blocks keep code 0).  Input preparation for the NVFP4 'dynamic MSE'
    checkpoints (paperlayer summary §5.2)."""
    c0 = _nearest(np.abs(g).max(-1) / (6.0 * float(S)), e4).astype(np.int64)
    e2 = _e2m1_values()
    best, best_err = c0.copy(), np.full(c0.shape, np.inf)
    for off in range(above, -below - 1, -1):
        c = np.clip(c0 + off, 1, 126)
        den = e4[c] * float(S)
        y = g / den[..., None]
        v = e2[_nearest(y, e2)] * np.where(np.signbit(y), -1.0, 1.0)
        err = np.sum((g - v * den[..., None]) ** 2, axis=-1)
        better = err < best_err
        best_err = np.where(better, err, best_err)
        best = np.where(better, c, best)
    return np.where(c0 > 0, best, 0).astype(np.uint8)


def _encode_rows(w, fmt, rows=2048):
    """Encode in row chunks (bounded float64 temporaries).  The NVFP4 tensor
    scale needs the whole-matrix maximum first."""
    N = w.shape[0]
    if fmt == "mxfp8":
        qs, ss = zip(*(encode_mxfp8(w[r:r + rows]) for r in range(0, N, rows)))
        return np.concatenate(qs), np.concatenate(ss)
    amax = float(np.abs(w).max())
    S = np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)
    e4, out_q, out_s = _e4m3_values(), [], []
    for r in range(0, N, rows):
        g = np.asarray(w[r:r + rows], dtype=np.float64)
        n, K = g.shape
        g = g.reshape(n, K // 16, 16)
        if fmt == "nvfp4_mse":
            sb = _nvfp4_block_codes(g, S, e4)
        else:
            sb = _nearest(np.abs(g).max(-1) / (6.0 * float(S)), e4).astype(np.uint8)
        den = e4[sb] * float(S)
        y = g / np.where(den > 0, den, 1.0)[..., None]
        c = _nearest(y, _e2m1_values()) | np.where(np.signbit(y), 0x8, 0)
        c = np.where(den[..., None] > 0, c, 0).reshape(n, K).astype(np.uint8)
        out_q.append(((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8))
        out_s.append(sb)
    return (np.concatenate(out_q), np.concatenate(out_s),
            np.array([S], dtype=np.float32))


def quantize_weights(weights, fmt, workers=None):
    """Copy of `weights` with the block projections in `fmt` ('mxfp8',
    'nvfp4', or 'nvfp4_mse': the NVFP4 format with block scales chosen by
    minimum squared error); embeddings, LM head and vectors unchanged.  Matrices are
    encoded on a thread pool (NumPy releases the GIL in the bulk work)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    if fmt not in ("mxfp8", "nvfp4", "nvfp4_mse"):
        raise ValueError(fmt)
    names = [n for n in weights if n.split(".", 1)[-1] in QUANT_LEAVES]
    out = {n: t for n, t in weights.items() if n not in names}
    workers = workers or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=workers) as ex:
        res = list(ex.map(lambda n: _encode_rows(bf16_bits_to_f32(weights[n]),
                                                 fmt), names))
    for n, r in zip(names, res):
        out[n + ".q"], out[n + ".s"] = r[0], r[1]
        if fmt != "mxfp8":
            out[n + ".t"] = r[2]
    return out
