"""Counter-based synthetic KV-cache contents ("context already cached").

The long-context workloads start from a cache that already holds n_ctx
tokens.  Both the CUDA path (the library's cache-fill entry point) and the
oracle tests generate those entries from the same published counter-based
generator, SplitMix64 (Steele, Lea and Flood, OOPSLA 2014), so no cache byte
travels from one side to the other.

Entry (kind, block, slot, b, kvh, pos, j), kind 0 = K, 1 = V, j < head_dim:
    c = ((((((kind * 64 + block) * 8 + slot) * 4096 + b) * 64 + kvh)
          * 2**20 + pos) * 512 + j)
    z = splitmix64(seed + c);   u = (z >> 40) * 2**-24   (24-bit uniform)
    K = bf16((2u - 1) * f32(sqrt(3 / head_dim)))   -> E|K|^2 = 1
    V = bf16((2u - 1) * f32(sqrt(3 / d)))          -> variance 1/d
All steps are exact in float32 except the final round-to-nearest-even to
BF16, so both sides produce identical bytes.
"""
import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)


def splitmix64(x):
    """SplitMix64 output function on uint64 arrays (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = (np.asarray(x, dtype=np.uint64) + np.uint64(0x9E3779B97F4A7C15))
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def counter(kind, block, slot, b, kvh, pos, j):
    c = np.uint64(kind)
    for v, m in ((block, 64), (slot, 8), (b, 4096), (kvh, 64)):
        c = c * np.uint64(m) + np.asarray(v, dtype=np.uint64)
    c = c * np.uint64(1 << 20) + np.asarray(pos, dtype=np.uint64)
    return c * np.uint64(512) + np.asarray(j, dtype=np.uint64)


def kv_rows(shape, seed, block, slot, b, kvh, positions):
    """K, V float32 arrays [len(positions), head_dim] (BF16-exact values)."""
    from .gen import f32_to_bf16_bits, bf16_bits_to_f32
    hd = shape.head_dim
    pos = np.asarray(positions, dtype=np.uint64)[:, None]
    j = np.arange(hd, dtype=np.uint64)[None, :]
    out = []
    for kind, c in ((0, np.float32(np.sqrt(3.0 / hd))),
                    (1, np.float32(np.sqrt(3.0 / shape.d)))):
        with np.errstate(over="ignore"):
            z = splitmix64(np.uint64(seed) + counter(kind, block, slot, b, kvh,
                                                     pos, j))
        u = (z >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)
        x = (np.float32(2.0) * u - np.float32(1.0)) * c
        out.append(bf16_bits_to_f32(f32_to_bf16_bits(x)))
    return out[0], out[1]
