"""Seeded weight and prompt generators (shapes and random draws only)."""
import os
import numpy as np


def f32_to_bf16_bits(a):
    """Round float32 to BF16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b):
    """Exact widening of BF16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32)


def tensor_names(shape):
    """Stable, ordered list of the weight tensors of a model shape."""
    names = ["embed", "lm_head", "s_z"]
    for i in range(shape.n_blocks):
        p = f"blk{i}."
        names += [p + "w_qkvg", p + "s_q", p + "s_k", p + "w_o",
                  p + "alpha_a", p + "w_gu", p + "w_down", p + "alpha_m"]
    return names


def tensor_spec(shape, name):
    """(kind, dims): kind 'mat' = BF16 row-normalised matrix, else a float32
    vector family ('alpha', 'qk_scale', 'logit_scale')."""
    d, F = shape.d, shape.ffn
    if name in ("embed", "lm_head"):
        return "mat", (shape.vocab, d)
    if name == "s_z":
        return "logit_scale", (shape.vocab,)
    leaf = name.split(".", 1)[1]
    return {
        "w_qkvg": ("mat", (shape.qkvg_rows, d)),
        "s_q": ("qk_scale", (shape.n_q_heads, shape.head_dim)),
        "s_k": ("qk_scale", (shape.n_kv_heads, shape.head_dim)),
        "w_o": ("mat", (d, shape.qdim)),
        "alpha_a": ("alpha", (d,)),
        "w_gu": ("mat", (2 * F, d)),      # F gate rows, then F up rows
        "w_down": ("mat", (d, F)),
        "alpha_m": ("alpha", (d,)),
    }[leaf]


def make_tensor(shape, name, seed=0):
    """Generate one tensor.  Matrices come back as uint16 BF16 bits."""
    idx = tensor_names(shape).index(name)
    rng = np.random.default_rng([seed, idx])
    kind, dims = tensor_spec(shape, name)
    if kind == "mat":
        rows, cols = dims
        out = np.empty(dims, dtype=np.uint16)
        step = max(1, (1 << 24) // cols)          # bounded temporaries
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            g = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
            nrm = np.sqrt(np.einsum("ij,ij->i", g, g, dtype=np.float64))
            g /= nrm[:, None].astype(np.float32)
            out[r0:r1] = f32_to_bf16_bits(g)
        return out
    noise = rng.standard_normal(dims).astype(np.float32) * np.float32(1e-3)
    if kind == "alpha":
        return np.float32(0.05) + noise
    if kind == "qk_scale":
        return np.float32(1.0) + noise
    if kind == "logit_scale":
        return np.float32(np.sqrt(shape.d)) * (np.float32(1.0) + noise)
    raise ValueError(kind)


def make_weights(shape, seed=0, names=None, workers=None):
    """All (or the listed) tensors as {name: ndarray}.

    ``workers`` > 1 draws tensors on a thread pool: NumPy's generator and the
    array arithmetic release the GIL, so threads scale without copying the
    tensors between processes.
    """
    names = list(names) if names is not None else tensor_names(shape)
    if workers is None:
        big = shape.params_per_block() * shape.n_blocks > 50_000_000
        workers = min(32, os.cpu_count() or 1) if big else 1
    if workers <= 1:
        return {n: make_tensor(shape, n, seed) for n in names}
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=workers) as ex:
        outs = list(ex.map(lambda n: make_tensor(shape, n, seed), names))
    return dict(zip(names, outs))


def make_prompt(shape, batch, length, seed=1):
    """Uniform random token ids in [0, vocab), int32 [batch, length]."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, shape.vocab, size=(batch, length), dtype=np.int64
                        ).astype(np.int32)
