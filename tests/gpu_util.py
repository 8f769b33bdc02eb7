"""Helpers shared by the GPU tests: run the oracle and the CUDA path on the
same seeded inputs (teacher-forced greedy decode) and compare."""
import numpy as np
import torch

from oracle.model import Model

LOGIT_TOL = 3e-2          # max |delta logits|, BF16 path vs oracle
TOP1_MIN = 0.995          # top-1 agreement
NORM_TOL = 2e-3           # | ||s|| - 1 |


def oracle_run(shape, w, prompt, n_loops, kv_mode, n_decode, chunks=None):
    """Oracle logits for every prompt position, then n_decode greedy steps.
    Returns (prompt_logits [B,T,V], decode tokens [n_decode,B], decode
    logits [n_decode,B,V])."""
    B, T = prompt.shape
    m = Model(shape, w, batch=B, kv_mode=kv_mode)
    chunks = chunks or [T]
    zs, t0 = [], 0
    for c in chunks:
        zs.append(m.forward(prompt[:, t0:t0 + c], n_loops, all_logits=True))
        t0 += c
    zp = np.concatenate(zs, axis=1)
    toks, zd = [], []
    nxt = np.argmax(zp[:, -1], axis=-1)
    for _ in range(n_decode):
        toks.append(nxt.astype(np.int32))
        z = m.decode_step(nxt, n_loops)
        zd.append(z)
        nxt = np.argmax(z, axis=-1)
    return zp, np.array(toks), np.array(zd), m


def gpu_run(gm, prompt, n_loops, kv_mode, toks, chunks=None, max_ctx=None):
    B, T = prompt.shape
    chunks = chunks or [T]
    max_chunk = max(chunks)
    max_ctx = max_ctx or (T + len(toks) + 8)
    cache = gm.new_cache(B, max_ctx, max_chunk, kv_mode=kv_mode,
                         max_loops=max(n_loops, 1))
    ws = gm.workspace(B, max_chunk)
    dev = gm.device
    zs, am, t0 = [], [], 0
    for c in chunks:
        t = torch.from_numpy(np.ascontiguousarray(prompt[:, t0:t0 + c])).to(dev)
        z, a = gm.prefill(cache, t, n_loops, ws, logits_all=True)
        zs.append(z.cpu().numpy())
        am.append(a.cpu().numpy())
        t0 += c
    zd, ad, states = [], [], []
    for j in range(len(toks)):
        t = torch.from_numpy(toks[j]).to(dev)
        z, a = gm.decode_step(cache, t, n_loops, ws)
        zd.append(z.cpu().numpy())
        ad.append(a.cpu().numpy())
        states.append(gm.copy_state(ws, B, 1).cpu().numpy())
    torch.cuda.synchronize()
    assert gm.sync_status() == 0
    return (np.concatenate(zs, axis=1), np.concatenate(am, axis=1),
            np.array(zd), np.array(ad), states, cache)


def compare(z_gpu, z_ref, label):
    """Element-wise logits bound, and a valid greedy pick at every position:
    the GPU's top-1 token must score within LOGIT_TOL of the oracle's best
    (with random-init weights the top two logits can be closer than BF16
    rounding, and then either token is a correct argmax).  Returns
    (max|dz|, raw top-1 agreements, positions) for pooled agreement checks."""
    d = float(np.abs(z_gpu - z_ref).max())
    g = np.argmax(z_gpu, -1)
    r = np.argmax(z_ref, -1)
    picked = np.take_along_axis(z_ref, g[..., None], -1)[..., 0]
    slack = float((z_ref.max(-1) - picked).max())
    agree = int(np.sum(g == r))
    print(f"{label}: max|dz| {d:.3e}  top-1 {agree}/{g.size}  "
          f"worst pick slack {slack:.2e}")
    assert d <= LOGIT_TOL, f"{label}: max|dz| {d:.3e} > {LOGIT_TOL}"
    assert slack <= LOGIT_TOL, f"{label}: a greedy pick is {slack:.3e} below"
    return d, agree, g.size
