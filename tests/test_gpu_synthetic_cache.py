"""A cache filled with seeded synthetic context (dory_cache_fill_synthetic)
decodes like the oracle given the same entries from synthetic.kvgen:
tiny model, B=2, 40 cached tokens (more than the 16-token window, so the
rings wrap), k=2, both KV modes, 6 teacher-forced decode steps."""
import numpy as np
import pytest
import torch

from oracle.model import Model
from synthetic import TINY, make_weights
from synthetic.kvgen import kv_rows
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


def oracle_with_cache(w, B, n_ctx, seed, kv_mode, k):
    m = Model(TINY, w, batch=B, kv_mode=kv_mode)
    gin, grec, gout = TINY.block_groups()
    for i in range(TINY.n_blocks):
        slots = range(1, k + 1) if (i in grec and kv_mode == "per_loop") else [0]
        for s in slots:
            K = np.zeros((B, TINY.n_kv_heads, n_ctx, TINY.head_dim))
            V = np.zeros_like(K)
            for b in range(B):
                for h in range(TINY.n_kv_heads):
                    kk, vv = kv_rows(TINY, seed, i, s, b, h, np.arange(n_ctx))
                    K[b, h], V[b, h] = kk, vv
            m.cache[(i, s)] = (K, V)
    m.n_ctx = n_ctx
    return m


@pytest.mark.parametrize("kv_mode", ["per_loop", "last_loop"])
def test_synthetic_context_decode(kv_mode):
    import looped_ngpt_b200 as lb
    w = make_weights(TINY, seed=0)
    gm = lb.DoryModel(TINY, w, device="cuda:0")
    B, n_ctx, seed, k = 2, 40, 2, 2
    ref = oracle_with_cache(w, B, n_ctx, seed, kv_mode, k)
    cache = gm.new_cache(B, 64, 1, kv_mode=kv_mode, max_loops=k)
    cache.fill_synthetic(n_ctx, seed)
    ws = gm.workspace(B, 1)
    tok = np.array([3, 700])
    zr, zg = [], []
    for _ in range(6):
        z = ref.decode_step(tok, k)
        g, _ = gm.decode_step(cache, torch.from_numpy(tok.astype(np.int32)).cuda(),
                              k, ws)
        zr.append(z)
        zg.append(g.cpu().numpy().copy())
        tok = np.argmax(z, axis=-1)
    assert gm.sync_status() == 0
    assert cache.length() == n_ctx + 6
    compare(np.array(zg), np.array(zr), f"synthetic {kv_mode}")
