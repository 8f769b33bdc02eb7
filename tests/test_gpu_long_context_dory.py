"""Decode over seeded synthetic cached context at the full Dory1.0-4B shape,
in the launch configuration bench.py times for long context: B=64 sequences,
k=2, per_loop and last_loop (one 16-block cluster per (sequence, KV head) in
the decode attention, split-K tensor-core GEMMs for the batch-64
projections).

  * 4096 cached tokens: sequences 0 and 63 against the float64 oracle given
    the same cache entries (synthetic.kvgen), one decode step: the logits
    bound and valid greedy picks.  At 4096 tokens every cluster block holds
    several key tiles and the 1024-token sliding-window rings have wrapped.
    (The oracle keeps float64 caches for every slot; at 32768 tokens that
    would be about 19 GB of host memory per sampled sequence.)
  * 32768 cached tokens (the bench size): properties that hold at any size,
    for all 64 sequences: finite logits, unit-norm final states, valid
    greedy picks, a clean device status and the cache length advanced."""
import numpy as np
import pytest
import torch

from oracle.model import Model
from synthetic import DORY, make_weights
from synthetic.kvgen import kv_rows
from tests.gpu_util import compare, NORM_TOL

pytestmark = pytest.mark.gpu

B, K_LOOPS, SEED = 64, 2, 2


@pytest.fixture(scope="module")
def dory_long():
    import looped_ngpt_b200 as lb
    w = make_weights(DORY, seed=0)
    return w, lb.DoryModel(DORY, w, device="cuda:0")


def oracle_for(w, seqs, n_ctx, kv_mode="per_loop"):
    """Oracle model whose batch rows are the sampled sequences `seqs`, each
    slot's cache filled with that sequence's synthetic entries (the
    generator's slot index is the loop t for per_loop recurrent blocks, 0
    for every single-slot block)."""
    m = Model(DORY, w, batch=len(seqs), kv_mode=kv_mode)
    _, grec, _ = DORY.block_groups()
    pos = np.arange(n_ctx)
    for i in range(DORY.n_blocks):
        per_loop = i in grec and kv_mode == "per_loop"
        for s in (range(1, K_LOOPS + 1) if per_loop else [0]):
            Kc = np.zeros((len(seqs), DORY.n_kv_heads, n_ctx, DORY.head_dim))
            Vc = np.zeros_like(Kc)
            for r, b in enumerate(seqs):
                for h in range(DORY.n_kv_heads):
                    Kc[r, h], Vc[r, h] = kv_rows(DORY, SEED, i, s, b, h, pos)
            m.cache[(i, s)] = (Kc, Vc)
    m.n_ctx = n_ctx
    return m


def gpu_step(gm, n_ctx, tok, kv_mode="per_loop"):
    cache = gm.new_cache(B, n_ctx + 8, 1, kv_mode=kv_mode, max_loops=K_LOOPS)
    cache.fill_synthetic(n_ctx, SEED)
    ws = gm.workspace(B, 1)
    z, a = gm.decode_step(cache, torch.from_numpy(tok).cuda(), K_LOOPS, ws)
    s = gm.copy_state(ws, B, 1)
    torch.cuda.synchronize()
    out = (z.cpu().numpy(), a.cpu().numpy(), s.cpu().numpy(), cache.length(),
           gm.sync_status())
    del cache, ws, z, a, s
    torch.cuda.empty_cache()
    return out


@pytest.mark.parametrize("kv_mode", ["per_loop", "last_loop"])
def test_b64_ctx4k_sampled_sequences_match_oracle(dory_long, kv_mode):
    w, gm = dory_long
    n_ctx = 4096
    tok = np.random.default_rng(7).integers(0, DORY.vocab, size=B).astype(np.int32)
    z, a, s, length, status = gpu_step(gm, n_ctx, tok, kv_mode)
    assert status == 0 and length == n_ctx + 1
    seqs = [0, B - 1]
    ref = oracle_for(w, seqs, n_ctx, kv_mode)
    zr = ref.decode_step(tok[seqs], K_LOOPS)
    compare(z[seqs], zr, f"dory B=64 ctx 4096 {kv_mode} sampled")
    assert np.array_equal(a, np.argmax(z, -1))
    assert np.abs(np.linalg.norm(s, axis=-1) - 1).max() <= NORM_TOL


def test_b64_ctx32k_properties(dory_long):
    _, gm = dory_long
    n_ctx = 32768
    tok = np.random.default_rng(8).integers(0, DORY.vocab, size=B).astype(np.int32)
    z, a, s, length, status = gpu_step(gm, n_ctx, tok)
    assert status == 0 and length == n_ctx + 1
    assert np.isfinite(z).all()
    assert np.array_equal(a, np.argmax(z, -1))
    assert np.abs(np.linalg.norm(s, axis=-1) - 1).max() <= NORM_TOL
