"""Prefix caching and chunked prefill at 256K context (long-context serving;
MXFP8 explainer page, deployment section: contexts up to 256K).

* A prompt prefix prefilled once in one cache and copied into every
  sequence of another (dory_cache_copy_prefix) continues exactly like the
  oracle that ran prefix and suffix as two calls: suffix prefill (every
  position) and two decode steps, k = 2, both KV modes, prefix longer than
  the sliding window.  The copy refuses what it cannot provide.
* Chunked prefill at the end of a 256K context: the Dory widths with one
  input, one recurrent and one output block (sliding window, full, sliding
  window), 261624 seeded synthetic cached tokens, then two 256-token chunks
  at k = 2, last_loop, reaching position 262143; every position of both
  chunks against the oracle given the same cache entries (RoPE angles near
  2^18 with base 1e7 on the full-attention block)."""
import numpy as np
import pytest
import torch

from oracle.model import Model
from synthetic import TINY, ModelShape, make_weights, make_prompt
from synthetic.kvgen import kv_rows
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    import looped_ngpt_b200 as lb
    w = make_weights(TINY, seed=0)
    return w, lb.DoryModel(TINY, w, device="cuda:0")


@pytest.mark.parametrize("kv_mode", ["per_loop", "last_loop"])
def test_prefix_copy_continues_like_two_calls(tiny, kv_mode):
    w, gm = tiny
    k, Tp, Ts = 2, 30, 10
    prefix = make_prompt(TINY, 1, Tp, seed=40)
    suffix = make_prompt(TINY, 2, Ts, seed=41)
    src = gm.new_cache(1, 64, Tp, kv_mode=kv_mode, max_loops=k)
    ws1 = gm.workspace(1, Tp)
    gm.prefill(src, torch.from_numpy(prefix).cuda(), k, ws1)
    for t in (3, 9, 27):                      # the source moves on
        gm.decode_step(src, torch.tensor([t], dtype=torch.int32,
                                         device="cuda"), k, ws1)
    dst = gm.new_cache(2, 64, Ts, kv_mode=kv_mode, max_loops=k)
    dst.copy_prefix_from(src, 0, Tp)
    assert dst.length() == Tp
    ws2 = gm.workspace(2, Ts)
    zg, _ = gm.prefill(dst, torch.from_numpy(suffix).cuda(), k, ws2,
                       logits_all=True)
    zg = zg.cpu().numpy()
    ref = Model(TINY, w, batch=2, kv_mode=kv_mode)
    ref.forward(np.repeat(prefix, 2, axis=0), k)
    zr = ref.forward(suffix, k, all_logits=True)
    tok = np.argmax(zr[:, -1], -1)
    dr, dg = [], []
    for _ in range(2):
        dr.append(ref.decode_step(tok, k))
        g, _ = gm.decode_step(dst, torch.from_numpy(tok.astype(np.int32)).cuda(),
                              k, ws2)
        dg.append(g.cpu().numpy().copy())
        tok = np.argmax(dr[-1], -1)
    assert gm.sync_status() == 0
    compare(zg, zr, f"prefix-cached suffix {kv_mode}")
    compare(np.array(dg), np.array(dr), f"prefix-cached decode {kv_mode}")


def test_prefix_copy_refusals(tiny):
    import looped_ngpt_b200 as lb
    w, gm = tiny
    ws = gm.workspace(1, 8)
    src = gm.new_cache(1, 128, 8, kv_mode="last_loop")
    for c in range(12):                       # 96 tokens; ring of 64 slots
        gm.prefill(src, torch.from_numpy(make_prompt(TINY, 1, 8, seed=c)).cuda(),
                   1, ws)
    dst = gm.new_cache(2, 128, 8, kv_mode="last_loop")
    other = gm.new_cache(2, 128, 8, kv_mode="per_loop", max_loops=1)
    for cache, n, code in ((dst, 97, -3),     # past the source's length
                           (other, 40, -3),   # another KV mode
                           (dst, 20, -3)):    # ring slots already reused
        with pytest.raises(lb.DoryError) as e:
            cache.copy_prefix_from(src, 0, n)
        assert e.value.code == code
    dst.copy_prefix_from(src, 0, 90)          # still held by the ring
    assert dst.length() == 90
    assert gm.sync_status() == 0


LSHAPE = ModelShape(name="dory-widths-1-1-1-v8192", d=2560, n_q_heads=16,
                    n_kv_heads=4, head_dim=160, ffn=10240, vocab=8192,
                    n_in=1, n_rec=1, n_out=1, swa_window=1024,
                    layer_types=(0, 1, 0))


def test_chunked_prefill_at_256k_context():
    import looped_ngpt_b200 as lb
    k, chunk, n_chunks, seed = 2, 256, 2, 2
    max_ctx = 1 << 18
    n_ctx = max_ctx - n_chunks * chunk - 8
    w = make_weights(LSHAPE, seed=0)
    gm = lb.DoryModel(LSHAPE, w, device="cuda:0")
    cache = gm.new_cache(1, max_ctx, chunk, kv_mode="last_loop")
    cache.fill_synthetic(n_ctx, seed)
    ws = gm.workspace(1, chunk)
    prompt = make_prompt(LSHAPE, 1, n_chunks * chunk, seed=44)
    zg = []
    for c in range(n_chunks):
        z, _ = gm.prefill(cache, torch.from_numpy(
            prompt[:, c * chunk:(c + 1) * chunk].copy()).cuda(), k, ws,
            logits_all=True)
        zg.append(z.cpu().numpy())
    assert gm.sync_status() == 0
    assert cache.length() == n_ctx + n_chunks * chunk
    del gm, cache, ws
    torch.cuda.empty_cache()
    ref = Model(LSHAPE, w, kv_mode="last_loop")
    H, hd, total = LSHAPE.n_kv_heads, LSHAPE.head_dim, n_ctx + n_chunks * chunk
    for i in range(LSHAPE.n_blocks):
        full = LSHAPE.layer_types[i] == 1
        lo = 0 if full else n_ctx - LSHAPE.swa_window
        pos = np.arange(lo, n_ctx)
        K = np.zeros((1, H, total, hd))
        V = np.zeros_like(K)
        for h in range(H):
            K[0, h, lo:n_ctx], V[0, h, lo:n_ctx] = kv_rows(LSHAPE, seed, i, 0, 0,
                                                          h, pos)
        ref.cache[(i, 0)] = (K, V)
    ref.n_ctx = n_ctx
    zr = [ref.forward(prompt[:, c * chunk:(c + 1) * chunk], k, all_logits=True)
          for c in range(n_chunks)]
    compare(np.concatenate(zg, 1), np.concatenate(zr, 1),
            f"chunked prefill at {n_ctx} cached tokens")
