"""GPU vs oracle at the full Dory1.0-4B shape (d=2560, 16/4 heads of 160,
blocks 8/20/8, SwiGLU 10240, vocab 131072), seeded random-init BF16 weights.

Sampled cases the float64 oracle finishes in a few minutes on the host:
  * an 8-token prompt at k=2 (last_loop) plus 3 teacher-forced decode steps,
    every prompt position compared (GEMV decode path, tensor-core prefill);
  * a 1040-token prompt at k=1 (longer than the 1024-token window, so the
    sliding-window mask, ring and paged cache are exercised at full size),
    every position compared and raw top-1 agreement >= 99.5% gated;
  * k=4 (192 sublayers) in both KV modes: a 1040-token prompt and two
    teacher-forced decode steps (raw top-1 gated at 99%: every
    disagreement must still be a valid greedy pick).
Bounds as for the tiny model: max |dlogits| <= 3e-2, valid greedy picks,
| ||s|| - 1 | <= 2e-3."""
import numpy as np
import pytest
import torch

from synthetic import DORY, make_weights, make_prompt
from tests.gpu_util import compare, NORM_TOL, TOP1_MIN

TOP1_MIN_DEEP = 0.99     # raw top-1 gate at k = 4 (see the test)
from oracle.model import Model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dory():
    import looped_ngpt_b200 as lb
    w = make_weights(DORY, seed=0)
    return w, lb.DoryModel(DORY, w, device="cuda:0")


def test_dory_short_prompt_k2_decode(dory):
    w, gm = dory
    prompt = make_prompt(DORY, 1, 8, seed=5)
    ref = Model(DORY, w, kv_mode="last_loop")
    zp = ref.forward(prompt, 2, all_logits=True)
    toks, zd = [], []
    nxt = int(np.argmax(zp[0, -1]))
    for _ in range(3):
        toks.append(nxt)
        z = ref.decode_step([nxt], 2)
        zd.append(z)
        nxt = int(np.argmax(z[0]))
    cache = gm.new_cache(1, 64, 8, kv_mode="last_loop")
    ws = gm.workspace(1, 8)
    t = torch.from_numpy(prompt).to("cuda:0")
    gp, _ = gm.prefill(cache, t, 2, ws, logits_all=True)
    gp = gp.cpu().numpy()
    gd, norms = [], []
    for tk in toks:
        z, _ = gm.decode_step(cache, torch.tensor([tk], dtype=torch.int32,
                                                  device="cuda:0"), 2, ws)
        gd.append(z.cpu().numpy())
        norms.append(np.linalg.norm(gm.copy_state(ws, 1, 1).cpu().numpy()))
    assert gm.sync_status() == 0
    compare(gp, zp, "dory prefill")
    compare(np.array(gd), np.array(zd), "dory decode")
    assert max(abs(n - 1) for n in norms) <= NORM_TOL


def test_dory_prompt_longer_than_window_k1(dory):
    w, gm = dory
    T = DORY.swa_window + 16
    prompt = make_prompt(DORY, 1, T, seed=6)
    ref = Model(DORY, w, kv_mode="per_loop")
    zp = ref.forward(prompt, 1, all_logits=True)
    cache = gm.new_cache(1, T + 8, T, kv_mode="per_loop", max_loops=1)
    ws = gm.workspace(1, T)
    gp, _ = gm.prefill(cache, torch.from_numpy(prompt).to("cuda:0"), 1, ws,
                       logits_all=True)
    s = gm.copy_state(ws, 1, T, logits_all=True).cpu().numpy()
    assert gm.sync_status() == 0
    _, agree, n = compare(gp.cpu().numpy(), zp, "dory long prefill")
    assert np.abs(np.linalg.norm(s, axis=-1) - 1).max() <= NORM_TOL
    assert agree / n >= TOP1_MIN, f"top-1 agreement {agree}/{n}"


def _last_loop_from_per_loop(pl, k):
    """Oracle in last_loop mode holding what a last_loop prefill leaves: every
    recurrent layer's single cache holds the final loop's entries, the other
    layers' caches are unchanged.  One prefill call gives the same states in
    both modes (the pinned oracle properties "last_loop prefill logits equal
    per_loop" and "last_loop decode reads final-loop entries")."""
    ll = Model(DORY, pl.w, kv_mode="last_loop")
    _, grec, _ = DORY.block_groups()
    for (i, slot), (K, V) in pl.cache.items():
        if i not in grec or slot == k:
            ll.cache[(i, 0)] = (K.copy(), V.copy())
    ll.n_ctx = pl.n_ctx
    return ll


def test_dory_k4_prompt_and_decode_both_modes(dory):
    """k = 4 (192 sublayers) at the full shape: a 1040-token prompt (across
    the 1024-token window; every position compared, raw top-1 gated) and
    two teacher-forced decode steps in each KV mode (last_loop decode reads
    the final loop's entries of the prompt, per_loop each loop's own)."""
    w, gm = dory
    T, k, steps = DORY.swa_window + 16, 4, 2
    prompt = make_prompt(DORY, 1, T, seed=8)
    pl = Model(DORY, w, kv_mode="per_loop")
    zp = pl.forward(prompt, k, all_logits=True)
    refs = {"per_loop": pl, "last_loop": _last_loop_from_per_loop(pl, k)}
    for kv_mode, ref in refs.items():
        toks, zd = [], []
        nxt = int(np.argmax(zp[0, -1]))
        for _ in range(steps):
            toks.append(nxt)
            z = ref.decode_step([nxt], k)
            zd.append(z)
            nxt = int(np.argmax(z[0]))
        cache = gm.new_cache(1, T + 8, T, kv_mode=kv_mode, max_loops=k)
        ws = gm.workspace(1, T)
        gp, _ = gm.prefill(cache, torch.from_numpy(prompt).to("cuda:0"), k, ws,
                           logits_all=True)
        gp = gp.cpu().numpy()
        gd, norms = [], []
        for tk in toks:
            z, _ = gm.decode_step(cache, torch.tensor(
                [tk], dtype=torch.int32, device="cuda:0"), k, ws)
            gd.append(z.cpu().numpy().copy())
            norms.append(np.linalg.norm(gm.copy_state(ws, 1, 1).cpu().numpy()))
        assert gm.sync_status() == 0
        _, agree, n = compare(gp, zp, f"dory k=4 {kv_mode} prefill")
        compare(np.array(gd), np.array(zd), f"dory k=4 {kv_mode} decode")
        assert max(abs(x - 1) for x in norms) <= NORM_TOL
        # compare() already forces agreement wherever the oracle's top two
        # logits are more than the logit tolerance apart; at 192 sublayers
        # the logit error (~1.4e-2) exceeds more near-ties of 131072
        # random-init logits, and raw agreement measures 99.2%
        assert agree / n >= TOP1_MIN_DEEP, f"top-1 agreement {agree}/{n}"
        del cache, ws
        torch.cuda.empty_cache()
