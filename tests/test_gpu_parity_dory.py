"""GPU vs oracle at the full Dory1.0-4B shape (d=2560, 16/4 heads of 160,
blocks 8/20/8, SwiGLU 10240, vocab 131072), seeded random-init BF16 weights.

Sampled cases the float64 oracle finishes in a few minutes on the host:
  * an 8-token prompt at k=2 (last_loop) plus 3 teacher-forced decode steps,
    every prompt position compared (GEMV decode path, tensor-core prefill);
  * a 1040-token prompt at k=1 (longer than the 1024-token window, so the
    sliding-window mask, ring and paged cache are exercised at full size),
    the last 8 positions compared.
Bounds as for the tiny model: max |dlogits| <= 3e-2, valid greedy picks,
| ||s|| - 1 | <= 2e-3."""
import numpy as np
import pytest
import torch

from synthetic import DORY, make_weights, make_prompt
from tests.gpu_util import compare, NORM_TOL
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
    compare(gp.cpu().numpy()[:, -8:], zp[:, -8:], "dory long prefill")
    assert np.abs(np.linalg.norm(s, axis=-1) - 1).max() <= NORM_TOL
