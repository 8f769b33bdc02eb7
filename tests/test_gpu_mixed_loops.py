"""Mixed loop counts in one batch (elastic depth per request; paper
summary, 研究动机 / 核心方法: one checkpoint, the loop count chosen per
request): every sequence of a batch computes what a call with its own loop
count computes.  Tiny model, loop counts (1, 4, 2) at batch 3 (decode
GEMV path) and a 10-sequence batch cycling 1..4 (tensor-core GEMM path),
both KV modes: a 16-token mixed prefill (every position) and three
teacher-forced mixed decode steps, each sequence against an oracle run with
its own loop count."""
import numpy as np
import pytest
import torch

from oracle.model import Model
from synthetic import TINY, make_weights, make_prompt
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    import looped_ngpt_b200 as lb
    w = make_weights(TINY, seed=0)
    return w, lb.DoryModel(TINY, w, device="cuda:0")


@pytest.mark.parametrize("kv_mode", ["per_loop", "last_loop"])
@pytest.mark.parametrize("loops", [(1, 4, 2), (1, 2, 3, 4, 1, 2, 3, 4, 2, 1)])
def test_mixed_loop_counts_match_per_sequence_oracle(tiny, kv_mode, loops):
    w, gm = tiny
    B, T, steps = len(loops), 16, 3
    kmax = max(loops)
    prompt = make_prompt(TINY, B, T, seed=50)
    rl = torch.tensor(loops, dtype=torch.int32, device="cuda:0")
    cache = gm.new_cache(B, T + steps + 8, T, kv_mode=kv_mode, max_loops=kmax)
    ws = gm.workspace(B, T)
    zg, _ = gm.prefill_mixed(cache, torch.from_numpy(prompt).cuda(), rl, ws,
                             logits_all=True)
    zg = zg.cpu().numpy()
    refs = [Model(TINY, w, batch=1, kv_mode=kv_mode) for _ in range(B)]
    zr = np.concatenate([refs[b].forward(prompt[b:b + 1], loops[b], True)
                         for b in range(B)])
    tok = np.argmax(zr[:, -1], -1)
    dg, dr = [], []
    for _ in range(steps):
        dr.append(np.concatenate([refs[b].decode_step(tok[b:b + 1], loops[b])
                                  for b in range(B)]))
        g, _ = gm.decode_step_mixed(cache, torch.from_numpy(
            tok.astype(np.int32)).cuda(), rl, kmax, ws)
        dg.append(g.cpu().numpy().copy())
        tok = np.argmax(dr[-1], -1)
    assert gm.sync_status() == 0
    assert cache.length() == T + steps
    compare(zg, zr, f"mixed {loops} prefill {kv_mode}")
    compare(np.array(dg), np.array(dr), f"mixed {loops} decode {kv_mode}")
