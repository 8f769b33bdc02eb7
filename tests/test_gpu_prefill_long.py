"""Prefill parity in the launch configuration of the long-prompt benchmark:
one 8192-token uniform-random prompt at k = 4 loops, per_loop KV cache, the
Dory1.0-4B widths (d 2560, 16/4 heads of 160, SwiGLU 10240) with one input,
one recurrent and one output block (sliding window, full, sliding window),
so that every tensor-core GEMM and prefill-attention launch has the shape it
has in the full model (M = 8192 rows, a 1024-token window band and a full
causal 8192 x 8192 triangle), at a depth the float64 oracle finishes in
about a minute.  The vocabulary is cut to 8192 rows so that every position's
logits can be compared; 309 positions are compared (every 32nd, both sides
of the 1024-token window edge, and the last), with the BF16 bounds:
max |dlogits| <= 3e-2, valid greedy picks, | ||s|| - 1 | <= 2e-3 at every
position."""
import numpy as np
import pytest
import torch

from oracle.model import Model
from synthetic import ModelShape, make_weights, make_prompt
from tests.gpu_util import compare, NORM_TOL

pytestmark = pytest.mark.gpu

PSHAPE = ModelShape(name="dory-widths-1-1-1-v8192", d=2560, n_q_heads=16,
                    n_kv_heads=4, head_dim=160, ffn=10240, vocab=8192,
                    n_in=1, n_rec=1, n_out=1, swa_window=1024,
                    layer_types=(0, 1, 0))


def test_t8192_k4_per_loop_prefill_matches_oracle():
    import looped_ngpt_b200 as lb
    T, k = 8192, 4
    w = make_weights(PSHAPE, seed=0)
    prompt = make_prompt(PSHAPE, 1, T)
    gm = lb.DoryModel(PSHAPE, w, device="cuda:0")
    cache = gm.new_cache(1, T + 16, T, kv_mode="per_loop", max_loops=k)
    ws = gm.workspace(1, T)
    gz, ga = gm.prefill(cache, torch.from_numpy(prompt).to("cuda:0"), k, ws,
                        logits_all=True)
    states = gm.copy_state(ws, 1, T, logits_all=True).cpu().numpy()
    pos = np.unique(np.concatenate([np.arange(0, T, 32),
                                    np.arange(1000, 1050), [T - 1]]))
    gz = gz.cpu().numpy()[:, pos]
    ga = ga.cpu().numpy()[:, pos]
    assert gm.sync_status() == 0
    del gm, cache, ws
    torch.cuda.empty_cache()
    assert np.array_equal(ga, np.argmax(gz, -1))
    assert np.abs(np.linalg.norm(states, axis=-1) - 1).max() <= NORM_TOL
    ref = Model(PSHAPE, w, kv_mode="per_loop")
    zr = ref.forward(prompt, k, all_logits=True)[:, pos]
    compare(gz, zr, f"T={T} k={k} per_loop prefill ({len(pos)} positions)")
