"""Allocation-free decode step (dory_decode_step_static).

Some callers cannot call cudaMalloc -- code running under an allocator that
owns all device memory, or a process that must not grow its device footprint
once serving -- so they cannot hand dory_decode_step a workspace.  The static
entry point takes its workspace from a library-owned device array instead.
This test drives it through the C ABI and checks that two decode calls in a
row give the same logits (within the parity tolerance) and the same greedy
tokens as dory_decode_step with a caller-allocated workspace.  It is collected
last so that a stop-at-first-failure run has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

from looped_ngpt_b200 import _lib
from synthetic import TINY, make_weights, make_prompt
from tests.gpu_util import LOGIT_TOL

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _ptr(t):
    return P(t.data_ptr())


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def test_static_decode_matches_workspace_decode():
    import looped_ngpt_b200 as lb
    lib = _lib.load()
    w = make_weights(TINY, seed=0)
    gm = lb.DoryModel(TINY, w, device="cuda:0")
    prompt = torch.from_numpy(make_prompt(TINY, 2, 30, seed=3)).to("cuda:0")
    k, mode = 2, "last_loop"
    caches = [gm.new_cache(2, 64, 30, kv_mode=mode) for _ in range(2)]
    ws = gm.workspace(2, 30)
    for c in caches:
        gm.prefill(c, prompt, k, ws)
    V = TINY.vocab
    toks = torch.tensor([5, 900], dtype=torch.int32, device="cuda:0")
    for step in range(2):                      # two calls in a row
        z_ref = torch.empty((2, V), dtype=torch.float32, device="cuda:0")
        a_ref = torch.empty((2,), dtype=torch.int32, device="cuda:0")
        z_st = torch.full((2, V), float("nan"), device="cuda:0")
        a_st = torch.full((2,), -1, dtype=torch.int32, device="cuda:0")
        assert lib.dory_decode_step(
            gm.handle, caches[0].handle, _ptr(toks), 2, k, 1, _ptr(z_ref),
            _ptr(a_ref), _ptr(ws), ws.numel(), _stream()) == 0
        assert lib.dory_decode_step_static(
            gm.handle, caches[1].handle, _ptr(toks), 2, k, 1, _ptr(z_st),
            _ptr(a_st), _stream()) == 0
        torch.cuda.synchronize()
        assert lib.dory_sync_status(gm.handle, _stream()) == 0
        d = float((z_ref - z_st).abs().max())
        assert d <= LOGIT_TOL, f"step {step}: max|dz| {d}"
        assert torch.equal(a_ref, a_st)
        toks = a_ref.clone()
    assert caches[0].length() == caches[1].length() == 32


def test_static_decode_rejects_oversized_batch():
    import looped_ngpt_b200 as lb
    lib = _lib.load()
    gm = lb.DoryModel(TINY, make_weights(TINY, seed=0), device="cuda:0")
    limit = 8 << 20
    need = ctypes.c_int64()
    B = 2
    while True:
        assert lib.dory_workspace_bytes(gm.handle, B, 1, ctypes.byref(need)) == 0
        if need.value > limit:
            break
        B *= 2
    cache = gm.new_cache(B, 8, 1, kv_mode="last_loop")
    toks = torch.zeros((B,), dtype=torch.int32, device="cuda:0")
    out = torch.empty((B,), dtype=torch.int32, device="cuda:0")
    assert lib.dory_decode_step_static(gm.handle, cache.handle, _ptr(toks), B,
                                       1, 1, None, _ptr(out), _stream()) == -6
    assert cache.length() == 0
