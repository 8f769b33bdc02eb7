"""Allocation-free decode step (dory_decode_step_static).

Some callers cannot call cudaMalloc -- code running under an allocator that
owns all device memory, or a process that must not grow its device footprint
once serving -- so they cannot hand dory_decode_step a workspace.  The static
entry point takes its workspace from a library-owned device array instead.
This test drives it through the C ABI and checks that two decode calls in a
row give the same logits (bit for bit, and so within the parity tolerance)
and the same greedy tokens as dory_decode_step with a caller-allocated
workspace, and that they leave the device's free memory unchanged.  It is collected
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
    """Two static calls in a row give bit-identical logits and tokens to the
    workspace entry (the same kernels on the same inputs), after a larger
    batch has left other contents in the shared array, and the static calls
    change the device's free memory by nothing."""
    import looped_ngpt_b200 as lb
    lib = _lib.load()
    w = make_weights(TINY, seed=0)
    gm = lb.DoryModel(TINY, w, device="cuda:0")
    dev = "cuda:0"
    prompt = torch.from_numpy(make_prompt(TINY, 2, 30, seed=3)).to(dev)
    k, mode = 2, "last_loop"
    caches = [gm.new_cache(2, 64, 30, kv_mode=mode) for _ in range(3)]
    ws = gm.workspace(2, 30)
    for c in caches:
        gm.prefill(c, prompt, k, ws)
    V = TINY.vocab
    # a larger batch first, so that the array holds another call's words
    big = gm.new_cache(6, 8, 1, kv_mode=mode)
    tb = torch.arange(6, dtype=torch.int32, device=dev) * 37
    ab = torch.empty((6,), dtype=torch.int32, device=dev)
    zb = torch.empty((6, V), dtype=torch.float32, device=dev)
    assert lib.dory_decode_step_static(gm.handle, big.handle, _ptr(tb), 6, k,
                                       1, _ptr(zb), _ptr(ab), _stream()) == 0
    # warm-up on a spare cache: every kernel of the B=2 step is loaded
    toks0 = torch.tensor([5, 900], dtype=torch.int32, device=dev)
    zw = torch.empty((2, V), dtype=torch.float32, device=dev)
    aw = torch.empty((2,), dtype=torch.int32, device=dev)
    assert lib.dory_decode_step_static(gm.handle, caches[2].handle,
                                       _ptr(toks0), 2, k, 1, _ptr(zw),
                                       _ptr(aw), _stream()) == 0
    # outputs of both steps allocated up front
    toks = [toks0, torch.empty((2,), dtype=torch.int32, device=dev)]
    z_st = [torch.full((2, V), float("nan"), device=dev) for _ in range(2)]
    a_st = [torch.full((2,), -1, dtype=torch.int32, device=dev)
            for _ in range(2)]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for step in range(2):                      # two calls in a row
        assert lib.dory_decode_step_static(
            gm.handle, caches[1].handle, _ptr(toks[step]), 2, k, 1,
            _ptr(z_st[step]), _ptr(a_st[step]), _stream()) == 0
        if step == 0:
            toks[1].copy_(a_st[0])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "a static call allocated"
    assert lib.dory_sync_status(gm.handle, _stream()) == 0
    for step in range(2):
        z_ref = torch.empty((2, V), dtype=torch.float32, device=dev)
        a_ref = torch.empty((2,), dtype=torch.int32, device=dev)
        assert lib.dory_decode_step(
            gm.handle, caches[0].handle, _ptr(toks[step]), 2, k, 1,
            _ptr(z_ref), _ptr(a_ref), _ptr(ws), ws.numel(), _stream()) == 0
        torch.cuda.synchronize()
        assert lib.dory_sync_status(gm.handle, _stream()) == 0
        d = float((z_ref - z_st[step]).abs().max())
        assert d <= LOGIT_TOL, f"step {step}: max|dz| {d}"
        assert torch.equal(z_ref, z_st[step]), f"step {step}: not bit-equal"
        assert torch.equal(a_ref, a_st[step])
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
