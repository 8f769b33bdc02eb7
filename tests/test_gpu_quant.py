"""MXFP8 / NVFP4 weight-only models on the GPU.

* In-register weight decode is bit-exact against the oracle's decode of the
  same bytes (dequantised weights must match bit for bit).  NVFP4 is also
  run with block scales chosen by minimum squared error (the same format,
  other bytes).
* Quantised decode (prompt fed one token per call, k=2, last_loop) matches
  the oracle run on the same quantised bytes within the BF16 tolerances, and
  so do quantised prefill and decode batches over 8 (tensor-core path)."""
import numpy as np
import pytest
import torch

from oracle import quant
from oracle.model import Model
from synthetic import TINY, make_weights, make_prompt
from synthetic.quantize import quantize_weights
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["mxfp8", "nvfp4", "nvfp4_mse"])
def qmodel(request):
    import looped_ngpt_b200 as lb
    qw = quantize_weights(make_weights(TINY, seed=0), request.param)
    return request.param, qw, lb.DoryModel(TINY, qw, device="cuda:0")


@pytest.mark.parametrize("name,K", [("blk0.w_qkvg", 256), ("blk3.w_o", 256),
                                    ("blk5.w_gu", 256), ("blk7.w_down", 768)])
def test_dequant_bit_exact(qmodel, name, K):
    fmt, qw, gm = qmodel
    q, s = qw[name + ".q"], qw[name + ".s"]
    if fmt == "mxfp8":
        ref = quant.dequant_mxfp8(q, s)
    else:
        ref = quant.dequant_nvfp4(q, s)          # tensor scale applied later
    N = ref.shape[0]
    got = gm.debug_dequant(name, 0, N, K).cpu().numpy()
    assert got.dtype == np.float32
    assert np.array_equal(got.astype(np.float64), ref)


def test_quantised_decode_matches_oracle(qmodel):
    fmt, qw, gm = qmodel
    prompt = make_prompt(TINY, 2, 12, seed=4)[:, :]
    ref = Model(TINY, qw, batch=2, kv_mode="last_loop")
    cache = gm.new_cache(2, 32, 1, kv_mode="last_loop")
    ws = gm.workspace(2, 1)
    zr, zg = [], []
    for t in range(prompt.shape[1]):
        zr.append(ref.decode_step(prompt[:, t], 2))
        g, _ = gm.decode_step(cache, torch.from_numpy(prompt[:, t].copy()).cuda(),
                              2, ws)
        zg.append(g.cpu().numpy().copy())
    assert gm.sync_status() == 0
    compare(np.array(zg), np.array(zr), f"{fmt} decode")


def test_quantised_prefill_and_batch_over_8(qmodel):
    """Multi-token calls and batches over 8 run the tensor-core GEMM on the
    projection dequantised to bf16 (exact) just before it, with the NVFP4
    tensor scale applied to the products: a 20-token prompt per sequence
    (every position compared) and two teacher-forced decode steps at B = 10,
    k = 2, per_loop."""
    fmt, qw, gm = qmodel
    B, T, k = 10, 20, 2
    prompt = make_prompt(TINY, B, T, seed=17)
    ref = Model(TINY, qw, batch=B, kv_mode="per_loop")
    zr = ref.forward(prompt, k, all_logits=True)
    cache = gm.new_cache(B, 32, T, kv_mode="per_loop", max_loops=k)
    ws = gm.workspace(B, T)
    zg, _ = gm.prefill(cache, torch.from_numpy(prompt).cuda(), k, ws,
                       logits_all=True)
    zg = zg.cpu().numpy()
    tok = np.argmax(zr[:, -1], -1)
    dr, dg = [], []
    for _ in range(2):
        dr.append(ref.decode_step(tok, k))
        g, _ = gm.decode_step(cache, torch.from_numpy(tok.astype(np.int32)).cuda(),
                              k, ws)
        dg.append(g.cpu().numpy().copy())
        tok = np.argmax(dr[-1], -1)
    assert gm.sync_status() == 0
    compare(zg, zr, f"{fmt} prefill B={B} T={T}")
    compare(np.array(dg), np.array(dr), f"{fmt} decode B={B}")
