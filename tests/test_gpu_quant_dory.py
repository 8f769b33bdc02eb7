"""MXFP8 / NVFP4 weight-only decode at the Dory1.0-4B widths (d 2560, 16/4
heads of 160, SwiGLU 10240), one input, one recurrent and one output block
(sliding window, full, sliding window), so that every projection shape of
the full model is exercised at a fraction of its size.

* The production decode GEMV (the kernel the forward pass launches, through
  dory_debug_gemv) multiplies the quantised weights by one-hot activation
  rows x = e_k: each output is weight (n, k) times its group scale (and the
  NVFP4 tensor scale), rounded once to f32, and must equal the oracle's
  decode of the same bytes bit for bit (MXFP8 explainer page, deployment
  section: E4M3 values with an E8M0 scale per 32 weights; paper summary,
  前置知识: NVFP4 = E2M1 values with E4M3 block scales), at K = 2560 and
  K = 10240, for batch rows 1, 2, 4 and 8.
* A 1100-token prefill at k = 2 through the tensor-core path (projections
  dequantised to bf16 just before each GEMM), every position compared.
* Batch-4 decode at k = 2, last_loop, after a seeded synthetic context of
  131000 cached tokens (the long-context quantised workload: RoPE angles at
  positions near 131072, base 1e7 on the full-attention block), sequences 0
  and 3 against the oracle given the same cache entries, two steps."""
import numpy as np
import pytest
import torch

from oracle import quant
from oracle.model import Model
from synthetic import ModelShape, make_weights
from synthetic.kvgen import kv_rows
from synthetic.quantize import quantize_weights
from tests.gpu_util import compare, NORM_TOL

pytestmark = pytest.mark.gpu

QSHAPE = ModelShape(name="dory-widths-1-1-1", d=2560, n_q_heads=16,
                    n_kv_heads=4, head_dim=160, ffn=10240, vocab=8192,
                    n_in=1, n_rec=1, n_out=1, swa_window=1024,
                    layer_types=(0, 1, 0))


@pytest.fixture(scope="module")
def bf16_weights():
    return make_weights(QSHAPE, seed=0)


@pytest.fixture(scope="module", params=["mxfp8", "nvfp4"])
def qmodel(request, bf16_weights):
    import looped_ngpt_b200 as lb
    qw = quantize_weights(bf16_weights, request.param)
    return request.param, qw, lb.DoryModel(QSHAPE, qw, device="cuda:0")


def _columns(K, rng):
    ks = list(range(32)) + list(range(K - 8, K))
    rest = rng.choice(np.arange(32, K - 8), size=24, replace=False)
    return np.array(ks + sorted(rest.tolist()))


def _expected(fmt, qw, name):
    """Oracle decode of the stored bytes, rounded the way the GEMV rounds:
    MXFP8 e4m3 * 2^(e8m0 - 127) is exact in f32; NVFP4 (e2m1 * e4m3) is
    exact and the f32 tensor scale is applied by one rounded multiply."""
    q, s = qw[name + ".q"], qw[name + ".s"]
    if fmt == "mxfp8":
        return quant.dequant_mxfp8(q, s).astype(np.float32)
    w = quant.dequant_nvfp4(q, s).astype(np.float32)
    return w * np.float32(qw[name + ".t"][0])


@pytest.mark.parametrize("name,K", [("blk0.w_qkvg", 2560), ("blk1.w_o", 2560),
                                    ("blk2.w_gu", 2560), ("blk1.w_down", 10240)])
def test_production_gemv_decode_bit_exact(qmodel, name, K):
    fmt, qw, gm = qmodel
    ref = _expected(fmt, qw, name)
    assert ref.shape[1] == K
    cols = _columns(K, np.random.default_rng(K))
    one = np.uint16(0x3F80)                       # bf16 1.0
    groups, i = [], 0
    for B in (1, 2, 4) + (8,) * ((len(cols) - 7 + 7) // 8):
        if i >= len(cols):
            break
        groups.append(cols[i:i + B])
        i += B
    for g in groups:
        x = np.zeros((len(g), K), dtype=np.uint16)
        x[np.arange(len(g)), g] = one
        dx = torch.from_numpy(x.view(np.int16)).to("cuda:0")
        parts = gm.debug_gemv(name, dx).cpu().numpy().astype(np.float64)
        got = parts.sum(0).astype(np.float32)        # other slabs are 0
        want = ref[:, g].T
        assert got.shape == want.shape
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (f"{fmt} {name} columns {g.tolist()}: "
                               f"{bad.size} weights differ, first "
                               f"{got.flat[bad[0]]!r} vs {want.flat[bad[0]]!r}")
    assert gm.sync_status() == 0


def _oracle_with_context(qw, seqs, n_ctx, extra, seed):
    m = Model(QSHAPE, qw, batch=len(seqs), kv_mode="last_loop")
    hd, H = QSHAPE.head_dim, QSHAPE.n_kv_heads
    for i in range(QSHAPE.n_blocks):
        full = QSHAPE.layer_types[i] == 1
        lo = 0 if full else n_ctx - QSHAPE.swa_window
        pos = np.arange(lo, n_ctx)
        K = np.zeros((len(seqs), H, n_ctx + extra, hd))
        V = np.zeros_like(K)
        for r, b in enumerate(seqs):
            for h in range(H):
                K[r, h, lo:n_ctx], V[r, h, lo:n_ctx] = kv_rows(
                    QSHAPE, seed, i, 0, b, h, pos)
        m.cache[(i, 0)] = (K, V)
    m.n_ctx = n_ctx
    return m


def test_quantised_decode_at_131k_context(qmodel):
    fmt, qw, gm = qmodel
    B, n_ctx, k, seed, steps = 4, 131000, 2, 2, 2
    seqs = [0, B - 1]
    cache = gm.new_cache(B, n_ctx + 8, 1, kv_mode="last_loop")
    cache.fill_synthetic(n_ctx, seed)
    ws = gm.workspace(B, 1)
    toks = np.random.default_rng(21).integers(0, QSHAPE.vocab,
                                              size=(steps, B)).astype(np.int32)
    zg, sg = [], []
    for j in range(steps):
        z, _ = gm.decode_step(cache, torch.from_numpy(toks[j]).cuda(), k, ws)
        zg.append(z.cpu().numpy()[seqs])
        sg.append(gm.copy_state(ws, B, 1).cpu().numpy())
    assert gm.sync_status() == 0
    assert cache.length() == n_ctx + steps
    del cache, ws
    torch.cuda.empty_cache()
    ref = _oracle_with_context(qw, seqs, n_ctx, steps, seed)
    zr = [ref.decode_step(toks[j][seqs], k) for j in range(steps)]
    compare(np.array(zg), np.array(zr), f"{fmt} B=4 ctx 131000")
    assert max(np.abs(np.linalg.norm(s, axis=-1) - 1).max() for s in sg) <= NORM_TOL


def test_quantised_prefill_dory_widths(qmodel):
    """A 1100-token prompt (across the 1024-token window) at k = 2, per_loop,
    through the tensor-core path with dequantised projections: every
    position against the oracle on the same quantised bytes."""
    from synthetic import make_prompt
    fmt, qw, gm = qmodel
    T, k = 1100, 2
    prompt = make_prompt(QSHAPE, 1, T, seed=23)
    cache = gm.new_cache(1, T + 8, T, kv_mode="per_loop", max_loops=k)
    ws = gm.workspace(1, T)
    zg, _ = gm.prefill(cache, torch.from_numpy(prompt).cuda(), k, ws,
                       logits_all=True)
    zg = zg.cpu().numpy()
    assert gm.sync_status() == 0
    del cache, ws
    torch.cuda.empty_cache()
    zr = Model(QSHAPE, qw, kv_mode="per_loop").forward(prompt, k, True)
    compare(zg, zr, f"{fmt} prefill T={T} Dory widths")


@pytest.mark.parametrize("B", [2, 3, 4, 8])
@pytest.mark.parametrize("name", ["blk0.w_qkvg", "blk1.w_o", "blk2.w_gu",
                                  "blk1.w_down"])
def test_bf16_batched_gemv_matches_float64(bf16_weights, name, B):
    """The BF16 decode GEMV for 2..8 activation rows (whole-row projections
    on the warp MMA, the 8 weight rows of a stage as the MMA columns; the
    K-split down projection on the SIMT loop) against a float64 product of
    the same bf16 values."""
    import looped_ngpt_b200 as lb
    from synthetic.gen import bf16_bits_to_f32, f32_to_bf16_bits
    gm = lb.DoryModel(QSHAPE, bf16_weights, device="cuda:0")
    W = bf16_bits_to_f32(bf16_weights[name]).astype(np.float64)
    K = W.shape[1]
    rng = np.random.default_rng(B * 7 + K)
    x = f32_to_bf16_bits(rng.standard_normal((B, K)).astype(np.float32) /
                         np.float32(np.sqrt(K)))
    dx = torch.from_numpy(x.view(np.int16)).to("cuda:0")
    got = gm.debug_gemv(name, dx).cpu().numpy().astype(np.float64).sum(0)
    want = bf16_bits_to_f32(x).astype(np.float64) @ W.T
    assert gm.sync_status() == 0
    tol = 2e-5 * np.sqrt(K) * (np.abs(want).max() + 1e-3)
    assert np.abs(got - want).max() <= tol, np.abs(got - want).max()
