"""The seeded quantised checkpoints (synthetic.quantize, used by bench.py)
are byte-identical to the oracle's own quantisers, and the oracle decodes a
quantised model (tiny shape) consistently with its BF16 original."""
import numpy as np
import pytest

from oracle import quant
from oracle.model import Model
from synthetic import TINY, make_weights, make_prompt
from synthetic.gen import bf16_bits_to_f32
from synthetic.quantize import encode_mxfp8, encode_nvfp4, quantize_weights


@pytest.fixture(scope="module")
def w():
    return make_weights(TINY, seed=0)


@pytest.mark.parametrize("name", ["blk0.w_qkvg", "blk3.w_down", "blk5.w_gu"])
def test_encoders_match_oracle_quantisers(w, name):
    m = bf16_bits_to_f32(w[name])
    q1, e1 = encode_mxfp8(m)
    q2, e2 = quant.quant_mxfp8(m)
    assert np.array_equal(q1, q2) and np.array_equal(e1, e2)
    p1, s1, t1 = encode_nvfp4(m)
    p2, s2, t2 = quant.quant_nvfp4(m)
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)
    assert np.float32(t1[0]) == np.float32(t2)


@pytest.mark.parametrize("name", ["blk0.w_qkvg", "blk3.w_down"])
def test_mse_encoder_matches_oracle(w, name):
    from synthetic.quantize import _encode_rows
    m = bf16_bits_to_f32(w[name])
    p1, s1, t1 = _encode_rows(m, "nvfp4_mse", rows=100)
    p2, s2, t2 = quant.quant_nvfp4_mse(m)
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)
    assert np.float32(t1[0]) == np.float32(t2)


@pytest.mark.parametrize("fmt,tol", [("mxfp8", 0.05), ("nvfp4", 0.35),
                                     ("nvfp4_mse", 0.35)])
def test_quantised_model_close_to_bf16(w, fmt, tol):
    """Weight-only quantisation perturbs the logits by a bounded amount
    (E4M3: ~2^-4 relative per weight; E2M1 much coarser)."""
    qw = quantize_weights(w, fmt)
    assert "blk0.w_qkvg" not in qw and "blk0.w_qkvg.q" in qw
    assert "embed" in qw and "lm_head" in qw
    toks = make_prompt(TINY, 1, 6)
    z0 = Model(TINY, w).forward(toks, 2)
    z1 = Model(TINY, qw).forward(toks, 2)
    rel = np.linalg.norm(z1 - z0) / np.linalg.norm(z0)
    assert 0 < rel < tol, rel
