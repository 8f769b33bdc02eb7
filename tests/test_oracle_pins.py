"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/structure.json), closed forms, special cases,
invariants, or a brute-force restatement on tiny inputs.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import model as om
from synthetic import TINY, DORY, make_weights, make_prompt, tiny_with_blocks

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _golden():
    with open(os.path.join(GOLD, "structure.json")) as f:
        return json.load(f)


# ---------------------------------------------------------------- structure
def test_dory_shape_matches_printed_config():
    g = _golden()
    c = g["config"]["values"]
    assert DORY.d == c["hidden_size"]
    assert DORY.n_q_heads == c["num_attention_heads"]
    assert DORY.n_kv_heads == c["num_key_value_heads"]
    assert DORY.swa_window == c["sliding_window"]
    assert DORY.rope_theta_swa == c["rope_theta_swa"]
    assert DORY.rope_theta_full == c["rope_theta_full"]
    assert DORY.vocab == c["vocab"]
    assert DORY.n_q_heads * DORY.head_dim == DORY.d
    b = g["blocks"]["values"]
    assert (DORY.n_in, DORY.n_rec, DORY.n_out) == (b["input"], b["recurrent"],
                                                  b["output"])
    cnt = g["sublayer_counts"]["values"]
    assert sum(1 for t in DORY.layer_types if t == 0) == cnt["swa_attention"]
    assert sum(1 for t in DORY.layer_types if t == 1) == cnt["full_attention"]
    assert DORY.n_blocks == cnt["mlp"]


@pytest.mark.parametrize("k", [1, 2, 4])
def test_depth_is_32_plus_40k(k):
    """Effective depth printed on the pages: 72 / 112 / 192 sublayers."""
    want = _golden()["depth_by_loops"]["values"][str(k)]
    sh = tiny_with_blocks(8, 20, 8)
    m = om.Model(sh, make_weights(sh), batch=1)
    m.forward(make_prompt(sh, 1, 3), n_loops=k)
    assert m.sublayers == want == 32 + 40 * k


# ---------------------------------------------------------------- primitives
def test_l2n_unit_and_zero_guard():
    v = rng.standard_normal((5, 7))
    assert np.allclose(np.linalg.norm(om.l2n(v), axis=-1), 1.0)
    assert np.all(om.l2n(np.zeros(4)) == 0.0)
    assert np.allclose(om.l2n(np.array([3.0, 4.0])), [0.6, 0.8])


def test_rope_matches_complex_rotation():
    """Rotate-half RoPE == multiplying (v_i + i v_{i+h/2}) by e^{i p theta^(-2i/h)}."""
    h, theta = 8, 1.0e4
    v = rng.standard_normal((3, h))
    pos = np.array([0, 5, 1000])
    out = om.rope(v, pos, theta)
    z = v[:, :h // 2] + 1j * v[:, h // 2:]
    f = np.array([theta ** (-2.0 * i / h) for i in range(h // 2)])
    zr = z * np.exp(1j * pos[:, None] * f[None, :])
    assert np.allclose(out[:, :h // 2], zr.real)
    assert np.allclose(out[:, h // 2:], zr.imag)


def test_rope_norm_identity_relative():
    h = 16
    v = rng.standard_normal((4, h))
    pos = np.array([0, 3, 77, 130000])
    r = om.rope(v, pos, 1e7)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(v, axis=-1))
    assert np.allclose(om.rope(v[:1], [0], 1e4), v[:1])            # p = 0
    q, k = rng.standard_normal(h), rng.standard_normal(h)
    d1 = om.rope(q[None], [10], 1e4) @ om.rope(k[None], [4], 1e4).T
    d2 = om.rope(q[None], [106], 1e4) @ om.rope(k[None], [100], 1e4).T
    assert np.allclose(d1, d2)                                    # i - j only


def test_ngpt_update_special_cases():
    s = om.l2n(rng.standard_normal(6))
    h = rng.standard_normal(6)
    assert np.allclose(om.ngpt_update(s, h, np.zeros(6)), s)
    assert np.allclose(om.ngpt_update(s, h, np.ones(6)), om.l2n(h))
    a = np.full(6, 0.3)
    want = om.l2n(0.7 * s + 0.3 * om.l2n(h))                      # span form
    assert np.allclose(om.ngpt_update(s, h, a), want)
    # the result is invariant to the scale of h (the sublayer output is normalised)
    assert np.allclose(om.ngpt_update(s, 1e-3 * h, a), want)


def test_swiglu_closed_form():
    g = np.array([0.0, 1.0, -2.0])
    u = np.array([1.0, 2.0, 3.0])
    silu = np.array([0.0, 1.0 / (1.0 + np.exp(-1.0)),
                     -2.0 / (1.0 + np.exp(2.0))])
    want = silu * u / np.linalg.norm(silu * u)
    assert np.allclose(om.swiglu(g, u), want)


def test_inner_norm_cancels_under_update():
    """N(W N(m)) == N(W m): the norm before an output projection does not change
    the normalised sublayer output (used by the CUDA path, which skips it)."""
    W = rng.standard_normal((5, 9))
    m = rng.standard_normal(9) * 1e-3
    assert np.allclose(om.l2n(W @ om.l2n(m)), om.l2n(W @ m))


def test_greedy_lowest_index_on_ties():
    z = np.array([[0.1, 0.7, 0.7, 0.2], [1.0, 1.0, 1.0, 1.0]])
    assert list(om.greedy(z)) == [1, 0]


# ---------------------------------------------------------------- attention
def _rand_attn(Hq, Hkv, T, P, h):
    q = rng.standard_normal((Hq, T, h))
    K = rng.standard_normal((Hkv, P, h))
    V = rng.standard_normal((Hkv, P, h))
    return q, K, V


@pytest.mark.parametrize("window", [0, 3, 6])
def test_attention_equals_bruteforce(window):
    q, K, V = _rand_attn(4, 2, 5, 9, 6)
    qp = np.arange(4, 9)
    kp = np.arange(9)
    a = om.attention(q, K, V, qp, kp, window, 0.7)
    b = om.attention_bruteforce(q, K, V, qp, kp, window, 0.7)
    assert np.allclose(a, b)


def test_attention_single_key_returns_value():
    q, K, V = _rand_attn(2, 1, 1, 1, 4)
    out = om.attention(q, K, V, [0], [0], 0, 3.0)
    assert np.allclose(out[0, 0], V[0, 0]) and np.allclose(out[1, 0], V[0, 0])


def test_attention_uniform_scores_average_values():
    """Equal scores (q = 0) give the mean of the visible values; with a window
    of W only the last W keys count."""
    V = rng.standard_normal((1, 6, 3))
    K = rng.standard_normal((1, 6, 3))
    q = np.zeros((1, 1, 3))
    out = om.attention(q, K, V, [5], np.arange(6), 0, 1.0)
    assert np.allclose(out[0, 0], V[0].mean(axis=0))
    out = om.attention(q, K, V, [5], np.arange(6), 2, 1.0)
    assert np.allclose(out[0, 0], V[0, 4:6].mean(axis=0))


def test_swa_equals_full_when_short():
    q, K, V = _rand_attn(4, 2, 7, 7, 5)
    p = np.arange(7)
    assert np.allclose(om.attention(q, K, V, p, p, 7, 1.1),
                       om.attention(q, K, V, p, p, 0, 1.1))
    assert not np.allclose(om.attention(q, K, V, p, p, 3, 1.1),
                           om.attention(q, K, V, p, p, 0, 1.1))


def test_gqa_with_replicated_kv_equals_mha():
    q, K, V = _rand_attn(4, 2, 3, 5, 6)
    p, kp = np.arange(2, 5), np.arange(5)
    Kr, Vr = np.repeat(K, 2, axis=0), np.repeat(V, 2, axis=0)
    assert np.allclose(om.attention(q, K, V, p, kp, 0, 0.5),
                       om.attention(q, Kr, Vr, p, kp, 0, 0.5))
    # head j uses kv head j // 2: swapping kv heads swaps output head pairs
    sw = om.attention(q[[2, 3, 0, 1]], K[[1, 0]], V[[1, 0]], p, kp, 0, 0.5)
    assert np.allclose(sw, om.attention(q, K, V, p, kp, 0, 0.5)[[2, 3, 0, 1]])


# ---------------------------------------------------------------- full model
@pytest.fixture(scope="module")
def tiny_w():
    return make_weights(TINY, seed=0)


def test_every_state_is_unit_norm(tiny_w):
    seen = []
    m = om.Model(TINY, tiny_w, batch=2, trace=lambda k, i, s: seen.append(s))
    m.forward(make_prompt(TINY, 2, 20), n_loops=2)
    assert len(seen) > 20
    for s in seen:
        assert np.allclose(np.linalg.norm(s, axis=-1), 1.0, atol=1e-12)


def test_k1_equals_plain_stack(tiny_w):
    """At k=1, u_1 = N(s_0 + x) = N(2x) = x, so the looped model is the plain
    36-block-style stack input -> recurrent -> output."""
    toks = make_prompt(TINY, 1, 24)
    z1 = om.Model(TINY, tiny_w).forward(toks, 1, all_logits=True)
    m = om.Model(TINY, tiny_w)
    T = toks.shape[1]
    pos = np.arange(T)
    s = om.l2n(m.rows("embed", toks))
    for i in range(TINY.n_blocks):
        s = m.block(i, s, pos, 1)
    z2 = m.lm_head(s)
    assert np.allclose(z1, z2, atol=1e-10)


def test_loop_count_changes_result(tiny_w):
    toks = make_prompt(TINY, 1, 8)
    z1 = om.Model(TINY, tiny_w).forward(toks, 1)
    z2 = om.Model(TINY, tiny_w).forward(toks, 2)
    assert not np.allclose(z1, z2)


def test_last_loop_equals_per_loop_at_k1(tiny_w):
    toks = make_prompt(TINY, 1, 30)
    a = om.Model(TINY, tiny_w, kv_mode="per_loop")
    b = om.Model(TINY, tiny_w, kv_mode="last_loop")
    za, zb = a.forward(toks, 1), b.forward(toks, 1)
    for t in [5, 9, 1]:
        za = np.concatenate([za, a.decode_step([t], 1)[:, None]], axis=1)
        zb = np.concatenate([zb, b.decode_step([t], 1)[:, None]], axis=1)
    assert np.array_equal(za, zb)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_last_loop_footprint_is_k1_size(tiny_w, k):
    toks = make_prompt(TINY, 1, 10)
    m = om.Model(TINY, tiny_w, kv_mode="last_loop")
    m.forward(toks, k)
    assert len(m.kv_slots()) == TINY.n_blocks
    p = om.Model(TINY, tiny_w, kv_mode="per_loop")
    p.forward(toks, k)
    assert len(p.kv_slots()) == TINY.n_in + TINY.n_out + k * TINY.n_rec


def test_per_loop_incremental_equals_prefill(tiny_w):
    toks = make_prompt(TINY, 2, 22)
    full = om.Model(TINY, tiny_w, batch=2).forward(toks, 2, all_logits=True)
    m = om.Model(TINY, tiny_w, batch=2)
    m.forward(toks[:, :18], 2)
    for j in range(18, 22):
        z = m.decode_step(toks[:, j], 2)
        assert np.allclose(z, full[:, j], atol=1e-10)


def test_last_loop_prefill_logits_equal_per_loop(tiny_w):
    """One call: every loop rewrites the call's own tokens before they are read,
    so a single prefill gives the same logits in both modes."""
    toks = make_prompt(TINY, 1, 40)
    a = om.Model(TINY, tiny_w, kv_mode="per_loop").forward(toks, 2, True)
    b = om.Model(TINY, tiny_w, kv_mode="last_loop").forward(toks, 2, True)
    assert np.allclose(a, b, atol=1e-12)


def test_last_loop_decode_reads_final_loop_entries(tiny_w):
    """After a prefill, a last_loop decode must equal a per_loop decode whose
    every recurrent slot was replaced by the final loop's entries for the prior
    tokens (earlier-loop queries see final-loop K/V)."""
    k = 3
    toks = make_prompt(TINY, 1, 25)
    ll = om.Model(TINY, tiny_w, kv_mode="last_loop")
    pl = om.Model(TINY, tiny_w, kv_mode="per_loop")
    ll.forward(toks, k)
    pl.forward(toks, k)
    _, grec, _ = TINY.block_groups()
    for i in grec:
        K, V = pl.cache[(i, k)]
        assert np.allclose(K, ll.cache[(i, 0)][0], atol=1e-12)
        for t in range(1, k):
            pl.cache[(i, t)] = (K.copy(), V.copy())
    za = ll.decode_step([7], k)
    zb = pl.decode_step([7], k)
    assert np.allclose(za, zb, atol=1e-10)
    # and it differs from the true per_loop decode
    ref = om.Model(TINY, tiny_w, kv_mode="per_loop")
    ref.forward(toks, k)
    assert not np.allclose(ref.decode_step([7], k), za, atol=1e-6)


def test_per_loop_rejects_other_loop_count(tiny_w):
    m = om.Model(TINY, tiny_w, kv_mode="per_loop")
    m.forward(make_prompt(TINY, 1, 4), 2)
    with pytest.raises(ValueError):
        m.decode_step([3], 1)
    m2 = om.Model(TINY, tiny_w, kv_mode="last_loop")
    m2.forward(make_prompt(TINY, 1, 4), 2)
    m2.decode_step([3], 4)                 # any count in last_loop mode


def test_batch_rows_independent(tiny_w):
    toks = make_prompt(TINY, 3, 12)
    zb = om.Model(TINY, tiny_w, batch=3).forward(toks, 2, True)
    for b in range(3):
        z1 = om.Model(TINY, tiny_w, batch=1).forward(toks[b:b + 1], 2, True)
        assert np.allclose(zb[b], z1[0], atol=1e-10)


def test_loop_boundaries_follow_printed_equation(tiny_w):
    """Recorded states satisfy s_0 = x, u_t = N(s_{t-1} + x), ||s_t|| = 1 and
    the recurrent blocks run between u_t and s_t (the paper summary's loop
    equation), for k = 3."""
    rec = []
    m = om.Model(TINY, tiny_w, trace=lambda kind, i, s: rec.append((kind, i, s)))
    m.forward(make_prompt(TINY, 1, 9), 3)
    gin, grec, gout = TINY.block_groups()
    x = [s for kind, i, s in rec if kind == "mlp" and i == gin[-1]][0]
    ins = [s for kind, i, s in rec if kind == "loop_in"]
    outs = [s for kind, i, s in rec if kind == "loop_out"]
    assert len(ins) == len(outs) == 3
    prev = x
    for u, s in zip(ins, outs):
        want = (prev + x) / np.linalg.norm(prev + x, axis=-1, keepdims=True)
        assert np.allclose(u, want, atol=1e-12)
        prev = s
    order = [(kind, i) for kind, i, _ in rec if kind in ("attn", "mlp")]
    n_in = 2 * len(gin)
    assert order[:n_in] == [(k, i) for i in gin for k in ("attn", "mlp")]
    loop = [(k, i) for i in grec for k in ("attn", "mlp")]
    assert order[n_in:n_in + 3 * len(loop)] == loop * 3
    assert order[n_in + 3 * len(loop):] == [(k, i) for i in gout
                                            for k in ("attn", "mlp")]


# ------------------------------------------------- sublayers from raw slices
def _bf(t):
    return (np.asarray(t).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def _small_shape(**kw):
    return tiny_with_blocks(1, 1, 0, **kw)


def _n(v):
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _unit_rows(T, d, seed):
    r = np.random.default_rng(seed).standard_normal((1, T, d))
    return _n(r)


def _expected_attn_uniform(w, sh, s, window):
    """Attention sublayer output when every score is equal (no key carries
    information): each query averages the values of its visible positions
    (paperlayer summary §2: gated, normalised attention output blended into
    the residual; paper summary, 技术新颖性: sigmoid output gate), written
    from the raw rows of w_qkvg in the order q, k, v, gate."""
    qd, kvd, h = sh.qdim, sh.kvdim, sh.head_dim
    G = sh.n_q_heads // sh.n_kv_heads
    W = _bf(w["blk0.w_qkvg"])
    Wv, Wg = W[qd + kvd:qd + 2 * kvd], W[qd + 2 * kvd:]
    T = s.shape[1]
    out = np.empty_like(s)
    for p in range(T):
        lo = max(0, p - window + 1) if window else 0
        vmean = np.mean([Wv @ s[0, j] for j in range(lo, p + 1)], axis=0)
        o = np.concatenate([vmean[(hq // G) * h:(hq // G + 1) * h]
                            for hq in range(sh.n_q_heads)])
        a = _n(_sig(Wg @ s[0, p]) * o)
        hA = _bf(w["blk0.w_o"]) @ a
        al = np.asarray(w["blk0.alpha_a"], np.float64)
        out[0, p] = _n(s[0, p] + al * (_n(hA) - s[0, p]))
    return out


@pytest.mark.parametrize("zero", ["q", "k"])
def test_attn_sublayer_uniform_scores_closed_form(zero):
    """With the query rows (or the key rows) of w_qkvg set to zero, every
    score is 0 and each query's output is the mean of the visible values.
    The expected state is written from the raw v / gate / W_o rows, so a
    wrong q/k/v/gate slice, a missing sigmoid, another gate granularity or
    another GQA head order fails here."""
    sh = _small_shape()
    w = dict(make_weights(sh, seed=3))
    qd, kvd = sh.qdim, sh.kvdim
    W = w["blk0.w_qkvg"].copy()
    if zero == "q":
        W[:qd] = 0
    else:
        W[qd:qd + kvd] = 0
    w["blk0.w_qkvg"] = W
    T = 13                          # longer than the 8-token window
    s = _unit_rows(T, sh.d, 11)
    for full, window in ((0, sh.swa_window), (1, 0)):
        lt = (full,) + sh.layer_types[1:]
        sh2 = _small_shape(layer_types=lt)
        m = om.Model(sh2, w)
        got = m.attn_sublayer(0, s, np.arange(T), 0)
        want = _expected_attn_uniform(w, sh2, s, window)
        assert np.allclose(got, want, atol=1e-12)


def test_attn_sublayer_single_token_returns_gated_value():
    """One token, empty cache: the softmax over one key is 1, so head h
    outputs v of KV head h // (Hq/Hkv) whatever q and k are."""
    sh = _small_shape()
    w = make_weights(sh, seed=4)
    s = _unit_rows(1, sh.d, 12)
    got = om.Model(sh, w).attn_sublayer(0, s, np.arange(1), 0)
    want = _expected_attn_uniform(w, sh, s, 0)
    assert np.allclose(got, want, atol=1e-12)


def test_mlp_sublayer_gate_rows_then_up_rows():
    """SwiGLU over the fused gate/up matrix: rows [0, F) are the gate (through
    silu), rows [F, 2F) the up projection (paperlayer summary §2: SwiGLU
    activations normalised before the down projection).  Swapping the halves
    gives another state, so the test sees the order."""
    sh = _small_shape()
    w = make_weights(sh, seed=5)
    F = sh.ffn
    s = _unit_rows(3, sh.d, 13)
    Wgu = _bf(w["blk0.w_gu"])
    g, u = s @ Wgu[:F].T, s @ Wgu[F:].T
    al = np.asarray(w["blk0.alpha_m"], np.float64)

    def state(gate, up):
        m = _n(gate * _sig(gate) * up)
        hM = m @ _bf(w["blk0.w_down"]).T
        return _n(s + al * (_n(hM) - s))

    got = om.Model(sh, w).mlp_sublayer(0, s)
    assert np.allclose(got, state(g, u), atol=1e-12)
    assert not np.allclose(got, state(u, g), atol=1e-6)


def test_lm_head_across_row_chunks_with_logit_scale():
    """z = s_z * (W_lm s) for a vocabulary larger than the oracle's 16384-row
    chunk, with a non-uniform logit scale (paperlayer summary §2: logit-scale
    parameters)."""
    sh = _small_shape(vocab=40000)
    w = dict(make_weights(sh, seed=6, names=["lm_head", "s_z"]))
    w["s_z"] = np.linspace(0.5, 3.0, sh.vocab).astype(np.float32)
    s = _unit_rows(2, sh.d, 14)
    got = om.Model(sh, w).lm_head(s)
    want = w["s_z"].astype(np.float64) * (s @ _bf(w["lm_head"]).T)
    assert got.shape == (1, 2, sh.vocab)
    assert np.allclose(got, want, atol=1e-12)
