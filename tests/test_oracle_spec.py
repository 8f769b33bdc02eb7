"""Pins of the speculative acceptance rule (oracle/spec.py) against what the
mathematics of rejection sampling fixes (paperlayer summary §6.2: the output
keeps the verifier's sampling distribution)."""
import numpy as np

from oracle import spec


def test_greedy_keeps_matching_prefix_then_verifier_argmax():
    V = 7
    z = np.zeros((4, V))
    z[0, 3] = z[1, 5] = z[2, 1] = z[3, 6] = 1.0       # argmax 3, 5, 1, 6
    out, n = spec.accept_batch([[9, 3, 5, 2]], z[None], None, 0)
    assert n == 3 and list(out[0]) == [3, 5, 1, -1]
    out, n = spec.accept_batch([[9, 3, 5, 1]], z[None], None, 0)
    assert n == 4 and list(out[0]) == [3, 5, 1, 6]     # all kept + bonus
    out, n = spec.accept_batch([[9, 0, 5, 1]], z[None], None, 0)
    assert n == 1 and list(out[0]) == [3, -1, -1, -1]


def test_first_token_is_distributed_as_the_verifier():
    """P(emit x) = p(d) for x = d, else (1 - p(d)) p(x) / (1 - p(d)) = p(x):
    Monte Carlo over the uniforms, chi-square against p."""
    rng = np.random.default_rng(0)
    V, T = 6, 0.8
    z = rng.standard_normal((2, V)) * 2
    p = spec.softmax_t(z[0], T)
    d = int(np.argsort(p)[-2])                      # a likely, non-top draft
    N = 60000
    counts = np.zeros(V)
    for _ in range(N):
        u = rng.random(2)
        out, _ = spec.accept_batch([[0, d]], z[None], u[None], T)
        counts[out[0, 0]] += 1
    chi2 = float(((counts - N * p) ** 2 / (N * p)).sum())
    assert chi2 < 25.0, (chi2, counts / N, p)         # 5 dof, p ~ 1e-4


def test_all_kept_bonus_and_batch_minimum():
    rng = np.random.default_rng(1)
    V, T = 5, 1.0
    z = rng.standard_normal((2, 3, V))
    d = np.array([[0, 1, 2], [0, 3, 4]])
    u = np.zeros((2, 3))                             # u = 0 keeps any draft
    u[:, 2] = 0.999
    out, n = spec.accept_batch(d, z, u, T)
    assert n == 3
    for b in range(2):                               # bonus: inverse CDF of p
        assert out[b, 2] == spec.inverse_cdf(spec.softmax_t(z[b, 2], T), 0.999)
    u[1, 1] = 0.9999999                              # row 1 rejects draft 2
    out, n = spec.accept_batch(d, z, u, T)
    assert n == 2
    assert out[0, 1] == d[0, 2]                      # row 0 kept its own
    p = spec.softmax_t(z[1, 1], T)
    p[d[1, 2]] = 0
    assert out[1, 1] == spec.inverse_cdf(p, 0.999)
    assert list(out[:, 2]) == [-1, -1]


def test_inverse_cdf_closed_form():
    w = np.array([0.1, 0.0, 0.3, 0.6])
    assert spec.inverse_cdf(w, 0.0) == 0
    assert spec.inverse_cdf(w, 0.099) == 0
    assert spec.inverse_cdf(w, 0.2) == 2
    assert spec.inverse_cdf(w, 0.41) == 3
    assert spec.inverse_cdf(w, 0.999999) == 3
