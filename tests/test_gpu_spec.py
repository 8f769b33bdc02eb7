"""Self-speculative decoding on the GPU ("Dory1.0-4B: A Looped
Normalized-GPT", §6.2: draft at one loop, verify at four, rejection
sampling keeps the verifier's distribution).

* The acceptance kernels against the oracle's rule (oracle/spec.py) on the
  same logits, proposals and uniforms: greedy and sampled, a batch of
  sequences advancing together.
* The first emitted token of the sampled rule is distributed as the
  verifier's softmax (chi-square over 4000 draws).
* End to end on the tiny model, per_loop cache: greedy speculative decoding
  emits the greedy tokens of the four-loop model; every emitted token is a
  valid greedy pick of the oracle run over the same sequence, and the
  sequence equals the GPU's own one-token-at-a-time k = 4 decoding."""
import ctypes

import numpy as np
import pytest
import torch

from looped_ngpt_b200 import _lib
from oracle import spec
from oracle.model import Model
from synthetic import TINY, make_weights, make_prompt
from tests.gpu_util import LOGIT_TOL

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _ptr(t, off=0):
    return P(t.data_ptr() + off)


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _near_boundary(drafts, logits, uniforms, temperature, eps=1e-5):
    """Whether a decision the oracle rule takes lies within eps of its
    threshold (f32 and f64 arithmetic may then decide differently): the
    keep/reject tests each row runs, and the one inverse-CDF draw."""
    B, G1 = drafts.shape
    gamma = G1 - 1
    r = [spec.accepted(drafts[b], logits[b], uniforms[b], temperature)
         for b in range(B)]
    n = min(r)
    for b in range(B):
        for j in range(min(r[b] + 1, gamma)):
            p = spec.softmax_t(logits[b, j], temperature)
            if abs(uniforms[b, j] - p[drafts[b, j + 1]]) < eps:
                return True
        if r[b] == n:
            q = spec.softmax_t(logits[b, n], temperature)
            if n < gamma:
                q[drafts[b, n + 1]] = 0.0
            c = np.cumsum(q) / q.sum()
            if np.min(np.abs(c - uniforms[b, gamma])) < eps:
                return True
    return False


@pytest.mark.parametrize("temperature", [0.0, 0.7])
def test_accept_kernel_matches_oracle_rule(temperature):
    lib = _lib.load()
    rng = np.random.default_rng(31)
    B, gamma, V = 3, 4, 1024
    G1 = gamma + 1
    checked = 0
    for trial in range(40):
        z = (rng.standard_normal((B, G1, V)) * 3).astype(np.float32)
        am = np.argmax(z, -1)
        drafts = rng.integers(0, V, size=(B, G1))
        take = rng.random((B, G1)) < 0.8          # mostly the verifier's pick
        drafts[:, 1:] = np.where(take[:, 1:], am[:, :-1], drafts[:, 1:])
        u = rng.random((B, G1)).astype(np.float32)
        if temperature > 0 and _near_boundary(drafts, z, u, temperature):
            continue
        want, n_want = spec.accept_batch(drafts, z.astype(np.float64),
                                         u.astype(np.float64), temperature)
        d_dr = torch.from_numpy(drafts.astype(np.int32)).cuda()
        d_tg = torch.from_numpy(am.astype(np.int32)).cuda()
        d_z = torch.from_numpy(z).cuda()
        d_u = torch.from_numpy(u).cuda()
        out = torch.full((B, G1), -7, dtype=torch.int32, device="cuda")
        scr = torch.zeros(B + 2, dtype=torch.int32, device="cuda")
        assert lib.dory_debug_spec_accept(
            _ptr(d_dr), _ptr(d_tg), _ptr(d_z), _ptr(d_u), B, gamma, V,
            ctypes.c_float(temperature), _ptr(out), _ptr(scr), _stream()) == 0
        torch.cuda.synchronize()
        assert int(scr[0]) == n_want, trial
        assert np.array_equal(out.cpu().numpy(), want), trial
        checked += 1
    assert checked >= 30


def test_accept_kernel_first_token_distribution():
    lib = _lib.load()
    rng = np.random.default_rng(5)
    V, T, N = 64, 1.0, 4000
    z = (rng.standard_normal((1, 2, V)) * 1.5).astype(np.float32)
    p = spec.softmax_t(z[0, 0].astype(np.float64), T)
    d = int(np.argsort(p)[-1])
    drafts = torch.tensor([[0, d]], dtype=torch.int32, device="cuda")
    tg = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    dz = torch.from_numpy(z).cuda()
    u = torch.from_numpy(rng.random((N, 2)).astype(np.float32)).cuda()
    out = torch.empty((N, 2), dtype=torch.int32, device="cuda")
    scr = torch.zeros((N, 3), dtype=torch.int32, device="cuda")
    for i in range(N):
        assert lib.dory_debug_spec_accept(
            _ptr(drafts), _ptr(tg), _ptr(dz), _ptr(u, i * 8), 1, 1, V,
            ctypes.c_float(T), _ptr(out, i * 8), _ptr(scr, i * 12),
            _stream()) == 0
    torch.cuda.synchronize()
    first = out[:, 0].cpu().numpy()
    counts = np.bincount(first, minlength=V).astype(np.float64)
    keep = N * p > 5                                # pool the rare tokens
    obs = np.append(counts[keep], counts[~keep].sum())
    exp = np.append(N * p[keep], N * p[~keep].sum())
    chi2 = float(((obs - exp) ** 2 / exp).sum())
    dof = len(obs) - 1
    assert chi2 < dof + 6 * np.sqrt(2 * dof), (chi2, dof)


@pytest.fixture(scope="module")
def tiny():
    import looped_ngpt_b200 as lb
    w = make_weights(TINY, seed=0)
    return w, lb.DoryModel(TINY, w, device="cuda:0")


def _plain_greedy(gm, prompt, k, n_tok):
    cache = gm.new_cache(1, 128, 32, kv_mode="per_loop", max_loops=k)
    ws = gm.workspace(1, 32)
    _, a = gm.prefill(cache, torch.from_numpy(prompt).cuda(), k, ws)
    toks, gaps = [int(a.cpu()[0])], []
    for _ in range(n_tok - 1):
        z, a = gm.decode_step(cache, a.clone(), k, ws)
        zs = np.sort(z.cpu().numpy()[0])
        gaps.append(zs[-1] - zs[-2])
        toks.append(int(a.cpu()[0]))
    return toks, gaps


def test_spec_greedy_equals_k4_greedy(tiny):
    w, gm = tiny
    k_draft, k_verify, gamma = 1, 4, 4
    prompt = make_prompt(TINY, 1, 20, seed=13)
    cache = gm.new_cache(1, 128, 32, kv_mode="per_loop", max_loops=k_verify)
    ws = gm.workspace(1, 32)
    sws = gm.spec_workspace(1, gamma)
    _, a = gm.prefill(cache, torch.from_numpy(prompt).cuda(), k_verify, ws)
    last = a.clone()
    gen = [int(last.cpu()[0])]
    counts = []
    while len(gen) < 33:
        out, n = gm.spec_decode_step(cache, last, gamma, k_draft, k_verify, sws)
        o = out.cpu().numpy()[0]
        assert 1 <= n <= gamma + 1 and (o[n:] == -1).all()
        gen += [int(t) for t in o[:n]]
        counts.append(n)
        last = out[:, n - 1].contiguous()
    assert gm.sync_status() == 0
    assert cache.length() == prompt.shape[1] + len(gen) - 1
    # every emitted token is a valid greedy pick of the oracle at k = 4 over
    # the same sequence (one multi-token pass = one-token steps, per_loop)
    seq = np.concatenate([prompt[0], np.array(gen[:-1])])[None]
    z = Model(TINY, w, kv_mode="per_loop").forward(seq, k_verify, True)[0]
    T0 = prompt.shape[1]
    for i, t in enumerate(gen):
        row = z[T0 - 1 + i]
        assert row.max() - row[t] <= LOGIT_TOL, (i, t, int(np.argmax(row)))
    # and it is the GPU's own k = 4 greedy decoding, up to the first step
    # whose top two logits are closer than the tolerance
    plain, gaps = _plain_greedy(gm, prompt, k_verify, len(gen))
    for i in range(len(gen)):
        if i > 0 and gaps[i - 1] < 2 * LOGIT_TOL:
            break
        assert gen[i] == plain[i], (i, gen[:i + 1], plain[:i + 1])
    print(f"spec greedy: {len(gen)} tokens in {len(counts)} steps "
          f"(emitted per step {counts})")


def test_spec_sampled_runs_and_keeps_cache_consistent(tiny):
    w, gm = tiny
    gamma = 3
    prompt = make_prompt(TINY, 2, 12, seed=14)
    cache = gm.new_cache(2, 96, 16, kv_mode="per_loop", max_loops=4)
    ws = gm.workspace(2, 16)
    sws = gm.spec_workspace(2, gamma)
    _, a = gm.prefill(cache, torch.from_numpy(prompt).cuda(), 4, ws)
    last = a.clone()
    total = 0
    rng = np.random.default_rng(2)
    for _ in range(6):
        u = torch.from_numpy(rng.random((2, gamma + 1)).astype(np.float32)).cuda()
        out, n = gm.spec_decode_step(cache, last, gamma, 1, 4, sws,
                                     temperature=0.8, uniform=u)
        o = out.cpu().numpy()
        assert 1 <= n <= gamma + 1
        assert ((o[:, :n] >= 0) & (o[:, :n] < TINY.vocab)).all()
        assert (o[:, n:] == -1).all()
        total += n
        last = out[:, n - 1].contiguous()
    assert gm.sync_status() == 0
    assert cache.length() == 12 + total
    # a last_loop cache is refused (a verify pass would not be one-token
    # decoding there)
    import looped_ngpt_b200 as lb
    c2 = gm.new_cache(2, 32, 8, kv_mode="last_loop")
    with pytest.raises(lb.DoryError) as e:
        gm.spec_decode_step(c2, last, gamma, 1, 4, sws)
    assert e.value.code == -3
