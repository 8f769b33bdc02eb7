"""Acceptance rule of self-speculative decoding (TEST INFRASTRUCTURE, see the
package docstring).

"Dory1.0-4B: A Looped Normalized-GPT" (paperlayer summary), §6.2
Self-Speculative Decoding: the same checkpoint drafts at one loop and
verifies the proposed tokens at four loops; rejection sampling accepts
proposals and corrects rejections so that the output keeps the verifier's
sampling distribution.

Readings where the page is silent:
  * the draft is greedy: each proposal is the draft model's argmax, i.e. a
    point-mass proposal q = delta(d).  For it the rejection-sampling rule of
    speculative sampling becomes: keep proposal d with probability p(d)
    (p = the verifier's distribution at that position); at the first
    rejection draw from the residual max(0, p - q), normalised, which is p
    restricted to x != d; if every proposal is kept, draw once more from p
    at the last position;
  * p = softmax(z / temperature) of the verifier's logits z; temperature 0
    is greedy decoding (keep d iff it is the verifier's argmax, lowest index
    on ties; the token after the kept proposals is the verifier's argmax);
  * the random numbers are inputs: u_j in [0, 1) decides proposal j + 1,
    and one more, u_gamma, drives the single draw (inverse CDF: the smallest
    token whose cumulative weight exceeds u * total);
  * sequences decoded together advance by the same count n = 1 + min_b r_b
    (r_b = proposals row b kept); a row that kept more emits its own kept
    proposal at position n - 1.
"""
import numpy as np


def softmax_t(z, temperature):
    """p = softmax(z / temperature) in float64."""
    z = np.asarray(z, dtype=np.float64) / temperature
    e = np.exp(z - z.max())
    return e / e.sum()


def inverse_cdf(w, u):
    """Smallest index whose running sum of the weights w exceeds u * sum(w)."""
    c = np.cumsum(np.asarray(w, dtype=np.float64))
    idx = int(np.searchsorted(c, u * c[-1], side="right"))
    nz = np.flatnonzero(np.asarray(w) > 0)
    return min(idx, int(nz[-1]))


def accepted(draft, logits, uniform, temperature):
    """Number r of proposals one sequence keeps: draft [gamma + 1] (last
    accepted token, then the proposals), logits [gamma + 1, V] of the
    verifier, uniform [gamma + 1]."""
    gamma = len(draft) - 1
    for j in range(gamma):
        d = int(draft[j + 1])
        if temperature == 0:
            keep = d == int(np.argmax(logits[j]))
        else:
            keep = uniform[j] < softmax_t(logits[j], temperature)[d]
        if not keep:
            return j
    return gamma


def token_at(draft, logits, uniform, temperature, n_kept, own_kept):
    """The token a sequence emits after n_kept proposals (own_kept: how many
    this sequence kept itself)."""
    gamma = len(draft) - 1
    if temperature == 0:
        return int(np.argmax(logits[n_kept]))
    if own_kept > n_kept:
        return int(draft[n_kept + 1])
    p = softmax_t(logits[n_kept], temperature)
    if n_kept < gamma:
        p = p.copy()
        p[int(draft[n_kept + 1])] = 0.0
    return inverse_cdf(p, uniform[gamma])


def accept_batch(drafts, logits, uniforms, temperature):
    """Emitted tokens [B, gamma + 1] (-1 past n) and n for a batch of
    sequences advancing together."""
    drafts = np.asarray(drafts)
    B, G1 = drafts.shape
    r = [accepted(drafts[b], logits[b], uniforms[b] if uniforms is not None
                  else None, temperature) for b in range(B)]
    n = min(r)
    out = np.full((B, G1), -1, dtype=np.int64)
    for b in range(B):
        out[b, :n] = drafts[b, 1:n + 1]
        out[b, n] = token_at(drafts[b], logits[b], uniforms[b] if uniforms
                             is not None else None, temperature, n, r[b])
    return out, n + 1
