"""CPU oracle of the Dory1.0-4B looped normalized-GPT forward pass.

TEST INFRASTRUCTURE.  This package is a plain, slow, obviously-correct NumPy
restatement of the method as the Dory1.0-4B pages describe it.  It exists to
check the CUDA path; it is not part of the product.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and its
reference arm) may import it.  It shares no code with the CUDA path and
imports nothing from ``looped_ngpt_b200``; the two meet only through the
seeded generators in ``synthetic``.

Arithmetic is float64 throughout (the pages fix no precision for the
reference computation).  Weights are the same BF16 bytes the GPU reads,
widened exactly.

Parity status by function (what pins each is listed in the tests):
  l2n, rope, attention, attention_bruteforce, ngpt_update, swiglu,
  Model.forward (loop, re-injection, both KV modes), quant decoders and
  quantisers: pinned by closed forms, special cases, brute force and
  format-definition values.
  query/key scale and softmax temperature (sqrt(head_dim)): parity
  unpinned -- the pages name a query-key scale but print no value or
  formula for the temperature; the reading taken is the nGPT one.
"""
from .model import (Model, l2n, rope, attention, attention_bruteforce,
                    ngpt_update, swiglu, silu, sigmoid, greedy)
from . import quant

__all__ = ["Model", "l2n", "rope", "attention", "attention_bruteforce",
           "ngpt_update", "swiglu", "silu", "sigmoid", "greedy", "quant"]
