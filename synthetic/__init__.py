"""Seeded synthetic inputs for the looped nGPT forward pass.

This module is shared by the CPU oracle (``oracle/``) and by the CUDA path
(``looped_ngpt_b200``).  It holds model *shapes* and random-number recipes
only; no step of the forward pass (normalisation of states, projections,
attention, the loop) is computed here.  The recipe follows the workload
descriptions of the Dory1.0-4B pages:

* every weight matrix: N(0, 1) entries, each row scaled to unit L2 norm
  (the nGPT convention of unit-norm embedding rows), then rounded to BF16
  with round-to-nearest-even;
* residual rates alpha_A, alpha_M: 0.05 + N(0, 1e-3) per channel
  ("ngpt_alpha_init 0.05", Dory model card, config section);
* query/key scales s_q, s_k: 1 + N(0, 1e-3) per head and dimension;
* logit scale s_z: sqrt(d) * (1 + N(0, 1e-3)) per vocabulary entry, so that
  logits of unit vectors have a spread of about one;
* prompts: uniform integers in [0, vocab), seed 1.

Each tensor is drawn from its own PCG64 stream ``default_rng([seed, idx])``
(idx = the tensor's position in ``tensor_names``), so any subset of tensors
can be generated alone and the draw does not depend on the order of calls.
"""
from .shapes import ModelShape, TINY, DORY, tiny_with_blocks, dory_with_blocks
from .gen import (tensor_names, tensor_spec, make_tensor, make_weights,
                  make_prompt, bf16_bits_to_f32, f32_to_bf16_bits)

__all__ = ["ModelShape", "TINY", "DORY", "tiny_with_blocks", "dory_with_blocks", "tensor_names",
           "tensor_spec", "make_tensor", "make_weights", "make_prompt",
           "bf16_bits_to_f32", "f32_to_bf16_bits"]
