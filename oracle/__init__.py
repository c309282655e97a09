"""CPU oracle of the GPT-2 decoder: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the C-ABI library
and its Python binding) never imports, calls or falls back to it.

* ``gpt2_oracle``: fp64 NumPy forward pass, logits and shifted
  cross-entropy, written from the pages' definitions.
* ``gpt2_backward``: fp64 NumPy gradients of that loss with respect to
  every weight (the chain rule through each forward step, in reverse).
* ``brute``: pure-Python scalar loops of the same forward pass for tiny
  shapes, used to pin ``gpt2_oracle``.
"""
from . import gpt2_oracle, gpt2_backward, brute  # noqa: F401
from .gpt2_oracle import (  # noqa: F401
    LN_EPS, layer_norm, gelu, linear, causal_mask, softmax_last,
    causal_self_attention, block, embed, hidden_states, forward,
    logsumexp_last, shifted_cross_entropy,
)
