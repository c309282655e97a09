"""Seeded synthetic inputs for the GPT-2 decoder forward pass.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path's
tests and bench. It holds none of the model's arithmetic: only the five
workload shapes, the random draws that fill the weights and token ids, the
bf16 storage rounding of those draws, and the position-aligned next-token
target array that the C ABI takes as input.

Workloads (sizes of GPT-2 small/medium/large/XL as listed in "Hand-writing
GPT-2 from scratch: the Transformer decoder core modules in PyTorch",
section 2.3, and the 124M config table of "Implementing GPT-2 from scratch:
a PyTorch guide to building an LLM", "configuration system"):

====  ==============================================  =====================
name  shape                                           init
====  ==============================================  =====================
tiny  L2 H2 C64 V512 ctx32, B2 T4, fp32               "dist": W,emb N(0,.02),
                                                      c_proj N(0,.02/sqrt(2L)),
                                                      b N(0,.01), g 1+N(0,.1),
                                                      beta N(0,.1)
124M  L12 H12 C768 V50257 ctx1024, B4 T1024, bf16     "dist"
350M  L24 H16 C1024, B8 T1024, bf16, loss only        "gpt2": N(0,.02),
                                                      c_proj /sqrt(2L),
                                                      b=0, g=1, beta=0
774M  L36 H20 C1280, B4, lengths 128/512/1000/1024    "gpt2"
      right-padded to T1024, bf16
1.5B  L48 H25 C1600, B16 T1024, bf16, loss only       "gpt2"
====  ==============================================  =====================

The "gpt2" init is the one described in "Reproducing GPT-2 124M", section
2.4 (Linear and embedding weights N(0, 0.02), LayerNorm gamma 1 and beta 0,
c_proj weights scaled by 1/sqrt(2*n_layer)).

Seeds: weights use ``numpy.random.default_rng(1000 + index)``; token ids use
``default_rng(1500 + index)``. Draws are made in float32 in a fixed tensor
order (wte, wpe, then per layer ln1_g, ln1_b, attn_w, attn_b, attn_proj_w,
attn_proj_b, ln2_g, ln2_b, fc_w, fc_b, mlp_proj_w, mlp_proj_b, then lnf_g,
lnf_b). For bf16 workloads every weight is rounded once to the nearest bf16
(ties to even) here, so the CUDA path and the oracle see identical values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

LAYER_KEYS = (
    "ln1_g", "ln1_b", "attn_w", "attn_b", "attn_proj_w", "attn_proj_b",
    "ln2_g", "ln2_b", "fc_w", "fc_b", "mlp_proj_w", "mlp_proj_b",
)


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    n_layer: int
    n_head: int
    n_embd: int
    vocab: int
    n_ctx: int
    batch: int
    seq: int
    dtype: str                    # "fp32" or "bf16": storage type of weights/activations
    init: str                     # "dist" or "gpt2"
    outputs: str                  # "logits+loss" or "loss"
    lengths: Optional[tuple] = None   # per-sequence valid lengths (right-padded)

    @property
    def d_head(self) -> int:
        return self.n_embd // self.n_head

    def scaled(self, **kw) -> "Workload":
        """A copy with some fields replaced (smaller parity cases)."""
        return dataclasses.replace(self, **kw)


WORKLOADS: List[Workload] = [
    Workload(0, "gpt2-tiny-fp32", 2, 2, 64, 512, 32, 2, 4, "fp32", "dist", "logits+loss"),
    Workload(1, "gpt2-124M", 12, 12, 768, 50257, 1024, 4, 1024, "bf16", "dist", "logits+loss"),
    Workload(2, "gpt2-350M", 24, 16, 1024, 50257, 1024, 8, 1024, "bf16", "gpt2", "loss"),
    Workload(3, "gpt2-774M", 36, 20, 1280, 50257, 1024, 4, 1024, "bf16", "gpt2", "logits+loss",
             lengths=(128, 512, 1000, 1024)),
    Workload(4, "gpt2-1.5B", 48, 25, 1600, 50257, 1024, 16, 1024, "bf16", "gpt2", "loss"),
]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); return float32.

    NaN/Inf do not occur in these draws. The result is exactly representable
    in bf16, so converting it to torch.bfloat16 on the device is lossless.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u >> 16) & 1) + 0x7FFF
    out = (((u + r) >> 16) << 16).astype(np.uint32)
    return out.view(np.float32).reshape(a.shape)


def _normal(rng, shape, std):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def make_weights(w: Workload) -> Dict[str, object]:
    """Draw all weights of workload ``w``.

    Returns a dict with float32 numpy arrays:
    ``wte`` [V,C], ``wpe`` [n_ctx,C], ``layers`` (list of dicts keyed by
    LAYER_KEYS, Linear weights in nn.Linear [out,in] layout), ``lnf_g``,
    ``lnf_b`` [C]. For bf16 workloads the values are bf16-exact.
    """
    rng = np.random.default_rng(1000 + w.index)
    C, L = w.n_embd, w.n_layer
    proj_std = 0.02 / np.sqrt(2.0 * L)

    def vec_bias(n):
        return _normal(rng, (n,), 0.01) if w.init == "dist" else np.zeros(n, np.float32)

    def vec_gamma(n):
        if w.init == "dist":
            return (1.0 + _normal(rng, (n,), 0.1)).astype(np.float32)
        return np.ones(n, np.float32)

    def vec_beta(n):
        return _normal(rng, (n,), 0.1) if w.init == "dist" else np.zeros(n, np.float32)

    out: Dict[str, object] = {}
    out["wte"] = _normal(rng, (w.vocab, C), 0.02)
    out["wpe"] = _normal(rng, (w.n_ctx, C), 0.02)
    layers = []
    for _ in range(L):
        d = {}
        d["ln1_g"] = vec_gamma(C)
        d["ln1_b"] = vec_beta(C)
        d["attn_w"] = _normal(rng, (3 * C, C), 0.02)
        d["attn_b"] = vec_bias(3 * C)
        d["attn_proj_w"] = _normal(rng, (C, C), proj_std)
        d["attn_proj_b"] = vec_bias(C)
        d["ln2_g"] = vec_gamma(C)
        d["ln2_b"] = vec_beta(C)
        d["fc_w"] = _normal(rng, (4 * C, C), 0.02)
        d["fc_b"] = vec_bias(4 * C)
        d["mlp_proj_w"] = _normal(rng, (C, 4 * C), proj_std)
        d["mlp_proj_b"] = vec_bias(C)
        layers.append(d)
    out["layers"] = layers
    out["lnf_g"] = vec_gamma(C)
    out["lnf_b"] = vec_beta(C)
    if w.dtype == "bf16":
        out["wte"] = round_to_bf16(out["wte"])
        out["wpe"] = round_to_bf16(out["wpe"])
        for d in layers:
            for k in LAYER_KEYS:
                d[k] = round_to_bf16(d[k])
        out["lnf_g"] = round_to_bf16(out["lnf_g"])
        out["lnf_b"] = round_to_bf16(out["lnf_b"])
    return out


def make_ids(w: Workload) -> np.ndarray:
    """Token ids int32 [B,T], uniform in [0, vocab); positions past a
    sequence's length (right padding) hold id 0."""
    rng = np.random.default_rng(1500 + w.index)
    ids = rng.integers(0, w.vocab, size=(w.batch, w.seq), dtype=np.int64).astype(np.int32)
    if w.lengths is not None:
        for b, n in enumerate(w.lengths):
            ids[b, n:] = 0
    return ids


def lengths_of(w: Workload) -> np.ndarray:
    """Valid length of each sequence (T for every sequence unless padded)."""
    if w.lengths is None:
        return np.full(w.batch, w.seq, dtype=np.int64)
    return np.asarray(w.lengths, dtype=np.int64)


def next_token_targets(ids: np.ndarray, lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """Position-aligned targets int32 [B,T] for the C ABI: position t of
    sequence b is scored against ids[b, t+1] while t+1 < length[b]; every
    other position holds -1 (ignored)."""
    B, T = ids.shape
    if lengths is None:
        lengths = np.full(B, T, dtype=np.int64)
    tg = np.full((B, T), -1, dtype=np.int32)
    for b in range(B):
        n = int(lengths[b])
        if n > 1:
            tg[b, : n - 1] = ids[b, 1:n]
    return tg


def random_case(seed: int, n_layer: int, n_head: int, n_embd: int, vocab: int, n_ctx: int,
                batch: int, seq: int, dtype: str = "bf16", init: str = "dist",
                lengths: Optional[tuple] = None) -> Workload:
    """A small ad-hoc workload (parity cases that span several tiles and a
    ragged tail). ``seed`` plays the role of the index in the seed rule."""
    return Workload(seed, f"case{seed}", n_layer, n_head, n_embd, vocab, n_ctx, batch, seq,
                    dtype, init, "logits+loss", lengths)
