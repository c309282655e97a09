"""CPU oracle for the GPT-2 decoder forward pass (test infrastructure only).

This is a plain, slow, fp64 NumPy restatement of what the forward pass
computes, written from the pages' definitions. It exists to check the CUDA
path: only the tests, the smoke check and the bench's CPU-baseline leg may
import it. It shares no code with the CUDA path; its only shared input is the
seeded generator in ``synthetic``.

Every step is the plain definition, with NumPy's matmul, exp, log, tanh,
sin, cos and SciPy's erf as the only library primitives. There is no blocking, fusion or
reordering: attention materialises the full masked score matrix, the
cross-entropy materialises the full logits.

Sources (page titles; the sections cited per function):
  [P1] "Hand-writing GPT-2 from scratch: the Transformer decoder core modules
       in PyTorch" (blog.csdn.net)
  [P3] "GPT-2 architecture analysis and implementation guide"
       (intelliparadigm.com)
  [P4] "Reproducing GPT-2 124M" (nzsm.cn)
  [P5] "Implementing GPT-2 from scratch: a PyTorch guide to building an LLM"
       (zingnex.cn)

Pins (tests/test_oracle_pins.py) tie every function below to something other
than itself: a pure-Python brute force, library routines (torch fp64
layer_norm / scaled_dot_product_attention / gelu / cross_entropy), closed
forms and the invariants the pages state. No function here is parity
unpinned.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np
from scipy.special import erf as _erf

LN_EPS = 1e-5  # [P1] sections 3.2 and 4.2; [P4] section 2.1


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """LayerNorm over the last axis with the biased variance.

    [P4] section 2.1 (hand-written LayerNorm: mean and the variance without
    Bessel's correction over the feature axis, eps added inside the square
    root, then gamma scale and beta shift); [P1] sections 3.2 and 4.2 fix
    eps = 1e-5.
    """
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return gamma * (x - mu) / np.sqrt(var + eps) + beta


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU, 0.5 x (1 + erf(x / sqrt 2)).

    [P3] section 2.2 applies F.gelu (the exact erf form); [P1] section 3.4
    recommends approximate=False. This is the default activation; gelu_tanh
    is the flag-selected variant.
    """
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """Tanh-approximation GELU, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).

    [P1] section 3.4 and [P4] section 2.4 give this form as the one of the
    original GPT-2 implementation (the model's GPT2_FLAG_GELU_TANH variant).
    """
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def sinusoidal_wpe(n_ctx: int, C: int) -> np.ndarray:
    """Fixed sinusoidal position table [n_ctx, C] ([P1] section 3.1):
    pe[pos, 2i] = sin(pos / 10000^(2i/C)), pe[pos, 2i+1] = cos(pos / 10000^(2i/C)),
    pos from 0, i in [0, C/2)."""
    pos = np.arange(n_ctx, dtype=np.float64)[:, None]
    i = np.arange(C // 2, dtype=np.float64)[None, :]
    angle = pos / np.power(10000.0, 2.0 * i / C)
    pe = np.empty((n_ctx, C), dtype=np.float64)
    pe[:, 0::2] = np.sin(angle)
    pe[:, 1::2] = np.cos(angle)
    return pe


def linear(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    """nn.Linear: y = x W^T + b with W in [out, in] layout ([P1] section 3.4)."""
    y = x @ w.T
    return y if b is None else y + b


def causal_mask(T: int) -> np.ndarray:
    """Boolean [T,T] mask, True where key j lies in the future of query i
    (j > i): the upper triangle above the diagonal ([P1] section 3.3, the
    tril / triu(diagonal=1) forms; [P3] section 2.1 get_mask)."""
    return np.triu(np.ones((T, T), dtype=bool), k=1)


def softmax_last(s: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (max-subtracted; exp(-inf) = 0)."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def causal_self_attention(qkv: np.ndarray, n_head: int, return_probs: bool = False):
    """Multi-head causal self-attention on the c_attn output.

    qkv: [B, T, 3C]. Columns [0,C) are q, [C,2C) k, [2C,3C) v; head h uses
    columns h*D..(h+1)*D of each ([P4] section 2.1: split by n_embd, then a
    view to [B,T,H,D] and a transpose to [B,H,T,D]).
    Scores q k^T * (1/sqrt(D)), then -inf where j > i, then softmax over
    keys, then P v, then heads concatenated back to [B,T,C]
    ([P4] sections 2.1-2.2; [P3] section 2.1).
    """
    B, T, C3 = qkv.shape
    C = C3 // 3
    D = C // n_head
    q = qkv[:, :, 0:C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    k = qkv[:, :, C:2 * C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    v = qkv[:, :, 2 * C:3 * C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    mask = causal_mask(T)
    y = np.empty((B, n_head, T, D), dtype=qkv.dtype)
    probs = np.empty((B, n_head, T, T), dtype=qkv.dtype) if return_probs else None
    scale = 1.0 / math.sqrt(D)
    for b in range(B):  # one sequence at a time bounds the [H,T,T] score memory
        s = (q[b] @ k[b].transpose(0, 2, 1)) * scale
        s = np.where(mask, -np.inf, s)
        p = softmax_last(s)
        y[b] = p @ v[b]
        if return_probs:
            probs[b] = p
    out = y.transpose(0, 2, 1, 3).reshape(B, T, C)
    return (out, probs) if return_probs else out


def block(x: np.ndarray, lw: Dict[str, np.ndarray], n_head: int, eps: float = LN_EPS,
          act=None) -> np.ndarray:
    """One Pre-LN block: x += attn(ln_1(x)); x += mlp(ln_2(x)).

    [P1] section 3.2 (LN, attention, residual add, LN, MLP, residual add);
    [P3] section 1.1 (GPT2Block.forward). Dropout is the identity in a
    forward pass without training.
    """
    h = layer_norm(x, lw["ln1_g"], lw["ln1_b"], eps)
    qkv = linear(h, lw["attn_w"], lw["attn_b"])
    y = causal_self_attention(qkv, n_head)
    x = x + linear(y, lw["attn_proj_w"], lw["attn_proj_b"])
    h = layer_norm(x, lw["ln2_g"], lw["ln2_b"], eps)
    f = (gelu if act is None else act)(linear(h, lw["fc_w"], lw["fc_b"]))
    x = x + linear(f, lw["mlp_proj_w"], lw["mlp_proj_b"])
    return x


def embed(weights: Dict[str, object], ids: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Token plus learned position embedding: wte[ids] + wpe[0..T-1]
    ([P1] section 4.1 forward steps 1; [P3] section 1.2, learned positions;
    [P4] section 2.1)."""
    T = ids.shape[1]
    wte = np.asarray(weights["wte"], dtype=dtype)
    wpe = np.asarray(weights["wpe"], dtype=dtype)
    return wte[ids] + wpe[:T][None, :, :]


def _as(d: Dict[str, np.ndarray], dtype) -> Dict[str, np.ndarray]:
    return {k: np.asarray(v, dtype=dtype) for k, v in d.items()}


def hidden_states(weights: Dict[str, object], ids: np.ndarray, n_head: int,
                  dtype=np.float64, eps: float = LN_EPS, act=None) -> np.ndarray:
    """Residual stream after every block, then ln_f: returns [B,T,C]
    ([P1] section 4.1 forward steps 1-3). `act` is the MLP activation
    (None: gelu, the exact form)."""
    x = embed(weights, ids, dtype)
    for lw in weights["layers"]:
        x = block(x, _as(lw, dtype), n_head, eps, act)
    return layer_norm(x, np.asarray(weights["lnf_g"], dtype), np.asarray(weights["lnf_b"], dtype), eps)


def forward(weights: Dict[str, object], ids: np.ndarray, n_head: int,
            dtype=np.float64, eps: float = LN_EPS, act=None) -> np.ndarray:
    """Logits [B,T,V] = ln_f(x) wte^T, the lm_head tied to the token
    embedding with no bias ([P1] sections 2.2 and 4.1 step 4; [P4] section
    2.1 weight tying)."""
    hf = hidden_states(weights, ids, n_head, dtype, eps, act)
    return hf @ np.asarray(weights["wte"], dtype).T


def logsumexp_last(z: np.ndarray) -> np.ndarray:
    """log sum_j exp(z_j) over the last axis, max-subtracted."""
    m = z.max(axis=-1)
    return m + np.log(np.exp(z - m[..., None]).sum(axis=-1))


def shifted_cross_entropy(logits: np.ndarray, ids: np.ndarray,
                          lengths: Optional[np.ndarray] = None) -> Tuple[float, np.ndarray]:
    """Next-token cross-entropy, mean over the scored positions.

    [P1] section 4.1 step 5: logits[..., :-1, :] against labels[..., 1:],
    CrossEntropyLoss with its default mean reduction; [P4] section 3.3: the
    target sequence is the input shifted by one. For right-padded sequences
    of valid length n, positions t >= n-1 have no target and are left out
    (the reading this build takes; the pages do not pad).

    Returns (loss, token_loss) where token_loss[b, t] is the loss of
    position t (NaN where not scored).
    """
    B, T, V = logits.shape
    if lengths is None:
        lengths = np.full(B, T, dtype=np.int64)
    z = logits[:, :-1, :]
    y = ids[:, 1:]
    lse = logsumexp_last(z)
    zt = np.take_along_axis(z, y[..., None].astype(np.int64), axis=-1)[..., 0]
    per = lse - zt
    token_loss = np.full((B, T), np.nan, dtype=np.float64)
    valid = np.zeros((B, T), dtype=bool)
    for b in range(B):
        n = int(lengths[b])
        if n > 1:
            token_loss[b, : n - 1] = per[b, : n - 1]
            valid[b, : n - 1] = True
    count = int(valid.sum())
    loss = float(token_loss[valid].sum() / count) if count else float("nan")
    return loss, token_loss
