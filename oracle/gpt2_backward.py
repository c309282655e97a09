"""CPU oracle of the GPT-2 backward pass (test infrastructure only).

The gradient of the mean shifted cross-entropy with respect to every weight
of the model, in fp64 NumPy, by the chain rule applied step by step to the
forward pass of ``gpt2_oracle`` in reverse order. Like the forward oracle it
exists only to check the CUDA path: only the tests, the smoke check and the
bench's CPU-baseline leg may import it, and it shares no code with the CUDA
path.

The pages train the model with loss.backward() followed by gradient
clipping ("Hand-writing GPT-2 from scratch: the Transformer decoder core
modules in PyTorch", section 4.3) and check hand-written modules against
finite differences with torch.autograd.gradcheck in double precision
(section 5.2). The tied lm_head (the same page, section 2.2: lm_head.weight
is wte.weight) makes the gradient of wte the sum of two terms: the token
embedding's scatter of the residual gradient into the rows of the ids, and
the lm_head's product of the logits gradient with the final hidden state.

Each function is the derivative of one forward step, written out:

* cross-entropy: d loss / d z = (softmax(z) - onehot(target)) / n_scored at
  scored positions, 0 elsewhere;
* tied head z = hf wte^T: d hf = dz wte, d wte += dz^T hf;
* LayerNorm y = g (x - mu) r + b with r = (var + eps)^-1/2 (biased var):
  with xh = (x - mu) r and gx = dy g,
  dx = r (gx - mean_c(gx) - xh mean_c(gx xh)), dg = sum_tokens dy xh,
  db = sum_tokens dy;
* Linear y = x W^T + b: dx = dy W, dW = dy^T x, db = sum_tokens dy;
* exact GELU g(u) = u Phi(u): g'(u) = Phi(u) + u phi(u);
  tanh form g(u) = u (1 + tanh(k (u + c u^3))) / 2:
  g'(u) = (1 + t) / 2 + u (1 - t^2) k (1 + 3 c u^2) / 2;
* attention per sequence and head, S = q k^T / sqrt(D) masked, P = softmax(S),
  y = P v: dv = P^T dy, dP = dy v^T, dS = P (dP - rowsum(dP P)),
  dq = dS k / sqrt(D), dk = dS^T q / sqrt(D);
* embedding x = wte[ids] + wpe[t]: dwte[id] += dx, dwpe[t] += sum_b dx.

Pins (tests/test_oracle_backward_pins.py): central finite differences of
the forward oracle's loss (the gradcheck of section 5.2, on every weight of
tiny models), torch fp64 autograd through a forward composed of torch's own
library routines, invariants (the logits gradient of each scored row sums
to 0, LayerNorm's input gradient is orthogonal to 1 and has the closed-form
product with the centred input), and planted mistakes that the pins must
catch.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np
from scipy.special import erf as _erf

from . import gpt2_oracle as F

GELU_TANH_K = math.sqrt(2.0 / math.pi)
GELU_TANH_C = 0.044715


def layer_norm_backward(x: np.ndarray, gamma: np.ndarray, dy: np.ndarray,
                        eps: float = F.LN_EPS) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of LayerNorm over the last axis (biased variance, eps inside
    the square root; "Reproducing GPT-2 124M", section 2.1). x, dy: [..., C].
    Returns (dx, dgamma, dbeta), dgamma and dbeta summed over every token."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(var + eps)
    xh = (x - mu) * r
    gx = dy * gamma
    dx = r * (gx - gx.mean(axis=-1, keepdims=True) - xh * (gx * xh).mean(axis=-1, keepdims=True))
    C = x.shape[-1]
    dgamma = (dy * xh).reshape(-1, C).sum(axis=0)
    dbeta = dy.reshape(-1, C).sum(axis=0)
    return dx, dgamma, dbeta


def linear_backward(x: np.ndarray, w: np.ndarray, dy: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of nn.Linear y = x W^T + b (W [out, in]): (dx, dW, db)."""
    dx = dy @ w
    dw = dy.reshape(-1, dy.shape[-1]).T @ x.reshape(-1, x.shape[-1])
    db = dy.reshape(-1, dy.shape[-1]).sum(axis=0)
    return dx, dw, db


def gelu_backward(u: np.ndarray, dout: np.ndarray) -> np.ndarray:
    """d gelu(u) / du times dout for the exact form u Phi(u) ("GPT-2
    architecture analysis and implementation guide", section 2.2, F.gelu)."""
    phi_cdf = 0.5 * (1.0 + _erf(u / math.sqrt(2.0)))
    phi_pdf = np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    return dout * (phi_cdf + u * phi_pdf)


def gelu_tanh_backward(u: np.ndarray, dout: np.ndarray) -> np.ndarray:
    """Derivative of the tanh-form GELU ("Hand-writing GPT-2 from scratch:
    the Transformer decoder core modules in PyTorch", section 3.4) times dout."""
    t = np.tanh(GELU_TANH_K * (u + GELU_TANH_C * u ** 3))
    return dout * (0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * GELU_TANH_K * (1.0 + 3.0 * GELU_TANH_C * u * u))


def causal_self_attention_backward(qkv: np.ndarray, n_head: int, dy: np.ndarray) -> np.ndarray:
    """Gradient with respect to the c_attn output qkv [B, T, 3C] of the
    masked multi-head attention of gpt2_oracle.causal_self_attention, given
    dy [B, T, C] (heads concatenated). The probabilities are recomputed from
    qkv exactly as the forward computes them."""
    B, T, C3 = qkv.shape
    C = C3 // 3
    D = C // n_head
    scale = 1.0 / math.sqrt(D)
    q = qkv[:, :, 0:C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    k = qkv[:, :, C:2 * C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    v = qkv[:, :, 2 * C:3 * C].reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    g = dy.reshape(B, T, n_head, D).transpose(0, 2, 1, 3)
    mask = F.causal_mask(T)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for b in range(B):
        s = (q[b] @ k[b].transpose(0, 2, 1)) * scale
        s = np.where(mask, -np.inf, s)
        p = F.softmax_last(s)                                  # [H, T, T]
        dv[b] = p.transpose(0, 2, 1) @ g[b]
        dp = g[b] @ v[b].transpose(0, 2, 1)
        ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))   # masked entries have p = 0
        dq[b] = (ds @ k[b]) * scale
        dk[b] = (ds.transpose(0, 2, 1) @ q[b]) * scale
    out = np.empty_like(qkv)
    out[:, :, 0:C] = dq.transpose(0, 2, 1, 3).reshape(B, T, C)
    out[:, :, C:2 * C] = dk.transpose(0, 2, 1, 3).reshape(B, T, C)
    out[:, :, 2 * C:3 * C] = dv.transpose(0, 2, 1, 3).reshape(B, T, C)
    return out


def scored_mask(ids: np.ndarray, lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """[B, T] bool: position t of sequence b has a next-token target
    (t + 1 < length[b]), the positions the loss averages over."""
    B, T = ids.shape
    if lengths is None:
        lengths = np.full(B, T, dtype=np.int64)
    return np.arange(T)[None, :] + 1 < np.asarray(lengths)[:, None]


def shifted_cross_entropy_backward(logits: np.ndarray, ids: np.ndarray,
                                   lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """d loss / d logits [B, T, V] for the mean next-token cross-entropy of
    gpt2_oracle.shifted_cross_entropy ("Hand-writing GPT-2 from scratch: the
    Transformer decoder core modules in PyTorch", section 4.1 step 5): at a
    scored position (softmax(z) - onehot(ids[t + 1])) / n_scored, 0 at the
    others."""
    B, T, V = logits.shape
    sc = scored_mask(ids, lengths)
    n = int(sc.sum())
    dz = np.zeros_like(logits)
    if n == 0:
        return dz
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    p = e / e.sum(axis=-1, keepdims=True)
    for b in range(B):
        for t in range(T):
            if sc[b, t]:
                dz[b, t] = p[b, t]
                dz[b, t, ids[b, t + 1]] -= 1.0
    return dz / n


def embed_backward(ids: np.ndarray, dx: np.ndarray, vocab: int, n_ctx: int) -> Tuple[np.ndarray, np.ndarray]:
    """Gradients of x = wte[ids] + wpe[0..T-1] ("Hand-writing GPT-2 from
    scratch: the Transformer decoder core modules in PyTorch", section 4.1
    step 1): the rows of dx added into the rows of their token ids (a token
    seen twice gets both), and summed over the batch into the first T rows
    of the position table."""
    B, T, C = dx.shape
    dwte = np.zeros((vocab, C), dtype=dx.dtype)
    np.add.at(dwte, ids.reshape(-1), dx.reshape(-1, C))
    dwpe = np.zeros((n_ctx, C), dtype=dx.dtype)
    dwpe[:T] = dx.sum(axis=0)
    return dwte, dwpe


def forward_backward(weights: Dict[str, object], ids: np.ndarray, n_head: int,
                     lengths: Optional[np.ndarray] = None, act: str = "erf",
                     dtype=np.float64, eps: float = F.LN_EPS, trace: Optional[dict] = None):
    """Loss and gradients of every weight, [P1] section 4.3's
    loss.backward() written out.

    Runs the forward of gpt2_oracle keeping what the backward needs (the
    residual stream entering each LayerNorm, the LayerNorm outputs, qkv, the
    attention output, the c_fc output before GELU), then walks back through
    the tied head, ln_f, the blocks in reverse order and the embedding.

    Returns (loss, grads) with grads shaped like `weights` ("wte", "wpe",
    "layers": [{LAYER_KEYS}], "lnf_g", "lnf_b"). The wte gradient is the sum
    of the lm_head and token-embedding terms. If `trace` is a dict it
    receives the intermediates (forward activations and their gradients) for
    step-by-step comparisons.
    """
    fgelu = F.gelu if act == "erf" else F.gelu_tanh
    bgelu = gelu_backward if act == "erf" else gelu_tanh_backward
    W = weights
    V, C = np.asarray(W["wte"]).shape
    n_ctx = np.asarray(W["wpe"]).shape[0]
    wte = np.asarray(W["wte"], dtype)
    layers = [{k: np.asarray(v, dtype) for k, v in lw.items()} for lw in W["layers"]]
    lnf_g = np.asarray(W["lnf_g"], dtype)
    lnf_b = np.asarray(W["lnf_b"], dtype)

    # ---- forward, keeping the activations
    x = F.embed(W, ids, dtype)
    saved = []
    for lw in layers:
        x_in = x
        h1 = F.layer_norm(x_in, lw["ln1_g"], lw["ln1_b"], eps)
        qkv = F.linear(h1, lw["attn_w"], lw["attn_b"])
        y = F.causal_self_attention(qkv, n_head)
        x_mid = x_in + F.linear(y, lw["attn_proj_w"], lw["attn_proj_b"])
        h2 = F.layer_norm(x_mid, lw["ln2_g"], lw["ln2_b"], eps)
        u = F.linear(h2, lw["fc_w"], lw["fc_b"])
        f = fgelu(u)
        x = x_mid + F.linear(f, lw["mlp_proj_w"], lw["mlp_proj_b"])
        saved.append(dict(x_in=x_in, h1=h1, qkv=qkv, y=y, x_mid=x_mid, h2=h2, u=u, f=f))
    x_final = x
    hf = F.layer_norm(x_final, lnf_g, lnf_b, eps)
    z = hf @ wte.T
    loss, _ = F.shifted_cross_entropy(z, ids, lengths)

    # ---- backward
    dz = shifted_cross_entropy_backward(z, ids, lengths)
    dhf = dz @ wte
    dwte_head = dz.reshape(-1, V).T @ hf.reshape(-1, C)
    dx, dlnf_g, dlnf_b = layer_norm_backward(x_final, lnf_g, dhf, eps)
    if trace is not None:
        trace.update(z=z, dz=dz, hf=hf, dhf=dhf, x_final=x_final, dx_final=dx, layers=[])
    grads_layers = [None] * len(layers)
    for li in range(len(layers) - 1, -1, -1):
        lw, s = layers[li], saved[li]
        g = {}
        # x = x_mid + c_proj(gelu(c_fc(ln_2(x_mid))))
        dff, g["mlp_proj_w"], g["mlp_proj_b"] = linear_backward(s["f"], lw["mlp_proj_w"], dx)
        du = bgelu(s["u"], dff)
        dh2, g["fc_w"], g["fc_b"] = linear_backward(s["h2"], lw["fc_w"], du)
        dx_ln2, g["ln2_g"], g["ln2_b"] = layer_norm_backward(s["x_mid"], lw["ln2_g"], dh2, eps)
        dx_mid = dx + dx_ln2
        # x_mid = x_in + c_proj(attn(c_attn(ln_1(x_in))))
        dy, g["attn_proj_w"], g["attn_proj_b"] = linear_backward(s["y"], lw["attn_proj_w"], dx_mid)
        dqkv = causal_self_attention_backward(s["qkv"], n_head, dy)
        dh1, g["attn_w"], g["attn_b"] = linear_backward(s["h1"], lw["attn_w"], dqkv)
        dx_ln1, g["ln1_g"], g["ln1_b"] = layer_norm_backward(s["x_in"], lw["ln1_g"], dh1, eps)
        if trace is not None:
            trace["layers"].insert(0, dict(s, dx_out=dx, df=dff, du=du, dh2=dh2, dx_mid=dx_mid, dy=dy,
                                           dqkv=dqkv, dh1=dh1, dx_in=dx_mid + dx_ln1))
        dx = dx_mid + dx_ln1
        grads_layers[li] = g
    dwte_emb, dwpe = embed_backward(ids, dx, V, n_ctx)
    if trace is not None:
        trace.update(dx_embed=dx, dwte_head=dwte_head, dwte_embed=dwte_emb)
    grads = {"wte": dwte_head + dwte_emb, "wpe": dwpe, "layers": grads_layers, "lnf_g": dlnf_g, "lnf_b": dlnf_b}
    return loss, grads
