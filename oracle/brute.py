"""Scalar-loop brute force of the GPT-2 forward pass (test infrastructure only).

Pure Python floats (IEEE double) and the ``math`` module, one scalar at a
time, written independently of ``gpt2_oracle`` so that the two can pin each
other on tiny shapes (the tiny fp32 workload: 2 layers, C=64, T=4, V=512).
Attention here is the per-query loop of the pages' causal rule: query i
visits keys 0..i only, with an explicit exp-sum, instead of a masked score
matrix. Only the tests may import this module.

Sources: "Hand-writing GPT-2 from scratch: the Transformer decoder core
modules in PyTorch" (sections 3.2-3.4, 4.1); "Reproducing GPT-2 124M"
(sections 2.1-2.2).
"""
from __future__ import annotations

import math
from typing import List, Sequence


def _ln(row: Sequence[float], g: Sequence[float], b: Sequence[float], eps: float) -> List[float]:
    n = len(row)
    mu = 0.0
    for v in row:
        mu += v
    mu /= n
    var = 0.0
    for v in row:
        var += (v - mu) * (v - mu)
    var /= n
    inv = 1.0 / math.sqrt(var + eps)
    return [(row[c] - mu) * inv * g[c] + b[c] for c in range(n)]


def _lin(row: Sequence[float], w, bias) -> List[float]:
    out = []
    for o in range(len(w)):
        acc = 0.0
        wo = w[o]
        for c in range(len(row)):
            acc += row[c] * wo[c]
        out.append(acc + (bias[o] if bias is not None else 0.0))
    return out


def _gelu(v: float) -> float:
    return 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0)))


def forward(weights, ids, n_head: int, eps: float = 1e-5):
    """Returns logits as nested lists [B][T][V]."""
    tolist = lambda a: a.tolist() if hasattr(a, "tolist") else a
    wte = tolist(weights["wte"])
    wpe = tolist(weights["wpe"])
    B = len(ids)
    T = len(ids[0])
    C = len(wte[0])
    D = C // n_head
    layers = [{k: tolist(v) for k, v in lw.items()} for lw in weights["layers"]]
    lnf_g, lnf_b = tolist(weights["lnf_g"]), tolist(weights["lnf_b"])
    logits = []
    for bi in range(B):
        x = [[wte[int(ids[bi][t])][c] + wpe[t][c] for c in range(C)] for t in range(T)]
        for lw in layers:
            qkv = [_lin(_ln(x[t], lw["ln1_g"], lw["ln1_b"], eps), lw["attn_w"], lw["attn_b"]) for t in range(T)]
            y = [[0.0] * C for _ in range(T)]
            for h in range(n_head):
                qo, ko, vo = h * D, C + h * D, 2 * C + h * D
                for i in range(T):
                    scores = []
                    for j in range(i + 1):           # keys 0..i only
                        s = 0.0
                        for d in range(D):
                            s += qkv[i][qo + d] * qkv[j][ko + d]
                        scores.append(s / math.sqrt(D))
                    mx = max(scores)
                    ex = [math.exp(s - mx) for s in scores]
                    den = sum(ex)
                    for d in range(D):
                        acc = 0.0
                        for j in range(i + 1):
                            acc += ex[j] / den * qkv[j][vo + d]
                        y[i][h * D + d] = acc
            for t in range(T):
                a = _lin(y[t], lw["attn_proj_w"], lw["attn_proj_b"])
                x[t] = [x[t][c] + a[c] for c in range(C)]
            for t in range(T):
                f = [_gelu(v) for v in _lin(_ln(x[t], lw["ln2_g"], lw["ln2_b"], eps), lw["fc_w"], lw["fc_b"])]
                m = _lin(f, lw["mlp_proj_w"], lw["mlp_proj_b"])
                x[t] = [x[t][c] + m[c] for c in range(C)]
        rows = []
        for t in range(T):
            hf = _ln(x[t], lnf_g, lnf_b, eps)
            rows.append(_lin(hf, wte, None))
        logits.append(rows)
    return logits


def shifted_cross_entropy(logits, ids, lengths=None):
    """Mean over scored positions of log-sum-exp minus the next-token logit."""
    B = len(logits)
    T = len(logits[0])
    total, count = 0.0, 0
    for b in range(B):
        n = T if lengths is None else int(lengths[b])
        for t in range(n - 1):
            z = logits[b][t]
            mx = max(z)
            s = 0.0
            for v in z:
                s += math.exp(v - mx)
            total += mx + math.log(s) - z[int(ids[b][t + 1])]
            count += 1
    return total / count
