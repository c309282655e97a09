"""Pins of the backward oracle (oracle/gpt2_backward.py) to things other
than itself (no GPU needed).

* Central finite differences of the forward oracle's loss, element by
  element over every weight of tiny models: the gradcheck of "Hand-writing
  GPT-2 from scratch: the Transformer decoder core modules in PyTorch",
  section 5.2 (double precision, step 1e-6), here over the whole model
  rather than one module.
* torch fp64 autograd through a forward built from torch's own routines
  (embedding lookup, F.layer_norm, F.linear, scaled_dot_product_attention
  with is_causal, F.gelu, F.cross_entropy with ignored targets).
* Invariants and special cases: each scored row of the logits gradient sums
  to 0 and is negative only at its target; LayerNorm's input gradient is
  orthogonal to the ones vector (the output does not change when x is
  shifted) and its product with the centred input is the closed form of
  the derivative along a scaling of x; T = 1 attention passes dy to v
  and nothing to q or k; GELU's derivative at 0 is 1/2.
* Planted mistakes (on the CPU, in the oracle): each must fail a pin.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

import synthetic
from oracle import gpt2_backward as B
from oracle import gpt2_oracle as O


def tiny_case(seed=3, L=1, H=2, C=8, V=13, T=5, nb=2, lengths=(5, 3), init="dist"):
    w = synthetic.random_case(seed, L, H, C, V, 8, nb, T, dtype="fp32", init=init, lengths=lengths)
    W = synthetic.make_weights(w)
    # larger weights than the 0.02 init, so every term of the gradient matters
    rng = np.random.default_rng(seed)
    for lw in W["layers"]:
        for k in ("attn_w", "attn_proj_w", "fc_w", "mlp_proj_w"):
            lw[k] = lw[k] * 20.0
    W["wte"] = W["wte"] + rng.standard_normal(W["wte"].shape).astype(np.float32) * 0.5
    W["wpe"] = W["wpe"] + rng.standard_normal(W["wpe"].shape).astype(np.float32) * 0.5
    return w, W, synthetic.make_ids(w), synthetic.lengths_of(w)


def _loss(W, ids, n_head, lengths, act):
    f = O.gelu if act == "erf" else O.gelu_tanh
    z = O.forward(W, ids, n_head, act=f)
    return O.shifted_cross_entropy(z, ids, lengths)[0]


def _tensors(W):
    """(name, array) of every weight tensor, as float64 copies in place in W."""
    out = [("wte", W, "wte"), ("wpe", W, "wpe"), ("lnf_g", W, "lnf_g"), ("lnf_b", W, "lnf_b")]
    for i, lw in enumerate(W["layers"]):
        for k in synthetic.LAYER_KEYS:
            out.append((f"layers.{i}.{k}", lw, k))
    return out


def _grad_of(grads, name):
    if name.startswith("layers."):
        _, i, k = name.split(".")
        return grads["layers"][int(i)][k]
    return grads[name]


def finite_difference_check(w, W, ids, lengths, act="erf", h=1e-6, rtol=1e-6, atol=1e-9):
    Wd = {"wte": np.asarray(W["wte"], np.float64).copy(), "wpe": np.asarray(W["wpe"], np.float64).copy(),
          "lnf_g": np.asarray(W["lnf_g"], np.float64).copy(), "lnf_b": np.asarray(W["lnf_b"], np.float64).copy(),
          "layers": [{k: np.asarray(v, np.float64).copy() for k, v in lw.items()} for lw in W["layers"]]}
    _, grads = B.forward_backward(Wd, ids, w.n_head, lengths, act=act)
    worst = 0.0
    for name, holder, key in _tensors(Wd):
        a = holder[key]
        g = _grad_of(grads, name)
        assert g.shape == a.shape, name
        num = np.empty_like(a)
        flat, nflat = a.reshape(-1), num.reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            flat[i] = v + h
            lp = _loss(Wd, ids, w.n_head, lengths, act)
            flat[i] = v - h
            lm = _loss(Wd, ids, w.n_head, lengths, act)
            flat[i] = v
            nflat[i] = (lp - lm) / (2 * h)
        err = np.abs(num - g)
        bound = atol + rtol * np.abs(num).max()
        worst = max(worst, float(err.max() / bound))
        assert err.max() <= bound, (name, float(err.max()), float(np.abs(num).max()))
    return worst


@pytest.mark.parametrize("act", ["erf", "tanh"])
def test_gradients_equal_central_finite_differences(act):
    w, W, ids, lengths = tiny_case()
    finite_difference_check(w, W, ids, lengths, act=act)


def test_finite_differences_two_layers_repeated_tokens():
    """Two blocks, and a token that occurs several times (its wte row gathers
    every occurrence plus the head term)."""
    w, W, ids, lengths = tiny_case(seed=5, L=2, H=2, C=8, V=7, T=6, nb=2, lengths=(6, 6))
    ids[0, :3] = 4
    ids[1, 2] = 4
    finite_difference_check(w, W, ids, lengths)


# ---------------------------------------------------------------- torch fp64 autograd

def _torch_loss(W, ids, n_head, lengths, act):
    t = {k: torch.tensor(np.asarray(W[k], np.float64), requires_grad=True) for k in ("wte", "wpe", "lnf_g", "lnf_b")}
    tl = [{k: torch.tensor(np.asarray(v, np.float64), requires_grad=True) for k, v in lw.items()} for lw in W["layers"]]
    idt = torch.tensor(ids, dtype=torch.long)
    Bn, T = ids.shape
    C = t["wte"].shape[1]
    x = TF.embedding(idt, t["wte"]) + t["wpe"][:T][None]
    for lw in tl:
        h = TF.layer_norm(x, (C,), lw["ln1_g"], lw["ln1_b"], 1e-5)
        qkv = TF.linear(h, lw["attn_w"], lw["attn_b"])
        q, k, v = qkv.split(C, dim=-1)
        sh = lambda a: a.view(Bn, T, n_head, C // n_head).transpose(1, 2)
        y = TF.scaled_dot_product_attention(sh(q), sh(k), sh(v), is_causal=True)
        y = y.transpose(1, 2).reshape(Bn, T, C)
        x = x + TF.linear(y, lw["attn_proj_w"], lw["attn_proj_b"])
        h = TF.layer_norm(x, (C,), lw["ln2_g"], lw["ln2_b"], 1e-5)
        f = TF.gelu(TF.linear(h, lw["fc_w"], lw["fc_b"]), approximate="none" if act == "erf" else "tanh")
        x = x + TF.linear(f, lw["mlp_proj_w"], lw["mlp_proj_b"])
    hf = TF.layer_norm(x, (C,), t["lnf_g"], t["lnf_b"], 1e-5)
    z = hf @ t["wte"].T
    tgt = torch.full((Bn, T), -100, dtype=torch.long)
    for b in range(Bn):
        n = int(lengths[b])
        tgt[b, : n - 1] = idt[b, 1:n]
    loss = TF.cross_entropy(z.reshape(-1, z.shape[-1]), tgt.reshape(-1), ignore_index=-100)
    loss.backward()
    grads = {k: t[k].grad.numpy() for k in t}
    grads["layers"] = [{k: v.grad.numpy() for k, v in lw.items()} for lw in tl]
    return float(loss.item()), grads


@pytest.mark.parametrize("act", ["erf", "tanh"])
def test_gradients_equal_torch_autograd(act):
    w = synthetic.random_case(17, 2, 4, 64, 300, 64, 3, 24, dtype="fp32", lengths=(24, 7, 17))
    W = synthetic.make_weights(w)
    ids = synthetic.make_ids(w)
    lengths = synthetic.lengths_of(w)
    loss, g = B.forward_backward(W, ids, w.n_head, lengths, act=act)
    tloss, tg = _torch_loss(W, ids, w.n_head, lengths, act)
    assert abs(loss - tloss) <= 1e-12
    for name, _, _ in _tensors(W):
        a, r = _grad_of(g, name), _grad_of(tg, name)
        assert np.abs(a - r).max() <= 1e-10 * max(1.0, np.abs(r).max()), name


# ---------------------------------------------------------------- invariants, special cases

def test_logits_gradient_rows_sum_to_zero_and_point_at_target():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((2, 6, 40)) * 3
    ids = rng.integers(0, 40, size=(2, 6))
    lengths = np.array([6, 4])
    dz = B.shifted_cross_entropy_backward(z, ids, lengths)
    sc = B.scored_mask(ids, lengths)
    assert int(sc.sum()) == 5 + 3
    assert np.abs(dz.sum(-1)).max() <= 1e-15
    assert (dz[~sc] == 0).all()
    for b, t in zip(*np.nonzero(sc)):
        row = dz[b, t]
        assert row[ids[b, t + 1]] < 0 and (np.delete(row, ids[b, t + 1]) > 0).all()
        # magnitude of the target entry: (1 - p_target) / n_scored
        p = np.exp(z[b, t] - O.logsumexp_last(z[b, t]))
        assert abs(row[ids[b, t + 1]] + (1 - p[ids[b, t + 1]]) / 8) <= 1e-15


def test_layer_norm_gradient_orthogonal_to_shift_and_scale():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7, 33)) * 2 + 3
    g = rng.standard_normal(33)
    dy = rng.standard_normal((5, 7, 33))
    dx, dg, db = B.layer_norm_backward(x, g, dy)
    xc = x - x.mean(-1, keepdims=True)
    var = (xc ** 2).mean(-1)
    xh = xc / np.sqrt(var + 1e-5)[..., None]
    # shifting x leaves the output unchanged: dx . 1 = 0
    assert np.abs(dx.sum(-1)).max() <= 1e-12
    # scaling the centred input by a: d/da of the output at a = 1 is xh eps / (var + eps),
    # so dx . xc = eps / (var + eps) * sum(dy g xh) (0 when eps = 0)
    want = 1e-5 / (var + 1e-5) * (dy * g * xh).sum(-1)
    assert np.abs((dx * xc).sum(-1) - want).max() <= 1e-12
    assert np.allclose(db, dy.reshape(-1, 33).sum(0), rtol=0, atol=1e-12)


def test_attention_gradient_single_position():
    rng = np.random.default_rng(2)
    qkv = rng.standard_normal((3, 1, 3 * 16))
    dy = rng.standard_normal((3, 1, 16))
    d = B.causal_self_attention_backward(qkv, 2, dy)
    assert np.abs(d[:, :, :32]).max() == 0.0          # one key: softmax is constant 1
    assert np.array_equal(d[:, :, 32:], dy)


def test_gelu_derivative_values():
    u = np.array([0.0, 8.0, -8.0, 1.0])
    d = B.gelu_backward(u, np.ones_like(u))
    assert abs(d[0] - 0.5) <= 1e-15 and abs(d[1] - 1.0) <= 1e-12 and abs(d[2]) <= 1e-12
    # d/du [u Phi(u)] at 1 = Phi(1) + phi(1)
    assert abs(d[3] - (0.5 * (1 + math.erf(1 / math.sqrt(2))) + math.exp(-0.5) / math.sqrt(2 * math.pi))) <= 1e-15
    dt = B.gelu_tanh_backward(u, np.ones_like(u))
    assert abs(dt[0] - 0.5) <= 1e-15 and abs(dt[1] - 1.0) <= 1e-9


def test_embedding_gradient_gathers_repeats_and_positions():
    ids = np.array([[2, 2, 0], [1, 2, 4]])
    dx = np.arange(2 * 3 * 2, dtype=np.float64).reshape(2, 3, 2)
    dwte, dwpe = B.embed_backward(ids, dx, vocab=6, n_ctx=5)
    assert np.array_equal(dwte[2], dx[0, 0] + dx[0, 1] + dx[1, 1])
    assert np.array_equal(dwte[3], np.zeros(2)) and np.array_equal(dwte[5], np.zeros(2))
    assert np.array_equal(dwpe[:3], dx.sum(0)) and (dwpe[3:] == 0).all()


def test_tied_gradient_is_embedding_plus_head_term():
    w, W, ids, lengths = tiny_case()
    tr = {}
    _, g = B.forward_backward(W, ids, w.n_head, lengths, trace=tr)
    assert np.array_equal(g["wte"], tr["dwte_head"] + tr["dwte_embed"])
    assert np.abs(tr["dwte_head"]).max() > 0 and np.abs(tr["dwte_embed"]).max() > 0


# ---------------------------------------------------------------- planted mistakes

def _mutants():
    def ln_no_projection(x, gamma, dy, eps=O.LN_EPS):
        mu = x.mean(-1, keepdims=True)
        r = 1 / np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + eps)
        gx = dy * gamma
        dx = r * (gx - gx.mean(-1, keepdims=True))
        C = x.shape[-1]
        return dx, (dy * (x - mu) * r).reshape(-1, C).sum(0), dy.reshape(-1, C).sum(0)

    def attn_no_scale(qkv, n_head, dy):
        D = qkv.shape[-1] // 3 // n_head
        out = B_orig["attn"](qkv, n_head, dy)
        out[:, :, : 2 * qkv.shape[-1] // 3] *= math.sqrt(D)
        return out

    def ce_not_averaged(logits, ids, lengths=None):
        return B_orig["ce"](logits, ids, lengths) * max(1, int(B.scored_mask(ids, lengths).sum()))

    def embed_forgets_head_tie(ids, dx, vocab, n_ctx):
        dwte, dwpe = B_orig["embed"](ids, dx, vocab, n_ctx)
        return np.zeros_like(dwte), dwpe

    def gelu_wrong_form(u, dout):
        return B_orig["gelu_tanh"](u, dout * 1.02)

    return {
        "layer_norm_backward": ln_no_projection,
        "causal_self_attention_backward": attn_no_scale,
        "shifted_cross_entropy_backward": ce_not_averaged,
        "embed_backward": embed_forgets_head_tie,
        "gelu_backward": gelu_wrong_form,
    }


B_orig = {"attn": B.causal_self_attention_backward, "ce": B.shifted_cross_entropy_backward,
          "embed": B.embed_backward, "gelu_tanh": B.gelu_tanh_backward}


@pytest.mark.parametrize("fn", sorted(_mutants()))
def test_planted_mistake_fails_finite_differences(fn, monkeypatch):
    monkeypatch.setattr(B, fn, _mutants()[fn])
    w, W, ids, lengths = tiny_case()
    with pytest.raises(AssertionError):
        finite_difference_check(w, W, ids, lengths)
