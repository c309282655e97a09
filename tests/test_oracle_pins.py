"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a brute force, a library routine, a
closed form, an invariant the pages state, or a value the pages print
(tests/golden/page_values.json). The mutation tests at the end plant
plausible mistakes in the oracle (on the CPU) and check that a pin catches
each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synthetic
from oracle import brute
from oracle import gpt2_oracle as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_values.json")))


def tiny():
    w = synthetic.WORKLOADS[0]
    return w, synthetic.make_weights(w), synthetic.make_ids(w)


def small_case(seed=7, L=2, H=4, C=64, V=300, T=24, B=2, init="dist"):
    w = synthetic.random_case(seed, L, H, C, V, 64, B, T, dtype="fp32", init=init)
    return w, synthetic.make_weights(w), synthetic.make_ids(w)


# --------------------------------------------------------------------------
# brute force


def test_oracle_equals_scalar_loop_brute_force_tiny():
    w, W, ids = tiny()
    z = O.forward(W, ids, w.n_head)
    zb = np.asarray(brute.forward(W, ids.tolist(), w.n_head))
    assert z.shape == (w.batch, w.seq, w.vocab)
    scale = np.abs(zb).max()
    assert np.abs(z - zb).max() <= 1e-12 * max(scale, 1.0)
    loss, _ = O.shifted_cross_entropy(z, ids)
    lb = brute.shifted_cross_entropy(zb.tolist(), ids.tolist())
    assert abs(loss - lb) <= 1e-12


def test_oracle_equals_brute_force_with_padding():
    w, W, ids = small_case(seed=11, L=1, H=2, C=32, V=97, T=6, B=3)
    lengths = np.array([6, 2, 4])
    z = O.forward(W, ids, w.n_head)
    zb = np.asarray(brute.forward(W, ids.tolist(), w.n_head))
    assert np.abs(z - zb).max() <= 1e-12
    loss, tok = O.shifted_cross_entropy(z, ids, lengths)
    lb = brute.shifted_cross_entropy(zb.tolist(), ids.tolist(), lengths.tolist())
    assert abs(loss - lb) <= 1e-12
    assert np.isnan(tok[1, 1:]).all() and np.isfinite(tok[1, 0])
    assert int(np.isfinite(tok).sum()) == 5 + 1 + 3


# --------------------------------------------------------------------------
# library routines (torch fp64 on the CPU)


def test_layer_norm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7, 96)) * 3 + 1.5
    g = rng.standard_normal(96)
    b = rng.standard_normal(96)
    ref = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b), eps=1e-5).numpy()
    assert np.abs(O.layer_norm(x, g, b) - ref).max() <= 1e-12


def test_attention_matches_torch_sdpa_causal():
    rng = np.random.default_rng(1)
    B, T, H, D = 2, 37, 3, 16
    C = H * D
    qkv = rng.standard_normal((B, T, 3 * C))
    y = O.causal_self_attention(qkv, H)
    t = torch.from_numpy(qkv)
    q, k, v = t.split(C, dim=2)
    q, k, v = (a.view(B, T, H, D).transpose(1, 2) for a in (q, k, v))
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B, T, C).numpy()
    assert np.abs(y - ref).max() <= 1e-12


def test_gelu_matches_math_erf_and_torch():
    xs = np.linspace(-8, 8, 161)
    g = O.gelu(xs)
    ref = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in xs])
    assert np.abs(g - ref).max() <= 1e-15 * 8
    ref2 = F.gelu(torch.from_numpy(xs), approximate="none").numpy()
    assert np.abs(g - ref2).max() <= 1e-14
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([10.0]))[0] - 10.0) < 1e-12
    assert abs(O.gelu(np.array([-10.0]))[0]) < 1e-12
    # hand check of the pages (all-ones weights and input): c_fc output is C*1+b
    C = 8
    pre = np.ones((1, C)) @ np.ones((4 * C, C)).T
    assert np.allclose(O.gelu(pre), 0.5 * C * (1 + math.erf(C / math.sqrt(2))), atol=0, rtol=1e-15)


def test_gelu_tanh_matches_torch_and_its_identities():
    xs = np.linspace(-8, 8, 161)
    g = O.gelu_tanh(xs)
    # library routine: torch's tanh-approximate GELU in fp64
    ref = F.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    assert np.abs(g - ref).max() <= 1e-14
    # 0.5 x (1 + tanh u) is odd-symmetric around x/2: g(x) - g(-x) = x exactly
    assert np.abs((g - O.gelu_tanh(-xs)) - xs).max() <= 1e-14
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    # it approximates the exact form to within 5e-4 (and is not identical to it)
    d = np.abs(g - O.gelu(xs))
    assert d.max() <= 5e-4 and d.max() >= 1e-5


def test_sinusoidal_wpe_closed_forms():
    n_ctx, C = 64, 16
    pe = O.sinusoidal_wpe(n_ctx, C)
    assert pe.shape == (n_ctx, C)
    # position 0: sin 0 = 0 in even columns, cos 0 = 1 in odd columns
    assert np.array_equal(pe[0], np.tile([0.0, 1.0], C // 2))
    # pair i = 0 has frequency 1: columns 0 and 1 are sin(pos), cos(pos)
    pos = np.arange(n_ctx)
    assert np.abs(pe[:, 0] - np.sin(pos)).max() <= 1e-15
    assert np.abs(pe[:, 1] - np.cos(pos)).max() <= 1e-15
    # every (sin, cos) pair lies on the unit circle
    assert np.abs(pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2 - 1.0).max() <= 1e-14
    # the angle of pair i at position 1 is 10000^(-2i/C): a geometric progression
    ang = np.arctan2(pe[1, 0::2], pe[1, 1::2])
    assert np.allclose(ang[1:] / ang[:-1], 10000.0 ** (-2.0 / C), rtol=1e-12, atol=0)
    assert abs(ang[0] - 1.0) <= 1e-15


def test_cross_entropy_matches_torch():
    rng = np.random.default_rng(2)
    B, T, V = 3, 9, 41
    z = rng.standard_normal((B, T, V)) * 4
    ids = rng.integers(0, V, size=(B, T))
    loss, tok = O.shifted_cross_entropy(z, ids)
    ref = F.cross_entropy(torch.from_numpy(z[:, :-1].reshape(-1, V)), torch.from_numpy(ids[:, 1:].reshape(-1)))
    assert abs(loss - float(ref)) <= 1e-12
    assert np.isnan(tok[:, -1]).all()


def test_full_model_matches_torch_library_composition():
    """The whole forward against torch library modules (fp64, CPU) on a shape
    too large for the brute force: 4 heads, T=48, two layers."""
    w, W, ids = small_case(seed=5, L=2, H=4, C=64, V=300, T=48, B=2)
    z = O.forward(W, ids, w.n_head)
    tt = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    C, H, D, T = w.n_embd, w.n_head, w.d_head, w.seq
    x = tt(W["wte"])[torch.from_numpy(ids.astype(np.int64))] + tt(W["wpe"])[:T]
    for lw in W["layers"]:
        h = F.layer_norm(x, (C,), tt(lw["ln1_g"]), tt(lw["ln1_b"]), 1e-5)
        q, k, v = F.linear(h, tt(lw["attn_w"]), tt(lw["attn_b"])).split(C, dim=2)
        q, k, v = (a.view(-1, T, H, D).transpose(1, 2) for a in (q, k, v))
        y = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(-1, T, C)
        x = x + F.linear(y, tt(lw["attn_proj_w"]), tt(lw["attn_proj_b"]))
        h = F.layer_norm(x, (C,), tt(lw["ln2_g"]), tt(lw["ln2_b"]), 1e-5)
        x = x + F.linear(F.gelu(F.linear(h, tt(lw["fc_w"]), tt(lw["fc_b"]))), tt(lw["mlp_proj_w"]), tt(lw["mlp_proj_b"]))
    ref = F.linear(F.layer_norm(x, (C,), tt(W["lnf_g"]), tt(W["lnf_b"]), 1e-5), tt(W["wte"])).numpy()
    assert np.abs(z - ref).max() <= 1e-11


# --------------------------------------------------------------------------
# invariants and closed forms


def test_softmax_rows_sum_to_one_and_mask_is_exact():
    rng = np.random.default_rng(3)
    B, T, H, D = 2, 17, 2, 8
    qkv = rng.standard_normal((B, T, 3 * H * D)) * 2
    _, p = O.causal_self_attention(qkv, H, return_probs=True)
    assert np.abs(p.sum(-1) - 1).max() <= 1e-12
    upper = np.triu(np.ones((T, T), bool), 1)
    assert (p[..., upper] == 0).all()
    assert (p[..., ~upper] > 0).all()       # diagonal and past keys are visible


def test_attention_with_zero_queries_is_cumulative_mean():
    """q = 0 makes every visible score equal, so y_i = mean(v_0..v_i):
    the closed form of a causal mask that includes the diagonal."""
    rng = np.random.default_rng(4)
    B, T, H, D = 1, 11, 2, 4
    C = H * D
    qkv = rng.standard_normal((B, T, 3 * C))
    qkv[:, :, :C] = 0
    y = O.causal_self_attention(qkv, H)
    v = qkv[:, :, 2 * C:]
    cm = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None]
    assert np.abs(y - cm).max() <= 1e-13


def test_attention_single_position_returns_v():
    rng = np.random.default_rng(5)
    qkv = rng.standard_normal((3, 1, 3 * 12))
    assert np.array_equal(O.causal_self_attention(qkv, 3), qkv[:, :, 24:])


def test_layer_norm_pre_affine_moments():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((64, 200)) * 0.05 + 0.3
    y = O.layer_norm(x, np.ones(200), np.zeros(200))
    var = x.var(axis=-1)
    assert np.abs(y.mean(-1)).max() <= 1e-13
    assert np.abs(y.var(-1) - var / (var + 1e-5)).max() <= 1e-12


def test_uniform_logits_give_log_vocab():
    """ln_f gamma = beta = 0 makes every logit 0, so the loss is ln V exactly."""
    w, W, ids = tiny()
    W = dict(W)
    W["lnf_g"] = np.zeros_like(W["lnf_g"])
    W["lnf_b"] = np.zeros_like(W["lnf_b"])
    z = O.forward(W, ids, w.n_head)
    assert (z == 0).all()
    loss, _ = O.shifted_cross_entropy(z, ids)
    assert abs(loss - math.log(512)) <= 1e-12
    z2 = np.zeros((1, 3, 50257))
    assert abs(O.shifted_cross_entropy(z2, np.array([[1, 2, 3]]))[0] - math.log(50257)) <= 1e-12


def test_causality_future_tokens_do_not_change_the_past():
    w, W, ids = small_case(seed=9, T=20)
    z = O.forward(W, ids, w.n_head)
    for t in (0, 7, 18):
        ids2 = ids.copy()
        ids2[:, t + 1:] = (ids2[:, t + 1:] + 13) % w.vocab
        z2 = O.forward(W, ids2, w.n_head)
        assert np.array_equal(z[:, : t + 1], z2[:, : t + 1])
        assert not np.array_equal(z[:, t + 1:], z2[:, t + 1:])


def test_lm_head_is_tied_to_wte():
    """Changing one wte row changes the embedding of that token and the
    logit column of that token: the head reads the same buffer."""
    w, W, ids = tiny()
    r = 77
    assert r not in set(ids.ravel().tolist())
    z = O.forward(W, ids, w.n_head)
    W2 = dict(W)
    W2["wte"] = W["wte"].copy()
    W2["wte"][r] += 0.5
    z2 = O.forward(W2, ids, w.n_head)
    changed = np.abs(z2 - z).max(axis=(0, 1)) > 0
    assert changed[r] and changed.sum() == 1    # only column r: token r is never an input
    hf = O.hidden_states(W, ids, w.n_head)
    assert np.allclose(z2[..., r] - z[..., r], hf @ np.full(w.n_embd, 0.5), atol=1e-13)


def test_zero_linear_weights_closed_form():
    """With every Linear weight zero each block adds b_proj + b_mproj to the
    residual stream (attention of a constant v returns v), so the output is
    ln_f(wte[id] + wpe[t] + sum of those biases) wte^T."""
    w, W, ids = small_case(seed=12, L=3, T=10)
    Z = dict(W)
    Z["layers"] = []
    for lw in W["layers"]:
        d = dict(lw)
        for k in ("attn_w", "attn_proj_w", "fc_w", "mlp_proj_w"):
            d[k] = np.zeros_like(lw[k])
        Z["layers"].append(d)
    z = O.forward(Z, ids, w.n_head)
    shift = sum(lw["attn_proj_b"].astype(np.float64) + lw["mlp_proj_b"] for lw in W["layers"])
    x = W["wte"].astype(np.float64)[ids] + W["wpe"][: w.seq] + shift
    mu = x.mean(-1, keepdims=True)
    sd = np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + 1e-5)
    ref = ((x - mu) / sd * W["lnf_g"] + W["lnf_b"]) @ W["wte"].astype(np.float64).T
    assert np.abs(z - ref).max() <= 1e-12


def test_shift_pairs_position_t_with_token_t_plus_1():
    V = 10
    ids = np.array([[3, 1, 4, 1, 5]])
    z = np.full((1, 5, V), -50.0)
    for t in range(4):
        z[0, t, ids[0, t + 1]] = 50.0      # a perfect next-token predictor
    loss, _ = O.shifted_cross_entropy(z, ids)
    assert loss < 1e-40
    assert synthetic.next_token_targets(ids).tolist() == [[1, 4, 1, 5, -1]]


# --------------------------------------------------------------------------
# values printed on the pages


def test_page_demo_output_shape():
    w = synthetic.random_case(21, 1, 2, 16, 50257, 8, 2, 4, dtype="fp32")
    W, ids = synthetic.make_weights(w), synthetic.make_ids(w)
    assert list(O.forward(W, ids, w.n_head).shape) == GOLDEN["demo_output_shape"]["value"]


def test_page_124m_config_and_parameter_count():
    w = synthetic.WORKLOADS[1]
    g = GOLDEN["gpt2_124m_config"]["value"]
    assert (w.vocab, w.n_ctx, w.n_embd, w.n_head, w.n_layer) == (g["vocab"], g["n_ctx"], g["n_embd"], g["n_head"], g["n_layer"])
    C, V, L = w.n_embd, w.vocab, w.n_layer
    per_layer = 2 * C + 3 * C * C + 3 * C + C * C + C + 2 * C + 4 * C * C + 4 * C + 4 * C * C + C
    n = V * C + w.n_ctx * C + L * per_layer + 2 * C
    assert n == 124_439_808
    e = GOLDEN["embedding_plus_head_params_124m"]
    assert abs(2 * V * C - e["value"]) <= e["tolerance"]


def test_page_initial_loss_near_10_9():
    """A random-init 124M model scores about 10.9 ([P4] section 4.4). Run on
    one 64-token prefix of the 124M workload (causality makes a prefix exact)."""
    w = synthetic.WORKLOADS[1]
    W = synthetic.make_weights(w)
    ids = synthetic.make_ids(w)[:1, :64]
    z = O.forward(W, ids, w.n_head)
    loss, _ = O.shifted_cross_entropy(z, ids)
    g = GOLDEN["initial_loss"]
    assert abs(loss - g["value"]) <= g["tolerance"]
    assert O.LN_EPS == GOLDEN["ln_eps"]["value"]


# --------------------------------------------------------------------------
# planted mistakes: each must be caught by a pin above


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_eps_1e6_is_caught(monkeypatch):
    orig = O.layer_norm
    monkeypatch.setattr(O, "layer_norm", lambda x, g, b, eps=1e-5: orig(x, g, b, 1e-6))
    assert _fails(test_layer_norm_matches_torch)
    assert _fails(test_full_model_matches_torch_library_composition)


def test_planted_unbiased_variance_is_caught(monkeypatch):
    def ln_unbiased(x, g, b, eps=1e-5):
        mu = x.mean(-1, keepdims=True)
        var = ((x - mu) ** 2).sum(-1, keepdims=True) / (x.shape[-1] - 1)
        return g * (x - mu) / np.sqrt(var + eps) + b
    monkeypatch.setattr(O, "layer_norm", ln_unbiased)
    assert _fails(test_layer_norm_matches_torch)
    assert _fails(test_layer_norm_pre_affine_moments)


def test_planted_mask_without_diagonal_is_caught(monkeypatch):
    monkeypatch.setattr(O, "causal_mask", lambda T: np.triu(np.ones((T, T), dtype=bool), k=0))
    with np.errstate(invalid="ignore"):
        assert _fails(test_attention_matches_torch_sdpa_causal)
        assert _fails(test_attention_with_zero_queries_is_cumulative_mean)


def test_planted_transposed_mask_is_caught(monkeypatch):
    monkeypatch.setattr(O, "causal_mask", lambda T: np.tril(np.ones((T, T), dtype=bool), k=-1))
    assert _fails(test_attention_matches_torch_sdpa_causal)
    assert _fails(test_causality_future_tokens_do_not_change_the_past)


def test_planted_tanh_gelu_is_caught(monkeypatch):
    monkeypatch.setattr(O, "gelu", lambda x: 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3))))
    assert _fails(test_gelu_matches_math_erf_and_torch)
    assert _fails(test_oracle_equals_scalar_loop_brute_force_tiny)


def test_planted_unshifted_targets_are_caught(monkeypatch):
    def ce_unshifted(logits, ids, lengths=None):
        lse = O.logsumexp_last(logits)
        zt = np.take_along_axis(logits, ids[..., None].astype(np.int64), -1)[..., 0]
        per = lse - zt
        return float(per.mean()), per
    monkeypatch.setattr(O, "shifted_cross_entropy", ce_unshifted)
    assert _fails(test_cross_entropy_matches_torch)
    assert _fails(test_shift_pairs_position_t_with_token_t_plus_1)


def test_planted_missing_scale_is_caught(monkeypatch):
    orig_softmax = O.softmax_last
    monkeypatch.setattr(O, "softmax_last", lambda s: orig_softmax(s * 4.0))
    assert _fails(test_attention_matches_torch_sdpa_causal)
    assert _fails(test_oracle_equals_scalar_loop_brute_force_tiny)


def test_planted_dropped_attention_branch_is_caught(monkeypatch):
    orig_linear = O.linear
    monkeypatch.setattr(O, "linear", lambda x, w, b: orig_linear(x, w, b) if w.shape[0] != w.shape[1] else orig_linear(x, w, b) * 0)
    assert _fails(test_full_model_matches_torch_library_composition)


def test_planted_sinusoidal_exponent_is_caught(monkeypatch):
    def pe_wrong(n_ctx, C):   # i / C instead of 2i / C
        pos = np.arange(n_ctx, dtype=np.float64)[:, None]
        i = np.arange(C // 2, dtype=np.float64)[None, :]
        a = pos / np.power(10000.0, i / C)
        pe = np.empty((n_ctx, C))
        pe[:, 0::2], pe[:, 1::2] = np.sin(a), np.cos(a)
        return pe
    monkeypatch.setattr(O, "sinusoidal_wpe", pe_wrong)
    assert _fails(test_sinusoidal_wpe_closed_forms)


def test_planted_gelu_tanh_coefficient_is_caught(monkeypatch):
    monkeypatch.setattr(O, "gelu_tanh",
                        lambda x: 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.0447 * x ** 3))))
    assert _fails(test_gelu_tanh_matches_torch_and_its_identities)
