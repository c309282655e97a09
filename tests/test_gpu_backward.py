"""Backward pass through the C ABI (include/gpt2_train.h) against the
backward oracle (oracle/gpt2_backward.py), step by step and for the whole
model.

Tolerances. Each product reads bf16 operands (relative rounding 2^-9) and
accumulates in fp32, as the forward does:
* one product on bf16-exact inputs written in fp32: the accumulation error
  only, far below 1e-3 of the result's scale (max-abs <= 1e-3 * scale);
* a result rounded once to bf16: within 2^-8 of itself;
* a chain of products (attention backward, the whole model): the bf16
  roundings of the intermediate operands (P, dS, dz, the residual gradient
  at each GEMM input) compound; per gradient tensor relative L2 error
  <= 2e-2 against the fp64 oracle, and the loss within 1e-2 as in the
  forward parity tests. The measured errors are printed (GRAD lines).
"""
import json
import math

import numpy as np
import pytest
import torch

import synthetic
from oracle import gpt2_backward as OB
from oracle import gpt2_oracle as O
from tests._cmp import max_abs, rel_l2

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 2e-2


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_decoder_lm_b200 as g
    return g


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)


def bf16_exact(rng, shape, scale=1.0):
    return synthetic.round_to_bf16(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def report(name, **kw):
    print("GRAD " + json.dumps({"case": name, **kw}), flush=True)


# (tokens M, out N, in K); the last two are weight gradients with few output
# tiles and many tokens, which run as two K halves added into a zeroed output
LIN_SHAPES = [(200, 192, 320), (1000, 768, 2304), (4096, 768, 3072), (77, 64, 128), (1500, 384, 256),
              (4096, 768, 768)]


@pytest.mark.parametrize("shape", LIN_SHAPES)
def test_linear_dgrad_and_wgrad(G, shape):
    """dx = dy W (fp32 and bf16 out) and dW = dy^T x on the MN-major tcgen05
    layouts, against oracle.linear_backward; M ragged (not a multiple of 64
    or 128) in all but one shape."""
    M, N, K = shape
    rng = np.random.default_rng(M + N + K)
    dy = bf16_exact(rng, (M, N))
    W = bf16_exact(rng, (N, K), 1.0 / math.sqrt(N))
    x = bf16_exact(rng, (M, K))
    rdx, rdw, _ = OB.linear_backward(x.astype(np.float64), W.astype(np.float64), dy.astype(np.float64))
    st = status_word()
    dx32 = torch.empty(M, K, dtype=torch.float32, device="cuda")
    dx16 = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty(N, K, dtype=torch.float32, device="cuda")
    d_dy, d_W, d_x = dev(dy, "bf16"), dev(W, "bf16"), dev(x, "bf16")
    G.gpt2_op_linear_dgrad(d_dy, d_W, M, N, K, dx32, True, st)
    G.gpt2_op_linear_dgrad(d_dy, d_W, M, N, K, dx16, False, st)
    G.gpt2_op_linear_wgrad(d_dy, d_x, M, N, K, dw, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g32, g16, gw = dx32.cpu().numpy(), dx16.float().cpu().numpy(), dw.cpu().numpy()
    report(f"linear{shape}", dgrad_max_abs=max_abs(g32, rdx), wgrad_max_abs=max_abs(gw, rdw))
    assert max_abs(g32, rdx) <= 1e-3 * max(1.0, np.abs(rdx).max())
    assert np.all(np.abs(g16 - rdx) <= np.abs(rdx) * 2.0 ** -8 + 1e-3)
    assert max_abs(gw, rdw) <= 1e-3 * max(1.0, np.abs(rdw).max())
    # a second call gives the same bits (also when the K range is split in two)
    dw2 = torch.empty_like(dw)
    G.gpt2_op_linear_wgrad(d_dy, d_x, M, N, K, dw2, st)
    torch.cuda.synchronize()
    assert torch.equal(dw, dw2)


@pytest.mark.parametrize("tanh_form", [0, 1])
def test_dgrad_with_gelu_derivative(G, tanh_form):
    M, N, K = 300, 768, 3072
    rng = np.random.default_rng(11 + tanh_form)
    dy = bf16_exact(rng, (M, N))
    W = bf16_exact(rng, (N, K), 1.0 / math.sqrt(N))
    u = bf16_exact(rng, (M, K), 2.0)
    df = dy.astype(np.float64) @ W.astype(np.float64)
    ref = (OB.gelu_tanh_backward if tanh_form else OB.gelu_backward)(u.astype(np.float64), df)
    out = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    st = status_word()
    G.gpt2_op_linear_dgrad_gelu(dev(dy, "bf16"), dev(W, "bf16"), dev(u, "bf16"), M, N, K, tanh_form, out, st)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert int(st.item()) == 0
    report(f"dgrad_gelu_tanh{tanh_form}", max_abs=max_abs(got, ref), rel_l2=rel_l2(got, ref))
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 2e-3)


@pytest.mark.parametrize("C", [64, 768, 1600])
def test_layernorm_backward(G, C):
    M = 333
    rng = np.random.default_rng(C)
    x = (rng.standard_normal((M, C)) * 2 + 0.5).astype(np.float32)
    g = bf16_exact(rng, (C,), 1.0)
    dh = rng.standard_normal((M, C)).astype(np.float32)
    dx_in = rng.standard_normal((M, C)).astype(np.float32)
    rdx, rdg, rdb = OB.layer_norm_backward(x.astype(np.float64), g.astype(np.float64), dh.astype(np.float64))
    ws = torch.empty(G.gpt2_op_layernorm_backward_workspace_bytes(M, C), dtype=torch.uint8, device="cuda")
    dx = torch.empty(M, C, dtype=torch.float32, device="cuda")
    dg = torch.empty(C, dtype=torch.float32, device="cuda")
    db = torch.empty(C, dtype=torch.float32, device="cuda")
    G.gpt2_op_layernorm_backward(dev(x, "fp32"), dev(g, "bf16"), dev(dh, "fp32"), dev(dx_in, "fp32"), M, C, dx, dg,
                                 db, ws)
    torch.cuda.synchronize()
    got = dx.cpu().numpy()
    assert max_abs(got, rdx + dx_in) <= 1e-4 * max(1.0, np.abs(rdx).max())
    assert max_abs(dg.cpu().numpy(), rdg) <= 1e-4 * max(1.0, np.abs(rdg).max())
    assert max_abs(db.cpu().numpy(), rdb) <= 1e-4 * max(1.0, np.abs(rdb).max())
    # a second call gives the same bits (fixed-order column sums)
    dg2 = torch.empty_like(dg)
    G.gpt2_op_layernorm_backward(dev(x, "fp32"), dev(g, "bf16"), dev(dh, "fp32"), None, M, C, dx, dg2, db, ws)
    torch.cuda.synchronize()
    assert torch.equal(dg, dg2)
    assert max_abs(dx.cpu().numpy(), rdx) <= 1e-4 * max(1.0, np.abs(rdx).max())


@pytest.mark.parametrize("B,T,H", [(2, 200, 2), (1, 64, 1), (4, 1024, 12), (3, 77, 4)])
def test_attention_backward(G, B, T, H):
    """The training forward's row log-sum-exp and the attention backward,
    against the oracle's probabilities and causal_self_attention_backward."""
    C = 64 * H
    rng = np.random.default_rng(B * 1000 + T + H)
    qkv = bf16_exact(rng, (B, T, 3 * C))
    dy = bf16_exact(rng, (B, T, C))
    d_qkv = dev(qkv, "bf16")
    y = torch.empty(B * T, C, dtype=torch.bfloat16, device="cuda")
    lse2 = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
    st = status_word()
    G.gpt2_op_attention_train(d_qkv, B, T, H, C, y, lse2, st)
    # the oracle's normaliser in the same units: log2 sum_j 2^(s_ij log2(e) / sqrt(D))
    q = qkv[:, :, :C].reshape(B, T, H, 64).transpose(0, 2, 1, 3).astype(np.float64)
    k = qkv[:, :, C:2 * C].reshape(B, T, H, 64).transpose(0, 2, 1, 3).astype(np.float64)
    s = (q @ k.transpose(0, 1, 3, 2)) / 8.0
    s = np.where(O.causal_mask(T), -np.inf, s)
    ref_lse2 = (O.logsumexp_last(s)) / math.log(2.0)
    ws = torch.empty(G.gpt2_op_attention_backward_workspace_bytes(B, T, H, C), dtype=torch.uint8, device="cuda")
    dqkv = torch.empty(B * T, 3 * C, dtype=torch.bfloat16, device="cuda")
    G.gpt2_op_attention_backward(d_qkv, y, dev(dy, "bf16"), lse2, B, T, H, C, dqkv, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert max_abs(lse2.cpu().numpy(), ref_lse2) <= 1e-3
    # reference gradient at the kernel's own rounded output y (the forward is tested elsewhere)
    ref = OB.causal_self_attention_backward(qkv.astype(np.float64), H, dy.astype(np.float64))
    got = dqkv.float().cpu().numpy().reshape(B, T, 3 * C)
    parts = {n: (got[:, :, i * C:(i + 1) * C], ref[:, :, i * C:(i + 1) * C]) for i, n in enumerate("qkv")}
    errs = {n: rel_l2(a, r) for n, (a, r) in parts.items()}
    report(f"attention_bwd B{B} T{T} H{H}", **{f"rel_l2_d{n}": e for n, e in errs.items()})
    for n, e in errs.items():
        assert e <= GRAD_REL_L2, (n, e)


def test_lmhead_ce_backward(G):
    """dz, dhf = dz wte and the head's dwte = dz^T hf on a vocabulary that is
    not a multiple of the tile width, with unscored rows."""
    M, C, V = 300, 256, 1000
    rng = np.random.default_rng(5)
    hf = bf16_exact(rng, (M, C))
    wte = bf16_exact(rng, (V, C), 0.05)
    tg = rng.integers(0, V, size=M).astype(np.int32)
    tg[::7] = -1
    z = hf.astype(np.float64) @ wte.astype(np.float64).T
    sc = tg >= 0
    p = np.exp(z - O.logsumexp_last(z)[:, None])
    dz = p.copy()
    dz[np.arange(M)[sc], tg[sc]] -= 1.0
    dz[~sc] = 0.0
    dz /= sc.sum()
    ref_loss = float((O.logsumexp_last(z)[sc] - z[np.arange(M)[sc], tg[sc]]).mean())
    ref_dhf = dz @ wte.astype(np.float64)
    ref_dwte = dz.T @ hf.astype(np.float64)
    ws = torch.empty(G.gpt2_op_lmhead_ce_backward_workspace_bytes(M, V), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    dhf = torch.empty(M, C, dtype=torch.float32, device="cuda")
    dwte = torch.empty(V, C, dtype=torch.float32, device="cuda")
    st = status_word()
    G.gpt2_op_lmhead_ce_backward(dev(hf, "bf16"), dev(wte, "bf16"), torch.from_numpy(tg).cuda(), M, C, V, loss, dhf,
                                 dwte, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    a, b = rel_l2(dhf.cpu().numpy(), ref_dhf), rel_l2(dwte.cpu().numpy(), ref_dwte)
    report("lmhead_ce_bwd", loss_err=abs(float(loss.item()) - ref_loss), rel_l2_dhf=a, rel_l2_dwte=b)
    assert abs(float(loss.item()) - ref_loss) <= 1e-3
    assert a <= GRAD_REL_L2 and b <= GRAD_REL_L2


def _grad_tensors(g):
    out = [("wte", g["wte"]), ("wpe", g["wpe"]), ("lnf_g", g["lnf_g"]), ("lnf_b", g["lnf_b"])]
    for i, lg in enumerate(g["layers"]):
        for k in synthetic.LAYER_KEYS:
            out.append((f"{i}.{k}", lg[k]))
    return out


def run_model_backward(G, wl, W, ids, lengths=None, act="erf"):
    flags = G.GPT2_FLAG_GELU_TANH if act == "tanh" else 0
    model = G.GPT2Model.from_workload(wl, W, flags=flags)
    grads = model.new_grads()
    ws = model.new_train_workspace()
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(synthetic.next_token_targets(ids, lengths)).cuda()
    loss = model.forward_backward(d_ids, d_tg, grads, ws)
    torch.cuda.synchronize()
    assert model.status() == 0
    host = {"wte": grads["wte"].cpu().numpy(), "wpe": grads["wpe"].cpu().numpy(),
            "lnf_g": grads["lnf_g"].cpu().numpy(), "lnf_b": grads["lnf_b"].cpu().numpy(),
            "layers": [{k: v.cpu().numpy() for k, v in lg.items()} for lg in grads["layers"]]}
    out = (float(loss.item()), host)
    model.close()
    del model, grads, ws
    torch.cuda.empty_cache()
    return out


def compare_grads(name, loss, g, ref_loss, ref):
    errs = {}
    for (n, a), (_, r) in zip(_grad_tensors(g), _grad_tensors(ref)):
        assert a.shape == r.shape, n
        errs[n] = rel_l2(a, r)
    worst = max(errs, key=errs.get)
    report(name, loss_err=abs(loss - ref_loss), worst=worst, worst_rel_l2=errs[worst],
           median_rel_l2=float(np.median(list(errs.values()))), wte=errs["wte"])
    assert abs(loss - ref_loss) <= 1e-2
    for n, e in errs.items():
        assert e <= GRAD_REL_L2, (n, e)


SMALL = synthetic.random_case(61, n_layer=2, n_head=4, n_embd=256, vocab=1000, n_ctx=256, batch=3, seq=200,
                              lengths=(200, 131, 47))


@pytest.mark.parametrize("act", ["erf", "tanh"])
def test_small_model_gradients(G, act):
    W = synthetic.make_weights(SMALL)
    ids = synthetic.make_ids(SMALL)
    lengths = synthetic.lengths_of(SMALL)
    loss, g = run_model_backward(G, SMALL, W, ids, lengths, act)
    ref_loss, ref = OB.forward_backward(W, ids, SMALL.n_head, lengths, act=act)
    compare_grads(f"small-{act}", loss, g, ref_loss, ref)
    # the tied wte: rows of tokens that never occur get the head term only
    present = np.zeros(SMALL.vocab, bool)
    present[ids.reshape(-1)] = True
    assert (~present).any()


def test_124m_gradients_one_sequence(G):
    """GPT-2 124M shapes (12 layers, C 768, V 50257) on one 1024-token sequence."""
    wl = synthetic.WORKLOADS[1].scaled(batch=1)
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(synthetic.WORKLOADS[1])[:1]
    loss, g = run_model_backward(G, wl, W, ids)
    ref_loss, ref = OB.forward_backward(W, ids, wl.n_head)
    compare_grads("124M-B1", loss, g, ref_loss, ref)


def test_forward_backward_errors(G):
    wl = SMALL
    W = synthetic.make_weights(wl)
    model = G.GPT2Model.from_workload(wl, W)
    grads = model.new_grads()
    ws = model.new_train_workspace()
    ids = torch.from_numpy(synthetic.make_ids(wl)).cuda()
    tg = torch.from_numpy(synthetic.next_token_targets(synthetic.make_ids(wl))).cuda()
    with pytest.raises(G.GPT2Error) as e:
        model.forward_backward(ids, tg, grads, ws[: ws.numel() // 2])
    assert e.value.code == G.binding.ERR_CODE["GPT2_ERR_WORKSPACE"]
    with pytest.raises(G.GPT2Error) as e:            # 16 positions or fewer: the few-row path has no backward
        model.forward_backward(ids[:1, :16].contiguous(), tg[:1, :16].contiguous(), grads, ws)
    assert e.value.code == G.binding.ERR_CODE["GPT2_ERR_UNSUPPORTED"]
    model.close()
    f32 = G.GPT2Model.from_workload(wl, W, dtype="fp32")
    with pytest.raises(G.GPT2Error):
        f32.new_train_workspace()
    f32.close()
