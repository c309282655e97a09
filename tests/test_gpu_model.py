"""Whole forward pass through the C ABI (gpt2_create / gpt2_forward /
gpt2_loss / gpt2_forward_loss) against the CPU oracle on small seeded
workloads, plus the error paths of the ABI."""
import math

import numpy as np
import pytest
import torch

import synthetic
from oracle import gpt2_oracle as O
from tests import _cmp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_decoder_lm_b200 as g
    return g


def run_case(G, wl, dtype=None, ids=None, lengths=None):
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl) if ids is None else ids
    model = G.GPT2Model.from_workload(wl, W, dtype=dtype)
    targets = synthetic.next_token_targets(ids, lengths)
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(targets).cuda()
    tok = torch.empty(ids.shape, dtype=torch.float32, device="cuda")
    logits, loss = model.forward_loss(d_ids, d_tg, token_loss=tok)
    torch.cuda.synchronize()
    assert model.status() == 0
    return W, ids, model, logits.cpu().numpy(), float(loss.item()), tok.cpu().numpy()


def test_tiny_fp32_workload(G):
    wl = synthetic.WORKLOADS[0]
    W, ids, model, z, loss, tok = run_case(G, wl)
    ref = O.forward(W, ids, wl.n_head)
    ref_loss, ref_tok = O.shifted_cross_entropy(ref, ids)
    assert z.shape == (2, 4, 512)
    assert _cmp.rel_l2(z, ref) <= _cmp.FP32_REL_L2
    assert abs(loss - ref_loss) <= 1e-5
    assert np.allclose(tok[:, :-1], ref_tok[:, :-1], atol=1e-5) and (tok[:, -1] == 0).all()


SMALL = synthetic.random_case(31, n_layer=2, n_head=4, n_embd=256, vocab=1000, n_ctx=256, batch=3, seq=200)


def test_small_bf16_case_spans_tiles_and_tails(G):
    W, ids, model, z, loss, tok = run_case(G, SMALL)
    ref = O.forward(W, ids, SMALL.n_head)
    ref_loss, _ = O.shifted_cross_entropy(ref, ids)
    assert _cmp.rel_l2(z, ref) <= _cmp.BF16_REL_L2
    assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS
    assert abs(loss - ref_loss) <= _cmp.BF16_LOSS_ABS
    lit, tie = _cmp.top1(z, ref)
    assert tie >= _cmp.BF16_TOP1


@pytest.mark.parametrize("B,T", [(1, 1), (3, 1), (2, 5), (1, 17), (1, 256), (8, 2)])
def test_degenerate_and_edge_shapes(G, B, T):
    """A single position (no scored target: logits only), a batch of a few
    rows (M <= 16: the few-row GEMV path with separate LayerNorms), one row
    past it (M = 17: the tensor-core path with one ragged 128-row tile), a
    sequence of the full context n_ctx, and many sequences of two positions
    (one scored position each) against the oracle."""
    wl = SMALL.scaled(batch=B, seq=T)
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    model = G.GPT2Model.from_workload(wl, W)
    d_ids = torch.from_numpy(ids).cuda()
    ref = O.forward(W, ids, wl.n_head)
    z = model.forward(d_ids).cpu().numpy()
    assert model.status() == 0
    assert z.shape == (B, T, wl.vocab)
    assert _cmp.rel_l2(z, ref) <= _cmp.BF16_REL_L2
    assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS
    if T >= 2:
        ref_loss, _ = O.shifted_cross_entropy(ref, ids)
        d_tg = torch.from_numpy(synthetic.next_token_targets(ids)).cuda()
        z2, loss = model.forward_loss(d_ids, d_tg)
        assert model.status() == 0
        assert torch.equal(z2.cpu(), torch.from_numpy(z))
        assert abs(loss.item() - ref_loss) <= _cmp.BF16_LOSS_ABS


def test_small_case_all_fp32_debug_mode(G):
    W, ids, model, z, loss, tok = run_case(G, SMALL, dtype="fp32")
    ref = O.forward(W, ids, SMALL.n_head)
    ref_loss, _ = O.shifted_cross_entropy(ref, ids)
    assert _cmp.rel_l2(z, ref) <= _cmp.FP32_REL_L2
    assert abs(loss - ref_loss) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_gelu_tanh_flag(G, dtype):
    """GPT2_FLAG_GELU_TANH: the MLP uses the tanh form; parity with the oracle
    run with gelu_tanh (and, in fp32, clearly closer to it than to the erf form)."""
    W = synthetic.make_weights(SMALL)
    ids = synthetic.make_ids(SMALL)
    model = G.GPT2Model.from_workload(SMALL, W, dtype=dtype, flags=G.GPT2_FLAG_GELU_TANH)
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(synthetic.next_token_targets(ids)).cuda()
    logits, loss = model.forward_loss(d_ids, d_tg)
    torch.cuda.synchronize()
    assert model.status() == 0
    z = logits.cpu().numpy()
    ref = O.forward(W, ids, SMALL.n_head, act=O.gelu_tanh)
    ref_loss, _ = O.shifted_cross_entropy(ref, ids)
    if dtype == "bf16":
        assert _cmp.rel_l2(z, ref) <= _cmp.BF16_REL_L2
        assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS
        assert abs(float(loss.item()) - ref_loss) <= _cmp.BF16_LOSS_ABS
    else:
        assert _cmp.rel_l2(z, ref) <= _cmp.FP32_REL_L2
        assert abs(float(loss.item()) - ref_loss) <= 1e-4
        ref_erf = O.forward(W, ids, SMALL.n_head)
        assert _cmp.rel_l2(z, ref) * 10 < _cmp.rel_l2(z, ref_erf)
    model.close()


def test_model_with_device_filled_sinusoidal_wpe(G):
    """A model whose wpe is the fixed sinusoidal table filled on the device
    (gpt2_fill_sinusoidal_wpe) against the oracle with the oracle's table."""
    wl = SMALL
    W = synthetic.make_weights(wl)
    W["wpe"] = synthetic.round_to_bf16(O.sinusoidal_wpe(wl.n_ctx, wl.n_embd).astype(np.float32))
    Wd = G.upload_weights(synthetic.make_weights(wl), "bf16")
    wpe = torch.empty(wl.n_ctx, wl.n_embd, dtype=torch.bfloat16, device="cuda")
    G.gpt2_fill_sinusoidal_wpe(G.GPT2_BF16, wpe, wl.n_ctx, wl.n_embd)
    Wd["wpe"] = wpe
    ids = synthetic.make_ids(wl)
    model = G.GPT2Model.from_workload(wl, Wd)
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(synthetic.next_token_targets(ids)).cuda()
    logits, loss = model.forward_loss(d_ids, d_tg)
    torch.cuda.synchronize()
    assert model.status() == 0
    z = logits.cpu().numpy()
    ref = O.forward(W, ids, wl.n_head)
    ref_loss, _ = O.shifted_cross_entropy(ref, ids)
    assert _cmp.rel_l2(z, ref) <= _cmp.BF16_REL_L2
    assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS
    assert abs(float(loss.item()) - ref_loss) <= _cmp.BF16_LOSS_ABS
    model.close()


def test_head_dim_32_bf16(G):
    wl = synthetic.random_case(32, n_layer=1, n_head=4, n_embd=128, vocab=777, n_ctx=160, batch=2, seq=150)
    W, ids, model, z, loss, tok = run_case(G, wl)
    ref = O.forward(W, ids, wl.n_head)
    assert _cmp.rel_l2(z, ref) <= _cmp.BF16_REL_L2
    assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_causality_on_device_is_exact(G, dtype):
    """Changing tokens after position t leaves logits at positions <= t
    bit-identical: every kernel keeps rows independent and masked keys get
    exactly zero weight."""
    wl = SMALL.scaled(batch=2, seq=130)
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    model = G.GPT2Model.from_workload(wl, W, dtype=dtype)
    z1 = model.forward(torch.from_numpy(ids).cuda()).cpu()
    t = 70
    ids2 = ids.copy()
    ids2[:, t + 1:] = (ids2[:, t + 1:] * 7 + 3) % wl.vocab
    z2 = model.forward(torch.from_numpy(ids2).cuda()).cpu()
    assert torch.equal(z1[:, : t + 1], z2[:, : t + 1])
    assert not torch.equal(z1[:, t + 1:], z2[:, t + 1:])


def test_padded_batch_loss_ignores_pads(G):
    wl = SMALL.scaled(batch=3, seq=96, lengths=(96, 17, 50))
    lengths = synthetic.lengths_of(wl)
    W, ids, model, z, loss, tok = run_case(G, wl, lengths=lengths)
    ref = O.forward(W, ids, wl.n_head)
    ref_loss, ref_tok = O.shifted_cross_entropy(ref, ids, lengths)
    assert abs(loss - ref_loss) <= _cmp.BF16_LOSS_ABS
    scored = np.isfinite(ref_tok)
    assert int(scored.sum()) == 95 + 16 + 49
    assert np.abs(tok[scored] - ref_tok[scored]).max() <= 2e-2
    assert (tok[~scored] == 0).all()


def test_loss_only_matches_forward_loss(G):
    W = synthetic.make_weights(SMALL)
    ids = synthetic.make_ids(SMALL)
    model = G.GPT2Model.from_workload(SMALL, W)
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(synthetic.next_token_targets(ids)).cuda()
    l1 = model.loss(d_ids, d_tg).item()
    _, l2 = model.forward_loss(d_ids, d_tg)
    assert l1 == l2.item()


def test_uniform_logits_loss_is_log_vocab(G):
    W = synthetic.make_weights(SMALL)
    W["lnf_g"] = np.zeros_like(W["lnf_g"])
    W["lnf_b"] = np.zeros_like(W["lnf_b"])
    ids = synthetic.make_ids(SMALL)
    model = G.GPT2Model.from_workload(SMALL, W)
    loss = model.loss(torch.from_numpy(ids).cuda(), torch.from_numpy(synthetic.next_token_targets(ids)).cuda())
    assert abs(loss.item() - math.log(SMALL.vocab)) <= 1e-5


def test_error_paths(G):
    W = synthetic.make_weights(SMALL)
    model = G.GPT2Model.from_workload(SMALL, W, max_B=2, max_T=64)
    ids = torch.zeros(2, 64, dtype=torch.int32, device="cuda")
    with pytest.raises(G.GPT2Error) as e:
        model.forward(torch.zeros(3, 64, dtype=torch.int32, device="cuda"))      # B > max_B
    assert e.value.code == 1
    bad = ids.clone()
    bad[1, 3] = SMALL.vocab
    model.forward(bad)
    assert model.status() == 5                # GPT2_ERR_BAD_TOKEN, reported once
    assert model.status() == 0
    tg = torch.full((2, 64), -1, dtype=torch.int32, device="cuda")
    loss = model.loss(ids, tg)
    assert math.isnan(loss.item()) and model.status() == 7
