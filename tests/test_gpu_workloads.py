"""Parity at the full workload sizes, in the launch configuration bench.py
times (gpt2_forward_loss on the whole batch).

The oracle checks every logit of the 124M workload. For the larger
workloads it checks sampled outputs it can afford: whole short sequences and
the first tokens of long ones, which causality makes exact (outputs at
positions < t depend only on tokens < t). Properties that hold at any size
cover the rest: the loss equals the mean of the per-position losses, pads
never change scored outputs, and the scored-position count.

Each test prints one PARITY line with the measured agreement figures.
"""
import json
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


def report(name, **kw):
    print("PARITY " + json.dumps({"workload": name, **kw}), flush=True)


def gpu_run(G, wl, W, ids, lengths=None, want_logits=True, dtype=None):
    model = G.GPT2Model.from_workload(wl, W, dtype=dtype)
    d_ids = torch.from_numpy(ids).cuda()
    d_tg = torch.from_numpy(synthetic.next_token_targets(ids, lengths)).cuda()
    tok = torch.empty(ids.shape, dtype=torch.float32, device="cuda")
    logits, loss = model.forward_loss(d_ids, d_tg, want_logits=want_logits, token_loss=tok)
    torch.cuda.synchronize()
    assert model.status() == 0
    out = (None if logits is None else logits.cpu().numpy(), float(loss.item()), tok.cpu().numpy())
    model.close()
    del model
    torch.cuda.empty_cache()
    return out


def test_124m_full_logits_and_loss(G):
    wl = synthetic.WORKLOADS[1]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    z, loss, tok = gpu_run(G, wl, W, ids)
    ref = O.forward(W, ids, wl.n_head)
    ref_loss, ref_tok = O.shifted_cross_entropy(ref, ids)
    rl, ma = _cmp.rel_l2(z, ref), _cmp.max_abs(z, ref)
    lit, tie = _cmp.top1(z, ref)
    report(wl.name, rel_l2=rl, max_abs=ma, top1_literal=lit, top1_tie_aware=tie, loss=loss, oracle_loss=ref_loss,
           loss_err=abs(loss - ref_loss))
    assert rl <= _cmp.BF16_REL_L2
    assert ma <= _cmp.BF16_MAX_ABS
    assert abs(loss - ref_loss) <= _cmp.BF16_LOSS_ABS
    assert tie >= _cmp.BF16_TOP1
    assert lit >= 0.97          # literal argmax agreement: near-ties on random weights keep it under 99.5%
    assert abs(loss - tok[:, :-1].mean()) <= 1e-5


def test_124m_all_fp32_debug_mode(G):
    wl = synthetic.WORKLOADS[1]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)[:2]
    wl2 = wl.scaled(batch=2)
    z, loss, tok = gpu_run(G, wl2, W, ids, dtype="fp32")
    ref = O.forward(W, ids, wl.n_head)
    ref_loss, _ = O.shifted_cross_entropy(ref, ids)
    rl = _cmp.rel_l2(z, ref)
    report(wl.name + "-fp32", rel_l2=rl, loss=loss, oracle_loss=ref_loss)
    assert rl <= _cmp.FP32_REL_L2
    assert abs(loss - ref_loss) <= 1e-4


def _sampled_token_losses(W, wl, ids, rows, prefix):
    z = O.forward(W, ids[rows, :prefix], wl.n_head)
    _, t = O.shifted_cross_entropy(z, ids[rows, :prefix])
    return z, t[:, : prefix - 1]


def test_350m_loss_only_sampled(G):
    wl = synthetic.WORKLOADS[2]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    _, loss, tok = gpu_run(G, wl, W, ids, want_logits=False)
    rows, prefix = [0, 5], 160
    _, ref_t = _sampled_token_losses(W, wl, ids, rows, prefix)
    got = tok[rows, : prefix - 1]
    report(wl.name, loss=loss, sampled_mean_abs_err=float(np.abs(got - ref_t).mean()),
           sampled_max_abs_err=float(np.abs(got - ref_t).max()), sampled_tokens=int(ref_t.size))
    assert abs(got.mean() - ref_t.mean()) <= _cmp.BF16_LOSS_ABS
    assert np.abs(got - ref_t).max() <= _cmp.BF16_MAX_ABS
    assert abs(loss - tok[:, :-1].mean()) <= 1e-5
    assert (tok[:, -1] == 0).all()


def test_774m_padded_sampled(G):
    wl = synthetic.WORKLOADS[3]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    lengths = synthetic.lengths_of(wl)
    z, loss, tok = gpu_run(G, wl, W, ids, lengths)
    # sequence 0 (length 128) in full, the first 128 tokens of the others
    prefix = 128
    ref = O.forward(W, ids[:, :prefix], wl.n_head)
    _, ref_t = O.shifted_cross_entropy(ref, ids[:, :prefix])
    got = z[:, :prefix]
    rl, ma = _cmp.rel_l2(got, ref), _cmp.max_abs(got, ref)
    lit, tie = _cmp.top1(got, ref)
    scored = synthetic.next_token_targets(ids, lengths) >= 0
    report(wl.name, rel_l2=rl, max_abs=ma, top1_literal=lit, top1_tie_aware=tie, loss=loss,
           scored=int(scored.sum()))
    assert rl <= _cmp.BF16_REL_L2 and ma <= _cmp.BF16_MAX_ABS and tie >= _cmp.BF16_TOP1
    assert np.abs(tok[:, : prefix - 1] - ref_t[:, : prefix - 1]).max() <= _cmp.BF16_MAX_ABS
    assert int(scored.sum()) == 127 + 511 + 999 + 1023
    assert abs(loss - tok[scored].mean()) <= 1e-5
    assert (tok[~scored] == 0).all()
    # pads never reach a scored output: change the pad id and nothing scored moves
    ids2 = ids.copy()
    for b, n in enumerate(lengths):
        ids2[b, n:] = 4321
    z2, loss2, tok2 = gpu_run(G, wl, W, ids2, lengths)
    for b, n in enumerate(lengths):
        assert np.array_equal(z[b, :n], z2[b, :n])
    assert loss2 == loss


def test_1p5b_loss_only_sampled(G):
    wl = synthetic.WORKLOADS[4]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    _, loss, tok = gpu_run(G, wl, W, ids, want_logits=False)
    rows, prefix = [3, 15], 64
    _, ref_t = _sampled_token_losses(W, wl, ids, rows, prefix)
    got = tok[rows, : prefix - 1]
    report(wl.name, loss=loss, sampled_mean_abs_err=float(np.abs(got - ref_t).mean()),
           sampled_max_abs_err=float(np.abs(got - ref_t).max()))
    assert abs(got.mean() - ref_t.mean()) <= _cmp.BF16_LOSS_ABS
    assert np.abs(got - ref_t).max() <= _cmp.BF16_MAX_ABS
    assert abs(loss - tok[:, :-1].mean()) <= 1e-5
    assert math.isfinite(loss) and abs(loss - 10.9) < 0.5
