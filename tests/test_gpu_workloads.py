"""Parity at the full workload sizes, in the launch configuration bench.py
times (gpt2_forward_loss on the whole batch).

The oracle checks every logit of the 124M workload and of the 774M
workload's valid positions (all four sequences, each run alone at its own
length), and whole 1024-token sequences of the loss-only 350M (two of eight)
and 1.5B (one of sixteen) workloads: every per-position loss of those
sequences. Causality makes a sequence run alone exact against the batched
run. Properties that hold at any size cover the rest: the loss equals the
mean of the per-position losses, pads never change scored outputs, and the
scored-position count.

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


def _oracle_sequences(W, wl, ids, rows, lengths=None):
    """Oracle logits and per-position losses of whole sequences `rows`, each
    run alone at its own valid length (causality: a sequence's outputs do not
    depend on the pads after it or on the other sequences of the batch)."""
    out = []
    for b in rows:
        n = wl.seq if lengths is None else int(lengths[b])
        z = O.forward(W, ids[b:b + 1, :n], wl.n_head)
        _, t = O.shifted_cross_entropy(z, ids[b:b + 1, :n])
        out.append((b, n, z[0], t[0, : n - 1]))
    return out


def _check_token_losses(name, loss, tok, seqs, scored_mask, extra=None):
    """Per-position losses of the oracle's whole sequences against the GPU's,
    the mean over them, and the GPU loss as the mean of its own per-position
    losses over every scored position of the batch."""
    got = np.concatenate([tok[b, : n - 1] for b, n, _, _ in seqs])
    ref = np.concatenate([t for _, _, _, t in seqs])
    err = np.abs(got.astype(np.float64) - ref)
    report(name, loss=loss, sequences=[int(b) for b, _, _, _ in seqs], scored_checked=int(ref.size),
           last_position=int(max(n for _, n, _, _ in seqs) - 1), token_loss_max_abs_err=float(err.max()),
           token_loss_mean_abs_err=float(err.mean()), mean_gpu=float(got.mean()), mean_oracle=float(ref.mean()),
           **(extra or {}))
    assert err.max() <= _cmp.BF16_MAX_ABS
    assert abs(got.mean() - ref.mean()) <= _cmp.BF16_LOSS_ABS
    assert abs(loss - tok[scored_mask].mean()) <= 1e-5
    assert (tok[~scored_mask] == 0).all()


def test_350m_loss_only_whole_sequences(G):
    """350M, B 8, T 1024, loss only: sequences 0 and 5 in full (2046 scored
    positions, keys up to position 1023) against the oracle."""
    wl = synthetic.WORKLOADS[2]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    _, loss, tok = gpu_run(G, wl, W, ids, want_logits=False)
    seqs = _oracle_sequences(W, wl, ids, [0, 5])
    scored = synthetic.next_token_targets(ids) >= 0
    _check_token_losses(wl.name, loss, tok, seqs, scored)


def test_774m_padded_whole_batch(G):
    """774M, lengths 128/512/1000/1024 right-padded to 1024: every sequence in
    full, so every logit at a valid position, every per-position loss and the
    batch loss itself (all 2660 scored positions) are compared with the
    oracle; then pad invariance and the scored count."""
    wl = synthetic.WORKLOADS[3]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    lengths = synthetic.lengths_of(wl)
    z, loss, tok = gpu_run(G, wl, W, ids, lengths)
    seqs = _oracle_sequences(W, wl, ids, range(wl.batch), lengths)
    got_z = np.concatenate([z[b, :n] for b, n, _, _ in seqs])
    ref_z = np.concatenate([r for _, _, r, _ in seqs])
    rl, ma = _cmp.rel_l2(got_z, ref_z), _cmp.max_abs(got_z, ref_z)
    lit, tie = _cmp.top1(got_z, ref_z)
    ref_loss = float(np.concatenate([t for _, _, _, t in seqs]).mean())
    scored = synthetic.next_token_targets(ids, lengths) >= 0
    _check_token_losses(wl.name, loss, tok, seqs, scored,
                        dict(rel_l2=rl, max_abs=ma, top1_literal=lit, top1_tie_aware=tie, oracle_loss=ref_loss,
                             loss_err=abs(loss - ref_loss), scored=int(scored.sum()), logit_rows=int(got_z.shape[0])))
    assert rl <= _cmp.BF16_REL_L2 and ma <= _cmp.BF16_MAX_ABS and tie >= _cmp.BF16_TOP1
    assert abs(loss - ref_loss) <= _cmp.BF16_LOSS_ABS
    assert int(scored.sum()) == 127 + 511 + 999 + 1023
    # pads never reach a scored output: change the pad id and nothing scored moves
    ids2 = ids.copy()
    for b, n in enumerate(lengths):
        ids2[b, n:] = 4321
    z2, loss2, tok2 = gpu_run(G, wl, W, ids2, lengths)
    for b, n in enumerate(lengths):
        assert np.array_equal(z[b, :n], z2[b, :n])
    assert loss2 == loss


def test_1p5b_loss_only_whole_sequence(G):
    """1.5B, B 16, T 1024, loss only: sequence 15 in full (1023 scored
    positions) against the oracle."""
    wl = synthetic.WORKLOADS[4]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    _, loss, tok = gpu_run(G, wl, W, ids, want_logits=False)
    seqs = _oracle_sequences(W, wl, ids, [15])
    scored = synthetic.next_token_targets(ids) >= 0
    _check_token_losses(wl.name, loss, tok, seqs, scored)
    assert math.isfinite(loss) and abs(loss - 10.9) < 0.5
