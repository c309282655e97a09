"""The data-parallel forward on the device: two ranks, each running libgpt2
on its own shard of the batch, the loss combined over ranks.

Both ranks are processes on the one GPU of the test machine, joined by a
gloo process group on the host. Nothing on the device waits on the other
rank: each rank's kernels run to completion on their own, and the only
exchange is the host all-reduce of (sum of per-position losses, scored
count) in transformer_decoder_lm_b200.dist ("Hand-writing GPT-2 from
scratch: the Transformer decoder core modules in PyTorch", section 6.2,
data-parallel ranks; here only the forward's loss is combined). The combined
loss and every rank's per-position losses are compared with the oracle on
the whole batch.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic
from oracle import gpt2_oracle as O
from tests import _cmp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASE = synthetic.random_case(43, n_layer=2, n_head=4, n_embd=256, vocab=1000, n_ctx=256, batch=5, seq=200,
                             lengths=(200, 57, 130, 200, 9))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import synthetic as S
    import transformer_decoder_lm_b200 as G
    from transformer_decoder_lm_b200 import dist as D
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        torch.cuda.set_device(0)
        W = S.make_weights(CASE)
        ids = S.make_ids(CASE)
        tg = S.next_token_targets(ids, S.lengths_of(CASE))
        a, b = D.shard_sequences(CASE.batch, rank, world)
        model = G.GPT2Model.from_workload(CASE, W, max_B=b - a)
        d_ids = torch.from_numpy(np.ascontiguousarray(ids[a:b])).cuda()
        d_tg = torch.from_numpy(np.ascontiguousarray(tg[a:b])).cuda()
        tok = torch.empty(d_ids.shape, dtype=torch.float32, device="cuda")
        _, loss = model.forward_loss(d_ids, d_tg, want_logits=False, token_loss=tok)
        torch.cuda.synchronize()
        rc = model.status()
        count = int((tg[a:b] >= 0).sum())
        combined = D.global_mean_loss(loss.cpu(), count)
        out[rank] = (rc, float(combined.item()), tok.cpu().numpy(), a, b)
        model.close()
    finally:
        dist.destroy_process_group()


def test_two_ranks_on_libgpt2_match_whole_batch_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    W = synthetic.make_weights(CASE)
    ids = synthetic.make_ids(CASE)
    lengths = synthetic.lengths_of(CASE)
    ref_loss, ref_tok = O.shifted_cross_entropy(O.forward(W, ids, CASE.n_head), ids, lengths)
    tok = np.zeros(ids.shape, dtype=np.float64)
    for r in range(world):
        rc, combined, t, a, b = out[r]
        assert rc == 0
        assert abs(combined - ref_loss) <= _cmp.BF16_LOSS_ABS
        tok[a:b] = t
    assert (out[0][3], out[0][4], out[1][3], out[1][4]) == (0, 3, 3, 5)
    assert out[0][1] == out[1][1]          # every rank holds the same combined loss
    scored = synthetic.next_token_targets(ids, lengths) >= 0
    assert np.abs(tok[scored] - ref_tok[scored]).max() <= _cmp.BF16_MAX_ABS
    assert (tok[~scored] == 0).all()
    # the combined loss is the mean over every scored position of the batch
    assert abs(out[0][1] - tok[scored].mean()) <= 1e-5
