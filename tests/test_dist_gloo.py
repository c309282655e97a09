"""Host logic of the data-parallel forward on CPU: world_size 2 over gloo.

Each rank scores its own shard of a batch with the CPU oracle; the combined
loss from transformer_decoder_lm_b200.dist must equal the oracle's loss on
the whole batch, and the max-over-ranks timing helper must return the
largest rank value. (The dist helpers import only torch: no GPU and no
libgpt2.so needed.)
"""
import importlib.util
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_dist():
    # the helpers are plain torch; load the file alone so no GPU library is needed
    spec = importlib.util.spec_from_file_location("g2dist", os.path.join(ROOT, "transformer_decoder_lm_b200", "dist.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import synthetic
    from oracle import gpt2_oracle as O
    D = _load_dist()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synthetic.random_case(41, n_layer=1, n_head=2, n_embd=32, vocab=97, n_ctx=16, batch=5, seq=12,
                                   dtype="fp32", lengths=(12, 3, 12, 7, 1))
        W = synthetic.make_weights(wl)
        ids = synthetic.make_ids(wl)
        lengths = synthetic.lengths_of(wl)
        a, b = D.shard_sequences(wl.batch, rank, world)
        z = O.forward(W, ids[a:b], wl.n_head)
        local, tok = O.shifted_cross_entropy(z, ids[a:b], lengths[a:b])
        count = int(np.isfinite(tok).sum())
        g = D.global_mean_loss(torch.tensor([local], dtype=torch.float32), count)
        mx = D.max_over_ranks(float(rank) * 1.5 + 2.0, "cpu")
        out[rank] = (float(g.item()), mx, a, b)
    finally:
        dist.destroy_process_group()


def test_shard_sequences_covers_batch_once():
    D = _load_dist()
    for B in (0, 1, 4, 5, 16):
        for W in (1, 2, 3, 8):
            spans = [D.shard_sequences(B, r, W) for r in range(W)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(spans[i][1] == spans[i + 1][0] for i in range(W - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        D.shard_sequences(4, 2, 2)


def test_two_rank_loss_equals_whole_batch_loss():
    import synthetic
    from oracle import gpt2_oracle as O
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    wl = synthetic.random_case(41, n_layer=1, n_head=2, n_embd=32, vocab=97, n_ctx=16, batch=5, seq=12,
                               dtype="fp32", lengths=(12, 3, 12, 7, 1))
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    whole, _ = O.shifted_cross_entropy(O.forward(W, ids, wl.n_head), ids, synthetic.lengths_of(wl))
    for r in range(world):
        g, mx, a, b = out[r]
        assert abs(g - whole) <= 1e-5 * max(1.0, abs(whole))
        assert mx == 3.5
    assert (out[0][2], out[0][3], out[1][2], out[1][3]) == (0, 3, 3, 5)
    assert math.isfinite(whole)
