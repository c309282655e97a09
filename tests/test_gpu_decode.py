"""Incremental decoding with the key/value cache, through the C ABI.

The logits of a new token at position p must equal row p of the full
forward over positions 0..p (the causal mask makes every earlier row
independent of later tokens), which the oracle computes directly: the
decode path is checked against O.forward on the growing prefix at every
step, after a prefill whose own logits are checked too.
"""
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


CASES = {
    "bf16": synthetic.random_case(51, n_layer=2, n_head=4, n_embd=256, vocab=1000, n_ctx=96, batch=3, seq=40),
    "fp32": synthetic.random_case(52, n_layer=2, n_head=2, n_embd=64, vocab=512, n_ctx=64, batch=2, seq=24,
                                  dtype="fp32"),
    "bf16_d32": synthetic.random_case(53, n_layer=1, n_head=4, n_embd=128, vocab=700, n_ctx=64, batch=2, seq=20),
}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_then_decode_matches_full_forward(G, name):
    wl = CASES[name]
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    B, T = ids.shape
    T0 = T // 2
    model = G.GPT2Model.from_workload(wl, W)
    cache = model.new_kv_cache()
    d_ids = torch.from_numpy(ids).cuda()
    z0 = model.prefill(d_ids[:, :T0].contiguous(), cache).cpu().numpy()
    ref0 = O.forward(W, ids[:, :T0], wl.n_head)
    bf16 = wl.dtype == "bf16"
    lim = _cmp.BF16_REL_L2 if bf16 else _cmp.FP32_REL_L2
    assert _cmp.rel_l2(z0, ref0) <= lim
    for pos in range(T0, T):
        z = model.decode_step(d_ids[:, pos].contiguous(), pos, cache).cpu().numpy()
        ref = O.forward(W, ids[:, :pos + 1], wl.n_head)[:, pos]
        assert _cmp.rel_l2(z, ref) <= lim, pos
        if bf16:
            assert _cmp.max_abs(z, ref) <= _cmp.BF16_MAX_ABS, pos
    assert model.status() == 0
    model.close()


def test_decode_from_empty_cache_and_errors(G):
    """Decoding every position from 0 (no prefill) gives the full forward
    too; bad positions and batch sizes are rejected on the host."""
    wl = CASES["bf16"].scaled(batch=2, seq=12)
    W = synthetic.make_weights(wl)
    ids = synthetic.make_ids(wl)
    model = G.GPT2Model.from_workload(wl, W)
    cache = model.new_kv_cache()
    d_ids = torch.from_numpy(ids).cuda()
    ref = O.forward(W, ids, wl.n_head)
    for pos in range(ids.shape[1]):
        z = model.decode_step(d_ids[:, pos].contiguous(), pos, cache).cpu().numpy()
        assert _cmp.rel_l2(z, ref[:, pos]) <= _cmp.BF16_REL_L2, pos
    with pytest.raises(G.GPT2Error):
        model.decode_step(d_ids[:, 0].contiguous(), wl.n_ctx, cache)          # pos >= n_ctx
    with pytest.raises(G.GPT2Error):
        model.decode_step(torch.zeros(wl.batch + 1, dtype=torch.int32, device="cuda"), 1, cache)   # B > max_B
    # a cache sized for fewer sequences than the handle's max_B is refused on the host
    small = torch.empty(G.gpt2_kv_cache_bytes(model.cfg, wl.batch - 1), dtype=torch.uint8, device="cuda")
    for call in (lambda: model.decode_step(d_ids[:, 0].contiguous(), 0, small),
                 lambda: model.prefill(d_ids[:, :4].contiguous(), small, want_logits=False)):
        with pytest.raises(G.GPT2Error) as e:
            call()
        assert e.value.code == G.binding.ERR_CODE["GPT2_ERR_WORKSPACE"]
    assert model.status() == 0
    model.close()
