"""The allocation-free lm_head + cross-entropy entry point.

gpt2_op_lmhead_ce_noalloc exists for callers that cannot call cudaMalloc
(a plugin in a host application that owns all device memory, or a
latency-critical path that cannot afford cudaMalloc's device
synchronisation); its scratch is a fixed array inside libgpt2.so. This file
checks, through the C ABI, that two calls in a row give the same logits,
per-position losses and mean loss as the workspace-taking
gpt2_op_lmhead_ce (the second call with different inputs, so a stale
scratch from the first would show), and that a request larger than the
fixed scratch is refused before any launch. The file name makes pytest
collect it last.
"""
import math

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_decoder_lm_b200 as g
    return g


def _case(seed, M, C, V):
    rng = np.random.default_rng(seed)
    hf = synthetic.round_to_bf16(rng.standard_normal((M, C)).astype(np.float32))
    wte = synthetic.round_to_bf16((rng.standard_normal((V, C)) * 0.05).astype(np.float32))
    tg = rng.integers(0, V, size=M).astype(np.int32)
    tg[:: 5 + seed % 3] = -1
    to = lambda a, dt: torch.from_numpy(a).to("cuda", dt)
    return to(hf, torch.bfloat16), to(wte, torch.bfloat16), to(tg, torch.int32)


def _with_workspace(G, hf, wte, tg, M, C, V):
    ws = torch.empty(G.gpt2_op_lmhead_ce_workspace_bytes(G.GPT2_BF16, M, V), dtype=torch.uint8, device="cuda")
    logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
    tok = torch.empty(M, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    G.gpt2_op_lmhead_ce(G.GPT2_BF16, hf, wte, tg, M, C, V, logits, tok, loss, ws)
    return logits, tok, loss


def _no_alloc(G, hf, wte, tg, M, C, V):
    logits = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
    tok = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
    loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.gpt2_op_lmhead_ce_noalloc(G.GPT2_BF16, hf, wte, tg, M, C, V, logits, tok, loss, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return logits, tok, loss


@pytest.mark.parametrize("M,C,V", [(300, 768, 1000), (4096, 768, 50257)])
def test_no_alloc_matches_workspace_entry_point_twice(G, M, C, V):
    for call, seed in enumerate((101, 202)):
        hf, wte, tg = _case(seed + M, M, C, V)
        ref_logits, ref_tok, ref_loss = _with_workspace(G, hf, wte, tg, M, C, V)
        logits, tok, loss = _no_alloc(G, hf, wte, tg, M, C, V)
        # the same kernels on the same inputs: equal to within the lm_head test tolerances
        assert torch.allclose(logits, ref_logits, rtol=0, atol=1e-4), call
        assert torch.allclose(tok, ref_tok, rtol=0, atol=1e-4), call
        assert abs(float(loss.item()) - float(ref_loss.item())) <= 1e-5, call
        assert math.isfinite(float(loss.item()))


def test_no_alloc_refuses_requests_beyond_its_scratch(G):
    C, V = 768, 50257
    per_row = 16 * ((V + 127) // 128)
    M = G.GPT2_NOALLOC_SCRATCH_BYTES // per_row + 64
    hf, wte, tg = _case(7, 128, C, 1000)     # never read: the size check comes first
    with pytest.raises(G.GPT2Error) as e:
        G.gpt2_op_lmhead_ce_noalloc(G.GPT2_BF16, hf, wte, tg, M, C, V, None, None, None)
    assert e.value.code == 8                 # GPT2_ERR_SCRATCH_LIMIT
    assert "scratch" in G.gpt2_error_string(8)
