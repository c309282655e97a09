"""Per-step parity of the CUDA kernels against the CPU oracle, through the
C-ABI single-step entry points (gpt2_op_*). Sizes span several tiles and a
ragged tail; every tcgen05 tile width is exercised."""
import math
import os

import numpy as np
import pytest
import torch

import synthetic
from oracle import gpt2_oracle as O
from tests._cmp import rel_l2, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_decoder_lm_b200 as g   # fails loudly if libgpt2.so is missing
    return g


def dev(a, dtype):
    td = {"bf16": torch.bfloat16, "fp32": torch.float32, "i32": torch.int32}[dtype]
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(td)


def bf16_exact(rng, shape, scale=1.0):
    return synthetic.round_to_bf16((rng.standard_normal(shape) * scale).astype(np.float32))


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ---------------------------------------------------------------- embedding


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_embed(G, dtype):
    rng = np.random.default_rng(10)
    V, C, T, Bn = 1000, 768, 37, 3
    wte = bf16_exact(rng, (V, C), 0.02)
    wpe = bf16_exact(rng, (64, C), 0.02)
    ids = rng.integers(0, V, size=(Bn, T)).astype(np.int32)
    x = torch.empty(Bn * T, C, dtype=torch.float32, device="cuda")
    st = status_word()
    code = G.GPT2_BF16 if dtype == "bf16" else G.GPT2_FP32
    G.gpt2_op_embed(code, dev(ids, "i32"), dev(wte, dtype), dev(wpe, dtype), Bn * T, T, C, V, x, st)
    ref = O.embed({"wte": wte, "wpe": wpe}, ids).reshape(Bn * T, C)
    assert max_abs(x.cpu().numpy(), ref) <= 1e-7
    assert int(st.item()) == 0
    bad = ids.copy()
    bad[1, 5] = V + 3
    G.gpt2_op_embed(code, dev(bad, "i32"), dev(wte, dtype), dev(wpe, dtype), Bn * T, T, C, V, x, st)
    torch.cuda.synchronize()
    assert int(st.item()) & 1                 # recorded, and row 0 was read instead
    assert np.allclose(x.cpu().numpy()[T + 5], wte[0] + wpe[5], atol=1e-7)


# ---------------------------------------------------------------- LayerNorm


@pytest.mark.parametrize("C", [64, 768, 1600])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_layernorm(G, dtype, C):
    rng = np.random.default_rng(C)
    M = 301
    x = (rng.standard_normal((M, C)) * 1.7 + 0.4).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(C)).astype(np.float32)
    b = (0.1 * rng.standard_normal(C)).astype(np.float32)
    if dtype == "bf16":
        g, b = synthetic.round_to_bf16(g), synthetic.round_to_bf16(b)
    out = torch.empty(M, C, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    code = G.GPT2_BF16 if dtype == "bf16" else G.GPT2_FP32
    G.gpt2_op_layernorm(code, dev(x, "fp32"), dev(g, dtype), dev(b, dtype), M, C, out)
    ref = O.layer_norm(x.astype(np.float64), g, b)
    got = out.float().cpu().numpy()
    if dtype == "fp32":
        assert max_abs(got, ref) <= 2e-5
    else:
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)


# ------------------------------------------------------------------- Linear

LINEAR_SHAPES = [
    (300, 2304, 768),     # c_attn-like, ragged M
    (128, 200, 64),       # one m-tile, N tail inside a 64-column group
    (515, 776, 256),      # N tail past 768
    (64, 1600, 1600),     # partial m-tile only
    (5, 2304, 768),       # a few rows: the few-row path (8 rows held, 4 columns per warp)
    (16, 776, 3072),      # its largest row count, N tail, long K (one column per warp, K streamed)
    (4, 3072, 768),       # the decoding step's c_fc shape
    (1, 768, 3072),       # one row, long K
    (12, 200, 1024),      # 16 rows held, 2 columns per warp, N tail
]


def pin_gemm(monkeypatch, bn, pair):
    """Pin the tcgen05 GEMM's tile width ("" = cost model) and whether CTA
    pairs (256-row tiles over two SMs, opt-in) run ("1") or not ("0")."""
    if bn:
        monkeypatch.setenv("G2_GEMM_BN", bn)
    else:
        monkeypatch.delenv("G2_GEMM_BN", raising=False)
    monkeypatch.setenv("G2_GEMM_PAIR", pair)


# (pair, tile width): a pair's tiles are at least 128 columns wide
GEMM_PINS = [(p, bn) for p in ("0", "1") for bn in ("64", "128", "192", "256", "") if not (p == "1" and bn == "64")]


@pytest.mark.parametrize("pair,bn", GEMM_PINS)
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
@pytest.mark.parametrize("shape", LINEAR_SHAPES)
def test_linear_bf16_tcgen05(G, shape, epi, pair, bn, monkeypatch):
    pin_gemm(monkeypatch, bn, pair)
    M, N, K = shape
    rng = np.random.default_rng(M * 7 + N + K + epi)
    A = bf16_exact(rng, (M, K))
    W = bf16_exact(rng, (N, K), 1.0 / math.sqrt(K))
    bias = bf16_exact(rng, (N,), 0.1)
    st = status_word()
    ref = O.linear(A.astype(np.float64), W.astype(np.float64), bias.astype(np.float64))
    if epi == 2:
        x0 = rng.standard_normal((M, N)).astype(np.float32)
        out = dev(x0, "fp32")
        ref = ref + x0
    else:
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        if epi == 1:
            ref = O.gelu(ref)
        if epi == 3:
            ref = O.gelu_tanh(ref)
    G.gpt2_op_linear(G.GPT2_BF16, epi, dev(A, "bf16"), dev(W, "bf16"), dev(bias, "bf16"), M, N, K, out, st)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert int(st.item()) == 0
    if epi == 2:
        assert max_abs(got, ref) <= 1e-4 * max(1.0, math.sqrt(K) / 16)
    else:
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-4)


@pytest.mark.parametrize("pair", ["0", "1"])
@pytest.mark.parametrize("M,N,K,epi", [(4096, 2304, 768, 0), (4096, 3072, 768, 1), (4096, 768, 768, 2),
                                       (4096, 768, 3072, 2)])
def test_linear_bf16_block_shapes(G, M, N, K, epi, pair, monkeypatch):
    """The four Linear layers of a 124M block at B 4, T 1024 (several waves of
    tiles per SM or SM pair), with the tile widths the cost model picks."""
    pin_gemm(monkeypatch, "", pair)
    rng = np.random.default_rng(M + N + K + epi)
    A = bf16_exact(rng, (M, K))
    W = bf16_exact(rng, (N, K), 1.0 / math.sqrt(K))
    bias = bf16_exact(rng, (N,), 0.1)
    ref = O.linear(A.astype(np.float64), W.astype(np.float64), bias.astype(np.float64))
    if epi == 2:
        x0 = rng.standard_normal((M, N)).astype(np.float32)
        out = dev(x0, "fp32")
        ref = ref + x0
    else:
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        if epi == 1:
            ref = O.gelu(ref)
    st = status_word()
    G.gpt2_op_linear(G.GPT2_BF16, epi, dev(A, "bf16"), dev(W, "bf16"), dev(bias, "bf16"), M, N, K, out, st)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert int(st.item()) == 0
    if epi == 2:
        assert max_abs(got, ref) <= 1e-4 * max(1.0, math.sqrt(K) / 16)
    else:
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-4)


def test_gelu_epilogue_within_one_bf16_ulp(G):
    """The c_fc epilogue's GELU on exactly representable pre-activations in
    [-8, 8] (identity weights, zero bias) against the fp64 erf form, after the
    same bf16 rounding: at most one bf16 ulp apart (the erf approximation's
    error, a few 1e-7 absolute, only matters at rounding boundaries)."""
    M = N = K = 64 * 4
    xs = synthetic.round_to_bf16(np.linspace(-8, 8, M).astype(np.float32))
    A = np.zeros((M, K), np.float32)
    A[np.arange(M), np.arange(M) % K] = xs
    W = np.eye(N, K, dtype=np.float32)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    G.gpt2_op_linear(G.GPT2_BF16, 1, dev(A, "bf16"), dev(W, "bf16"), dev(np.zeros(N, np.float32), "bf16"), M, N, K,
                     out)
    got = out.float().cpu().numpy()[np.arange(M), np.arange(M) % K]
    exact = O.gelu(xs.astype(np.float64))
    ref = torch.from_numpy(exact).to(torch.bfloat16).float().numpy()
    # one bf16 ulp, plus 1e-6 absolute: for x < -5 the exact value is below
    # 1e-6 and fp32's 1 + erf(x / sqrt 2) cancels to 0 (as CUDA's erff does)
    ulp = np.abs(ref) * 2.0 ** -7
    assert np.all(np.abs(got - ref) <= ulp + 1e-6)
    assert np.abs(got - exact).max() <= 2.0 ** -8 * 8


@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_linear_fp32_simt(G, epi):
    M, N, K = 130, 200, 72
    rng = np.random.default_rng(40 + epi)
    A = rng.standard_normal((M, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32) / math.sqrt(K)
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    ref = O.linear(A.astype(np.float64), W.astype(np.float64), bias.astype(np.float64))
    if epi == 2:
        x0 = rng.standard_normal((M, N)).astype(np.float32)
        out = dev(x0, "fp32")
        ref = ref + x0
    else:
        out = torch.empty(M, N, dtype=torch.float32, device="cuda")
        if epi == 1:
            ref = O.gelu(ref)
        if epi == 3:
            ref = O.gelu_tanh(ref)
    G.gpt2_op_linear(G.GPT2_FP32, epi, dev(A, "fp32"), dev(W, "fp32"), dev(bias, "fp32"), M, N, K, out)
    assert max_abs(out.cpu().numpy(), ref) <= 2e-5


# ---------------------------------------------------------------- attention


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("B,T,H,C", [(2, 200, 4, 256), (1, 64, 2, 64), (3, 1, 12, 768), (1, 333, 12, 768),
                                     (1, 1024, 12, 768), (2, 1000, 4, 256), (1, 2048, 2, 128)])
def test_attention(G, dtype, B, T, H, C):
    # the longer cases split their last query tiles into two key ranges merged at the end
    rng = np.random.default_rng(B * 1000 + T + H)
    qkv = bf16_exact(rng, (B * T, 3 * C))
    y = torch.empty(B * T, C, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    code = G.GPT2_BF16 if dtype == "bf16" else G.GPT2_FP32
    G.gpt2_op_attention(code, dev(qkv, dtype), B, T, H, C, y)
    ref = O.causal_self_attention(qkv.astype(np.float64).reshape(B, T, 3 * C), H).reshape(B * T, C)
    got = y.float().cpu().numpy()
    if dtype == "fp32":
        assert max_abs(got, ref) <= 1e-5
    else:
        assert rel_l2(got, ref) <= 5e-3
        assert max_abs(got, ref) <= 2e-2
        # a second launch (split flags and counters reset by the first) gives the same bits
        y2 = torch.empty_like(y)
        G.gpt2_op_attention(code, dev(qkv, dtype), B, T, H, C, y2)
        assert torch.equal(y, y2)


# ------------------------------------------------------- lm_head + cross-entropy


@pytest.mark.parametrize("pair,bn", GEMM_PINS)
@pytest.mark.parametrize("M,C,V", [(300, 768, 1000), (128, 128, 50257), (300, 128, 50257)])
def test_lmhead_ce_bf16(G, M, C, V, pair, bn, monkeypatch):
    pin_gemm(monkeypatch, bn, pair)
    rng = np.random.default_rng(M + C + V)
    hf = bf16_exact(rng, (M, C))
    wte = bf16_exact(rng, (V, C), 0.05)
    targets = rng.integers(0, V, size=M).astype(np.int32)
    targets[::7] = -1                         # ignored positions
    targets[3] = V - 1                        # last real column (inside the padded tile)
    ws = torch.empty(G.gpt2_op_lmhead_ce_workspace_bytes(G.GPT2_BF16, M, V), dtype=torch.uint8, device="cuda")
    logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
    tok = torch.empty(M, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    st = status_word()
    G.gpt2_op_lmhead_ce(G.GPT2_BF16, dev(hf, "bf16"), dev(wte, "bf16"), dev(targets, "i32"), M, C, V, logits, tok,
                        loss, ws, st)
    torch.cuda.synchronize()
    z = hf.astype(np.float64) @ wte.astype(np.float64).T
    lse = O.logsumexp_last(z)
    valid = targets >= 0
    ref_tok = np.where(valid, lse - z[np.arange(M), np.maximum(targets, 0)], 0.0)
    assert int(st.item()) == 0
    assert max_abs(logits.cpu().numpy(), z) <= 1e-4 * math.sqrt(C) / 8
    assert max_abs(tok.cpu().numpy(), ref_tok) <= 1e-4
    assert abs(float(loss.item()) - ref_tok[valid].mean()) <= 1e-5
    # loss-only call (no logits) gives the same losses
    tok2 = torch.empty_like(tok)
    G.gpt2_op_lmhead_ce(G.GPT2_BF16, dev(hf, "bf16"), dev(wte, "bf16"), dev(targets, "i32"), M, C, V, None, tok2,
                        loss, ws, st)
    assert torch.equal(tok, tok2)


def test_lmhead_ce_fp32(G):
    M, C, V = 70, 64, 512
    rng = np.random.default_rng(3)
    hf = rng.standard_normal((M, C)).astype(np.float32)
    wte = (rng.standard_normal((V, C)) * 0.1).astype(np.float32)
    targets = rng.integers(-1, V, size=M).astype(np.int32)
    ws = torch.empty(G.gpt2_op_lmhead_ce_workspace_bytes(G.GPT2_FP32, M, V), dtype=torch.uint8, device="cuda")
    logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
    tok = torch.empty(M, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    G.gpt2_op_lmhead_ce(G.GPT2_FP32, dev(hf, "fp32"), dev(wte, "fp32"), dev(targets, "i32"), M, C, V, logits, tok,
                        loss, ws)
    z = hf.astype(np.float64) @ wte.astype(np.float64).T
    lse = O.logsumexp_last(z)
    valid = targets >= 0
    ref_tok = np.where(valid, lse - z[np.arange(M), np.maximum(targets, 0)], 0.0)
    assert max_abs(logits.cpu().numpy(), z) <= 1e-5
    assert max_abs(tok.cpu().numpy(), ref_tok) <= 1e-5
    assert abs(float(loss.item()) - ref_tok[valid].mean()) <= 1e-6


def test_lmhead_ce_no_targets_sets_status(G):
    M, C, V = 16, 64, 100
    hf = torch.zeros(M, C, dtype=torch.float32, device="cuda")
    wte = torch.zeros(V, C, dtype=torch.float32, device="cuda")
    tg = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(G.gpt2_op_lmhead_ce_workspace_bytes(G.GPT2_FP32, M, V), dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    st = status_word()
    G.gpt2_op_lmhead_ce(G.GPT2_FP32, hf, wte, tg, M, C, V, None, None, loss, ws, st)
    torch.cuda.synchronize()
    assert math.isnan(float(loss.item()))
    assert int(st.item()) & 4


# ------------------------------------------------------ sinusoidal position table


@pytest.mark.parametrize("n_ctx,C", [(1024, 768), (7, 10), (1, 2)])
def test_fill_sinusoidal_wpe(G, n_ctx, C):
    ref = O.sinusoidal_wpe(n_ctx, C)
    f32 = torch.empty(n_ctx, C, dtype=torch.float32, device="cuda")
    G.gpt2_fill_sinusoidal_wpe(G.GPT2_FP32, f32, n_ctx, C)
    torch.cuda.synchronize()
    assert max_abs(f32.cpu().numpy(), ref) <= 1e-7          # one fp32 rounding of values in [-1, 1]
    b16 = torch.empty(n_ctx, C, dtype=torch.bfloat16, device="cuda")
    G.gpt2_fill_sinusoidal_wpe(G.GPT2_BF16, b16, n_ctx, C)
    torch.cuda.synchronize()
    got = b16.float().cpu().numpy()
    # one round-to-nearest to bf16 (8 significant bits): |error| <= 2^-8 |value|
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 * 1.0001)
    with pytest.raises(G.GPT2Error):
        G.gpt2_fill_sinusoidal_wpe(G.GPT2_FP32, f32, n_ctx, C + 1)   # odd C


@pytest.mark.parametrize("C", [768, 1024, 1600])
def test_embed_layernorm_fused(G, C):
    """The embedding sum and ln_1 in one kernel: x as gpt2_op_embed writes it,
    h = LayerNorm(x) against the oracle (one bf16 rounding)."""
    M, T, V = 3 * 77, 77, 999
    rng = np.random.default_rng(C + 1)
    ids = rng.integers(0, V, size=M).astype(np.int32)
    wte, wpe = bf16_exact(rng, (V, C), 0.5), bf16_exact(rng, (T, C), 0.5)
    g, b = bf16_exact(rng, (C,), 1.0), bf16_exact(rng, (C,), 0.2)
    x = torch.empty(M, C, dtype=torch.float32, device="cuda")
    h = torch.empty(M, C, dtype=torch.bfloat16, device="cuda")
    st = status_word()
    G.gpt2_op_embed_layernorm(torch.from_numpy(ids).cuda(), dev(wte, "bf16"), dev(wpe, "bf16"), M, T, C, V,
                              dev(g, "bf16"), dev(b, "bf16"), x, h, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rx = wte[ids].astype(np.float64) + wpe[np.arange(M) % T]
    assert max_abs(x.cpu().numpy(), rx) <= 1e-6
    rh = O.layer_norm(rx, g.astype(np.float64), b.astype(np.float64))
    got = h.float().cpu().numpy()
    assert np.all(np.abs(got - rh) <= np.abs(rh) * 2.0 ** -8 + 1e-4)
