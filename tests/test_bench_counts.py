"""The counts behind bench.py's rates: the parameter count equals the sizes of
the weights the generator draws, the model FLOPs per step are the products of
the forward pass counted term by term, and the lm_head's FLOPs are its one
product."""
import bench
import synthetic


def test_parameter_count_matches_the_drawn_weights():
    for wl in (synthetic.WORKLOADS[0], synthetic.random_case(5, 3, 4, 96, 700, 48, 2, 8)):
        W = synthetic.make_weights(wl)
        n = W["wte"].size + W["wpe"].size + W["lnf_g"].size + W["lnf_b"].size
        n += sum(d[k].size for d in W["layers"] for k in synthetic.LAYER_KEYS)
        assert bench.n_params(wl) == n


def test_model_flops_term_by_term():
    wl = bench.WL   # GPT-2 124M, B 4, T 1024
    B, T, C, V, L = wl.batch, wl.seq, wl.n_embd, wl.vocab, wl.n_layer
    tokens = B * T
    linear = L * (C * 3 * C + C * C + C * 4 * C + 4 * C * C)          # weights of the four Linear layers
    elementwise = L * (3 * C + C + 4 * C + C + 4 * C) + 2 * C         # biases and the LayerNorm scales / shifts
    head = V * C                                                      # the tied lm_head
    attention = L * B * 2 * (2 * C) * (T * (T + 1) // 2)              # QK^T and PV over the causal pairs
    expected = 2.0 * (linear + elementwise + head) * tokens + attention
    assert bench.model_flops(wl) == expected
    assert abs(expected / 1e12 - 1.0904) < 0.0005                    # ~1.090 TFLOP per step
    assert bench.lmhead_flops(wl, tokens) == 2.0 * tokens * V * C
