"""The seeded input generator (synthetic/) holds to its stated recipe: the
same seed gives the same values, bf16 workloads are bf16-exact, the draws
have the stated distributions, padding and targets follow the position-aligned
shift. Both the oracle and the GPU path read these inputs, so a change here
would move both sides at once; these checks pin the recipe itself."""
import numpy as np
import torch

import synthetic

TINY = synthetic.WORKLOADS[0]
CASE = synthetic.random_case(900, n_layer=2, n_head=4, n_embd=256, vocab=3000, n_ctx=64, batch=3, seq=40)


def test_same_seed_same_values():
    a, b = synthetic.make_weights(CASE), synthetic.make_weights(CASE)
    assert np.array_equal(a["wte"], b["wte"]) and np.array_equal(a["lnf_b"], b["lnf_b"])
    for la, lb in zip(a["layers"], b["layers"]):
        for k in synthetic.LAYER_KEYS:
            assert np.array_equal(la[k], lb[k])
    assert np.array_equal(synthetic.make_ids(CASE), synthetic.make_ids(CASE))
    other = synthetic.make_weights(CASE.scaled(index=901))
    assert not np.array_equal(other["wte"], a["wte"])


def test_round_to_bf16_is_nearest_even_and_exact():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(10000).astype(np.float32) * 3
    r = synthetic.round_to_bf16(x)
    # exactly representable: a round trip through torch's bf16 changes nothing
    assert np.array_equal(torch.from_numpy(r).to(torch.bfloat16).float().numpy(), r)
    # the same rounding as torch's (nearest, ties to even)
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), r)
    # a tie goes to the even mantissa: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert synthetic.round_to_bf16(np.array([1 + 2.0 ** -8], np.float32))[0] == 1.0
    assert synthetic.round_to_bf16(np.array([1 + 3 * 2.0 ** -8], np.float32))[0] == 1 + 2.0 ** -6


def test_bf16_workloads_are_bf16_exact_and_fp32_ones_are_not_rounded():
    w = synthetic.make_weights(CASE)
    for arr in [w["wte"], w["wpe"], w["lnf_g"], w["layers"][1]["fc_w"], w["layers"][0]["attn_b"]]:
        assert np.array_equal(synthetic.round_to_bf16(arr), arr)
    t = synthetic.make_weights(TINY)   # fp32 workload: full float32 draws
    assert not np.array_equal(synthetic.round_to_bf16(t["wte"]), t["wte"])


def test_stated_distributions():
    w = synthetic.make_weights(CASE)            # init "dist"
    L = CASE.n_layer
    assert abs(w["wte"].std() - 0.02) < 0.02 * 0.02
    assert abs(w["wte"].mean()) < 1e-3
    proj = np.concatenate([d["mlp_proj_w"].ravel() for d in w["layers"]])
    assert abs(proj.std() - 0.02 / np.sqrt(2 * L)) < 0.02 * 0.02
    g = np.concatenate([d["ln1_g"] for d in w["layers"]])
    assert abs(g.mean() - 1.0) < 0.02 and abs(g.std() - 0.1) < 0.01
    gpt2_init = synthetic.make_weights(CASE.scaled(init="gpt2"))
    assert (gpt2_init["layers"][0]["ln1_g"] == 1).all() and (gpt2_init["layers"][0]["fc_b"] == 0).all()
    ids = synthetic.make_ids(CASE)
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < CASE.vocab
    big = synthetic.make_ids(CASE.scaled(batch=64, seq=1000))
    counts = np.bincount(big.ravel(), minlength=CASE.vocab)
    assert counts.min() > 0   # 64000 uniform draws over 3000 ids leave none empty


def test_padding_and_targets():
    wl = CASE.scaled(batch=3, seq=10, lengths=(10, 4, 1))
    ids = synthetic.make_ids(wl)
    assert (ids[1, 4:] == 0).all() and (ids[2, 1:] == 0).all()
    lengths = synthetic.lengths_of(wl)
    tg = synthetic.next_token_targets(ids, lengths)
    assert tg.dtype == np.int32 and tg.shape == ids.shape
    assert np.array_equal(tg[0, :9], ids[0, 1:]) and tg[0, 9] == -1
    assert np.array_equal(tg[1, :3], ids[1, 1:4]) and (tg[1, 3:] == -1).all()
    assert (tg[2] == -1).all()    # a one-token sequence has nothing to predict
    full = synthetic.next_token_targets(ids)
    assert np.array_equal(full[:, :-1], ids[:, 1:]) and (full[:, -1] == -1).all()
