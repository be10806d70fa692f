"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- the numbers the pages print, closed forms, library routines for a
special case, and brute force on tiny inputs.  CPU only."""

import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import indexer_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)["facts"]


def _printed(n, fact):
    """Round n to the number of significant digits the page prints."""
    return round(n / fact["scale"], fact["digits"] - len(str(int(fact["mantissa"])))) == fact["mantissa"]


# ---------------------------------------------------------------- page numbers

def test_shapes_follow_the_pages():
    f = _facts()
    shapes = oracle.parameter_shapes(f["model_width"]["value"], f["q_latent_dim"]["value"],
                                     f["indexer_heads"]["value"], f["indexer_head_dim"]["value"])
    assert shapes["W_q"] == (f["q_latent_dim"]["value"], f["q_projection_out"]["value"])
    assert shapes["W_w"] == (f["weight_projection_in"]["value"], f["weight_projection_out"]["value"])
    assert shapes["W_k"][1] == f["key_dim"]["value"]
    assert f["indexer_heads"]["value"] * f["indexer_head_dim"]["value"] == f["q_projection_out"]["value"]
    assert f["index_rope_dim"]["value"] == 0  # the oracle applies no rotary step at all


def test_parameter_count_matches_printed_figures():
    f = _facts()
    n = oracle.parameter_count()
    assert n == 7_438_592
    assert _printed(n, f["params_per_layer_printed"])
    assert _printed(f["indexer_layers"]["value"] * n, f["params_total_printed"])


def test_parameter_count_rejects_biased_projections():
    # Bias vectors on the three projections (4,096 + 128 + 32 per layer) still
    # print as 7.44M per layer but not as 178.5M over 24 layers.
    f = _facts()
    biased = oracle.parameter_count() + 4096 + 128 + 32
    assert _printed(biased, f["params_per_layer_printed"])
    assert not _printed(f["indexer_layers"]["value"] * biased, f["params_total_printed"])


def test_project_consumes_exactly_the_counted_parameters():
    rng = np.random.default_rng(0)
    T, hd, ql, H, D = 3, 16, 8, 2, 4
    shapes = oracle.parameter_shapes(hd, ql, H, D)
    ws = {k: rng.standard_normal(s) for k, s in shapes.items()}
    q, k, w = oracle.project(rng.standard_normal((T, hd)), rng.standard_normal((T, ql)),
                             ws["W_q"], ws["W_k"], ws["W_w"], ws["ln_gamma"], ws["ln_beta"],
                             n_heads=H, head_dim=D)
    assert q.shape == (T, H, D) and k.shape == (T, D) and w.shape == (T, H)
    bad = dict(ws)
    bad["W_k"] = np.concatenate([ws["W_k"], np.zeros((1, D))])  # a bias row folded in
    with pytest.raises(ValueError):
        oracle.project(rng.standard_normal((T, hd)), rng.standard_normal((T, ql)),
                       bad["W_q"], bad["W_k"], bad["W_w"], bad["ln_gamma"], bad["ln_beta"],
                       n_heads=H, head_dim=D)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_conversion_of_fp32_values():
    rng = np.random.default_rng(1)
    mant = rng.uniform(1.0, 2.0, 200_000)
    expo = rng.integers(-149, 128, 200_000)
    sign = rng.choice([-1.0, 1.0], 200_000)
    x32 = (sign * np.ldexp(mant, expo)).astype(np.float32)   # includes fp32 subnormals and near-max values
    x32 = x32[np.isfinite(x32)]
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(x32.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_go_to_even():
    ulp = 2.0 ** -7
    assert oracle.bf16_round(1.0 + ulp / 2) == 1.0                 # tie, 1.0 is even
    assert oracle.bf16_round(1.0 + 3 * ulp / 2) == 1.0 + 2 * ulp   # tie, goes up to even
    assert oracle.bf16_round(1.0 + ulp / 2 + 2.0 ** -30) == 1.0 + ulp
    assert oracle.bf16_round(-(1.0 + ulp / 2)) == -1.0
    assert oracle.bf16_round(2.0 ** 128 * (1 - 2.0 ** -9)) == np.inf  # rounds past the largest finite bf16
    assert oracle.bf16_round(0.0) == 0.0


def test_bf16_bits_round_trip():
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)
    vals = oracle.bf16_bits_to_float64(bits)
    np.testing.assert_array_equal(oracle.float64_to_bf16_bits(vals), bits)
    np.testing.assert_array_equal(oracle.bf16_round(vals), vals)


# ---------------------------------------------------------------- LayerNorm

def test_layer_norm_matches_torch_float64():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128)) * 3 + 0.5
    g = 1 + 0.02 * rng.standard_normal(128)
    b = 0.02 * rng.standard_normal(128)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (128,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.layer_norm(x, g, b, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_layer_norm_closed_form():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 128)) * 0.1
    eps = 1e-3
    y = oracle.layer_norm(x, np.ones(128), np.zeros(128), eps)
    v = x.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), v / (v + eps), rtol=1e-12)
    # scale invariance up to eps, and the affine part is applied after normalising
    np.testing.assert_allclose(oracle.layer_norm(7 * x, np.ones(128), np.zeros(128), 0.0),
                               oracle.layer_norm(x, np.ones(128), np.zeros(128), 0.0), rtol=1e-10)
    g = rng.standard_normal(128)
    b = rng.standard_normal(128)
    np.testing.assert_allclose(oracle.layer_norm(x, g, b, eps), y * g + b, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- projections, brute force

def _py_project(hidden, q_latent, Wq, Wk, Ww, gamma, beta, eps, H, D):
    """Pure-Python loops, dyadic inputs (every sum exact in float64)."""
    T = len(hidden)
    q = [[[sum(q_latent[t][i] * Wq[i][h * D + d] for i in range(len(Wq))) for d in range(D)]
          for h in range(H)] for t in range(T)]
    kraw = [[sum(hidden[t][i] * Wk[i][d] for i in range(len(Wk))) for d in range(D)] for t in range(T)]
    k = []
    for row in kraw:
        mu = sum(row) / D
        var = sum((v - mu) ** 2 for v in row) / D
        k.append([(row[d] - mu) / (var + eps) ** 0.5 * gamma[d] + beta[d] for d in range(D)])
    w = [[sum(hidden[t][i] * Ww[i][h] for i in range(len(Ww))) for h in range(H)] for t in range(T)]
    return np.array(q), np.array(k), np.array(w)


def test_project_matches_python_loops_on_tiny_dyadic_inputs():
    rng = np.random.default_rng(4)
    T, hd, ql, H, D = 5, 12, 10, 3, 4
    hidden = rng.integers(-4, 5, (T, hd)).astype(np.float64)
    q_latent = rng.integers(-4, 5, (T, ql)).astype(np.float64)
    Wq = rng.integers(-8, 9, (ql, H * D)) / 8.0
    Wk = rng.integers(-8, 9, (hd, D)) / 8.0
    Ww = rng.integers(-8, 9, (hd, H)) / 8.0
    gamma = 1 + rng.integers(-4, 5, D) / 64.0
    beta = rng.integers(-4, 5, D) / 64.0
    eps = 2.0 ** -10
    q, k, w = oracle.project(hidden, q_latent, Wq, Wk, Ww, gamma, beta, eps, H, D)
    pq, pk, pw = _py_project(hidden.tolist(), q_latent.tolist(), Wq.tolist(), Wk.tolist(),
                             Ww.tolist(), gamma.tolist(), beta.tolist(), eps, H, D)
    np.testing.assert_array_equal(q, oracle.bf16_round(pq))       # sums are exact, one rounding
    np.testing.assert_allclose(k, oracle.bf16_round(pk), rtol=2.0 ** -8)  # sqrt may differ in the last fp64 bit
    np.testing.assert_array_equal(w, pw.astype(np.float32).astype(np.float64))
    # q head h is columns h*D .. h*D+D-1 of the projection
    np.testing.assert_array_equal(q.reshape(T, H * D), oracle.bf16_round(q_latent @ Wq))


# ---------------------------------------------------------------- score and selection, brute force

def _py_scores(q_t, w_t, keys):
    out = []
    for k in keys:
        tot = 0.0
        for h in range(len(q_t)):
            dot = sum(q_t[h][d] * k[d] for d in range(len(k)))
            tot += w_t[h] * max(0.0, dot)
        out.append(tot)
    return out


@pytest.mark.parametrize("H,D,top_k", [(1, 2, 1), (1, 4, 3), (2, 2, 3), (2, 4, 1), (2, 4, 3)])
def test_topk_matches_bruteforce_on_tiny_inputs(H, D, top_k):
    rng = np.random.default_rng(100 + 10 * H + D + top_k)
    T = 12
    q = rng.integers(-3, 4, (T, H, D)).astype(np.float64)
    w = rng.integers(-2, 3, (T, H)) / 2.0
    keys = rng.integers(-3, 4, (T, D)).astype(np.float64)
    pos = np.arange(T)
    offs = np.array([0, T])
    idx, sc = oracle.topk(q, w, pos, offs, keys, offs, top_k=top_k)
    for t in range(T):
        I = _py_scores(q[t].tolist(), w[t].tolist(), keys[: t + 1].tolist())
        n = t + 1
        if n <= top_k:
            assert idx[t].tolist() == list(range(n)) + [-1] * (top_k - n)
            continue
        sel = idx[t].tolist()
        assert len(set(sel)) == top_k and all(0 <= s <= t for s in sel)   # causal, inclusive
        # the chosen set is a best set: it maximises the sum and the minimum over all subsets
        best_sum = max(sum(I[s] for s in c) for c in itertools.combinations(range(n), top_k))
        best_min = max(min(I[s] for s in c) for c in itertools.combinations(range(n), top_k))
        assert sum(I[s] for s in sel) == best_sum
        assert min(I[s] for s in sel) == best_min
        # order: score descending, position ascending
        keyed = [(-I[s], s) for s in sel]
        assert keyed == sorted(keyed)
        # ties at the boundary go to the lower positions
        thr = min(I[s] for s in sel)
        unsel = [s for s in range(n) if s not in sel]
        assert all(I[s] < thr or s > max(x for x in sel if I[x] == thr) for s in unsel)
        np.testing.assert_array_equal(sc[t], [I[s] for s in sel])


def test_scores_match_python_loops():
    rng = np.random.default_rng(5)
    q = rng.integers(-5, 6, (4, 8)).astype(np.float64)
    w = rng.integers(-4, 5, 4) / 4.0
    keys = rng.integers(-5, 6, (30, 8)).astype(np.float64)
    I, A = oracle.index_scores(q, w, keys)
    np.testing.assert_array_equal(I, _py_scores(q.tolist(), w.tolist(), keys.tolist()))
    np.testing.assert_array_equal(A, [sum(abs(w[h] * (q[h] @ k)) for h in range(4)) for k in keys])


# ---------------------------------------------------------------- invariants and special cases

def _rand_case(seed, T=40, H=4, D=8):
    rng = np.random.default_rng(seed)
    q = oracle.bf16_round(rng.standard_normal((T, H, D)))
    w = rng.standard_normal((T, H)).astype(np.float32).astype(np.float64)
    keys = oracle.bf16_round(rng.standard_normal((T, D)))
    return q, w, keys


def test_zero_head_weights_give_zero_scores():
    q, w, keys = _rand_case(6)
    I, A = oracle.index_scores(q[0], np.zeros(4), keys)
    assert np.all(I == 0.0)


def test_relu_terms_nonnegative_for_nonnegative_weights():
    q, w, keys = _rand_case(7)
    for t in range(10):
        I, A = oracle.index_scores(q[t], np.abs(w[t]), keys)
        assert np.all(I >= 0.0)
        assert np.all(I <= A + 1e-12)
    # every head term alone carries the sign of its weight
    for h in range(4):
        wh = np.zeros(4)
        wh[h] = -abs(w[0, h]) - 0.5
        I, _ = oracle.index_scores(q[0], wh, keys)
        assert np.all(I <= 0.0)


def test_single_head_unit_weight_is_textbook_relu_topk():
    rng = np.random.default_rng(8)
    D, n, k = 16, 500, 37
    q = oracle.bf16_round(rng.standard_normal((1, D)))
    keys = oracle.bf16_round(rng.standard_normal((n, D)))
    I, _ = oracle.index_scores(q, np.ones(1), keys)
    relu = np.maximum(keys @ q[0], 0)
    np.testing.assert_array_equal(I, relu)
    sel = oracle.select_topk(I, k)
    ref = np.argpartition(-relu, k - 1)[:k]
    np.testing.assert_array_equal(np.sort(relu[sel]), np.sort(relu[ref]))


def test_short_prefix_selects_everything_in_position_order():
    q, w, keys = _rand_case(9, T=40)
    pos = np.arange(40)
    offs = np.array([0, 40])
    idx, sc = oracle.topk(q, w, pos, offs, keys, offs, top_k=16)
    for t in range(16):
        assert idx[t].tolist() == list(range(t + 1)) + [-1] * (15 - t)
        assert np.all(np.isneginf(sc[t, t + 1:]))
    for t in range(16, 40):
        assert np.all(idx[t] >= 0) and np.all(idx[t] <= t)


def test_future_keys_do_not_matter():
    q, w, keys = _rand_case(10, T=40)
    pos = np.arange(40)
    offs = np.array([0, 40])
    a = oracle.topk(q, w, pos, offs, keys, offs, top_k=8)[0]
    for t in (5, 20, 33):
        keys2 = keys.copy()
        keys2[t + 1:] = oracle.bf16_round(np.random.default_rng(t).standard_normal(keys2[t + 1:].shape)) * 9
        b = oracle.topk(q[t:t + 1], w[t:t + 1], pos[t:t + 1], np.array([0, 1]), keys2, offs, top_k=8)[0]
        np.testing.assert_array_equal(a[t], b[0])


def test_permuting_visible_keys_permutes_indices():
    q, w, keys = _rand_case(11, T=60)
    perm = np.random.default_rng(12).permutation(60)
    t = 59
    one = np.array([0, 1])
    offs = np.array([0, 60])
    a = oracle.topk(q[t:t + 1], w[t:t + 1], np.array([59]), one, keys, offs, top_k=10)[0][0]
    b = oracle.topk(q[t:t + 1], w[t:t + 1], np.array([59]), one, keys[perm], offs, top_k=10)[0][0]
    assert set(perm[b].tolist()) == set(a.tolist())


def test_positive_weight_scale_keeps_the_set():
    q, w, keys = _rand_case(13, T=60)
    pos = np.arange(60)
    offs = np.array([0, 60])
    a = oracle.topk(q, w, pos, offs, keys, offs, top_k=9)[0]
    b = oracle.topk(q, w * 8.0, pos, offs, keys, offs, top_k=9)[0]
    np.testing.assert_array_equal(a, b)


def test_sequences_are_independent():
    q, w, keys = _rand_case(14, T=40)
    # sequence 0: tokens 0..24 at positions 0..24; sequence 1: tokens 25..39 at positions 0..14
    pos = np.concatenate([np.arange(25), np.arange(15)])
    qoff = np.array([0, 25, 40])
    coff = np.array([0, 25, 40])
    idx, _ = oracle.topk(q, w, pos, qoff, keys, coff, top_k=6)
    a = oracle.topk(q[:25], w[:25], pos[:25], np.array([0, 25]), keys[:25], np.array([0, 25]), top_k=6)[0]
    b = oracle.topk(q[25:], w[25:], pos[25:], np.array([0, 15]), keys[25:], np.array([0, 15]), top_k=6)[0]
    np.testing.assert_array_equal(idx, np.concatenate([a, b]))


def test_sorted_order_helper():
    I = np.array([0.5, 2.0, 2.0, -1.0, 3.0])
    assert oracle.sort_selected(np.array([0, 1, 2, 4, -1]), I).tolist() == [4, 1, 2, 0, -1]


# ---------------------------------------------------------------- planted mistakes are caught

def _bruteforce_ok(score_fn):
    rng = np.random.default_rng(200)
    q = rng.integers(-3, 4, (8, 2, 4)).astype(np.float64)
    w = rng.integers(-2, 3, (8, 2)) / 2.0
    keys = rng.integers(-3, 4, (8, 4)).astype(np.float64)
    for t in range(8):
        I, _ = score_fn(q[t], w[t], keys[: t + 1])
        if not np.array_equal(I, _py_scores(q[t].tolist(), w[t].tolist(), keys[: t + 1].tolist())):
            return False
    return True


@pytest.mark.parametrize("mistake", ["no_relu", "relu_after_weight", "transposed_heads", "abs_weight"])
def test_planted_score_mistakes_fail_the_bruteforce_pin(mistake):
    def wrong(q_t, w_t, keys):
        logits = keys @ q_t.T
        if mistake == "no_relu":
            I = logits @ w_t
        elif mistake == "relu_after_weight":
            I = np.maximum(logits * w_t, 0).sum(axis=1)
        elif mistake == "transposed_heads":
            I = np.maximum(logits, 0) @ w_t[::-1]
        else:
            I = np.maximum(logits, 0) @ np.abs(w_t)
        return I, np.abs(logits) @ np.abs(w_t)
    assert _bruteforce_ok(O.index_scores)
    assert not _bruteforce_ok(wrong)


def test_planted_layernorm_mistakes_fail_the_closed_form():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((16, 128))
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (128,), eps=1e-6).numpy()
    ones, zeros = np.ones(128), np.zeros(128)
    unbiased = (x - x.mean(1, keepdims=True)) / np.sqrt(x.var(1, ddof=1, keepdims=True) + 1e-6)
    rms = x / np.sqrt((x ** 2).mean(1, keepdims=True) + 1e-6)
    assert np.allclose(oracle.layer_norm(x, ones, zeros, 1e-6), ref, atol=1e-10)
    assert not np.allclose(unbiased, ref, atol=1e-6)
    assert not np.allclose(rms, ref, atol=1e-6)


# ---------------------------------------------------------------- index reuse (draft steps)

def test_reuse_gives_every_draft_its_anchors_bruteforce_selection():
    # the first step's selection of each anchor comes from brute-force scoring of its prefix;
    # a draft token at a later position reuses exactly that row ('MTP' row, GLM-5.2)
    rng = np.random.default_rng(31)
    H, D, k, T = 2, 4, 3, 9
    q = rng.standard_normal((T, H, D))
    w = rng.standard_normal((T, H))
    keys = rng.standard_normal((T, D))
    pos = np.arange(T)
    anchors = np.array([4, 6])
    idx, sc = oracle.topk(q[anchors], w[anchors], pos[anchors], np.array([0, 2]), keys, np.array([0, T]),
                          top_k=k)
    drafts = np.array([0, 0, 0, 1, 1, 5])      # anchor row of each draft token; 5 has none
    ri, rs = oracle.reuse_topk(idx, sc, drafts)
    for d, a in enumerate(drafts):
        if a >= len(anchors):
            assert np.all(ri[d] == -1) and np.all(np.isneginf(rs[d]))
            continue
        p = pos[anchors[a]]
        best = max(itertools.combinations(range(p + 1), k),
                   key=lambda c: (sorted((sum(w[anchors[a], h] * max(0.0, q[anchors[a], h] @ keys[s])
                                              for h in range(H)) for s in c)), [-s for s in c]))
        assert set(ri[d].tolist()) == set(best)
        assert ri[d].max() <= p      # causal for the anchor, hence for every later draft position


# ---------------------------------------------------------------- FP8 key cache

def test_e4m3_round_matches_torch_conversion_inside_the_range():
    rng = np.random.default_rng(41)
    mant = rng.uniform(1.0, 2.0, 100_000)
    ex = rng.integers(-12, 9, 100_000)
    x = (np.ldexp(mant, ex) * rng.choice([-1, 1], 100_000)).astype(np.float32).astype(np.float64)
    x = x[np.abs(x) <= 448.0]
    want = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_round(x), want)


def test_e4m3_grid_and_ties():
    # the 126 finite positive codes: 7 subnormals k 2^-9, then (1 + m/8) 2^(e-7)
    grid = [k * 2.0 ** -9 for k in range(1, 8)] + [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16)
                                                      for m in range(8) if not (e == 15 and m == 7)]
    assert len(grid) == 126 and max(grid) == 448.0
    g = np.array(grid)
    assert np.array_equal(oracle.e4m3_round(g), g)
    # midpoints go to the even mantissa; beyond 448 saturates
    assert oracle.e4m3_round(np.array([0.59375]))[0] == 0.625       # between 0.5625 (odd) and 0.625
    assert oracle.e4m3_round(np.array([1.0625]))[0] == 1.0          # between 1.0 (even) and 1.125
    assert oracle.e4m3_round(np.array([3 * 2.0 ** -10]))[0] == 2.0 ** -8   # subnormal tie to even
    assert oracle.e4m3_round(np.array([1000.0, -500.0])).tolist() == [448.0, -448.0]


def test_quantize_fp8_bounds_and_exact_max():
    rng = np.random.default_rng(42)
    v = rng.standard_normal((500, 128)).astype(np.float32)
    codes, scale = oracle.quantize_fp8(v)
    assert codes.shape == v.shape and scale.shape == (500,)
    assert np.all(np.abs(codes) <= 448.0)
    # the row maximum lands on 448 (up to one float32 rounding of v * inv)
    am = np.argmax(np.abs(v), axis=1)
    assert np.all(np.abs(codes[np.arange(500), am]) == 448.0)
    # relative error of a normal-range value is at most half a mantissa step (2^-4)
    deq = codes * scale[:, None]
    big = np.abs(v) >= 2.0 ** -6 * scale[:, None]
    assert np.all(np.abs(deq - v)[big] <= 2.0 ** -4 * np.abs(v)[big] * (1 + 1e-6))
    z, zs = oracle.quantize_fp8(np.zeros((2, 8), np.float32))
    assert np.all(z == 0) and np.all(zs == 0)


def test_fp8_scores_equal_scores_of_the_dequantised_operands():
    # the scale factoring (s_k out of the ReLU, s_q into the head weight) is exact algebra:
    # compare with index_scores of code * scale
    rng = np.random.default_rng(43)
    H, D, n = 4, 16, 50
    q = rng.standard_normal((H, D)).astype(np.float32)
    k = rng.standard_normal((n, D)).astype(np.float32)
    w = rng.standard_normal(H)
    q8, sq = oracle.quantize_fp8(q)
    k8, sk = oracle.quantize_fp8(k)
    I, A = oracle.fp8_index_scores(q8, sq, w, k8, sk)
    I2, A2 = oracle.index_scores(q8 * sq[:, None], w, k8 * sk[:, None])
    assert np.allclose(I, I2, rtol=1e-12, atol=1e-12) and np.allclose(A, A2, rtol=1e-12, atol=1e-12)
    # planted mistake: the key scale left out
    bad = (np.maximum(k8 @ q8.T, 0.0) @ (w * sq))
    assert not np.allclose(bad, I2)


def test_fp8_selection_tracks_the_bf16_selection():
    # quantisation moves scores by a few percent of A: the FP8 top-k keeps almost all of the
    # bf16 top-k on N(0,1) data (the recall the engines accept by caching keys in FP8)
    rng = np.random.default_rng(44)
    T, S = 3, 6000
    q = oracle.bf16_round(rng.standard_normal((T, 32, 128)))
    k = oracle.bf16_round(rng.standard_normal((S, 128)))
    w = rng.standard_normal((T, 32))
    pos = np.array([S - 1, S - 2, 4000])
    idx_b, _ = oracle.topk(q, w, pos, np.array([0, T]), k, np.array([0, S]))
    q8, sq = oracle.quantize_fp8(q.astype(np.float32))
    k8, sk = oracle.quantize_fp8(k.astype(np.float32))
    idx_f, _ = oracle.topk_fp8(q8, sq, w, pos, np.array([0, T]), k8, sk, np.array([0, S]))
    for r in range(T):
        assert len(np.intersect1d(idx_b[r], idx_f[r])) / 2048 > 0.9


# ---------------------------------------------------------------- DeepSeek-V3.2 form: 64 heads, RoPE on 64 dims

def test_rope_identity_cases():
    rng = np.random.default_rng(51)
    x = rng.standard_normal((5, 128))
    assert np.array_equal(oracle.rope(x, np.zeros(5), 64), x)            # position 0
    assert np.array_equal(oracle.rope(x, np.arange(5), 0), x)            # no rotary dims
    y = oracle.rope(x, np.arange(5) * 1000, 64)
    assert np.array_equal(y[:, 64:], x[:, 64:])                          # only the first 64 dims move


def test_rope_is_a_rotation_with_relative_positions():
    rng = np.random.default_rng(52)
    q = rng.standard_normal((7, 128))
    k = rng.standard_normal((7, 128))
    p = rng.integers(0, 100_000, 7).astype(np.float64)
    s = rng.integers(0, 100_000, 7).astype(np.float64)
    rq = oracle.rope(q, p, 64)
    # each rotated pair keeps its length
    assert np.allclose(np.hypot(rq[:, 0:64:2], rq[:, 1:64:2]), np.hypot(q[:, 0:64:2], q[:, 1:64:2]), rtol=1e-12)
    # composition: rotating by p1 then p2 is rotating by p1 + p2
    assert np.allclose(oracle.rope(oracle.rope(q, p, 64), s, 64), oracle.rope(q, p + s, 64), atol=1e-9)
    # the dot product depends on the positions only through their difference
    d = 12345.0
    a = np.sum(oracle.rope(q, p, 64) * oracle.rope(k, s, 64), axis=1)
    b = np.sum(oracle.rope(q, p + d, 64) * oracle.rope(k, s + d, 64), axis=1)
    assert np.allclose(a, b, rtol=1e-9, atol=1e-9)
    # the lowest pair turns by one radian per position, the highest by theta^(-62/64) of one
    e = np.zeros((1, 128))
    e[0, 0] = 1.0
    e[0, 62] = 1.0
    r = oracle.rope(e, np.array([3.0]), 64)
    assert np.isclose(np.arctan2(r[0, 1], r[0, 0]), 3.0 - 0.0)
    assert np.isclose(np.arctan2(r[0, 63], r[0, 62]), 3.0 * 10000.0 ** (-62 / 64))


def test_project_64_heads_with_rope():
    # the 64-head form: W_q 1,536 -> 8,192, W_w 7,168 -> 64 (shapes scaled down here), rotary
    # step on the first 64 dims of q (every head) and of the normalised key
    rng = np.random.default_rng(53)
    T, hd, ql, H, D = 6, 32, 16, 4, 128
    shapes = oracle.parameter_shapes(hd, ql, H, D)
    ws = {k_: rng.standard_normal(s_) * 0.3 for k_, s_ in shapes.items()}
    x, xq = rng.standard_normal((T, hd)), rng.standard_normal((T, ql))
    pos = np.array([0, 1, 7, 100, 5000, 70000])
    q0, k0, w0 = oracle.project(x, xq, ws["W_q"], ws["W_k"], ws["W_w"], ws["ln_gamma"], ws["ln_beta"],
                                n_heads=H, head_dim=D)
    q1, k1, w1 = oracle.project(x, xq, ws["W_q"], ws["W_k"], ws["W_w"], ws["ln_gamma"], ws["ln_beta"],
                                n_heads=H, head_dim=D, positions=pos, rope_dim=64)
    assert np.array_equal(w0, w1)
    assert np.array_equal(q0[0], q1[0]) and np.array_equal(k0[0], k1[0])       # position 0
    assert np.array_equal(q0[:, :, 64:], q1[:, :, 64:]) and np.array_equal(k0[:, 64:], k1[:, 64:])
    assert not np.allclose(q0[3:, :, :64], q1[3:, :, :64])
    # the rotated values are the rounding of the rotated unrounded projection
    raw = (xq @ ws["W_q"]).reshape(T, H, D)
    assert np.array_equal(q1, oracle.bf16_round(oracle.rope(raw, pos[:, None], 64)))
    with pytest.raises(ValueError):
        oracle.project(x, xq, ws["W_q"], ws["W_k"], ws["W_w"], ws["ln_gamma"], ws["ln_beta"], n_heads=H,
                       head_dim=D, rope_dim=64)


# ---------------------------------------------------------------- sparse MLA over the selection

def _mla_case(seed=0, T=3, H=4, n_rows=(40, 30), K=16, pad=4):
    rng = np.random.default_rng(seed)
    co = np.concatenate([[0], np.cumsum(n_rows)])
    qo = np.array([0, 2, T])                      # queries 0,1 in sequence 0; the rest in sequence 1
    kv = rng.standard_normal((int(co[-1]), oracle.MLA_DIM))
    q = rng.standard_normal((T, H, oracle.MLA_DIM)) * 0.1
    idx = np.full((T, K), -1, np.int64)
    for t in range(T):
        b = 0 if t < 2 else 1
        idx[t, : K - pad] = rng.choice(n_rows[b], K - pad, replace=False)
    return q, kv, co, qo, idx


def test_sparse_mla_matches_torch_attention():
    import torch
    q, kv, co, qo, idx = _mla_case()
    scale = 1.0 / np.sqrt(192.0)
    o, lse = oracle.sparse_mla(q, kv, co, qo, idx, scale)
    for t in range(q.shape[0]):
        b = 0 if t < 2 else 1
        rows = torch.tensor(kv[co[b] + idx[t][idx[t] >= 0]])
        qt = torch.tensor(q[t])[None]                        # [1, H, 576] as (batch, len, dim)
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, rows[None], rows[None, :, : oracle.MLA_LATENT], scale=scale)[0]
        assert np.allclose(o[t], ref.numpy(), rtol=1e-10, atol=1e-12)
        s = scale * (torch.tensor(q[t]) @ rows.T)
        assert np.allclose(lse[t], torch.logsumexp(s, dim=1).numpy(), rtol=1e-12)


def test_sparse_mla_latent_form_equals_the_per_head_192_128_form():
    # The per-head form of the 'Latent attention (MLA)' row: q/k heads of 192 = 128 no-rope
    # + 64 rope dims, v heads of 128; keys and values are up-projected from the 512-dim latent
    # c (k_nope = W_UK c, v = W_UV c) and the 64-dim rope key is shared by the heads.  Taking
    # q_nope into the latent space (W_UK^T q_nope) gives the 576-value query the oracle takes,
    # and W_UV applied to its 512-dim output gives the 128-dim head output: checked here with
    # torch's attention on the up-projected keys and values.
    import torch
    rng = np.random.default_rng(11)
    H, n = 3, 20
    c = rng.standard_normal((n, 512))
    k_rope = rng.standard_normal((n, 64))
    W_UK = rng.standard_normal((H, 128, 512)) / np.sqrt(512)
    W_UV = rng.standard_normal((H, 128, 512)) / np.sqrt(512)
    q_nope = rng.standard_normal((H, 128))
    q_rope = rng.standard_normal((H, 64))
    scale = 1.0 / np.sqrt(192.0)
    kv = np.concatenate([c, k_rope], axis=1)                          # the cached 576-value rows
    q_lat = np.concatenate([np.einsum("hdc,hd->hc", W_UK, q_nope), q_rope], axis=1)
    o_lat, lse = oracle.sparse_mla(q_lat[None], kv, np.array([0, n]), np.array([0, 1]),
                                   np.arange(n)[None], scale)
    o_head = np.einsum("hdc,hc->hd", W_UV, o_lat[0])                  # [H, 128]
    for h in range(H):
        k_h = torch.tensor(np.concatenate([c @ W_UK[h].T, k_rope], axis=1))   # [n, 192]
        v_h = torch.tensor(c @ W_UV[h].T)                                       # [n, 128]
        q_h = torch.tensor(np.concatenate([q_nope[h], q_rope[h]]))[None, None]  # [1, 1, 192]
        ref = torch.nn.functional.scaled_dot_product_attention(q_h, k_h[None], v_h[None], scale=scale)
        assert np.allclose(o_head[h], ref[0, 0].numpy(), rtol=1e-10, atol=1e-12)
        assert np.isclose(lse[0, h], torch.logsumexp(scale * (k_h @ q_h[0, 0]), 0).item(), rtol=1e-12)


def test_sparse_mla_brute_force_loops():
    q, kv, co, qo, idx = _mla_case(seed=3, T=2, H=2, n_rows=(9, 7), K=5, pad=1)
    scale = 0.7
    o, lse = oracle.sparse_mla(q, kv, co, qo, idx, scale)
    import math
    for t in range(2):
        base = 0                                   # both queries are in sequence 0
        for h in range(2):
            sc = []
            for j in idx[t]:
                if j < 0:
                    continue
                row = kv[base + j]
                sc.append((scale * sum(q[t, h, d] * row[d] for d in range(oracle.MLA_DIM)), row))
            mx = max(s for s, _ in sc)
            z = sum(math.exp(s - mx) for s, _ in sc)
            for d in (0, 100, 511):
                want = sum(math.exp(s - mx) / z * row[d] for s, row in sc)
                assert abs(o[t, h, d] - want) < 1e-12
            assert abs(lse[t, h] - (mx + math.log(z))) < 1e-12


def test_sparse_mla_special_cases():
    q, kv, co, qo, idx = _mla_case(seed=5)
    scale = 0.3
    # one selected token: the output is that token's latent, lse its score
    one = np.full_like(idx, -1)
    one[:, 0] = 7
    o, lse = oracle.sparse_mla(q, kv, co, qo, one, scale)
    for t in range(q.shape[0]):
        row = kv[co[0 if t < 2 else 1] + 7]
        assert np.allclose(o[t], np.broadcast_to(row[: oracle.MLA_LATENT], o[t].shape))
        assert np.allclose(lse[t], scale * q[t] @ row)
    # identical rows: the output is the row whatever the query; lse = score + log(count)
    kv2 = np.tile(kv[:1], (kv.shape[0], 1))
    o, lse = oracle.sparse_mla(q, kv2, co, qo, idx, scale)
    n = (idx >= 0).sum(axis=1)
    assert np.allclose(o, kv2[0, : oracle.MLA_LATENT])
    assert np.allclose(lse, scale * (q @ kv2[0]) + np.log(n)[:, None])
    # -1 entries are no token: dropping them changes nothing
    comp = np.array([np.concatenate([r[r >= 0], r[r < 0]]) for r in idx])
    o1, l1 = oracle.sparse_mla(q, kv, co, qo, idx, scale)
    o2, l2 = oracle.sparse_mla(q, kv, co, qo, comp, scale)
    assert np.allclose(o1, o2) and np.allclose(l1, l2)
    # nothing selected: zeros and -inf
    o, lse = oracle.sparse_mla(q, kv, co, qo, np.full_like(idx, -1), scale)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_sparse_mla_reads_the_query_sequence_rows():
    # a planted difference in sequence 1's rows changes only sequence 1's queries
    q, kv, co, qo, idx = _mla_case(seed=7)
    o1, _ = oracle.sparse_mla(q, kv, co, qo, idx, 0.5)
    kv2 = kv.copy()
    kv2[co[1]:] += 1.0
    o2, _ = oracle.sparse_mla(q, kv2, co, qo, idx, 0.5)
    assert np.allclose(o1[:2], o2[:2]) and not np.allclose(o1[2:], o2[2:])
