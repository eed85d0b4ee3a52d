"""Pins of the fp64 oracle to things other than itself: hand-worked fixtures
(tests/golden/), closed forms, invariants, brute force on tiny inputs and a
library routine (torch's fp64 scaled_dot_product_attention on the CPU).
CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f(x):
    return float(x) if not isinstance(x, str) else float(x.replace("inf", "inf"))


# ---------------------------------------------------------------- fixtures

def test_attention_hand_cases():
    for case in _load("attention_hand.json")["cases"]:
        out, lse = O.masked_attention(np.array(case["q"], float), np.array(case["K"], float),
                                      np.array(case["V"], float), case["seqlen"], case["blocks"],
                                      case["block_size"], case["scale"])
        np.testing.assert_allclose(out, np.array(case["out"], float), rtol=0, atol=1e-14,
                                   err_msg=case["name"])
        np.testing.assert_allclose(lse, np.array(case["lse"], float), rtol=0, atol=1e-14,
                                   err_msg=case["name"])


def test_gate_hand_case():
    d = _load("gate_hand.json")
    s = O.gate_scores(np.array(d["q"], float), np.array(d["W"], float),
                      np.array(d["kbar"], float), d["scale"])
    np.testing.assert_allclose(s, d["scores"], rtol=0, atol=1e-14)


def test_pool_hand_case():
    d = _load("pool_hand.json")
    kbar = O.pool_keys(np.array(d["K"], float), d["seqlen"], d["block_size"])
    np.testing.assert_array_equal(kbar, np.array(d["kbar"], float))


def test_combine_hand_case():
    d = _load("combine_hand.json")
    lse = np.array([[_f(v) for v in row] for row in d["lse"]])
    out, lse_out = O.combine(np.array(d["o"], float), lse)
    np.testing.assert_allclose(out, d["out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse_out, d["lse_out"], rtol=0, atol=1e-15)


def test_k_rules():
    d = _load("k_rules.json")
    for c in d["sparsity"]:
        assert O.k_from_sparsity(c["nb"], c["permille"]) == c["k"], c
    for c in d["budget"]:
        assert O.k_from_budget(c["nb"], c["budget"], c["block_size"]) == c["k"], c


def test_select_hand_cases():
    for c in _load("select_hand.json")["cases"]:
        scores = [_f(v) for v in c["scores"]]
        got = O.select_blocks(scores, c["k"], c["force_newest"]).tolist()
        assert got == c["indices"], c


# ---------------------------------------------------------------- selection

def _beats(s, i, j):
    """Block i outranks block j: higher score, or equal score and lower index;
    NaN below everything, -0.0 == +0.0."""
    a, b = s[i], s[j]
    if math.isnan(a):
        return math.isnan(b) and i < j
    if math.isnan(b):
        return True
    return a > b or (a == b and i < j)


def _brute_select(s, k, force):
    """Exhaustive: the unique k-subset (holding the forced block) in which
    every block chosen on merit outranks every block left out."""
    nb = len(s)
    k = min(k, nb)
    found = []
    for subset in itertools.combinations(range(nb), k):
        if force and k > 0 and nb - 1 not in subset:
            continue
        merit = [i for i in subset if not (force and i == nb - 1)]
        out = [j for j in range(nb) if j not in subset]
        if all(_beats(s, i, j) for i in merit for j in out):
            found.append(list(subset))
    assert len(found) == 1, (s, k, force, found)
    return found[0]


def test_select_matches_brute_force_with_ties_and_specials():
    rng = np.random.default_rng(7)
    specials = [0.0, -0.0, -math.inf, math.inf, math.nan]
    for trial in range(400):
        nb = int(rng.integers(1, 9))
        s = [float(v) for v in rng.integers(-2, 3, nb)]
        for pos in range(nb):
            if rng.random() < 0.2:
                s[pos] = specials[int(rng.integers(0, len(specials)))]
        k = int(rng.integers(1, nb + 2))
        force = bool(rng.integers(0, 2))
        got = O.select_blocks(s, k, force).tolist()
        assert got == _brute_select(s, k, force), (s, k, force)
        assert O.selection_is_valid(s, got, k, force, 0.0)


def test_selection_margin_and_validity():
    s = [0.5, 0.9, 0.1, 0.7]
    assert O.selection_margin(s, 2, False) == pytest.approx(0.2)
    assert O.selection_margin(s, 4, False) == math.inf
    # forced newest (0.7) leaves 1 merit slot: 0.9 vs next 0.5
    assert O.selection_margin(s, 2, True) == pytest.approx(0.4)
    assert O.selection_is_valid(s, [1, 3], 2, False, 0.0)
    assert not O.selection_is_valid(s, [0, 1], 2, False, 0.0)
    assert O.selection_is_valid(s, [0, 1], 2, False, 0.25)
    assert not O.selection_is_valid(s, [3, 1], 2, False, 0.0)   # not ascending
    assert not O.selection_is_valid(s, [0, 1], 2, True, 1.0)    # forced block missing


# ---------------------------------------------------------------- pooling and gate

def test_pool_closed_forms():
    rng = np.random.default_rng(1)
    c = rng.standard_normal(16)
    K = np.tile(c, (200, 1))
    kbar = O.pool_keys(K, 200, 64)
    assert kbar.shape == (4, 16)
    np.testing.assert_allclose(kbar, np.tile(c, (4, 1)), rtol=1e-15, atol=1e-15)
    # linear in K; every row of a block moved by the same vector moves the mean by it
    K2 = rng.standard_normal((130, 16))
    shift = rng.standard_normal(16)
    a = O.pool_keys(K2, 130, 64)
    b = O.pool_keys(K2 + shift, 130, 64)
    np.testing.assert_allclose(b - a, np.tile(shift, (3, 1)), atol=1e-12)
    # a single valid token in the newest block is its own mean
    np.testing.assert_array_equal(a[2], K2[128:130].mean(axis=0))


def test_gate_closed_forms():
    D = 8
    scale = 1 / math.sqrt(D)
    eye = np.eye(D)
    for i in range(D):
        for j in range(D):
            s = O.gate_scores(eye[i][None, :], eye, eye[j][None, :], scale)
            assert s[0] == (scale if i == j else 0.0)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, D))
    W = rng.standard_normal((D, D))
    kb = rng.standard_normal((9, D))
    base = O.gate_scores(q, W, kb, scale)
    np.testing.assert_allclose(O.gate_scores(2 * q, W, kb, scale), 2 * base, rtol=1e-13)
    # the group score of G identical heads equals the single-head score
    np.testing.assert_allclose(O.gate_scores(np.tile(q[:1], (4, 1)), W, kb, scale),
                               O.gate_scores(q[:1], W, kb, scale), rtol=1e-13)
    # permuting blocks permutes scores
    perm = rng.permutation(9)
    np.testing.assert_allclose(O.gate_scores(q, W, kb[perm], scale), base[perm], rtol=1e-13)


# ---------------------------------------------------------------- attention

def _sdpa_dense(q, K, V, scale):
    """torch's fp64 CPU scaled_dot_product_attention: a library routine."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1),
        torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1), scale=scale)
    return out[0, :, 0, :].numpy()


@pytest.mark.parametrize("L,bs", [(200, 64), (256, 64), (300, 128), (1, 64), (65, 64)])
def test_all_blocks_selected_equals_library_dense_attention(L, bs):
    rng = np.random.default_rng(L)
    G, D = 5, 32
    q, K, V = rng.standard_normal((G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    nb = O.num_blocks(L, bs)
    out, lse = O.masked_attention(q, K, V, L, range(nb), bs, 1 / math.sqrt(D))
    np.testing.assert_allclose(out, _sdpa_dense(q, K, V, 1 / math.sqrt(D)), rtol=1e-12, atol=1e-13)
    x = q @ K.T / math.sqrt(D)
    from scipy.special import logsumexp
    np.testing.assert_allclose(lse, logsumexp(x, axis=1), rtol=1e-13)


def test_sparse_equals_library_attention_on_the_selected_rows():
    rng = np.random.default_rng(11)
    G, D, L, bs = 4, 16, 500, 64
    q, K, V = rng.standard_normal((G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    blocks = [1, 4, 7]
    rows = np.concatenate([np.arange(j * bs, min((j + 1) * bs, L)) for j in blocks])
    out, _ = O.masked_attention(q, K, V, L, blocks, bs, 0.25)
    np.testing.assert_allclose(out, _sdpa_dense(q, K[rows], V[rows], 0.25), rtol=1e-12, atol=1e-13)


def test_attention_closed_forms_and_invariants():
    rng = np.random.default_rng(5)
    G, D, L, bs = 3, 16, 1000, 64
    q, K, V = rng.standard_normal((G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    blocks = [0, 3, 15]      # block 15 is partial: rows 960..999
    # one selected token: output is that V row exactly
    out, lse = O.masked_attention(q, K, V, 961, [15], bs, 0.3)
    np.testing.assert_array_equal(out, np.tile(V[960], (G, 1)))
    np.testing.assert_allclose(lse, q @ K[960] * 0.3, rtol=1e-15)
    # q = 0: the plain mean of the selected rows
    out, _ = O.masked_attention(np.zeros((G, D)), K, V, L, blocks, bs, 0.3)
    rows = np.r_[0:64, 192:256, 960:1000]
    np.testing.assert_allclose(out, np.tile(V[rows].mean(axis=0), (G, 1)), rtol=1e-12, atol=1e-14)
    # constant V rows: output is that constant (weights sum to 1)
    c = rng.standard_normal(D)
    out, _ = O.masked_attention(q, K, np.tile(c, (L, 1)), L, blocks, bs, 0.3)
    np.testing.assert_allclose(out, np.tile(c, (G, 1)), rtol=1e-12)
    # one-hot V (V_t = e_{t mod D}): each output row is a probability vector
    onehot = np.eye(D)[np.arange(L) % D]
    out, _ = O.masked_attention(q, K, onehot, L, blocks, bs, 0.3)
    np.testing.assert_allclose(out.sum(axis=1), 1.0, rtol=1e-13)
    assert (out >= 0).all()
    # unselected blocks and tail slots never matter, not even as NaN
    base, base_lse = O.masked_attention(q, K, V, L - 7, blocks, bs, 0.3)
    K2, V2 = K.copy(), V.copy()
    for j in set(range(16)) - set(blocks):
        K2[j * bs:(j + 1) * bs] = np.nan
        V2[j * bs:(j + 1) * bs] = 1e30
    K2[L - 7:] = np.nan
    V2[L - 7:] = np.nan
    out2, lse2 = O.masked_attention(q, K2, V2, L - 7, blocks, bs, 0.3)
    np.testing.assert_array_equal(out2, base)
    np.testing.assert_array_equal(lse2, base_lse)
    # the order of the index list does not matter
    out3, _ = O.masked_attention(q, K, V, L - 7, blocks[::-1], bs, 0.3)
    np.testing.assert_array_equal(out3, base)


@pytest.mark.parametrize("S", [1, 2, 3, 8, 13])
def test_split_then_combine_equals_unsplit(S):
    rng = np.random.default_rng(S)
    G, D, L, bs = 4, 16, 777, 64
    q, K, V = rng.standard_normal((G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    blocks = [0, 2, 5, 6, 9, 12]
    o, l = O.split_partials(q, K, V, L, blocks, bs, 0.25, S)
    assert o.shape == (S, G, D) and l.shape == (S, G)
    if S > len(blocks):
        assert np.isneginf(l).any()
    out, lse = O.combine(o, l)
    ref, ref_lse = O.masked_attention(q, K, V, L, blocks, bs, 0.25)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)
    # the pieces are contiguous runs of the ascending list that cover it once
    n = len(blocks)
    pieces = [blocks[(s * n) // S:((s + 1) * n) // S] for s in range(S)]
    assert sum(pieces, []) == blocks


def test_decode_row_picks_planted_blocks():
    """Compose pool -> gate -> select -> attention on a case built so that the
    answer is known: blocks 2 and 5 carry keys along the gate direction."""
    rng = np.random.default_rng(9)
    G, D, bs, L = 2, 16, 8, 60
    W = np.eye(D)
    q = np.zeros((G, D)); q[:, 3] = 1.0
    K = 0.01 * rng.standard_normal((L, D))
    K[2 * bs:3 * bs, 3] += 2.0
    K[5 * bs:6 * bs, 3] += 1.0
    V = rng.standard_normal((L, D))
    r = O.decode_row(q, W, K, V, L, bs, 2, False, 1 / math.sqrt(D), 1 / math.sqrt(D))
    assert r["indices"].tolist() == [2, 5]
    r = O.decode_row(q, W, K, V, L, bs, 2, True, 1 / math.sqrt(D), 1 / math.sqrt(D))
    assert r["indices"].tolist() == [2, 7]     # newest block 7 (rows 56..59) forced
    ref, _ = O.masked_attention(q, K, V, L, [2, 7], bs, 1 / math.sqrt(D))
    np.testing.assert_array_equal(r["out"], ref)


def test_bf16_conversion_is_exact():
    x = torch.randn(1000).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), x.double().numpy())



# ---------------------------------------------------------------- block mass

def test_block_mass_hand_cases():
    for case in _load("attention_hand.json")["cases"]:
        if "block_mass" not in case:
            continue
        got = O.block_mass(np.array(case["q"], float), np.array(case["K"], float), case["seqlen"],
                           case["blocks"], case["block_size"], case["scale"])
        np.testing.assert_allclose(got, np.array(case["block_mass"], float), atol=1e-14,
                                   err_msg=case["name"])


def test_block_mass_dense_equals_library_softmax_block_sums():
    from scipy.special import softmax
    rng = np.random.default_rng(12)
    G, D, L, bs = 3, 16, 300, 64
    q, K = rng.standard_normal((G, D)), rng.standard_normal((L, D))
    nb = O.num_blocks(L, bs)
    got = O.block_mass(q, K, L, range(nb), bs, 0.25)
    p = softmax(q @ K.T * 0.25, axis=1)
    want = np.stack([p[:, j * bs:min((j + 1) * bs, L)].sum(axis=1) for j in range(nb)], axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=1e-13)


def test_block_mass_sparse_properties():
    rng = np.random.default_rng(13)
    G, D, L, bs = 4, 16, 500, 64
    q, K = rng.standard_normal((G, D)), rng.standard_normal((L, D))
    sel = [0, 3, 7]
    got = O.block_mass(q, K, L, sel, bs, 0.3)
    assert got.shape == (G, 8)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=1e-13)
    assert (got[:, [1, 2, 4, 5, 6]] == 0).all()
    # masses weight the selected blocks' values: out = sum_j mass_j * (p-weighted block mean)
    V = np.ones((L, D))
    out, _ = O.masked_attention(q, K, V, L, sel, bs, 0.3)
    np.testing.assert_allclose(out[:, 0], got.sum(axis=1), rtol=1e-13)
    # a V whose column j is the indicator of block j turns the attention output into the masses
    Vb = np.zeros((L, D))
    Vb[np.arange(L), np.arange(L) // bs] = 1.0
    outb, _ = O.masked_attention(q, K, Vb, L, sel, bs, 0.3)
    np.testing.assert_allclose(outb[:, :8], got, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- unified cross-head selection

def test_unified_select_hand_cases():
    for c in _load("select_unified_hand.json")["cases"]:
        ph = np.array([[_f(v) for v in row] for row in c["per_head"]])
        agg = O.unified_scores(ph)
        want = np.array([_f(v) for v in c["aggregate"]])
        assert np.array_equal(agg, want, equal_nan=True), c
        assert O.select_blocks_unified(ph, c["k"], c["force_newest"]).tolist() == c["indices"], c
        per_head = [O.select_blocks(r, c["k"], c["force_newest"]).tolist() for r in ph]
        assert per_head == c["per_head_indices"], c


def test_unified_select_brute_force_and_reductions():
    rng = np.random.default_rng(17)
    for trial in range(300):
        H = int(rng.integers(1, 4))
        nb = int(rng.integers(1, 8))
        ph = rng.integers(-2, 3, (H, nb)).astype(float)
        k = int(rng.integers(1, nb + 2))
        force = bool(rng.integers(0, 2))
        # aggregate written out column by column, then the exhaustive search
        col = [sum(float(ph[h, j]) for h in range(H)) for j in range(nb)]
        got = O.select_blocks_unified(ph, k, force).tolist()
        assert got == _brute_select(col, k, force), (ph, k, force)
        # head order does not matter; one head is the per-head selection;
        # identical heads select what each head alone selects
        assert O.select_blocks_unified(ph[::-1], k, force).tolist() == got
        assert O.select_blocks_unified(ph[:1], k, force).tolist() == \
            O.select_blocks(ph[0], k, force).tolist()
        same = np.repeat(ph[:1], 3, axis=0)
        assert O.select_blocks_unified(same, k, force).tolist() == \
            O.select_blocks(ph[0], k, force).tolist()


def test_unified_f32_aggregate_is_the_in_order_fp32_sum():
    rng = np.random.default_rng(19)
    ph = rng.standard_normal((5, 300)).astype(np.float32)
    got = O.unified_scores_f32(ph)
    want = ph[0].copy()
    for h in range(1, 5):
        want = np.float32(want + ph[h])
    assert got.dtype == np.float32 and np.array_equal(got, want)
    # within fp32 rounding of the fp64 sum
    np.testing.assert_allclose(got, O.unified_scores(ph), rtol=0, atol=4e-6)


# ---------------------------------------------------------------- prefill with query pooling

def test_prefill_dense_equals_library_causal_attention():
    """Every block selected: the prefill path is causal attention, checked
    against torch's fp64 scaled_dot_product_attention(is_causal=True)."""
    import torch
    rng = np.random.default_rng(21)
    L, G, D, bs = 150, 3, 16, 32
    Q, K, V = rng.standard_normal((L, G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    nb = O.num_blocks(L, bs)
    sel = [np.arange(i + 1) for i in range(nb)]
    out, lse = O.prefill_attention(Q, K, V, L, sel, bs, 0.25)
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]            # [1][G][L][D]
    k = torch.from_numpy(K)[None, None].expand(1, G, L, D)
    v = torch.from_numpy(V)[None, None].expand(1, G, L, D)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.25)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
    x = np.einsum("tgd,sd->gts", Q, K) * 0.25
    x[:, np.triu(np.ones((L, L), bool), 1)] = -np.inf
    from scipy.special import logsumexp
    np.testing.assert_allclose(lse, logsumexp(x, axis=2).T, rtol=1e-12)


def test_prefill_sparse_equals_library_masked_attention():
    import torch
    rng = np.random.default_rng(22)
    L, G, D, bs = 200, 2, 8, 32
    Q, K, V = rng.standard_normal((L, G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    nb = O.num_blocks(L, bs)
    sel = [np.array(sorted(set(rng.choice(i + 1, size=min(i + 1, 2), replace=False).tolist()) | {i}))
           for i in range(nb)]
    out, _ = O.prefill_attention(Q, K, V, L, sel, bs, 0.3)
    allowed = np.zeros((L, L), bool)
    for i, blocks in enumerate(sel):
        rows = slice(i * bs, min((i + 1) * bs, L))
        for j in blocks:
            allowed[rows, j * bs:min((j + 1) * bs, L)] = True
    allowed &= ~np.triu(np.ones((L, L), bool), 1)
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K)[None, None].expand(1, G, L, D)
    v = torch.from_numpy(V)[None, None].expand(1, G, L, D)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(allowed),
                                                           scale=0.3)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_prefill_closed_forms_and_hand_case():
    rng = np.random.default_rng(23)
    L, G, D, bs = 70, 2, 4, 32
    Q, K, V = rng.standard_normal((L, G, D)), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    # token 0 sees only itself; the first token of any block with only its own
    # block selected sees only itself too
    out, lse = O.prefill_attention(Q, K, V, L, [np.array([0]), np.array([1]), np.array([2])], bs, 1.0)
    np.testing.assert_allclose(out[0], np.stack([V[0]] * G), rtol=0, atol=0)
    np.testing.assert_allclose(out[32], np.stack([V[32]] * G), rtol=0, atol=0)
    np.testing.assert_allclose(lse[0], Q[0] @ K[0], rtol=1e-14)
    # pooled queries: the mean over the block's tokens and the group's heads
    qbar = O.pool_queries(Q, L, bs)
    np.testing.assert_allclose(qbar[2], Q[64:70].reshape(-1, D).mean(axis=0), rtol=1e-14)
    # gate by hand: W = I, kbar = e_j: score(i, j) = qbar_i[j] * scale, -inf above the diagonal
    kb = np.eye(3, D)
    sc = O.prefill_gate_scores(Q, np.eye(D), kb, L, bs, 0.5)
    np.testing.assert_allclose(sc[2, :3], qbar[2, :3] * 0.5, rtol=1e-13)
    assert np.isneginf(sc[0, 1]) and np.isneginf(sc[1, 2])
    # selection: the diagonal block is always in and counts toward k
    s = np.array([[0, -np.inf, -np.inf], [5, 1, -np.inf], [5, 9, -3]], float)
    got = O.prefill_select(s, lambda i: 1)
    assert [g.tolist() for g in got] == [[0], [1], [2]]
    got = O.prefill_select(s, lambda i: 2)
    assert [g.tolist() for g in got] == [[0], [0, 1], [1, 2]]

    # the one-row and one-token forms the full-size tests sample
    np.testing.assert_allclose(O.prefill_gate_row(Q, np.eye(D), kb, L, bs, 0.5, 2),
                               qbar[2, :3] * 0.5, rtol=1e-13)
    o, l = O.prefill_attention_token(Q, K, V, L, 40, [1], bs, 0.7)
    x = Q[40] @ K[32:41].T * 0.7                                # keys 32..40 of block 1
    from scipy.special import logsumexp, softmax
    np.testing.assert_allclose(o, softmax(x, axis=1) @ V[32:41], rtol=1e-12)
    np.testing.assert_allclose(l, logsumexp(x, axis=1), rtol=1e-13)


def test_prefill_gate_hand_case():
    """The pooled-query gate on a hand-worked case with a partial last block:
    pooled queries, pooled keys, the causal score matrix and the per-block
    selection with the diagonal block forced (tests/golden/prefill_gate_hand.json,
    derivation in the file)."""
    c = _load("prefill_gate_hand.json")
    Q, K, Wm = (np.array(c[n], float) for n in ("Q", "K", "W"))
    L, bs = c["seqlen"], c["block_size"]
    np.testing.assert_array_equal(O.pool_queries(Q, L, bs), np.array(c["qbar"], float))
    kbar = O.pool_keys(K, L, bs)
    np.testing.assert_array_equal(kbar, np.array(c["kbar"], float))
    want = np.array([[_f(x) for x in row] for row in c["scores"]])
    got = O.prefill_gate_scores(Q, Wm, kbar, L, bs, c["scale"])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    for i in range(want.shape[0]):
        np.testing.assert_allclose(O.prefill_gate_row(Q, Wm, kbar, L, bs, c["scale"], i),
                                   want[i, :i + 1], rtol=0, atol=1e-15)
    ks = [O.k_from_sparsity(i + 1, c["sparsity_permille"]) for i in range(want.shape[0])]
    assert ks == c["k"]
    sel = O.prefill_select(got, lambda i: ks[i])
    assert [s.tolist() for s in sel] == c["selected"]
    # the whole prefill row reaches the same selection
    row = O.prefill_row(Q, Wm, K, K, L, bs, lambda i: ks[i], c["scale"], 1.0)
    assert [s.tolist() for s in row["selected"]] == c["selected"]
