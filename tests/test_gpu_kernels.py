"""Per-kernel parity of the CUDA library against the fp64 oracle, each kernel
fed fixed inputs so that a selection difference cannot hide an attention bug
(and the reverse).  Small shapes that still span several tiles, ragged tails,
paged and contiguous caches, both block sizes and every group size the
workloads use."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import seer
from block_sparse_attention_step_b200 import workloads as W
from oracle import seer_oracle as O

from gpu_util import (TOL_MAX_ABS, TOL_REL_L2, assert_f32_close, assert_out_close, f64,
                      require_gpu, row_inputs, scale_of)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def small(name, **kw):
    return W.WORKLOADS[name].replace(**kw)


# shapes: (workload, overrides)
SHAPES = {
    "contig_bs64_g4": small("b8_h32_L8k_bs64_s90_newest", batch=2, q_heads=8, kv_heads=2, seqlen=700),
    "paged_bs64_g8": small("b64_ragged_h64_paged_bs64", batch=3, q_heads=16, kv_heads=2,
                           seqlen_range=(1, 900)),
    "contig_bs128_g5": small("b16_h40_L32k_bs128_budget4k_newest", batch=2, q_heads=10, kv_heads=2,
                             seqlen=1000),
    "paged_bs128_g16": small("b64_ragged_h64_paged_bs64", batch=2, q_heads=16, kv_heads=1,
                             block_size=128, seqlen_range=(100, 1100)),
    "contig_bs64_g1": small("b1_g4_L4k_bs64_budget512", batch=2, q_heads=2, kv_heads=2, seqlen=257),
}


def dims_for(w, data):
    return seer.make_dims(w.batch, w.q_heads, w.kv_heads, w.head_dim, w.block_size,
                          data["nb_max"], data["num_pages"])


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


# ------------------------------------------------------------------ a0 pool

@pytest.mark.parametrize("shape", list(SHAPES))
def test_pool_keys_full_and_incremental(shape):
    w = SHAPES[shape]
    data = W.generate(w, 11, DEV)
    d = dims_for(w, data)
    B, H, nbm = w.batch, w.kv_heads, data["nb_max"]
    kbar = torch.full((B, H, nbm, 128), 7.0, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_pool_keys(d, data["k_pool"], data["page_table"], data["seqlens"], 0, kbar, status)
    got = f64(kbar)
    for b in range(B):
        for h in range(H):
            _, _, K, _, L = row_inputs(w, data, b, h)
            ref = O.pool_keys(K, L, w.block_size)
            nb = ref.shape[0]
            np.testing.assert_allclose(got[b, h, :nb], ref, rtol=1e-5, atol=2e-6)
            assert (got[b, h, nb:] == 0).all()
    # incremental: only the newest block of every (b, h) is rewritten
    kbar.fill_(7.0)
    seer.seer_pool_keys(d, data["k_pool"], data["page_table"], data["seqlens"], 1, kbar, status)
    got = f64(kbar)
    for b in range(B):
        for h in range(H):
            _, _, K, _, L = row_inputs(w, data, b, h)
            ref = O.pool_keys(K, L, w.block_size)
            nb = ref.shape[0]
            if nb:
                np.testing.assert_allclose(got[b, h, nb - 1], ref[nb - 1], rtol=1e-5, atol=2e-6)
            keep = np.ones(nbm, bool)
            if nb:
                keep[nb - 1] = False
            assert (got[b, h, keep] == 7.0).all()
    assert status.item() == 0


def test_pool_keys_head_major_layout():
    """A pool laid out [P][Hkv][bs][D] through the strides gives the same kbar."""
    w = SHAPES["paged_bs64_g8"]
    data = W.generate(w, 12, DEV)
    d = dims_for(w, data)
    hm = data["k_pool"].permute(0, 2, 1, 3).contiguous()      # [P][H][bs][D]
    d2 = dims_for(w, data)
    d2.stride_page, d2.stride_token, d2.stride_head = hm.stride(0), hm.stride(2), hm.stride(1)
    a = torch.zeros((w.batch, w.kv_heads, data["nb_max"], 128), device=DEV)
    b = torch.zeros_like(a)
    seer.seer_pool_keys(d, data["k_pool"], data["page_table"], data["seqlens"], 0, a)
    seer.seer_pool_keys(d2, hm, data["page_table"], data["seqlens"], 0, b)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ a1 gate

@pytest.mark.parametrize("shape", list(SHAPES))
def test_gate_scores_given_kbar(shape):
    w = SHAPES[shape]
    data = W.generate(w, 13, DEV)
    d = dims_for(w, data)
    B, H, nbm, G = w.batch, w.kv_heads, data["nb_max"], w.group
    # kbar from the oracle (fp32), so only the gate is under test
    kbar = torch.zeros((B, H, nbm, 128), dtype=torch.float32)
    refs = {}
    for b in range(B):
        for h in range(H):
            q, Wg, K, _, L = row_inputs(w, data, b, h)
            kb = O.pool_keys(K, L, w.block_size)
            kbar[b, h, :kb.shape[0]] = torch.from_numpy(kb).float()
            refs[b, h] = (q, Wg, kbar[b, h, :kb.shape[0]].double().numpy())
    kbar = kbar.to(DEV)
    scores = torch.full((B, H, nbm), 123.0, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_gate_scores(d, data["q"], data["w_gate"], kbar, data["seqlens"], scale_of(w), scores,
                          status)
    got = f64(scores)
    for (b, h), (q, Wg, kb) in refs.items():
        ref = O.gate_scores(q, Wg, kb, scale_of(w))
        nb = ref.shape[0]
        bound = 1e-5 * max(1e-3, float(np.abs(ref).max())) if nb else 0
        assert np.abs(got[b, h, :nb] - ref).max(initial=0) <= bound, (b, h)
        assert np.isneginf(got[b, h, nb:]).all()
    assert status.item() == 0


def test_gate_closed_form_identity():
    """W = I, q = e_i in every head, kbar = e_j: score = [i == j] / sqrt(D)."""
    D, NB = 128, 130
    d = seer.make_dims(1, 3, 1, D, 64, NB, NB)
    q = torch.zeros((1, 3, D), dtype=torch.bfloat16, device=DEV)
    q[0, :, 5] = 1.0
    Wg = torch.eye(D, device=DEV)[None].contiguous()
    kbar = torch.zeros((1, 1, NB, D), device=DEV)
    for j in range(NB):
        kbar[0, 0, j, j % D] = 1.0
    seqlens = torch.tensor([NB * 64], dtype=torch.int32, device=DEV)
    scores = torch.empty((1, 1, NB), device=DEV)
    seer.seer_gate_scores(d, q, Wg, kbar, seqlens, 1 / math.sqrt(D), scores)
    expect = torch.tensor([(1 / math.sqrt(D)) if j % D == 5 else 0.0 for j in range(NB)])
    assert torch.equal(scores[0, 0].cpu(), expect.float())


# ------------------------------------------------------------------ a2 select

def _planted_scores(rng, shape):
    s = rng.standard_normal(shape).astype(np.float32)
    kind = rng.random(shape)
    s[kind < 0.25] = np.round(s[kind < 0.25] * 2) / 2          # many exact ties
    s[(kind >= 0.25) & (kind < 0.27)] = -0.0
    s[(kind >= 0.27) & (kind < 0.29)] = 0.0
    s[(kind >= 0.29) & (kind < 0.30)] = -np.inf
    return s


@pytest.mark.parametrize("nbm,bs,force", [(1, 64, False), (7, 64, True), (64, 64, False),
                                          (100, 128, True), (512, 64, False), (1000, 64, True),
                                          (4096, 64, False), (4096, 128, True)])
def test_block_select_bit_exact(nbm, bs, force):
    rng = np.random.default_rng(nbm + bs + force)
    B, H = 5, 3
    seqlens = rng.integers(0, nbm * bs + 1, B)
    seqlens[0] = nbm * bs
    seqlens[1] = min(1, nbm * bs)
    ks = rng.integers(1, nbm + 3, B)
    ks[2] = 1
    k_max = int(min(max(ks.max(), 1), nbm))
    ks = np.minimum(ks, k_max)
    s = _planted_scores(rng, (B, H, nbm))
    d = seer.make_dims(B, H, H, 128, bs, nbm, B * nbm)
    scores = torch.from_numpy(s).to(DEV)
    idx = torch.full((B, H, k_max), 77, dtype=torch.int32, device=DEV)
    n_sel = torch.full((B, H), 77, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_block_select(d, scores, torch.from_numpy(seqlens).int().to(DEV),
                           torch.from_numpy(ks).int().to(DEV), force, k_max, idx, n_sel, status)
    idx, n_sel = idx.cpu().numpy(), n_sel.cpu().numpy()
    for b in range(B):
        nb = -(-int(seqlens[b]) // bs)
        for h in range(H):
            ref = O.select_blocks(s[b, h, :nb].astype(np.float64), int(ks[b]), force)
            assert n_sel[b, h] == len(ref), (b, h)
            assert idx[b, h, :len(ref)].tolist() == ref.tolist(), (b, h)
            assert (idx[b, h, len(ref):] == -1).all()
    assert status.item() == 0


def _extreme_rows(rng, nbm):
    """Rows that crowd one score bin or break a naive value range: all equal,
    one huge outlier, denormal spread, ±3e38 with +inf, half-integer ties."""
    rows = [np.zeros(nbm, np.float32),
            rng.standard_normal(nbm).astype(np.float32),
            (rng.standard_normal(nbm) * 1e-40).astype(np.float32),
            rng.standard_normal(nbm).astype(np.float32),
            (np.round(rng.standard_normal(nbm) * 2) / 2).astype(np.float32),
            np.full(nbm, -np.inf, np.float32)]
    rows[1][nbm // 3] = 1e30
    rows[3][:3] = [-3e38, 3e38, np.inf]
    rows[5][::7] = 1.0
    return np.stack(rows)


@pytest.mark.parametrize("nbm", [300, 512, 1024, 3000])
def test_block_select_crowded_and_extreme_rows(nbm):
    rng = np.random.default_rng(nbm)
    s = _extreme_rows(rng, nbm)[:, None, :]          # [B=6][H=1][nbm]
    B = s.shape[0]
    bs = 64
    for force in (False, True):
        for k in (1, 13, nbm // 10, nbm - 1):
            d = seer.make_dims(B, 1, 1, 128, bs, nbm, B * nbm)
            idx = torch.full((B, 1, nbm), 77, dtype=torch.int32, device=DEV)
            n_sel = torch.full((B, 1), 77, dtype=torch.int32, device=DEV)
            status = torch.zeros(1, dtype=torch.int32, device=DEV)
            seqlens = torch.full((B,), nbm * bs, dtype=torch.int32, device=DEV)
            ks = torch.full((B,), k, dtype=torch.int32, device=DEV)
            seer.seer_block_select(d, torch.from_numpy(s).to(DEV), seqlens, ks, force, nbm, idx,
                                   n_sel, status)
            idx_h, n_h = idx.cpu().numpy(), n_sel.cpu().numpy()
            for b in range(B):
                ref = O.select_blocks(s[b, 0].astype(np.float64), k, force)
                assert n_h[b, 0] == len(ref), (nbm, force, k, b)
                assert idx_h[b, 0, :len(ref)].tolist() == ref.tolist(), (nbm, force, k, b)
                assert (idx_h[b, 0, len(ref):] == -1).all()
            assert status.item() == 0


def test_block_select_nan_flags_status():
    d = seer.make_dims(1, 1, 1, 128, 64, 6, 6)
    s = torch.tensor([[[1.0, float("nan"), 3.0, float("-inf"), float("nan"), 2.0]]], device=DEV)
    idx = torch.empty((1, 1, 5), dtype=torch.int32, device=DEV)
    n_sel = torch.empty((1, 1), dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_block_select(d, s, torch.tensor([384], dtype=torch.int32, device=DEV),
                           torch.tensor([5], dtype=torch.int32, device=DEV), False, 5, idx, n_sel,
                           status)
    assert idx.cpu().tolist() == [[[0, 1, 2, 3, 5]]]
    assert status.item() & seer.DEV_NONFINITE_SCORE


# ------------------------------------------------------------------ a3 + a4

def _random_selection(w, data, rng, k_frac=0.3):
    """Index rows chosen by the oracle from random scores (exact, no ties)."""
    B, H, nbm = w.batch, w.kv_heads, data["nb_max"]
    L = data["seqlens"].cpu().numpy()
    k_max = max(1, int(math.ceil(k_frac * nbm)))
    idx = np.full((B, H, k_max), -1, np.int32)
    n_sel = np.zeros((B, H), np.int32)
    for b in range(B):
        nb = -(-int(L[b]) // w.block_size)
        for h in range(H):
            sel = O.select_blocks(rng.standard_normal(nb), min(k_max, max(1, int(k_frac * nb) + 1)),
                                  bool(rng.integers(0, 2)))
            idx[b, h, :len(sel)] = sel
            n_sel[b, h] = len(sel)
    return idx, n_sel, k_max


def _run_decode(w, data, idx, n_sel, k_max, S, q=None, k_pool=None, v_pool=None, dims=None):
    d = dims or dims_for(w, data)
    B, Hq = w.batch, w.q_heads
    o_part = torch.full((B, Hq, S, 128), 5.0, device=DEV)
    lse_part = torch.full((B, Hq, S), 5.0, device=DEV)
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx_t = torch.from_numpy(idx).to(DEV)
    nsel_t = torch.from_numpy(n_sel).to(DEV)
    seer.seer_sparse_decode(d, data["q"] if q is None else q,
                            data["k_pool"] if k_pool is None else k_pool,
                            data["v_pool"] if v_pool is None else v_pool, data["page_table"],
                            data["seqlens"], idx_t, nsel_t, k_max, S, scale_of(w), o_part, lse_part,
                            status)
    seer.seer_combine(d, o_part, lse_part, S, out, lse)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out, lse, o_part, lse_part


@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("S", [1, 3, 8])
def test_sparse_decode_and_combine_given_indices(shape, S):
    w = SHAPES[shape]
    data = W.generate(w, 21 + S, DEV)
    rng = np.random.default_rng(S)
    idx, n_sel, k_max = _random_selection(w, data, rng)
    out, lse, o_part, lse_part = _run_decode(w, data, idx, n_sel, k_max, S)
    out, lse, o_part, lse_part = f64(out), f64(lse), f64(o_part), f64(lse_part)
    G = w.group
    worst, worst_plain, worst_f32 = 0.0, 0.0, 0.0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            q, _, K, V, L = row_inputs(w, data, b, h)
            sel = idx[b, h, :n_sel[b, h]]
            ref, ref_lse = O.masked_attention(q, K, V, L, sel, w.block_size, scale_of(w))
            rows = slice(h * G, (h + 1) * G)
            e = assert_out_close(out[b, rows], ref, (b, h))
            worst, worst_plain = max(worst, e[0]), max(worst_plain, e[2])
            fin = np.isfinite(ref_lse)
            np.testing.assert_allclose(lse[b, rows][fin], ref_lse[fin], atol=1e-3)
            assert np.isneginf(lse[b, rows][~fin]).all()
            po, pl = O.split_partials(q, K, V, L, sel, w.block_size, scale_of(w), S)
            for s in range(S):
                if np.isneginf(pl[s]).all():
                    assert np.isneginf(lse_part[b, rows, s]).all()
                    assert (o_part[b, rows, s] == 0).all()
                else:
                    piece = sel[(s * len(sel)) // S:((s + 1) * len(sel)) // S]
                    toks = np.concatenate([np.arange(j * w.block_size,
                                                     min((j + 1) * w.block_size, L))
                                           for j in piece])
                    v_scale = float(np.abs(V[toks]).max()) if toks.size else 1.0
                    e = assert_f32_close(o_part[b, rows, s], po[s], v_scale, (b, h, s))
                    worst_f32 = max(worst_f32, e[0] / max(1.0, v_scale))
                    np.testing.assert_allclose(lse_part[b, rows, s], pl[s], atol=1e-3)
    print(f"{shape} S={S}: out worst max-abs beyond bf16 rounding {worst:.2e} "
          f"(plain {worst_plain:.2e}); o_part worst max-abs / max(1, |V|) {worst_f32:.2e}")


def test_decode_unselected_and_tail_slots_never_matter():
    """NaN / huge values outside the selected blocks and past seqlen leave the
    output bitwise unchanged (they are never read into the math)."""
    w = SHAPES["paged_bs64_g8"]
    data = W.generate(w, 31, DEV)
    rng = np.random.default_rng(3)
    idx, n_sel, k_max = _random_selection(w, data, rng)
    base = _run_decode(w, data, idx, n_sel, k_max, 3)
    kp, vp = data["k_pool"].clone(), data["v_pool"].clone()
    L = data["seqlens"].cpu().numpy()
    table = data["page_table"].cpu().numpy()
    for b in range(w.batch):
        nb = -(-int(L[b]) // 64)
        for j in range(nb):
            pg = table[b, j]
            for h in range(w.kv_heads):
                if j not in set(idx[b, h, :n_sel[b, h]].tolist()):
                    kp[pg, :, h] = float("nan")
                    vp[pg, :, h] = float("inf")
        tail = int(L[b]) - (nb - 1) * 64
        if 0 < tail < 64:
            kp[table[b, nb - 1], tail:] = float("nan")
            vp[table[b, nb - 1], tail:] = float("nan")
    again = _run_decode(w, data, idx, n_sel, k_max, 3, k_pool=kp, v_pool=vp)
    assert torch.equal(base[0], again[0])
    assert torch.equal(base[1], again[1])


def test_decode_deterministic_split_invariant_and_index_order():
    w = SHAPES["contig_bs128_g5"]
    data = W.generate(w, 41, DEV)
    rng = np.random.default_rng(4)
    idx, n_sel, k_max = _random_selection(w, data, rng, k_frac=0.6)
    a = _run_decode(w, data, idx, n_sel, k_max, 4)
    b = _run_decode(w, data, idx, n_sel, k_max, 4)
    assert torch.equal(a[0], b[0]) and torch.equal(a[2], b[2])
    one = _run_decode(w, data, idx, n_sel, k_max, 1)
    eight = _run_decode(w, data, idx, n_sel, k_max, 8)
    np.testing.assert_allclose(f64(one[1]), f64(eight[1]), atol=1e-5)
    np.testing.assert_allclose(f64(one[0]), f64(eight[0]), rtol=2 ** -7, atol=1e-3)
    rev = idx.copy()
    for bb in range(w.batch):
        for h in range(w.kv_heads):
            n = n_sel[bb, h]
            rev[bb, h, :n] = idx[bb, h, :n][::-1]
    r = _run_decode(w, data, rev, n_sel, k_max, 1)
    np.testing.assert_allclose(f64(r[1]), f64(one[1]), atol=1e-5)
    np.testing.assert_allclose(f64(r[0]), f64(one[0]), rtol=2 ** -7, atol=1e-3)


def test_decode_closed_forms():
    """q = 0 gives the mean of the selected V rows; constant V gives the constant."""
    w = SHAPES["contig_bs64_g4"]
    data = W.generate(w, 51, DEV)
    rng = np.random.default_rng(5)
    idx, n_sel, k_max = _random_selection(w, data, rng)
    zq = torch.zeros_like(data["q"])
    out = f64(_run_decode(w, data, idx, n_sel, k_max, 2, q=zq)[0])
    for b in range(w.batch):
        for h in range(w.kv_heads):
            _, _, _, V, L = row_inputs(w, data, b, h)
            rows = np.concatenate([np.arange(j * 64, min(j * 64 + 64, L)) for j in idx[b, h, :n_sel[b, h]]])
            mean = V[rows].mean(axis=0)
            for g in range(w.group):
                np.testing.assert_allclose(out[b, h * w.group + g], mean, atol=4e-3, rtol=2 ** -7)
    cv = torch.full_like(data["v_pool"], 0.375)
    out = f64(_run_decode(w, data, idx, n_sel, k_max, 2, v_pool=cv)[0])
    np.testing.assert_allclose(out, 0.375, rtol=4e-3)


def test_decode_head_major_layout_matches():
    w = SHAPES["paged_bs128_g16"]
    data = W.generate(w, 61, DEV)
    rng = np.random.default_rng(6)
    idx, n_sel, k_max = _random_selection(w, data, rng)
    base = _run_decode(w, data, idx, n_sel, k_max, 2)
    kh = data["k_pool"].permute(0, 2, 1, 3).contiguous()
    vh = data["v_pool"].permute(0, 2, 1, 3).contiguous()
    d2 = dims_for(w, data)
    d2.stride_page, d2.stride_token, d2.stride_head = kh.stride(0), kh.stride(2), kh.stride(1)
    other = _run_decode(w, data, idx, n_sel, k_max, 2, k_pool=kh, v_pool=vh, dims=d2)
    assert torch.equal(base[0], other[0])


def test_combine_hand_case():
    """The hand-worked combine fixture through the kernel."""
    d = seer.make_dims(1, 1, 1, 128, 64, 1, 1)
    o = torch.zeros((1, 1, 3, 128), device=DEV)
    o[0, 0, 0, 0] = 1.0
    o[0, 0, 1, 1] = 1.0
    lse = torch.tensor([[[0.0, math.log(3.0), float("-inf")]]], device=DEV)
    out = torch.empty((1, 1, 128), dtype=torch.bfloat16, device=DEV)
    lo = torch.empty((1, 1), device=DEV)
    seer.seer_combine(d, o, lse, 3, out, lo)
    assert out[0, 0, 0].item() == 0.25 and out[0, 0, 1].item() == 0.75
    assert abs(lo.item() - math.log(4.0)) < 1e-6
