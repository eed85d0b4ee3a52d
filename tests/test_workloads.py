"""The seeded input generator: shapes, determinism and the paged layout (CPU)."""
import torch

from block_sparse_attention_step_b200 import workloads as W


def _small(name, **kw):
    base = W.WORKLOADS[name]
    return base.replace(**kw)


def test_generate_is_deterministic_and_shaped():
    w = _small("b8_h32_L8k_bs64_s90_newest", batch=2, seqlen=300)
    a = W.generate(w, 5)
    b = W.generate(w, 5)
    c = W.generate(w, 6)
    for key in ("q", "w_gate", "k_pool", "v_pool", "page_table", "seqlens"):
        assert torch.equal(a[key], b[key]), key
    assert not torch.equal(a["k_pool"], c["k_pool"])
    assert a["q"].shape == (2, 32, 128) and a["q"].dtype == torch.bfloat16
    assert a["w_gate"].shape == (8, 128, 128) and a["w_gate"].dtype == torch.float32
    assert a["k_pool"].shape == (2 * 5, 64, 8, 128)
    assert a["nb_max"] == 5
    assert a["page_table"].tolist() == [[0, 1, 2, 3, 4], [5, 6, 7, 8, 9]]


def test_paged_ragged_table_is_a_permutation():
    w = _small("b64_ragged_h64_paged_bs64", batch=6, seqlen_range=(70, 700))
    d = W.generate(w, 1)
    L = d["seqlens"].tolist()
    assert all(70 <= x <= 700 for x in L)
    nb = [-(-x // 64) for x in L]
    t = d["page_table"]
    used = []
    for b in range(6):
        used += t[b, :nb[b]].tolist()
        assert (t[b, nb[b]:] == -1).all()
    assert sorted(used) == list(range(d["num_pages"]))
    # gather_rows walks the table: row t of sequence b is slot t % bs of its page
    b, h = 3, 5
    rows = W.gather_rows(d["k_pool"], t, b, h, L[b], 64)
    assert rows.shape == (L[b], 128)
    page = t[b, 1].item()
    assert torch.equal(rows[64 + 7], d["k_pool"][page, 7, h])


def test_offsets_shift_each_page_by_one_vector():
    w = _small("b8_h32_L8k_bs64_s90_newest", batch=1, seqlen=640, offset_var=400.0)
    d = W.generate(w, 2)
    k = d["k_pool"].float()
    # with a huge offset variance the rows of a page share their mean direction
    m = k.mean(dim=1)                       # [P][H][D]
    spread = (k - m[:, None]).std()
    assert m.abs().mean() > 5 * spread
    t = _small("b16_h40_L32k_bs128_budget4k_newest", batch=1, seqlen=1024)
    d = W.generate(t, 2)
    assert torch.isfinite(d["k_pool"].float()).all()


def test_head_major_layout_holds_the_same_values():
    w = _small("b64_ragged_h64_paged_bs64", batch=3, seqlen_range=(10, 300))
    a = W.generate(w, 4, layout="nhd")
    b = W.generate(w, 4, layout="hnd")
    assert b["k_pool"].shape == (a["num_pages"], 8, 64, 128)
    assert W.pool_strides(b) == (8 * 64 * 128, 128, 64 * 128)
    assert W.pool_strides(a) == (64 * 8 * 128, 8 * 128, 128)
    for bb in range(3):
        L = int(a["seqlens"][bb])
        for h in (0, 7):
            x = W.gather_rows(a["v_pool"], a["page_table"], bb, h, L, 64, "nhd")
            y = W.gather_rows(b["v_pool"], b["page_table"], bb, h, L, 64, "hnd")
            assert torch.equal(x, y)


def test_gate_recall_hand_case():
    """Recall = mass of the chosen blocks, per query head, padding ignored;
    choosing every block keeps all of a normalised row."""
    from block_sparse_attention_step_b200.runner import gate_recall
    m = torch.tensor([[[0.1, 0.2, 0.3, 0.4], [0.25, 0.25, 0.25, 0.25],
                       [0.7, 0.1, 0.1, 0.1], [0.0, 0.0, 0.5, 0.5]]])      # B 1, Hq 4, NB 4
    idx = torch.tensor([[[3, 1, -1, -1], [0, 1, 2, 3]]], dtype=torch.int32)  # Hkv 2, G 2
    n_sel = torch.tensor([[2, 4]], dtype=torch.int32)
    got = gate_recall(m, idx, n_sel, 2)
    assert torch.allclose(got, torch.tensor([[0.6, 0.5, 1.0, 1.0]]))
