"""Unified cross-head selection (one block set per sequence shared by all its
KV heads) against the oracle: the standalone select bit for bit on given fp32
scores (both sides rank the in-order fp32 aggregate), and the whole step with
the unified flag (indices under the margin rule, outputs on the GPU's own
index set)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import seer
from block_sparse_attention_step_b200 import workloads as W
from block_sparse_attention_step_b200.runner import StepBuffers
from oracle import seer_oracle as O

from gpu_util import MARGIN, assert_out_close, f64, require_gpu, row_inputs, scale_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _planted(rng, shape):
    s = rng.standard_normal(shape).astype(np.float32)
    kind = rng.random(shape)
    s[kind < 0.3] = np.round(s[kind < 0.3] * 2) / 2          # ties after the head sum
    s[(kind >= 0.3) & (kind < 0.32)] = -0.0
    s[(kind >= 0.32) & (kind < 0.33)] = -np.inf
    return s


@pytest.mark.parametrize("nbm,Hkv,force", [(1, 1, False), (9, 3, True), (130, 8, False),
                                           (700, 2, True), (1500, 4, False), (4096, 8, True)])
def test_unified_select_bit_exact(nbm, Hkv, force):
    rng = np.random.default_rng(nbm * 10 + Hkv)
    B, bs = 4, 64
    seqlens = rng.integers(0, nbm * bs + 1, B)
    seqlens[0] = nbm * bs
    ks = rng.integers(1, nbm + 3, B)
    k_max = int(min(max(ks.max(), 1), nbm))
    ks = np.minimum(ks, k_max)
    s = _planted(rng, (B, Hkv, nbm))
    d = seer.make_dims(B, Hkv, Hkv, 128, bs, nbm, B * nbm)
    idx = torch.full((B, Hkv, k_max), 77, dtype=torch.int32, device=DEV)
    n_sel = torch.full((B, Hkv), 77, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_block_select_unified(d, torch.from_numpy(s).to(DEV),
                                   torch.from_numpy(seqlens).int().to(DEV),
                                   torch.from_numpy(ks).int().to(DEV), force, k_max, idx, n_sel,
                                   status)
    idx, n_sel = idx.cpu().numpy(), n_sel.cpu().numpy()
    for b in range(B):
        nb = -(-int(seqlens[b]) // bs)
        agg = O.unified_scores_f32(s[b, :, :nb])
        ref = O.select_blocks(agg.astype(np.float64), int(ks[b]), force)
        for h in range(Hkv):
            assert n_sel[b, h] == len(ref), (b, h)
            assert idx[b, h, :len(ref)].tolist() == ref.tolist(), (b, h)
            assert (idx[b, h, len(ref):] == -1).all()
    assert status.item() == 0


def test_unified_select_nan_flags_status():
    d = seer.make_dims(1, 2, 2, 128, 64, 5, 5)
    s = torch.tensor([[[1.0, float("nan"), 3.0, 0.0, 2.0],
                       [1.0, 5.0, float("-inf"), 0.0, 2.0]]], device=DEV)
    idx = torch.empty((1, 2, 5), dtype=torch.int32, device=DEV)
    n_sel = torch.empty((1, 2), dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seer.seer_block_select_unified(d, s, torch.tensor([320], dtype=torch.int32, device=DEV),
                                   torch.tensor([4], dtype=torch.int32, device=DEV), False, 5,
                                   idx, n_sel, status)
    # aggregate [2, nan, -inf, 0, 4] -> top 4: 4, 0, 3, then -inf (2) over NaN (1)
    assert idx.cpu().tolist() == [[[0, 2, 3, 4, -1], [0, 2, 3, 4, -1]]]
    assert status.item() & seer.DEV_NONFINITE_SCORE


def _check_unified_rows(w, data, run, report):
    views = run.workspace_views()
    idx = views["idx"].cpu().numpy()
    n_sel = views["n_sel"].cpu().numpy()
    out, lse = f64(run.out), f64(run.lse)
    k_per_seq = run.k_per_seq.cpu().numpy()
    G = w.group
    for b in range(w.batch):
        per_head, rows = [], []
        for h in range(w.kv_heads):
            q, Wg, K, V, L = row_inputs(w, data, b, h)
            kbar = O.pool_keys(K, L, w.block_size)
            per_head.append(O.gate_scores(q, Wg, kbar, scale_of(w)))
            rows.append((q, K, V, L))
        agg = O.unified_scores(np.stack(per_head)) if per_head[0].size else np.zeros(0)
        k = int(k_per_seq[b])
        got = idx[b, 0, :n_sel[b, 0]]
        for h in range(w.kv_heads):       # one row for every head
            assert n_sel[b, h] == n_sel[b, 0]
            assert np.array_equal(idx[b, h], idx[b, 0])
        margin = O.selection_margin(agg, k, run.force_newest)
        # the aggregate adds Hkv fp32 scores: scale the gate margin with it
        if margin > MARGIN * w.kv_heads:
            assert got.tolist() == O.select_blocks(agg, k, run.force_newest).tolist(), (b, margin)
            report["exact"] += 1
        else:
            assert O.selection_is_valid(agg, got, k, run.force_newest, MARGIN * w.kv_heads), b
            report["near_tie"] += 1
        for h, (q, K, V, L) in enumerate(rows):
            o, l = O.masked_attention(q, K, V, L, got, w.block_size, scale_of(w))
            sl = slice(h * G, (h + 1) * G)
            assert_out_close(out[b, sl], o, (b, h))
            fin = np.isfinite(l)
            np.testing.assert_allclose(lse[b, sl][fin], l[fin], atol=1e-3)


CASES = {
    "contig_bs64_s90": W.WORKLOADS["b16_h40_L32k_bs64_s90"].replace(batch=3, seqlen=5000),
    "newest_bs64_offsets": W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=3,
                                                                             seqlen=3000),
    "budget_bs128_t": W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(batch=2,
                                                                                seqlen=9000),
    "ragged_paged": W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=4,
                                                                     seqlen_range=(1, 70000)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_step_unified_matches_oracle(name):
    w = CASES[name]
    data = W.generate(w, 31, DEV)
    run = StepBuffers(w, data, unified=True)
    run.step(update_kbar=2)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    report = {"exact": 0, "near_tie": 0}
    _check_unified_rows(w, data, run, report)
    assert report["exact"] >= 1


def test_step_unified_equals_standalone_gate_then_unified_select():
    w = W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=24, q_heads=16, kv_heads=8,
                                                         seqlen_range=(100, 30000))
    data = W.generate(w, 37, DEV)
    run = StepBuffers(w, data, unified=True)
    run.pool_full()
    run.step(update_kbar=1)
    torch.cuda.synchronize()
    v = run.workspace_views()
    scores = torch.empty_like(v["scores"])
    idx = torch.full_like(v["idx"], 77)
    n_sel = torch.full_like(v["n_sel"], 77)
    seer.seer_gate_scores(run.dims, data["q"], data["w_gate"], run.kbar, data["seqlens"],
                          run.scale, scores, run.status)
    seer.seer_block_select_unified(run.dims, scores, data["seqlens"], run.k_per_seq,
                                   run.force_newest, run.k_max, idx, n_sel, run.status)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    assert torch.equal(scores, v["scores"])
    assert torch.equal(idx, v["idx"]) and torch.equal(n_sel, v["n_sel"])
