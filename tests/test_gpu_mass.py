"""Per-block attention mass (the dense-mode target of the self-distilled gate)
against the fp64 oracle: dense mode (every block selected) and sparse
selections, both block sizes, paged and contiguous caches, G up to 16; the
decode partials of the mass variant equal the plain decode's bit for bit."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import seer
from block_sparse_attention_step_b200 import workloads as W
from block_sparse_attention_step_b200.runner import StepBuffers
from oracle import seer_oracle as O

from gpu_util import f64, require_gpu, row_inputs, scale_of

pytestmark = pytest.mark.gpu
DEV = "cuda"
MASS_ATOL = 2e-5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_mass(w, data, run, rows):
    v = run.workspace_views()
    idx = v["idx"].cpu().numpy()
    n_sel = v["n_sel"].cpu().numpy()
    mass = f64(run.block_mass)
    G = w.group
    for (b, h) in rows:
        q, _, K, _, L = row_inputs(w, data, b, h)
        sel = idx[b, h, :n_sel[b, h]]
        ref = O.block_mass(q, K, L, sel, w.block_size, scale_of(w))
        nb = ref.shape[1]
        got = mass[b, h * G:(h + 1) * G]
        np.testing.assert_allclose(got[:, :nb], ref, atol=MASS_ATOL, err_msg=str((b, h)))
        assert (got[:, nb:] == 0).all()
        if len(sel):
            np.testing.assert_allclose(got.sum(axis=1), 1.0, atol=1e-4)


CASES = {
    "dense_paged_bs64_g8": (W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(
        batch=3, seqlen_range=(1, 2000), sparsity_permille=0), None),
    "sparse_paged_bs64_g8": (W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(
        batch=3, seqlen_range=(64, 3000), sparsity_permille=900), None),
    "dense_contig_bs128_g5": (W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(
        batch=2, seqlen=1500, budget_tokens=None, sparsity_permille=0, force_newest=False), None),
    "sparse_contig_bs128_g16": (W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(
        batch=2, q_heads=32, kv_heads=2, seqlen=3000, budget_tokens=1024), 3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_step_block_mass_matches_oracle(name):
    w, splits = CASES[name]
    data = W.generate(w, 41, DEV)
    run = StepBuffers(w, data, num_splits=splits, mass=True)
    run.step(update_kbar=2)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    _check_mass(w, data, run, [(b, h) for b in range(w.batch) for h in range(w.kv_heads)])


def test_mass_decode_partials_equal_plain_decode():
    w = W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=3, seqlen_range=(64, 3000))
    data = W.generate(w, 43, DEV)
    run = StepBuffers(w, data, mass=True)
    run.step(update_kbar=2)
    v = run.workspace_views()
    d = data
    o1, l1 = v["o_part"].clone(), v["lse_part"].clone()
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    seer.seer_sparse_decode(run.dims, d["q"], d["k_pool"], d["v_pool"], run.page_table,
                            d["seqlens"], v["idx"], v["n_sel"], run.k_max, run.num_splits,
                            run.scale, o2, l2)
    bl = torch.full_like(run.block_lse, float("nan"))
    o3, l3 = torch.empty_like(o1), torch.empty_like(l1)
    seer.seer_sparse_decode_mass(run.dims, d["q"], d["k_pool"], d["v_pool"], run.page_table,
                                 d["seqlens"], v["idx"], v["n_sel"], run.k_max, run.num_splits,
                                 run.scale, o3, l3, bl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
    mass2 = torch.empty_like(run.block_mass)
    seer.seer_block_mass(run.dims, v["idx"], v["n_sel"], run.k_max, d["seqlens"], bl, run.lse,
                         mass2)
    torch.cuda.synchronize()
    assert torch.equal(mass2, run.block_mass)


def test_decode_item_counter_gives_the_same_bits_and_resets():
    """Items handed out through the shared counter (as in the step) or round-
    robin give bit-identical partials; the counter is zero after every launch."""
    w = W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=5, seqlen_range=(64, 5000))
    data = W.generate(w, 47, DEV)
    run = StepBuffers(w, data, num_splits=5)
    run.step(update_kbar=2)
    v = run.workspace_views()
    d = data
    ctr = torch.zeros(2, dtype=torch.int32, device=DEV)
    outs = []
    for counter in (None, ctr, ctr):
        o, l = torch.empty_like(v["o_part"]), torch.empty_like(v["lse_part"])
        seer.seer_sparse_decode(run.dims, d["q"], d["k_pool"], d["v_pool"], run.page_table,
                                d["seqlens"], v["idx"], v["n_sel"], run.k_max, run.num_splits,
                                run.scale, o, l, run.status, work_counter=counter)
        torch.cuda.synchronize()
        assert ctr.tolist() == [0, 0]
        outs.append((o, l))
    assert run.status.item() == 0
    for o, l in outs:
        assert torch.equal(o, v["o_part"]) and torch.equal(l, v["lse_part"])


def test_gate_recall_matches_oracle():
    """Gate recall (the dense block masses kept by the sparse selection) from
    the GPU's dense-mass step and sparse step against the oracle's dense
    block masses summed over the GPU's own selection."""
    from block_sparse_attention_step_b200.runner import gate_recall
    w = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=2, seqlen=2500)
    data = W.generate(w, 43, DEV)
    dense = StepBuffers(w, data, sparsity_permille=0, budget_tokens=0, mass=True)
    dense.step(update_kbar=2)
    sparse = StepBuffers(w, data)
    sparse.step(update_kbar=2)
    torch.cuda.synchronize()
    assert dense.status.item() == 0 and sparse.status.item() == 0
    v = sparse.workspace_views()
    rec = gate_recall(dense.block_mass, v["idx"], v["n_sel"], w.group).cpu().numpy()
    idx, n_sel = v["idx"].cpu().numpy(), v["n_sel"].cpu().numpy()
    G = w.group
    for b in range(w.batch):
        for h in range(w.kv_heads):
            q, _, K, _, L = row_inputs(w, data, b, h)
            allb = np.arange(O.num_blocks(L, w.block_size))
            ref = O.block_mass(q, K, L, allb, w.block_size, scale_of(w))     # [G][nb]
            chosen = idx[b, h, :n_sel[b, h]]
            np.testing.assert_allclose(rec[b, h * G:(h + 1) * G], ref[:, chosen].sum(axis=1),
                                       atol=1e-4, err_msg=str((b, h)))
    assert (rec <= 1 + 1e-4).all() and (rec > 0).all()
    # the dense selection keeps everything
    dv = dense.workspace_views()
    full = gate_recall(dense.block_mass, dv["idx"], dv["n_sel"], G)
    assert torch.allclose(full, torch.ones_like(full), atol=1e-4)
