"""The single-launch step (seer_decode_step_fused) against the per-stage step:
the same bits everywhere (kbar, scores, indices, output, lse) on every
workload shape, the control words back at rest after each launch, the KV
append (the cache rows it writes, and the step over the appended cache against
the oracle), and the calls it refuses."""
import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import seer
from block_sparse_attention_step_b200 import workloads as W
from block_sparse_attention_step_b200.runner import StepBuffers

from gpu_util import require_gpu
from test_gpu_step import check_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


CASES = {
    "headline_small": W.WORKLOADS["b16_h40_L32k_bs64_s90"].replace(batch=4, seqlen=9000),
    "newest_offsets": W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=3, seqlen=2100),
    "bs128_budget": W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(batch=3,
                                                                              seqlen=12000),
    "ragged_paged": W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=6,
                                                                     seqlen_range=(1, 40000)),
    "many_rows": W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(
        batch=40, q_heads=16, kv_heads=8, seqlen_range=(64, 9000), sparsity_permille=800),
    "g16": W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(
        batch=2, q_heads=32, kv_heads=2, seqlen=5000, budget_tokens=1024),
    "single_row": W.WORKLOADS["b1_g4_L4k_bs64_budget512"],
}


def _snapshot(run):
    v = run.workspace_views()
    return {"kbar": run.kbar.clone(), "scores": v["scores"].clone(), "idx": v["idx"].clone(),
            "n_sel": v["n_sel"].clone(), "out": run.out.clone(), "lse": run.lse.clone()}


def _assert_same(a, b):
    for key in a:
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("update_kbar", [1, 2, 0])
@pytest.mark.parametrize("name", list(CASES))
def test_fused_step_equals_per_stage_step(name, update_kbar):
    w = CASES[name]
    data = W.generate(w, 51, DEV)
    run = StepBuffers(w, data)
    run.pool_full()
    kbar0 = run.kbar.clone()
    run.step(update_kbar=update_kbar)
    torch.cuda.synchronize()
    ref = _snapshot(run)
    # the per-stage step advances the epoch too when its gate grid publishes rows
    e0 = run.workspace_views()["ctl"].tolist()[2]
    for rep in range(3):  # successive launches on one workspace
        run.kbar.copy_(kbar0)
        run.out.zero_()
        run.lse.zero_()
        run.step(update_kbar=update_kbar, fused=True)
        torch.cuda.synchronize()
        assert run.status.item() == 0
        _assert_same(ref, _snapshot(run))
        v = run.workspace_views()
        ctl = v["ctl"].tolist()
        assert ctl[:2] == [0, 0] and ctl[3:7] == [0, 0, 0, 0]   # counters at rest
        assert ctl[2] == e0 + rep + 1                           # one epoch per launch
        assert (v["row_flag"] == e0 + rep + 1).all()


def _append_inputs(w, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (w.batch, w.kv_heads, w.head_dim)
    k_new = torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV)
    v_new = torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV)
    return k_new, v_new


def _expected_pools(w, data, k_new, v_new):
    """The pools with the new token's rows written at L - 1 (host-side copy)."""
    kp, vp = data["k_pool"].clone(), data["v_pool"].clone()
    table = data["page_table"]
    L = data["seqlens"].tolist()
    for b in range(w.batch):
        if L[b] == 0:
            continue
        t = L[b] - 1
        page = int(table[b, t // w.block_size]) if w.paged else b * data["nb_max"] + t // w.block_size
        kp[page, t % w.block_size] = k_new[b]
        vp[page, t % w.block_size] = v_new[b]
    return kp, vp


@pytest.mark.parametrize("name", ["newest_offsets", "ragged_paged", "bs128_budget"])
def test_kv_append_both_paths(name):
    w = CASES[name]
    data = W.generate(w, 53, DEV)
    k_new, v_new = _append_inputs(w, 7)
    kp_want, vp_want = _expected_pools(w, data, k_new, v_new)
    k0, v0 = data["k_pool"].clone(), data["v_pool"].clone()
    run = StepBuffers(w, data)
    run.pool_full()
    kbar0 = run.kbar.clone()
    results = []
    for fused in (False, True):
        data["k_pool"].copy_(k0)
        data["v_pool"].copy_(v0)
        run.kbar.copy_(kbar0)
        run.step(args=run.args(update_kbar=1, k_new=k_new, v_new=v_new), fused=fused)
        torch.cuda.synchronize()
        assert run.status.item() == 0
        assert torch.equal(data["k_pool"], kp_want) and torch.equal(data["v_pool"], vp_want)
        results.append(_snapshot(run))
    _assert_same(results[0], results[1])
    # the step over the appended cache (incremental pooled key included) vs the oracle
    report = {"exact": 0, "near_tie": 0}
    check_rows(w, data, run, [(b, h) for b in range(w.batch) for h in range(w.kv_heads)], report)


def test_fused_step_refuses_unified_and_mass_and_bad_append():
    w = CASES["newest_offsets"]
    data = W.generate(w, 55, DEV)
    run = StepBuffers(w, data, unified=True)
    with pytest.raises(seer.SeerError) as e:
        run.step(update_kbar=2, fused=True)
    assert e.value.status == 2
    run2 = StepBuffers(w, data, mass=True)
    with pytest.raises(seer.SeerError) as e:
        run2.step(update_kbar=2, fused=True)
    assert e.value.status == 2
    k_new, _ = _append_inputs(w, 3)
    with pytest.raises(seer.SeerError) as e:
        run.step(args=run.args(update_kbar=1, k_new=k_new, v_new=None), fused=False)
    assert e.value.status == 1


def test_fused_step_edge_cases():
    """seqlen 0 and 1, a partial newest block, more splits than blocks."""
    w = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=4, q_heads=8, kv_heads=2,
                                                           seqlen=200)
    data = W.generate(w, 5, DEV)
    data["seqlens"] = torch.tensor([0, 1, 65, 200], dtype=torch.int32, device=DEV)
    run = StepBuffers(w, data, num_splits=16)
    run.pool_full()
    kbar0 = run.kbar.clone()
    run.step(update_kbar=1)
    torch.cuda.synchronize()
    ref = _snapshot(run)
    run.kbar.copy_(kbar0)
    run.step(update_kbar=1, fused=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    _assert_same(ref, _snapshot(run))


@pytest.mark.parametrize("name", ["b16_h40_L32k_bs64_s90", "b16_h40_L32k_bs128_budget4k_newest"])
def test_fused_step_full_size_equals_per_stage_step(name):
    """At full size with the benchmark's seed and incremental pooled-key
    update, the single launch gives the per-stage step's bits (the per-stage
    step is checked against the oracle at full size on sampled rows)."""
    w = W.WORKLOADS[name]
    data = W.generate(w, 1, DEV)
    run = StepBuffers(w, data)
    run.pool_full()
    kbar0 = run.kbar.clone()
    run.step(update_kbar=1)
    torch.cuda.synchronize()
    ref = _snapshot(run)
    run.kbar.copy_(kbar0)
    run.out.zero_()
    run.lse.zero_()
    run.step(update_kbar=1, fused=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    _assert_same(ref, _snapshot(run))
