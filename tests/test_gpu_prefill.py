"""Prefill with query pooling against the fp64 oracle: pooled keys, the
block-to-block gate scores of the pooled queries, the diagonal-forced
selection of every query block (bit-exact where the fp64 margin is clear,
valid otherwise) and the causal block-sparse attention of every query token
over the GPU's own selection; paged and contiguous caches, bs 64 and 128,
ragged lengths, sparsity and budget rules, and the dense case (every block
chosen) as plain causal attention."""
import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import workloads as W
from block_sparse_attention_step_b200.runner import PrefillBuffers
from oracle import seer_oracle as O

from gpu_util import MARGIN, assert_out_close, f64, require_gpu, scale_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


CASES = {
    "paged_bs64_s80": (W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(
        batch=2, q_heads=8, kv_heads=2, seqlen_range=(300, 1100)), 800, 0),
    "contig_bs64_dense": (W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(
        batch=2, q_heads=8, kv_heads=2, seqlen=450), 0, 0),
    "contig_bs128_budget": (W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(
        batch=1, q_heads=10, kv_heads=2, seqlen=1500, budget_tokens=512), 0, 512),
    "paged_bs64_s95_g8": (W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(
        batch=1, q_heads=16, kv_heads=2, seqlen_range=(2000, 2600)), 950, 0),
}


def _k_of(permille, budget, bs):
    if budget > 0:
        return lambda i: O.k_from_budget(i + 1, budget, bs)
    return lambda i: O.k_from_sparsity(i + 1, permille)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_oracle(name):
    w, permille, budget = CASES[name]
    data = W.generate(w, 61, DEV)
    q = W.prefill_queries(w, 61, data["nb_max"], DEV)
    run = PrefillBuffers(w, data, q, sparsity_permille=permille, budget_tokens=budget,
                         keep_scores=True)
    run.run(pool_keys=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    idx, n_sel = (t.cpu().numpy() for t in run.selection())
    kbar, scores = f64(run.kbar), f64(run.scores)
    out, lse = f64(run.out), f64(run.lse)
    G, bs = w.group, w.block_size
    k_of = _k_of(permille, budget, bs)
    exact = near = 0
    for b in range(w.batch):
        L = int(data["seqlens"][b])
        nb = O.num_blocks(L, bs)
        for h in range(w.kv_heads):
            Qg = f64(q[b, :L, h * G:(h + 1) * G])
            K = f64(W.gather_rows(data["k_pool"], data["page_table"], b, h, L, bs))
            V = f64(W.gather_rows(data["v_pool"], data["page_table"], b, h, L, bs))
            ref_kbar = O.pool_keys(K, L, bs)
            np.testing.assert_allclose(kbar[b, h, :nb], ref_kbar, rtol=1e-5, atol=2e-6)
            ref_sc = O.prefill_gate_scores(Qg, f64(data["w_gate"][h]), ref_kbar, L, bs, scale_of(w))
            got_sel = []
            for i in range(nb):
                row = ref_sc[i, : i + 1]
                bound = 1e-5 * max(1e-3, float(np.abs(row).max()))
                assert np.abs(scores[b, h, i, : i + 1] - row).max() <= bound + 2e-6, (b, h, i)
                assert np.isneginf(scores[b, h, i, i + 1:]).all()
                k = k_of(i)
                got = idx[b, h, i, : n_sel[b, h, i]]
                assert (idx[b, h, i, n_sel[b, h, i]:] == -1).all()
                if O.selection_margin(row, k, True) > MARGIN:
                    assert got.tolist() == O.select_blocks(row, k, True).tolist(), (b, h, i)
                    exact += 1
                else:
                    assert O.selection_is_valid(row, got, k, True, MARGIN), (b, h, i)
                    near += 1
                got_sel.append(got)
            ref_out, ref_lse = O.prefill_attention(Qg, K, V, L, got_sel, bs, scale_of(w))
            for g in range(G):
                assert_out_close(out[b, :L, h * G + g], ref_out[:, g], (b, h, g))
                np.testing.assert_allclose(lse[b, h * G + g, :L], ref_lse[:, g], atol=1e-3)
    assert exact > 0


def test_prefill_dense_is_causal_attention():
    """Sparsity 0: every block is chosen, so each output row is plain causal
    attention (checked against torch's fp64 SDPA, not the oracle)."""
    w = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=1, q_heads=4, kv_heads=1,
                                                           seqlen=333)
    data = W.generate(w, 63, DEV)
    q = W.prefill_queries(w, 63, data["nb_max"], DEV)
    run = PrefillBuffers(w, data, q, sparsity_permille=0, budget_tokens=0)
    run.run(pool_keys=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0   # also: no wait ran out (every tile streams several stages)
    L = 333
    Q = q[0, :L].double().permute(1, 0, 2)[None]                  # [1][4][L][D]
    K = W.gather_rows(data["k_pool"], data["page_table"], 0, 0, L, 64).double()
    V = W.gather_rows(data["v_pool"], data["page_table"], 0, 0, L, 64).double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cpu(), K.cpu()[None, None].expand(1, 4, L, 128), V.cpu()[None, None].expand(1, 4, L, 128),
        is_causal=True, scale=scale_of(w))[0].permute(1, 0, 2).numpy()
    assert_out_close(f64(run.out[0, :L]), ref, "dense")


@pytest.mark.parametrize("q_heads", [4, 3])
def test_prefill_growing_scores_rescale_the_accumulator(q_heads):
    """Keys whose scale grows block by block push every row's running maximum
    up past the kernel's rescale threshold (a factor of 2^8) several times,
    so the output accumulated in tensor memory is rescaled on the way; the
    result must still be plain causal attention (torch's fp64 SDPA).  Three
    query heads leave the last head pair with one real head."""
    w = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=1, q_heads=q_heads, kv_heads=1,
                                                           seqlen=700)
    data = W.generate(w, 67, DEV)
    q = W.prefill_queries(w, 67, data["nb_max"], DEV)
    kp = data["k_pool"]                                   # contiguous: page j = block j
    grow = 1.0 + 0.75 * torch.arange(kp.shape[0], device=DEV, dtype=torch.float32)
    data["k_pool"] = (kp.float() * grow[:, None, None, None]).to(torch.bfloat16)
    run = PrefillBuffers(w, data, q, sparsity_permille=0, budget_tokens=0)
    run.run(pool_keys=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    L, G = 700, q_heads
    Q = q[0, :L].double().permute(1, 0, 2)[None]
    K = W.gather_rows(data["k_pool"], data["page_table"], 0, 0, L, 64).double()
    V = W.gather_rows(data["v_pool"], data["page_table"], 0, 0, L, 64).double()
    x = torch.einsum("gtd,sd->gts", Q[0].cpu(), K.cpu()) * scale_of(w) * 1.4426950408889634
    causal = torch.tril(torch.ones(L, L, dtype=torch.bool))
    run_max = x.masked_fill(~causal, float("-inf")).amax(-1)      # each row's final maximum
    first = x[:, :, :64].masked_fill(~causal[:, :64], float("-inf")).amax(-1)
    grown = (run_max - first)[:, 320:]                            # rows from block 5 on
    assert float((grown > 8.0).double().mean()) > 0.5             # most of them rescale
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.cpu(), K.cpu()[None, None].expand(1, G, L, 128), V.cpu()[None, None].expand(1, G, L, 128),
        is_causal=True, scale=scale_of(w))[0].permute(1, 0, 2).numpy()
    assert_out_close(f64(run.out[0, :L]), ref, "rescaled")
    lse_ref = torch.logsumexp(x.masked_fill(~causal, float("-inf")) / 1.4426950408889634, -1)
    np.testing.assert_allclose(f64(run.lse[0, :, :L]), lse_ref.numpy(), atol=1e-3, rtol=1e-5)


def test_prefill_tail_garbage_never_matters():
    """NaN in the cache slots past each sequence's end changes nothing."""
    w, permille, budget = CASES["paged_bs64_s80"]
    data = W.generate(w, 65, DEV)
    q = W.prefill_queries(w, 65, data["nb_max"], DEV)
    a = PrefillBuffers(w, data, q, sparsity_permille=permille)
    a.run()
    torch.cuda.synchronize()
    out_a = a.out.clone()
    table = data["page_table"]
    for b in range(w.batch):
        L = int(data["seqlens"][b])
        if L % w.block_size:
            page = int(table[b, L // w.block_size])
            data["k_pool"][page, L % w.block_size:] = float("nan")
            data["v_pool"][page, L % w.block_size:] = float("nan")
    b_run = PrefillBuffers(w, data, q, sparsity_permille=permille)
    b_run.kbar.copy_(a.kbar)
    b_run.run(pool_keys=False)
    torch.cuda.synchronize()
    assert a.status.item() == 0 and b_run.status.item() == 0
    assert torch.equal(out_a, b_run.out)


@pytest.mark.parametrize("name", ["paged_bs64_s80", "contig_bs128_budget"])
def test_prefill_attention_alone_gives_the_same_bits(name):
    """seer_prefill_attention over the selection seer_prefill left in its
    workspace writes exactly seer_prefill's output and lse."""
    w, permille, budget = CASES[name]
    data = W.generate(w, 69, DEV)
    q = W.prefill_queries(w, 69, data["nb_max"], DEV)
    run = PrefillBuffers(w, data, q, sparsity_permille=permille, budget_tokens=budget)
    run.run(pool_keys=True)
    out2 = torch.zeros_like(run.out)
    lse2 = torch.full_like(run.lse, 7.0)
    run.attention(out=out2, lse=lse2)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    for b in range(w.batch):
        L = int(data["seqlens"][b])
        assert torch.equal(out2[b, :L], run.out[b, :L])
        assert torch.equal(lse2[b, :, :L], run.lse[b, :, :L])


def test_prefill_full_size_sampled():
    """The prefill at the size and seeds the benchmark times (batch 2, 16K-token
    prompt, 40/8 heads, bs 64, 90 %): every pooled key, and for sampled query
    blocks (first, second, middle, last and seeded picks) the gate row, the
    selection and the output and lse of sampled query tokens against the
    oracle computed one by one."""
    w = W.WORKLOADS[W.HEADLINE].replace(batch=2, seqlen=16384)
    seed = 1
    data = W.generate(w, seed, DEV)
    q = W.prefill_queries(w, seed, data["nb_max"], DEV)
    run = PrefillBuffers(w, data, q, keep_scores=True)
    run.run(pool_keys=True)
    torch.cuda.synchronize()
    assert run.status.item() == 0
    idx, n_sel = (t.cpu().numpy() for t in run.selection())
    kbar, scores = f64(run.kbar), f64(run.scores)
    G, bs, scale = w.group, w.block_size, scale_of(w)
    rng = np.random.default_rng(7)
    exact = 0
    for b in range(w.batch):
        L = int(data["seqlens"][b])
        nb = O.num_blocks(L, bs)
        for h in range(w.kv_heads):
            K = f64(W.gather_rows(data["k_pool"], data["page_table"], b, h, L, bs))
            ref_kbar = O.pool_keys(K, L, bs)
            np.testing.assert_allclose(kbar[b, h, :nb], ref_kbar, rtol=1e-5, atol=2e-6)
            V = f64(W.gather_rows(data["v_pool"], data["page_table"], b, h, L, bs))
            Qg = f64(q[b, :L, h * G:(h + 1) * G])
            blocks = sorted({0, 1, nb // 2, nb - 1, *rng.integers(0, nb, 2).tolist()})
            for i in blocks:
                row = O.prefill_gate_row(Qg, f64(data["w_gate"][h]), ref_kbar, L, bs, scale, i)
                bound = 1e-5 * max(1e-3, float(np.abs(row).max()))
                assert np.abs(scores[b, h, i, : i + 1] - row).max() <= bound + 2e-6, (b, h, i)
                k = O.k_from_sparsity(i + 1, w.sparsity_permille)
                got = idx[b, h, i, : n_sel[b, h, i]]
                if O.selection_margin(row, k, True) > MARGIN:
                    assert got.tolist() == O.select_blocks(row, k, True).tolist(), (b, h, i)
                    exact += 1
                else:
                    assert O.selection_is_valid(row, got, k, True, MARGIN), (b, h, i)
                lo, hi = i * bs, min((i + 1) * bs, L)
                for t in sorted({lo, hi - 1, int(rng.integers(lo, hi))}):
                    ref_o, ref_l = O.prefill_attention_token(Qg, K, V, L, t, got, bs, scale)
                    assert_out_close(f64(run.out[b, t, h * G:(h + 1) * G]), ref_o, (b, h, t))
                    np.testing.assert_allclose(f64(run.lse[b, h * G:(h + 1) * G, t]), ref_l,
                                               atol=1e-3)
    assert exact > 0
