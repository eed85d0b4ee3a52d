"""seer_decode_step_noalloc against seer_decode_step, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device
memory (a host runtime that owns all GPU memory through its own pool, or a
decode loop that must never enter the CUDA allocator): it runs the same step
with the library's fixed 16 MiB device array as workspace.  Both paths run the
same deterministic kernels on the same inputs, so two calls in a row must
each give exactly the caller-workspace step's bits (a scratch carve at a wrong
offset would show), and a size beyond the array must be refused.  This file is
collected last on purpose, so a failure here comes after every other test has
run; it also passes alone in a fresh process.
"""
import pytest
import torch

from block_sparse_attention_step_b200 import seer
from block_sparse_attention_step_b200 import workloads as W
from block_sparse_attention_step_b200.runner import StepBuffers

from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def test_noalloc_step_matches_workspace_step_twice():
    require_gpu()
    w = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"].replace(batch=4, seqlen=3000)
    data = W.generate(w, 17, "cuda")
    run = StepBuffers(w, data)
    run.pool_full()
    run.step(update_kbar=0)
    torch.cuda.synchronize()
    ref_out, ref_lse = run.out.clone(), run.lse.clone()
    v = run.workspace_views()
    ref_idx, ref_nsel = v["idx"].clone(), v["n_sel"].clone()
    assert run.status.item() == 0

    need = seer.seer_step_workspace_bytes(run.dims, run.k_max, run.num_splits)
    assert 0 < need <= seer.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        run.out.fill_(0)
        run.lse.fill_(0)
        seer.seer_decode_step_noalloc(run.dims, run.args(update_kbar=0))
        torch.cuda.synchronize()
        assert torch.equal(run.out, ref_out), ("call", call)
        assert torch.equal(run.lse, ref_lse), ("call", call)
        assert run.status.item() == 0
    # the caller's workspace was not touched by the no-allocation calls
    assert torch.equal(v["idx"], ref_idx) and torch.equal(v["n_sel"], ref_nsel)

    # a request larger than the fixed array is refused before any work
    big = seer.make_dims(64, 64, 8, 128, 64, 4096, 64 * 4096)
    args = run.args(update_kbar=0)
    args.k_max = 4096
    args.num_splits = 64
    assert seer.seer_step_workspace_bytes(big, 4096, 64) > seer.NOALLOC_SCRATCH_BYTES
    with pytest.raises(seer.SeerError) as e:
        seer.seer_decode_step_noalloc(big, args)
    assert e.value.status == 4          # SEER_ERR_WORKSPACE


def test_noalloc_steps_of_different_shapes_in_turn():
    """Differently shaped steps through the one fixed array, in turn.  The control words
    and row flags sit at an offset that depends on the shape, so each call lands on what
    the call before it left in the array (partials, indices, or its own flags at another
    offset); every call must still give the caller-workspace step's bits."""
    require_gpu()
    base = W.WORKLOADS["b8_h32_L8k_bs64_s90_newest"]
    shapes = [
        base.replace(batch=20, seqlen=2000),   # 160 rows: the row-claiming gate, row flags on
        base.replace(batch=3, seqlen=5000),    # 24 rows: one gate CTA per row
        W.WORKLOADS["b16_h40_L32k_bs128_budget4k_newest"].replace(batch=2, seqlen=4000),
    ]
    runs = []
    for i, w in enumerate(shapes):
        run = StepBuffers(w, W.generate(w, 30 + i, "cuda"))
        run.pool_full()
        run.step(update_kbar=0)
        torch.cuda.synchronize()
        assert run.status.item() == 0, i
        assert seer.seer_step_workspace_bytes(run.dims, run.k_max, run.num_splits) \
            <= seer.NOALLOC_SCRATCH_BYTES
        runs.append((run, run.out.clone(), run.lse.clone()))
    for rep in range(2):
        for i, (run, ref_out, ref_lse) in enumerate(runs):
            run.out.fill_(0)
            run.lse.fill_(0)
            seer.seer_decode_step_noalloc(run.dims, run.args(update_kbar=0))
            torch.cuda.synchronize()
            assert run.status.item() == 0, (rep, i)
            assert torch.equal(run.out, ref_out), (rep, i)
            assert torch.equal(run.lse, ref_lse), (rep, i)
