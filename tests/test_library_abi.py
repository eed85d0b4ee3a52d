"""The C-ABI library on the CPU: it loads, exports every symbol include/seer.h
declares, and its host-only helpers agree with the oracle and the fixtures.
No call here reaches the GPU (only argument checks that fail before any CUDA
work, and pure host helpers)."""
import ctypes
import json
import os
import re

import pytest

from block_sparse_attention_step_b200 import seer
from oracle import seer_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "seer.h")).read()
    return sorted(set(re.findall(r"SEER_API\s+[\w\s\*]+?\b(seer_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(seer.LIB_PATH):
        from block_sparse_attention_step_b200 import build
        build.build()
    return seer.library()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(declared) == sorted(seer.EXPORTS)
    assert seer.version() == 10000


def test_k_helpers_match_fixtures_and_oracle(lib):
    d = json.load(open(os.path.join(ROOT, "tests", "golden", "k_rules.json")))
    for c in d["sparsity"]:
        assert seer.seer_k_from_sparsity(c["nb"], c["permille"]) == c["k"]
    for c in d["budget"]:
        assert seer.seer_k_from_budget(c["nb"], c["budget"], c["block_size"]) == c["k"]
    for nb in list(range(0, 70)) + [127, 128, 129, 511, 512, 513, 1023, 1024]:
        for pm in (0, 1, 499, 500, 800, 900, 950, 999, 1000):
            assert seer.seer_k_from_sparsity(nb, pm) == O.k_from_sparsity(nb, pm), (nb, pm)
        for budget, bs in ((512, 64), (4096, 128), (4096, 64), (63, 64), (0, 64)):
            assert seer.seer_k_from_budget(nb, budget, bs) == O.k_from_budget(nb, budget, bs)
    with pytest.raises(seer.SeerError):
        seer.seer_k_from_sparsity(10, 1001)
    with pytest.raises(seer.SeerError):
        seer.seer_k_from_budget(10, 100, 0)


def test_dims_validation(lib):
    d = seer.make_dims(16, 40, 8, 128, 64, 512, 16 * 512)
    assert (d.stride_head, d.stride_token, d.stride_page) == (128, 8 * 128, 64 * 8 * 128)
    for bad, code in (((16, 40, 8, 64, 64, 512, 10), 2),      # D != 128
                      ((16, 40, 8, 128, 32, 512, 10), 2),      # block 32
                      ((16, 40, 7, 128, 64, 512, 10), 1),      # Hq % Hkv
                      ((16, 136, 8, 128, 64, 512, 10), 2),     # G = 17
                      ((16, 40, 8, 128, 64, 4097, 10), 2),     # too many blocks
                      ((0, 40, 8, 128, 64, 512, 10), 1)):      # empty batch
        with pytest.raises(seer.SeerError) as e:
            seer.make_dims(*bad)
        assert e.value.status == code, bad


def test_invalid_arguments_fail_before_any_launch(lib):
    d = seer.make_dims(2, 8, 2, 128, 64, 4, 8)
    null = None
    # null pointers -> SEER_ERR_INVALID_ARG, checked on the host
    assert lib.seer_pool_keys(ctypes.byref(d), null, null, null, 0, null, null, null) == 1
    assert lib.seer_gate_scores(ctypes.byref(d), null, null, null, null, 1.0, null, null, null) == 1
    assert lib.seer_block_select(ctypes.byref(d), null, null, null, 0, 4, null, null, null, null) == 1
    assert lib.seer_combine(ctypes.byref(d), null, null, 1, null, null, null) == 1
    fake = ctypes.c_void_p(4096)
    # k_max beyond max_blocks, splits out of range
    assert lib.seer_block_select(ctypes.byref(d), fake, fake, fake, 0, 5, fake, fake, null, null) == 1
    assert lib.seer_combine(ctypes.byref(d), fake, fake, 0, fake, null, null) == 1
    assert lib.seer_combine(ctypes.byref(d), fake, fake, 65, fake, null, null) == 1
    # misaligned pool pointer -> SEER_ERR_UNSUPPORTED
    odd = ctypes.c_void_p(4096 + 2)
    assert lib.seer_sparse_decode(ctypes.byref(d), fake, odd, fake, null, fake, fake, fake, 4, 1,
                                  0.1, fake, fake, null, null, null) == 2
    # o_part not 16-byte aligned (the merge writes float4 rows)
    assert lib.seer_sparse_decode(ctypes.byref(d), fake, fake, fake, null, fake, fake, fake, 4, 1,
                                  0.1, ctypes.c_void_p(4096 + 8), fake, null, null, null) == 2
    # misaligned item counter
    assert lib.seer_sparse_decode(ctypes.byref(d), fake, fake, fake, null, fake, fake, fake, 4, 1,
                                  0.1, fake, fake, ctypes.c_void_p(4096 + 4), null, null) == 2
    # unaligned strides
    d2 = seer.make_dims(2, 8, 2, 128, 64, 4, 8)
    d2.stride_token = 130
    assert lib.seer_pool_keys(ctypes.byref(d2), fake, null, fake, 0, fake, null, null) == 2
    # step without workspace
    a = seer.seer_step_args()
    a.k_per_seq = fake
    a.kbar = fake
    a.k_max = 4
    a.num_splits = 1
    assert lib.seer_decode_step(ctypes.byref(d), ctypes.byref(a), null) == 4
    # the host-buffer form checks the step before it enqueues q's copy (a copy
    # enqueued first would fail here with a CUDA error, or land on a GPU)
    a.out = fake
    assert lib.seer_decode_step_host(ctypes.byref(d), ctypes.byref(a), fake, fake, fake,
                                     null) == 4


def test_workspace_and_default_splits(lib):
    d = seer.make_dims(16, 40, 8, 128, 64, 512, 16 * 512)
    ws = seer.seer_step_workspace_bytes(d, 52, 8)
    r = lambda x: (x + 255) // 256 * 256
    expect = (r(16 * 8 * 512 * 4) + r(16 * 8 * 52 * 4) + r(16 * 8 * 4) +
              r(16 * 40 * 8 * 128 * 4) + r(16 * 40 * 8 * 4) + r(8 * 4) + r(16 * 8 * 4))
    assert ws == expect
    assert seer.seer_step_workspace_bytes(d, 0, 8) == 0
    s = seer.seer_default_splits(d, 52, 148)
    assert 1 <= s <= 26 and 16 * 8 * s >= 4 * 148
    d1 = seer.make_dims(1, 4, 1, 128, 64, 64, 64)
    assert seer.seer_default_splits(d1, 8, 148) == 4     # capped at k_max / 2
    assert seer.seer_default_splits(d1, 1, 148) == 1


def test_prefill_and_fused_host_checks(lib):
    d = seer.make_dims(2, 8, 2, 128, 64, 256, 2 * 256)
    # k of the last query block bounds every k_i: 10 % of 256 blocks, or 4096 / 64
    assert seer.seer_prefill_k_max(d, 900, 0) == O.k_from_sparsity(256, 900) == 26
    assert seer.seer_prefill_k_max(d, 0, 4096) == O.k_from_budget(256, 4096, 64) == 64
    rows = 2 * 2 * 256
    r = lambda x: (x + 255) // 256 * 256
    assert seer.seer_prefill_workspace_bytes(d, 26) == r(rows * 26 * 4) + r(rows * 4)
    null = None
    a = seer.seer_prefill_args()
    assert lib.seer_prefill(ctypes.byref(d), ctypes.byref(a), null) == 1      # no inputs
    # the attention stage alone: no selection, then no inputs
    assert lib.seer_prefill_attention(ctypes.byref(d), ctypes.byref(a), null, null, null) == 1
    sel = ctypes.c_void_p(4096)
    assert lib.seer_prefill_attention(ctypes.byref(d), ctypes.byref(a), sel, sel, null) == 1
    a.q = a.k_pool = a.v_pool = a.seqlens = a.out = ctypes.cast(ctypes.c_void_p(4096 + 8),
                                                                ctypes.c_void_p)
    a.k_max = 4
    assert lib.seer_prefill_attention(ctypes.byref(d), ctypes.byref(a), sel, sel, null) == 2
    fake = ctypes.c_void_p(4096)
    b = seer.seer_step_args()
    b.k_per_seq = b.kbar = fake
    b.k_max, b.num_splits, b.unified_heads = 4, 1, 1
    assert lib.seer_decode_step_fused(ctypes.byref(d), ctypes.byref(b), null) == 2   # unified
    b.unified_heads, b.k_new = 0, fake                                             # k_new alone
    assert lib.seer_decode_step_fused(ctypes.byref(d), ctypes.byref(b), null) == 1
    assert lib.seer_step_workspace_init(ctypes.byref(d), 4, 1, null, 0, null) == 4
    assert lib.seer_block_select_unified(ctypes.byref(d), null, null, null, 0, 4, null, null,
                                         null, null) == 1
    assert lib.seer_last_cuda_error().decode() == "no error"



def test_noalloc_scratch_size_matches_the_header():
    """The binding's copy of the no-allocation array size is the header's."""
    import re
    from block_sparse_attention_step_b200 import seer
    hdr = open(os.path.join(ROOT, "include", "seer.h")).read()
    m = re.search(r"#define SEER_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m, "SEER_NOALLOC_SCRATCH_BYTES not found in include/seer.h"
    assert seer.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
