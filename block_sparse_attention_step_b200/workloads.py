"""Seeded synthetic workloads for the block-sparse decode step.

This module only draws inputs: shapes, seeded random tensors and a paged
layout.  It holds none of the step's arithmetic (no pooling, scoring,
selection, k rule or attention), so both the CUDA library's tests and the CPU
oracle can take their inputs from it without sharing any of the method.

Value recipe (per workload, all seeded through one ``torch.Generator`` on the
target device, drawn in fixed-size page chunks so that a seed always gives the
same tensors):

* q ~ N(0, 1) rounded to bf16 (round-to-nearest-even), [B][Hq][D];
* gate projection W ~ N(0, 1/D) in fp32, [Hkv][D][D] (one D x D matrix per
  KV head, g = W q);
* K, V ~ N(0, 1) plus, where the workload says so, a per-(page, KV head)
  offset vector added to every row of that page before rounding to bf16:
  N(0, var) entries, or Student-t entries with nu = 3 drawn from its
  definition Z / sqrt(chi2_3 / 3);
* sequence lengths fixed, or uniform integers in [lo, hi] for ragged batches;
* a paged cache [P][page][Hkv][D] whose pages are a seeded random permutation
  (``paged``), else the identity table (page of block j of sequence b is
  b * NBmax + j, i.e. a contiguous [B][NBmax * bs][Hkv][D] cache).

The published workloads these stand in for (reasoning traces of a trained
model) are not reproducible here; the shapes, block sizes, budgets and
sparsities match the step's specification.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_CHUNK_PAGES = 2048  # pages drawn per randn call; fixed so seeds are stable


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    block_size: int
    seqlen: Optional[int] = None            # fixed length for every sequence
    seqlen_range: Optional[Tuple[int, int]] = None  # inclusive, ragged batch
    paged: bool = False
    offsets: str = "none"                   # "none" | "normal" | "student_t"
    offset_var: float = 0.0
    budget_tokens: Optional[int] = None
    sparsity_permille: Optional[int] = None
    force_newest: bool = False
    num_splits: Optional[int] = None
    # seed of the full-size draw; where it is not 1 it was picked by rejection
    # so that every (b, KV head) row's gate margin at the k / k+1 boundary
    # exceeds 1e-4 (see ``seed_note``)
    seed: int = 1
    seed_note: str = ""

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # one GQA-4 group, 4K context, budget of 512 tokens (8 of 64 blocks)
    "b1_g4_L4k_bs64_budget512": Workload(
        "b1_g4_L4k_bs64_budget512", batch=1, q_heads=4, kv_heads=1,
        head_dim=128, block_size=64, seqlen=4096, budget_tokens=512),
    # 8 x 32/8 heads, 8K context, 90% sparsity (13 of 128), newest forced,
    # per-block N(0, 0.5) offsets so the gate separates blocks
    "b8_h32_L8k_bs64_s90_newest": Workload(
        "b8_h32_L8k_bs64_s90_newest", batch=8, q_heads=32, kv_heads=8,
        head_dim=128, block_size=64, seqlen=8192, offsets="normal",
        offset_var=0.5, sparsity_permille=900, force_newest=True, seed=2,
        seed_note="seed 1 draws a row with a 1.6e-6 gate margin; seed 2's smallest "
                  "margin over all 64 rows is 2.7e-4"),
    # 16 x 40/8 heads, 32K context, 90% sparsity (52 of 512), 8 splits
    "b16_h40_L32k_bs64_s90": Workload(
        "b16_h40_L32k_bs64_s90", batch=16, q_heads=40, kv_heads=8,
        head_dim=128, block_size=64, seqlen=32768, sparsity_permille=900,
        num_splits=8),
    # 16 x 40/8 heads, 32K context, block 128, 4096-token budget (32 of 256),
    # Student-t(3) block offsets, newest forced
    "b16_h40_L32k_bs128_budget4k_newest": Workload(
        "b16_h40_L32k_bs128_budget4k_newest", batch=16, q_heads=40,
        kv_heads=8, head_dim=128, block_size=128, seqlen=32768,
        offsets="student_t", budget_tokens=4096, force_newest=True),
    # ragged 64 sequences, L ~ U[4096, 65536], 64/8 heads, paged random table
    "b64_ragged_h64_paged_bs64": Workload(
        "b64_ragged_h64_paged_bs64", batch=64, q_heads=64, kv_heads=8,
        head_dim=128, block_size=64, seqlen_range=(4096, 65536), paged=True,
        sparsity_permille=900),
}

HEADLINE = "b16_h40_L32k_bs64_s90"


def _ceil_div(a, b):
    return -(-a // b)


def _offsets(w: Workload, shape, g, device):
    if w.offsets == "none":
        return None
    if w.offsets == "normal":
        return torch.randn(shape, generator=g, device=device) * (w.offset_var ** 0.5)
    if w.offsets == "student_t":
        z = torch.randn(shape, generator=g, device=device)
        chi2 = torch.randn((3,) + tuple(shape), generator=g, device=device).pow(2).sum(0)
        return z / torch.sqrt(chi2 / 3.0)
    raise ValueError(f"unknown offsets kind {w.offsets!r}")


def _draw_pool(w: Workload, num_pages: int, g, device):
    """[P][bs][Hkv][D] bf16 pool drawn in fixed page chunks."""
    bs, H, D = w.block_size, w.kv_heads, w.head_dim
    pool = torch.empty((num_pages, bs, H, D), dtype=torch.bfloat16, device=device)
    for p0 in range(0, num_pages, _CHUNK_PAGES):
        n = min(_CHUNK_PAGES, num_pages - p0)
        x = torch.randn((n, bs, H, D), generator=g, device=device)
        off = _offsets(w, (n, H, D), g, device)
        if off is not None:
            x += off[:, None, :, :]
        pool[p0:p0 + n] = x.to(torch.bfloat16)
        del x, off
    return pool


def generate(w: Workload, seed: int, device="cpu", layout: str = "nhd") -> dict:
    """Draw one workload.  Returns a dict of tensors on ``device``:
    q [B][Hq][D] bf16, w_gate [Hkv][D][D] f32, k_pool / v_pool bf16 pages,
    page_table [B][NBmax] i32 (-1 past a sequence's last block), seqlens [B]
    i32, plus ``nb_max``, ``num_pages`` and ``layout`` ("nhd": pages
    [P][bs][Hkv][D], token-major; "hnd": pages [P][Hkv][bs][D], head-major --
    the same values, stored permuted)."""
    if layout not in ("nhd", "hnd"):
        raise ValueError(f"unknown layout {layout!r}")
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    B, bs, D = w.batch, w.block_size, w.head_dim
    if w.seqlen_range is not None:
        lo, hi = w.seqlen_range
        seqlens = torch.randint(lo, hi + 1, (B,), generator=g, device=device,
                                dtype=torch.int64)
    else:
        seqlens = torch.full((B,), int(w.seqlen), dtype=torch.int64, device=device)
    nb = [_ceil_div(int(L), bs) for L in seqlens.tolist()]
    nb_max = max(nb)
    if w.paged:
        num_pages = sum(nb)
        perm = torch.randperm(num_pages, generator=g, device=device)
        table = torch.full((B, nb_max), -1, dtype=torch.int64, device=device)
        off = 0
        for b in range(B):
            table[b, :nb[b]] = perm[off:off + nb[b]]
            off += nb[b]
    else:
        num_pages = B * nb_max
        table = torch.arange(num_pages, dtype=torch.int64, device=device).view(B, nb_max)
        for b in range(B):
            table[b, nb[b]:] = -1
    q = torch.randn((B, w.q_heads, D), generator=g, device=device).to(torch.bfloat16)
    w_gate = torch.randn((w.kv_heads, D, D), generator=g, device=device) * (1.0 / D) ** 0.5
    k_pool = _draw_pool(w, num_pages, g, device)
    v_pool = _draw_pool(w, num_pages, g, device)
    if layout == "hnd":
        k_pool = k_pool.permute(0, 2, 1, 3).contiguous()
        v_pool = v_pool.permute(0, 2, 1, 3).contiguous()
    return {
        "q": q.contiguous(),
        "w_gate": w_gate.float().contiguous(),
        "k_pool": k_pool,
        "v_pool": v_pool,
        "page_table": table.to(torch.int32).contiguous(),
        "seqlens": seqlens.to(torch.int32).contiguous(),
        "nb_max": int(nb_max),
        "num_pages": int(num_pages),
        "layout": layout,
    }


def pool_strides(data: dict):
    """(stride_page, stride_token, stride_head) in elements of the pools."""
    k = data["k_pool"]
    if data.get("layout", "nhd") == "hnd":
        return k.stride(0), k.stride(2), k.stride(1)
    return k.stride(0), k.stride(1), k.stride(2)


def gather_rows(pool: torch.Tensor, page_table: torch.Tensor, b: int, h: int,
                seqlen: int, block_size: int, layout: str = "nhd") -> torch.Tensor:
    """Token-ordered rows [L][D] of KV head h of sequence b, copied to the
    host in the pool's dtype (a layout walk, no arithmetic)."""
    nb = _ceil_div(int(seqlen), block_size)
    pages = page_table[b, :nb].to(device=pool.device, dtype=torch.int64)
    picked = pool.index_select(0, pages)
    if layout == "nhd":                   # [P][bs][Hkv][D]
        rows = picked[:, :, h, :]
    else:                                 # [P][Hkv][bs][D]
        rows = picked[:, h, :, :]
    return rows.reshape(nb * block_size, -1)[:seqlen].cpu()


def prefill_queries(w: Workload, seed: int, max_blocks: int, device="cpu") -> torch.Tensor:
    """Prompt queries for the prefill path: [B][max_blocks * bs][Hq][D] bf16,
    N(0, 1) rounded to nearest, drawn from their own seeded generator (the
    decode draw of the same seed is left unchanged)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed * 7919 + 17)
    shape = (w.batch, max_blocks * w.block_size, w.q_heads, w.head_dim)
    return torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
