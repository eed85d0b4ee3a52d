"""Device buffers for one decode step over a drawn workload (plumbing only).

``StepBuffers`` owns the torch allocations a caller of ``seer_decode_step``
needs besides the inputs (pooled keys, k per sequence, workspace, output,
status word) and issues the C-ABI calls through the ctypes binding.  Every
number it produces comes from the library's kernels.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import seer


def gate_recall(dense_mass: torch.Tensor, idx: torch.Tensor, n_sel: torch.Tensor,
                group: int) -> torch.Tensor:
    """Gate recall per (b, query head): the share of the dense attention
    distribution that a sparse selection keeps, i.e. the sum over the chosen
    blocks j of mass[b, qh, j], with `dense_mass` the block masses of a step
    that selected every block (the self-distilled gate's training target) and
    `idx` / `n_sel` the selection of the sparse step on the same inputs
    (query head qh reads the row of KV head qh // group).  An analysis
    metric over the step's outputs (a gather and a sum), not a step of the
    path.  Returns [B][Hq] fp32; 1 means the selection holds all the mass."""
    k_max = idx.shape[-1]
    live = torch.arange(k_max, device=idx.device)[None, None, :] < n_sel[..., None]
    j = idx.long().clamp(min=0).repeat_interleave(group, dim=1)       # [B][Hq][k_max]
    live = live.repeat_interleave(group, dim=1)
    return (torch.gather(dense_mass, 2, j) * live).sum(-1)


class StepBuffers:
    def __init__(self, w, data: dict, num_splits: Optional[int] = None,
                 sparsity_permille: Optional[int] = None, budget_tokens: Optional[int] = None,
                 force_newest: Optional[bool] = None, k_max: Optional[int] = None,
                 device: Optional[torch.device] = None, mass: bool = False,
                 unified: bool = False):
        self.w = w
        self.data = data
        dev = device or data["q"].device
        self.device = dev
        B, Hkv, D = w.batch, w.kv_heads, w.head_dim
        self.nb_max = data["nb_max"]
        from .workloads import pool_strides
        sp, st, sh = pool_strides(data)
        self.dims = seer.make_dims(B, w.q_heads, Hkv, D, w.block_size, self.nb_max,
                                   data["num_pages"], sp, st, sh)
        self.budget = w.budget_tokens if budget_tokens is None else budget_tokens
        self.permille = w.sparsity_permille if sparsity_permille is None else sparsity_permille
        if self.budget is None and self.permille is None:
            raise ValueError("workload has neither a budget nor a sparsity")
        self.force_newest = w.force_newest if force_newest is None else force_newest
        self.unified = bool(unified)   # one block set per sequence for all KV heads
        self.k_per_seq = torch.empty(B, dtype=torch.int32, device=dev)
        seer.seer_fill_k(self.dims, data["seqlens"], self.permille or 0, self.budget or 0,
                         self.k_per_seq)
        self.k_max = int(k_max) if k_max is not None else int(self.k_per_seq.max().item())
        self.k_max = max(1, min(self.k_max, self.nb_max))
        if num_splits is None:
            num_splits = w.num_splits or seer.seer_default_splits(self.dims, self.k_max, 0)
        self.num_splits = int(num_splits)
        self.kbar = torch.empty((B, Hkv, self.nb_max, D), dtype=torch.float32, device=dev)
        ws = seer.seer_step_workspace_bytes(self.dims, self.k_max, self.num_splits)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        # control words of the single-launch step start at zero
        seer.seer_step_workspace_init(self.dims, self.k_max, self.num_splits, self.workspace)
        self.out = torch.empty((B, w.q_heads, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, w.q_heads), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.scale = 1.0 / math.sqrt(D)
        # a contiguous cache needs no page table (identity pages)
        self.page_table = data["page_table"] if w.paged else None
        # optional per-block attention mass of every step
        self.block_lse = self.block_mass = None
        if mass:
            self.block_lse = torch.empty(seer.seer_block_lse_elems(self.dims), dtype=torch.float32,
                                         device=dev)
            self.block_mass = torch.empty((B, w.q_heads, self.nb_max), dtype=torch.float32,
                                          device=dev)

    # views into the workspace, in the order the library carves it
    def workspace_views(self):
        B, Hkv, Hq, S, D = self.w.batch, self.w.kv_heads, self.w.q_heads, self.num_splits, self.w.head_dim

        def r256(x):
            return (x + 255) // 256 * 256
        off = 0
        out = {}
        for name, n, dt in (("scores", B * Hkv * self.nb_max, torch.float32),
                            ("idx", B * Hkv * self.k_max, torch.int32),
                            ("n_sel", B * Hkv, torch.int32),
                            ("o_part", B * Hq * S * D, torch.float32),
                            ("lse_part", B * Hq * S, torch.float32),
                            ("ctl", 8, torch.int32),
                            ("row_flag", B * Hkv, torch.int32)):
            nbytes = n * 4
            out[name] = self.workspace[off:off + nbytes].view(dt)
            off += r256(nbytes)
        out["scores"] = out["scores"].view(B, Hkv, self.nb_max)
        out["idx"] = out["idx"].view(B, Hkv, self.k_max)
        out["n_sel"] = out["n_sel"].view(B, Hkv)
        out["o_part"] = out["o_part"].view(B, Hq, S, D)
        out["lse_part"] = out["lse_part"].view(B, Hq, S)
        return out

    def pool_full(self, stream=None):
        d = self.data
        seer.seer_pool_keys(self.dims, d["k_pool"], self.page_table, d["seqlens"], 0, self.kbar,
                            self.status, stream)

    def args(self, update_kbar: int = 0, q=None, k_new=None,
             v_new=None) -> "seer.seer_step_args":
        d = self.data
        return seer.step_args(d["q"] if q is None else q, d["k_pool"], d["v_pool"], self.page_table,
                              d["seqlens"], d["w_gate"], self.kbar, self.k_per_seq,
                              update_kbar=update_kbar, force_newest=self.force_newest,
                              k_max=self.k_max, num_splits=self.num_splits, gate_scale=self.scale,
                              softmax_scale=self.scale, workspace=self.workspace, out=self.out,
                              lse_out=self.lse, dev_status=self.status,
                              block_lse=self.block_lse, block_mass=self.block_mass,
                              unified_heads=self.unified, k_new=k_new, v_new=v_new)

    def step(self, update_kbar: int = 0, stream=None, args=None, fused: bool = False):
        call = seer.seer_decode_step_fused if fused else seer.seer_decode_step
        call(self.dims, args if args is not None else self.args(update_kbar), stream)


class PrefillBuffers:
    """Device buffers for the prefill path over a drawn workload: prompt
    queries (seeded), pooled keys, workspace, output, lse, gate scores."""

    def __init__(self, w, data: dict, q, sparsity_permille: Optional[int] = None,
                 budget_tokens: Optional[int] = None, keep_scores: bool = False):
        from .workloads import pool_strides
        self.w, self.data, self.q = w, data, q
        dev = q.device
        B, Hkv, D = w.batch, w.kv_heads, w.head_dim
        self.nb_max = data["nb_max"]
        sp, st, sh = pool_strides(data)
        self.dims = seer.make_dims(B, w.q_heads, Hkv, D, w.block_size, self.nb_max,
                                   data["num_pages"], sp, st, sh)
        self.budget = (w.budget_tokens if budget_tokens is None else budget_tokens) or 0
        self.permille = (w.sparsity_permille if sparsity_permille is None else sparsity_permille) or 0
        self.k_max = max(1, seer.seer_prefill_k_max(self.dims, self.permille, self.budget))
        self.kbar = torch.empty((B, Hkv, self.nb_max, D), dtype=torch.float32, device=dev)
        ws = seer.seer_prefill_workspace_bytes(self.dims, self.k_max)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        Lq = self.nb_max * w.block_size
        self.out = torch.zeros((B, Lq, w.q_heads, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, w.q_heads, Lq), dtype=torch.float32, device=dev)
        self.scores = (torch.empty((B, Hkv, self.nb_max, self.nb_max), dtype=torch.float32,
                                   device=dev) if keep_scores else None)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.scale = 1.0 / math.sqrt(D)
        self.page_table = data["page_table"] if w.paged else None

    def selection(self):
        rows = self.w.batch * self.w.kv_heads * self.nb_max
        idx = self.workspace[:rows * self.k_max * 4].view(torch.int32).view(
            self.w.batch, self.w.kv_heads, self.nb_max, self.k_max)
        off = (rows * self.k_max * 4 + 255) // 256 * 256
        n_sel = self.workspace[off:off + rows * 4].view(torch.int32).view(
            self.w.batch, self.w.kv_heads, self.nb_max)
        return idx, n_sel

    def attention(self, out=None, lse=None, stream=None):
        """The attention stage alone over the selection the last run() left
        in the workspace (seer_prefill_attention)."""
        idx, n_sel = self.selection()
        d = self.data
        seer.seer_prefill_attention(self.dims, self.q, d["k_pool"], d["v_pool"], self.page_table,
                                    d["seqlens"], idx, n_sel, k_max=self.k_max,
                                    softmax_scale=self.scale,
                                    out=self.out if out is None else out,
                                    lse_out=self.lse if lse is None else lse,
                                    dev_status=self.status, stream=stream)

    def run(self, pool_keys: bool = True, stream=None):
        d = self.data
        seer.seer_prefill(self.dims, self.q, d["k_pool"], d["v_pool"], self.page_table,
                          d["seqlens"], d["w_gate"], self.kbar, pool_keys=pool_keys,
                          sparsity_permille=self.permille, budget_tokens=self.budget,
                          k_max=self.k_max, gate_scale=self.scale, softmax_scale=self.scale,
                          workspace=self.workspace, out=self.out, lse_out=self.lse,
                          scores_out=self.scores, dev_status=self.status, stream=stream)
