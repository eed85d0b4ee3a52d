"""fp64 CPU oracle for the SeerAttention-R block-sparse decode step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers, tables or constants); it works on
plain numpy float64 arrays that the caller has already converted from the
seeded inputs.

What the step computes, and where each part comes from
------------------------------------------------------
Sources are the pages this project was specified from, cited by page title and
section:

* "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning" (paper
  summary page, Abstract): a self-distilled gate picks KV blocks for each
  decode query; query pooling is removed for auto-regressive decoding; blocks
  are large (64 or 128 tokens); accuracy holds at a 4K-token budget; the
  sparse decoding kernel runs at 90% sparsity.
* "Sparse Attention Reasoning" (Agent Skill page), Step 1 "Design Sparse
  Attention Gate": k from a sparsity ratio and a top-k over scores.
* Same page, Step 4 "Optimized Kernel Implementation": the meaning of sparse
  attention -- scores Q.K^T / sqrt(head_dim), unselected keys filled with
  -inf, softmax over keys, weights times V.
* The step specification this library implements (gate = mean-pooled block
  keys dotted with the gate-projected query, in fp32 on the GPU; per-KV-head
  top-k with ties to the lower block index and an optional forced newest
  block; split-KV partials merged by a log-sum-exp combine).

Readings taken where the pages are silent (each is also listed in the design
notes): the GQA group's score is the mean of its query heads' scores; the gate
scale is 1/sqrt(D); k = max(1, ceil((1000 - permille) * NB / 1000)) from a
sparsity, k = max(1, min(NB, budget // bs)) from a token budget; a forced
newest block counts toward k; indices come out ascending; NaN scores rank
below -inf and -0.0 equals +0.0; split s of S covers the selected blocks
[floor(s*n/S), floor((s+1)*n/S)) of the ascending list.

Every function here is pinned by ``tests/test_oracle_pins.py`` to closed
forms, brute force, library routines or the hand-worked fixtures in
``tests/golden/``; none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "num_blocks",
    "pool_keys",
    "gate_scores",
    "k_from_sparsity",
    "k_from_budget",
    "select_blocks",
    "selection_margin",
    "selection_is_valid",
    "masked_attention",
    "split_partials",
    "combine",
    "decode_row",
    "block_mass",
    "unified_scores",
    "unified_scores_f32",
    "select_blocks_unified",
    "pool_queries",
    "prefill_gate_scores",
    "prefill_gate_row",
    "prefill_select",
    "prefill_attention",
    "prefill_attention_token",
    "prefill_row",
]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> float64: a bf16 value is the top 16 bits of a float32."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def num_blocks(seqlen: int, block_size: int) -> int:
    """NB = ceil(L / bs): the number of KV blocks of a sequence of length L
    (the newest one possibly partial).  Block granularity: paper summary page,
    Abstract ("large sparse attention block sizes (64/128)")."""
    return -(-int(seqlen) // int(block_size))


def pool_keys(K: np.ndarray, seqlen: int, block_size: int) -> np.ndarray:
    """Mean-pooled block keys of one (sequence, KV head).

    K: [>= seqlen][D] float64 key rows in token order.  Returns kbar [NB][D]
    where kbar[j] is the plain mean of the valid rows t (t < seqlen) of block
    j.  Only keys are pooled: the paper summary page's Abstract removes query
    pooling for decoding, so the query enters the gate unpooled.
    """
    L = int(seqlen)
    nb = num_blocks(L, block_size)
    D = K.shape[1]
    kbar = np.zeros((nb, D), dtype=np.float64)
    for j in range(nb):
        lo = j * block_size
        hi = min(lo + block_size, L)
        kbar[j] = K[lo:hi].sum(axis=0) / float(hi - lo)
    return kbar


def gate_scores(q_group: np.ndarray, W: np.ndarray, kbar: np.ndarray,
                scale: float) -> np.ndarray:
    """Gate score of every block for one KV head.

    q_group: [G][D] the GQA group's decode queries; W: [D][D] this KV head's
    gate projection (g = W q, row-major: g[i] = sum_j W[i][j] q[j]); kbar:
    [NB][D].  Each query head scores block j as (W q).kbar[j]; the group's
    score is the mean over its G heads, times ``scale`` (1/sqrt(D)).  Written
    head by head and averaged last, deliberately not in the order a GPU would
    use (average the queries first).
    """
    per_head = np.empty((q_group.shape[0], kbar.shape[0]), dtype=np.float64)
    for g in range(q_group.shape[0]):
        projected = W @ q_group[g]
        per_head[g] = kbar @ projected
    return per_head.mean(axis=0) * float(scale)


def k_from_sparsity(nb: int, sparsity_permille: int) -> int:
    """Blocks kept at a sparsity given in permille: the fraction (1 - s) of
    the NB blocks, rounded up, at least one.  Agent Skill page, Step 1, keeps
    "the top (1 - sparsity) fraction"; rounding up is the reading that gives
    13 of 128 and 52 of 512 blocks at 90%."""
    if not 0 <= sparsity_permille <= 1000:
        raise ValueError("sparsity_permille must be within [0, 1000]")
    kept = (1000 - int(sparsity_permille)) * int(nb)
    return max(1, -(-kept // 1000))


def k_from_budget(nb: int, budget_tokens: int, block_size: int) -> int:
    """Blocks kept under a token budget (paper summary page, Abstract: a 4K
    token budget): floor(budget / bs) whole blocks, capped at NB, at least
    one."""
    return max(1, min(int(nb), int(budget_tokens) // int(block_size)))


def _rank_key(score: float, index: int):
    """Sort key of a block: finite and infinite scores by value descending,
    then NaN last; equal scores (with -0.0 == +0.0, which Python's == already
    gives) by lower index first."""
    if math.isnan(score):
        return (1, 0.0, index)
    return (0, -score, index)


def select_blocks(scores: Sequence[float], k: int,
                  force_newest: bool) -> np.ndarray:
    """Top-k blocks of one KV head, returned in ascending block order.

    scores: [NB] (the valid blocks only).  The newest block NB-1, when
    forced, is taken first and counts toward k; the other k-1 (or k) places go
    to the best remaining blocks under (score descending, index ascending).
    Agent Skill page, Step 1 (top-k over importance scores); the tie rule and
    the forced block come from the step specification.
    """
    s = [float(x) for x in np.asarray(scores, dtype=np.float64)]
    nb = len(s)
    k = min(int(k), nb)
    taken = []
    candidates = list(range(nb))
    if force_newest and nb > 0 and k > 0:
        taken.append(nb - 1)
        candidates.remove(nb - 1)
    candidates.sort(key=lambda j: _rank_key(s[j], j))
    taken.extend(candidates[: max(0, k - len(taken))])
    return np.array(sorted(taken), dtype=np.int64)


def selection_margin(scores: Sequence[float], k: int,
                     force_newest: bool) -> float:
    """Gap between the last block taken on merit and the first one left out
    (forced block excluded from the ranking).  +inf when nothing is left out
    or nothing is chosen on merit.  Rows whose margin exceeds the gate
    tolerance must select bit-identically on both sides."""
    s = np.asarray(scores, dtype=np.float64)
    nb = len(s)
    k = min(int(k), nb)
    pool = list(range(nb))
    kk = k
    if force_newest and nb > 0 and k > 0:
        pool.remove(nb - 1)
        kk -= 1
    if kk <= 0 or kk >= len(pool):
        return math.inf
    ranked = sorted(pool, key=lambda j: _rank_key(float(s[j]), j))
    a, b = float(s[ranked[kk - 1]]), float(s[ranked[kk]])
    if math.isnan(a) or math.isnan(b):
        return 0.0
    return float(a - b)


def selection_is_valid(scores: Sequence[float], chosen: Sequence[int], k: int,
                       force_newest: bool, tol: float) -> bool:
    """Whether an index list is a correct top-k up to ``tol``: right count,
    ascending, unique, in range, forced block present, and every block chosen
    on merit scores at least every block left out, minus ``tol``."""
    s = np.asarray(scores, dtype=np.float64)
    nb = len(s)
    k = min(int(k), nb)
    chosen = [int(c) for c in chosen]
    if len(chosen) != k or chosen != sorted(set(chosen)):
        return False
    if any(c < 0 or c >= nb for c in chosen):
        return False
    merit = set(chosen)
    if force_newest and k > 0:
        if nb - 1 not in merit:
            return False
        merit.discard(nb - 1)
    left_out = [j for j in range(nb) if j not in chosen]
    if not merit or not left_out:
        return True
    def value(j):  # NaN ranks with -inf here: below every real score
        return -math.inf if math.isnan(s[j]) else float(s[j])
    worst_in = min(value(j) for j in merit)
    best_out = max(value(j) for j in left_out)
    return bool(worst_in >= best_out - tol)


def masked_attention(q_group: np.ndarray, K: np.ndarray, V: np.ndarray,
                     seqlen: int, blocks: Sequence[int], block_size: int,
                     scale: float):
    """Exact softmax attention of G decode queries over the selected blocks.

    Agent Skill page, Step 4: scores = q.K^T * scale over all L cached keys,
    every key outside the selected blocks (and every tail slot t >= L of a
    partial block) set to -inf, softmax over keys, weights times V.  The
    current token's K/V sits at position L-1 already, so no causal mask is
    needed beyond t < L.  The weighted sum runs over the selected keys only:
    every other weight is exactly zero, and skipping them keeps garbage (NaN)
    in unselected or tail slots out of the result.

    Returns (out [G][D], lse [G]) with lse the natural-log log-sum-exp of the
    scaled scores; an empty selection gives (zeros, -inf).
    """
    L = int(seqlen)
    G, D = q_group.shape
    keep = np.zeros(L, dtype=bool)
    for j in blocks:
        lo = int(j) * block_size
        keep[lo:min(lo + block_size, L)] = True
    if not keep.any():
        return np.zeros((G, V.shape[1])), np.full(G, -np.inf)
    x = np.full((G, L), -np.inf, dtype=np.float64)
    x[:, keep] = (q_group @ K[:L][keep].T) * float(scale)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    total = e.sum(axis=1, keepdims=True)
    p = e / total
    out = p[:, keep] @ V[:L][keep]
    lse = (m + np.log(total))[:, 0]
    return out, lse


def split_partials(q_group, K, V, seqlen, blocks, block_size, scale,
                   num_splits: int):
    """Split-KV partials: the ascending block list cut into ``num_splits``
    contiguous pieces, piece s holding entries [floor(s*n/S), floor((s+1)*n/S)),
    each attended on its own with ``masked_attention``.  An empty piece gives
    o = 0 and lse = -inf.  Returns (o [S][G][D], lse [S][G])."""
    blocks = list(int(b) for b in blocks)
    n = len(blocks)
    S = int(num_splits)
    outs, lses = [], []
    for s in range(S):
        piece = blocks[(s * n) // S:((s + 1) * n) // S]
        o, l = masked_attention(q_group, K, V, seqlen, piece, block_size, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def combine(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Log-sum-exp merge of split partials (the step specification's combine).

    o_parts: [S][G][D] per-piece normalised outputs; lse_parts: [S][G].  The
    merged lse is log(sum_s exp(lse_s)); the output is sum_s exp(lse_s - lse)
    * o_s.  Pieces with lse = -inf weigh nothing.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - safe_m[None, :])
    total = w.sum(axis=0)
    lse = np.where(total > 0, safe_m + np.log(np.where(total > 0, total, 1.0)), -np.inf)
    weights = np.where(total[None, :] > 0, w / np.where(total > 0, total, 1.0)[None, :], 0.0)
    out = np.einsum("sg,sgd->gd", weights, np.asarray(o_parts, dtype=np.float64))
    return out, lse


def decode_row(q_group, W, K, V, seqlen, block_size, k, force_newest,
               gate_scale, softmax_scale):
    """The whole step for one (sequence, KV head): pool keys, gate scores,
    top-k selection, then masked softmax attention of the G query heads over
    the chosen blocks.  Returns a dict with kbar, scores, indices, out, lse."""
    kbar = pool_keys(K, seqlen, block_size)
    scores = gate_scores(q_group, W, kbar, gate_scale)
    idx = select_blocks(scores, k, force_newest)
    out, lse = masked_attention(q_group, K, V, seqlen, idx, block_size,
                                softmax_scale)
    return {"kbar": kbar, "scores": scores, "indices": idx, "out": out,
            "lse": lse}


def block_mass(q_group, K, seqlen, blocks, block_size, scale):
    """Attention mass of every block: mass[g][j] = sum of query head g's
    softmax weights (the Agent Skill page's Step 4 definition, over the
    selected blocks) on the tokens t < L of block j; 0 for blocks that were
    not selected.  With every block selected this is the dense model's
    block-level attention distribution, the target the self-distilled gate
    is trained toward (paper summary page, Abstract: "self-distilled gating").
    Returns [G][NB]."""
    L = int(seqlen)
    G = q_group.shape[0]
    nb = num_blocks(L, block_size)
    mass = np.zeros((G, nb), dtype=np.float64)
    blocks = sorted(int(j) for j in blocks)
    if not blocks:
        return mass
    rows = np.concatenate([np.arange(j * block_size, min((j + 1) * block_size, L)) for j in blocks])
    x = (q_group @ K[rows].T) * float(scale)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    p = e / e.sum(axis=1, keepdims=True)
    owner = rows // block_size
    for j in blocks:
        mass[:, j] = p[:, owner == j].sum(axis=1)
    return mass


def unified_scores(per_head_scores) -> np.ndarray:
    """Cross-head block ranking of one sequence: one block set shared by every
    KV head, as in the unified cross-head selection of the LessIsMore
    abstract on the author page (aggregate the heads' evidence, then rank
    once).  Reading taken: each block's aggregate is the sum over KV heads of
    its gate score (ranking by the sum is ranking by the mean).  fp64; NaN or
    +inf with -inf in a column give NaN, -inf alone gives -inf.
    per_head_scores: [Hkv][NB].  Returns [NB]."""
    s = np.asarray(per_head_scores, dtype=np.float64)
    out = np.zeros(s.shape[1], dtype=np.float64)
    for h in range(s.shape[0]):
        out = out + s[h]
    return out


def unified_scores_f32(per_head_scores_f32) -> np.ndarray:
    """The same aggregate in fp32, heads added in order h = 0, 1, ...: the
    values the GPU's unified select ranks when it is given fp32 scores, so
    that a test on given scores can demand identical indices (the integer
    decision is taken in the kernel's precision on both sides)."""
    s = np.asarray(per_head_scores_f32, dtype=np.float32)
    out = np.zeros(s.shape[1], dtype=np.float32)
    for h in range(s.shape[0]):
        out = (out + s[h]).astype(np.float32)
    return out


def select_blocks_unified(per_head_scores, k: int, force_newest: bool) -> np.ndarray:
    """Top-k of the cross-head aggregate (``unified_scores``) under the same
    order, forced block and ascending output as ``select_blocks``; every KV
    head of the sequence then attends these blocks."""
    return select_blocks(unified_scores(per_head_scores), k, force_newest)


# ---------------------------------------------------------------- prefill with query pooling
#
# SeerAttention-R removes query pooling to decode token by token (paper
# summary page, Abstract: it extends SeerAttention, whose gate pools queries).
# The prefill path here is that pooled form, in the notation of the decode
# step.  Readings (the pages give no formula for it): query block i holds the
# query tokens [i*bs, min((i+1)*bs, L)); its pooled query is the mean over
# those tokens and over the G heads of the group; block j scores
# gate_scale * (W qbar_i) . kbar_j for j <= i only (a query never sees later
# keys); block i itself is always selected (it holds the query's own recent
# keys, the prefill form of the forced newest block) and counts toward k;
# every query token then attends, causally, the tokens of its block's chosen
# blocks that do not come after it.


def pool_queries(Q_group: np.ndarray, seqlen: int, block_size: int) -> np.ndarray:
    """Pooled queries of one (sequence, KV head): Q_group [>= L][G][D];
    returns qbar [NB][D], the mean over the valid tokens of query block i and
    over the group's G heads."""
    L = int(seqlen)
    nb = num_blocks(L, block_size)
    qbar = np.zeros((nb, Q_group.shape[2]), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * block_size, min((i + 1) * block_size, L)
        rows = Q_group[lo:hi].reshape(-1, Q_group.shape[2])
        qbar[i] = rows.sum(axis=0) / float(rows.shape[0])
    return qbar


def prefill_gate_scores(Q_group: np.ndarray, W: np.ndarray, kbar: np.ndarray, seqlen: int,
                        block_size: int, scale: float) -> np.ndarray:
    """Block-to-block gate scores [NB][NB] of one (sequence, KV head): entry
    (i, j) is scale * (W qbar_i) . kbar_j for j <= i and -inf above the
    diagonal.  Written token by token and head by head and averaged last (the
    mean of the per-query scores equals the score of the pooled query), not
    in the order a GPU would use."""
    L = int(seqlen)
    nb = num_blocks(L, block_size)
    out = np.full((nb, nb), -np.inf, dtype=np.float64)
    for i in range(nb):
        out[i, : i + 1] = prefill_gate_row(Q_group, W, kbar, L, block_size, scale, i)
    return out


def prefill_gate_row(Q_group: np.ndarray, W: np.ndarray, kbar: np.ndarray, seqlen: int,
                     block_size: int, scale: float, i: int) -> np.ndarray:
    """Row i of ``prefill_gate_scores`` on its causal prefix: [i + 1] scores
    of query block i against key blocks 0..i (each query token and head of
    block i scored on its own, the mean taken last)."""
    lo, hi = i * block_size, min((i + 1) * block_size, int(seqlen))
    acc = np.zeros(i + 1, dtype=np.float64)
    count = 0
    for t in range(lo, hi):
        for g in range(Q_group.shape[1]):
            acc += kbar[: i + 1] @ (W @ Q_group[t, g])
            count += 1
    return acc / count * float(scale)


def prefill_select(scores: np.ndarray, k_of_block) -> list:
    """Per query block i: the top-k_i of row i over blocks 0..i with block i
    forced (``select_blocks`` with the forced newest block on the causal
    prefix).  k_of_block(i) gives k_i.  Returns a list of ascending arrays."""
    return [select_blocks(scores[i, : i + 1], k_of_block(i), True) for i in range(scores.shape[0])]


def prefill_attention(Q_group: np.ndarray, K: np.ndarray, V: np.ndarray, seqlen: int,
                      selected: list, block_size: int, scale: float):
    """Causal softmax attention of every query token over its query block's
    selected key blocks: token t of block i, head g attends the keys s of the
    blocks in selected[i] with s <= t (Agent Skill page, Step 4's masked
    softmax, with the causal mask of a prefill).  Returns (out [L][G][D],
    lse [L][G])."""
    L = int(seqlen)
    G, D = Q_group.shape[1], V.shape[1]
    out = np.zeros((L, G, D), dtype=np.float64)
    lse = np.full((L, G), -np.inf, dtype=np.float64)
    for i, blocks in enumerate(selected):
        for t in range(i * block_size, min((i + 1) * block_size, L)):
            out[t], lse[t] = prefill_attention_token(Q_group, K, V, L, t, blocks, block_size,
                                                     scale)
    return out, lse


def prefill_attention_token(Q_group: np.ndarray, K: np.ndarray, V: np.ndarray, seqlen: int,
                            t: int, blocks, block_size: int, scale: float):
    """One query token t of ``prefill_attention``: its G heads attend the keys
    s <= t of the given blocks.  Returns (out [G][D], lse [G])."""
    L = int(seqlen)
    keep = np.zeros(L, dtype=bool)
    for j in blocks:
        keep[int(j) * block_size:min((int(j) + 1) * block_size, L)] = True
    keep[t + 1:] = False
    keys = np.nonzero(keep)[0]
    x = (Q_group[t] @ K[keys].T) * float(scale)          # [G][n]
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    tot = e.sum(axis=1, keepdims=True)
    return (e / tot) @ V[keys], (m + np.log(tot))[:, 0]


def prefill_row(Q_group, W, K, V, seqlen, block_size, k_of_block, gate_scale, softmax_scale):
    """The prefill path for one (sequence, KV head): pooled keys, gate scores
    of the pooled queries, per-block selection, causal block-sparse attention.
    Returns a dict with kbar, scores, selected, out, lse."""
    kbar = pool_keys(K, seqlen, block_size)
    scores = prefill_gate_scores(Q_group, W, kbar, seqlen, block_size, gate_scale)
    selected = prefill_select(scores, k_of_block)
    out, lse = prefill_attention(Q_group, K, V, seqlen, selected, block_size, softmax_scale)
    return {"kbar": kbar, "scores": scores, "selected": selected, "out": out, "lse": lse}

