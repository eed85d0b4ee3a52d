"""Shared helpers of the GPU parity tests: copying seeded inputs to the host
as float64 for the oracle, and the comparison measures with their bounds."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_step_b200 import workloads as W

# Output tolerance of the step against the fp64 oracle (max-abs, rel-L2).
TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 1e-2
# Gate scores closer than this (fp64 margin at the k/k+1 boundary) may
# legitimately select differently in fp32; such rows get a validity check.
MARGIN = 1e-4


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_attention_step_b200 import seer
    seer.library()  # raises if the library is missing: no fallback
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip(f"built for sm_100a, device is sm_{major}{minor}")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def row_inputs(w, data, b, h):
    """(q_group [G][D], W [D][D], K [L][D], V [L][D], L) as float64 on the host."""
    L = int(data["seqlens"][b].item())
    G = w.group
    q = f64(data["q"][b, h * G:(h + 1) * G])
    Wg = f64(data["w_gate"][h])
    K = f64(W.gather_rows(data["k_pool"], data["page_table"], b, h, L, w.block_size, data.get("layout", "nhd")))
    V = f64(W.gather_rows(data["v_pool"], data["page_table"], b, h, L, w.block_size, data.get("layout", "nhd")))
    return q, Wg, K, V, L


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x|: the rounding every bf16
    output carries whatever the kernel computed."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def out_errors(got: np.ndarray, ref: np.ndarray):
    """(max-abs, rel-L2, plain max-abs) of a bf16 output against the fp64
    oracle.  The first max-abs is taken over the error beyond the output's
    own bf16 rounding (|got - ref| - half an ulp of ref); below |ref| = 4
    that allowance is at most 2^-7, so for unit-scale outputs this is the
    plain max-abs bound.  The plain max-abs |got - ref| is reported beside
    it."""
    err = got - ref
    excess = np.abs(err) - bf16_half_ulp(ref)
    max_abs = float(excess.max()) if err.size else 0.0
    plain = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    return max_abs, rel, plain


def assert_out_close(got, ref, what=""):
    """The bf16 output bound: max-abs beyond the bf16 rounding <= 2e-2 and
    rel-L2 <= 1e-2.  For bf16 outputs only."""
    max_abs, rel, plain = out_errors(got, ref)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, (what, max_abs, rel, plain)
    return max_abs, rel, plain


# fp32 results (split partials): no output rounding to allow for.  The
# kernel's own error: q.K products of bf16 values are exact in fp32 and 128 of
# them add with relative error <= 128 * 2^-24 of the sum of |products|; the
# softmax weights reach the P.V product as a bf16 hi + lo pair (about 2^-16
# relative); V is exact; accumulators are fp32.  A weight error e moves the
# output by at most e * max|V| over the attended rows, so the bound scales
# with that magnitude (1 for unit-variance data, larger for heavy-tailed).
TOL_F32_MAX_ABS = 1e-3
TOL_F32_REL_L2 = 1e-4


def f32_errors(got: np.ndarray, ref: np.ndarray):
    """(plain max-abs, rel-L2) of an fp32 result against the fp64 oracle."""
    err = np.asarray(got, dtype=np.float64) - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def assert_f32_close(got, ref, v_scale=1.0, what=""):
    """The fp32 bound: plain max-abs <= 1e-3 * max(1, v_scale) (v_scale =
    the largest |V| entry the result averages) and rel-L2 <= 1e-4."""
    max_abs, rel = f32_errors(got, ref)
    bound = TOL_F32_MAX_ABS * max(1.0, float(v_scale))
    assert max_abs <= bound and rel <= TOL_F32_REL_L2, (what, max_abs, bound, rel)
    return max_abs, rel


def scale_of(w):
    return 1.0 / math.sqrt(w.head_dim)
