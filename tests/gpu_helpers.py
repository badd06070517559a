"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding and compare with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

from oracle import sla2_oracle as O

SCORE_TIE = 1e-6          # oracle-logit gap under which two blocks may swap in the mask
REL_L2_Q = 2e-2           # quantised output vs the quantisation-emulating oracle
MAX_ABS_Q = 5e-2
REL_L2_U = 1e-3           # unquantised fp32 output vs the exact oracle


def to_dev(inp):
    return {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "proj_q", "proj_k", "alpha")}


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def head_np(inp, b, h):
    f = lambda t: t[b, h].double().numpy()
    return (f(inp.q), f(inp.k), f(inp.v), inp.proj_q[h].double().numpy(), inp.proj_k[h].double().numpy(),
            inp.alpha[h].double().numpy())


def check_mask_rows(gpu_mask, ref_mask, ref_scores, k):
    """Rows must agree except for swaps of blocks whose oracle logits lie
    within SCORE_TIE of the row's k-th largest logit. Returns the set of rows
    that differ (all of them near-ties)."""
    gpu_mask = np.asarray(gpu_mask)
    ref_mask = np.asarray(ref_mask)
    assert gpu_mask.shape == ref_mask.shape
    assert (gpu_mask.sum(axis=-1) == k).all(), "every row keeps exactly k blocks"
    bad = np.argwhere((gpu_mask != ref_mask).any(axis=-1))
    rows = set()
    for r in bad:
        r = tuple(r)
        s = ref_scores[r]
        kth = np.sort(s)[::-1][k - 1]
        diff = np.nonzero(gpu_mask[r] != ref_mask[r])[0]
        gap = np.max(np.abs(s[diff] - kth))
        assert gap < SCORE_TIE, f"mask row {r} differs beyond the near-tie rule (gap {gap:.3e})"
        rows.add(r)
    return rows
