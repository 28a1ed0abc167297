"""Shared helpers of the GPU parity tests: run the library on a workload and
compare with the fp64 oracle under the acceptance rules.

Acceptance (bf16 inputs, fp32 accumulation): kept-channel indices and the
thinner key cache bit-exact; decode output max-abs <= 2e-3 and relative L2
<= 1e-3. fp32 inputs: max-abs <= 1e-5 and relative L2 <= 1e-6.  The fp32
decode converts its exact fp32 inputs to fp64 and carries every later step
(logits, exponentials, running sums, split merge) in fp64, so the error that
reaches the output is the final rounding to fp32 (relative 2^-24 = 6e-8 per
element) plus fp64 rounding (~1e-15): 1e-6 leaves a margin of more than 10x.
Index lists may
differ only at a near-tie: every channel in which they differ must have an
oracle score within 1e-6 relative of the cut (the T-th largest score).

Scores: bf16 keys are squared exactly and summed four rows at a time in fp32
(three roundings, relative error below 3 * 2^-24 = 1.8e-7 per partial, and so
for the channel energy, which is a sum of non-negative partials), then in
fp64; the square root halves that.  The scores are checked within 1e-6
relative, and two channels whose oracle scores differ by more than
2 * 1.8e-7 relative keep their order, which the near-tie rule covers.  fp32
keys are squared exactly in fp64 (checked within 1e-12).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: (2e-3, 1e-3), torch.float32: (1e-5, 1e-6)}
NEAR_TIE_REL = 1e-6


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


SCORE_RTOL = {torch.bfloat16: 1e-6, torch.float32: 1e-12}


def check_scores(gpu_scores: torch.Tensor, ora_scores: np.ndarray, rtol: float | None = None,
                 dtype: torch.dtype = torch.bfloat16):
    g = f64(gpu_scores)
    np.testing.assert_allclose(g, ora_scores, rtol=SCORE_RTOL[dtype] if rtol is None else rtol, atol=0)


def idx_mismatch_heads(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, T: int):
    """Return the list of (b, h) whose index lists differ; assert every difference
    is a near-tie at the cut and that the GPU list is a valid ascending set."""
    bad = []
    B, H, _ = ora_idx.shape
    for b in range(B):
        for h in range(H):
            gi = gpu_idx[b, h]
            assert np.all(np.diff(gi) > 0), f"idx not strictly ascending at {(b, h)}: {gi}"
            assert gi.min() >= 0 and gi.max() < ora_scores.shape[-1]
            if np.array_equal(gi, ora_idx[b, h]):
                continue
            s = ora_scores[b, h]
            cut = np.sort(s)[::-1][T - 1]
            diff = np.setxor1d(gi, ora_idx[b, h])
            for c in diff:
                assert abs(s[c] - cut) <= NEAR_TIE_REL * abs(cut), (
                    f"head {(b, h)}: channel {c} score {s[c]!r} is not a near-tie of cut {cut!r}")
            bad.append((b, h))
    return bad


def check_out(gpu_out: torch.Tensor, ora_out: np.ndarray, dtype, where: str = ""):
    g = f64(gpu_out)
    max_abs_tol, rel_l2_tol = TOL[dtype]
    err = np.abs(g - ora_out)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(g - ora_out) / max(np.linalg.norm(ora_out), 1e-300))
    assert np.all(np.isfinite(g)), f"{where}: non-finite output"
    assert max_abs <= max_abs_tol and rel_l2 <= rel_l2_tol, (
        f"{where}: max_abs {max_abs:.3e} (tol {max_abs_tol}) rel_l2 {rel_l2:.3e} (tol {rel_l2_tol})")
    return max_abs, rel_l2


def kp_logical(k_pruned: torch.Tensor, N: int) -> np.ndarray:
    """Thinner cache buffer [B,Hkv,T,ldk] -> K'[B,Hkv,N,T] values (fp64)."""
    return f64(k_pruned[..., :N].transpose(-1, -2))


# Width decisions: GPU scores are within 1e-6 relative of the oracle's, so
# each squared score within 2e-6, and so every cumulative energy and the total
# (sums of non-negative terms): a width may differ only where the oracle's
# cumulative energy is within about 4e-6 of tau * E; the window is 1e-5.
ADAPTIVE_ENERGY_REL = 1e-5


def width_is_near_tie(s, tau, T_min, T_max, k_gpu, k_ora):
    """Whether two widths of one head can both follow from scores within the
    score tolerance of the oracle's: the oracle's cumulative squared-score
    energy (rank order) must lie within ADAPTIVE_ENERGY_REL of tau * E at every
    width from the smaller choice up to (not including) the larger one, so that
    the cut could fall on either side."""
    order = sorted(range(len(s)), key=lambda c: (-s[c], c))
    e = np.array([s[c] * s[c] for c in order])
    cum = np.cumsum(e)
    E = cum[-1]
    lo, hi = min(k_gpu, k_ora), max(k_gpu, k_ora)
    if lo < T_min or hi > T_max:
        return False
    return all(abs(cum[k - 1] - tau * E) <= ADAPTIVE_ENERGY_REL * tau * E for k in range(lo, hi))
