"""Comparison helpers shared by the GPU parity tests (no method arithmetic here).

Tolerances (bf16 inputs, fp32 accumulation), each set by the arithmetic of what it checks:
  pooled K/V    an fp32 sum then one rounding to bf16, so within 1 bf16 ulp of the correctly
                rounded mean (the fp32 sum may move a value across a rounding boundary),
                >= 99.9 % bit-identical
  lse           fp32 exp2 sums and one log: |d| <= 2e-5 absolute (natural-log units)
  scores        fp32 sums of fp32 probabilities: |d| <= 1e-5 * (largest score of the row) + 1e-9
  o_cmp, o_sel  P is rounded to bf16 for the P V product (2^-9 relative per term):
                |d| <= 2^-8 * max|V| + 1e-6 elementwise, relative L2 <= 4e-3
  combine       one rounding of the fp32 result to bf16: |d| <= 1 bf16 ulp + 1e-7
  whole path    indices equal where the oracle's k-th/(k+1)-th score gap > 1e-4 (fp32 scores
                cannot order closer ties the way fp64 does); every selected block within
                tau = 1e-6 * max(1, S_(k)) of the k-th best oracle score; output against the
                oracle run on the GPU's indices: max-abs <= 2e-2, rel-L2 <= 5e-3 (the bf16 output
                rounding plus the branch errors above)
"""
from __future__ import annotations

import numpy as np
import torch

GAP_EXACT = 1e-4
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1e-300)))
    return np.where(ax > 0, np.exp2(np.maximum(e, -126) - 7), 2.0 ** -133)


def check_pooled(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Returns the exact fraction; asserts the 1-ulp bound."""
    diff = np.abs(gpu - ref)
    assert np.all(diff <= bf16_ulp(ref) * (1 + 1e-9)), float(diff.max())
    return float(np.mean(diff == 0))


def check_close(name, gpu, ref, atol, rl2=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    assert float(err.max()) <= atol, f"{name}: max-abs {err.max():.3e} > {atol:.3e}"
    if rl2 is not None:
        r = rel_l2(gpu, ref)
        assert r <= rl2, f"{name}: rel-L2 {r:.3e} > {rl2:.3e}"


# backward: g*P and dS are rounded to bf16 for the tensor-core products (2^-9 relative per term)
# and D = g <dout, O> comes from the fp32 forward outputs (about 2^-8 of |V|); both enter each
# gradient at about 2^-8 relative. The absolute floor covers gradients that are exactly zero
# (a single key: P = 1, dS = 0), where fp32 leaves a residue of about 2^-24 |dP|.
GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2
GRAD_ABS_FLOOR = 1e-6


def check_grad(name, got, ref):
    """A gradient against the oracle's: max-abs <= 2e-2 max|ref| + 1e-6, rel-L2 <= 1e-2."""
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    scale = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    bound = GRAD_MAX_REL * scale + GRAD_ABS_FLOOR
    assert err <= bound, f"{name}: max-abs {err:.3e} > {bound:.3e}"
    if scale > 0:
        r = rel_l2(got, ref)
        assert r <= GRAD_REL_L2, f"{name}: rel-L2 {r:.3e}"


def check_selection(gpu_idx: np.ndarray, ref_idx: np.ndarray, gap: np.ndarray,
                    scores: np.ndarray, k: int, forced: int = 0) -> dict:
    """Index parity of one selection [H, nq, forced + k] against the oracle.

    The forced blocks 0 .. forced-1 must open every list. Of the rest (the top-k among blocks
    forced .. nb-1): where the oracle's gap exceeds GAP_EXACT the sets must be equal; everywhere,
    every selected block must be score-optimal within tau of the oracle's k-th best score."""
    if forced:
        assert (gpu_idx[..., :forced] == np.arange(forced)).all(), "forced blocks missing"
        assert (ref_idx[..., :forced] == np.arange(forced)).all()
        gpu_idx, ref_idx = gpu_idx[..., forced:] - forced, ref_idx[..., forced:] - forced
        scores = scores[..., forced:]
    gs = np.sort(gpu_idx, -1)
    rs = np.sort(ref_idx, -1)
    sep = gap > GAP_EXACT
    assert np.array_equal(gs[sep], rs[sep]), "index sets differ on gap-separated query blocks"
    nb = scores.shape[-1]
    assert gpu_idx.min() >= 0 and gpu_idx.max() < nb
    assert all(len(set(r)) == k for r in gpu_idx.reshape(-1, k).tolist()), "duplicate indices"
    kth = np.sort(scores, -1)[..., nb - k]
    tau = 1e-6 * np.maximum(1.0, kth)
    got = np.take_along_axis(scores, gpu_idx.astype(np.int64), -1)
    worst = float((got - (kth - tau)[..., None]).min())
    assert worst >= 0, f"a selected block is not score-optimal (short by {-worst:.3e})"
    return {"gap_separated": float(sep.mean()),
            "sets_equal": float(np.mean(np.all(gs == rs, -1)))}


def check_output(gpu_out: np.ndarray, ref_out: np.ndarray) -> dict:
    err = np.abs(gpu_out - ref_out)
    r = rel_l2(gpu_out, ref_out)
    assert float(err.max()) <= OUT_MAX_ABS, f"max-abs {err.max():.3e}"
    assert r <= OUT_REL_L2, f"rel-L2 {r:.3e}"
    return {"max_abs": float(err.max()), "rel_l2": r}
