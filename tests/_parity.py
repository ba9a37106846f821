"""Host-side comparison of the CUDA path against the oracle.

Acceptance (the block's stated tolerances):
  * expert indices identical, except on tokens whose oracle fp32 logits have a
    gap below 1e-4 between the k-th and the (k+1)-th largest -- those tokens are
    excluded from the index AND the output checks, and counted;
  * max |y - y_ref| <= 2e-2 * max |y_ref|;
  * mean relative error, read as sum|y - y_ref| / sum|y_ref| over the kept
    tokens, <= 5e-3.
Where several indices are correct (excluded tokens) the chosen set is still
checked for validity: k distinct experts in range.
"""
from __future__ import annotations

import numpy as np

GAP = 1e-4
MAX_REL = 2e-2
MEAN_REL = 5e-3


def excluded_tokens(logits: np.ndarray, k: int) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest logits are closer than GAP."""
    T, E = logits.shape
    if k >= E:
        return np.zeros(T, dtype=bool)
    s = -np.sort(-logits.astype(np.float64), axis=1)
    return (s[:, k - 1] - s[:, k]) < GAP


def compare_block(y_gpu: np.ndarray, idx_gpu: np.ndarray, w_gpu: np.ndarray, ref: dict, k: int,
                  E: int) -> dict:
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = ref["y"]
    excl = excluded_tokens(ref["logits"], k)
    keep = ~excl
    # validity of every chosen set
    assert idx_gpu.shape == ref["idx"].shape
    assert np.all((idx_gpu >= 0) & (idx_gpu < E)), "expert index out of range"
    for t in range(idx_gpu.shape[0]):
        assert len(set(idx_gpu[t].tolist())) == k, "repeated expert for token %d" % t
    idx_mismatch = int(np.sum(np.any(idx_gpu[keep] != ref["idx"][keep], axis=1)))
    w_err = float(np.max(np.abs(w_gpu[keep] - ref["w"][keep]))) if keep.any() else 0.0
    if keep.any():
        diff = np.abs(y_gpu[keep] - y_ref[keep])
        max_rel = float(diff.max() / max(np.abs(y_ref[keep]).max(), 1e-30))
        mean_rel = float(diff.sum() / max(np.abs(y_ref[keep]).sum(), 1e-30))
    else:
        max_rel = mean_rel = 0.0
    return dict(n_tokens=int(y_gpu.shape[0]), n_excluded=int(excl.sum()), idx_mismatch=idx_mismatch,
                w_max_err=w_err, max_rel=max_rel, mean_rel=mean_rel,
                ok=(idx_mismatch == 0 and max_rel <= MAX_REL and mean_rel <= MEAN_REL))
