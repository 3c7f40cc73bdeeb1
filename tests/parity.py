"""Comparison helpers between the CUDA path and the oracle.

Quantised inputs (values k/64) make every fp32 dot product exact, so there the
comparison is bit-for-bit.  On unit-norm fp16 inputs the tensor cores sum in
fp32 in their own order; the rule is: a returned index may differ from the
oracle's only where the oracle's top-2 score gap is below TOL, the oracle
score of the returned index must then be within TOL of the oracle's best, and
every returned score must be within TOL of the oracle's best.
"""
import numpy as np
import torch

import oracle

TOL = 1e-3


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().cuda()


def check_nn_tolerant(Q, X, idx, score, ref: "oracle.NNResult", tol=TOL):
    """Apply the tolerance rule to a GPU NN result; returns the mismatch count."""
    idx = np.asarray(idx)
    score = np.asarray(score, dtype=np.float64)
    diff = np.nonzero(idx != ref.arg)[0]
    assert np.all(ref.gap[diff] < tol), "index differs where the oracle gap is >= tol"
    if len(diff):
        s = oracle.pair_scores(Q, X, diff.astype(np.int32), idx[diff])
        assert np.all(s >= ref.best[diff] - tol)
    assert np.all(np.abs(score - ref.best) <= tol)
    return len(diff)


def check_mnn_tolerant(gpu_pairs, ref: "oracle.MNNResult", tol=TOL):
    g = {tuple(p) for p in np.asarray(gpu_pairs).tolist()}
    o = {tuple(p) for p in ref.pairs.tolist()}
    for (i, j) in g ^ o:
        assert ref.row.gap[i] < tol or ref.col.gap[j] < tol, (i, j)
    return len(g ^ o)


def seed_state_np(res, b=0):
    st = res.seed_state[b].cpu().numpy()
    return st[:, 0], st[:, 1], st[:, 2], st[:, 3].astype(bool)


def pairs_from_seeds(u, v, conv):
    return sorted({(int(a), int(b)) for a, b, c in zip(u, v, conv) if c})
