"""Parity of the 3-D point path on the GPU (needs a B200): exact Euclidean NN,
the reciprocal set and FRM on point maps, against the double-precision oracle
(its Euclidean metric at d = 3, pinned to scipy's K-d tree in test_oracle).

Coordinates that are multiples of 1/64 inside [-16, 16] make every fp32
squared distance exact, so those cases compare bit for bit, ties included.
Continuous coordinates use a relative rule: a returned index may differ from
the oracle's only where the oracle's best and second squared distances are
within REL of each other, and every returned squared distance is within REL
of the oracle's best.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import seed_state_np

pytestmark = pytest.mark.gpu

REL = 2e-6


def _cuda32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _check_rel(Q, X, idx, d2, ref):
    best = -ref.best
    second = -ref.second
    diff = np.nonzero(idx != ref.arg)[0]
    gap = second - best
    assert np.all(gap[diff] <= REL * np.maximum(best[diff], 1e-30)), diff[:10]
    if len(diff):
        got = ((Q[diff] - X[idx[diff]]) ** 2).sum(axis=1)
        assert np.all(got <= best[diff] * (1 + REL) + 1e-30)
    assert np.all(np.abs(d2 - best) <= REL * np.maximum(best, 1e-30) + 1e-30)
    return len(diff)


# ----------------------------------------------------------------- NN queries

@pytest.mark.parametrize("nq,nx", [(1, 1), (100, 1), (1, 100), (1000, 2000), (5000, 20000),
                                   (777, 4097)])
def test_pts_nn_quantised_bitexact(nq, nx):
    rng = np.random.default_rng(nq + 7 * nx)
    X = synth.quantised_points(rng, nx, repeat=0.1)
    Q = synth.quantised_points(rng, nq)
    if nq > 10 and nx > 10:
        Q[:10] = X[:10]                                   # queries on data points
    idx, d2 = rnn.pts_nn(_cuda32(Q), _cuda32(X))
    ref = oracle.nn(Q.astype(np.float32), X.astype(np.float32), metric="l2")
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(d2.cpu().numpy().astype(np.float64), -ref.best)


def test_pts_nn_queries_outside_the_box():
    rng = np.random.default_rng(8)
    X = synth.quantised_points(rng, 3000, clusters=2, spread=0.5)
    X = np.clip(X, -4, 4)
    Q = np.round(rng.uniform(-20, 20, size=(2000, 3)) * 64) / 64
    idx, d2 = rnn.pts_nn(_cuda32(Q), _cuda32(X))
    ref = oracle.nn(Q, X, metric="l2")
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(d2.cpu().numpy().astype(np.float64), -ref.best)


@pytest.mark.parametrize("shape", ["same", "line", "plane", "two"])
def test_pts_nn_degenerate_sets(shape):
    rng = np.random.default_rng(9)
    n = 1500
    if shape == "same":
        X = np.tile([[1.5, -2.0, 3.25]], (n, 1))
    elif shape == "line":
        t = np.round(rng.uniform(-10, 10, n) * 64) / 64
        X = np.stack([t, 0.5 * np.ones(n), -t], axis=1)
    elif shape == "plane":
        X = np.round(rng.uniform(-10, 10, (n, 3)) * 64) / 64
        X[:, 2] = 2.0
    else:                                                  # two far clusters
        X = synth.quantised_points(rng, n, clusters=1, spread=0.2)
        X[n // 2:] = np.clip(X[n // 2:] + 14, -16, 16)
        X[: n // 2] = np.clip(X[: n // 2] - 1, -16, 16)
    Q = synth.quantised_points(rng, 700)
    idx, d2 = rnn.pts_nn(_cuda32(Q), _cuda32(X))
    ref = oracle.nn(Q, X, metric="l2")
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(d2.cpu().numpy().astype(np.float64), -ref.best)


def test_pts_nn_no_queries():
    X = _cuda32(np.zeros((5, 3)))
    idx, d2 = rnn.pts_nn(_cuda32(np.zeros((0, 3))), X)
    assert idx.numel() == 0 and d2.numel() == 0


def test_pts_nn_continuous_relative():
    rng = np.random.default_rng(10)
    X = (rng.standard_normal((30000, 3)) * np.array([4.0, 3.0, 0.5])).astype(np.float32)
    Q = (rng.standard_normal((5000, 3)) * 5.0).astype(np.float32)
    Q[:20] *= 100.0                                        # far queries
    idx, d2 = rnn.pts_nn(_cuda32(Q), _cuda32(X))
    ref = oracle.nn(Q, X, metric="l2")
    n = _check_rel(Q.astype(np.float64), X.astype(np.float64), idx.cpu().numpy(),
                   d2.cpu().numpy().astype(np.float64), ref)
    assert n <= 2


# ------------------------------------------------------------ reciprocal set

@pytest.mark.parametrize("s1,s2", [((32, 40), (32, 40)), ((37, 41), (29, 53)), ((1, 1), (3, 5))])
def test_pts_mnn_quantised_bitexact(s1, s2):
    P1, _ = synth.pointmap_pair(70 + s1[0], *s1, quantised=True)
    _, P2 = synth.pointmap_pair(71 + s2[0], *s2, quantised=True)
    r = rnn.pts_mnn(_cuda32(P1), _cuda32(P2), with_nn=True)
    ref = oracle.mnn(P1, P2, metric="l2")
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.rowmax.cpu().numpy().astype(np.float64), -ref.row.best)
    assert np.array_equal(r.colmax.cpu().numpy().astype(np.float64), -ref.col.best)


def test_pts_mnn_full_size_sampled():
    """384x512 point maps (the size of the descriptor workloads): NN of a
    sample of pixels in both directions, and the mutual pairs among them."""
    P1, P2 = synth.pointmap_pair(80, 384, 512)
    A, B = P1.reshape(-1, 3).astype(np.float32), P2.reshape(-1, 3).astype(np.float32)
    r = rnn.pts_mnn(_cuda32(P1), _cuda32(P2), with_nn=True)
    rowarg, colarg = r.rowarg.cpu().numpy(), r.colarg.cpu().numpy()
    rng = np.random.default_rng(81)
    si = rng.choice(len(A), 3000, replace=False)
    sj = rng.choice(len(B), 3000, replace=False)
    ref_r = oracle.nn(A[si], B, metric="l2")
    ref_c = oracle.nn(B[sj], A, metric="l2")
    _check_rel(A[si].astype(np.float64), B.astype(np.float64), rowarg[si],
               r.rowmax.cpu().numpy()[si].astype(np.float64), ref_r)
    _check_rel(B[sj].astype(np.float64), A.astype(np.float64), colarg[sj],
               r.colmax.cpu().numpy()[sj].astype(np.float64), ref_c)
    pairs = r.trimmed().cpu().numpy()
    assert np.all(np.diff(pairs[:, 0]) > 0)
    assert np.array_equal(colarg[pairs[:, 1]], pairs[:, 0])
    assert np.array_equal(rowarg[pairs[:, 0]], pairs[:, 1])
    assert len(pairs) == int(np.sum(colarg[rowarg] == np.arange(len(A))))


# ---------------------------------------------------------------------- FRM

@pytest.mark.parametrize("S,max_iter", [(4, 10), (2, 3), (1, 10), (3, 1)])
def test_pts_frm_quantised_bitexact(S, max_iter):
    P1, P2 = synth.pointmap_pair(90 + S, 40, 56, quantised=True)
    r = rnn.pts_frm_match(_cuda32(P1), _cuda32(P2), seed_stride=S, max_iter=max_iter,
                          with_seed_state=True)
    ref = oracle.frm_ex(P1, P2, S, max_iter, metric="l2")
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    u, v, q, c = seed_state_np(r)
    assert np.array_equal(u, ref.seed_u) and np.array_equal(v, ref.seed_v)
    assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)


def test_pts_frm_batched_starts_tol_basin():
    B, H, W = 3, 24, 36
    maps = [synth.pointmap_pair(100 + b, H, W, quantised=True) for b in range(B)]
    a = np.stack([m[0] for m in maps])
    b = np.stack([m[1] for m in maps])
    rng = np.random.default_rng(101)
    starts = rng.integers(0, H * W, size=(B, 150)).astype(np.int32)
    starts[:, 3] = starts[:, 0]
    r = rnn.pts_frm_match(_cuda32(a), _cuda32(b), max_iter=1, pixel_tol=2.0,
                          init=torch.from_numpy(starts).cuda(), with_seed_state=True)
    for i in range(B):
        ref = oracle.frm_refine(a[i], b[i], starts[i], pixel_tol=2.0, metric="l2")
        got = r.pairs[i, : int(r.count[i])].cpu().numpy()
        assert np.array_equal(got, ref.pairs.reshape(-1, 2)), i
    rb = rnn.pts_frm_match(_cuda32(a), _cuda32(b), seed_stride=2, max_iter=5, with_basin=True)
    for i in range(B):
        ref = oracle.frm_ex(a[i], b[i], 2, 5, basin=True, metric="l2")
        assert np.array_equal(rb.pairs[i, : int(rb.count[i])].cpu().numpy(),
                              ref.pairs.reshape(-1, 2)), i
        assert np.array_equal(rb.basin[i].cpu().numpy(), ref.basin), i


def test_pts_frm_continuous_matches_oracle():
    P1, P2 = synth.pointmap_pair(110, 96, 128, noise=0.01)
    r = rnn.pts_frm_match(_cuda32(P1), _cuda32(P2), seed_stride=4, max_iter=10)
    ref = oracle.frm_ex(P1.astype(np.float32), P2.astype(np.float32), 4, 10, metric="l2")
    got = {tuple(p) for p in r.trimmed().cpu().numpy().tolist()}
    exp = {tuple(p) for p in ref.pairs.tolist()}
    # continuous coordinates: an fp32 near-tie could flip a trajectory, so a
    # handful of pairs out of the whole set may differ
    assert len(got ^ exp) <= max(2, len(exp) // 200)
    assert len(exp) > 100


def test_pts_frm_starts_out_of_image_are_dropped():
    H, W = 20, 30
    P1, P2 = synth.pointmap_pair(120, H, W, quantised=True)
    rng = np.random.default_rng(121)
    good = rng.integers(0, H * W, 80).astype(np.int32)
    starts = np.concatenate([good, np.array([-1, H * W, H * W + 9, -50], np.int32)])
    r = rnn.pts_frm_match(_cuda32(P1), _cuda32(P2), max_iter=1, pixel_tol=1.5,
                          init=torch.from_numpy(starts).cuda())
    ref = oracle.frm_refine(P1, P2, good, pixel_tol=1.5, metric="l2")
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))
