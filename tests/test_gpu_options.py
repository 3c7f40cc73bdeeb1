"""Parity of the quoted matcher's other options on the GPU (needs a B200):
the Euclidean metric, FRM from given start pixels with the pixel tolerance,
and the basin output, against the double-precision oracle.

Quantised inputs (values k/64) keep every augmented score exact, so they are
compared bit for bit (squared distances included).  Unit-norm fp16 inputs
use the tolerance rule in squared-distance units: |a-b|^2 = 2 - 2 a.b there,
so the dot rule's 1e-3 becomes 2e-3.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import dev, seed_state_np

pytestmark = pytest.mark.gpu

TOL_L2 = 2e-3


def _q(seed, n, d):
    rng = np.random.default_rng(seed)
    return synth.quantised_map(rng, 1, n, d).reshape(n, d)


def _neg_sqdist(A, B, ia, ib):
    a = oracle.as_f64(A).reshape(-1, A.shape[-1])[ia]
    b = oracle.as_f64(B).reshape(-1, B.shape[-1])[ib]
    return -((a - b) ** 2).sum(axis=1)


# ------------------------------------------------------------ Euclidean metric

@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("nq,nx,d", [(1, 1, 8), (300, 700, 16), (1000, 1537, 24),
                                     (130, 5000, 32), (200, 700, 256)])
def test_nn_l2_quantised_bitexact(dt, nq, nx, d):
    Q = synth.to_storage(_q(1 + d, nq, d), dt)
    X = synth.to_storage(_q(2 + d, nx, d), dt)
    idx, score = rnn.nn_argmax(dev(Q), dev(X), metric="l2")
    ref = oracle.nn(Q, X, metric="l2")
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    # the squared distance of the chosen neighbour, exact
    assert np.array_equal(score.cpu().numpy().astype(np.float64), -ref.best)


def test_nn_l2_unit_fp16_tolerance():
    D1, D2 = synth.smooth_pair(31, 40, 50, 24)
    Q = synth.to_storage(D1.reshape(-1, 24), "f16")
    X = synth.to_storage(D2.reshape(-1, 24), "f16")
    idx, score = rnn.nn_argmax(dev(Q), dev(X), metric="l2")
    idx, score = idx.cpu().numpy(), score.cpu().numpy().astype(np.float64)
    ref = oracle.nn(Q, X, metric="l2")
    diff = np.nonzero(idx != ref.arg)[0]
    assert np.all(ref.gap[diff] < TOL_L2)
    assert np.all(_neg_sqdist(Q, X, diff, idx[diff]) >= ref.best[diff] - TOL_L2)
    assert np.all(np.abs(-score - ref.best) <= TOL_L2)


@pytest.mark.parametrize("s1,s2,d", [((32, 32), (32, 32), 16), ((37, 41), (29, 53), 24),
                                     ((20, 30), (25, 21), 32), ((9, 7), (11, 5), 8),
                                     ((31, 33), (27, 35), 56), ((24, 26), (22, 28), 64)])
def test_mnn_l2_quantised_bitexact(s1, s2, d):
    """Under the Euclidean metric d <= 56 runs the one-pass kernel on the
    symmetric forms (-|q - x|^2/2 for every pair), d = 64 the two sweeps."""
    rng = np.random.default_rng(5 + d)
    D1 = synth.to_storage(synth.quantised_map(rng, *s1, d), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, *s2, d), "f16")
    r = rnn.mnn_exhaustive(dev(D1), dev(D2), with_nn=True, metric="l2")
    ref = oracle.mnn(D1, D2, metric="l2")
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.rowmax.cpu().numpy().astype(np.float64), -ref.row.best)
    assert np.array_equal(r.colmax.cpu().numpy().astype(np.float64), -ref.col.best)


@pytest.mark.parametrize("S,max_iter", [(4, 10), (3, 2)])
def test_frm_l2_quantised_bitexact(S, max_iter):
    rng = np.random.default_rng(40 + S)
    D1 = synth.to_storage(synth.quantised_map(rng, 40, 56, 24), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, 36, 60, 24), "f16")
    r = rnn.frm_match_ex(dev(D1), dev(D2), seed_stride=S, max_iter=max_iter, metric="l2",
                         with_seed_state=True)
    ref = oracle.frm_ex(D1, D2, S, max_iter, metric="l2")
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    u, v, q, c = seed_state_np(r)
    assert np.array_equal(u, ref.seed_u) and np.array_equal(v, ref.seed_v)
    assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)


# ------------------------------------------------------ given starts, pixel_tol

def _starts(rng, n1, n, dup=True):
    s = rng.integers(0, n1, size=n).astype(np.int32)
    if dup:
        s[3] = s[0]
        s[7] = s[1]
    return s


@pytest.mark.parametrize("metric", ["dot", "l2"])
@pytest.mark.parametrize("tol", [0.0, 1.5, 3.0])
def test_refine_batched_quantised_bitexact(metric, tol):
    B, H1, W1, H2, W2, d, n = 3, 24, 40, 28, 36, 24, 200
    rng = np.random.default_rng(61)
    maps = [(synth.quantised_map(rng, H1, W1, d), synth.quantised_map(rng, H2, W2, d))
            for _ in range(B)]
    a = torch.stack([synth.to_storage(m[0], "f16") for m in maps])
    b = torch.stack([synth.to_storage(m[1], "f16") for m in maps])
    starts = np.stack([_starts(rng, H1 * W1, n) for _ in range(B)])
    r = rnn.frm_match_ex(dev(a), dev(b), max_iter=1, metric=metric,
                         init=torch.from_numpy(starts).cuda(), pixel_tol=tol,
                         with_seed_state=True)
    for i in range(B):
        ref = oracle.frm_refine(a[i], b[i], starts[i], pixel_tol=tol, metric=metric)
        got = r.pairs[i, : int(r.count[i])].cpu().numpy()
        assert np.array_equal(got, ref.pairs.reshape(-1, 2)), i
        u, v, q, c = seed_state_np(r, i)
        k = len(ref.seeds)
        assert np.array_equal(u[:k], ref.seed_u) and np.array_equal(v[:k], ref.seed_v)
        assert np.array_equal(q[:k], ref.seed_queries)
        assert np.array_equal(c[:k], ref.seed_converged)
        assert np.all(u[k:] == -1) and np.all(q[k:] == 0) and not c[k:].any()


def test_refine_drops_out_of_image_starts():
    H, W, d = 16, 24, 16
    rng = np.random.default_rng(62)
    D1 = synth.to_storage(synth.quantised_map(rng, H, W, d), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, H, W, d), "f16")
    good = _starts(rng, H * W, 50, dup=False)
    starts = np.concatenate([good, np.array([-1, H * W, H * W + 5, -100], np.int32)])
    r = rnn.frm_refine(dev(D1), dev(D2), torch.from_numpy(starts).cuda(), 2.0)
    ref = oracle.frm_refine(D1, D2, good, pixel_tol=2.0)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))


# ----------------------------------------------------------------- basin mode

@pytest.mark.parametrize("S,max_iter", [(2, 10), (3, 2), (1, 10)])
def test_basin_batched_quantised_bitexact(S, max_iter):
    B, H, W, d = 2, 20, 28, 16
    rng = np.random.default_rng(70 + S)
    maps = [(synth.quantised_map(rng, H, W, d), synth.quantised_map(rng, H, W, d))
            for _ in range(B)]
    a = torch.stack([synth.to_storage(m[0], "f16") for m in maps])
    b = torch.stack([synth.to_storage(m[1], "f16") for m in maps])
    r = rnn.frm_match_ex(dev(a), dev(b), seed_stride=S, max_iter=max_iter, with_basin=True,
                         with_seed_state=True)
    for i in range(B):
        ref = oracle.frm_ex(a[i], b[i], S, max_iter, basin=True)
        assert np.array_equal(r.pairs[i, : int(r.count[i])].cpu().numpy(),
                              ref.pairs.reshape(-1, 2)), i
        assert np.array_equal(r.basin[i].cpu().numpy(), ref.basin), i
        _, _, q, c = seed_state_np(r, i)
        assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)


# ------------------------------------------------- hand-worked cases, on the GPU

def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _pad8(x):
    x = np.asarray(x, np.float64)
    out = np.zeros(x.shape[:-1] + (8,), np.float64)
    out[..., : x.shape[-1]] = x
    return out


def test_golden_nn_l2_ties_on_gpu(golden_dir):
    g = _golden(golden_dir, "nn_l2_ties.json")
    Q = synth.to_storage(_pad8(g["Q"]), "f16")
    X = synth.to_storage(_pad8(g["X"]), "f16")
    assert rnn.nn_argmax(dev(Q), dev(X), metric="l2")[0].cpu().tolist() == g["l2_arg"]
    assert rnn.nn_argmax(dev(Q), dev(X))[0].cpu().tolist() == g["dot_arg"]


@pytest.mark.parametrize("case", range(5))
def test_golden_refine_on_gpu(golden_dir, case):
    g = _golden(golden_dir, "frm_refine_1x3_1x2.json")
    c = g["cases"][case]
    D1 = synth.to_storage(_pad8(g["D1"]).reshape(g["H1"], g["W1"], 8), "f16")
    D2 = synth.to_storage(_pad8(g["D2"]).reshape(g["H2"], g["W2"], 8), "f16")
    init = torch.tensor(g["init"], dtype=torch.int32, device="cuda")
    r = rnn.frm_refine(dev(D1), dev(D2), init, c["pixel_tol"], metric=c["metric"])
    assert r.trimmed().cpu().tolist() == c["pairs"]


@pytest.mark.parametrize("case", range(5))
def test_golden_basin_on_gpu(golden_dir, case):
    g = _golden(golden_dir, "frm_basin_chain_2x2_1x4.json")
    c = g["cases"][case]
    S = np.array(g["scores"], np.float64)
    D1 = synth.to_storage(_pad8(S).reshape(g["H1"], g["W1"], 8), "f16")
    D2 = synth.to_storage(_pad8(np.eye(g["d"])).reshape(g["H2"], g["W2"], 8), "f16")
    r = rnn.frm_match_ex(dev(D1), dev(D2), seed_stride=c["stride"], max_iter=c["max_iter"],
                         with_basin=True, with_seed_state=True)
    assert r.trimmed().cpu().tolist() == c["pairs"]
    assert r.basin[0].cpu().tolist() == c["basin"]
    if "seed_queries" in c:
        assert seed_state_np(r)[2].tolist() == c["seed_queries"]


# ------------------------------------------ reciprocal set from NN arrays

def test_mnn_mutual_matches_numpy():
    rng = np.random.default_rng(90)
    n1, n2 = 20000, 13001
    rowarg = rng.integers(0, n2, n1).astype(np.int32)
    colarg = rng.integers(0, n1, n2).astype(np.int32)
    # plant mutual pairs and a few out-of-range indices
    i = rng.choice(n1, 3000, replace=False)
    j = rng.choice(n2, 3000, replace=False)
    rowarg[i] = j
    colarg[j] = i
    rowarg[:5] = [-1, n2, n2 + 7, -100, 2 ** 30]
    pairs, count = rnn.mnn_mutual(torch.from_numpy(rowarg).cuda(), torch.from_numpy(colarg).cuda())
    ok = np.array([0 <= rowarg[k] < n2 and colarg[rowarg[k]] == k for k in range(n1)])
    ref = np.stack([np.nonzero(ok)[0], rowarg[ok]], axis=1)
    assert np.array_equal(pairs[: int(count.item())].cpu().numpy(), ref)


def test_sharded_single_rank_equals_exhaustive():
    from reciprocal_nearest_neighbour_b200 import replicas

    rng = np.random.default_rng(91)
    D1 = synth.to_storage(synth.quantised_map(rng, 37, 41, 24), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, 29, 53, 24), "f16")
    pairs, count = replicas.mnn_sharded(dev(D1), dev(D2), 1, 0)
    ref = oracle.mnn(D1, D2).pairs
    assert np.array_equal(pairs[: int(count.item())].cpu().numpy(), ref)
    # the rank-0 half of a two-rank split finds the NN of its own rows exactly
    r1 = replicas.row_slice(37 * 41, 2, 0)
    idx, _ = rnn.nn_argmax(dev(D1).reshape(-1, 24)[r1.start:r1.stop], dev(D2).reshape(-1, 24))
    ref_rows = oracle.nn(D1.reshape(-1, 24)[r1.start:r1.stop], D2.reshape(-1, 24)).arg
    assert len(ref_rows) == len(r1)
    assert np.array_equal(idx.cpu().numpy(), ref_rows)
