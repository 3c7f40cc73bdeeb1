"""Full-size parity (needs a B200): the whole exhaustive set at 512x384 in
both input modes, every pair of the 64-pair batched FRM workload, and the
one-pass exhaustive kernel's chunk and edge cases.

The oracle's results on the full workloads come from
``tests/golden/make_full_size_refs.py`` (stored with the SHA-256 of their
inputs and of the oracle's sources); when a stored file does not match its
inputs, the oracle runs here instead (minutes on the host).

M = {(i,j) | j = NN2(D1_i) and i = NN1(D2_j)} (cv-learn.com "MASt3R" note,
paragraph "Fast reciprocal matching (FRM)"): with the oracle's NN arrays the
reference pair list is that definition written out.
"""
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import TOL, check_mnn_tolerant, check_nn_tolerant, dev, pairs_from_seeds, \
    seed_state_np

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
import make_full_size_refs as refs  # noqa: E402

pytestmark = pytest.mark.gpu


def _mutual_pairs(rowarg, colarg):
    """M from NN arrays: (i, rowarg[i]) where colarg[rowarg[i]] == i, increasing i."""
    i = np.nonzero(colarg[rowarg] == np.arange(len(rowarg)))[0]
    return np.stack([i, rowarg[i]], axis=1).astype(np.int32).reshape(-1, 2)


def _mnn_ref(mode, a, b, metric="dot"):
    z = refs.load("mnn_512x384_" + mode + ("" if metric == "dot" else "_" + metric), a, b)
    if z is not None:
        return z
    r = oracle.mnn(a, b, metric=metric)
    z = dict(rowarg=r.row.arg, colarg=r.col.arg)
    if mode == "q":
        z.update(rowbest4096=np.round(r.row.best * 4096).astype(np.int32),
                 colbest4096=np.round(r.col.best * 4096).astype(np.int32))
    else:
        z.update(rowbest=r.row.best, colbest=r.col.best, rowgap=r.row.gap, colgap=r.col.gap)
    return z


def test_mnn_full_size_quantised_bitexact():
    """The whole 512x384, d = 24 set on k/64 maps: every NN index and score of
    both directions and the pair list, bit for bit."""
    w, a, b = refs.mnn_inputs("q")
    z = _mnn_ref("q", a, b)
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    rowarg, colarg = r.rowarg.cpu().numpy(), r.colarg.cpu().numpy()
    assert np.array_equal(rowarg, z["rowarg"])
    assert np.array_equal(colarg, z["colarg"])
    rowmax = r.rowmax.cpu().numpy().astype(np.float64) * 4096.0
    colmax = r.colmax.cpu().numpy().astype(np.float64) * 4096.0
    assert np.array_equal(rowmax, z["rowbest4096"].astype(np.float64))
    assert np.array_equal(colmax, z["colbest4096"].astype(np.float64))
    ref_pairs = _mutual_pairs(z["rowarg"], z["colarg"])
    assert np.array_equal(r.trimmed().cpu().numpy(), ref_pairs)
    assert len(ref_pairs) > 1000


def test_mnn_full_size_quantised_bf16_bitexact():
    """The same quantised maps stored as bf16 (k/64 with |k| <= 127 has at
    most 7 significant bits, so bf16 holds it exactly): the whole set equals
    the oracle's, bit for bit."""
    w, a, b = refs.mnn_inputs("q")
    z = _mnn_ref("q", a, b)
    a2, b2 = a.to(torch.bfloat16), b.to(torch.bfloat16)
    assert torch.equal(a2.float(), a.float()) and torch.equal(b2.float(), b.float())
    r = rnn.mnn_exhaustive(dev(a2), dev(b2), with_nn=True)
    assert np.array_equal(r.rowarg.cpu().numpy(), z["rowarg"])
    assert np.array_equal(r.colarg.cpu().numpy(), z["colarg"])
    rowmax = r.rowmax.cpu().numpy().astype(np.float64) * 4096.0
    colmax = r.colmax.cpu().numpy().astype(np.float64) * 4096.0
    assert np.array_equal(rowmax, z["rowbest4096"].astype(np.float64))
    assert np.array_equal(colmax, z["colbest4096"].astype(np.float64))
    assert np.array_equal(r.trimmed().cpu().numpy(), _mutual_pairs(z["rowarg"], z["colarg"]))


def test_mnn_full_size_l2_quantised_bitexact():
    """The whole 512x384, d = 24 set on k/64 maps under the Euclidean metric
    (the one-pass kernel on the symmetric forms): every nearest index by
    distance, every squared distance and the pair list, bit for bit."""
    w, a, b = refs.mnn_inputs("q")
    z = _mnn_ref("q", a, b, metric="l2")
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True, metric="l2")
    assert np.array_equal(r.rowarg.cpu().numpy(), z["rowarg"])
    assert np.array_equal(r.colarg.cpu().numpy(), z["colarg"])
    # the oracle scores -|a - b|^2, the library reports |a - b|^2
    rowmax = r.rowmax.cpu().numpy().astype(np.float64) * 4096.0
    colmax = r.colmax.cpu().numpy().astype(np.float64) * 4096.0
    assert np.array_equal(rowmax, -z["rowbest4096"].astype(np.float64))
    assert np.array_equal(colmax, -z["colbest4096"].astype(np.float64))
    assert np.array_equal(r.trimmed().cpu().numpy(), _mutual_pairs(z["rowarg"], z["colarg"]))


def test_mnn_full_size_fp16_tolerance():
    """The whole 512x384, d = 24 set on unit-norm fp16 maps: every index and
    score under the tolerance rule, and the pair list differing from the
    oracle's only where a row or column is a near-tie."""
    w, a, b = refs.mnn_inputs("f")
    z = _mnn_ref("f", a, b)
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    A, B = a.reshape(-1, w.d), b.reshape(-1, w.d)
    row = SimpleNamespace(arg=z["rowarg"], best=z["rowbest"].astype(np.float64),
                          gap=z["rowgap"].astype(np.float64))
    col = SimpleNamespace(arg=z["colarg"], best=z["colbest"].astype(np.float64),
                          gap=z["colgap"].astype(np.float64))
    nd_row = check_nn_tolerant(A, B, r.rowarg.cpu().numpy(), r.rowmax.cpu().numpy(), row)
    nd_col = check_nn_tolerant(B, A, r.colarg.cpu().numpy(), r.colmax.cpu().numpy(), col)
    ref = SimpleNamespace(pairs=_mutual_pairs(z["rowarg"], z["colarg"]), row=row, col=col)
    nd_m = check_mnn_tolerant(r.trimmed().cpu().numpy(), ref)
    # near-ties are rare: the sets agree almost everywhere
    assert nd_row < 200 and nd_col < 200 and nd_m < 200, (nd_row, nd_col, nd_m)
    assert len(ref.pairs) > 100000


def test_frm_batched_workload_all_pairs():
    """All 64 pairs of 512x288 (30 % occlusion) in one launch sequence:
    seeds whose oracle trajectory has no near-tie match the oracle exactly
    (final U, V, queries, converged); every output pair is the oracle's or
    mutual under the tolerance rule."""
    w, a, b = refs.frm64_inputs()
    z = refs.load(w.name, a, b)
    r = rnn.frm_match_batched(dev(a), dev(b), w.seed_stride, w.max_iter, with_seed_state=True)
    unstable = 0
    for i in range(w.pairs):
        if z is None:
            o = oracle.frm(a[i], b[i], w.seed_stride, w.max_iter)
            ou, ov, oq, oc, og = (o.seed_u, o.seed_v, o.seed_queries, o.seed_converged,
                                  o.seed_min_gap)
        else:
            ou, ov, oq = z["seed_u"][i], z["seed_v"][i], z["seed_queries"][i]
            oc, og = z["seed_converged"][i].astype(bool), z["seed_min_gap"][i]
        u, v, q, c = seed_state_np(r, i)
        stable = og >= TOL
        unstable += int((~stable).sum())
        assert np.array_equal(u[stable], ou[stable]), i
        assert np.array_equal(v[stable], ov[stable]), i
        assert np.array_equal(q[stable], oq[stable]), i
        assert np.array_equal(c[stable], oc[stable]), i
        got = r.pairs[i, : int(r.count[i])].cpu().numpy()
        assert got.tolist() == [list(p) for p in pairs_from_seeds(u, v, c)], i
        ref_pairs = set(pairs_from_seeds(ou, ov, oc))
        assert set(pairs_from_seeds(ou[stable], ov[stable], oc[stable])) <= \
            {tuple(p) for p in got.tolist()}, i
        # pairs the oracle did not output: mutual nearest neighbours under the rule
        extra = np.array([p for p in got.tolist() if tuple(p) not in ref_pairs],
                         dtype=np.int32).reshape(-1, 2)
        if len(extra):
            A, B = a[i].reshape(-1, w.d), b[i].reshape(-1, w.d)
            s = oracle.pair_scores(A, B, extra[:, 0], extra[:, 1])
            assert np.all(s >= oracle.nn(A[extra[:, 0]], B).best - TOL), i
            assert np.all(s >= oracle.nn(B[extra[:, 1]], A).best - TOL), i
    # about 9 % of the seeds pass a near-tie somewhere along their trajectory
    # (occluded and out-of-view pixels hold fresh random vectors); the rest is
    # compared exactly above
    assert unstable < 0.15 * w.pairs * len(oracle.frm_seeds(w.H, w.W, w.seed_stride))


# ------------------------------------------------ one-pass kernel edge cases

@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_mnn_multi_unit_ragged_bitexact(dt):
    """A set large enough for whole 16 x 8-tile units in both directions, with
    ragged last blocks (the NaN rows past both maps), quantised, bit for bit."""
    D1, D2 = synth.quantised_pair(77, 160, 161, 190, 257, 24)
    a, b = synth.to_storage(D1, dt), synth.to_storage(D2, dt)
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    ref = oracle.mnn(a, b)
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.rowmax.cpu().numpy().astype(np.float64), ref.row.best)
    assert np.array_equal(r.colmax.cpu().numpy().astype(np.float64), ref.col.best)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_mnn_l2_multi_unit_ragged_bitexact(dt):
    """The Euclidean metric on the same multi-unit ragged shapes: nearest
    neighbours by distance in both directions, squared distances, bit for bit."""
    D1, D2 = synth.quantised_pair(78, 160, 161, 190, 257, 24)
    a, b = synth.to_storage(D1, dt), synth.to_storage(D2, dt)
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True, metric="l2")
    ref = oracle.mnn(a, b, metric="l2")
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.rowmax.cpu().numpy().astype(np.float64), -ref.row.best)
    assert np.array_equal(r.colmax.cpu().numpy().astype(np.float64), -ref.col.best)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))


@pytest.mark.parametrize("d", [8, 16, 24, 32, 64])
def test_mnn_ties_across_chunks(d):
    """Rows copied far from their originals in both maps (other quadrants,
    m-tiles and candidate tiles), so equal maxima sit in different chunks of
    both directions: the lowest index must win everywhere."""
    rng = np.random.default_rng(100 + d)
    H, W = 41, 97
    n = H * W
    D1 = synth.quantised_map(rng, H, W, d).reshape(n, d)
    D2 = synth.quantised_map(rng, H, W, d).reshape(n, d)
    for M in (D1, D2):
        src = rng.choice(n // 2, 400, replace=False)
        dst = n // 2 + rng.choice(n - n // 2, 400, replace=False)
        M[dst] = M[src]
    a = synth.to_storage(D1.reshape(H, W, d), "f16")
    b = synth.to_storage(D2.reshape(H, W, d), "f16")
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    ref = oracle.mnn(a, b)
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))
    # the copies made ties that reached the maximum in both directions
    assert np.any(ref.row.gap == 0) and np.any(ref.col.gap == 0)


def test_mnn_all_scores_equal():
    """Constant maps: every score is equal, so every NN is index 0 and M is
    {(0, 0)}; sizes spanning several units, quadrants and candidate tiles."""
    for shape1, shape2 in (((50, 60), (45, 70)), ((1, 3000), (2500, 1))):
        a = torch.full((*shape1, 16), 0.25, dtype=torch.float16)
        b = torch.full((*shape2, 16), -0.5, dtype=torch.float16)
        r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
        assert torch.all(r.rowarg == 0) and torch.all(r.colarg == 0)
        assert r.trimmed().cpu().tolist() == [[0, 0]]
        assert torch.all(r.rowmax == -2.0)
