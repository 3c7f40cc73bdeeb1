"""Parity of small query counts on the GPU (needs a B200).

Launches with a few queries per problem (small nearest-neighbour calls, the
late FRM half-steps) leave most rows of the 128-row query tile empty.  These
cases pin them against the double-precision oracle: query counts up to and
past 32, ragged candidate tails inside a 32-candidate chunk, a 128-candidate
half and a 256-candidate tile, and ties placed in different lanes, warps,
halves and tiles, which must resolve to the lowest index.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import check_nn_tolerant, dev

pytestmark = pytest.mark.gpu


def _q(seed, n, d):
    rng = np.random.default_rng(seed)
    return synth.quantised_map(rng, 1, n, d).reshape(n, d)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("nq", [1, 7, 16, 17, 31, 32, 33])
@pytest.mark.parametrize("nx,d", [(1, 8), (255, 24), (257, 16), (5000, 24), (70001, 40),
                                  (3000, 64)])
def test_small_nn_quantised_bitexact(dt, nq, nx, d):
    Q = synth.to_storage(_q(nq * 11 + d, nq, d), dt)
    X = synth.to_storage(_q(nx * 5 + d, nx, d), dt)
    idx, score = rnn.nn_argmax(dev(Q), dev(X))
    ref = oracle.nn(Q, X)
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(score.cpu().numpy().astype(np.float64), ref.best)


@pytest.mark.parametrize("positions", [(40, 300, 1000), (31, 32, 33), (127, 128, 129),
                                       (255, 256, 4000), (5, 37, 69, 101), (1023, 770, 600)])
def test_small_ties_take_lowest_index(positions):
    rng = np.random.default_rng(sum(positions))
    n, d = 5000, 24
    X = synth.quantised_map(rng, 1, n, d).reshape(n, d) * 0.25    # small scores
    Q = synth.quantised_map(rng, 1, 20, d).reshape(20, d)
    # one vector with a score above every other candidate's, at several positions
    X[list(positions)] = np.round(Q[0] * 64) / 64
    Qt, Xt = synth.to_storage(Q, "f16"), synth.to_storage(X, "f16")
    idx, _ = rnn.nn_argmax(dev(Qt), dev(Xt))
    ref = oracle.nn(Qt, Xt)
    got = idx.cpu().numpy()
    assert np.array_equal(got, ref.arg)
    assert got[0] == min(positions)


def test_small_identical_candidates():
    zeros = torch.zeros((777, 16), dtype=torch.float16)
    idx, score = rnn.nn_argmax(dev(zeros[:9]), dev(zeros))
    assert idx.cpu().tolist() == [0] * 9 and score.cpu().tolist() == [0.0] * 9
    rng = np.random.default_rng(4)
    base = synth.quantised_map(rng, 1, 300, 16).reshape(300, 16)
    X = np.concatenate([base, base, base], axis=0)
    Q = synth.quantised_map(rng, 1, 25, 16).reshape(25, 16)
    Qt, Xt = synth.to_storage(Q, "f16"), synth.to_storage(X, "f16")
    idx, _ = rnn.nn_argmax(dev(Qt), dev(Xt))
    ref = oracle.nn(Qt, Xt)
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.all(ref.arg < 300)


@pytest.mark.parametrize("nq", [3, 32])
def test_small_unit_fp16_tolerance(nq):
    D1, D2 = synth.smooth_pair(60 + nq, 96, 128, 24)
    Q = synth.to_storage(D1.reshape(-1, 24)[:: (96 * 128) // nq][:nq], "f16")
    X = synth.to_storage(D2.reshape(-1, 24), "f16")
    idx, score = rnn.nn_argmax(dev(Q), dev(X))
    ref = oracle.nn(Q, X)
    check_nn_tolerant(Q, X, idx.cpu().numpy(), score.cpu().numpy(), ref)


def test_small_euclidean_bitexact():
    Q = synth.to_storage(_q(71, 29, 24), "f16")
    X = synth.to_storage(_q(72, 4099, 24), "f16")
    idx, score = rnn.nn_argmax(dev(Q), dev(X), metric="l2")
    ref = oracle.nn(Q, X, metric="l2")
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(score.cpu().numpy().astype(np.float64), -ref.best)


def test_small_frm_tail_matches_oracle():
    """Batched FRM whose late half-steps have a handful of live seeds per
    pair."""
    rng = np.random.default_rng(80)
    B, H, W, d = 4, 48, 64, 24
    D1 = synth.to_storage(np.stack([synth.quantised_map(rng, H, W, d) for _ in range(B)]), "f16")
    D2 = synth.to_storage(np.stack([synth.quantised_map(rng, H, W, d) for _ in range(B)]), "f16")
    r = rnn.frm_match_batched(dev(D1), dev(D2), seed_stride=12, max_iter=10,
                              with_seed_state=True)
    for b in range(B):
        ref = oracle.frm_ex(D1[b], D2[b], 12, 10)
        assert np.array_equal(r.pairs[b, : int(r.count[b])].cpu().numpy(),
                              ref.pairs.reshape(-1, 2)), b
        st = r.seed_state[b].cpu().numpy()
        assert np.array_equal(st[: len(ref.seed_queries), 2], ref.seed_queries), b
