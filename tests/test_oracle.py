"""Pins for the double-precision oracle (CPU only).

Each test ties the oracle to something other than itself: hand-worked golden
cases, an exact integer brute force written independently here, closed forms
(FRM with stride 1 equals the reciprocal set; an identity warp matches every
pixel to itself) and the invariants the pages state (every FRM pair is a
mutual match, FRM output is a subset of M, scores never decrease along a
trajectory).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from reciprocal_nearest_neighbour_b200 import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _chain_maps(g):
    S = np.array(g["scores"], dtype=np.float64)
    D1 = S.reshape(g["H1"], g["W1"], g["d"])
    D2 = np.eye(g["d"]).reshape(g["H2"], g["W2"], g["d"])
    return D1, D2


# ---------------------------------------------------------------- golden cases

def test_golden_chain_nn_and_mnn(golden_dir):
    g = _load(golden_dir, "frm_chain_2x2_1x4.json")
    D1, D2 = _chain_maps(g)
    r = oracle.mnn(D1, D2)
    assert r.row.arg.tolist() == g["nn2"]
    assert r.col.arg.tolist() == g["nn1"]
    assert r.pairs.tolist() == g["mnn"]


@pytest.mark.parametrize("case", range(6))
def test_golden_chain_frm(golden_dir, case):
    g = _load(golden_dir, "frm_chain_2x2_1x4.json")
    c = g["frm"][case]
    D1, D2 = _chain_maps(g)
    r = oracle.frm(D1, D2, seed_stride=c["stride"], max_iter=c["max_iter"])
    assert r.pairs.reshape(-1, 2).tolist() == c["pairs"]
    if "seed_queries" in c:
        assert r.seed_queries.tolist() == c["seed_queries"]
    if "seed_converged" in c:
        assert r.seed_converged.tolist() == c["seed_converged"]
    if "traj" in c:
        assert r.traj.tolist() == c["traj"]


def test_golden_seed_grid(golden_dir):
    g = _load(golden_dir, "seed_grid.json")
    for c in g["cases"]:
        s = oracle.frm_seeds(c["H"], c["W"], c["S"])
        if "seeds" in c:
            assert s.tolist() == c["seeds"], c
        else:
            assert len(s) == c["count"] and s[0] == c["first"] and s[-1] == c["last"], c
        assert np.all(np.diff(s) > 0)


def test_golden_nn_ties(golden_dir):
    g = _load(golden_dir, "nn_ties.json")
    for c in g["cases"]:
        sc = np.array(c["scores"], dtype=np.float64)
        X = np.zeros((len(sc), 4))
        X[:, 0] = sc
        q = np.zeros((1, 4))
        q[0, 0] = 1.0
        r = oracle.nn(q, X)
        assert r.arg[0] == c["arg"], c
        want = math.inf if c["gap"] == "inf" else c["gap"]
        assert r.gap[0] == want, c


# ------------------------------------------------------- exact integer brute force

def _int_codes(H, W, d, seed):
    rng = np.random.default_rng(seed)
    return synth.quantised_map(rng, H, W, d)


def _brute(K1, K2):
    """Exact integer scores (k1 . k2) and lowest-index argmax both ways."""
    A = np.rint(K1.reshape(-1, K1.shape[-1]) * 64).astype(np.int64)
    B = np.rint(K2.reshape(-1, K2.shape[-1]) * 64).astype(np.int64)
    S = A @ B.T
    rowarg = S.argmax(axis=1)          # numpy argmax returns the first maximum
    colarg = S.argmax(axis=0)
    mutual = [(i, int(rowarg[i])) for i in range(S.shape[0]) if colarg[rowarg[i]] == i]
    return S, rowarg, colarg, mutual


@pytest.mark.parametrize("shape", [((7, 9), (8, 6), 16), ((16, 16), (16, 16), 8),
                                   ((5, 13), (11, 3), 24), ((32, 32), (32, 32), 16)])
def test_mnn_matches_integer_bruteforce(shape):
    (H1, W1), (H2, W2), d = shape
    rng = np.random.default_rng(11 + d)
    D1 = synth.quantised_map(rng, H1, W1, d)
    D2 = synth.quantised_map(rng, H2, W2, d)
    S, ra, ca, mutual = _brute(D1, D2)
    r = oracle.mnn(D1, D2)
    assert np.array_equal(r.row.arg, ra)
    assert np.array_equal(r.col.arg, ca)
    assert [tuple(p) for p in r.pairs.tolist()] == mutual
    # scores are exact: best * 4096 is the integer maximum
    assert np.array_equal(r.row.best * 4096, S.max(axis=1).astype(np.float64))
    assert np.array_equal(r.col.best * 4096, S.max(axis=0).astype(np.float64))
    srt = np.sort(S, axis=1)
    assert np.array_equal(r.row.gap * 4096, (srt[:, -1] - srt[:, -2]).astype(np.float64))


def test_tiny_workload_matches_bruteforce():
    w = synth.WORKLOADS["tiny_q32"]
    D1, D2 = synth.make_workload(w)
    _, ra, ca, mutual = _brute(D1, D2)
    r = oracle.mnn(D1, D2)
    assert np.array_equal(r.row.arg, ra) and np.array_equal(r.col.arg, ca)
    assert [tuple(p) for p in r.pairs.tolist()] == mutual


def test_ties_on_duplicated_candidates():
    rng = np.random.default_rng(5)
    D1 = synth.quantised_map(rng, 4, 4, 8)
    base = synth.quantised_map(rng, 2, 4, 8)
    D2 = np.concatenate([base, base], axis=0)        # candidates j and j+8 are equal
    r = oracle.mnn(D1, D2)
    assert np.all(r.row.arg < 8)                      # lowest index wins
    assert np.all(r.row.gap == 0)
    zeros = np.zeros((3, 3, 8))
    z = oracle.mnn(zeros, zeros)                      # every score is 0
    assert np.all(z.row.arg == 0) and np.all(z.col.arg == 0)
    assert z.pairs.tolist() == [[0, 0]]


# ------------------------------------------------------------------ closed forms

@pytest.mark.parametrize("max_iter", [1, 3, 10])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_frm_stride1_equals_mnn(seed, max_iter):
    rng = np.random.default_rng(100 + seed)
    D1 = synth.quantised_map(rng, 9, 11, 16)
    D2 = synth.quantised_map(rng, 10, 7, 16)
    m = oracle.mnn(D1, D2)
    f = oracle.frm(D1, D2, seed_stride=1, max_iter=max_iter)
    assert f.pairs.tolist() == m.pairs.tolist()


def _unit_iid(rng, H, W, d):
    v = rng.standard_normal((H, W, d))
    v /= np.linalg.norm(v, axis=-1, keepdims=True)
    return synth.to_storage(v, "f16").double().numpy()


def test_identity_warp():
    rng = np.random.default_rng(7)
    D = _unit_iid(rng, 20, 24, 32)
    m = oracle.mnn(D, D)
    n = 20 * 24
    assert m.pairs.tolist() == [[i, i] for i in range(n)]
    f = oracle.frm(D, D, seed_stride=4, max_iter=10)
    seeds = oracle.frm_seeds(20, 24, 4)
    assert f.pairs.tolist() == [[s, s] for s in seeds]
    assert np.all(f.seed_queries == 2)               # converged in the first iteration
    assert np.all(f.seed_converged)


def test_identity_warp_quantised():
    # for vectors that are not unit length, (i,i) is in M iff NN2(i) = i, and M
    # only holds diagonal pairs or symmetric off-diagonal pairs
    rng = np.random.default_rng(8)
    D = synth.quantised_map(rng, 12, 12, 16)
    m = oracle.mnn(D, D)
    P = {tuple(p) for p in m.pairs.tolist()}
    for i in range(144):
        assert ((i, i) in P) == (m.row.arg[i] == i)
    for (i, j) in P:
        assert i == j or (j, i) in P


# ------------------------------------------------------------------- invariants

@pytest.mark.parametrize("seed", range(4))
def test_frm_subset_mutual_monotone(seed):
    rng = np.random.default_rng(200 + seed)
    D1 = synth.quantised_map(rng, 16, 20, 16)
    D2 = synth.quantised_map(rng, 18, 14, 16)
    S, ra, ca, mutual = _brute(D1, D2)
    f = oracle.frm(D1, D2, seed_stride=2, max_iter=10)
    for (u, v) in f.pairs.tolist():
        assert ra[u] == v and ca[v] == u              # every output pair is mutual
    assert set(map(tuple, f.pairs.tolist())) <= set(mutual)
    assert f.pairs.tolist() == sorted(map(list, set(map(tuple, f.pairs.tolist()))))
    # scores never decrease along a trajectory
    for s in range(len(f.seeds)):
        seq = []
        prev_u = f.seeds[s]
        for t in range(10):
            u_in, v, u_out = f.traj[s, t]
            if u_in < 0:
                break
            assert u_in == prev_u
            seq.append(S[u_in, v])
            if u_out >= 0:
                seq.append(S[u_out, v])
                prev_u = u_out
        assert all(a <= b for a, b in zip(seq, seq[1:])), seq


def test_mnn_symmetry_and_uniqueness():
    rng = np.random.default_rng(9)
    D1 = synth.quantised_map(rng, 13, 17, 24)
    D2 = synth.quantised_map(rng, 15, 12, 24)
    a = oracle.mnn(D1, D2).pairs
    b = oracle.mnn(D2, D1).pairs
    assert sorted(map(tuple, a.tolist())) == sorted((j, i) for i, j in b.tolist())
    assert len(set(a[:, 0])) == len(a) and len(set(a[:, 1])) == len(a)


def test_frm_on_smooth_pair_converges_and_is_mutual():
    D1, D2 = synth.smooth_pair(3, 48, 64, 24)
    D1 = synth.to_storage(D1, "f16")
    D2 = synth.to_storage(D2, "f16")
    f = oracle.frm(D1, D2, seed_stride=8, max_iter=10)
    m = oracle.mnn(D1, D2)
    assert len(f.pairs) > 0.5 * len(f.seeds)
    assert set(map(tuple, f.pairs.tolist())) <= set(map(tuple, m.pairs.tolist()))
    # the active counts shrink and match the per-seed query counts
    assert f.active_per_half.sum() == f.seed_queries.sum()


def test_thread_count_does_not_change_results():
    D1, D2 = synth.quantised_pair(4, 20, 20, 18, 22, 16)
    a = oracle.frm(D1, D2, seed_stride=3, max_iter=10, threads=1)
    b = oracle.frm(D1, D2, seed_stride=3, max_iter=10, threads=0)
    assert np.array_equal(a.pairs, b.pairs) and np.array_equal(a.traj, b.traj)
    m1 = oracle.mnn(D1, D2, threads=1)
    m2 = oracle.mnn(D1, D2, threads=0)
    assert np.array_equal(m1.pairs, m2.pairs)


def test_quantised_values_exact_in_storage_types():
    rng = np.random.default_rng(1)
    q = synth.quantised_map(rng, 8, 8, 16)
    k = q * 64
    assert np.all(np.abs(k) <= 127) and np.array_equal(k, np.rint(k))
    for dt in ("f16", "bf16"):
        assert np.array_equal(synth.to_storage(q, dt).double().numpy(), q)


def test_workloads_have_stated_shapes():
    w = synth.WORKLOADS["frm_512x384"]
    assert (w.H, w.W, w.d, w.seed_stride, w.max_iter) == (384, 512, 24, 8, 10)
    assert len(oracle.frm_seeds(w.H, w.W, w.seed_stride)) == 3072
    b = synth.WORKLOADS["frm_batched_64x512x288"]
    assert (b.pairs, b.H, b.W, b.occlusion) == (64, 288, 512, 0.30)


# ------------------------------------------------- metric, start pixels, basin
# Pins for the quoted function's other options (see oracle.frm_ex): the
# Euclidean metric of its brute-force matcher, FRM from given start pixels
# with the pixel tolerance, and the basin output.

def _ints(D):
    """Integer numerators k of a quantised map (values k/64)."""
    return np.rint(np.asarray(D, dtype=np.float64).reshape(-1, np.asarray(D).shape[-1]) * 64
                   ).astype(np.int64)


def _nn_int(A, B, metric):
    """Exact NN of each row of A among the rows of B (integers), first index on ties."""
    if metric == "dot":
        return (A @ B.T).argmax(axis=1)
    d2 = ((A[:, None, :] - B[None, :, :]) ** 2).sum(axis=2)
    return d2.argmin(axis=1)


def test_golden_nn_l2_ties(golden_dir):
    g = _load(golden_dir, "nn_l2_ties.json")
    X, Q = np.array(g["X"], float), np.array(g["Q"], float)
    assert oracle.nn(Q, X, metric="l2").arg.tolist() == g["l2_arg"]
    assert oracle.nn(Q, X, metric="dot").arg.tolist() == g["dot_arg"]


@pytest.mark.parametrize("shape", [((7, 9), (8, 6), 16), ((5, 13), (11, 3), 24),
                                   ((16, 16), (16, 16), 8)])
def test_l2_nn_and_mnn_match_integer_bruteforce(shape):
    (H1, W1), (H2, W2), d = shape
    rng = np.random.default_rng(31 + d)
    D1 = synth.quantised_map(rng, H1, W1, d)
    D2 = synth.quantised_map(rng, H2, W2, d)
    A, B = _ints(D1), _ints(D2)
    ra, ca = _nn_int(A, B, "l2"), _nn_int(B, A, "l2")
    r = oracle.mnn(D1, D2, metric="l2")
    assert np.array_equal(r.row.arg, ra) and np.array_equal(r.col.arg, ca)
    mutual = [(i, int(ra[i])) for i in range(len(ra)) if ca[ra[i]] == i]
    assert [tuple(p) for p in r.pairs.tolist()] == mutual
    # best = -min squared distance, exact (multiples of 1/4096)
    d2 = ((A[:, None, :] - B[None, :, :]) ** 2).sum(axis=2)
    assert np.array_equal(-r.row.best * 4096, d2.min(axis=1).astype(np.float64))


def test_l2_equals_dot_on_unit_vectors():
    """For unit vectors |a-b|^2 = 2 - 2 a.b, so both metrics pick the same NN."""
    rng = np.random.default_rng(5)
    A = rng.standard_normal((200, 16))
    B = rng.standard_normal((300, 16))
    A /= np.linalg.norm(A, axis=1, keepdims=True)
    B /= np.linalg.norm(B, axis=1, keepdims=True)
    dot, l2 = oracle.nn(A, B), oracle.nn(A, B, metric="l2")
    sep = dot.gap > 1e-9
    assert sep.mean() > 0.99
    assert np.array_equal(dot.arg[sep], l2.arg[sep])


@pytest.mark.parametrize("case", range(5))
def test_golden_refine(golden_dir, case):
    g = _load(golden_dir, "frm_refine_1x3_1x2.json")
    c = g["cases"][case]
    D1 = np.array(g["D1"], float).reshape(g["H1"], g["W1"], g["d"])
    D2 = np.array(g["D2"], float).reshape(g["H2"], g["W2"], g["d"])
    r = oracle.frm_refine(D1, D2, g["init"], pixel_tol=c["pixel_tol"], metric=c["metric"])
    assert r.seeds.tolist() == [0, 1, 2]
    assert r.pairs.tolist() == c["pairs"]
    assert r.seed_queries.tolist() == [2, 2, 2]


def _refine_numpy(A, B, H1, W1, init, tol, metric):
    """The pixel-tolerance round trip from each unique start, written out."""
    pairs = set()
    for u in np.unique(init):
        v = int(_nn_int(A[u:u + 1], B, metric)[0])
        u2 = int(_nn_int(B[v:v + 1], A, metric)[0])
        if tol > 0:
            conv = math.hypot(u // W1 - u2 // W1, u % W1 - u2 % W1) < tol
        else:
            conv = u2 == u
        if conv:
            pairs.add((int(u), v))
    return sorted(pairs)


@pytest.mark.parametrize("metric", ["dot", "l2"])
@pytest.mark.parametrize("tol", [0.0, 1.0, 1.5, 2.3])
def test_refine_matches_numpy_roundtrip(metric, tol):
    rng = np.random.default_rng(77)
    H1, W1, H2, W2, d = 9, 11, 8, 10, 16
    D1 = synth.quantised_map(rng, H1, W1, d)
    D2 = synth.quantised_map(rng, H2, W2, d)
    init = rng.integers(0, H1 * W1, size=60).astype(np.int32)
    init[5] = init[0]                                # a duplicate
    r = oracle.frm_refine(D1, D2, init, pixel_tol=tol, metric=metric)
    ref = _refine_numpy(_ints(D1), _ints(D2), H1, W1, init, tol, metric)
    assert [tuple(p) for p in r.pairs.tolist()] == ref
    assert np.array_equal(r.seeds, np.unique(init))


@pytest.mark.parametrize("case", range(5))
def test_golden_basin(golden_dir, case):
    g = _load(golden_dir, "frm_basin_chain_2x2_1x4.json")
    c = g["cases"][case]
    D1, D2 = _chain_maps(g)
    r = oracle.frm_ex(D1, D2, c["stride"], c["max_iter"], basin=True)
    assert r.pairs.tolist() == c["pairs"]
    assert r.basin.tolist() == c["basin"]
    if "seed_queries" in c:
        assert r.seed_queries.tolist() == c["seed_queries"]


def _basin_numpy(A, B, seeds, max_iter):
    """Replay of the basin-mode loop with exact integer NN queries."""
    n1 = A.shape[0]
    U = seeds.astype(np.int64).copy()
    V = np.full_like(U, -1)
    Uold = U.copy()
    active = np.ones(len(U), bool)
    basin = np.full(n1 + 1, -1, np.int64)
    t = 0
    while active.any():
        idx = np.nonzero(active)[0]
        V[idx] = _nn_int(A[U[idx]], B, "dot")
        U[idx] = _nn_int(B[V[idx]], A, "dot")
        basin[Uold[idx]] = U[idx]
        active[idx] = U[idx] != Uold[idx]
        t += 1
        if t >= max_iter:
            break
        Uold = U.copy()
    conv = ~active
    pairs = sorted({(int(U[s]), int(V[s])) for s in range(len(U)) if conv[s]})
    return pairs, basin


@pytest.mark.parametrize("S,max_iter", [(2, 10), (3, 2), (1, 10)])
def test_basin_matches_numpy_replay_and_plain_frm(S, max_iter):
    rng = np.random.default_rng(90 + S)
    H, W, d = 10, 12, 16
    D1 = synth.quantised_map(rng, H, W, d)
    D2 = synth.quantised_map(rng, H, W, d)
    r = oracle.frm_ex(D1, D2, S, max_iter, basin=True)
    pairs, basin = _basin_numpy(_ints(D1), _ints(D2), oracle.frm_seeds(H, W, S), max_iter)
    assert [tuple(p) for p in r.pairs.tolist()] == pairs
    assert np.array_equal(r.basin, basin)
    # skipping the first half-step's test changes no output pair
    assert np.array_equal(r.pairs, oracle.frm(D1, D2, S, max_iter).pairs)


# ------------------------------------------------------------------ 3-D points
# MASt3R's NN function on 3-D points is a K-d tree query (scipy's cKDTree
# here): the oracle's Euclidean metric at d = 3 must give its answers.

def test_points_nn_matches_kdtree():
    from scipy.spatial import cKDTree

    rng = np.random.default_rng(123)
    X = rng.standard_normal((3000, 3)) * np.array([3.0, 2.0, 1.0])
    Q = rng.standard_normal((1000, 3)) * 4.0            # some queries far outside
    r = oracle.nn(Q, X, metric="l2")
    dist, idx = cKDTree(X).query(Q)
    assert np.array_equal(r.arg, idx)
    assert np.allclose(-r.best, dist ** 2, rtol=1e-12, atol=0.0)


def test_points_nn_ties_lowest_index_via_ball_query():
    """Repeated points and equal distances: the distance is the tree's, and
    the index is the lowest of all points at that distance (a ball query
    collects them; their squared distances are compared as integers)."""
    from scipy.spatial import cKDTree

    rng = np.random.default_rng(124)
    X = synth.quantised_points(rng, 2000, repeat=0.2)
    Q = synth.quantised_points(rng, 400)
    Q[:50] = X[rng.integers(0, len(X), 50)]               # queries on data points
    r = oracle.nn(Q, X, metric="l2")
    tree = cKDTree(X)
    dist, _ = tree.query(Q)
    assert np.allclose(-r.best, dist ** 2, rtol=1e-12, atol=0.0)
    Xi, Qi = np.rint(X * 64).astype(np.int64), np.rint(Q * 64).astype(np.int64)
    for t in range(len(Q)):
        near = np.array(tree.query_ball_point(Q[t], dist[t] * (1 + 1e-9) + 1e-12))
        d2 = ((Xi[near] - Qi[t]) ** 2).sum(axis=1)
        low = near[d2 == d2.min()].min()
        assert r.arg[t] == low, t
        assert -r.best[t] * 4096 == d2.min()


def _frm_kdtree(P1, P2, seeds, max_iter):
    """The FRM loop on point maps with K-d tree queries as the NN function,
    written out (grid seeds, V = NN2(U), U = NN1(V), the two convergence
    tests, max_iter), as the quoted function runs it on the CPU."""
    from scipy.spatial import cKDTree

    A, B = P1.reshape(-1, 3), P2.reshape(-1, 3)
    t1, t2 = cKDTree(A), cKDTree(B)
    U = seeds.astype(np.int64).copy()
    V = np.full_like(U, -1)
    Uold, Vold = U.copy(), V.copy()
    active = np.ones(len(U), bool)
    for it in range(max_iter):
        idx = np.nonzero(active)[0]
        if len(idx) == 0:
            break
        V[idx] = t2.query(A[U[idx]])[1]
        active[idx] = V[idx] != Vold[idx]
        idx = np.nonzero(active)[0]
        U[idx] = t1.query(B[V[idx]])[1]
        active[idx] = U[idx] != Uold[idx]
        Uold, Vold = U.copy(), V.copy()
    return sorted({(int(U[s]), int(V[s])) for s in range(len(U)) if not active[s]})


@pytest.mark.parametrize("S,max_iter", [(4, 10), (2, 3), (1, 10)])
def test_points_frm_matches_kdtree_replay(S, max_iter):
    P1, P2 = synth.pointmap_pair(51 + S, 24, 32, noise=0.01)
    r = oracle.frm_ex(P1, P2, S, max_iter, metric="l2")
    ref = _frm_kdtree(P1, P2, oracle.frm_seeds(24, 32, S), max_iter)
    assert [tuple(p) for p in r.pairs.tolist()] == ref
    assert len(ref) > 0


def test_points_mnn_matches_kdtree():
    from scipy.spatial import cKDTree

    P1, P2 = synth.pointmap_pair(60, 20, 28, noise=0.01)
    A, B = P1.reshape(-1, 3), P2.reshape(-1, 3)
    r = oracle.mnn(P1, P2, metric="l2")
    ra, ca = cKDTree(B).query(A)[1], cKDTree(A).query(B)[1]
    assert np.array_equal(r.row.arg, ra) and np.array_equal(r.col.arg, ca)
    mutual = [(i, int(ra[i])) for i in range(len(ra)) if ca[ra[i]] == i]
    assert [tuple(p) for p in r.pairs.tolist()] == mutual


def test_pointmap_generator_ranges():
    P1, P2 = synth.pointmap_pair(3, 48, 64, quantised=True)
    for P in (P1, P2):
        assert P.shape == (48, 64, 3)
        assert np.abs(P).max() <= 16.0
        assert np.array_equal(P * 64, np.rint(P * 64))
    Q = synth.quantised_points(np.random.default_rng(1), 1000)
    assert np.abs(Q).max() <= 16.0 and np.array_equal(Q * 64, np.rint(Q * 64))


# ------------------------------------------------------------- coarse-to-fine

def test_golden_c2f_crops(golden_dir):
    g = _load(golden_dir, "c2f_crops_8x12.json")
    for L, c, want in g["origins"]:
        assert oracle.c2f_crop_origins(L, c) == want
    for i, Hc, Wc, H, W, want in g["fine_pixel"]:
        assert list(oracle.c2f_fine_pixel(i, Hc, Wc, H, W)) == want
    sizes = (g["Hc1"], g["Wc1"], g["Hc2"], g["Wc2"], g["H1"], g["W1"], g["H2"], g["W2"])
    for m, key in ((1, "crops_min1"), (2, "crops_min2")):
        t = oracle.c2f_crops(g["coarse"], *sizes, tuple(g["crop"]), min_coarse=m)
        assert t.tolist() == g[key]


def _pool(D, s):
    """Mean over s x s pixel blocks, renormalised (the coarse stand-in)."""
    H, W, d = D.shape
    P = D[: H // s * s, : W // s * s].reshape(H // s, s, W // s, s, d).mean(axis=(1, 3))
    return P / np.linalg.norm(P, axis=-1, keepdims=True)


def test_c2f_one_crop_is_plain_frm():
    """A crop as large as the images leaves one crop pair, (0,0)-(0,0): the
    result is FRM on the full-resolution maps."""
    F1, F2 = synth.smooth_pair(21, 24, 32, 16)
    C1, C2 = _pool(F1, 4), _pool(F2, 4)
    r = oracle.c2f(C1, C2, F1, F2, crop=(64, 64), seed_stride=3, max_iter=10)
    assert r.crops.tolist() == [[0, 0, 0, 0, len(r.coarse), 1]]
    assert np.array_equal(r.pairs, oracle.frm_ex(F1, F2, 3, 10).pairs)


def test_c2f_pairs_are_mutual_in_their_crops():
    F1, F2 = synth.smooth_pair(22, 40, 48, 16)
    C1, C2 = _pool(F1, 4), _pool(F2, 4)
    crop = (16, 20)
    r = oracle.c2f(C1, C2, F1, F2, crop=crop, seed_stride=2, max_iter=10)
    assert len(r.pairs) > 50 and r.crops[:, 5].sum() >= 4
    W1 = W2 = 48
    seen = set()
    for y0, x0, y2, x2, n, on in r.crops.tolist():
        if not on:
            continue
        a, b = F1[y0:y0 + 16, x0:x0 + 20], F2[y2:y2 + 16, x2:x2 + 20]
        m = oracle.mnn(a, b)
        for u, v in m.pairs.tolist():
            seen.add(((y0 + u // 20) * W1 + x0 + u % 20, (y2 + v // 20) * W2 + x2 + v % 20))
    # every output pair is a reciprocal pair of some crop pair's windows
    assert all((int(u), int(v)) in seen for u, v in r.pairs)
    assert np.all(np.diff(r.pairs[:, 0]) > 0)
