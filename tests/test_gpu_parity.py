"""Parity of the CUDA path against the double-precision oracle (needs a B200).

Sizes span several 128-row query tiles and 256-row candidate tiles with
ragged tails; quantised inputs are compared bit for bit, unit-norm fp16
inputs under the tolerance rule of ``parity.py``.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import (TOL, check_mnn_tolerant, check_nn_tolerant, dev, pairs_from_seeds,
                    seed_state_np)

pytestmark = pytest.mark.gpu

DTYPES = ["f16", "bf16"]


def _q(seed, n, d):
    rng = np.random.default_rng(seed)
    return synth.quantised_map(rng, 1, n, d).reshape(n, d)


# ------------------------------------------------------------------ nn_argmax

@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("nq,nx,d", [(1, 1, 8), (5, 300, 16), (1000, 1537, 24), (130, 5000, 32),
                                     (257, 700, 40), (300, 2000, 64), (129, 513, 128),
                                     (200, 700, 256), (128, 256, 24)])
def test_nn_argmax_quantised_bitexact(dt, nq, nx, d):
    Q = synth.to_storage(_q(nq * 7 + d, nq, d), dt)
    X = synth.to_storage(_q(nx * 3 + d + 1, nx, d), dt)
    idx, score = rnn.nn_argmax(dev(Q), dev(X))
    ref = oracle.nn(Q, X)
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.array_equal(score.cpu().numpy().astype(np.float64), ref.best)


def test_nn_argmax_ties_take_lowest_index():
    rng = np.random.default_rng(3)
    base = synth.quantised_map(rng, 1, 300, 16).reshape(300, 16)
    X = np.concatenate([base, base, base], axis=0)      # each candidate appears 3 times
    Q = synth.quantised_map(rng, 1, 500, 16).reshape(500, 16)
    Qt, Xt = synth.to_storage(Q, "f16"), synth.to_storage(X, "f16")
    idx, _ = rnn.nn_argmax(dev(Qt), dev(Xt))
    ref = oracle.nn(Qt, Xt)
    assert np.array_equal(idx.cpu().numpy(), ref.arg)
    assert np.all(ref.arg < 300)
    zeros = torch.zeros((70, 8), dtype=torch.float16)
    idx, score = rnn.nn_argmax(dev(zeros[:5]), dev(zeros))
    assert idx.cpu().tolist() == [0] * 5 and score.cpu().tolist() == [0.0] * 5


def test_nn_argmax_unit_fp16_tolerance():
    D1, D2 = synth.smooth_pair(21, 40, 50, 24)
    Q = synth.to_storage(D1.reshape(-1, 24), "f16")
    X = synth.to_storage(D2.reshape(-1, 24), "f16")
    idx, score = rnn.nn_argmax(dev(Q), dev(X))
    ref = oracle.nn(Q, X)
    check_nn_tolerant(Q, X, idx.cpu().numpy(), score.cpu().numpy(), ref)


def test_nn_argmax_empty_queries():
    X = torch.ones((10, 8), dtype=torch.float16, device="cuda")
    Q = torch.ones((0, 8), dtype=torch.float16, device="cuda")
    idx, score = rnn.nn_argmax(Q, X)
    assert idx.numel() == 0


# ------------------------------------------------------------ exhaustive M

@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("s1,s2,d", [((32, 32), (32, 32), 16), ((37, 41), (29, 53), 24),
                                     ((1, 1), (3, 5), 8), ((20, 33), (20, 33), 32),
                                     ((9, 70), (11, 40), 256)])
def test_mnn_quantised_bitexact(dt, s1, s2, d):
    D1, D2 = synth.quantised_pair(sum(s1) * 31 + d, *s1, *s2, d)
    a, b = synth.to_storage(D1, dt), synth.to_storage(D2, dt)
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    ref = oracle.mnn(a, b)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.rowmax.cpu().numpy().astype(np.float64), ref.row.best)
    assert np.array_equal(r.colmax.cpu().numpy().astype(np.float64), ref.col.best)


def test_mnn_tiny_workload_and_identity():
    w = synth.WORKLOADS["tiny_q32"]
    D1, D2 = synth.make_workload(w)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.mnn_exhaustive(dev(a), dev(b))
    assert np.array_equal(r.trimmed().cpu().numpy(), oracle.mnn(a, b).pairs)
    rng = np.random.default_rng(4)
    v = rng.standard_normal((24, 20, 32))
    v /= np.linalg.norm(v, axis=-1, keepdims=True)
    u = synth.to_storage(v, "f16")
    r = rnn.mnn_exhaustive(dev(u), dev(u))
    assert r.trimmed().cpu().tolist() == [[i, i] for i in range(480)]


def test_mnn_unit_fp16_tolerance():
    D1, D2 = synth.smooth_pair(22, 48, 64, 24)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    ref = oracle.mnn(a, b)
    check_nn_tolerant(a, b, r.rowarg.cpu().numpy(), r.rowmax.cpu().numpy(), ref.row)
    check_nn_tolerant(b, a, r.colarg.cpu().numpy(), r.colmax.cpu().numpy(), ref.col)
    check_mnn_tolerant(r.trimmed().cpu().numpy(), ref)


def test_mnn_full_size_sampled_bitexact():
    """512x384, d=24 quantised, in the bench's launch configuration; sampled rows."""
    w = synth.WORKLOADS["mnn_512x384_q"]
    D1, D2 = synth.make_workload(w)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    rowarg, colarg = r.rowarg.cpu().numpy(), r.colarg.cpu().numpy()
    pairs = r.trimmed().cpu().numpy()
    rng = np.random.default_rng(0)
    n = w.H * w.W
    rows = np.unique(np.concatenate([rng.choice(n, 384, replace=False), [0, n - 1]]))
    A, B = a.reshape(n, -1), b.reshape(n, -1)
    ref_row = oracle.nn(A[rows], B)
    assert np.array_equal(rowarg[rows], ref_row.arg)
    cols = np.unique(np.concatenate([rng.choice(n, 384, replace=False), ref_row.arg]))
    ref_col = oracle.nn(B[cols], A)
    assert np.array_equal(colarg[cols], ref_col.arg)
    # membership of the sampled rows in M, from the oracle's own NN1 of their NN2
    colmap = dict(zip(cols.tolist(), ref_col.arg.tolist()))
    gpu_m = {int(i): int(j) for i, j in pairs}
    for i, j in zip(rows.tolist(), ref_row.arg.tolist()):
        assert (colmap[j] == i) == (gpu_m.get(i) == j)
    # global properties at any size: sorted, unique, mutual under the GPU's own NN
    assert np.all(np.diff(pairs[:, 0]) > 0)
    assert np.array_equal(rowarg[pairs[:, 0]], pairs[:, 1])
    assert np.array_equal(colarg[pairs[:, 1]], pairs[:, 0])
    mutual = np.nonzero(colarg[rowarg] == np.arange(n))[0]
    assert np.array_equal(mutual, pairs[:, 0])


# --------------------------------------------------------------------- FRM

def _frm_compare_exact(a, b, S, max_iter):
    ref = oracle.frm(a, b, S, max_iter)
    r = rnn.frm_match(dev(a), dev(b), S, max_iter, with_seed_state=True)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs.reshape(-1, 2))
    u, v, q, c = seed_state_np(r)
    assert np.array_equal(u, ref.seed_u) and np.array_equal(v, ref.seed_v)
    assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)
    return ref


@pytest.mark.parametrize("dt", DTYPES)
def test_frm_tiny_workload_bitexact(dt):
    w = synth.WORKLOADS["tiny_q32"]
    D1, D2 = synth.make_workload(w)
    _frm_compare_exact(synth.to_storage(D1, dt), synth.to_storage(D2, dt), w.seed_stride,
                       w.max_iter)


@pytest.mark.parametrize("S,max_iter,shape", [(1, 10, ((19, 23), (21, 17))), (3, 1, ((40, 37), (33, 45))),
                                              (3, 4, ((40, 37), (33, 45))), (5, 10, ((64, 70), (60, 75))),
                                              (2, 10, ((45, 47), (45, 47)))])
def test_frm_quantised_bitexact(S, max_iter, shape):
    (H1, W1), (H2, W2) = shape
    D1, D2 = synth.quantised_pair(H1 * W2 + S, H1, W1, H2, W2, 16)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    ref = _frm_compare_exact(a, b, S, max_iter)
    if S == 1:  # closed form: stride 1 gives the whole reciprocal set
        assert ref.pairs.tolist() == oracle.mnn(a, b).pairs.tolist()


def test_frm_golden_chain(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "frm_chain_2x2_1x4.json")))
    S = np.array(g["scores"], dtype=np.float64) / 16.0
    D1 = np.zeros((g["H1"], g["W1"], 8))
    D1.reshape(-1, 8)[:, :4] = S
    D2 = np.zeros((g["H2"], g["W2"], 8))
    D2.reshape(-1, 8)[:, :4] = np.eye(4)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    for c in g["frm"]:
        r = rnn.frm_match(dev(a), dev(b), c["stride"], c["max_iter"], with_seed_state=True)
        assert r.trimmed().cpu().tolist() == c["pairs"], c
        if "seed_queries" in c:
            assert seed_state_np(r)[2].tolist() == c["seed_queries"]
    m = rnn.mnn_exhaustive(dev(a), dev(b))
    assert m.trimmed().cpu().tolist() == g["mnn"]


def test_frm_no_seeds_and_single_pixel():
    a = torch.ones((1, 4, 8), dtype=torch.float16)
    r = rnn.frm_match(dev(a), dev(a), 2, 10)
    assert int(r.count[0]) == 0
    one = torch.ones((1, 1, 8), dtype=torch.float16)
    r = rnn.frm_match(dev(one), dev(one), 1, 10)
    assert r.trimmed().cpu().tolist() == [[0, 0]]


def _frm_tolerant(a, b, S, max_iter, res, b_index=0):
    """FRM parity on fp16: stable seeds exact, the rest mutual under the rule."""
    ref = oracle.frm(a, b, S, max_iter)
    u, v, q, c = seed_state_np(res, b_index)
    stable = ref.seed_min_gap >= TOL
    assert np.array_equal(u[stable], ref.seed_u[stable])
    assert np.array_equal(v[stable], ref.seed_v[stable])
    assert np.array_equal(q[stable], ref.seed_queries[stable])
    assert np.array_equal(c[stable], ref.seed_converged[stable])
    got = res.pairs[b_index, : int(res.count[b_index])].cpu().numpy()
    assert got.tolist() == [list(p) for p in pairs_from_seeds(u, v, c)]
    if len(got):
        A = a.reshape(-1, a.shape[-1])
        B = b.reshape(-1, b.shape[-1])
        s = oracle.pair_scores(A, B, got[:, 0], got[:, 1])
        rb = oracle.nn(A[got[:, 0]], B).best
        cb = oracle.nn(B[got[:, 1]], A).best
        assert np.all(s >= rb - TOL) and np.all(s >= cb - TOL)
    stable_pairs = pairs_from_seeds(ref.seed_u[stable], ref.seed_v[stable],
                                    ref.seed_converged[stable])
    assert set(stable_pairs) <= {tuple(p) for p in got.tolist()}
    return int((~stable).sum())


def test_frm_unit_fp16_tolerance():
    D1, D2 = synth.smooth_pair(23, 96, 128, 24)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.frm_match(dev(a), dev(b), 8, 10, with_seed_state=True)
    _frm_tolerant(a, b, 8, 10, r)


def test_frm_full_size_fp16():
    """512x384, d=24, stride 8, max_iter 10: the whole oracle run (seconds on the host)."""
    w = synth.WORKLOADS["frm_512x384"]
    D1, D2 = synth.make_workload(w)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.frm_match(dev(a), dev(b), w.seed_stride, w.max_iter, with_seed_state=True)
    _frm_tolerant(a, b, w.seed_stride, w.max_iter, r)


def test_frm_batched_matches_oracle_per_pair():
    B, H, W, d = 5, 40, 56, 16
    maps = [synth.quantised_pair(300 + i, H, W, H, W, d) for i in range(B)]
    a = torch.stack([synth.to_storage(m[0], "f16") for m in maps])
    b = torch.stack([synth.to_storage(m[1], "f16") for m in maps])
    r = rnn.frm_match_batched(dev(a), dev(b), 4, 10, with_seed_state=True)
    for i in range(B):
        ref = oracle.frm(a[i], b[i], 4, 10)
        got = r.pairs[i, : int(r.count[i])].cpu().numpy()
        assert np.array_equal(got, ref.pairs.reshape(-1, 2)), i
        u, v, q, c = seed_state_np(r, i)
        assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)


def test_frm_batched_strided_padded_maps():
    """d = 24 (copied into zero-padded 32-wide rows) with batch strides wider
    than H*W*d, through the C ABI; every pair against the oracle."""
    B, H, W, d, S, it = 3, 24, 40, 24, 4, 10
    gap = 8 * 5                                   # elements between consecutive maps
    lib = rnn._lib.load()
    maps = [synth.quantised_pair(400 + i, H, W, H, W, d) for i in range(B)]
    n = H * W * d
    a = torch.zeros(B * (n + gap), dtype=torch.float16)
    b = torch.zeros(B * (n + gap), dtype=torch.float16)
    for i, (m1, m2) in enumerate(maps):
        a[i * (n + gap): i * (n + gap) + n] = synth.to_storage(m1, "f16").reshape(-1)
        b[i * (n + gap): i * (n + gap) + n] = synth.to_storage(m2, "f16").reshape(-1)
    a, b = dev(a), dev(b)
    k = int(lib.rnn_frm_num_seeds(H, W, S))
    cap = int(lib.rnn_frm_max_pairs(H, W, H, W, S))
    pairs = torch.empty((B, cap, 2), dtype=torch.int32, device="cuda")
    count = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(lib.rnn_frm_workspace_size(B, H, W, H, W, d, S), dtype=torch.uint8,
                     device="cuda")
    rnn._lib.check(lib.rnn_frm_match_batched(
        B, a.data_ptr(), n + gap, b.data_ptr(), n + gap, H, W, H, W, d, 0, S, it,
        pairs.data_ptr(), cap, count.data_ptr(), None, ws.data_ptr(), ws.numel(),
        torch.cuda.current_stream().cuda_stream), "rnn_frm_match_batched")
    torch.cuda.synchronize()
    assert k > 0
    for i, (m1, m2) in enumerate(maps):
        ref = oracle.frm(synth.to_storage(m1, "f16"), synth.to_storage(m2, "f16"), S, it)
        got = pairs[i, : int(count[i])].cpu().numpy()
        assert np.array_equal(got, ref.pairs.reshape(-1, 2)), i


def test_frm_batched_workload_sampled_pairs():
    """The 64-pair 512x288 workload in one launch sequence; two pairs checked."""
    w = synth.WORKLOADS["frm_batched_64x512x288"]
    a, b = synth.make_workload_storage(w, "f16", workers=os.cpu_count() or 1)
    r = rnn.frm_match_batched(dev(a), dev(b), w.seed_stride, w.max_iter, with_seed_state=True)
    for i in (0, w.pairs - 1):
        _frm_tolerant(a[i], b[i], w.seed_stride, w.max_iter, r, i)


def test_repeat_runs_are_identical():
    w = synth.WORKLOADS["frm_512x384"]
    D1, D2 = synth.make_workload(w)
    a, b = dev(synth.to_storage(D1, "f16")), dev(synth.to_storage(D2, "f16"))
    outs = [rnn.frm_match(a, b, 8, 10, with_seed_state=True) for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.seed_state, outs[0].seed_state)
        assert torch.equal(o.trimmed(), outs[0].trimmed())
    m = [rnn.mnn_exhaustive(a[:96], b[:96], with_nn=True) for _ in range(3)]
    for o in m[1:]:
        assert torch.equal(o.rowarg, m[0].rowarg) and torch.equal(o.colarg, m[0].colarg)


def test_workspace_status_ok_after_calls():
    a = dev(synth.to_storage(synth.quantised_pair(1, 16, 16, 16, 16, 16)[0], "f16"))
    ws = torch.empty(rnn._lib.load().rnn_frm_workspace_size(1, 16, 16, 16, 16, 16, 2),
                     dtype=torch.uint8, device="cuda")
    rnn.frm_match(a, a, 2, 10, workspace=ws)
    rnn.workspace_status(ws)


def test_frm_large_map_fp16():
    """1024x768 maps, d = 32, 2 % outlier pixels, stride 8 (12 288 seeds),
    max_iter 15: the whole oracle run."""
    w = synth.WORKLOADS["frm_1024x768"]
    D1, D2 = synth.make_workload(w)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.frm_match(dev(a), dev(b), w.seed_stride, w.max_iter, with_seed_state=True)
    # at 786 432 candidates about a tenth of the trajectories pass a top-2 gap
    # below 1e-3 somewhere; those are held to the tolerance rule, the rest
    # must match exactly
    _frm_tolerant(a, b, w.seed_stride, w.max_iter, r)
    assert int(r.count[0]) > 1000


def test_mnn_coarse_tokens_fp16():
    """The coarse reciprocal set on 80x64 tokens, d = 256, fp16 unit vectors."""
    w = synth.WORKLOADS["mnn_coarse_80x64"]
    D1, D2 = synth.make_workload(w)
    a, b = synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")
    r = rnn.mnn_exhaustive(dev(a), dev(b), with_nn=True)
    ref = oracle.mnn(a, b)
    A, B = a.reshape(-1, w.d), b.reshape(-1, w.d)
    check_nn_tolerant(A, B, r.rowarg.cpu().numpy(), r.rowmax.cpu().numpy(), ref.row)
    check_nn_tolerant(B, A, r.colarg.cpu().numpy(), r.colmax.cpu().numpy(), ref.col)
    assert check_mnn_tolerant(r.trimmed().cpu().numpy(), ref) <= 5
    assert len(ref.pairs) > 1000


def test_repeat_runs_are_identical_other_paths():
    """Deterministic reductions: three runs of coarse-to-fine, point-map FRM
    and the Euclidean exhaustive set give identical bits (a race would show
    as run-to-run differences)."""
    w = synth.WORKLOADS["frm_512x384"]
    D1, D2 = synth.make_workload(w)
    a, b = dev(synth.to_storage(D1, "f16")), dev(synth.to_storage(D2, "f16"))
    C1 = dev(synth.to_storage(synth.coarse_map(D1, 48, 64), "f16"))
    C2 = dev(synth.to_storage(synth.coarse_map(D2, 48, 64), "f16"))
    c = [rnn.c2f_match(C1, C2, a, b, crop=(192, 256), seed_stride=4) for _ in range(3)]
    for o in c[1:]:
        assert torch.equal(o.trimmed(), c[0].trimmed()) and torch.equal(o.crops, c[0].crops)
    P1, P2 = synth.pointmap_pair(9, w.H, w.W)
    p1 = torch.from_numpy(P1.astype(np.float32)).cuda()
    p2 = torch.from_numpy(P2.astype(np.float32)).cuda()
    f = [rnn.pts_frm_match(p1, p2, seed_stride=8, with_seed_state=True) for _ in range(3)]
    for o in f[1:]:
        assert torch.equal(o.seed_state, f[0].seed_state)
        assert torch.equal(o.trimmed(), f[0].trimmed())
    m = [rnn.mnn_exhaustive(a[:128], b[:128], with_nn=True, metric="l2") for _ in range(3)]
    for o in m[1:]:
        assert torch.equal(o.rowmax, m[0].rowmax) and torch.equal(o.colarg, m[0].colarg)
        assert torch.equal(o.trimmed(), m[0].trimmed())
