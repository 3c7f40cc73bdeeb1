"""Double-precision CPU oracle for reciprocal nearest-neighbour matching.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``reciprocal_nearest_neighbour_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``rnn_oracle.c`` (plain C, double precision, OpenMP
over independent queries); this module compiles it with gcc on first use and
marshals numpy arrays in and out.  Inputs may be numpy arrays of any float
type or CPU torch tensors (fp16/bf16 are converted to double exactly).

What each function computes, with its source:

* ``nn``: nearest neighbour = the lowest index with the largest dot product
  (cv-learn.com "MASt3R" note, paragraph "Fast reciprocal matching (FRM)":
  NN1/NN2; the argmax and tie readings are stated in the C file).
* ``mnn``: the reciprocal set M = {(i,j) | j = NN2(D1_i) and i = NN1(D2_j)}
  (same paragraph).
* ``frm_seeds`` / ``frm``: Fast Reciprocal Matching as the quoted
  ``fast_reciprocal_NNs`` runs it (staskaer.github.io blog on DUSt3R/MASt3R,
  MASt3R matching section): grid seeds, two half-steps with their tests,
  ``max_iter`` cap, unique sorted output.
* ``frm_ex``: the same function's other options: given start pixels (made
  unique and sorted), the ``pixel_tol`` convergence rule that returns the
  start pixel, the basin output, and the Euclidean-distance metric of its
  brute-force matcher (``metric="l2"``; also for ``nn`` and ``mnn``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rnn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math"]

_lib = None


def build(force: bool = False) -> str:
    """Compile ``rnn_oracle.c`` into ``liboracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def compiler_flags() -> str:
    return "gcc " + " ".join(_CFLAGS)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_nn.argtypes = [P, i64, P, i64, i32, P, P, P, i32]
    lib.oracle_nn.restype = None
    lib.oracle_pair_scores.argtypes = [P, P, i32, P, P, i64, P]
    lib.oracle_pair_scores.restype = None
    lib.oracle_mnn.argtypes = [P, i64, P, i64, i32, P, P, P, P, P, P, P, i32]
    lib.oracle_mnn.restype = ctypes.c_int64
    lib.oracle_frm_seeds.argtypes = [i32, i32, i32, P]
    lib.oracle_frm_seeds.restype = ctypes.c_int64
    lib.oracle_frm.argtypes = [P, i32, i32, P, i32, i32, i32, i32, i32, P, P, P, P, P, P, P,
                               P, i32]
    lib.oracle_frm.restype = ctypes.c_int64
    lib.oracle_nn_metric.argtypes = [P, i64, P, i64, i32, i32, P, P, P, i32]
    lib.oracle_nn_metric.restype = None
    lib.oracle_mnn_metric.argtypes = [P, i64, P, i64, i32, i32, P, P, P, P, P, P, P, i32]
    lib.oracle_mnn_metric.restype = ctypes.c_int64
    lib.oracle_frm_ex.argtypes = [P, i32, i32, P, i32, i32, i32, P, i64, i32, i32,
                                  ctypes.c_double, i32, i32, P, i64, P, P, P, P, P, P, i32]
    lib.oracle_frm_ex.restype = ctypes.c_int64
    _lib = lib
    return lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or CPU torch tensor."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _rows(x) -> np.ndarray:
    a = as_f64(x)
    return a.reshape(-1, a.shape[-1])


@dataclass
class NNResult:
    arg: np.ndarray      # int32 [nq]
    best: np.ndarray     # float64 [nq]
    second: np.ndarray   # float64 [nq] (best score over every other index)

    @property
    def gap(self) -> np.ndarray:
        return self.best - self.second


METRICS = {"dot": 0, "l2": 1}


def nn(Q, X, threads: int = 0, metric: str = "dot") -> NNResult:
    """Nearest neighbour of each row of Q in X, lowest index on ties: the
    largest dot product, or with ``metric="l2"`` the smallest Euclidean
    distance (``best``/``second`` are then negated squared distances)."""
    q, x = _rows(Q), _rows(X)
    assert q.shape[1] == x.shape[1]
    nq, nx, d = q.shape[0], x.shape[0], q.shape[1]
    arg = np.empty(nq, np.int32)
    best = np.empty(nq, np.float64)
    second = np.empty(nq, np.float64)
    if nq:
        _load().oracle_nn_metric(_ptr(q), nq, _ptr(x), nx, d, METRICS[metric], _ptr(arg),
                                 _ptr(best), _ptr(second), threads)
    return NNResult(arg, best, second)


def pair_scores(A, B, ia, ib) -> np.ndarray:
    """``s(ia[t], ib[t])`` between the rows of A and B, in double."""
    a, b = _rows(A), _rows(B)
    ia = np.ascontiguousarray(ia, dtype=np.int32)
    ib = np.ascontiguousarray(ib, dtype=np.int32)
    out = np.empty(len(ia), np.float64)
    if len(ia):
        _load().oracle_pair_scores(_ptr(a), _ptr(b), a.shape[1], _ptr(ia), _ptr(ib), len(ia),
                                   _ptr(out))
    return out


@dataclass
class MNNResult:
    pairs: np.ndarray    # int32 [|M|][2], increasing i
    row: NNResult        # NN2 of every D1 pixel
    col: NNResult        # NN1 of every D2 pixel


def mnn(D1, D2, threads: int = 0, metric: str = "dot") -> MNNResult:
    """The reciprocal nearest-neighbour set between two descriptor maps."""
    a, b = _rows(D1), _rows(D2)
    n1, n2, d = a.shape[0], b.shape[0], a.shape[1]
    pairs = np.empty((min(n1, n2), 2), np.int32)
    ra, ca = np.empty(n1, np.int32), np.empty(n2, np.int32)
    rb, rs = np.empty(n1), np.empty(n1)
    cb, cs = np.empty(n2), np.empty(n2)
    m = _load().oracle_mnn_metric(_ptr(a), n1, _ptr(b), n2, d, METRICS[metric], _ptr(pairs),
                                  _ptr(ra), _ptr(ca), _ptr(rb), _ptr(rs), _ptr(cb), _ptr(cs),
                                  threads)
    return MNNResult(pairs[:m].copy(), NNResult(ra, rb, rs), NNResult(ca, cb, cs))


def frm_seeds(H: int, W: int, S: int) -> np.ndarray:
    """Linear indices of the FRM grid seeds on an H x W image with stride S."""
    lib = _load()
    k = lib.oracle_frm_seeds(H, W, S, None)
    out = np.empty(k, np.int32)
    if k:
        lib.oracle_frm_seeds(H, W, S, _ptr(out))
    return out


@dataclass
class FRMResult:
    pairs: np.ndarray           # int32 [n][2], unique, sorted by U
    seeds: np.ndarray           # int32 [k]
    seed_u: np.ndarray          # int32 [k] final U
    seed_v: np.ndarray          # int32 [k] final V
    seed_queries: np.ndarray    # int32 [k] NN queries made for the seed
    seed_converged: np.ndarray  # bool  [k]
    seed_min_gap: np.ndarray    # float64 [k] smallest top-2 gap along the trajectory
    traj: np.ndarray            # int32 [k][max_iter][3] (U queried, V, U found)
    active_per_half: np.ndarray  # int64 [2*max_iter]


def frm(D1, D2, seed_stride: int = 8, max_iter: int = 10, threads: int = 0) -> FRMResult:
    """Fast Reciprocal Matching of two ``[H][W][d]`` maps."""
    a, b = as_f64(D1), as_f64(D2)
    H1, W1, d = a.shape
    H2, W2, d2 = b.shape
    assert d == d2
    a, b = a.reshape(-1, d), b.reshape(-1, d)
    seeds = frm_seeds(H1, W1, seed_stride)
    k = len(seeds)
    pairs = np.empty((max(k, 1), 2), np.int32)
    su, sv, sq = (np.empty(k, np.int32) for _ in range(3))
    sc = np.empty(k, np.uint8)
    sg = np.empty(k, np.float64)
    traj = np.empty((k, max_iter, 3), np.int32)
    aph = np.empty(2 * max_iter, np.int64)
    n = _load().oracle_frm(_ptr(a), H1, W1, _ptr(b), H2, W2, d, seed_stride, max_iter,
                           _ptr(pairs), _ptr(su), _ptr(sv), _ptr(sq), _ptr(sc), _ptr(sg),
                           _ptr(traj), _ptr(aph), threads)
    return FRMResult(pairs[:n].copy(), seeds, su, sv, sq, sc.astype(bool), sg, traj, aph)


@dataclass
class FRMExResult:
    pairs: np.ndarray           # int32 [n][2], unique, sorted
    seeds: np.ndarray           # int32 [k] start pixels, ascending
    seed_u: np.ndarray          # int32 [k] final U
    seed_v: np.ndarray          # int32 [k] final V
    seed_queries: np.ndarray    # int32 [k]
    seed_converged: np.ndarray  # bool  [k]
    basin: np.ndarray           # int32 [H1*W1 + 1] or None


def frm_ex(D1, D2, seed_stride: int = 8, max_iter: int = 10, init=None,
           pixel_tol: float = 0.0, basin: bool = False, metric: str = "dot",
           threads: int = 0) -> FRMExResult:
    """Fast Reciprocal Matching with the quoted function's options: start
    pixels ``init`` (linear indices; None = the grid), ``pixel_tol``, basin
    mode, metric."""
    a, b = as_f64(D1), as_f64(D2)
    H1, W1, d = a.shape
    H2, W2, d2 = b.shape
    assert d == d2
    a, b = a.reshape(-1, d), b.reshape(-1, d)
    if init is not None:
        init = np.ascontiguousarray(np.asarray(init, dtype=np.int32).reshape(-1))
        seeds = np.unique(init)
    else:
        seeds = frm_seeds(H1, W1, seed_stride)
    k = len(seeds)
    pairs = np.empty((max(k, 1), 2), np.int32)
    su, sv, sq = (np.empty(max(k, 1), np.int32) for _ in range(3))
    sc = np.empty(max(k, 1), np.uint8)
    bas = np.empty(H1 * W1 + 1, np.int32) if basin else None
    ns = ctypes.c_int64(0)
    n = _load().oracle_frm_ex(_ptr(a), H1, W1, _ptr(b), H2, W2, d,
                              _ptr(init) if init is not None else None,
                              len(init) if init is not None else 0, seed_stride, max_iter,
                              float(pixel_tol), int(bool(basin)), METRICS[metric], _ptr(pairs),
                              len(pairs), _ptr(su), _ptr(sv), _ptr(sq), _ptr(sc),
                              _ptr(bas) if bas is not None else None, ctypes.byref(ns),
                              threads)
    assert ns.value == k
    return FRMExResult(pairs[:n].copy(), seeds, su[:k], sv[:k], sq[:k], sc[:k].astype(bool),
                       bas)


def frm_refine(D1, D2, init, pixel_tol: float = 0.0, metric: str = "dot",
               threads: int = 0) -> FRMExResult:
    """The quoted function called with start pixels: one iteration
    (``max_iter`` = 1), the ``pixel_tol`` rule, (start, match) pairs."""
    return frm_ex(D1, D2, init=init, max_iter=1, pixel_tol=pixel_tol, metric=metric,
                  threads=threads)
