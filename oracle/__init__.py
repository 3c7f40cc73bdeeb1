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
* ``c2f_crops`` / ``c2f``: coarse-to-fine matching (cv-learn.com "MASt3R"
  note, paragraph "Coarse-to-fine matching"; staskaer.github.io blog, the
  step after FRM that returns to full resolution and matches again block by
  block): the reciprocal set of the coarse maps, crops of image 1 on a grid,
  each paired with a crop of image 2 centred on its coarse matches, FRM per
  crop pair on the full-resolution maps, and the matches mapped back.  The
  pages give no formulas for the crops; the integer rules written out in
  ``c2f_crops`` are this implementation's reading.
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


# --------------------------------------------------------- coarse-to-fine

def c2f_crop_origins(L: int, c: int) -> list:
    """Origins of the ceil(L/c) crops of length c that cover [0, L), the first
    at 0 and the last at L - c, spread evenly (floor)."""
    n = -(-L // c)
    if n <= 1:
        return [0]
    return [(a * (L - c)) // (n - 1) for a in range(n)]


def c2f_fine_pixel(i: int, Hc: int, Wc: int, H: int, W: int):
    """Full-resolution (y, x) of the centre of coarse pixel i = yc*Wc + xc:
    floor((2*yc + 1) * H / (2*Hc)), floor((2*xc + 1) * W / (2*Wc))."""
    yc, xc = divmod(int(i), Wc)
    return ((2 * yc + 1) * H) // (2 * Hc), ((2 * xc + 1) * W) // (2 * Wc)


def c2f_crop_size(H1, W1, H2, W2, crop):
    ch, cw = crop
    return min(ch, H1, H2), min(cw, W1, W2)


def c2f_crops(coarse_pairs, Hc1, Wc1, Hc2, Wc2, H1, W1, H2, W2, crop, min_coarse=1):
    """Crop table ``int32 [n][6]``: y0_1, x0_1, y0_2, x0_2, n_coarse, on.

    Crops of image 1 are the row-major grid of ``c2f_crop_origins`` along each
    axis.  A coarse pair (i, j) belongs to crop b when the full-resolution
    pixel of i lies inside it.  With n >= min_coarse such pairs, crop b is on
    and its image-2 crop is centred on the floor of the mean full-resolution
    position of their j, clamped into image 2; otherwise it is off (origin
    0, 0) and is not matched."""
    ch, cw = c2f_crop_size(H1, W1, H2, W2, crop)
    ys, xs = c2f_crop_origins(H1, ch), c2f_crop_origins(W1, cw)
    p1 = [c2f_fine_pixel(i, Hc1, Wc1, H1, W1) for i, _ in coarse_pairs]
    p2 = [c2f_fine_pixel(j, Hc2, Wc2, H2, W2) for _, j in coarse_pairs]
    rows = []
    for y0 in ys:
        for x0 in xs:
            inside = [t for t, (y, x) in enumerate(p1) if y0 <= y < y0 + ch and x0 <= x < x0 + cw]
            n = len(inside)
            if n >= max(min_coarse, 1):
                cy = sum(p2[t][0] for t in inside) // n
                cx = sum(p2[t][1] for t in inside) // n
                y2 = min(max(cy - ch // 2, 0), H2 - ch)
                x2 = min(max(cx - cw // 2, 0), W2 - cw)
                rows.append((y0, x0, y2, x2, n, 1))
            else:
                rows.append((y0, x0, 0, 0, n, 0))
    return np.array(rows, dtype=np.int32).reshape(-1, 6)


@dataclass
class C2FResult:
    pairs: np.ndarray    # int32 [n][2] full-resolution (u, v), one per u, sorted by u
    crops: np.ndarray    # int32 [ncrops][6] (see c2f_crops)
    coarse: np.ndarray   # int32 [m][2] reciprocal pairs of the coarse maps


def c2f(C1, C2, F1, F2, crop=(384, 512), seed_stride: int = 8, max_iter: int = 10,
        min_coarse: int = 1, metric: str = "dot", threads: int = 0) -> C2FResult:
    """Coarse-to-fine matching of full-resolution maps F1, F2 ``[H][W][d]``
    guided by coarse maps C1, C2 ``[Hc][Wc][dc]``: M of the coarse maps
    (``mnn``), the crop table (``c2f_crops``), FRM with grid seeds of stride
    ``seed_stride`` on every crop pair that is on (``frm_ex``), each pair
    mapped back by its crops' origins; where crops overlap, the first crop
    in table order that outputs an image-1 pixel gives its pair."""
    c1, c2 = as_f64(C1), as_f64(C2)
    f1, f2 = as_f64(F1), as_f64(F2)
    Hc1, Wc1, _ = c1.shape
    Hc2, Wc2, _ = c2.shape
    H1, W1, _ = f1.shape
    H2, W2, _ = f2.shape
    coarse = mnn(c1, c2, threads=threads, metric=metric).pairs
    crops = c2f_crops(coarse.tolist(), Hc1, Wc1, Hc2, Wc2, H1, W1, H2, W2, crop, min_coarse)
    ch, cw = c2f_crop_size(H1, W1, H2, W2, crop)
    best = {}
    for y0, x0, y2, x2, _, on in crops.tolist():
        if not on:
            continue
        a = f1[y0:y0 + ch, x0:x0 + cw]
        b = f2[y2:y2 + ch, x2:x2 + cw]
        r = frm_ex(a, b, seed_stride, max_iter, metric=metric, threads=threads)
        for u, v in r.pairs.tolist():
            gu = (y0 + u // cw) * W1 + (x0 + u % cw)
            gv = (y2 + v // cw) * W2 + (x2 + v % cw)
            if gu not in best:
                best[gu] = gv
    pairs = np.array(sorted(best.items()), dtype=np.int32).reshape(-1, 2)
    return C2FResult(pairs, crops, coarse)
