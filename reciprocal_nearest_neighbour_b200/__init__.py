"""Reciprocal nearest-neighbour matching on B200 (sm_100a).

Thin PyTorch binding of ``librnn.so`` (C ABI in ``include/rnn.h``): it checks
shapes, allocates outputs and workspaces with torch (device memory only) and
passes raw pointers and the current CUDA stream.  Every step of the matching
runs in the library's CUDA kernels; there is no CPU path.

Descriptor maps are ``[H, W, d]`` (or ``[B, H, W, d]`` for the batched FRM)
contiguous fp16/bf16 CUDA tensors; pixel index ``p = y*W + x``.

* ``nn_argmax(Q, X)``: NN of every query row among the rows of X (largest dot
  product, lowest index on ties) and its score.
* ``mnn_exhaustive(D1, D2)``: the reciprocal set
  M = {(i, j) | j = NN2(D1_i) and i = NN1(D2_j)} (cv-learn.com "MASt3R"
  note, paragraph "Fast reciprocal matching (FRM)").
* ``frm_match`` / ``frm_match_batched``: Fast Reciprocal Matching from grid
  seeds, with the loop of the quoted ``fast_reciprocal_NNs``
  (staskaer.github.io DUSt3R/MASt3R blog, MASt3R matching section).
* ``frm_match_ex`` / ``frm_refine``: the same function's other options: given
  start pixels, the pixel tolerance, the basin output.
* ``metric="l2"`` (``nn_argmax``, ``mnn_exhaustive``, ``frm_match_ex``,
  ``frm_refine``): the smallest Euclidean distance instead of the largest dot
  product; scores are then squared distances.
* ``c2f_match``: coarse-to-fine matching: the reciprocal set of coarse maps
  places crop pairs, FRM runs on the full-resolution windows, and the pairs
  are mapped back (cv-learn.com "MASt3R" note, "Coarse-to-fine matching").
* ``pts_nn`` / ``pts_mnn`` / ``pts_frm_match``: the same operations on 3-D
  points (fp32 ``[..., 3]``), where MASt3R's NN function is the exact nearest
  point in Euclidean distance (a K-d tree query in its reference code).

Results stay on the device; pair lists come back as ``(pairs, count)`` with
``pairs`` a ``[cap, 2]`` int32 buffer and ``count`` a device int32 tensor;
``trim(pairs, count)`` cuts the buffer to length (this synchronises).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import RNNError, RNNLibraryError  # noqa: F401

__all__ = [
    "nn_argmax", "mnn_exhaustive", "frm_match", "frm_match_batched", "frm_num_seeds",
    "frm_max_pairs", "workspace_status", "trim", "MNNResult", "FRMResult", "RNNError",
    "RNNLibraryError", "FRMPlan", "frm_match_ex", "frm_refine", "pts_nn", "pts_mnn",
    "pts_frm_match", "c2f_match", "C2FResult", "mnn_mutual", "FRMGraph",
]

_DT = {torch.float16: _lib.RNN_F16, torch.bfloat16: _lib.RNN_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"descriptors must be float16 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


def _check_map(t: torch.Tensor, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns blocks aligned to at least 512 bytes
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def workspace_status(workspace: torch.Tensor) -> None:
    """Raise RNNError(RNN_ETIMEOUT) if the last call on `workspace` gave up on a wait."""
    lib = _lib.load()
    _lib.check(lib.rnn_workspace_status(workspace.data_ptr(), _stream(workspace)),
               "rnn_workspace_status")


def trim(pairs: torch.Tensor, count: torch.Tensor) -> torch.Tensor:
    """``pairs[:count]`` (reads the count back to the host)."""
    return pairs[: int(count.reshape(-1)[0].item())]


def _metric(metric: str) -> int:
    if metric not in _lib.METRICS:
        raise ValueError(f"metric must be one of {sorted(_lib.METRICS)}, got {metric!r}")
    return _lib.METRICS[metric]


def nn_argmax(Q: torch.Tensor, X: torch.Tensor, *, workspace: Optional[torch.Tensor] = None,
              idx_out: Optional[torch.Tensor] = None, score_out: Optional[torch.Tensor] = None,
              with_scores: bool = True, metric: str = "dot"):
    """NN of each row of ``Q [nq, d]`` among the rows of ``X [nx, d]``.

    Returns ``(idx int32 [nq], score float32 [nq] or None)``; with
    ``metric="l2"`` the score is the squared distance.
    """
    _check_map(Q, "Q", 2)
    _check_map(X, "X", 2)
    if Q.dtype != X.dtype or Q.shape[1] != X.shape[1]:
        raise ValueError("Q and X must share dtype and d")
    lib = _lib.load()
    nq, d = Q.shape
    nx = X.shape[0]
    dev = Q.device
    if idx_out is None:
        idx_out = torch.empty(nq, dtype=torch.int32, device=dev)
    if score_out is None and with_scores:
        score_out = torch.empty(nq, dtype=torch.float32, device=dev)
    m = _metric(metric)
    need = lib.rnn_nn_workspace_size_ex(nq, nx, d, m)
    if workspace is None:
        workspace = _workspace(need, dev)
    _lib.check(lib.rnn_nn_argmax_ex(Q.data_ptr(), nq, X.data_ptr(), nx, d, _dtype_code(Q), m,
                                    idx_out.data_ptr(), _ptr(score_out), workspace.data_ptr(),
                                    workspace.numel(), _stream(Q)), "rnn_nn_argmax_ex")
    return idx_out, score_out


@dataclass
class MNNResult:
    pairs: torch.Tensor            # [cap, 2] int32 buffer; the first `count` rows hold M
    count: torch.Tensor            # [1] int32 on the device
    rowarg: Optional[torch.Tensor] = None   # [H1*W1] NN2 of every D1 pixel
    rowmax: Optional[torch.Tensor] = None
    colarg: Optional[torch.Tensor] = None   # [H2*W2] NN1 of every D2 pixel
    colmax: Optional[torch.Tensor] = None

    def trimmed(self) -> torch.Tensor:
        return trim(self.pairs, self.count)


def mnn_exhaustive(D1: torch.Tensor, D2: torch.Tensor, *, with_nn: bool = False,
                   workspace: Optional[torch.Tensor] = None,
                   out: Optional[MNNResult] = None, metric: str = "dot") -> MNNResult:
    """Exhaustive reciprocal NN set between ``D1 [H1, W1, d]`` and ``D2 [H2, W2, d]``."""
    _check_map(D1, "D1", 3)
    _check_map(D2, "D2", 3)
    if D1.dtype != D2.dtype or D1.shape[2] != D2.shape[2]:
        raise ValueError("D1 and D2 must share dtype and d")
    lib = _lib.load()
    H1, W1, d = D1.shape
    H2, W2, _ = D2.shape
    n1, n2 = H1 * W1, H2 * W2
    dev = D1.device
    if out is None:
        out = MNNResult(torch.empty((min(n1, n2), 2), dtype=torch.int32, device=dev),
                        torch.zeros(1, dtype=torch.int32, device=dev))
        if with_nn:
            out.rowarg = torch.empty(n1, dtype=torch.int32, device=dev)
            out.rowmax = torch.empty(n1, dtype=torch.float32, device=dev)
            out.colarg = torch.empty(n2, dtype=torch.int32, device=dev)
            out.colmax = torch.empty(n2, dtype=torch.float32, device=dev)
    m = _metric(metric)
    need = lib.rnn_mnn_workspace_size_ex(H1, W1, H2, W2, d, m)
    if workspace is None:
        workspace = _workspace(need, dev)
    _lib.check(lib.rnn_mnn_exhaustive_ex(
        D1.data_ptr(), H1, W1, D2.data_ptr(), H2, W2, d, _dtype_code(D1), m,
        out.pairs.data_ptr(), out.pairs.shape[0], out.count.data_ptr(), _ptr(out.rowarg),
        _ptr(out.rowmax), _ptr(out.colarg), _ptr(out.colmax), workspace.data_ptr(),
        workspace.numel(), _stream(D1)), "rnn_mnn_exhaustive_ex")
    return out


def mnn_mutual(rowarg: torch.Tensor, colarg: torch.Tensor, *,
               workspace: Optional[torch.Tensor] = None):
    """The reciprocal set from NN arrays: ``(i, rowarg[i])`` for every i with
    ``colarg[rowarg[i]] == i``, in increasing i.  ``rowarg`` (NN2 of every
    image-1 pixel) and ``colarg`` (NN1 of every image-2 pixel) are int32 CUDA
    tensors.  Returns ``(pairs [min(n1, n2), 2], count [1])``."""
    for t, n in ((rowarg, "rowarg"), (colarg, "colarg")):
        _check_map(t, n, 1)
        if t.dtype != torch.int32:
            raise ValueError(f"{n} must be int32")
    lib = _lib.load()
    n1, n2 = rowarg.numel(), colarg.numel()
    dev = rowarg.device
    pairs = torch.empty((max(1, min(n1, n2)), 2), dtype=torch.int32, device=dev)
    count = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _workspace(lib.rnn_mnn_mutual_workspace_size(n1), dev)
    _lib.check(lib.rnn_mnn_mutual(rowarg.data_ptr(), n1, colarg.data_ptr(), n2, pairs.data_ptr(),
                                  pairs.shape[0], count.data_ptr(), workspace.data_ptr(),
                                  workspace.numel(), _stream(rowarg)), "rnn_mnn_mutual")
    return pairs, count


def frm_num_seeds(H1: int, W1: int, seed_stride: int) -> int:
    return int(_lib.load().rnn_frm_num_seeds(H1, W1, seed_stride))


def frm_max_pairs(H1: int, W1: int, H2: int, W2: int, seed_stride: int) -> int:
    return int(_lib.load().rnn_frm_max_pairs(H1, W1, H2, W2, seed_stride))


@dataclass
class FRMResult:
    pairs: torch.Tensor                      # [B, cap, 2] int32 (B = 1 for frm_match)
    count: torch.Tensor                      # [B] int32 on the device
    seed_state: Optional[torch.Tensor] = None  # [B, k, 4]: U, V, queries, converged
    basin: Optional[torch.Tensor] = None       # [B, H1*W1 + 1] (basin mode)

    def trimmed(self, b: int = 0) -> torch.Tensor:
        return self.pairs[b, : int(self.count[b].item())]


class FRMPlan:
    """Preallocated workspace and outputs for repeated FRM calls of one shape.

    ``plan.run(D1, D2)`` only marshals pointers into the ABI, so it can be
    captured in a CUDA graph.
    """

    def __init__(self, B: int, H1: int, W1: int, H2: int, W2: int, d: int, dtype: torch.dtype,
                 seed_stride: int = 8, max_iter: int = 10, device="cuda",
                 with_seed_state: bool = False):
        lib = _lib.load()
        self.B, self.H1, self.W1, self.H2, self.W2, self.d = B, H1, W1, H2, W2, d
        self.dtype, self.seed_stride, self.max_iter = dtype, seed_stride, max_iter
        self.k = int(lib.rnn_frm_num_seeds(H1, W1, seed_stride))
        self.cap = max(1, int(lib.rnn_frm_max_pairs(H1, W1, H2, W2, seed_stride)))
        dev = torch.device(device)
        self.workspace = _workspace(
            lib.rnn_frm_workspace_size(B, H1, W1, H2, W2, d, seed_stride), dev)
        self.result = FRMResult(
            torch.empty((B, self.cap, 2), dtype=torch.int32, device=dev),
            torch.zeros(B, dtype=torch.int32, device=dev),
            torch.empty((B, max(self.k, 1), 4), dtype=torch.int32, device=dev)
            if with_seed_state else None)

    def run(self, D1: torch.Tensor, D2: torch.Tensor) -> FRMResult:
        batched = D1.dim() == 4
        _check_map(D1, "D1", 4 if batched else 3)
        _check_map(D2, "D2", 4 if batched else 3)
        B = D1.shape[0] if batched else 1
        if (B, *D1.shape[-3:]) != (self.B, self.H1, self.W1, self.d) or \
                tuple(D2.shape[-3:]) != (self.H2, self.W2, self.d) or \
                (batched and D2.shape[0] != B):
            raise ValueError("maps do not match the plan's shape")
        if D1.dtype != self.dtype or D2.dtype != self.dtype:
            raise ValueError("maps do not match the plan's dtype")
        lib = _lib.load()
        r = self.result
        n1, n2 = self.H1 * self.W1 * self.d, self.H2 * self.W2 * self.d
        _lib.check(lib.rnn_frm_match_batched(
            B, D1.data_ptr(), n1, D2.data_ptr(), n2, self.H1, self.W1, self.H2, self.W2, self.d,
            _DT[self.dtype], self.seed_stride, self.max_iter, r.pairs.data_ptr(), self.cap,
            r.count.data_ptr(), _ptr(r.seed_state), self.workspace.data_ptr(),
            self.workspace.numel(), _stream(D1)), "rnn_frm_match_batched")
        return r


def frm_match(D1: torch.Tensor, D2: torch.Tensor, seed_stride: int = 8, max_iter: int = 10, *,
              with_seed_state: bool = False, workspace: Optional[torch.Tensor] = None
              ) -> FRMResult:
    """Fast Reciprocal Matching of ``D1 [H1, W1, d]`` against ``D2 [H2, W2, d]``."""
    _check_map(D1, "D1", 3)
    _check_map(D2, "D2", 3)
    if D1.dtype != D2.dtype or D1.shape[2] != D2.shape[2]:
        raise ValueError("D1 and D2 must share dtype and d")
    lib = _lib.load()
    H1, W1, d = D1.shape
    H2, W2, _ = D2.shape
    dev = D1.device
    k = int(lib.rnn_frm_num_seeds(H1, W1, seed_stride)) if seed_stride >= 1 else 0
    cap = max(1, int(lib.rnn_frm_max_pairs(H1, W1, H2, W2, seed_stride)) if seed_stride >= 1
              else 1)
    out = FRMResult(torch.empty((1, cap, 2), dtype=torch.int32, device=dev),
                    torch.zeros(1, dtype=torch.int32, device=dev),
                    torch.empty((1, max(k, 1), 4), dtype=torch.int32, device=dev)
                    if with_seed_state else None)
    if workspace is None:
        workspace = _workspace(lib.rnn_frm_workspace_size(1, H1, W1, H2, W2, d, seed_stride),
                               dev)
    _lib.check(lib.rnn_frm_match(
        D1.data_ptr(), H1, W1, D2.data_ptr(), H2, W2, d, _dtype_code(D1), seed_stride, max_iter,
        out.pairs.data_ptr(), cap, out.count.data_ptr(), _ptr(out.seed_state),
        workspace.data_ptr(), workspace.numel(), _stream(D1)), "rnn_frm_match")
    return out


def frm_match_batched(D1: torch.Tensor, D2: torch.Tensor, seed_stride: int = 8,
                      max_iter: int = 10, *, with_seed_state: bool = False) -> FRMResult:
    """FRM over ``B`` independent pairs: ``D1 [B, H1, W1, d]``, ``D2 [B, H2, W2, d]``."""
    _check_map(D1, "D1", 4)
    _check_map(D2, "D2", 4)
    if D1.shape[0] != D2.shape[0] or D1.dtype != D2.dtype or D1.shape[3] != D2.shape[3]:
        raise ValueError("D1 and D2 must share B, dtype and d")
    B, H1, W1, d = D1.shape
    _, H2, W2, _ = D2.shape
    plan = FRMPlan(B, H1, W1, H2, W2, d, D1.dtype, seed_stride, max_iter, D1.device,
                   with_seed_state)
    return plan.run(D1, D2)


def frm_match_ex(D1: torch.Tensor, D2: torch.Tensor, *, seed_stride: int = 8,
                 max_iter: int = 10, metric: str = "dot", init: Optional[torch.Tensor] = None,
                 pixel_tol: float = 0.0, with_basin: bool = False,
                 with_seed_state: bool = False,
                 workspace: Optional[torch.Tensor] = None) -> FRMResult:
    """FRM with every option of the quoted ``fast_reciprocal_NNs``.

    ``D1``/``D2`` are ``[H, W, d]`` or ``[B, H, W, d]``.  ``init`` (CUDA int32,
    ``[n]`` or ``[B, n]``) gives the start pixels ``y*W1 + x`` instead of the
    grid; ``pixel_tol > 0`` (only with ``init``) outputs ``(start, match)``
    for the starts whose round trip lands closer than ``pixel_tol`` pixels;
    ``with_basin`` returns ``basin [B, H1*W1 + 1]`` (basin[p] = the pixel a
    round trip from p returned to, -1 if never visited).
    """
    batched = D1.dim() == 4
    _check_map(D1, "D1", 4 if batched else 3)
    _check_map(D2, "D2", 4 if batched else 3)
    if D1.dtype != D2.dtype or D1.shape[-1] != D2.shape[-1]:
        raise ValueError("D1 and D2 must share dtype and d")
    if batched and D1.shape[0] != D2.shape[0]:
        raise ValueError("D1 and D2 must share B")
    B = D1.shape[0] if batched else 1
    H1, W1, d = D1.shape[-3:]
    H2, W2, _ = D2.shape[-3:]
    lib = _lib.load()
    m = _metric(metric)
    dev = D1.device
    n_init = -1
    if init is not None:
        if not isinstance(init, torch.Tensor) or not init.is_cuda or init.dtype != torch.int32:
            raise ValueError("init must be a CUDA int32 tensor")
        init = init.reshape(B, -1).contiguous()
        n_init = init.shape[1]
        k = n_init
    else:
        k = int(lib.rnn_frm_num_seeds(H1, W1, seed_stride)) if seed_stride >= 1 else 0
    n2 = H2 * W2
    cap = max(1, k if pixel_tol > 0 else min(k, n2))
    out = FRMResult(torch.empty((B, cap, 2), dtype=torch.int32, device=dev),
                    torch.zeros(B, dtype=torch.int32, device=dev),
                    torch.empty((B, max(k, 1), 4), dtype=torch.int32, device=dev)
                    if with_seed_state else None,
                    torch.empty((B, H1 * W1 + 1), dtype=torch.int32, device=dev)
                    if with_basin else None)
    if workspace is None:
        workspace = _workspace(lib.rnn_frm_workspace_size_ex(B, H1, W1, H2, W2, d, m,
                                                             seed_stride, n_init), dev)
    _lib.check(lib.rnn_frm_match_ex(
        B, D1.data_ptr(), H1 * W1 * d, D2.data_ptr(), H2 * W2 * d, H1, W1, H2, W2, d,
        _dtype_code(D1), m, _ptr(init), max(n_init, 0), seed_stride, max_iter,
        float(pixel_tol), out.pairs.data_ptr(), cap, out.count.data_ptr(),
        _ptr(out.seed_state), _ptr(out.basin), workspace.data_ptr(), workspace.numel(),
        _stream(D1)), "rnn_frm_match_ex")
    return out


class FRMGraph:
    """FRM of two resident maps recorded once as a CUDA graph plan.

    ``FRMGraph(D1, D2, ...)`` takes the arguments of :func:`frm_match_ex`
    (without ``workspace``); ``launch()`` re-runs the match on the current
    contents of ``D1``/``D2`` into the same output tensors, on the current
    stream.  Iterations after the last active seed converged launch nothing.
    The plan keeps ``D1``, ``D2`` and ``init`` alive; launches must not
    overlap.
    """

    def __init__(self, D1: torch.Tensor, D2: torch.Tensor, *, seed_stride: int = 8,
                 max_iter: int = 10, metric: str = "dot", init: Optional[torch.Tensor] = None,
                 pixel_tol: float = 0.0, with_basin: bool = False,
                 with_seed_state: bool = False):
        batched = D1.dim() == 4
        _check_map(D1, "D1", 4 if batched else 3)
        _check_map(D2, "D2", 4 if batched else 3)
        if D1.dtype != D2.dtype or D1.shape[-1] != D2.shape[-1]:
            raise ValueError("D1 and D2 must share dtype and d")
        if batched and D1.shape[0] != D2.shape[0]:
            raise ValueError("D1 and D2 must share B")
        B = D1.shape[0] if batched else 1
        H1, W1, d = D1.shape[-3:]
        H2, W2, _ = D2.shape[-3:]
        lib = _lib.load()
        m = _metric(metric)
        dev = D1.device
        n_init = -1
        if init is not None:
            if not isinstance(init, torch.Tensor) or not init.is_cuda or \
                    init.dtype != torch.int32:
                raise ValueError("init must be a CUDA int32 tensor")
            init = init.reshape(B, -1).contiguous()
            n_init = k = init.shape[1]
        else:
            k = int(lib.rnn_frm_num_seeds(H1, W1, seed_stride)) if seed_stride >= 1 else 0
        cap = max(1, k if pixel_tol > 0 else min(k, H2 * W2))
        self._keep = (D1, D2, init)
        self.result = FRMResult(
            torch.empty((B, cap, 2), dtype=torch.int32, device=dev),
            torch.zeros(B, dtype=torch.int32, device=dev),
            torch.empty((B, max(k, 1), 4), dtype=torch.int32, device=dev)
            if with_seed_state else None,
            torch.empty((B, H1 * W1 + 1), dtype=torch.int32, device=dev)
            if with_basin else None)
        self.workspace = _workspace(lib.rnn_frm_workspace_size_ex(
            B, H1, W1, H2, W2, d, m, seed_stride, n_init), dev)
        r = self.result
        handle = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _lib.check(lib.rnn_frm_graph_create(
                B, D1.data_ptr(), H1 * W1 * d, D2.data_ptr(), H2 * W2 * d, H1, W1, H2, W2, d,
                _dtype_code(D1), m, _ptr(init), max(n_init, 0), seed_stride, max_iter,
                float(pixel_tol), r.pairs.data_ptr(), cap, r.count.data_ptr(),
                _ptr(r.seed_state), _ptr(r.basin), self.workspace.data_ptr(),
                self.workspace.numel(), ctypes.byref(handle)), "rnn_frm_graph_create")
        self._handle = handle

    def launch(self) -> FRMResult:
        if not self._handle:
            raise RuntimeError("the graph plan is closed")
        lib = _lib.load()
        _lib.check(lib.rnn_frm_graph_launch(self._handle, _stream(self._keep[0])),
                   "rnn_frm_graph_launch")
        return self.result

    def close(self) -> None:
        if getattr(self, "_handle", None):
            _lib.load().rnn_frm_graph_destroy(self._handle)
            self._handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the process releases the graph
            pass


def frm_refine(D1: torch.Tensor, D2: torch.Tensor, init: torch.Tensor, pixel_tol: float = 0.0,
               *, metric: str = "dot", with_seed_state: bool = False) -> FRMResult:
    """The quoted function called with start pixels: one round trip from each
    unique start, ``(start, match)`` pairs for the starts that come back
    (exactly, or within ``pixel_tol`` pixels)."""
    return frm_match_ex(D1, D2, max_iter=1, metric=metric, init=init, pixel_tol=pixel_tol,
                        with_seed_state=with_seed_state)


# ------------------------------------------------------------------ 3-D points

def _check_points(t: torch.Tensor, name: str, ndim: int) -> None:
    _check_map(t, name, ndim)
    if t.dtype != torch.float32 or t.shape[-1] != 3:
        raise ValueError(f"{name} must be float32 [..., 3], got {t.dtype} {tuple(t.shape)}")


def pts_nn(Q: torch.Tensor, X: torch.Tensor, *, workspace: Optional[torch.Tensor] = None):
    """Nearest point of ``X [nx, 3]`` to each of ``Q [nq, 3]`` (Euclidean,
    lowest index on ties).  Returns ``(idx int32 [nq], squared distance
    float32 [nq])``."""
    _check_points(Q, "Q", 2)
    _check_points(X, "X", 2)
    lib = _lib.load()
    nq, nx = Q.shape[0], X.shape[0]
    idx = torch.empty(nq, dtype=torch.int32, device=Q.device)
    d2 = torch.empty(nq, dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _workspace(lib.rnn_pts_nn_workspace_size(nq, nx), Q.device)
    _lib.check(lib.rnn_pts_nn(Q.data_ptr(), nq, X.data_ptr(), nx, idx.data_ptr(), d2.data_ptr(),
                              workspace.data_ptr(), workspace.numel(), _stream(Q)), "rnn_pts_nn")
    return idx, d2


def pts_mnn(P1: torch.Tensor, P2: torch.Tensor, *, with_nn: bool = False,
            workspace: Optional[torch.Tensor] = None) -> MNNResult:
    """Reciprocal set between point maps ``P1 [H1, W1, 3]`` and ``P2 [H2, W2, 3]``;
    ``rowmax``/``colmax`` hold squared distances."""
    _check_points(P1, "P1", 3)
    _check_points(P2, "P2", 3)
    lib = _lib.load()
    H1, W1, _ = P1.shape
    H2, W2, _ = P2.shape
    n1, n2 = H1 * W1, H2 * W2
    dev = P1.device
    out = MNNResult(torch.empty((min(n1, n2), 2), dtype=torch.int32, device=dev),
                    torch.zeros(1, dtype=torch.int32, device=dev))
    if with_nn:
        out.rowarg = torch.empty(n1, dtype=torch.int32, device=dev)
        out.rowmax = torch.empty(n1, dtype=torch.float32, device=dev)
        out.colarg = torch.empty(n2, dtype=torch.int32, device=dev)
        out.colmax = torch.empty(n2, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _workspace(lib.rnn_pts_mnn_workspace_size(H1, W1, H2, W2), dev)
    _lib.check(lib.rnn_pts_mnn(
        P1.data_ptr(), H1, W1, P2.data_ptr(), H2, W2, out.pairs.data_ptr(), out.pairs.shape[0],
        out.count.data_ptr(), _ptr(out.rowarg), _ptr(out.rowmax), _ptr(out.colarg),
        _ptr(out.colmax), workspace.data_ptr(), workspace.numel(), _stream(P1)), "rnn_pts_mnn")
    return out


def pts_frm_match(P1: torch.Tensor, P2: torch.Tensor, *, seed_stride: int = 8,
                  max_iter: int = 10, init: Optional[torch.Tensor] = None,
                  pixel_tol: float = 0.0, with_basin: bool = False,
                  with_seed_state: bool = False,
                  workspace: Optional[torch.Tensor] = None) -> FRMResult:
    """FRM on point maps ``[H, W, 3]`` or ``[B, H, W, 3]`` (fp32), with the
    options of ``frm_match_ex``."""
    batched = P1.dim() == 4
    _check_points(P1, "P1", 4 if batched else 3)
    _check_points(P2, "P2", 4 if batched else 3)
    if batched and P1.shape[0] != P2.shape[0]:
        raise ValueError("P1 and P2 must share B")
    B = P1.shape[0] if batched else 1
    H1, W1, _ = P1.shape[-3:]
    H2, W2, _ = P2.shape[-3:]
    lib = _lib.load()
    dev = P1.device
    n_init = -1
    if init is not None:
        if not isinstance(init, torch.Tensor) or not init.is_cuda or init.dtype != torch.int32:
            raise ValueError("init must be a CUDA int32 tensor")
        init = init.reshape(B, -1).contiguous()
        n_init = init.shape[1]
        k = n_init
    else:
        k = int(lib.rnn_frm_num_seeds(H1, W1, seed_stride)) if seed_stride >= 1 else 0
    cap = max(1, k if pixel_tol > 0 else min(k, H2 * W2))
    out = FRMResult(torch.empty((B, cap, 2), dtype=torch.int32, device=dev),
                    torch.zeros(B, dtype=torch.int32, device=dev),
                    torch.empty((B, max(k, 1), 4), dtype=torch.int32, device=dev)
                    if with_seed_state else None,
                    torch.empty((B, H1 * W1 + 1), dtype=torch.int32, device=dev)
                    if with_basin else None)
    if workspace is None:
        workspace = _workspace(lib.rnn_pts_frm_workspace_size(B, H1, W1, H2, W2, seed_stride,
                                                              n_init), dev)
    _lib.check(lib.rnn_pts_frm_match(
        B, P1.data_ptr(), H1 * W1 * 3, P2.data_ptr(), H2 * W2 * 3, H1, W1, H2, W2, _ptr(init),
        max(n_init, 0), seed_stride, max_iter, float(pixel_tol), out.pairs.data_ptr(), cap,
        out.count.data_ptr(), _ptr(out.seed_state), _ptr(out.basin), workspace.data_ptr(),
        workspace.numel(), _stream(P1)), "rnn_pts_frm_match")
    return out


# ------------------------------------------------------------ coarse-to-fine

@dataclass
class C2FResult:
    pairs: torch.Tensor    # [cap, 2] int32 full-resolution (image-1, image-2) pixels
    count: torch.Tensor    # [1] int32
    crops: torch.Tensor    # [ncrops, 6]: y0_1, x0_1, y0_2, x0_2, coarse pairs inside, on

    def trimmed(self) -> torch.Tensor:
        return trim(self.pairs, self.count)


def c2f_match(C1: torch.Tensor, C2: torch.Tensor, F1: torch.Tensor, F2: torch.Tensor, *,
              crop=(384, 512), seed_stride: int = 8, max_iter: int = 10, min_coarse: int = 1,
              metric: str = "dot", workspace: Optional[torch.Tensor] = None) -> C2FResult:
    """Coarse-to-fine matching of full-resolution maps ``F1 [H1, W1, d]``,
    ``F2 [H2, W2, d]`` guided by coarse maps ``C1 [Hc1, Wc1, dc]``,
    ``C2 [Hc2, Wc2, dc]`` (all one dtype); ``crop`` is ``(height, width)``."""
    for t, n in ((C1, "C1"), (C2, "C2"), (F1, "F1"), (F2, "F2")):
        _check_map(t, n, 3)
    if len({C1.dtype, C2.dtype, F1.dtype, F2.dtype}) != 1:
        raise ValueError("all four maps must share one dtype")
    if C1.shape[2] != C2.shape[2] or F1.shape[2] != F2.shape[2]:
        raise ValueError("C1/C2 and F1/F2 must share their depth")
    lib = _lib.load()
    Hc1, Wc1, dc = C1.shape
    Hc2, Wc2, _ = C2.shape
    H1, W1, d = F1.shape
    H2, W2, _ = F2.shape
    ch, cw = int(crop[0]), int(crop[1])
    m = _metric(metric)
    dev = F1.device
    nc = int(lib.rnn_c2f_num_crops(H1, W1, H2, W2, ch, cw))
    cap = max(1, int(lib.rnn_c2f_max_pairs(H1, W1, H2, W2, ch, cw, seed_stride)))
    out = C2FResult(torch.empty((cap, 2), dtype=torch.int32, device=dev),
                    torch.zeros(1, dtype=torch.int32, device=dev),
                    torch.empty((max(nc, 1), 6), dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = _workspace(lib.rnn_c2f_workspace_size(Hc1, Wc1, Hc2, Wc2, dc, H1, W1, H2,
                                                          W2, d, m, ch, cw, seed_stride), dev)
    _lib.check(lib.rnn_c2f_match(
        C1.data_ptr(), Hc1, Wc1, C2.data_ptr(), Hc2, Wc2, dc, F1.data_ptr(), H1, W1,
        F2.data_ptr(), H2, W2, d, _dtype_code(F1), m, ch, cw, seed_stride, max_iter, min_coarse,
        out.pairs.data_ptr(), cap, out.count.data_ptr(), out.crops.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(F1)), "rnn_c2f_match")
    return out
