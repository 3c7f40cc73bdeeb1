"""Seeded synthetic descriptor maps.

This module only draws inputs.  It holds none of the matching arithmetic
(scores, nearest neighbours, the reciprocal test, the FRM loop); both the
double-precision oracle and the CUDA path take their inputs from here.

The real workloads are MASt3R matching-head outputs: per-pixel descriptors
``D1, D2 in R^{H x W x d}`` normalised to unit length (cv-learn.com MASt3R note,
section "Method and architecture", matching head).  There are no trained
weights here, so these maps stand in for them:

* ``quantised_map``: values ``k/64`` with ``k = round(N(0, 40))`` clipped to
  [-127, 127].  Every value is exact in fp16 and bf16, and every fp32 sum of
  up to 1040 products of such values is exact, so the GPU can be checked
  bit-for-bit.
* ``smooth_pair``: a Gaussian-smoothed random field plus noise, normalised per
  pixel; the second map samples the first through a random similarity about
  the image centre, with fresh random vectors where the source falls outside
  the first image, optionally an occluded rectangle and a share of outlier
  pixels.
* ``pointmap_pair``: the 3-D inputs, two point maps ``[H][W][3]`` of one
  smooth surface in the first camera's frame (MASt3R regresses both point
  maps in that frame): a smooth random depth map back-projected through a
  pinhole camera, and the same surface sampled at pixel positions moved by a
  random similarity, plus noise; optionally rounded to multiples of 1/64.
* ``quantised_points``: ``n`` points with coordinates ``k/64`` in [-16, 16]
  drawn in clusters, with repeated points (ties).
* ``coarse_map``: the coarse maps of coarse-to-fine matching, standing in for
  the network's output on a downscaled image: the full-resolution map read at
  the centre pixel of each coarse cell, optionally through a fixed random
  projection to another depth and renormalised.

Arrays are float64 ``[H][W][d]`` (channel-last, row-major, pixel index
``y*W + x``) holding values that are exactly representable in the requested
storage type; ``to_storage`` rounds them to fp16 or bf16 (round to nearest
even).  Every generator takes an explicit integer seed and draws from
``numpy.random.default_rng(seed)`` in a fixed order.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.ndimage import gaussian_filter1d

__all__ = [
    "quantised_map",
    "quantised_pair",
    "smooth_pair",
    "pointmap_pair",
    "quantised_points",
    "coarse_map",
    "to_storage",
    "Workload",
    "WORKLOADS",
    "make_workload",
]


def _round_half_away(x: np.ndarray) -> np.ndarray:
    return np.sign(x) * np.floor(np.abs(x) + 0.5)


def quantised_map(rng: np.random.Generator, H: int, W: int, d: int) -> np.ndarray:
    """``k/64`` with ``k = round_half_away(N(0, 40^2))`` clipped to +-127."""
    k = _round_half_away(rng.standard_normal((H, W, d)) * 40.0)
    k = np.clip(k, -127.0, 127.0)
    return k / 64.0


def quantised_pair(seed: int, H1: int, W1: int, H2: int, W2: int, d: int):
    """Two independent quantised maps drawn from one stream (D1 first)."""
    rng = np.random.default_rng(seed)
    return quantised_map(rng, H1, W1, d), quantised_map(rng, H2, W2, d)


def _unit(v: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(v * v, axis=-1, keepdims=True))
    n = np.where(n > 0, n, 1.0)
    return v / n


def _smooth_field(rng: np.random.Generator, H: int, W: int, d: int, sigma: float) -> np.ndarray:
    f = rng.standard_normal((H, W, d))
    f = gaussian_filter1d(f, sigma, axis=0, mode="reflect", truncate=4.0)
    f = gaussian_filter1d(f, sigma, axis=1, mode="reflect", truncate=4.0)
    sd = f.std(axis=(0, 1), keepdims=True)
    return f / np.where(sd > 0, sd, 1.0)


def _bilinear(img: np.ndarray, x: np.ndarray, y: np.ndarray) -> np.ndarray:
    """Sample ``img[H][W][d]`` at real positions inside ``[0,W-1] x [0,H-1]``."""
    H, W, _ = img.shape
    x0 = np.clip(np.floor(x).astype(np.int64), 0, W - 1)
    y0 = np.clip(np.floor(y).astype(np.int64), 0, H - 1)
    x1 = np.minimum(x0 + 1, W - 1)
    y1 = np.minimum(y0 + 1, H - 1)
    fx = (x - x0)[:, None]
    fy = (y - y0)[:, None]
    flat = img.reshape(H * W, img.shape[2])   # row gathers on a flat view are faster
    top = flat[y0 * W + x0] * (1 - fx) + flat[y0 * W + x1] * fx
    bot = flat[y1 * W + x0] * (1 - fx) + flat[y1 * W + x1] * fx
    return top * (1 - fy) + bot * fy


def smooth_pair(seed: int, H: int, W: int, d: int, *, sigma: float = 2.0,
                noise1: float = 0.1, noise2: float = 0.05,
                max_rot_deg: float = 20.0, scale_range=(0.8, 1.25),
                occlusion: float = 0.0, outliers: float = 0.0):
    """Unit-norm pair related by a random similarity about the image centre.

    Draw order from ``default_rng(seed)``: smooth field (H*W*d normals), D1
    noise, rotation, log-scale, D2 noise, fresh vectors for out-of-view pixels,
    occlusion rectangle position and vectors, outlier choice and vectors.
    """
    rng = np.random.default_rng(seed)
    field = _smooth_field(rng, H, W, d, sigma)
    d1 = _unit(field + noise1 * rng.standard_normal((H, W, d)))

    theta = math.radians(rng.uniform(-max_rot_deg, max_rot_deg))
    scale = math.exp(rng.uniform(math.log(scale_range[0]), math.log(scale_range[1])))
    cx, cy = (W - 1) / 2.0, (H - 1) / 2.0
    ys, xs = np.mgrid[0:H, 0:W]
    px = (xs.reshape(-1) - cx).astype(np.float64)
    py = (ys.reshape(-1) - cy).astype(np.float64)
    c, s = math.cos(theta), math.sin(theta)
    sx = cx + scale * (c * px - s * py)
    sy = cy + scale * (s * px + c * py)
    inside = (sx >= 0) & (sx <= W - 1) & (sy >= 0) & (sy <= H - 1)

    n2 = noise2 * rng.standard_normal((H * W, d))
    d2 = np.empty((H * W, d))
    d2[inside] = _bilinear(d1, sx[inside], sy[inside])
    d2 = d2 + n2
    fresh = rng.standard_normal((H * W, d))
    d2[~inside] = fresh[~inside]

    if occlusion > 0:
        ow = max(1, int(round(W * math.sqrt(occlusion))))
        oh = max(1, int(round(H * math.sqrt(occlusion))))
        ox = int(rng.integers(0, W - ow + 1))
        oy = int(rng.integers(0, H - oh + 1))
        occ = np.zeros((H, W), dtype=bool)
        occ[oy:oy + oh, ox:ox + ow] = True
        occ = occ.reshape(-1)
        d2[occ] = rng.standard_normal((int(occ.sum()), d))
    if outliers > 0:
        n_out = int(round(outliers * H * W))
        idx = rng.choice(H * W, size=n_out, replace=False)
        d2[idx] = rng.standard_normal((n_out, d))

    d2 = _unit(d2).reshape(H, W, d)
    return d1, d2


def pointmap_pair(seed: int, H: int, W: int, *, depth=(2.0, 5.0), sigma: float = 6.0,
                  noise: float = 0.002, max_rot_deg: float = 10.0,
                  scale_range=(0.9, 1.1), quantised: bool = False):
    """Point maps ``P1, P2 [H][W][3]`` (float64) of one smooth surface.

    Depth ``z = depth[0] + (depth[1]-depth[0]) * (field + 2.5)/5`` clipped to
    the range (``field`` a unit-variance smooth random field), back-projected
    with focal length ``W`` about the image centre.  P2 samples the same depth
    at pixel positions moved by a random similarity about the centre (pixels
    sampled outside the image take the nearest border depth), then adds
    ``noise`` to every coordinate of both maps.  ``quantised`` rounds every
    coordinate to a multiple of 1/64 (then all squared distances are exact in
    fp32; the coordinates stay inside [-16, 16] for the default depths).

    Draw order from ``default_rng(seed)``: field (H*W normals), rotation,
    log-scale, P1 noise, P2 noise.
    """
    rng = np.random.default_rng(seed)
    field = _smooth_field(rng, H, W, 1, sigma)[..., 0]
    z = depth[0] + (depth[1] - depth[0]) * np.clip((field + 2.5) / 5.0, 0.0, 1.0)
    theta = math.radians(rng.uniform(-max_rot_deg, max_rot_deg))
    scale = math.exp(rng.uniform(math.log(scale_range[0]), math.log(scale_range[1])))
    f = float(W)
    cx, cy = (W - 1) / 2.0, (H - 1) / 2.0
    ys, xs = np.mgrid[0:H, 0:W].astype(np.float64)

    def backproject(u, v, zz):
        return np.stack([(u - cx) * zz / f, (v - cy) * zz / f, zz], axis=-1)

    p1 = backproject(xs, ys, z)
    c, s = math.cos(theta), math.sin(theta)
    px, py = xs - cx, ys - cy
    sx = np.clip(cx + scale * (c * px - s * py), 0, W - 1)
    sy = np.clip(cy + scale * (s * px + c * py), 0, H - 1)
    z2 = _bilinear(z[..., None], sx.reshape(-1), sy.reshape(-1)).reshape(H, W)
    p2 = backproject(sx, sy, z2)
    p1 = p1 + noise * rng.standard_normal(p1.shape)
    p2 = p2 + noise * rng.standard_normal(p2.shape)
    if quantised:
        p1 = np.clip(_round_half_away(p1 * 64.0), -1024, 1024) / 64.0
        p2 = np.clip(_round_half_away(p2 * 64.0), -1024, 1024) / 64.0
    return p1, p2


def quantised_points(rng: np.random.Generator, n: int, clusters: int = 8,
                     spread: float = 1.5, repeat: float = 0.05) -> np.ndarray:
    """``[n][3]`` points ``k/64`` in [-16, 16]: Gaussian clusters (centres
    uniform in [-12, 12]^3, standard deviation ``spread``), then a share
    ``repeat`` of the points replaced by copies of earlier ones."""
    centres = rng.uniform(-12.0, 12.0, size=(clusters, 3))
    which = rng.integers(0, clusters, size=n)
    p = centres[which] + spread * rng.standard_normal((n, 3))
    p = np.clip(_round_half_away(p * 64.0), -1024, 1024) / 64.0
    nrep = int(round(repeat * n))
    if nrep and n > 1:
        dst = rng.integers(1, n, size=nrep)
        src = (rng.random(nrep) * dst).astype(np.int64)
        p[dst] = p[src]
    return p


def coarse_map(F: np.ndarray, Hc: int, Wc: int, dc: int = 0, seed: int = 0) -> np.ndarray:
    """``[Hc][Wc][dc]`` map read from ``F [H][W][d]`` at row
    ``int((yc + 0.5) * H / Hc)`` and column ``int((xc + 0.5) * W / Wc)``.
    With ``dc`` > 0 the samples go through a fixed ``dc x d`` Gaussian matrix
    drawn from ``default_rng(seed)`` and are renormalised; otherwise they are
    the samples themselves (quantised inputs stay exact)."""
    H, W, d = F.shape
    ys = ((np.arange(Hc) + 0.5) * H / Hc).astype(np.int64)
    xs = ((np.arange(Wc) + 0.5) * W / Wc).astype(np.int64)
    S = F[ys][:, xs]
    if dc:
        R = np.random.default_rng(seed).standard_normal((dc, d))
        S = _unit(S @ R.T)
    return S


def to_storage(a: np.ndarray, dtype: str):
    """Round a float64 map to the storage type; returns a CPU torch tensor.

    ``dtype`` is ``"f16"`` (numpy's float64 -> float16 conversion, one
    round-to-nearest-even step) or ``"bf16"`` (torch's conversion, which goes
    through float32; each step rounds to nearest even).
    """
    import torch

    return torch.from_numpy(_storage_bits(a, dtype)).view(
        torch.float16 if dtype == "f16" else torch.bfloat16)


def _storage_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit patterns of ``a`` rounded to ``dtype`` (int16 array)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    if dtype == "f16":
        return a.astype(np.float16).view(np.int16)
    if dtype == "bf16":
        import torch

        return torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy()
    raise ValueError(f"unknown storage dtype {dtype!r}")


@dataclass(frozen=True)
class Workload:
    """One synthetic matching workload (sizes, generator and FRM settings)."""

    name: str
    kind: str          # "quantised" | "smooth"
    H: int
    W: int
    d: int
    seed: int
    pairs: int = 1
    seed_stride: int = 8
    max_iter: int = 10
    occlusion: float = 0.0
    outliers: float = 0.0


WORKLOADS = {
    # two 32x32 quantised maps, d=16, seed 0; FRM stride 4 (64 seeds)
    "tiny_q32": Workload("tiny_q32", "quantised", 32, 32, 16, 0, seed_stride=4),
    # FRM at 512x384 (W=512, H=384), d=24, unit-norm fp16, stride 8 (3072 seeds)
    "frm_512x384": Workload("frm_512x384", "smooth", 384, 512, 24, 2),
    # exhaustive mutual NN at 512x384, d=24, quantised (bit-exact mode)
    "mnn_512x384_q": Workload("mnn_512x384_q", "quantised", 384, 512, 24, 3),
    # exhaustive mutual NN at 512x384, d=24, unit-norm fp16 (same generator as FRM)
    "mnn_512x384_f": Workload("mnn_512x384_f", "smooth", 384, 512, 24, 2),
    # 64 independent pairs at 512x288, d=24, 30% occluded rectangle in D2
    "frm_batched_64x512x288": Workload("frm_batched_64x512x288", "smooth", 288, 512, 24, 1000,
                                       pairs=64, occlusion=0.30),
    # 1024x768, d=32, 2% outlier pixels in D2, max_iter 15
    "frm_1024x768": Workload("frm_1024x768", "smooth", 768, 1024, 32, 5, max_iter=15,
                             outliers=0.02),
    # coarse mutual NN on 80x64 tokens, d=256
    "mnn_coarse_80x64": Workload("mnn_coarse_80x64", "smooth", 64, 80, 256, 6),
}


def make_workload(w: Workload, pair: int = 0):
    """Return the float64 (D1, D2) maps of pair ``pair`` of workload ``w``.

    Pair ``b`` of a multi-pair workload uses seed ``w.seed + b``.
    """
    seed = w.seed + pair
    if w.kind == "quantised":
        return quantised_pair(seed, w.H, w.W, w.H, w.W, w.d)
    return smooth_pair(seed, w.H, w.W, w.d, occlusion=w.occlusion, outliers=w.outliers)


def _pair_storage(args):
    w, pair, dtype = args
    d1, d2 = make_workload(w, pair)
    # ship raw 16-bit patterns (bf16 has no numpy type)
    return _storage_bits(d1, dtype), _storage_bits(d2, dtype)


def make_workload_storage(w: Workload, dtype: str = "f16", pairs=None, workers: int = 0):
    """Pairs of workload ``w`` rounded to ``dtype``, as CPU tensors ``[P, H, W, d]``.

    ``pairs`` is an iterable of pair indices (default: all ``w.pairs``).  With
    ``workers > 1`` the pairs are drawn in a process pool started with the
    ``spawn`` method, so it is safe after CUDA has been initialised; the result
    does not depend on the worker count.
    """
    import torch

    idx = list(range(w.pairs)) if pairs is None else list(pairs)
    jobs = [(w, p, dtype) for p in idx]
    if workers and workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor

        with ProcessPoolExecutor(max_workers=min(workers, len(jobs)),
                                 mp_context=mp.get_context("spawn")) as ex:
            parts = list(ex.map(_pair_storage, jobs))
    else:
        parts = [_pair_storage(j) for j in jobs]
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    A = torch.from_numpy(np.stack([p[0] for p in parts])).view(tdt)
    B = torch.from_numpy(np.stack([p[1] for p in parts])).view(tdt)
    return A, B
