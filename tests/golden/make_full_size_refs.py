"""Write the oracle's results on the full-size workloads, keyed by input hash.

The exhaustive reciprocal set at 512x384 (196 608 pixels a map, d = 24) costs
the double-precision oracle about 2 x 1.9e12 flops: minutes on a host.  The
GPU parity tests compare the CUDA path against it element by element, so the
oracle's outputs are computed once here and stored next to this script.  Every
stored value comes from ``oracle/`` alone (nothing here calls the CUDA path);
each file records the SHA-256 of the input bytes and of the oracle's sources,
and a test that finds a different hash recomputes the oracle instead of
trusting the file.

Files (``tests/golden/full_size/``):

* ``mnn_512x384_q.npz``: quantised k/64 maps (bit-exact mode).  ``rowarg``,
  ``colarg`` (NN2 of every image-1 pixel, NN1 of every image-2 pixel) and
  ``rowbest4096``, ``colbest4096``: the best scores times 4096, which are
  integers (every score is a multiple of 2^-12).
* ``mnn_512x384_q_l2.npz``: the quantised maps under the Euclidean metric
  (nearest by |a - b|^2, lowest index on ties); the best scores (-|a - b|^2)
  times 4096, integers as above.
* ``mnn_512x384_f.npz``: the unit-norm fp16 maps.  ``rowarg``, ``colarg``,
  ``rowbest``, ``colbest`` and the top-2 gaps ``rowgap``, ``colgap``.  The
  scores are stored as float32: the tolerance rule compares them with a
  margin of 1e-3, far above float32 rounding (6e-8 here).
* ``frm_batched_64x512x288.npz``: FRM on every one of the 64 pairs of the
  batched workload (stride 8, max_iter 10): per pair and seed the final U, V,
  queries made, converged flag and the smallest top-2 gap along the seed's
  trajectory; the pairs follow from the converged seeds.

Usage: ``python tests/golden/make_full_size_refs.py [mnn_q] [mnn_q_l2] [mnn_f] [frm64]``
(default: all four).
"""
from __future__ import annotations

import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
OUT = os.path.join(HERE, "full_size")
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def oracle_sha256() -> str:
    """Hash of the oracle's sources (its arithmetic and its marshalling)."""
    h = hashlib.sha256()
    for name in ("rnn_oracle.c", "__init__.py"):
        with open(os.path.join(ROOT, "oracle", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def inputs_sha256(*tensors) -> str:
    """Hash of the 16-bit patterns of the input maps, in order."""
    h = hashlib.sha256()
    for t in tensors:
        a = t.contiguous().view(-1)
        import torch

        h.update(a.view(torch.int16).numpy().tobytes())
    return h.hexdigest()


def mnn_inputs(mode: str):
    from reciprocal_nearest_neighbour_b200 import synth

    w = synth.WORKLOADS["mnn_512x384_q" if mode == "q" else "mnn_512x384_f"]
    D1, D2 = synth.make_workload(w)
    return w, synth.to_storage(D1, "f16"), synth.to_storage(D2, "f16")


def frm64_inputs():
    from reciprocal_nearest_neighbour_b200 import synth

    w = synth.WORKLOADS["frm_batched_64x512x288"]
    a, b = synth.make_workload_storage(w, "f16", workers=min(8, os.cpu_count() or 1))
    return w, a, b


def path(name: str) -> str:
    return os.path.join(OUT, name + ".npz")


def write_mnn(mode: str, metric: str = "dot") -> str:
    import oracle

    w, a, b = mnn_inputs(mode)
    t0 = time.time()
    ref = oracle.mnn(a, b, metric=metric)
    dt = time.time() - t0
    meta = dict(inputs_sha256=inputs_sha256(a, b), oracle_sha256=oracle_sha256(),
                workload=w.name, oracle_seconds=dt, threads=oracle.max_threads())
    arrs = dict(rowarg=ref.row.arg, colarg=ref.col.arg)
    if mode == "q":
        for nm, r in (("row", ref.row), ("col", ref.col)):
            s = r.best * 4096.0
            assert np.array_equal(s, np.round(s)), "quantised scores are multiples of 2^-12"
            arrs[nm + "best4096"] = s.astype(np.int32)
    else:
        arrs.update(rowbest=ref.row.best.astype(np.float32), colbest=ref.col.best.astype(np.float32),
                    rowgap=ref.row.gap.astype(np.float32), colgap=ref.col.gap.astype(np.float32))
    os.makedirs(OUT, exist_ok=True)
    name = "mnn_512x384_" + mode + ("" if metric == "dot" else "_" + metric)
    np.savez_compressed(path(name), **arrs, **{k: np.array(v) for k, v in meta.items()})
    return f"{name}: |M| = {len(ref.pairs)}, oracle {dt:.0f} s"


def write_frm64() -> str:
    import oracle

    w, a, b = frm64_inputs()
    t0 = time.time()
    U, V, Q, C, G = [], [], [], [], []
    for i in range(w.pairs):
        r = oracle.frm(a[i], b[i], w.seed_stride, w.max_iter)
        U.append(r.seed_u), V.append(r.seed_v), Q.append(r.seed_queries)
        C.append(r.seed_converged), G.append(r.seed_min_gap)
    dt = time.time() - t0
    meta = dict(inputs_sha256=inputs_sha256(a, b), oracle_sha256=oracle_sha256(),
                workload=w.name, oracle_seconds=dt, threads=oracle.max_threads())
    os.makedirs(OUT, exist_ok=True)
    np.savez_compressed(path(w.name), seed_u=np.stack(U), seed_v=np.stack(V),
                        seed_queries=np.stack(Q), seed_converged=np.stack(C),
                        seed_min_gap=np.stack(G), **{k: np.array(v) for k, v in meta.items()})
    return f"{w.name}: {w.pairs} pairs, oracle {dt:.0f} s"


def load(name: str, *tensors):
    """The stored arrays of ``name`` if they were made from exactly these
    inputs by the current oracle sources, else None (the caller then runs the
    oracle itself)."""
    f = path(name)
    if not os.path.exists(f):
        return None
    z = np.load(f)
    if str(z["inputs_sha256"]) != inputs_sha256(*tensors):
        return None
    if str(z["oracle_sha256"]) != oracle_sha256():
        return None
    return {k: z[k] for k in z.files}


def main(argv) -> None:
    jobs = argv or ["mnn_q", "mnn_q_l2", "mnn_f", "frm64"]
    for j in jobs:
        if j == "mnn_q":
            print(write_mnn("q"), flush=True)
        elif j == "mnn_q_l2":
            print(write_mnn("q", "l2"), flush=True)
        elif j == "mnn_f":
            print(write_mnn("f"), flush=True)
        elif j == "frm64":
            print(write_frm64(), flush=True)
        else:
            raise SystemExit(f"unknown job {j!r}")


if __name__ == "__main__":
    main(sys.argv[1:])

