"""Failure detection on the GPU without a fault (needs a B200).

Every wait of the fused kernel is bounded.  The test hook
rnn_test_stall_loads makes its producer load no candidate tile, so the MMA
warps' wait on the first tile runs out (after 50 ms here): the kernel stops
all its warps, frees tensor memory and returns, the workspace status reads
RNN_ETIMEOUT, every index written is still in range, and the next call on the
same context and workspace is correct.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import dev

pytestmark = pytest.mark.gpu

LIMIT_NS = 50_000_000


def _stalled(fn):
    lib = rnn._lib.load()
    lib.rnn_test_stall_loads(1, LIMIT_NS)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        lib.rnn_test_stall_loads(0, 0)
    return out


def test_nn_wait_runs_out_and_is_reported():
    rng = np.random.default_rng(200)
    Q = synth.to_storage(synth.quantised_map(rng, 1, 300, 24).reshape(300, 24), "f16")
    X = synth.to_storage(synth.quantised_map(rng, 1, 5000, 24).reshape(5000, 24), "f16")
    lib = rnn._lib.load()
    ws = torch.empty(lib.rnn_nn_workspace_size_ex(300, 5000, 24, 0), dtype=torch.uint8,
                     device="cuda")
    idx, _ = _stalled(lambda: rnn.nn_argmax(dev(Q), dev(X), workspace=ws))
    with pytest.raises(rnn.RNNError) as e:
        rnn.workspace_status(ws)
    assert e.value.name == "RNN_ETIMEOUT"
    i = idx.cpu().numpy()
    assert i.min() >= 0 and i.max() < 5000
    # the context and the workspace are fine afterwards
    idx, _ = rnn.nn_argmax(dev(Q), dev(X), workspace=ws)
    rnn.workspace_status(ws)
    assert np.array_equal(idx.cpu().numpy(), oracle.nn(Q, X).arg)


def test_frm_wait_runs_out_and_is_reported():
    rng = np.random.default_rng(201)
    D1 = synth.to_storage(synth.quantised_map(rng, 24, 32, 16), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, 24, 32, 16), "f16")
    lib = rnn._lib.load()
    ws = torch.empty(lib.rnn_frm_workspace_size(1, 24, 32, 24, 32, 16, 4), dtype=torch.uint8,
                     device="cuda")
    r = _stalled(lambda: rnn.frm_match(dev(D1), dev(D2), 4, 3, workspace=ws))
    with pytest.raises(rnn.RNNError) as e:
        rnn.workspace_status(ws)
    assert e.value.name == "RNN_ETIMEOUT"
    p = r.trimmed().cpu().numpy()
    assert np.all((p >= 0) & (p < 24 * 32))
    r = rnn.frm_match(dev(D1), dev(D2), 4, 3, workspace=ws)
    rnn.workspace_status(ws)
    assert np.array_equal(r.trimmed().cpu().numpy(), oracle.frm(D1, D2, 4, 3).pairs)


def test_mnn_onepass_wait_runs_out_and_is_reported():
    """The exhaustive set's one-pass kernel (d <= 32): its MMA warp's wait on
    the first query tile runs out, every role of every CTA stops, and the
    status reads RNN_ETIMEOUT; indices stay in range and the next call on the
    same workspace is exact."""
    rng = np.random.default_rng(202)
    D1 = synth.to_storage(synth.quantised_map(rng, 40, 50, 24), "f16")
    D2 = synth.to_storage(synth.quantised_map(rng, 30, 70, 24), "f16")
    lib = rnn._lib.load()
    ws = torch.empty(lib.rnn_mnn_workspace_size(40, 50, 30, 70, 24), dtype=torch.uint8,
                     device="cuda")
    r = _stalled(lambda: rnn.mnn_exhaustive(dev(D1), dev(D2), workspace=ws, with_nn=True))
    with pytest.raises(rnn.RNNError) as e:
        rnn.workspace_status(ws)
    assert e.value.name == "RNN_ETIMEOUT"
    ra, ca = r.rowarg.cpu().numpy(), r.colarg.cpu().numpy()
    assert ra.min() >= 0 and ra.max() < 30 * 70 and ca.min() >= 0 and ca.max() < 40 * 50
    r = rnn.mnn_exhaustive(dev(D1), dev(D2), workspace=ws, with_nn=True)
    rnn.workspace_status(ws)
    ref = oracle.mnn(D1, D2)
    assert np.array_equal(r.rowarg.cpu().numpy(), ref.row.arg)
    assert np.array_equal(r.colarg.cpu().numpy(), ref.col.arg)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
