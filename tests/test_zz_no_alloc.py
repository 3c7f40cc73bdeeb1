"""The nearest-neighbour entry point that allocates nothing.

``rnn_nn_argmax_noalloc`` serves callers that cannot allocate device memory:
a plugin whose host framework owns every device buffer and only lends it the
inputs and outputs, or a latency-bound loop where cudaMalloc/cudaFree would
synchronise the device.  Its scratch is a fixed array inside the library.
These tests call it through the C ABI and check it against the oracle and
against the ordinary entry point (which takes a caller workspace) on two calls
in a row: the second call must not see anything the first one left in the
shared array.  Inputs are quantised, so the comparisons are exact.

This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def _noalloc(Q, X, with_scores=True):
    lib = _lib.load()
    nq, d = Q.shape
    idx = torch.full((nq,), -7, dtype=torch.int32, device="cuda")
    score = (torch.full((nq,), float("nan"), dtype=torch.float32, device="cuda")
             if with_scores else None)
    dt = _lib.RNN_BF16 if Q.dtype == torch.bfloat16 else _lib.RNN_F16
    status = lib.rnn_nn_argmax_noalloc(Q.data_ptr(), nq, X.data_ptr(), X.shape[0], d, dt,
                                       idx.data_ptr(), score.data_ptr() if with_scores else None,
                                       torch.cuda.current_stream().cuda_stream)
    return status, idx, score


def _status():
    return _lib.load().rnn_nn_argmax_noalloc_status(torch.cuda.current_stream().cuda_stream)


def _maps(seed, nq, nx, d, dt="f16"):
    rng = np.random.default_rng(seed)
    Q = synth.to_storage(synth.quantised_map(rng, 1, nq, d).reshape(nq, d), dt)
    X = synth.to_storage(synth.quantised_map(rng, 1, nx, d).reshape(nx, d), dt)
    return Q, X


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls(dt):
    Qh, X1h = _maps(123, 3000, 5000, 24, dt)
    # second candidate set with much smaller scores: keys left over from the
    # first call would win every comparison if the scratch were not cleared
    X2h = (X1h.float() / 8).to(X1h.dtype)
    Q = Qh.cuda()
    for Xh in (X1h, X2h):
        X = Xh.cuda()
        ref = oracle.nn(Qh, Xh)
        ref_idx, ref_score = rnn.nn_argmax(Q, X)
        status, idx, score = _noalloc(Q, X)
        torch.cuda.synchronize()
        assert status == 0, _lib.STATUS.get(status)
        assert _status() == 0
        assert np.array_equal(idx.cpu().numpy(), ref.arg)
        assert np.array_equal(score.cpu().numpy().astype(np.float64), ref.best)
        assert torch.equal(idx, ref_idx) and torch.equal(score, ref_score)


def test_noalloc_without_scores_and_at_the_query_limit():
    """score_out = NULL is allowed; exactly RNN_NN_NOALLOC_MAX_QUERIES queries
    fill the array and still match the oracle."""
    n = _lib.RNN_NN_NOALLOC_MAX_QUERIES
    Qh, Xh = _maps(7, n, 300, 8)
    status, idx, _ = _noalloc(Qh.cuda(), Xh.cuda(), with_scores=False)
    torch.cuda.synchronize()
    assert status == 0, _lib.STATUS.get(status)
    assert np.array_equal(idx.cpu().numpy(), oracle.nn(Qh, Xh).arg)


def test_noalloc_status_reports_a_wait_that_ran_out():
    """The test hook stalls the candidate loads, the fused kernel's bounded
    wait runs out: the call's own status is RNN_OK (nothing failed on the
    host) and the status word reads RNN_ETIMEOUT; the next call is exact and
    clears it."""
    Qh, Xh = _maps(9, 500, 4000, 24)
    Q, X = Qh.cuda(), Xh.cuda()
    lib = _lib.load()
    lib.rnn_test_stall_loads(1, 50_000_000)
    try:
        status, idx, _ = _noalloc(Q, X)
        torch.cuda.synchronize()
    finally:
        lib.rnn_test_stall_loads(0, 0)
    assert status == 0
    assert _lib.STATUS[_status()] == "RNN_ETIMEOUT"
    i = idx.cpu().numpy()
    assert i.min() >= 0 and i.max() < 4000
    status, idx, _ = _noalloc(Q, X)
    assert status == 0 and _status() == 0
    assert np.array_equal(idx.cpu().numpy(), oracle.nn(Qh, Xh).arg)


def test_noalloc_rejects_more_queries_than_its_scratch_holds():
    lib = _lib.load()
    n = _lib.RNN_NN_NOALLOC_MAX_QUERIES + 1
    Q = torch.zeros((n, 8), dtype=torch.float16, device="cuda")
    X = torch.zeros((4, 8), dtype=torch.float16, device="cuda")
    idx = torch.empty(n, dtype=torch.int32, device="cuda")
    status = lib.rnn_nn_argmax_noalloc(Q.data_ptr(), n, X.data_ptr(), 4, 8, _lib.RNN_F16,
                                       idx.data_ptr(), None,
                                       torch.cuda.current_stream().cuda_stream)
    assert _lib.STATUS[status] == "RNN_EUNSUPPORTED"
