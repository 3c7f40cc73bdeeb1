"""The nearest-neighbour entry point that allocates nothing.

``rnn_nn_argmax_noalloc`` serves callers that cannot allocate device memory:
a plugin whose host framework owns every device buffer and only lends it the
inputs and outputs, or a latency-bound loop where cudaMalloc/cudaFree would
synchronise the device.  Its scratch is a fixed array inside the library.
These tests call it through the C ABI and check it against the ordinary
entry point (which takes a caller workspace) on two calls in a row: the
second call must not see anything the first one left in the shared array.
Inputs are quantised, so the comparison is exact.

This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def _noalloc(Q, X):
    lib = _lib.load()
    nq, d = Q.shape
    idx = torch.full((nq,), -7, dtype=torch.int32, device="cuda")
    score = torch.full((nq,), float("nan"), dtype=torch.float32, device="cuda")
    status = lib.rnn_nn_argmax_noalloc(Q.data_ptr(), nq, X.data_ptr(), X.shape[0], d,
                                       _lib.RNN_F16, idx.data_ptr(), score.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    return status, idx, score


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    rng = np.random.default_rng(123)
    nq, nx, d = 3000, 5000, 24
    Q = synth.to_storage(synth.quantised_map(rng, 1, nq, d).reshape(nq, d), "f16").cuda()
    X1 = synth.to_storage(synth.quantised_map(rng, 1, nx, d).reshape(nx, d), "f16").cuda()
    # second candidate set with much smaller scores: keys left over from the
    # first call would win every comparison if the scratch were not cleared
    X2 = (X1.float() / 8).half()
    for X in (X1, X2):
        ref_idx, ref_score = rnn.nn_argmax(Q, X)
        status, idx, score = _noalloc(Q, X)
        torch.cuda.synchronize()
        assert status == 0, _lib.STATUS.get(status)
        assert torch.equal(idx, ref_idx)
        assert torch.equal(score, ref_score)


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
