"""FRM graph plans on the GPU (needs a B200): the recorded match, with its
conditional iterations, gives the oracle's result and the stream call's,
bit for bit (pairs, counts, seed state, basin), and a relaunch reads the
maps' new contents.  The same holds for FRM and coarse-to-fine calls that the
caller records into its own CUDA graph.  Quantised inputs (values k/64) make
every score exact.
"""
import numpy as np
import pytest
import torch

import oracle
import reciprocal_nearest_neighbour_b200 as rnn
from reciprocal_nearest_neighbour_b200 import synth
from parity import dev, seed_state_np

pytestmark = pytest.mark.gpu


def _maps(seed, H1, W1, H2, W2, d=24, B=None):
    rng = np.random.default_rng(seed)
    if B is None:
        return (synth.to_storage(synth.quantised_map(rng, H1, W1, d), "f16"),
                synth.to_storage(synth.quantised_map(rng, H2, W2, d), "f16"))
    return (synth.to_storage(np.stack([synth.quantised_map(rng, H1, W1, d) for _ in range(B)]),
                             "f16"),
            synth.to_storage(np.stack([synth.quantised_map(rng, H2, W2, d) for _ in range(B)]),
                             "f16"))


def _same(a: rnn.FRMResult, b: rnn.FRMResult):
    B = a.count.shape[0]
    assert torch.equal(a.count, b.count)
    for i in range(B):
        n = int(a.count[i])
        assert torch.equal(a.pairs[i, :n], b.pairs[i, :n]), i
    if a.seed_state is not None:
        assert torch.equal(a.seed_state, b.seed_state)
    if a.basin is not None:
        assert torch.equal(a.basin, b.basin)


@pytest.mark.parametrize("S,max_iter,metric", [(4, 10, "dot"), (2, 3, "dot"), (3, 1, "dot"),
                                               (4, 10, "l2"), (1, 64, "dot")])
def test_graph_matches_oracle_and_stream(S, max_iter, metric):
    D1, D2 = _maps(200 + S + max_iter, 40, 56, 36, 60)
    g = rnn.FRMGraph(dev(D1), dev(D2), seed_stride=S, max_iter=max_iter, metric=metric,
                     with_seed_state=True)
    r = g.launch()
    torch.cuda.synchronize()
    ref = oracle.frm_ex(D1, D2, S, max_iter, metric=metric)
    assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
    u, v, q, c = seed_state_np(r)
    assert np.array_equal(u, ref.seed_u) and np.array_equal(v, ref.seed_v)
    assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)
    s = rnn.frm_match_ex(dev(D1), dev(D2), seed_stride=S, max_iter=max_iter, metric=metric,
                         with_seed_state=True)
    _same(r, s)
    g.close()


def test_graph_relaunch_reads_new_maps():
    D1, D2 = _maps(210, 48, 64, 48, 64)
    E1, E2 = _maps(211, 48, 64, 48, 64)
    t1, t2 = dev(D1), dev(D2)
    g = rnn.FRMGraph(t1, t2, seed_stride=4, max_iter=10, with_seed_state=True)
    for A, B in [(D1, D2), (E1, E2), (D1, D2), (E1, E2)]:
        t1.copy_(dev(A))
        t2.copy_(dev(B))
        r = g.launch()
        ref = oracle.frm_ex(A, B, 4, 10)
        assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
        u, v, q, c = seed_state_np(r)
        assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)
    g.close()
    with pytest.raises(RuntimeError):
        g.launch()


def test_graph_batched_starts_tol_basin():
    B, H, W = 3, 24, 36
    D1, D2 = _maps(220, H, W, H, W, B=B)
    rng = np.random.default_rng(221)
    starts = torch.from_numpy(rng.integers(0, H * W, size=(B, 150)).astype(np.int32)).cuda()
    g = rnn.FRMGraph(dev(D1), dev(D2), max_iter=1, pixel_tol=2.0, init=starts,
                     with_seed_state=True)
    r = g.launch()
    s = rnn.frm_match_ex(dev(D1), dev(D2), max_iter=1, pixel_tol=2.0, init=starts,
                         with_seed_state=True)
    _same(r, s)
    for i in range(B):
        ref = oracle.frm_refine(D1[i], D2[i], starts[i].cpu().numpy(), pixel_tol=2.0)
        assert np.array_equal(r.pairs[i, : int(r.count[i])].cpu().numpy(),
                              ref.pairs.reshape(-1, 2)), i
    gb = rnn.FRMGraph(dev(D1), dev(D2), seed_stride=2, max_iter=6, with_basin=True,
                      with_seed_state=True)
    rb = gb.launch()
    sb = rnn.frm_match_ex(dev(D1), dev(D2), seed_stride=2, max_iter=6, with_basin=True,
                          with_seed_state=True)
    _same(rb, sb)
    for i in range(B):
        ref = oracle.frm_ex(D1[i], D2[i], 2, 6, basin=True)
        assert np.array_equal(rb.basin[i].cpu().numpy(), ref.basin), i


def test_graph_full_size_matches_stream():
    """512 x 384 maps, d = 24, stride 8, ten iterations (the FRM workload):
    the plan and the stream call agree bit for bit, over repeated launches."""
    D1, D2 = synth.smooth_pair(230, 384, 512, 24)
    t1 = dev(synth.to_storage(D1, "f16"))
    t2 = dev(synth.to_storage(D2, "f16"))
    s = rnn.frm_match_ex(t1, t2, seed_stride=8, max_iter=10, with_seed_state=True)
    g = rnn.FRMGraph(t1, t2, seed_stride=8, max_iter=10, with_seed_state=True)
    for _ in range(3):
        _same(g.launch(), s)
    assert int(s.count[0]) > 1000


# ------------------------------------------- FRM inside a caller's CUDA graph

def _capture(fn):
    """Record fn() into a torch CUDA graph (after one eager call on the side
    stream, as torch recommends); returns the graph and fn's outputs."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


@pytest.mark.parametrize("metric", ["dot", "l2"])
def test_caller_graph_capture_of_frm(metric):
    """An FRM call captured by the caller records its later iterations as
    conditional nodes; replays give the oracle's result on whatever the
    input tensors hold."""
    D1, D2 = _maps(240, 40, 56, 36, 60)
    E1, E2 = _maps(241, 40, 56, 36, 60)
    t1, t2 = dev(D1), dev(D2)
    g, r = _capture(lambda: rnn.frm_match_ex(t1, t2, seed_stride=3, max_iter=10, metric=metric,
                                             with_seed_state=True))
    for A, B in [(D1, D2), (E1, E2), (D1, D2)]:
        t1.copy_(dev(A))
        t2.copy_(dev(B))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.frm_ex(A, B, 3, 10, metric=metric)
        assert np.array_equal(r.trimmed().cpu().numpy(), ref.pairs)
        u, v, q, c = seed_state_np(r)
        assert np.array_equal(q, ref.seed_queries) and np.array_equal(c, ref.seed_converged)


def test_caller_graph_capture_of_c2f():
    A, B = synth.smooth_pair(250, 192, 256, 24)
    F1, F2 = dev(synth.to_storage(A, "f16")), dev(synth.to_storage(B, "f16"))
    C1 = dev(synth.to_storage(synth.coarse_map(A, 24, 32, dc=64, seed=3), "f16"))
    C2 = dev(synth.to_storage(synth.coarse_map(B, 24, 32, dc=64, seed=3), "f16"))
    kw = dict(crop=(96, 128), seed_stride=4, max_iter=12)
    eager = rnn.c2f_match(C1, C2, F1, F2, **kw)
    g, r = _capture(lambda: rnn.c2f_match(C1, C2, F1, F2, **kw))
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r.count, eager.count) and torch.equal(r.crops, eager.crops)
        n = int(eager.count[0])
        assert torch.equal(r.pairs[:n], eager.pairs[:n])
    assert int(eager.count[0]) > 100


def test_capture_in_a_fresh_thread_records_every_iteration():
    """A thread whose first FRM call is captured has no stream for the
    conditional bodies yet: every iteration is recorded, same results."""
    import threading
    D1, D2 = _maps(260, 32, 48, 32, 48)
    out = {}

    def body():
        try:
            t1, t2 = dev(D1), dev(D2)
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    r = rnn.frm_match_ex(t1, t2, seed_stride=2, max_iter=8,
                                         with_seed_state=True)
            g.replay()
            torch.cuda.synchronize()
            out["r"] = (r.trimmed().cpu().numpy(), seed_state_np(r))
        except Exception as e:  # reported below, in the test's thread
            out["e"] = e

    th = threading.Thread(target=body)
    th.start()
    th.join()
    assert "e" not in out, out.get("e")
    ref = oracle.frm_ex(D1, D2, 2, 8)
    pairs, (u, v, q, c) = out["r"]
    assert np.array_equal(pairs, ref.pairs)
    assert np.array_equal(q, ref.seed_queries)
