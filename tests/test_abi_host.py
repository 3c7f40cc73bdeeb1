"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

The library must load without a GPU, export every function ``include/rnn.h``
declares, compute workspace sizes and seed counts on the host, and reject bad
arguments before touching the device.
"""
import ctypes
import os
import re

import pytest

import oracle
from reciprocal_nearest_neighbour_b200 import _lib, build as rnn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    rnn_build.build()
    return _lib.load()


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(rnn_[a-z0-9_]+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(_lib.EXPORTS)
    so = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared:
        assert hasattr(so, name), name


def test_status_strings_and_version(lib):
    assert lib.rnn_abi_version() == 7
    for code, name in _lib.STATUS.items():
        assert lib.rnn_status_string(code).decode().startswith(name)


@pytest.mark.parametrize("H,W,S", [(5, 7, 2), (4, 4, 3), (1, 4, 2), (3, 3, 1), (384, 512, 8),
                                   (288, 512, 8), (768, 1024, 8), (32, 32, 4), (17, 9, 5)])
def test_seed_counts_match_oracle(lib, H, W, S):
    assert lib.rnn_frm_num_seeds(H, W, S) == len(oracle.frm_seeds(H, W, S))
    k = len(oracle.frm_seeds(H, W, S))
    assert lib.rnn_frm_max_pairs(H, W, H, W, S) == min(k, H * W)


def test_workspace_sizes(lib):
    assert lib.rnn_nn_workspace_size(1000) >= 1000 * 8
    assert lib.rnn_mnn_workspace_size(384, 512, 384, 512, 32) >= 2 * 384 * 512 * 8
    # d <= 32 (and d = 64) take the one-pass kernel, which reads copies of both
    # maps padded to the K-block (d = 24 -> 32 channels, 64 bytes a row) with
    # 2048 NaN rows past the last pixel
    n = 384 * 512
    assert (lib.rnn_mnn_workspace_size(384, 512, 384, 512, 24)
            >= 2 * n * 8 + 2 * (n + 2048) * 64)
    assert (lib.rnn_mnn_workspace_size(384, 512, 384, 512, 24)
            == lib.rnn_mnn_workspace_size(384, 512, 384, 512, 32))
    # the Euclidean metric takes the one-pass kernel too (d = 24: 24 channels and six
    # form columns in 32), on the same copies; at d = 64 it keeps the two sweeps with
    # a query and a candidate form per map (67 columns padded to 80, 160-byte rows)
    assert (lib.rnn_mnn_workspace_size_ex(384, 512, 384, 512, 24, 1)
            == lib.rnn_mnn_workspace_size(384, 512, 384, 512, 24))
    assert (lib.rnn_mnn_workspace_size_ex(384, 512, 384, 512, 64, 1)
            >= 2 * n * 8 + 4 * n * 160)
    one = lib.rnn_frm_workspace_size(1, 384, 512, 384, 512, 32, 8)
    many = lib.rnn_frm_workspace_size(64, 288, 512, 288, 512, 32, 8)
    assert one > 0 and many > 64 * 2304 * 8
    assert lib.rnn_frm_workspace_size(0, 384, 512, 384, 512, 32, 8) == 0
    assert lib.rnn_frm_workspace_size(1, 384, 512, 384, 512, 0, 8) == 0
    for v in (one, many):
        assert v % 256 == 0


FAKE = 0x10000  # never dereferenced: every call below fails validation first
EINVAL, EALIGN, ECAP, EUNSUP, EWS = 1, 2, 3, 6, 7


def test_nn_argmax_argument_errors(lib):
    ws = lib.rnn_nn_workspace_size(10)
    f = lib.rnn_nn_argmax
    assert f(None, 10, FAKE, 10, 24, 0, FAKE, None, FAKE, ws, None) == EINVAL
    assert f(FAKE, 10, FAKE, 0, 24, 0, FAKE, None, FAKE, ws, None) == EINVAL
    assert f(FAKE, -1, FAKE, 10, 24, 0, FAKE, None, FAKE, ws, None) == EINVAL
    assert f(FAKE, 10, FAKE, 10, 20, 0, FAKE, None, FAKE, ws, None) == EALIGN
    assert f(FAKE + 8, 10, FAKE, 10, 24, 0, FAKE, None, FAKE, ws, None) == EALIGN
    assert f(FAKE, 10, FAKE, 10, 264, 0, FAKE, None, FAKE, ws, None) == EUNSUP
    assert f(FAKE, 10, FAKE, 10, 24, 7, FAKE, None, FAKE, ws, None) == EINVAL
    assert f(FAKE, 10, FAKE, 10, 24, 0, None, None, FAKE, ws, None) == EINVAL
    assert f(FAKE, 10, FAKE, 10, 24, 0, FAKE, None, None, ws, None) == EWS
    assert f(FAKE, 10, FAKE, 10, 24, 0, FAKE, None, FAKE, ws - 8, None) == EWS
    assert f(FAKE, 10, FAKE, 10, 24, 0, FAKE, None, FAKE + 16, ws, None) == EWS


def test_mnn_argument_errors(lib):
    ws = lib.rnn_mnn_workspace_size(4, 4, 4, 4, 16)
    f = lib.rnn_mnn_exhaustive

    def call(**kw):
        a = dict(D1=FAKE, H1=4, W1=4, D2=FAKE, H2=4, W2=4, d=16, dt=0, pairs=FAKE, cap=16,
                 count=FAKE, ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["D1"], a["H1"], a["W1"], a["D2"], a["H2"], a["W2"], a["d"], a["dt"],
                 a["pairs"], a["cap"], a["count"], None, None, None, None, a["ws"], a["wsb"], None)

    assert call(H1=0) == EINVAL
    assert call(D2=None) == EINVAL
    assert call(pairs=None) == EINVAL
    assert call(count=None) == EINVAL
    assert call(d=12) == EALIGN
    assert call(cap=15) == ECAP
    assert call(wsb=ws - 1) == EWS


def test_frm_argument_errors(lib):
    ws = lib.rnn_frm_workspace_size(2, 8, 8, 8, 8, 16, 2)
    f = lib.rnn_frm_match_batched

    def call(**kw):
        a = dict(B=2, D1=FAKE, s1=8 * 8 * 16, D2=FAKE, s2=8 * 8 * 16, H1=8, W1=8, H2=8, W2=8,
                 d=16, dt=0, S=2, it=10, pairs=FAKE, cap=16, count=FAKE, ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["B"], a["D1"], a["s1"], a["D2"], a["s2"], a["H1"], a["W1"], a["H2"], a["W2"],
                 a["d"], a["dt"], a["S"], a["it"], a["pairs"], a["cap"], a["count"], None,
                 a["ws"], a["wsb"], None)

    assert call(B=0) == EINVAL
    assert call(B=_lib.RNN_MAX_BATCH + 1) == EUNSUP
    assert call(S=0) == EINVAL
    assert call(it=0) == EINVAL
    assert call(s1=8 * 8 * 16 - 8) == EINVAL
    assert call(s2=8 * 8 * 16 + 4) == EINVAL
    assert call(cap=15) == ECAP
    assert call(ws=None) == EWS
    assert call(d=4) == EALIGN
    single = lib.rnn_frm_match
    assert single(FAKE, 8, 8, FAKE, 8, 8, 16, 0, 2, 0, FAKE, 16, FAKE, None, FAKE, ws,
                  None) == EINVAL


def test_ex_workspace_sizes(lib):
    dot = lib.rnn_mnn_workspace_size_ex(384, 512, 384, 512, 24, _lib.RNN_DOT)
    assert dot == lib.rnn_mnn_workspace_size(384, 512, 384, 512, 24)
    # both metrics run the one-pass kernel at d = 24 on one padded copy of each
    # map (the Euclidean forms fit their six columns in the same 32 channels)
    l2 = lib.rnn_mnn_workspace_size_ex(384, 512, 384, 512, 24, _lib.RNN_L2)
    assert l2 == dot
    assert lib.rnn_nn_workspace_size_ex(100, 5000, 24, _lib.RNN_DOT) == \
        lib.rnn_nn_workspace_size(100)
    assert lib.rnn_nn_workspace_size_ex(100, 5000, 24, _lib.RNN_L2) >= \
        lib.rnn_nn_workspace_size(100) + (100 + 5000) * 32 * 2
    grid = lib.rnn_frm_workspace_size_ex(2, 64, 64, 64, 64, 16, _lib.RNN_DOT, 8, -1)
    assert grid == lib.rnn_frm_workspace_size(2, 64, 64, 64, 64, 16, 8)
    # given starts: sized by their count, whatever the stride
    assert lib.rnn_frm_workspace_size_ex(2, 64, 64, 64, 64, 16, _lib.RNN_DOT, 0, 1000) > \
        lib.rnn_frm_workspace_size_ex(2, 64, 64, 64, 64, 16, _lib.RNN_DOT, 0, 10)
    assert lib.rnn_frm_workspace_size_ex(2, 64, 64, 64, 64, 16, 7, 8, -1) == 0


def test_frm_ex_argument_errors(lib):
    n_init = 20
    ws = lib.rnn_frm_workspace_size_ex(2, 8, 8, 8, 8, 16, _lib.RNN_DOT, 2, n_init)
    f = lib.rnn_frm_match_ex

    def call(**kw):
        a = dict(B=2, D1=FAKE, s1=8 * 8 * 16, D2=FAKE, s2=8 * 8 * 16, H1=8, W1=8, H2=8, W2=8,
                 d=16, dt=0, metric=0, init=FAKE, n=n_init, S=2, it=1, tol=0.0, pairs=FAKE,
                 cap=20, count=FAKE, basin=None, ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["B"], a["D1"], a["s1"], a["D2"], a["s2"], a["H1"], a["W1"], a["H2"], a["W2"],
                 a["d"], a["dt"], a["metric"], a["init"], a["n"], a["S"], a["it"], a["tol"],
                 a["pairs"], a["cap"], a["count"], None, a["basin"], a["ws"], a["wsb"], None)

    assert call(metric=2) == EINVAL
    assert call(tol=-1.0) == EINVAL
    assert call(tol=float("nan")) == EINVAL
    assert call(init=None, tol=1.5) == EINVAL       # a tolerance needs given starts
    assert call(n=-1) == EINVAL
    assert call(init=None, S=0) == EINVAL
    assert call(it=0) == EINVAL
    # with a tolerance the (start, match) pairs are bounded by the starts only
    assert call(tol=1.5, cap=19) == ECAP
    assert call(wsb=ws - 1) == EWS
    assert call(d=4) == EALIGN
    nn = lib.rnn_nn_argmax_ex
    assert nn(FAKE, 10, FAKE, 10, 16, 0, 5, FAKE, None, FAKE, 1 << 20, None) == EINVAL
    mnn = lib.rnn_mnn_exhaustive_ex
    assert mnn(FAKE, 4, 4, FAKE, 4, 4, 16, 0, 9, FAKE, 16, FAKE, None, None, None, None, FAKE,
               1 << 20, None) == EINVAL


def test_pts_workspace_sizes(lib):
    n = 384 * 512
    nn = lib.rnn_pts_nn_workspace_size(1000, n)
    # sorted points (16 bytes), cell and rank (4 + 4) and about 2 cells per point
    assert nn >= n * (16 + 8) + 2 * n * 4
    mnn = lib.rnn_pts_mnn_workspace_size(384, 512, 384, 512)
    assert mnn >= 2 * n * (16 + 8 + 8) + 4 * n * 4
    one = lib.rnn_pts_frm_workspace_size(1, 384, 512, 384, 512, 8, -1)
    many = lib.rnn_pts_frm_workspace_size(4, 384, 512, 384, 512, 8, -1)
    assert many > 3 * one
    assert lib.rnn_pts_frm_workspace_size(1, 384, 512, 384, 512, 0, 500) > 0
    for v in (nn, mnn, one, many):
        assert v % 256 == 0


def test_pts_argument_errors(lib):
    ws = lib.rnn_pts_nn_workspace_size(10, 10)
    nn = lib.rnn_pts_nn
    assert nn(FAKE, 10, FAKE, 0, FAKE, None, FAKE, ws, None) == EINVAL
    assert nn(FAKE, -1, FAKE, 10, FAKE, None, FAKE, ws, None) == EINVAL
    assert nn(None, 10, FAKE, 10, FAKE, None, FAKE, ws, None) == EINVAL
    assert nn(FAKE, 10, None, 10, FAKE, None, FAKE, ws, None) == EINVAL
    assert nn(FAKE, 10, FAKE, 10, None, None, FAKE, ws, None) == EINVAL
    assert nn(FAKE + 2, 10, FAKE, 10, FAKE, None, FAKE, ws, None) == EALIGN
    assert nn(FAKE, 10, FAKE, (1 << 28) + 1, FAKE, None, FAKE, 1 << 40, None) == EUNSUP
    assert nn(FAKE, 10, FAKE, 10, FAKE, None, FAKE, ws - 4, None) == EWS
    assert nn(FAKE, 10, FAKE, 10, FAKE, None, FAKE + 16, ws, None) == EWS

    wm = lib.rnn_pts_mnn_workspace_size(4, 4, 4, 4)
    mnn = lib.rnn_pts_mnn
    assert mnn(FAKE, 0, 4, FAKE, 4, 4, FAKE, 16, FAKE, None, None, None, None, FAKE, wm,
               None) == EINVAL
    assert mnn(FAKE, 4, 4, FAKE + 1, 4, 4, FAKE, 16, FAKE, None, None, None, None, FAKE, wm,
               None) == EALIGN
    assert mnn(FAKE, 4, 4, FAKE, 4, 4, FAKE, 15, FAKE, None, None, None, None, FAKE, wm,
               None) == ECAP
    assert mnn(FAKE, 4, 4, FAKE, 4, 4, FAKE, 16, FAKE, None, None, None, None, FAKE, wm - 1,
               None) == EWS

    wf = lib.rnn_pts_frm_workspace_size(2, 8, 8, 8, 8, 2, -1)
    f = lib.rnn_pts_frm_match

    def call(**kw):
        a = dict(B=2, P1=FAKE, s1=8 * 8 * 3, P2=FAKE, s2=8 * 8 * 3, H1=8, W1=8, H2=8, W2=8,
                 init=None, n=0, S=2, it=10, tol=0.0, pairs=FAKE, cap=16, count=FAKE, ws=FAKE,
                 wsb=wf)
        a.update(kw)
        return f(a["B"], a["P1"], a["s1"], a["P2"], a["s2"], a["H1"], a["W1"], a["H2"],
                 a["W2"], a["init"], a["n"], a["S"], a["it"], a["tol"], a["pairs"], a["cap"],
                 a["count"], None, None, a["ws"], a["wsb"], None)

    assert call(B=0) == EINVAL
    assert call(B=_lib.RNN_MAX_BATCH + 1) == EUNSUP
    assert call(S=0) == EINVAL
    assert call(it=0) == EINVAL
    assert call(tol=1.0) == EINVAL                  # a tolerance needs given starts
    assert call(s1=8 * 8 * 3 - 1) == EINVAL
    assert call(P2=FAKE + 2) == EALIGN
    assert call(cap=15) == ECAP
    assert call(wsb=wf - 1) == EWS


def test_c2f_host_functions(lib):
    assert lib.rnn_c2f_num_crops(768, 1024, 768, 1024, 384, 512) == 4
    assert lib.rnn_c2f_num_crops(1000, 1000, 1000, 1000, 384, 384) == 9
    assert lib.rnn_c2f_num_crops(100, 100, 50, 60, 384, 512) == 4      # crop cut to 50x60
    assert lib.rnn_c2f_num_crops(0, 10, 10, 10, 4, 4) == 0
    k = len(oracle.frm_seeds(384, 512, 8))
    assert lib.rnn_c2f_max_pairs(768, 1024, 768, 1024, 384, 512, 8) == 4 * k
    assert lib.rnn_c2f_max_pairs(16, 16, 16, 16, 8, 8, 1) == 256      # one pair per pixel
    ws = lib.rnn_c2f_workspace_size(64, 80, 64, 80, 256, 768, 1024, 768, 1024, 32, 0, 384,
                                    512, 8)
    assert ws >= 2 * 4 * 384 * 512 * 32 * 2 and ws % 256 == 0
    assert lib.rnn_c2f_workspace_size(64, 80, 64, 80, 256, 768, 1024, 768, 1024, 32, 5, 384,
                                      512, 8) == 0


def test_c2f_argument_errors(lib):
    ws = lib.rnn_c2f_workspace_size(4, 4, 4, 4, 16, 16, 16, 16, 16, 16, 0, 8, 8, 2)
    cap = lib.rnn_c2f_max_pairs(16, 16, 16, 16, 8, 8, 2)
    f = lib.rnn_c2f_match

    def call(**kw):
        a = dict(C1=FAKE, Hc1=4, Wc1=4, C2=FAKE, Hc2=4, Wc2=4, dc=16, F1=FAKE, H1=16, W1=16,
                 F2=FAKE, H2=16, W2=16, d=16, dt=0, metric=0, ch=8, cw=8, S=2, it=10, mc=1,
                 pairs=FAKE, cap=cap, count=FAKE, ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["C1"], a["Hc1"], a["Wc1"], a["C2"], a["Hc2"], a["Wc2"], a["dc"], a["F1"],
                 a["H1"], a["W1"], a["F2"], a["H2"], a["W2"], a["d"], a["dt"], a["metric"],
                 a["ch"], a["cw"], a["S"], a["it"], a["mc"], a["pairs"], a["cap"], a["count"],
                 None, a["ws"], a["wsb"], None)

    assert call(Hc1=0) == EINVAL
    assert call(ch=0) == EINVAL
    assert call(S=0) == EINVAL
    assert call(it=0) == EINVAL
    assert call(metric=3) == EINVAL
    assert call(pairs=None) == EINVAL
    assert call(dc=12) == EALIGN
    assert call(F2=FAKE + 8) == EALIGN
    assert call(cap=cap - 1) == ECAP
    # 40 x 40 crops of 1 x 1 pixel: more crops than RNN_MAX_BATCH
    assert call(H1=40, W1=40, H2=40, W2=40, ch=1, cw=1) == EUNSUP


def test_mnn_mutual_argument_errors(lib):
    ws = lib.rnn_mnn_mutual_workspace_size(100)
    assert ws > 0 and ws % 256 == 0
    f = lib.rnn_mnn_mutual
    assert f(FAKE, 0, FAKE, 10, FAKE, 10, FAKE, FAKE, ws, None) == EINVAL
    assert f(None, 100, FAKE, 10, FAKE, 10, FAKE, FAKE, ws, None) == EINVAL
    assert f(FAKE, 100, FAKE, 10, FAKE, 9, FAKE, FAKE, ws, None) == ECAP
    assert f(FAKE, 100, FAKE, 10, FAKE, 10, FAKE, FAKE, ws - 1, None) == EWS
    assert f(FAKE, 100, FAKE, 10, FAKE, 10, FAKE, FAKE + 8, ws, None) == EWS


def test_stall_hook_is_a_host_switch(lib):
    # sets and clears process-global state only; nothing is launched
    lib.rnn_test_stall_loads(1, 1000)
    lib.rnn_test_stall_loads(0, 0)


def test_frm_graph_host_checks(lib):
    # checks made before any device query: no plan handle, too many iterations
    import ctypes
    h = ctypes.c_void_p()
    args = [1, FAKE, 64 * 24, FAKE, 64 * 24, 8, 8, 8, 8, 24, 0, 0, None, 0, 4]
    rest = [0.0, FAKE, 64, FAKE, None, None, FAKE, 1 << 20]
    assert lib.rnn_frm_graph_create(*args, 10, *rest, None) == EINVAL
    assert lib.rnn_frm_graph_create(*args, 65, *rest, ctypes.byref(h)) == EUNSUP
    assert not h.value
    assert lib.rnn_frm_graph_launch(None, None) == EINVAL
    lib.rnn_frm_graph_destroy(None)


def test_frm_graph_binding_rejects_bad_maps(lib):
    # the binding checks its arguments before the library is asked for a plan
    import torch
    import reciprocal_nearest_neighbour_b200 as rnn
    cpu = torch.zeros((8, 8, 24), dtype=torch.float16)
    with pytest.raises(ValueError):
        rnn.FRMGraph(cpu, cpu)
    g = rnn.FRMGraph.__new__(rnn.FRMGraph)   # a plan whose creation never ran
    g._handle = ctypes.c_void_p()
    with pytest.raises(RuntimeError):
        g.launch()
    g.close()                                 # closing it is a no-op


def test_noalloc_scratch_holds_the_largest_call(lib):
    """The no-allocation entry point passes its fixed array (256 + 8 *
    RNN_NN_NOALLOC_MAX_QUERIES bytes) as the workspace of the ordinary call;
    the workspace that call needs at the limit must fit in it.  Argument
    errors come back before any device work."""
    m = _lib.RNN_NN_NOALLOC_MAX_QUERIES
    assert lib.rnn_nn_workspace_size(m) <= 256 + 8 * m
    assert lib.rnn_nn_workspace_size_ex(m, 1 << 20, 64, _lib.RNN_DOT) <= 256 + 8 * m
    call = lib.rnn_nn_argmax_noalloc
    assert _lib.STATUS[call(FAKE, m + 1, FAKE, 4, 8, 0, FAKE, None, None)] == "RNN_EUNSUPPORTED"
    assert _lib.STATUS[call(FAKE, -1, FAKE, 4, 8, 0, FAKE, None, None)] == "RNN_EINVAL"
