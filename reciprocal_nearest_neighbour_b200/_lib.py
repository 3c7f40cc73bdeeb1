"""ctypes loader for ``librnn.so`` (the C ABI declared in ``include/rnn.h``).

There is no fallback: if the library is missing or fails to load, every call
raises ``RNNLibraryError``.  Build it with
``python -m reciprocal_nearest_neighbour_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librnn.so")

# every symbol include/rnn.h declares
EXPORTS = (
    "rnn_status_string",
    "rnn_abi_version",
    "rnn_workspace_status",
    "rnn_nn_workspace_size",
    "rnn_nn_argmax",
    "rnn_mnn_workspace_size",
    "rnn_mnn_exhaustive",
    "rnn_frm_num_seeds",
    "rnn_frm_max_pairs",
    "rnn_frm_workspace_size",
    "rnn_frm_match",
    "rnn_frm_match_batched",
    "rnn_launch_count",
    "rnn_set_kernel_timer",
    "rnn_nn_argmax_noalloc",
    "rnn_nn_argmax_noalloc_status",
    "rnn_nn_workspace_size_ex",
    "rnn_nn_argmax_ex",
    "rnn_mnn_workspace_size_ex",
    "rnn_mnn_exhaustive_ex",
    "rnn_frm_workspace_size_ex",
    "rnn_frm_match_ex",
    "rnn_pts_nn_workspace_size",
    "rnn_pts_nn",
    "rnn_pts_mnn_workspace_size",
    "rnn_pts_mnn",
    "rnn_pts_frm_workspace_size",
    "rnn_pts_frm_match",
    "rnn_c2f_num_crops",
    "rnn_c2f_max_pairs",
    "rnn_c2f_workspace_size",
    "rnn_c2f_match",
    "rnn_mnn_mutual_workspace_size",
    "rnn_mnn_mutual",
    "rnn_test_stall_loads",
    "rnn_frm_graph_create",
    "rnn_frm_graph_launch",
    "rnn_frm_graph_destroy",
)

STATUS = {
    0: "RNN_OK", 1: "RNN_EINVAL", 2: "RNN_EALIGN", 3: "RNN_ECAPACITY", 4: "RNN_ECUDA",
    5: "RNN_ETIMEOUT", 6: "RNN_EUNSUPPORTED", 7: "RNN_EWORKSPACE",
}
RNN_F16, RNN_BF16 = 0, 1
RNN_DOT, RNN_L2 = 0, 1
METRICS = {"dot": RNN_DOT, "l2": RNN_L2}
RNN_MAX_BATCH = 1024
RNN_NN_NOALLOC_MAX_QUERIES = 65536


class RNNLibraryError(RuntimeError):
    pass


class RNNError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {msg}")
        self.code = code
        self.name = STATUS.get(code, str(code))


_lib = None


def load():
    """Load librnn.so once and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RNNLibraryError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m reciprocal_nearest_neighbour_b200.build` (needs nvcc)")
    try:
        lib = ctypes.CDLL(LIB_PATH)
    except OSError as e:  # pragma: no cover
        raise RNNLibraryError(f"cannot load {LIB_PATH}: {e}") from e
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sigs = {
        "rnn_status_string": (ctypes.c_char_p, [I]),
        "rnn_abi_version": (I, []),
        "rnn_workspace_status": (I, [P, P]),
        "rnn_nn_workspace_size": (SZ, [I64]),
        "rnn_nn_argmax": (I, [P, I64, P, I64, I, I, P, P, P, SZ, P]),
        "rnn_mnn_workspace_size": (SZ, [I, I, I, I, I]),
        "rnn_mnn_exhaustive": (I, [P, I, I, P, I, I, I, I, P, I64, P, P, P, P, P, P, SZ, P]),
        "rnn_frm_num_seeds": (I64, [I, I, I]),
        "rnn_frm_max_pairs": (I64, [I, I, I, I, I]),
        "rnn_frm_workspace_size": (SZ, [I, I, I, I, I, I, I]),
        "rnn_frm_match": (I, [P, I, I, P, I, I, I, I, I, I, P, I64, P, P, P, SZ, P]),
        "rnn_frm_match_batched": (I, [I, P, I64, P, I64, I, I, I, I, I, I, I, I, P, I64, P, P, P,
                                      SZ, P]),
        "rnn_launch_count": (ctypes.c_uint64, []),
        "rnn_set_kernel_timer": (None, [P, P, I, P]),
        "rnn_nn_argmax_noalloc": (I, [P, I64, P, I64, I, I, P, P, P]),
        "rnn_nn_argmax_noalloc_status": (I, [P]),
        "rnn_nn_workspace_size_ex": (SZ, [I64, I64, I, I]),
        "rnn_nn_argmax_ex": (I, [P, I64, P, I64, I, I, I, P, P, P, SZ, P]),
        "rnn_mnn_workspace_size_ex": (SZ, [I, I, I, I, I, I]),
        "rnn_mnn_exhaustive_ex": (I, [P, I, I, P, I, I, I, I, I, P, I64, P, P, P, P, P, P, SZ,
                                      P]),
        "rnn_frm_workspace_size_ex": (SZ, [I, I, I, I, I, I, I, I, I64]),
        "rnn_frm_match_ex": (I, [I, P, I64, P, I64, I, I, I, I, I, I, I, P, I64, I, I,
                                 ctypes.c_float, P, I64, P, P, P, P, SZ, P]),
        "rnn_pts_nn_workspace_size": (SZ, [I64, I64]),
        "rnn_pts_nn": (I, [P, I64, P, I64, P, P, P, SZ, P]),
        "rnn_pts_mnn_workspace_size": (SZ, [I, I, I, I]),
        "rnn_pts_mnn": (I, [P, I, I, P, I, I, P, I64, P, P, P, P, P, P, SZ, P]),
        "rnn_pts_frm_workspace_size": (SZ, [I, I, I, I, I, I, I64]),
        "rnn_pts_frm_match": (I, [I, P, I64, P, I64, I, I, I, I, P, I64, I, I, ctypes.c_float,
                                  P, I64, P, P, P, P, SZ, P]),
        "rnn_c2f_num_crops": (I, [I, I, I, I, I, I]),
        "rnn_c2f_max_pairs": (I64, [I, I, I, I, I, I, I]),
        "rnn_c2f_workspace_size": (SZ, [I, I, I, I, I, I, I, I, I, I, I, I, I, I]),
        "rnn_c2f_match": (I, [P, I, I, P, I, I, I, P, I, I, P, I, I, I, I, I, I, I, I, I, I,
                              P, I64, P, P, P, SZ, P]),
        "rnn_mnn_mutual_workspace_size": (SZ, [I64]),
        "rnn_mnn_mutual": (I, [P, I64, P, I64, P, I64, P, P, SZ, P]),
        "rnn_test_stall_loads": (None, [I, ctypes.c_uint64]),
        "rnn_frm_graph_create": (I, [I, P, I64, P, I64, I, I, I, I, I, I, I, P, I64, I, I,
                                     ctypes.c_float, P, I64, P, P, P, P, SZ, P]),
        "rnn_frm_graph_launch": (I, [P, P]),
        "rnn_frm_graph_destroy": (None, [P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(code: int, where: str) -> None:
    if code != 0:
        msg = load().rnn_status_string(code).decode()
        raise RNNError(code, where, msg)
