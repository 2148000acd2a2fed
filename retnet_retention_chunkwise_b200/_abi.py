"""ctypes declarations for libretention.so (the C ABI in include/retention.h).

Marshalling only: this module loads the in-tree shared library and declares the
signatures.  There is no alternative implementation behind it; if the library
is missing or fails to load, importing the package raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# RETENTION_LIBRARY selects another build of the same library (the
# bounds-checked one for tests); by default the in-tree libretention.so.
LIB_PATH = os.environ.get("RETENTION_LIBRARY") or os.path.join(HERE, "libretention.so")

RET_OK, RET_EINVAL, RET_EUNSUPPORTED, RET_ECUDA, RET_ETIMEOUT, RET_EBOUNDS = 0, 1, 2, 3, 4, 5
RET_F32, RET_BF16 = 0, 1
RET_MAX_HEADS = 1024

# Every symbol include/retention.h declares.
EXPORTS = (
    "retention_parallel",
    "retention_chunkwise",
    "retention_chunkwise_workspace_bytes",
    "retention_recurrent_step",
    "retention_get_device_status",
    "retention_status_str",
    "retention_abi_version",
    "retention_chunkwise_static_ws",
    "retention_chunkwise_host",
    "retention_chunkwise_host_workspace_bytes",
    "retention_groupnorm",
    "retention_groupnorm_gated",
    "retention_chunkwise_gn_gated",
    "retention_chunkwise_gn",
    "retention_chunkwise_gn_workspace_bytes",
    "retention_parallel_backward",
    "retention_parallel_backward_workspace_bytes",
    "retention_chunkwise_backward",
    "retention_chunkwise_backward_workspace_bytes",
    "retention_chunkwise_backward_state",
    "retention_chunkwise_backward_state_workspace_bytes",
    "retention_chunkwise_state",
    "retention_chunkwise_state_workspace_bytes",
    "retention_state_fold",
)
GATE_ACTS = {"none": 0, "swish": 1, "sigmoid": 2}  # ret_gate_act
STATIC_WS_BYTES = 16 << 20  # scratch array behind retention_chunkwise_static_ws


class RetShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int)]


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libretention.so not found at {path}; build it with "
            "`python -m retnet_retention_chunkwise_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, fp, i, sz = ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_size_t
    lib.retention_parallel.argtypes = [vp, vp, vp, fp, vp, RetShape, i, vp]
    lib.retention_chunkwise.argtypes = [vp, vp, vp, fp, vp, vp, vp, i, RetShape, i, vp, sz, vp]
    lib.retention_chunkwise_workspace_bytes.argtypes = [i, RetShape, i]
    lib.retention_chunkwise_workspace_bytes.restype = sz
    lib.retention_recurrent_step.argtypes = [vp, vp, vp, fp, vp, vp, RetShape, i, vp]
    lib.retention_get_device_status.argtypes = [vp]
    lib.retention_status_str.argtypes = [i]
    lib.retention_status_str.restype = ctypes.c_char_p
    lib.retention_abi_version.argtypes = []
    lib.retention_chunkwise_static_ws.argtypes = [vp, vp, vp, fp, vp, vp, vp, i, RetShape, i, vp]
    lib.retention_chunkwise_static_ws.restype = ctypes.c_int
    lib.retention_chunkwise_host.argtypes = [vp, vp, vp, fp, vp, vp, vp, vp, vp, vp, vp, i, RetShape, i,
                                             vp, sz, i, vp]
    lib.retention_chunkwise_host.restype = ctypes.c_int
    lib.retention_chunkwise_host_workspace_bytes.argtypes = [i, RetShape, i, i]
    lib.retention_chunkwise_host_workspace_bytes.restype = sz
    f32 = ctypes.c_float
    lib.retention_groupnorm.argtypes = [vp, vp, f32, vp, vp, RetShape, i, vp]
    lib.retention_groupnorm.restype = ctypes.c_int
    lib.retention_groupnorm_gated.argtypes = [vp, vp, vp, f32, vp, vp, i, RetShape, i, vp]
    lib.retention_groupnorm_gated.restype = ctypes.c_int
    lib.retention_chunkwise_gn_gated.argtypes = [vp, vp, vp, fp, vp, vp, vp, i, RetShape, i, f32, vp, vp, vp, i,
                                                 vp, sz, vp]
    lib.retention_chunkwise_gn_gated.restype = ctypes.c_int
    lib.retention_chunkwise_gn.argtypes = [vp, vp, vp, fp, vp, vp, vp, i, RetShape, i, f32, vp, vp, vp, sz, vp]
    lib.retention_chunkwise_gn.restype = ctypes.c_int
    lib.retention_chunkwise_gn_workspace_bytes.argtypes = [i, RetShape, i]
    lib.retention_chunkwise_gn_workspace_bytes.restype = sz
    lib.retention_parallel_backward.argtypes = [vp, vp, vp, fp, vp, vp, vp, vp, RetShape, i, vp, sz, vp]
    lib.retention_parallel_backward.restype = ctypes.c_int
    lib.retention_parallel_backward_workspace_bytes.argtypes = [RetShape, i]
    lib.retention_parallel_backward_workspace_bytes.restype = sz
    lib.retention_chunkwise_backward.argtypes = [vp, vp, vp, fp, vp, vp, vp, vp, i, RetShape, i, vp, sz, vp]
    lib.retention_chunkwise_backward.restype = ctypes.c_int
    lib.retention_chunkwise_backward_workspace_bytes.argtypes = [i, RetShape, i]
    lib.retention_chunkwise_backward_workspace_bytes.restype = sz
    lib.retention_chunkwise_backward_state.argtypes = [vp, vp, vp, fp, vp, vp, vp, vp, vp, vp, vp, i, RetShape, i,
                                                       vp, sz, vp]
    lib.retention_chunkwise_backward_state.restype = ctypes.c_int
    lib.retention_chunkwise_backward_state_workspace_bytes.argtypes = [i, RetShape, i]
    lib.retention_chunkwise_backward_state_workspace_bytes.restype = sz
    lib.retention_chunkwise_state.argtypes = [vp, vp, fp, vp, vp, i, RetShape, i, vp, sz, vp]
    lib.retention_chunkwise_state.restype = ctypes.c_int
    lib.retention_chunkwise_state_workspace_bytes.argtypes = [i, RetShape, i]
    lib.retention_chunkwise_state_workspace_bytes.restype = sz
    lib.retention_state_fold.argtypes = [vp, ctypes.POINTER(ctypes.c_int), i, fp, vp, vp, RetShape, vp]
    lib.retention_state_fold.restype = ctypes.c_int
    for name in ("retention_parallel", "retention_chunkwise", "retention_recurrent_step",
                 "retention_get_device_status", "retention_abi_version"):
        getattr(lib, name).restype = ctypes.c_int
    return lib
