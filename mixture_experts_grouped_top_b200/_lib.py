"""ctypes loader for libmoe_grouped.so and the argument/return types of every C entry point."""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_grouped.so")

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/moe_grouped.h
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_device_status": (_i, [_vp]),
    "moe_launch_count": (ctypes.c_uint64, []),
    "moe_test_stall_gemm": (_i, [_i, ctypes.c_uint64]),
    "moe_route": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_route_bwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "moe_route_permute": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                               _vp]),
    "moe_permute_workspace_size": (_sz, [_i, _i, _i]),
    "moe_permute": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute_capacity_workspace_size": (_sz, [_i, _i, _i]),
    "moe_permute_capacity": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                  _vp]),
    "moe_permute_rows": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_permute_rows_mxfp8_workspace_size": (_sz, [_i, _i]),
    "moe_permute_rows_mxfp8": (_i, [_vp, _vp, _i, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_unpermute": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "mxfp8_quantize": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "fp8_quantize_workspace_size": (_sz, [_i]),
    "fp8_quantize": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "grouped_mlp_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "grouped_mlp_saved_size": (_sz, [_i, _i, _i, _i, _i]),
    "grouped_mlp_saved_offset": (_sz, [_i, _i, _i, _i, _i, _i]),
    "grouped_mlp_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "grouped_mlp_fwd_combine_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "grouped_mlp_fwd_combine": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _vp, _vp,
                                     _vp, _sz, _vp]),
    "grouped_mlp_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "grouped_mlp_bwd": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                             _vp]),
    "grouped_mlp_bwd_workspace_offset": (_sz, [_i, _i, _i, _i, _i, _i]),
    "grouped_mlp_bwd_mxfp8_operands": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                            _vp, _vp, _sz, _vp]),
    "mxfp8_quantize_weights": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "mxfp8_quantize_grouped": (_i, [_vp, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "mxfp8_grouped_atoms_bytes": (_sz, [_i, _i, _i]),
    "moe_gather_slots": (_i, [_vp, _vp, _i, _vp, _vp]),
}

class MxBwdOperands(ctypes.Structure):
    """moe_mxfp8_bwd_operands: (codes, atoms) pointer pairs, NULL where not given."""
    _fields_ = [(name, _vp) for name in ("dy_rows", "dy_rows_atoms", "dy_cols", "dy_cols_atoms", "xp_cols",
                                        "xp_cols_atoms", "w1_rows", "w1_rows_atoms", "w2_rows", "w2_rows_atoms")]


_lock = threading.Lock()
_handle = None


class LibraryMissing(RuntimeError):
    pass


def load() -> ctypes.CDLL:
    """Load the CUDA library (once). Raises LibraryMissing if it has not been built."""
    global _handle
    with _lock:
        if _handle is not None:
            return _handle
        if not os.path.exists(LIB_PATH):
            raise LibraryMissing(
                f"{LIB_PATH} is not built; run `python -m mixture_experts_grouped_top_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _handle = h
        return h
