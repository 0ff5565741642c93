"""The C-ABI library builds, loads without a GPU, exports every declared symbol and
rejects bad arguments synchronously (no GPU work is issued for those calls)."""
import ctypes
import os
import re

import pytest

import mixture_experts_grouped_top_b200 as moe_b200
from mixture_experts_grouped_top_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_grouped.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    h = moe_b200.lib()
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(h, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"
    # and the binding declares nothing the header does not
    assert set(_lib.SIGNATURES) == set(names)


def test_status_strings():
    assert moe_b200.moe_status_string(0) == "MOE_OK"
    assert moe_b200.moe_status_string(5) == "MOE_ERR_TIMEOUT"
    assert moe_b200.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_sizes():
    # the 16 blocks' expert histograms (256-byte aligned) plus 256 bytes for the fused
    # route + permutation call's counter
    assert moe_b200.moe_permute_workspace_size(8192, 2, 8) == 16 * 8 * 4 + (256 - 16 * 8 * 4 % 256) % 256 + 256
    assert moe_b200.grouped_mlp_workspace_size(8, 16384, 4096, 14336) >= 16384 * 14336 * 2
    assert moe_b200.grouped_mlp_saved_size(8, 100, 256, 128) >= 100 * 3 * 128 * 2
    assert moe_b200.grouped_mlp_bwd_workspace_size(8, 100, 256, 128) >= 100 * 256 * 2


@pytest.mark.parametrize("args", [
    (0, 10, 4, 5, 1),     # k > E
    (0, 10, 0, 1, 1),     # E = 0
    (0, -1, 4, 2, 1),     # T < 0
    (0, 10, 2000, 2, 1),  # E too large
])
def test_route_rejects_bad_arguments(args):
    h = moe_b200.lib()
    p, T, E, k, renorm = args
    rc = h.moe_route(ctypes.c_void_p(p), T, E, k, renorm, None, None, None)
    assert rc == 1


def test_router_backward_and_fused_route_reject_bad_arguments():
    h = moe_b200.lib()
    # k > E, no logits without renorm, workspace too small: refused before any launch
    assert h.moe_route_bwd(None, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 2, 3, 1,
                           ctypes.c_void_p(16), None) == 1
    assert h.moe_route_bwd(None, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 8, 2, 0,
                           ctypes.c_void_p(16), None) == 1
    p = ctypes.c_void_p(256)
    assert h.moe_route_permute(p, p, 16, 64, 8, 2, 1, 0, p, p, p, None, p, p, p, p, p, 16, None) == 1


def test_other_entry_points_reject_bad_arguments():
    h = moe_b200.lib()
    # unsupported shapes are reported before any launch
    assert h.grouped_mlp_fwd(None, None, None, 8, 16, 100, 256, None, None, None, None, None, 0, None, None,
                             None, 0, None) == 2                                       # H % 64 != 0
    assert h.grouped_mlp_fwd(None, None, None, 8, 16, 128, 200, None, None, None, None, None, 0, None, None,
                             None, 0, None) == 2                                       # F % 128 != 0
    assert h.grouped_mlp_fwd(None, None, None, 0, 16, 128, 256, None, None, None, None, None, 0, None, None,
                             None, 0, None) == 1                                       # E = 0
    assert h.grouped_mlp_bwd(None, None, 4, 16, 128, 256, None, None, None, None, 1, None, None, None, None,
                             None, None, 0, None) == 1                                 # null operands
    assert h.grouped_mlp_bwd(None, None, 4, 16, 128, 256, None, None, None, None, 7, None, None, None, None,
                             None, None, 0, None) == 1                                 # unknown precision
    assert h.mxfp8_quantize_grouped(None, 64, 100, None, 4, None, None, None) == 2    # C % 128
    assert h.grouped_mlp_bwd_workspace_offset(4, 64, 128, 256, 0, 1) == 2 ** 64 - 1  # no `a` part for BF16
    assert h.mxfp8_quantize(None, 1, 4, 33, 0, 0, 0, None, None, None) == 1            # null input
    assert h.mxfp8_quantize(None, 1, 4, 64, 0, 1, 0, None, None, None) == 1            # transpose with axis 0
    assert h.mxfp8_quantize(None, 1, 128, 128, 0, 0, 1, None, None, None) == 1         # MMA scales need axis 1
    assert h.mxfp8_quantize(None, 1, 96, 128, 1, 1, 1, None, None, None) == 2          # ... and 128-multiples
    assert h.moe_unpermute(None, None, None, 4, 12, 2, None, None) == 1                # H % 8
    assert h.moe_permute(None, None, None, 4, 64, 4, 8, 0, None, None, None, None, None, None, None, 0,
                         None) == 1                                                    # k > E


def test_zero_token_calls_are_noops():
    h = moe_b200.lib()
    assert h.moe_route(None, 0, 4, 2, 1, None, None, None) == 0
    assert h.moe_unpermute(None, None, None, 0, 64, 2, None, None) == 0
    assert h.mxfp8_quantize(None, 0, 32, 64, 1, 1, 0, None, None, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_handle", None)
    with pytest.raises(_lib.LibraryMissing):
        _lib.load()
