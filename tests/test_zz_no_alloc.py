"""moe_permute_noalloc: the permutation for callers that cannot allocate device memory
(a server or embedded runtime that fixes all device memory at start-up, or a C host with
no caching allocator). It uses the library's static scratch table instead of a caller
workspace, so its outputs must equal moe_permute's bit for bit — checked here on two
calls in a row through the C ABI, the second with a different shape and expert count so
that leftovers of the first call in the shared table would show."""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
import workloads

DEV = "cuda"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(T, H, E, k, precision):
    R = T * k
    o = {"xp": torch.full((R, H), 7, dtype=torch.bfloat16 if precision == 0 else torch.uint8, device=DEV),
         "row_map": torch.full((R,), -5, dtype=torch.int32, device=DEV),
         "probs_perm": torch.full((R,), -1.0, dtype=torch.float32, device=DEV),
         "split_sizes": torch.full((E,), -3, dtype=torch.int32, device=DEV),
         "offsets": torch.full((E + 1,), -3, dtype=torch.int32, device=DEV)}
    o["xp_scale"] = torch.full((R, H // 32), 9, dtype=torch.uint8, device=DEV) if precision == 1 else None
    return o


def _call_noalloc(x, idx, prob, E, precision, o):
    T, H = x.shape
    k = idx.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return mb.lib().moe_permute_noalloc(_p(x), _p(idx), _p(prob), T, H, E, k, precision, _p(o["xp"]),
                                        _p(o["xp_scale"]), _p(o["row_map"]), _p(o["probs_perm"]),
                                        _p(o["split_sizes"]), _p(o["offsets"]), stream)


@pytest.mark.gpu
def test_noalloc_permute_matches_workspace_permute_on_two_calls():
    cases = [(3000, 256, 128, 8, 0, 11), (700, 128, 6, 2, 1, 12)]   # (T, H, E, k, precision, seed)
    for T, H, E, k, precision, seed in cases:
        d = workloads.small_layer(T, H, 128, E, k, seed=seed, with_grad=False)
        x = d["x"].to(DEV)
        idx, prob = mb.moe_route(d["logits"].to(DEV), k)
        o = _outputs(T, H, E, k, precision)
        assert _call_noalloc(x, idx, prob, E, precision, o) == 0
        ref = mb.moe_permute(x, idx, prob, E, "bf16" if precision == 0 else "mxfp8")
        torch.cuda.synchronize()
        for name in ("xp", "xp_scale", "row_map", "probs_perm", "split_sizes", "offsets"):
            if o[name] is None:
                continue
            assert torch.equal(o[name], ref[name]), name
        assert int(o["split_sizes"].sum()) == T * k
    assert mb.moe_device_status() == 0


@pytest.mark.gpu
def test_noalloc_permute_rejects_sizes_beyond_the_table():
    # ceil(T*k/1024) * E = 4096 * 128 > MOE_PERMUTE_NOALLOC_MAX_COUNTS: refused before any launch
    rc = mb.lib().moe_permute_noalloc(None, None, None, 2097152, 64, 128, 2, 0, None, None, None, None, None,
                                      None, None)
    assert rc == 2
    assert np.int64(2097152) * 2 // 1024 * 128 > 262144
