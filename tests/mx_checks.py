"""Check that MXFP8 codes produced from fp32 arithmetic differ from the oracle's own
quantisation of the exact (fp64) values only where the two sit on opposite sides of a
rounding boundary.

A kernel that quantises its own fp32 result (the fc1 epilogue's `a`) cannot match the
oracle code for code: fp32 and fp64 values of the same quantity straddle an E4M3
rounding midpoint, or a power of two that decides the block scale, now and then. Every
other difference is a bug. So, per element and per 32-value block:

* a block scale may differ from the oracle's only by one step, and only where the exact
  block maximum lies within its error bound (or ``amax_tol`` relative) of a power of two;
* with the kernel's block scale X, an element's value may differ from the oracle's
  encoding of (exact value / X) only by one E4M3 step, and only where that exact value
  lies within its error bound / X (or ``step_tol`` of a step) of the midpoint between the
  two codes.

The per-element error bound ``err`` is what fp32 arithmetic can move the value by; for
the fc1 epilogue it comes from :func:`swiglu_fp32_error_bound`.
"""
import ml_dtypes
import numpy as np

from oracle import mxfp8 as oq

E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


U = 2.0 ** -24


def sigmoid_terms(g):
    """s = 1 / (1 + e^-g) and a bound on the relative error of the kernels' fp32 value of
    it. The kernels take e^-g from the fast exponential intrinsic (CUDA documents at most
    2 + floor(1.173 |x|) ulp), round 1 + e once and divide with the fast divide (at most
    2 ulp). An ulp of a float is at most 2 U of its value (U = 2^-24), and a relative
    error of e reaches s scaled by e / (1 + e) = 1 - s:
        rel(s) <= (1 - s) (4 + 2.346 |g|) U + U + 4 U."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-g))
    return s, (1.0 - s) * (4.0 + 2.346 * np.abs(g)) * U + 5.0 * U


def swiglu_fp32_error_bound(g, u, p, sum_abs_g, sum_abs_u, K: int):
    """Bound on |a_fp32 - a| for a = SiLU(g) * u * p when g and u are K-term dot products
    accumulated in fp32 by the tensor cores: each K=32 MMA step adds its partial sum into
    the fp32 accumulator, so K/32 + 1 roundings of at most u = 2**-24 times the running
    magnitude (at most sum_k |x_k w_k|) each; a factor 4 covers the MMA's internal
    alignment of its 32 products. The epilogue's own fp32 work: the sigmoid's relative
    error (sigmoid_terms) plus a few roundings of the products."""
    n_add = K // 32 + 1
    eps_g = 4.0 * n_add * U * np.asarray(sum_abs_g, dtype=np.float64)
    eps_u = 4.0 * n_add * U * np.asarray(sum_abs_u, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    s, rel_s = sigmoid_terms(g)
    silu = g * s
    dsilu = s * (1.0 + g * (1.0 - s))
    return np.abs(dsilu * u * p) * eps_g + np.abs(silu * p) * eps_u + (rel_s + 12.0 * U) * np.abs(silu * u * p)


def dswiglu_fp32_error_bounds(g, u, p, sum_abs_da, K: int):
    """Bounds on |x_fp32 - x| for the SwiGLU backward's dg, du and the recomputed a, when
    da is a K-term dot product accumulated in fp32 by the tensor cores (the bound of
    swiglu_fp32_error_bound on da) and g, u, p are exact inputs (|da| is at most
    sum |dy w|). The epilogue's own fp32 work: the sigmoid's error (sigmoid_terms) moves
    SiLU'(g) = s (1 + g (1 - s)) by |1 + g - 2 g s| s rel(s) and SiLU(g) by |g| s rel(s),
    plus a few roundings of each step."""
    eps_da = 4.0 * (K // 32 + 1) * U * np.asarray(sum_abs_da, dtype=np.float64)
    da_max = np.abs(np.asarray(sum_abs_da, dtype=np.float64))
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    s, rel_s = sigmoid_terms(g)
    silu = g * s
    dsilu = s * (1.0 + g * (1.0 - s))
    err_dsilu = np.abs(1.0 + g - 2.0 * g * s) * s * rel_s + 8.0 * U * (s + np.abs(g) * s * (1.0 - s))
    err_silu = np.abs(g) * s * rel_s + 2.0 * U * np.abs(silu)
    return (np.abs(p * u * dsilu) * eps_da + np.abs(p * u) * da_max * (err_dsilu + 8.0 * U * np.abs(dsilu)),
            np.abs(p * silu) * eps_da + np.abs(p) * da_max * (err_silu + 8.0 * U * np.abs(silu)),
            (rel_s + 12.0 * U) * np.abs(silu * u * p))


def boundary_flips_grouped_rows(codes, scales, exact, split, err=None, **tol):
    """The same check for codes quantised along each expert's rows (32-row blocks that
    restart at every expert): codes / exact / err [R, C], scales a per-expert list of
    [ceil(n_e/32), C]. Each expert's rows are padded to whole blocks with zeros and
    transposed, so that the blocks run along the last axis."""
    codes = np.asarray(codes, dtype=np.uint8)
    exact = np.asarray(exact, dtype=np.float64)
    err = np.zeros(exact.shape) if err is None else np.asarray(err, dtype=np.float64)
    total = {"scale_flips": 0, "code_flips": 0, "bad_scales": 0, "bad_codes": 0, "worst_mid_dist": 0.0}
    ok_all, r0 = True, 0
    for n, sc in zip(split, scales):
        n = int(n)
        if n == 0:
            continue
        npad = (n + 31) // 32 * 32
        pad = lambda a, dt: np.concatenate([a[r0:r0 + n], np.zeros((npad - n, a.shape[1]), dtype=dt)])
        ok, rep = boundary_flips(pad(codes, np.uint8).T, np.asarray(sc).T, pad(exact, np.float64).T,
                                 pad(err, np.float64).T, **tol)
        ok_all &= ok
        for k in total:
            total[k] = max(total[k], rep[k]) if k == "worst_mid_dist" else total[k] + rep[k]
        r0 += n
    return ok_all, total


def boundary_flips(codes, scales, exact, err=None, step_tol=1e-3, amax_tol=1e-4):
    """Return (ok, report) for kernel codes [n, C] / scales [n, C/32] against exact [n, C];
    ``err`` [n, C] bounds how far fp32 arithmetic can move each exact value."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    exact = np.asarray(exact, dtype=np.float64)
    n, C = exact.shape
    err = np.zeros((n, C)) if err is None else np.asarray(err, dtype=np.float64)
    blk = exact.reshape(n, C // 32, 32)
    amax = np.max(np.abs(blk), axis=-1)
    err_amax = np.take_along_axis(err.reshape(n, C // 32, 32), np.argmax(np.abs(blk), axis=-1)[..., None],
                                  axis=-1)[..., 0]
    own_s = oq.e8m0_for_amax(amax)
    report = {"scale_flips": 0, "code_flips": 0, "bad_scales": 0, "bad_codes": 0, "worst_mid_dist": 0.0}
    sdiff = scales != own_s
    if np.any(sdiff):
        am = amax[sdiff]
        with np.errstate(divide="ignore"):
            p2 = np.exp2(np.round(np.log2(np.where(am > 0, am, 1.0))))
        near = np.abs(am - p2) <= np.maximum(amax_tol * am, err_amax[sdiff])
        one_step = np.abs(scales[sdiff].astype(np.int64) - own_s[sdiff].astype(np.int64)) == 1
        bad = ~(near & one_step & (am > 0))
        report["scale_flips"] = int(np.sum(sdiff))
        report["bad_scales"] = int(np.sum(bad))
    X = np.ldexp(1.0, scales.astype(np.int64) - 127)
    v = (blk / X[..., None]).reshape(n, C)
    err_v = err / np.repeat(X, 32, axis=1)
    own_c = oq.e4m3_encode(v)
    diff = E4M3[codes] != E4M3[own_c]          # +0 and -0 are the same value
    if np.any(diff):
        g, o, vv = codes[diff], own_c[diff], v[diff]
        gm, om_ = g & 0x7F, o & 0x7F
        same_sign_or_zero = ((g >> 7) == (o >> 7)) | (gm == 0) | (om_ == 0)
        adjacent = (np.abs(gm.astype(np.int64) - om_.astype(np.int64)) == 1) & same_sign_or_zero
        gv, ov = E4M3[g], E4M3[o]
        step = np.abs(gv - ov)
        tol = np.maximum(step_tol * step, err_v[diff])
        dist = np.abs(vv - (gv + ov) / 2.0) / np.where(step > 0, step, 1.0)
        bad = ~(adjacent & (np.abs(vv - (gv + ov) / 2.0) <= tol))
        report["code_flips"] = int(np.sum(diff))
        report["bad_codes"] = int(np.sum(bad))
        report["worst_mid_dist"] = float(np.max(np.where(adjacent, dist, np.inf)))
    ok = report["bad_scales"] == 0 and report["bad_codes"] == 0
    return ok, report


def assert_boundary_flips(codes, scales, exact, name="codes", **tol):
    ok, rep = boundary_flips(codes, scales, exact, **tol)
    assert ok, f"{name}: MXFP8 codes differ from the oracle beyond rounding-boundary flips: {rep}"
    return rep
