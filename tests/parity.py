"""Tolerances and comparison for GPU-vs-oracle parity.

bf16 inputs, and fp16 inputs (held to the same bounds; their output
spacing is finer) (the stated bounds, applied as written):
  * every element whose reference |O| < 4: |dO| <= 1e-2;
  * every element: the error of the arithmetic before the output is rounded
    to bf16 is at most 1e-2.  The kernel's fp32 value is not visible, only its
    bf16 rounding O_gpu; every fp32 value that rounds to O_gpu lies within
    half a bf16 spacing of it, so the smallest arithmetic error consistent
    with the output is  max(0, |O_gpu - O_ref| - half_spacing(O_gpu)),  and
    that must be <= 1e-2.  (Rounding alone moves an element in [4, 8) by up
    to 0.0156, more than the stated bound, which is why elements of 4 and
    above are held to the arithmetic error.)
  * mean |dO| <= 1e-3;
  * |dLSE| <= 2e-3 + 2^-23 |LSE| (the relative term only matters where a fully
    masked row puts LSE near -1e9, where one fp32 ulp is 64).
fp32 inputs ("relative error <= 1e-5", read normwise): max |dO| <= 1e-5 max |O|,
and |dLSE| <= 1e-5 max(1, |LSE|) per element.  O is a weighted average of V
rows; where it nearly cancels, its error scales with the averaged terms, not
with |O| itself, so the per-element relative error is reported (against a
floor of 2^-7 max |O|) but not bounded.
An oracle LSE of -inf (a row with no finite logit) must come back as -inf
with O = 0.

Every check prints its statistics (max and mean |dO|, max |dLSE|, max |O|,
the arithmetic error bound above), so the margin shows in the log.
"""
import numpy as np
import torch

BF16_MAX_O = 1e-2
BF16_MEAN_O = 1e-3
BF16_LSE = 2e-3
BF16_STRICT_BELOW = 4.0
FP32_REL = 1e-5


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def half_spacing_bf16(x: np.ndarray, bits: int = 8) -> np.ndarray:
    """Half the distance between neighbouring numbers of a `bits`-significand
    format (bf16: 8, fp16: 11) at each representable value x: every real
    number that rounds to x lies within it (for x a power of two, the spacing
    below is half as wide; the larger one bounds both sides).  Normal range
    only (both formats' outputs here are far above their smallest normal)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - float(bits))


def check(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    o_gpu, lse_gpu, o_ref, lse_ref = map(_np, (o_gpu, lse_gpu, o_ref, lse_ref))
    assert o_gpu.shape == o_ref.shape and lse_gpu.shape == lse_ref.shape
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    dO = np.abs(o_gpu - o_ref)
    ninf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ninf), f"{what}: -inf LSE pattern differs"
    assert not np.any(np.isnan(lse_gpu)), f"{what}: NaN LSE"
    fin = ~ninf
    dL = np.abs(lse_gpu[fin] - lse_ref[fin])
    stats = {"max_dO": float(dO.max(initial=0)), "mean_dO": float(dO.mean()) if dO.size else 0.0,
             "max_dLSE": float(dL.max(initial=0)), "max_abs_O": float(np.abs(o_ref).max(initial=0))}
    if dtype in (torch.bfloat16, torch.float16):
        half = half_spacing_bf16(o_gpu, 8 if dtype == torch.bfloat16 else 11)
        stats["max_arith_err_lower_bound"] = float(np.maximum(dO - half, 0.0).max(initial=0))
        small = np.abs(o_ref) < BF16_STRICT_BELOW
        stats["max_dO_below_4"] = float(dO[small].max(initial=0))
        print(f"parity {what}: {stats}")
        assert stats["max_dO_below_4"] <= BF16_MAX_O, f"{what}: {stats}"
        assert stats["max_arith_err_lower_bound"] <= BF16_MAX_O, f"{what}: {stats}"
        assert stats["mean_dO"] <= BF16_MEAN_O, f"{what}: {stats}"
        bound = BF16_LSE + 2.0 ** -23 * np.abs(lse_ref[fin])
        assert np.all(dL <= bound), f"{what}: LSE {stats}"
    else:
        scale = max(stats["max_abs_O"], 1e-30)
        rel_el = dO / np.maximum(np.abs(o_ref), 2.0 ** -7 * scale)
        stats["max_rel_elementwise"] = float(rel_el.max(initial=0))
        print(f"parity {what}: {stats}")
        assert stats["max_dO"] <= FP32_REL * scale, f"{what}: {stats}"
        assert np.all(dL <= FP32_REL * np.maximum(1.0, np.abs(lse_ref[fin]))), f"{what}: LSE {stats}"
    return stats


# Backward pass.  The gradients are sums over many products whose factors the
# tensor-core path rounds to bf16 (weights p, logit gradients dt; O enters
# delta after its own rounding) before it accumulates in fp32, and the
# gradients are rounded to the input dtype at the end: each source moves a
# gradient by up to about 2^-9 of the size of its terms.  Held normwise per
# gradient tensor G against the float64 reference R:
#   bf16 / fp16:  max |G - R| <= 2^-6 max |R|  and  mean |G - R| <= 2^-7 mean |R|
#                 (eight and four times the 2^-9 rounding unit);
#   fp32:         max |G - R| <= 1e-5 max |R|  (the forward's normwise reading).
BWD_MAX_REL = 2.0 ** -6
BWD_MEAN_REL = 2.0 ** -7
BWD_FP32_MAX_REL = 1e-5


def check_grads(got: dict, ref: dict, dtype, what=""):
    stats = {}
    for name, r in ref.items():
        g = got[name]
        assert g is not None, f"{what}: {name} not computed"
        g, r = _np(g), _np(r)
        assert g.shape == r.shape, f"{what}: {name} shape {g.shape} vs {r.shape}"
        assert np.all(np.isfinite(g)), f"{what}: non-finite {name}"
        e = np.abs(g - r)
        rmax = float(np.abs(r).max(initial=0))
        rmean = float(np.abs(r).mean()) if r.size else 0.0
        s = {"max_err": float(e.max(initial=0)), "max_ref": rmax,
             "max_rel": float(e.max(initial=0)) / max(rmax, 1e-30),
             "mean_rel": (float(e.mean()) / max(rmean, 1e-30)) if e.size else 0.0}
        stats[name] = s
        if dtype in (torch.bfloat16, torch.float16):
            ok = s["max_err"] <= BWD_MAX_REL * rmax and float(e.mean()) <= BWD_MEAN_REL * rmean
        else:
            ok = s["max_err"] <= BWD_FP32_MAX_REL * rmax
        if rmax == 0.0:
            ok = s["max_err"] == 0.0
        assert ok, f"{what}: {name} {s}"
    print(f"grad parity {what}: " + ", ".join(
        f"{k} max_rel {v['max_rel']:.2e} mean_rel {v['mean_rel']:.2e}" for k, v in stats.items()))
    return stats
