"""Tolerances and comparison for GPU-vs-oracle parity.

bf16 inputs (the stated bounds, applied as written):
  * every element whose reference |O| < 4: |dO| <= 1e-2;
  * every element: |O_gpu - rne_bf16(O_ref)| <= 1e-2, the error of the
    arithmetic once the unavoidable rounding of the output to bf16 is taken
    out (an O element in [4, 8) is stored with a spacing of 2^-5, so rounding
    alone can move it by 0.0156);
  * mean |dO| <= 1e-3;
  * |dLSE| <= 2e-3 + 2^-23 |LSE| (the relative term only matters where a fully
    masked row puts LSE near -1e9, where one fp32 ulp is 64).
fp32 inputs: max |dO| <= 1e-5 max |O| (normwise), and per element
|dO| <= 1e-5 max(|O_ref|, 2^-7 max |O|); |dLSE| <= 1e-5 max(1, |LSE|).
An oracle LSE of -inf (a row with no finite logit) must come back as -inf
with O = 0.

Every check prints its statistics (max and mean |dO|, max |dLSE|, max |O|,
and the error excluding output rounding), so the margin shows in the log.
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


def rne_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 (ties to even), back in float64."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32).to(torch.bfloat16).to(
        torch.float64).numpy() if x.size else x.copy()


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
    if dtype == torch.bfloat16:
        # fp32 rounding to bf16 of an fp64 value: go through fp32 first, which
        # can only matter below 2^-126 (no output gets there meaningfully)
        d_excl = np.abs(o_gpu - rne_bf16(o_ref))
        stats["max_dO_excl_rounding"] = float(d_excl.max(initial=0))
        small = np.abs(o_ref) < BF16_STRICT_BELOW
        stats["max_dO_below_4"] = float(dO[small].max(initial=0))
        print(f"parity {what}: {stats}")
        assert stats["max_dO_below_4"] <= BF16_MAX_O, f"{what}: {stats}"
        assert stats["max_dO_excl_rounding"] <= BF16_MAX_O, f"{what}: {stats}"
        assert stats["mean_dO"] <= BF16_MEAN_O, f"{what}: {stats}"
        bound = BF16_LSE + 2.0 ** -23 * np.abs(lse_ref[fin])
        assert np.all(dL <= bound), f"{what}: LSE {stats}"
    else:
        scale = max(stats["max_abs_O"], 1e-30)
        rel_el = dO / np.maximum(np.abs(o_ref), 2.0 ** -7 * scale)
        stats["max_rel_elementwise"] = float(rel_el.max(initial=0))
        print(f"parity {what}: {stats}")
        assert stats["max_dO"] <= FP32_REL * scale, f"{what}: {stats}"
        assert stats["max_rel_elementwise"] <= FP32_REL, f"{what}: {stats}"
        assert np.all(dL <= FP32_REL * np.maximum(1.0, np.abs(lse_ref[fin]))), f"{what}: LSE {stats}"
    return stats
