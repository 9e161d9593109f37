"""Pins that tie the float64 oracle to something other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` instance and raises
AssertionError when the oracle disagrees with what the formula and the
mathematics fix.  The formula is the DeepSpeed DS4Sci_EvoformerAttention
guide's unit-test reference (hmyw.cn, section 4), with its section 5.2 bias
shapes and its section 5.4 log-sum-exp.  ``test_oracle.py`` runs them on the
real oracle; ``test_oracle_mutants.py`` runs them on deliberately broken
copies of the oracle and checks that every plausible mistake trips one.
"""
from __future__ import annotations

import json
import math
import os
from decimal import Context, Decimal, localcontext

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
_NS = {"log": math.log, "sqrt": math.sqrt, "exp": math.exp, "inf": math.inf}


def _expr(s) -> float:
    if isinstance(s, (int, float)):
        return float(s)
    return float(eval(s, {"__builtins__": {}}, dict(_NS)))  # fixture arithmetic only


def _sparse(spec, shape) -> np.ndarray:
    a = np.full(shape, _expr(spec["fill"]), dtype=np.float64)
    for idx, val in spec["set"]:
        a[tuple(idx)] = _expr(val)
    return a


def golden_cases():
    with open(GOLDEN) as f:
        data = json.load(f)
    out = []
    for c in data["cases"]:
        B, N, S, H, D = c["shape"]
        case = {
            "name": c["name"],
            "q": _sparse(c["q"], (B, N, S, H, D)),
            "k": _sparse(c["k"], (B, N, S, H, D)),
            "v": _sparse(c["v"], (B, N, S, H, D)),
            "mask": None if c["mask"] is None else _sparse(c["mask"], (B, N, S)).reshape(B, N, 1, 1, S),
            "pair": None if c["pair"] is None else _sparse(c["pair"], (B, H, S, S)).reshape(B, 1, H, S, S),
            "o": _sparse(c["expect_o"], (B, N, S, H, D)),
            "lse": _sparse(c["expect_lse"], (B, N, H, S)),
            "atol": float(c["atol"]),
        }
        out.append(case)
    return out


def _t(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a))


def _close(a, b, atol, rtol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
        err = np.where(both_inf, 0.0, np.abs(a - b))
        bound = atol + rtol * np.abs(np.where(np.isinf(b), 0.0, b))
        bad = ~(err <= bound)
    if bad.any():
        shown = np.where(bad & np.isfinite(err), err, 0.0).max()
        raise AssertionError(f"{what}: {int(bad.sum())} elements off, max finite err {shown} "
                             f"at {np.argwhere(bad)[:3].tolist()}")


# ---------------------------------------------------------------- closed forms
def pin_golden(orc):
    """Hand-derived closed forms in tests/golden/closed_forms.json."""
    for c in golden_cases():
        O, L = orc.attention(_t(c["q"]), _t(c["k"]), _t(c["v"]), _t(c["mask"]), _t(c["pair"]))
        _close(O.numpy(), c["o"], c["atol"], what=c["name"] + " O")
        _close(L.numpy(), c["lse"], c["atol"], rtol=1e-15, what=c["name"] + " LSE")


def pin_constant_keys_give_mean_of_values(orc):
    """Zero biases and K equal for every key: uniform weights, O = mean_j V,
    LSE = q.k/sqrt(D) + log S."""
    rng = np.random.default_rng(1)
    B, N, S, H, D = 1, 2, 7, 2, 5
    q = rng.standard_normal((B, N, S, H, D))
    krow = rng.standard_normal((B, N, 1, H, D))
    k = np.broadcast_to(krow, (B, N, S, H, D)).copy()
    v = rng.standard_normal((B, N, S, H, D))
    O, L = orc.attention(_t(q), _t(k), _t(v), None, None)
    mean_v = v.mean(axis=2, keepdims=True)
    _close(O.numpy(), np.broadcast_to(mean_v, O.shape), 1e-12, what="mean of V")
    logit = np.einsum("bnshd,bnhd->bnhs", q, krow[:, :, 0]) / math.sqrt(D)
    _close(L.numpy(), logit + math.log(S), 1e-12, what="LSE = logit + log S")


# ----------------------------------------------------------------- brute force
def _brute_force_decimal(q, k, v, mask, pair):
    """Softmax written straight from its definition, exp(t_j) / sum exp(t),
    without subtracting the row maximum, in 60-digit decimal arithmetic with an
    exponent range wide enough for exp(-1e9)."""
    B, N, S, H, D = q.shape
    O = np.zeros((B, N, S, H, D))
    L = np.zeros((B, N, H, S))
    with localcontext(Context(prec=60, Emin=-10**12, Emax=10**12)):
        sqrt_d = Decimal(D).sqrt()
        for b in range(B):
            for n in range(N):
                for h in range(H):
                    for i in range(S):
                        e = []
                        for j in range(S):
                            dot = Decimal(0)
                            for d in range(D):
                                dot += Decimal(float(q[b, n, i, h, d])) * Decimal(float(k[b, n, j, h, d]))
                            t = dot / sqrt_d
                            if mask is not None:
                                t += Decimal(float(mask[b, n, 0, 0, j]))
                            if pair is not None:
                                t += Decimal(float(pair[b, 0, h, i, j]))
                            e.append(t.exp())
                        z = Decimal(0)
                        for x in e:
                            z += x
                        if z == 0:
                            O[b, n, i, h, :] = 0.0
                            L[b, n, h, i] = -math.inf
                            continue
                        for d in range(D):
                            acc = Decimal(0)
                            for j in range(S):
                                acc += e[j] * Decimal(float(v[b, n, j, h, d]))
                            O[b, n, i, h, d] = float(acc / z)
                        L[b, n, h, i] = float(z.ln())
    return O, L


def _tiny_inputs(seed, B=1, N=2, S=6, H=2, D=3, mask_kind="mixed", pair=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, S, H, D)) * 1.5
    k = rng.standard_normal((B, N, S, H, D)) * 1.5
    v = rng.standard_normal((B, N, S, H, D))
    m = None
    if mask_kind == "mixed":       # finite values, a few -inf
        m = rng.standard_normal((B, N, 1, 1, S))
        m[rng.random(m.shape) < 0.2] = -math.inf
        m[..., 0] = rng.standard_normal()  # key 0 always finite: no empty rows
    elif mask_kind == "huge":      # the guide's 1e9 * (keep - 1), with one fully masked n
        keep = rng.random((B, N, 1, 1, S)) >= 0.3
        keep[:, 0] = False
        keep[:, 1:, ..., 0] = True
        m = 1e9 * (keep.astype(np.float64) - 1.0)
    p = rng.standard_normal((B, 1, H, S, S)) * 2.0 if pair else None
    return q, k, v, m, p


def pin_brute_force_finite(orc):
    """Oracle vs exact-arithmetic brute force on tiny inputs (finite and -inf
    mask entries, pair bias present / absent)."""
    for seed, pair, B, D in ((0, True, 1, 3), (1, False, 2, 2), (2, True, 2, 4)):
        q, k, v, m, p = _tiny_inputs(seed, B=B, D=D, pair=pair)
        O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
        Ob, Lb = _brute_force_decimal(q, k, v, m, p)
        _close(O.numpy(), Ob, 1e-12, what=f"brute force O (seed {seed})")
        _close(L.numpy(), Lb, 1e-12, rtol=1e-15, what=f"brute force LSE (seed {seed})")


def pin_brute_force_huge_mask(orc):
    """Oracle vs brute force with the guide's -1e9 mask, including an n whose
    every key is masked (the formula stays defined: a constant shift)."""
    q, k, v, m, p = _tiny_inputs(3, B=1, N=3, S=5, H=2, D=3, mask_kind="huge")
    O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    Ob, Lb = _brute_force_decimal(q, k, v, m, p)
    # a logit near -1e9 is rounded to ~1e-7 in double
    _close(O.numpy(), Ob, 1e-6, what="brute force O, -1e9 mask")
    _close(L.numpy(), Lb, 1e-6, rtol=1e-15, what="brute force LSE, -1e9 mask")


def pin_empty_rows(orc):
    """Every key -inf: no finite logit; the oracle's reading is O = 0,
    LSE = -inf (brute force gives sum exp = 0)."""
    q, k, v, m, p = _tiny_inputs(4, N=2, S=4, pair=True)
    m = np.zeros((1, 2, 1, 1, 4))
    m[:, 1] = -math.inf
    O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    Ob, Lb = _brute_force_decimal(q, k, v, m, p)
    _close(O.numpy(), Ob, 1e-12, what="empty rows O")
    _close(L.numpy(), Lb, 1e-12, rtol=1e-15, what="empty rows LSE")
    assert np.all(np.isneginf(L.numpy()[:, 1])) and np.all(O.numpy()[:, 1] == 0)


# -------------------------------------------------------------- library check
def pin_sdpa_float64(orc):
    """A special case that reduces to a library routine: float64
    scaled_dot_product_attention with the two biases summed into an additive
    float mask (default scale 1/sqrt(D)); LSE by torch.logsumexp of the same
    logits.  The attn_mask axes are [query, key], which pins the pair bias
    orientation."""
    rng = np.random.default_rng(7)
    B, N, S, H, D = 2, 3, 37, 3, 8
    q = rng.standard_normal((B, N, S, H, D))
    k = rng.standard_normal((B, N, S, H, D))
    v = rng.standard_normal((B, N, S, H, D))
    m = rng.standard_normal((B, N, 1, 1, S))
    m[..., S - 5:] = -1e4
    p = rng.standard_normal((B, 1, H, S, S)) * 1.7
    O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    qt = torch.from_numpy(q).permute(0, 1, 3, 2, 4)   # [B, N, H, S, D]
    kt = torch.from_numpy(k).permute(0, 1, 3, 2, 4)
    vt = torch.from_numpy(v).permute(0, 1, 3, 2, 4)
    bias = torch.from_numpy(m) + torch.from_numpy(p)   # [B, N, H, S, S] by broadcast
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=bias)
    logits = qt @ kt.transpose(-1, -2) / math.sqrt(D) + bias
    lse = torch.logsumexp(logits, dim=-1)
    _close(O.numpy(), ref.permute(0, 1, 3, 2, 4).numpy(), 1e-12, what="SDPA O")
    _close(L.numpy(), lse.numpy(), 1e-12, rtol=1e-15, what="logsumexp LSE")


# ------------------------------------------------------------------ invariants
def _rand(seed, B=1, N=3, S=9, H=2, D=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, S, H, D))
    k = rng.standard_normal((B, N, S, H, D))
    v = rng.standard_normal((B, N, S, H, D))
    m = rng.standard_normal((B, N, 1, 1, S))
    p = rng.standard_normal((B, 1, H, S, S))
    return rng, q, k, v, m, p


def pin_mask_shift(orc):
    """Adding c to every key's mask bias leaves O unchanged and adds c to LSE."""
    rng, q, k, v, m, p = _rand(11)
    O0, L0 = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    for c in (3.25, -40.0):
        O1, L1 = orc.attention(_t(q), _t(k), _t(v), _t(m + c), _t(p))
        _close(O1.numpy(), O0.numpy(), 1e-12, what="mask shift O")
        _close(L1.numpy(), L0.numpy() + c, 1e-12, what="mask shift LSE")
    # a shift of a whole pair row (one query) behaves the same way for that row
    p2 = p.copy()
    p2[:, :, :, 2, :] += 5.0
    O2, L2 = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p2))
    _close(O2.numpy(), O0.numpy(), 1e-12, what="pair row shift O")
    expect = L0.numpy().copy()
    expect[:, :, :, 2] += 5.0
    _close(L2.numpy(), expect, 1e-12, what="pair row shift LSE")


def pin_key_permutation(orc):
    """Permuting keys together with their K, V, mask and pair columns leaves
    O and LSE unchanged."""
    rng, q, k, v, m, p = _rand(12)
    perm = rng.permutation(q.shape[2])
    O0, L0 = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    O1, L1 = orc.attention(_t(q), _t(k[:, :, perm]), _t(v[:, :, perm]),
                           _t(m[..., perm]), _t(p[..., perm]))
    _close(O1.numpy(), O0.numpy(), 1e-12, what="key permutation O")
    _close(L1.numpy(), L0.numpy(), 1e-12, what="key permutation LSE")


def pin_query_permutation(orc):
    """Permuting queries with their Q rows and pair rows permutes the outputs."""
    rng, q, k, v, m, p = _rand(13)
    perm = rng.permutation(q.shape[2])
    O0, L0 = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    O1, L1 = orc.attention(_t(q[:, :, perm]), _t(k), _t(v), _t(m), _t(p[:, :, :, perm, :]))
    _close(O1.numpy(), O0.numpy()[:, :, perm], 1e-12, what="query permutation O")
    _close(L1.numpy(), L0.numpy()[..., perm], 1e-12, what="query permutation LSE")


def pin_value_affine(orc):
    """V -> a V + b gives O -> a O + b (the weights sum to one)."""
    rng, q, k, v, m, p = _rand(14)
    a, b = -2.5, 0.75
    O0, L0 = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    O1, L1 = orc.attention(_t(q), _t(k), _t(a * v + b), _t(m), _t(p))
    _close(O1.numpy(), a * O0.numpy() + b, 1e-12, what="V affine O")
    _close(L1.numpy(), L0.numpy(), 0.0, what="V affine LSE")


def pin_duplicate_n(orc):
    """The pair bias is shared across N: two n slices with identical Q, K, V
    and mask give identical outputs."""
    rng, q, k, v, m, p = _rand(15)
    for x in (q, k, v, m):
        x[:, 2] = x[:, 0]
    O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    _close(O.numpy()[:, 2], O.numpy()[:, 0], 0.0, what="duplicate n O")
    _close(L.numpy()[:, 2], L.numpy()[:, 0], 0.0, what="duplicate n LSE")


def pin_slices_match_full(orc):
    """The sampled entry point returns the same numbers as the full one."""
    rng, q, k, v, m, p = _rand(16, B=2, N=3, S=10, H=3, D=4)
    O, L = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    slices = [(1, 2, 0), (0, 0, 2), (1, 1, 1), (0, 2, 0)]
    Os, Ls = orc.attention_slices(_t(q), _t(k), _t(v), _t(m), _t(p), slices)
    for s, (b, n, h) in enumerate(slices):
        _close(Os[s], O.numpy()[b, n, :, h, :], 0.0, what="slice O")
        _close(Ls[s], L.numpy()[b, n, h, :], 0.0, what="slice LSE")


ALL_PINS = [
    pin_golden,
    pin_constant_keys_give_mean_of_values,
    pin_brute_force_finite,
    pin_brute_force_huge_mask,
    pin_empty_rows,
    pin_sdpa_float64,
    pin_mask_shift,
    pin_key_permutation,
    pin_query_permutation,
    pin_value_affine,
    pin_duplicate_n,
    pin_slices_match_full,
]
