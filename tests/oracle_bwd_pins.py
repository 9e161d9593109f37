"""Pins for the float64 oracle's backward pass.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle's gradients disagree with what the mathematics fixes.  The
guide (DeepSpeed DS4Sci_EvoformerAttention, hmyw.cn, sections 1 and 5.4)
says the backward pass returns the gradients of Q, K, V and of the biases,
recomputed from the inputs with the per-row delta as an intermediate; it
prints no formula and no worked example, so the gradients are pinned to:

* central finite differences of the FORWARD oracle (its own pins tie it to the
  formula), for every input element of small cases;
* float64 autograd of torch's scaled_dot_product_attention with the two
  biases summed into an additive mask (a library routine, so an independent
  implementation of the same derivative);
* hand-derived closed forms (tests/golden/bwd_closed_forms.json) and special
  cases with a closed form (uniform weights, one key, S = 1);
* invariants: the logit gradient sums to zero along each row, so dmask and
  every row of dpair sum to zero over keys; a constant shift of the mask
  changes no gradient; permuting keys permutes the key-side gradients;
  gradients are linear in dO.
``test_oracle_bwd.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on broken copies of it.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from tests.oracle_pins import _close, _sparse, _t

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bwd_closed_forms.json")


def _inputs(seed, B=1, N=2, S=5, H=2, D=3, mask_kind="finite", pair=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, S, H, D)) * 1.3
    k = rng.standard_normal((B, N, S, H, D)) * 1.3
    v = rng.standard_normal((B, N, S, H, D))
    do = rng.standard_normal((B, N, S, H, D))
    m = None
    if mask_kind == "finite":
        m = rng.standard_normal((B, N, 1, 1, S))
    elif mask_kind == "some_neg_inf":
        m = rng.standard_normal((B, N, 1, 1, S))
        m[..., 1] = -math.inf
    p = rng.standard_normal((B, 1, H, S, S)) * 1.5 if pair else None
    return q, k, v, m, p, do


def _bwd(orc, q, k, v, m, p, do):
    g = orc.attention_bwd(_t(q), _t(k), _t(v), _t(m), _t(p), _t(do))
    return {name: t.numpy() for name, t in g.items()}


def _loss(orc, q, k, v, m, p, do):
    O, _ = orc.attention(_t(q), _t(k), _t(v), _t(m), _t(p))
    return float((O.numpy() * do).sum())


# ------------------------------------------------------- finite differences
def pin_bwd_finite_differences(orc):
    """Every gradient element against the central difference of
    sum(dO * O) from the forward oracle (step 1e-5: truncation ~1e-10,
    rounding ~1e-11)."""
    for seed, mask_kind, pair in ((0, "finite", True), (1, "some_neg_inf", True), (2, None, False)):
        q, k, v, m, p, do = _inputs(seed, mask_kind=mask_kind, pair=pair)
        g = _bwd(orc, q, k, v, m, p, do)
        named = [("dq", q), ("dk", k), ("dv", v)]
        if m is not None:
            named.append(("dmask", m))
        if p is not None:
            named.append(("dpair", p))
        h = 1e-5
        for name, x in named:
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                if not np.isfinite(x[idx]):
                    continue            # a -inf key has zero weight and zero gradient
                keep = x[idx]
                x[idx] = keep + h
                lp = _loss(orc, q, k, v, m, p, do)
                x[idx] = keep - h
                lm = _loss(orc, q, k, v, m, p, do)
                x[idx] = keep
                fd[idx] = (lp - lm) / (2 * h)
            scale = max(1.0, float(np.abs(fd).max()))
            _close(g[name], fd, 2e-8 * scale, what=f"finite differences {name} (seed {seed})")


# ------------------------------------------------------------ library check
def _torch_grads(q, k, v, m, p, do):
    """float64 autograd of scaled_dot_product_attention, layout [B, N, H, S, D]."""
    B, N, S, H, D = q.shape
    tq, tk, tv = (torch.tensor(np.ascontiguousarray(x.transpose(0, 1, 3, 2, 4)), requires_grad=True)
                  for x in (q, k, v))
    bias = torch.zeros((B, N, H, S, S), dtype=torch.float64)
    tm = tp = None
    if m is not None:
        tm = torch.tensor(m, requires_grad=True)            # [B, N, 1, 1, S]
        bias = bias + tm.reshape(B, N, 1, 1, S)
    if p is not None:
        tp = torch.tensor(p, requires_grad=True)            # [B, 1, H, S, S]
        bias = bias + tp
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=bias)
    tdo = torch.tensor(np.ascontiguousarray(do.transpose(0, 1, 3, 2, 4)))
    (out * tdo).sum().backward()
    g = {name: t.grad.detach().numpy().transpose(0, 1, 3, 2, 4) for name, t in
         (("dq", tq), ("dk", tk), ("dv", tv))}
    if tm is not None:
        g["dmask"] = tm.grad.detach().numpy()
    if tp is not None:
        g["dpair"] = tp.grad.detach().numpy()
    return g


def pin_bwd_sdpa_autograd(orc):
    """float64 autograd of scaled_dot_product_attention (default scale
    1/sqrt(D), additive float mask = mask + pair broadcast to every slice)."""
    for seed, shape, mask_kind in ((3, (2, 3, 9, 2, 4), "some_neg_inf"), (4, (1, 4, 16, 3, 8), "finite")):
        B, N, S, H, D = shape
        q, k, v, m, p, do = _inputs(seed, B, N, S, H, D, mask_kind=mask_kind)
        g = _bwd(orc, q, k, v, m, p, do)
        ref = _torch_grads(q, k, v, m, p, do)
        for name in ("dq", "dk", "dv", "dmask", "dpair"):
            scale = max(1.0, float(np.abs(ref[name]).max()))
            _close(g[name], ref[name], 1e-12 * scale, what=f"autograd {name} (seed {seed})")


def pin_bwd_pair_rows_match_autograd(orc):
    """The row-sampling entry (one query row of dpair, summed over every n)
    against the autograd pair gradient."""
    q, k, v, m, p, do = _inputs(5, 1, 6, 11, 2, 4, mask_kind="some_neg_inf")
    ref = _torch_grads(q, k, v, m, p, do)["dpair"]
    rows = [(0, 0, 0), (0, 1, 7), (0, 0, 10)]
    got = orc.pair_grad_rows(_t(q), _t(k), _t(v), _t(m), _t(p), _t(do), rows, chunk=4)
    for r, (b, h, i) in enumerate(rows):
        _close(got[r], ref[b, 0, h, i], 1e-12, what=f"dpair row {(b, h, i)}")
    dq, dk, dv, cs = orc.attention_bwd_slices(_t(q), _t(k), _t(v), _t(m), _t(p), _t(do), [(0, 3, 1)])
    tg = _torch_grads(q, k, v, m, p, do)
    _close(dq[0], tg["dq"][0, 3, :, 1, :], 1e-12, what="sampled slice dq")
    _close(dk[0], tg["dk"][0, 3, :, 1, :], 1e-12, what="sampled slice dk")
    _close(dv[0], tg["dv"][0, 3, :, 1, :], 1e-12, what="sampled slice dv")


# ------------------------------------------------------------- closed forms
def golden_bwd_cases():
    with open(GOLDEN) as f:
        data = json.load(f)
    out = []
    for c in data["cases"]:
        B, N, S, H, D = c["shape"]
        case = {"name": c["name"], "atol": float(c["atol"])}
        for key in ("q", "k", "v", "do"):
            case[key] = _sparse(c[key], (B, N, S, H, D))
        case["mask"] = None if c["mask"] is None else _sparse(c["mask"], (B, N, S)).reshape(B, N, 1, 1, S)
        case["pair"] = None if c["pair"] is None else _sparse(c["pair"], (B, H, S, S)).reshape(B, 1, H, S, S)
        for key in ("dq", "dk", "dv"):
            case["expect_" + key] = _sparse(c["expect_" + key], (B, N, S, H, D))
        if c.get("expect_dmask") is not None:
            case["expect_dmask"] = _sparse(c["expect_dmask"], (B, N, S)).reshape(B, N, 1, 1, S)
        if c.get("expect_dpair") is not None:
            case["expect_dpair"] = _sparse(c["expect_dpair"], (B, H, S, S)).reshape(B, 1, H, S, S)
        out.append(case)
    return out


def pin_bwd_golden(orc):
    """Hand-derived gradients in tests/golden/bwd_closed_forms.json."""
    for c in golden_bwd_cases():
        g = _bwd(orc, c["q"], c["k"], c["v"], c["mask"], c["pair"], c["do"])
        for name in ("dq", "dk", "dv", "dmask", "dpair"):
            if "expect_" + name in c:
                _close(g[name], c["expect_" + name], c["atol"], what=f"{c['name']} {name}")


def pin_bwd_uniform_weights(orc):
    """Zero biases and K equal for every key: weights 1/S, so dv_j = mean_i
    dO_i for every j, dq = 0, and dt_ij = (dO_i . (v_j - mean v)) / S gives
    dk_j = sum_i dt_ij q_i / sqrt(D)."""
    rng = np.random.default_rng(6)
    B, N, S, H, D = 1, 2, 7, 2, 5
    q = rng.standard_normal((B, N, S, H, D))
    k = np.broadcast_to(rng.standard_normal((B, N, 1, H, D)), (B, N, S, H, D)).copy()
    v = rng.standard_normal((B, N, S, H, D))
    do = rng.standard_normal((B, N, S, H, D))
    g = _bwd(orc, q, k, v, None, None, do)
    _close(g["dq"], np.zeros_like(q), 1e-12, what="uniform dq")
    mean_do = do.sum(axis=2, keepdims=True) / S
    _close(g["dv"], np.broadcast_to(mean_do, v.shape), 1e-12, what="uniform dv")
    vc = v - v.mean(axis=2, keepdims=True)
    dt = np.einsum("bnihd,bnjhd->bnhij", do, vc) / S
    dk = np.einsum("bnhij,bnihd->bnjhd", dt, q) / math.sqrt(D)
    _close(g["dk"], dk, 1e-12, what="uniform dk")


def pin_bwd_single_key_and_s1(orc):
    """One finite key (the rest -inf): its weight is 1, so dv of that key is
    sum_i dO_i, every other dv is 0, and dq = dk = dmask = dpair = 0.  S = 1
    is the same case with one key."""
    for S, live in ((6, 2), (1, 0)):
        q, k, v, _, p, do = _inputs(7, N=2, S=S, mask_kind=None)
        m = np.full((1, 2, 1, 1, S), -math.inf)
        m[..., live] = 0.25
        g = _bwd(orc, q, k, v, m, p, do)
        dv = np.zeros_like(v)
        dv[:, :, live] = do.sum(axis=2)
        _close(g["dv"], dv, 1e-12, what=f"one key dv (S={S})")
        for name in ("dq", "dk", "dmask", "dpair"):
            _close(g[name], np.zeros_like(g[name]), 1e-12, what=f"one key {name} (S={S})")


def pin_bwd_empty_rows(orc):
    """An n whose keys are all -inf has no softmax (O = 0): its slices get
    zero gradients and add nothing to dpair."""
    q, k, v, m, p, do = _inputs(8, N=3, S=4, mask_kind="finite")
    m[:, 1] = -math.inf
    g = _bwd(orc, q, k, v, m, p, do)
    for name in ("dq", "dk", "dv"):
        _close(g[name][:, 1], np.zeros_like(g[name][:, 1]), 0.0, what=f"empty rows {name}")
    _close(g["dmask"][:, 1], np.zeros_like(g["dmask"][:, 1]), 0.0, what="empty rows dmask")
    keep = [0, 2]
    g2 = _bwd(orc, q[:, keep], k[:, keep], v[:, keep], m[:, keep], p, do[:, keep])
    _close(g["dpair"], g2["dpair"], 1e-13, what="empty rows add nothing to dpair")


# --------------------------------------------------------------- invariants
def pin_bwd_rows_sum_to_zero(orc):
    """Each row of the logit gradient sums to zero over keys (the softmax
    Jacobian annihilates constants), so dmask[b, n, :] and every row
    dpair[b, h, i, :] sum to zero."""
    q, k, v, m, p, do = _inputs(9, 2, 3, 8, 2, 4, mask_kind="some_neg_inf")
    g = _bwd(orc, q, k, v, m, p, do)
    scale = max(1.0, float(np.abs(g["dpair"]).max()))
    _close(g["dmask"].sum(axis=-1), np.zeros(g["dmask"].shape[:-1]), 1e-12 * scale, what="dmask sum")
    _close(g["dpair"].sum(axis=-1), np.zeros(g["dpair"].shape[:-1]), 1e-12 * scale, what="dpair row sums")
    # and the column sums differ from zero (the check above is not vacuous)
    assert np.abs(g["dpair"].sum(axis=-2)).max() > 1e-3


def pin_bwd_mask_shift(orc):
    """Adding a constant to every mask entry of an n shifts its logits by a
    constant: no gradient changes.  With -1e9 on every key of one n (the
    guide's mask for a fully padded column) the gradients equal those of the
    unmasked problem up to the double rounding of logits near -1e9."""
    q, k, v, m, p, do = _inputs(10, N=3, S=6, mask_kind="finite")
    g = _bwd(orc, q, k, v, m, p, do)
    m2 = m.copy()
    m2[:, 1] += 3.75
    g2 = _bwd(orc, q, k, v, m2, p, do)
    for name in g:
        _close(g2[name], g[name], 1e-11, what=f"shift {name}")
    m3 = m.copy()
    m3[:, 2] = -1e9 + m[:, 2]
    g3 = _bwd(orc, q, k, v, m3, p, do)
    for name in g:
        _close(g3[name], g[name], 2e-6, what=f"-1e9 shift {name}")


def pin_bwd_key_permutation(orc):
    """Permuting keys together with their K, V rows, mask entries and pair
    columns leaves dq unchanged and permutes dk, dv, dmask and the columns of
    dpair the same way."""
    q, k, v, m, p, do = _inputs(11, N=2, S=7, mask_kind="finite")
    perm = np.random.default_rng(12).permutation(7)
    g = _bwd(orc, q, k, v, m, p, do)
    gp = _bwd(orc, q, k[:, :, perm], v[:, :, perm], m[..., perm], p[..., perm], do)
    _close(gp["dq"], g["dq"], 1e-12, what="perm dq")
    _close(gp["dk"], g["dk"][:, :, perm], 1e-12, what="perm dk")
    _close(gp["dv"], g["dv"][:, :, perm], 1e-12, what="perm dv")
    _close(gp["dmask"], g["dmask"][..., perm], 1e-12, what="perm dmask")
    _close(gp["dpair"], g["dpair"][..., perm], 1e-12, what="perm dpair")


def pin_bwd_linear_in_do(orc):
    """The backward map is linear in the upstream gradient."""
    q, k, v, m, p, do = _inputs(13, N=2, S=5, mask_kind="finite")
    do2 = np.random.default_rng(14).standard_normal(do.shape)
    g1 = _bwd(orc, q, k, v, m, p, do)
    g2 = _bwd(orc, q, k, v, m, p, do2)
    g3 = _bwd(orc, q, k, v, m, p, 2.0 * do - 0.5 * do2)
    for name in g1:
        _close(g3[name], 2.0 * g1[name] - 0.5 * g2[name], 1e-12, what=f"linear {name}")


ALL_BWD_PINS = [
    pin_bwd_finite_differences,
    pin_bwd_sdpa_autograd,
    pin_bwd_pair_rows_match_autograd,
    pin_bwd_golden,
    pin_bwd_uniform_weights,
    pin_bwd_single_key_and_s1,
    pin_bwd_empty_rows,
    pin_bwd_rows_sum_to_zero,
    pin_bwd_mask_shift,
    pin_bwd_key_permutation,
    pin_bwd_linear_in_do,
]
