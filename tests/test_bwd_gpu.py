"""Backward pass on the GPU against the float64 oracle's gradients.

Each case runs the forward pass (evo_attn) and then the backward pass
(evo_attn_backward) through the C ABI on seeded inputs, and compares dQ, dK,
dV and the requested bias gradients with the oracle's chain-rule gradients
of the same inputs and upstream gradient, with the tolerances stated in
tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import workloads as W
from tests.parity import check_grads

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _upstream(case, seed):
    rng = np.random.Generator(np.random.PCG64(50_000 + seed))
    return torch.from_numpy(rng.standard_normal(case.q.shape, dtype=np.float32)).to(case.q.dtype)


def run_bwd(case, do, need_dmask=None, need_dpair=None):
    dev = _dev()
    to = (lambda t: None if t is None else t.to(dev))
    q, k, v, m, p = to(case.q), to(case.k), to(case.v), to(case.mask), to(case.pair)
    o, lse = evo.evo_attn(q, k, v, m, p)
    grads = evo.evo_attn_backward(q, k, v, m, p, o, lse, to(do), need_dmask=need_dmask, need_dpair=need_dpair)
    status = evo.evo_attn_sync_status()
    assert status == evo.EVO_OK, evo.evo_attn_strerror(status)
    names = ("dq", "dk", "dv", "dmask", "dpair")
    return {n: (None if g is None else g.cpu()) for n, g in zip(names, grads)}


def ref_grads(case, do):
    return oracle.attention_bwd(case.q, case.k, case.v, case.mask, case.pair, do)


def compare(case, seed, what, need_dmask=None, need_dpair=None):
    do = _upstream(case, seed)
    got = run_bwd(case, do, need_dmask, need_dpair)
    ref = ref_grads(case, do)
    if need_dmask is False:
        assert got["dmask"] is None
        ref.pop("dmask", None)
    if need_dpair is False:
        assert got["dpair"] is None
        ref.pop("dpair", None)
    return check_grads(got, ref, case.dtype, what)


def test_bwd_tiny_fp32():
    case = W.make_case("tiny_fp32", 0)
    compare(case, 0, "tiny_fp32")


# (B, N, S, H, D, mask, pair, spike_frac, fully_masked).  bf16 with D in
# {16, 32, 64} and a pair bias whose rows are whole 16-byte units (or none)
# runs on the tensor-core kernel; the rest on the SIMT kernels.
BF16_CASES = [
    (1, 4, 200, 2, 32, "tail", True, 0.01, 1),      # tensor cores, ragged blocks, a fully masked n
    (1, 3, 136, 2, 64, "head", True, 0.0, 0),       # tensor cores, D = 64
    (2, 3, 96, 3, 16, "bernoulli", False, 0.0, 0),  # tensor cores, D = 16, no pair bias
    (1, 2, 256, 2, 16, "tail", True, 0.01, 0),      # tensor cores, D = 16, two whole blocks
    (1, 3, 160, 2, 32, "neg_inf", True, 0.0, 0),    # tensor cores, -inf mask entries
    (1, 2, 64, 2, 32, "none", True, 0.0, 0),        # tensor cores, no mask
    (1, 2, 384, 4, 32, "tail", False, 0.0, 1),      # tensor cores, no pair bias, several blocks
    (1, 3, 130, 2, 64, "head", True, 0.0, 0),       # SIMT: pair rows not 16-byte units
    (1, 2, 77, 2, 48, "tail", True, 0.0, 0),        # SIMT: head dim 48
    (1, 1, 1, 1, 32, "zero", True, 0.0, 0),         # SIMT: S = 1
]


@pytest.mark.parametrize("shape", BF16_CASES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[5]}")
def test_bwd_bf16(shape):
    B, N, S, H, D, mask, pair, spike, full = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=S + D, mask=mask, pair=pair, spike_frac=spike,
                         fully_masked=full)
    compare(case, S, f"bf16 {shape}")


def test_bwd_fp32_random():
    case = W.random_case(2, 3, 77, 2, 24, torch.float32, seed=5, mask="tail", pair=True, fully_masked=1)
    compare(case, 5, "fp32 random")


def test_bwd_fp16_tensor_cores():
    case = W.random_case(1, 3, 264, 2, 64, torch.float16, seed=9, mask="bernoulli", pair=True, spike_frac=0.01)
    compare(case, 9, "fp16 D=64 tensor cores")
    case = W.random_case(2, 2, 128, 2, 32, torch.float16, seed=10, mask="none", pair=False)
    compare(case, 10, "fp16 D=32 tensor cores, no biases")


def test_bwd_fp16_d16_tensor_cores():
    case = W.random_case(2, 3, 200, 2, 16, torch.float16, seed=14, mask="head", pair=True)
    compare(case, 14, "fp16 D=16 tensor cores")


def test_bwd_fp16_fully_masked_rows_are_empty():
    # in fp16 the guide's -1e9 mask is -inf: a fully masked n has no softmax
    # and gets zero gradients
    case = W.random_case(1, 3, 120, 2, 32, torch.float16, seed=6, mask="tail", pair=True, fully_masked=1)
    stats = compare(case, 6, "fp16 with an empty n")
    assert stats["dq"]["max_ref"] > 0


def test_bwd_skips_bias_gradients_not_requested():
    case = W.random_case(1, 2, 64, 2, 32, torch.bfloat16, seed=7, mask="tail", pair=True)
    compare(case, 7, "no dmask", need_dmask=False)
    compare(case, 7, "no dpair", need_dpair=False)


def test_bwd_rejects_overlapping_outputs_on_device():
    dev = _dev()
    case = W.random_case(1, 2, 64, 2, 32, torch.bfloat16, seed=8, mask="none", pair=False)
    q, k, v = (t.to(dev) for t in (case.q, case.k, case.v))
    o, lse = evo.evo_attn(q, k, v)
    do = torch.ones_like(q)
    B, N, S, H, D = q.shape
    size = evo.evo_attn_bwd_workspace_size(B, N, S, H, D)
    ws = torch.empty(size, dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    args = lambda dq_ptr: (q.data_ptr(), k.data_ptr(), v.data_ptr(), None, None, o.data_ptr(), lse.data_ptr(),
                           do.data_ptr(), dq_ptr, dk.data_ptr(), dv.data_ptr(), None, None, ws.data_ptr(), size,
                           B, N, S, H, D, evo.EVO_DTYPE_BF16, None)
    assert evo.evo_attn_bwd(*args(q.data_ptr())) == evo.EVO_ERR_INVALID_ARG     # dQ over Q
    assert evo.evo_attn_bwd(*args(dk.data_ptr())) == evo.EVO_ERR_INVALID_ARG    # dQ over dK
    assert evo.evo_attn_bwd(*args(dq.data_ptr())) == evo.EVO_OK
    assert evo.evo_attn_sync_status() == evo.EVO_OK


def test_bwd_tri_1024_sampled():
    """The backward at the full triangle-attention size (B=1, N=S=1024, H=4,
    D=32, the forward's workload), compared on sampled outputs: dQ, dK, dV of
    whole (b, n, h) slices, dmask of whole n (all heads), and rows of dpair
    (each a sum over all 1024 n)."""
    case = W.make_case("tri_1024", 0)
    do = _upstream(case, 0)
    got = run_bwd(case, do)
    orc = oracle.default()
    B, N, S, H, D = case.shape
    fm = case.meta.get("tail", 0)
    slices = [(0, 0, 0), (0, 517, 3), (0, 1023, 1), (0, 301, 2)]
    dq, dk, dv, cs = orc.attention_bwd_slices(case.q, case.k, case.v, case.mask, case.pair, do, slices)
    pick = lambda g: np.stack([g[b, n, :, h, :].double().numpy() for (b, n, h) in slices])
    check_grads({"dq": pick(got["dq"]), "dk": pick(got["dk"]), "dv": pick(got["dv"])},
                {"dq": dq, "dk": dk, "dv": dv}, case.dtype, "tri_1024 sampled slices")
    # dmask of n = 517: the column sums of all four heads' slices
    hs = [(0, 517, h) for h in range(H)]
    _, _, _, cs = orc.attention_bwd_slices(case.q, case.k, case.v, case.mask, case.pair, do, hs)
    ref_m = cs.sum(axis=0)
    check_grads({"dmask": got["dmask"][0, 517, 0, 0].double().numpy()}, {"dmask": ref_m}, case.dtype,
                f"tri_1024 dmask (tail {fm})")
    rows = [(0, 0, 5), (0, 2, 700), (0, 3, 1023)]
    ref_p = orc.pair_grad_rows(case.q, case.k, case.v, case.mask, case.pair, do, rows, chunk=128)
    got_p = np.stack([got["dpair"][b, 0, h, i].double().numpy() for (b, h, i) in rows])
    check_grads({"dpair": got_p}, {"dpair": ref_p}, case.dtype, "tri_1024 dpair rows")


def test_bwd_msa_col_2048_sampled():
    """The backward at the full column-attention size (no pair bias; two n
    whose every key is masked, whose rows take the recomputed LSE): dQ, dK,
    dV of sampled slices including both fully masked n, and dmask of them."""
    case = W.make_case("msa_col_2048", 0)
    do = _upstream(case, 0)
    got = run_bwd(case, do)
    orc = oracle.default()
    B, N, S, H, D = case.shape
    full = case.meta["fully_masked_n"]
    slices = [(0, full[0], 0), (0, full[1], 5), (0, 17, 3), (0, 200, 7)]
    dq, dk, dv, _ = orc.attention_bwd_slices(case.q, case.k, case.v, case.mask, case.pair, do, slices)
    pick = lambda g: np.stack([g[b, n, :, h, :].double().numpy() for (b, n, h) in slices])
    check_grads({"dq": pick(got["dq"]), "dk": pick(got["dk"]), "dv": pick(got["dv"])},
                {"dq": dq, "dk": dk, "dv": dv}, case.dtype, "msa_col_2048 sampled slices")
    for n in (full[0], 17):
        hs = [(0, n, h) for h in range(H)]
        _, _, _, cs = orc.attention_bwd_slices(case.q, case.k, case.v, case.mask, case.pair, do, hs)
        check_grads({"dmask": got["dmask"][0, n, 0, 0].double().numpy()}, {"dmask": cs.sum(axis=0)},
                    case.dtype, f"msa_col_2048 dmask n={n}")
