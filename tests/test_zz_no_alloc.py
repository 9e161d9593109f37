"""evo_attn_bwd_noalloc (the backward on the library's static scratch) against
evo_attn_bwd (caller workspace): two calls in a row on one stream, each held
to the backward tolerances of tests/parity.py with the workspace entry
point's gradients as the reference; and the refusal of problems whose
scratch does not fit.  Named to be collected last; passes alone too."""
import numpy as np
import pytest
import torch

import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import workloads as W
from tests.parity import check_grads

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dmask", "dpair")


def _inputs(case, seed):
    dev = torch.device("cuda", 0)
    to = (lambda t: None if t is None else t.to(dev))
    rng = np.random.Generator(np.random.PCG64(60_000 + seed))
    do = torch.from_numpy(rng.standard_normal(case.q.shape, dtype=np.float32)).to(case.q.dtype)
    return to(case.q), to(case.k), to(case.v), to(case.mask), to(case.pair), to(do)


def _noalloc(q, k, v, m, p, o, lse, do, stream):
    B, N, S, H, D = q.shape
    out = [torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
           None if m is None else torch.empty_like(m), None if p is None else torch.empty_like(p)]
    ptr = (lambda t: None if t is None else t.data_ptr())
    st = evo.evo_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr(m), ptr(p), o.data_ptr(),
                                  lse.data_ptr(), do.data_ptr(), *[ptr(t) for t in out], B, N, S, H, D,
                                  {torch.bfloat16: evo.EVO_DTYPE_BF16, torch.float32: evo.EVO_DTYPE_FP32,
                                   torch.float16: evo.EVO_DTYPE_FP16}[q.dtype], stream.cuda_stream)
    assert st == evo.EVO_OK, evo.evo_attn_strerror(st)
    return out


@pytest.mark.parametrize("which", ["bf16_tensor_cores", "fp32_simt"])
def test_noalloc_matches_workspace_entry_two_calls(which):
    if which == "bf16_tensor_cores":
        case = W.random_case(1, 4, 200, 2, 32, torch.bfloat16, seed=11, mask="tail", pair=True, fully_masked=1)
    else:
        case = W.random_case(1, 3, 40, 2, 16, torch.float32, seed=12, mask="tail", pair=True)
    q, k, v, m, p, do = _inputs(case, 1)
    B, N, S, H, D = q.shape
    assert evo.evo_attn_bwd_workspace_size(B, N, S, H, D) <= evo.NOALLOC_SCRATCH_BYTES
    stream = torch.cuda.current_stream()
    o, lse = evo.evo_attn(q, k, v, m, p)
    ref = evo.evo_attn_backward(q, k, v, m, p, o, lse, do)
    first = _noalloc(q, k, v, m, p, o, lse, do, stream)
    second = _noalloc(q, k, v, m, p, o, lse, do, stream)
    assert evo.evo_attn_sync_status(stream.cuda_stream) == evo.EVO_OK
    r = {n: g.cpu() for n, g in zip(NAMES, ref) if g is not None}
    for call, got in (("first", first), ("second", second)):
        g = {n: t.cpu() for n, t in zip(NAMES, got) if t is not None}
        check_grads(g, {n: t.double() for n, t in r.items()}, case.dtype, f"noalloc {which} {call} call")


def test_noalloc_refuses_scratch_beyond_its_size():
    dev = torch.device("cuda", 0)
    B, N, S, H, D = 1, 384, 384, 4, 32   # needs about 83 MB of scratch
    need = evo.evo_attn_bwd_workspace_size(B, N, S, H, D)
    assert need > evo.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, N, S, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.zeros((B, N, H, S), dtype=torch.float32, device=dev)
    g = torch.full_like(q, 7.0)
    st = evo.evo_attn_bwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), None, None, q.data_ptr(),
                                  lse.data_ptr(), q.data_ptr(), g.data_ptr(), g.data_ptr(), g.data_ptr(), None, None,
                                  B, N, S, H, D, evo.EVO_DTYPE_BF16, None)
    assert st == evo.EVO_ERR_SCRATCH
    assert "scratch" in evo.evo_attn_strerror(st)
    torch.cuda.synchronize()
    assert bool((g == 7.0).all())        # nothing was launched


def test_noalloc_checks_arguments_like_the_workspace_entry():
    dev = torch.device("cuda", 0)
    case = W.random_case(1, 2, 64, 2, 32, torch.bfloat16, seed=13, mask="none", pair=False)
    q, k, v, m, p, do = _inputs(case, 2)
    o, lse = evo.evo_attn(q, k, v)
    B, N, S, H, D = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dm = torch.empty((B, N, 1, 1, S), dtype=q.dtype, device=dev)
    base = lambda **kw: evo.evo_attn_bwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), None, None, o.data_ptr(), lse.data_ptr(), do.data_ptr(),
        kw.get("dq", dq.data_ptr()), dk.data_ptr(), dv.data_ptr(), kw.get("dm"), None, B, N, S, H, D,
        kw.get("dtype", evo.EVO_DTYPE_BF16), None)
    assert base(dm=dm.data_ptr()) == evo.EVO_ERR_INVALID_ARG        # dmask without a mask
    assert base(dq=q.data_ptr()) == evo.EVO_ERR_INVALID_ARG         # dQ over Q
    assert base(dtype=5) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert base() == evo.EVO_OK
    assert evo.evo_attn_sync_status() == evo.EVO_OK
