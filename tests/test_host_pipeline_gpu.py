"""GPU: the host-memory entry point (evo_attn_fwd_host) returns exactly what
evo_attn_fwd returns on the same inputs, whatever the chunking, and orders
itself on the caller's stream."""
import pytest
import torch

import oracle
import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    evo.load_library()


def pinned(t):
    return None if t is None else t.pin_memory()


def on_device(case):
    dev = torch.device("cuda", 0)
    t = lambda x: None if x is None else x.to(dev)
    o, lse = evo.evo_attn(t(case.q), t(case.k), t(case.v), t(case.mask), t(case.pair))
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def from_host(case, chunk_n, stream=None):
    hin = [pinned(getattr(case, n)) for n in ("q", "k", "v", "mask", "pair")]
    o, lse = evo.evo_attn_from_host(*hin, device="cuda:0", chunk_n=chunk_n, stream=stream)
    if stream is None:
        torch.cuda.current_stream(0).synchronize()
    else:
        stream.synchronize()
    return o, lse


CASES = [
    # B, N, S, H, D, dtype, pair, mask
    (2, 5, 256, 2, 32, torch.bfloat16, True, "tail"),      # tensor-core kernel, two batch entries, odd N
    (1, 6, 200, 3, 64, torch.bfloat16, False, "bernoulli"),  # no pair bias, ragged S
    (1, 3, 70, 2, 48, torch.bfloat16, True, "tail"),       # SIMT bf16 shape
    (2, 3, 45, 2, 16, torch.float32, True, "zero"),        # fp32
]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{str(s[5])[6:]}")
@pytest.mark.parametrize("chunk_n", [0, 1, 2, 3, 100])
def test_host_entry_matches_device_call(shape, chunk_n):
    B, N, S, H, D, dt, pair, mask = shape
    case = W.random_case(B, N, S, H, D, dt, seed=17, mask=mask, pair=pair)
    o_ref, l_ref = on_device(case)
    o, lse = from_host(case, chunk_n)
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_host_entry_against_oracle_on_a_side_stream():
    case = W.random_case(1, 4, 384, 2, 32, torch.bfloat16, seed=3, mask="tail", pair=True)
    s = torch.cuda.Stream(0)
    o, lse = from_host(case, 1, stream=s)
    assert evo.evo_attn_sync_status(s.cuda_stream) == evo.EVO_OK
    o_ref, l_ref = oracle.attention(case.q, case.k, case.v, case.mask, case.pair)
    parity.check(o, lse, o_ref, l_ref, torch.bfloat16, "host entry")


def test_back_to_back_calls_reuse_device_buffers():
    """A second call into the same device buffers starts its copies only after
    the first call's kernels have read them."""
    a = W.random_case(1, 8, 256, 2, 32, torch.bfloat16, seed=1, mask="tail", pair=True)
    b = W.random_case(1, 8, 256, 2, 32, torch.bfloat16, seed=2, mask="tail", pair=True)
    dev = torch.device("cuda", 0)
    like = lambda t: torch.empty(t.shape, dtype=t.dtype, device=dev)
    bufs = (like(a.q), like(a.k), like(a.v), like(a.mask), like(a.pair), like(a.q),
            torch.empty((1, 8, 2, 256), dtype=torch.float32, device=dev))
    outs, host_inputs = [], []
    for c in (a, b):
        # the pinned inputs stay referenced until the synchronize below: the
        # copies run after the call returns
        hin = [pinned(getattr(c, n)) for n in ("q", "k", "v", "mask", "pair")]
        host_inputs.append(hin)
        outs.append(evo.evo_attn_from_host(*hin, device_buffers=bufs, chunk_n=2))
    torch.cuda.current_stream(0).synchronize()
    for c, (o, lse) in zip((a, b), outs):
        o_ref, l_ref = on_device(c)
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_pageable_host_memory_is_refused():
    case = W.random_case(1, 2, 64, 1, 32, torch.bfloat16, seed=4, mask="none", pair=False)
    dev = torch.device("cuda", 0)
    qd, kd, vd = (t.to(dev) for t in (case.q, case.k, case.v))
    od = torch.empty_like(qd)
    ld = torch.empty((1, 2, 1, 64), dtype=torch.float32, device=dev)
    oh = torch.empty_like(case.q)
    lh = torch.empty((1, 2, 1, 64), dtype=torch.float32)
    st = evo.evo_attn_fwd_host(case.q.data_ptr(), case.k.data_ptr(), case.v.data_ptr(), None, None,
                               oh.data_ptr(), lh.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), None, None,
                               od.data_ptr(), ld.data_ptr(), 1, 2, 64, 1, 32, evo.EVO_DTYPE_BF16, 0, None)
    assert st == evo.EVO_ERR_INVALID_ARG
