"""GPU: evo_attn_fwd can be captured in a CUDA graph and replayed; a replay
on new data in the same buffers gives what an eager call gives."""
import pytest
import torch

import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    evo.load_library()


SHAPES = [
    # B, N, S, H, D, dtype
    (1, 4, 256, 2, 32, torch.bfloat16),  # tensor-core kernel
    (1, 3, 70, 2, 48, torch.bfloat16),   # SIMT kernel, bf16
    (1, 2, 45, 2, 16, torch.float32),    # SIMT kernel, fp32
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{str(s[5])[6:]}")
def test_forward_replays_in_a_cuda_graph(shape):
    B, N, S, H, D, dt = shape
    dev = torch.device("cuda", 0)
    first = W.random_case(B, N, S, H, D, dt, seed=6, mask="tail", pair=True)
    second = W.random_case(B, N, S, H, D, dt, seed=7, mask="tail", pair=True)
    names = ("q", "k", "v", "mask", "pair")
    bufs = [getattr(first, n).to(dev) for n in names]
    out = torch.empty_like(bufs[0])
    lse = torch.empty((B, N, H, S), dtype=torch.float32, device=dev)

    def eager(case):
        o, l = evo.evo_attn(*(getattr(case, n).to(dev) for n in names))
        torch.cuda.synchronize()
        return o.clone(), l.clone()

    evo.evo_attn(*bufs, out=out, lse=lse)  # one eager call first, as a warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        evo.evo_attn(*bufs, out=out, lse=lse)
    for case in (first, second):
        for buf, n in zip(bufs, names):
            buf.copy_(getattr(case, n))
        out.zero_()
        lse.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert evo.evo_attn_sync_status() == evo.EVO_OK
        o_ref, l_ref = eager(case)
        assert torch.equal(out, o_ref) and torch.equal(lse, l_ref)


BWD_SHAPES = [
    # B, N, S, H, D, dtype: tensor-core backward (fp32 sums by TMA reductions), SIMT backward
    (1, 3, 192, 2, 32, torch.bfloat16),
    (1, 2, 45, 2, 16, torch.float32),
]


@pytest.mark.parametrize("shape", BWD_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{str(s[5])[6:]}")
def test_backward_replays_in_a_cuda_graph(shape):
    """evo_attn_bwd (its zeroing copies and kernels) captured once and replayed on
    new data in the same buffers matches an eager call: bitwise on the SIMT
    path, within the gradient tolerance on the tensor-core path, whose fp32
    sums are added in a varying order."""
    from tests.parity import check_grads
    B, N, S, H, D, dt = shape
    dev = torch.device("cuda", 0)
    cases = [W.random_case(B, N, S, H, D, dt, seed=s, mask="tail", pair=True, fully_masked=1) for s in (8, 9)]
    gen = torch.Generator().manual_seed(3)
    dos = [torch.randn((B, N, S, H, D), generator=gen).to(dt) for _ in cases]
    names = ("q", "k", "v", "mask", "pair")
    ins = [getattr(cases[0], n).to(dev) for n in names]
    do = dos[0].to(dev)
    o, lse = evo.evo_attn(*ins)
    grads = [torch.empty_like(ins[0]) for _ in range(3)] + [torch.empty_like(ins[3]), torch.empty_like(ins[4])]
    ws = torch.empty(evo.evo_attn_bwd_workspace_size(B, N, S, H, D), dtype=torch.uint8, device=dev)
    code = {torch.bfloat16: evo.EVO_DTYPE_BF16, torch.float32: evo.EVO_DTYPE_FP32}[dt]

    def call(stream):
        return evo.evo_attn_bwd(*(t.data_ptr() for t in ins), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                                *(g.data_ptr() for g in grads), ws.data_ptr(), ws.numel(), B, N, S, H, D, code,
                                stream)

    assert call(torch.cuda.current_stream().cuda_stream) == evo.EVO_OK   # eager warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        assert call(torch.cuda.current_stream().cuda_stream) == evo.EVO_OK
    for case, d_h in zip(cases, dos):
        for buf, n in zip(ins, names):
            buf.copy_(getattr(case, n))
        do.copy_(d_h)
        o2, l2 = evo.evo_attn(*ins)
        o.copy_(o2)
        lse.copy_(l2)
        for g in grads:
            g.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert evo.evo_attn_sync_status() == evo.EVO_OK
        ref = evo.evo_attn_backward(*ins, o, lse, do)
        torch.cuda.synchronize()
        got = {n: g.cpu() for n, g in zip(("dq", "dk", "dv", "dmask", "dpair"), grads)}
        want = {n: r.cpu() for n, r in zip(("dq", "dk", "dv", "dmask", "dpair"), ref)}
        if dt == torch.float32:
            for n in got:
                assert torch.equal(got[n], want[n]), n
        else:
            check_grads(got, {n: t.double() for n, t in want.items()}, dt, f"graph replay {shape}")
