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
