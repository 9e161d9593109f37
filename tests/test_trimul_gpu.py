"""Triangle multiplication on the GPU against the float64 oracle.

Bound, per element: the GPU computes each dot product over k with products
exact in fp32 (16-bit inputs) and fp32 accumulation, then rounds Z to the
input type.  With u = 2^-24 and gamma_N = N u / (1 - N u), an fp32 sum of N
terms in any order is within gamma_N * sum_k |a_k b_k| of the exact sum, and
rounding adds at most half the output spacing:
    |Z_gpu - Z_ref| <= half_spacing(Z_gpu) + 4 gamma_N (|A| x |B|)
(the factor 4 is margin for the tensor core's internal order; the largest
ratio of error to bound is printed).
"""
import numpy as np
import pytest
import torch

import triangle_biased_attention_b200 as evo
from oracle import trimul as T
from tests.parity import half_spacing_bf16
from triangle_biased_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def check(z_gpu, z_ref, z_abs, N, dtype, what):
    z_gpu = z_gpu.double().cpu().numpy() if isinstance(z_gpu, torch.Tensor) else np.asarray(z_gpu, dtype=np.float64)
    z_ref = np.asarray(z_ref, dtype=np.float64)
    assert np.all(np.isfinite(z_gpu)), what
    u = 2.0 ** -24
    gamma = N * u / (1 - N * u)
    bound = half_spacing_bf16(z_gpu, 8 if dtype == torch.bfloat16 else 11) + 4 * gamma * np.asarray(z_abs)
    err = np.abs(z_gpu - z_ref)
    ratio = float((err / np.maximum(bound, 1e-300)).max(initial=0))
    print(f"trimul parity {what}: max|dZ| {err.max(initial=0):.3e}, max|Z| {np.abs(z_ref).max(initial=0):.3e}, "
          f"max err/bound {ratio:.3f}")
    assert ratio <= 1.0, what


# (Bt, N, C, dtype)
SHAPES = [
    (1, 128, 8, torch.bfloat16),
    (2, 200, 5, torch.bfloat16),     # ragged tiles, channels not a multiple of 32
    (1, 37, 3, torch.bfloat16),      # N not a multiple of 8 (padded rows)
    (1, 1, 4, torch.bfloat16),       # N = 1
    (1, 256, 33, torch.float16),
    (1, 130, 64, torch.float16),
]


@pytest.mark.parametrize("outgoing", [True, False], ids=["outgoing", "incoming"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}x{s[2]}-{str(s[3])[6:]}")
def test_trimul_matches_oracle(shape, outgoing):
    Bt, N, C, dt = shape
    a, b = W.trimul_case(Bt, N, C, dt, seed=N + C)
    dev = torch.device("cuda", 0)
    z = evo.trimul(a.to(dev), b.to(dev), outgoing=outgoing)
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    ref = T.trimul(a, b, outgoing).numpy()
    zabs = T.trimul(a.abs(), b.abs(), outgoing).numpy()
    check(z, ref, zabs, N, dt, f"{shape} {'outgoing' if outgoing else 'incoming'}")


@pytest.mark.parametrize("outgoing", [True, False], ids=["outgoing", "incoming"])
def test_trimul_768_sampled(outgoing):
    """The bench size (Bt=1, N=768, C=128), on 512 sampled entries."""
    Bt, N, C = W.TRIMUL_WORKLOADS["trimul_768"]
    a, b = W.trimul_case(Bt, N, C, torch.bfloat16, seed=0)
    dev = torch.device("cuda", 0)
    z = evo.trimul(a.to(dev), b.to(dev), outgoing=outgoing).cpu()
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    rng = np.random.default_rng(5)
    ent = [(0, int(i), int(j), int(c)) for i, j, c in zip(rng.integers(0, N, 512), rng.integers(0, N, 512),
                                                          rng.integers(0, C, 512))]
    ent += [(0, N - 1, N - 1, C - 1), (0, 0, 0, 0), (0, 767, 0, 64)]
    ref = T.trimul_entries(a, b, outgoing, ent)
    zabs = T.trimul_entries(a.abs(), b.abs(), outgoing, ent)
    got = np.array([float(z[e]) for e in ent])
    check(got, ref, zabs, N, torch.bfloat16, f"trimul_768 sampled {'outgoing' if outgoing else 'incoming'}")


def test_trimul_rejects_bad_arguments_on_device():
    dev = torch.device("cuda", 0)
    a = torch.zeros((1, 16, 16, 4), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(evo.evo_trimul_workspace_size(1, 16, 4), dtype=torch.uint8, device=dev)
    z = torch.empty_like(a)
    call = lambda zp, wb, dt=evo.EVO_DTYPE_BF16: evo.evo_trimul(a.data_ptr(), a.data_ptr(), zp, ws.data_ptr(), wb,
                                                                1, 16, 4, 1, dt, None)
    assert call(a.data_ptr(), ws.numel()) == evo.EVO_ERR_INVALID_ARG         # Z over A
    assert call(z.data_ptr(), ws.numel() - 1) == evo.EVO_ERR_INVALID_ARG     # workspace too small
    assert call(z.data_ptr(), ws.numel(), evo.EVO_DTYPE_FP32) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert call(z.data_ptr(), ws.numel()) == evo.EVO_OK
    assert evo.evo_attn_sync_status() == evo.EVO_OK
