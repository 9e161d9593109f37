"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.  Small shapes are compared element by element; the
full-size workloads are compared on every element where the oracle finishes
in seconds and on sampled (b, n, h) slices otherwise."""
import dataclasses

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


def run_gpu(case, stream=None):
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (case.q, case.k, case.v))
    m = None if case.mask is None else case.mask.to(dev)
    p = None if case.pair is None else case.pair.to(dev)
    o, lse = evo.evo_attn(q, k, v, m, p, stream=stream)
    assert evo.evo_attn_sync_status(None if stream is None else stream.cuda_stream) == evo.EVO_OK
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check_full(case, what):
    o, lse = run_gpu(case)
    o_ref, lse_ref = oracle.attention(case.q, case.k, case.v, case.mask, case.pair)
    return parity.check(o, lse, o_ref, lse_ref, case.dtype, what)


def check_sampled(case, slices, what):
    o, lse = run_gpu(case)
    o_ref, lse_ref = oracle.attention_slices(case.q, case.k, case.v, case.mask, case.pair, slices)
    o_s = torch.stack([o[b, n, :, h, :] for (b, n, h) in slices])
    l_s = torch.stack([lse[b, n, h, :] for (b, n, h) in slices])
    return parity.check(o_s, l_s, o_ref, lse_ref, case.dtype, what)


# ------------------------------------------------------------------- fp32 path
@pytest.mark.parametrize("seed", [0, 1, 2, 3, 4])
def test_fp32_tiny_workload(seed):
    check_full(W.make_case("tiny_fp32", seed), f"tiny_fp32 seed {seed}")


FP32_SHAPES = [
    # B, N, S, H, D, pair, mask, fully_masked
    (1, 3, 45, 2, 7, True, "tail", 0),
    (2, 2, 130, 3, 64, True, "tail", 1),
    (1, 1, 1, 1, 1, True, "zero", 0),
    (1, 2, 70, 1, 128, False, "neg_inf", 0),
    (1, 2, 33, 2, 16, False, "none", 0),
]


@pytest.mark.parametrize("shape", FP32_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[6]}")
def test_fp32_random(shape):
    B, N, S, H, D, pair, mask, full = shape
    case = W.random_case(B, N, S, H, D, torch.float32, seed=11, mask=mask, pair=pair, fully_masked=full)
    check_full(case, str(shape))


# ------------------------------------------------------------------- bf16 path
BF16_SHAPES = [
    # B, N, S, H, D, pair, mask, fully_masked, spike_frac
    (1, 3, 200, 2, 32, True, "tail", 0, 0.0),      # ragged second key block, odd N
    (1, 4, 128, 2, 32, True, "bernoulli", 0, 0.0), # exactly one tile
    (2, 2, 136, 3, 64, True, "tail", 1, 0.0),      # D=64, a fully masked n
    (1, 5, 72, 1, 16, True, "tail", 0, 0.0),       # D=16, S below one tile
    (1, 2, 40, 2, 32, False, "tail", 0, 0.0),      # no pair bias
    (1, 3, 264, 2, 64, False, "neg_inf", 0, 0.0),  # -inf mask entries, 3 key blocks
    (1, 1, 8, 1, 32, True, "zero", 0, 0.0),        # tiny S
    (1, 2, 1, 1, 16, False, "none", 0, 0.0),       # S = 1
    (1, 2, 384, 4, 32, True, "none", 0, 0.0),      # no mask tensor
    (1, 2, 300, 2, 32, False, "tail", 2, 0.0),     # S not a multiple of 8, all n masked
    (1, 4, 256, 2, 32, True, "tail", 0, 0.01),     # peaky pair bias (+8 spikes)
    (1, 2, 512, 2, 64, True, "bernoulli", 0, 0.01),
    (1, 3, 640, 2, 32, True, "head", 1, 0.0),      # leading blocks fully masked, then not
    (1, 2, 520, 1, 16, False, "head", 0, 0.0),     # same without pair bias, ragged S
    (1, 2, 256, 2, 128, True, "bernoulli", 0, 0.01),  # D=128: two 128 B swizzle atoms per row
    (1, 3, 136, 1, 128, False, "tail", 1, 0.0),    # D=128, ragged, no pair, a fully masked n
    (2, 3, 384, 2, 64, True, "head", 1, 0.0),      # D=64 (two slices per tile), leading masked blocks
    (1, 7, 128, 1, 64, True, "tail", 0, 0.0),      # D=64, odd N: a tile with one slice
    (1, 4, 72, 2, 128, True, "none", 0, 0.0),      # D=128, S below one tile, S % 8 == 0 with pair bias
]


# Large pair-bias spikes scattered over several key blocks: rows whose maximum
# is raised by more than the kernel's lazy-rescale headroom in a later block
# take its rare recompute path (and rescale O in tensor memory).
SPIKE_SHAPES = [
    # B, N, S, H, D, mask, spike value, spike fraction, seed
    (1, 4, 512, 2, 32, "tail", 24.0, 0.002, 21),
    (1, 2, 384, 1, 128, "bernoulli", 28.0, 0.002, 24),
    (1, 2, 640, 2, 64, "bernoulli", 30.0, 0.001, 22),
    (1, 3, 384, 1, 16, "tail", -40.0, 0.01, 23),
]


@pytest.mark.parametrize("shape", SPIKE_SHAPES, ids=lambda s: f"S{s[2]}-D{s[4]}-spike{s[6]:+g}")
def test_bf16_late_maximum_raises(shape):
    B, N, S, H, D, mask, spike, frac, seed = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=seed, mask=mask, pair=True,
                         spike_frac=frac, spike=spike)
    check_full(case, str(shape))


# Pair bias rising by a fixed amount every 32 keys (one softmax step of the
# tensor-core kernel): with +6 per step (8.7 in log2 units) each new step's p
# reach 2^8.7 against the running maximum, so the step's p sum passes 2^15
# while no single p does (the check's rare path without a raise); with +12
# (17.3 in log2 units) every step raises the maximum and rescales P and O.
RAMP_SHAPES = [
    # B, N, S, H, D, ramp per 32 keys, seed
    (1, 3, 256, 2, 32, 6.0, 31),
    (1, 3, 384, 1, 32, 12.0, 32),
    (1, 2, 200, 2, 64, 6.0, 33),
    (1, 3, 160, 1, 16, 12.0, 34),
]


@pytest.mark.parametrize("shape", RAMP_SHAPES, ids=lambda s: f"S{s[2]}-D{s[4]}-ramp{s[5]:g}")
def test_bf16_rising_steps(shape):
    B, N, S, H, D, ramp, seed = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=seed, mask="none", pair=True)
    steps = (torch.arange(S) // 32).to(torch.float32) * ramp           # per key
    pair = (case.pair.float() + steps.view(1, 1, 1, 1, S)).to(torch.bfloat16)
    case = dataclasses.replace(case, pair=pair)
    check_full(case, str(shape))


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[5]}-{s[6]}")
def test_bf16_random(shape):
    B, N, S, H, D, pair, mask, full, spike = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=3, mask=mask, pair=pair,
                         fully_masked=full, spike_frac=spike)
    check_full(case, str(shape))


# bf16 head dims other than 16, 32, 64 and 128: the SIMT kernel with bf16
# inputs and output
BF16_SIMT_SHAPES = [
    # B, N, S, H, D, pair, mask, fully_masked
    (2, 2, 45, 3, 8, True, "tail", 0),     # small D, ragged S
    (1, 2, 130, 2, 48, False, "tail", 0),  # D not a multiple of 16
    (1, 2, 33, 1, 1, True, "zero", 0),     # D = 1
    (1, 2, 96, 2, 24, False, "neg_inf", 0),
]

# tensor-core shapes whose pair-bias rows are not whole 16-byte units
# (S % 8 != 0): the softmax reads the bias element by element from global
# memory instead of through the TMA ring
BF16_GLOBAL_BIAS_SHAPES = [
    # B, N, S, H, D, pair, mask, fully_masked
    (1, 3, 70, 2, 128, True, "tail", 1),   # D = 128, S < one tile
    (1, 4, 60, 2, 32, True, "tail", 0),    # D = 32
    (1, 5, 301, 2, 32, True, "bernoulli", 1),  # ragged, three key blocks, a fully masked n
    (2, 3, 131, 1, 64, True, "head", 0),   # D = 64, two slices
    (1, 2, 255, 2, 16, True, "none", 0),   # D = 16, no mask tensor (keys past S masked by the kernel)
]


@pytest.mark.parametrize("shape", BF16_GLOBAL_BIAS_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[6]}")
def test_bf16_pair_bias_rows_not_16_byte_units(shape):
    B, N, S, H, D, pair, mask, full = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=6, mask=mask, pair=pair, fully_masked=full)
    check_full(case, str(shape))


@pytest.mark.parametrize("shape", BF16_SIMT_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[5]}-{s[6]}")
def test_bf16_simt_shapes(shape):
    B, N, S, H, D, pair, mask, full = shape
    case = W.random_case(B, N, S, H, D, torch.bfloat16, seed=5, mask=mask, pair=pair, fully_masked=full)
    check_full(case, str(shape))


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("name", ["tri_start_384", "msa_row_512"])
def test_bf16_workload_full(name, seed):
    check_full(W.make_case(name, seed), f"{name} seed {seed}")


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("name", ["msa_col_2048", "tri_1024", "tri_1024_d64", "tri_512_d128"])
def test_bf16_workload_sampled(name, seed):
    case = W.make_case(name, seed)
    slices = W.sample_slices(case, 64, seed, must_include_n=case.meta.get("fully_masked_n", []))
    check_sampled(case, slices, f"{name} seed {seed}")


# --------------------------------------------------------------- behaviour
def test_outputs_stay_inside_their_buffers():
    """Guard regions around O and LSE keep their canary after a launch."""
    case = W.random_case(1, 3, 200, 2, 32, torch.bfloat16, seed=9, mask="tail", pair=True)
    dev = torch.device("cuda", 0)
    B, N, S, H, D = case.shape
    G = 4096
    o_buf = torch.full((G + B * N * S * H * D + G,), -77.0, dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((G + B * N * H * S + G,), -77.0, dtype=torch.float32, device=dev)
    o = o_buf[G:G + B * N * S * H * D].view(B, N, S, H, D)
    lse = l_buf[G:G + B * N * H * S].view(B, N, H, S)
    evo.evo_attn(case.q.to(dev), case.k.to(dev), case.v.to(dev), case.mask.to(dev), case.pair.to(dev),
                 out=o, lse=lse)
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    for buf, n in ((o_buf, B * N * S * H * D), (l_buf, B * N * H * S)):
        assert torch.all(buf[:G] == -77.0) and torch.all(buf[G + n:] == -77.0)
    o_ref, lse_ref = oracle.attention(case.q, case.k, case.v, case.mask, case.pair)
    parity.check(o.cpu(), lse.cpu(), o_ref, lse_ref, torch.bfloat16, "guarded")


def test_repeat_calls_are_bitwise_identical_and_stream_ordered():
    case = W.random_case(1, 4, 256, 2, 32, torch.bfloat16, seed=4, mask="tail", pair=True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1, l1 = run_gpu(case, stream=s)
    o2, l2 = run_gpu(case)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_zero_sized_call_is_a_noop():
    q = torch.empty(1, 0, 64, 2, 32, dtype=torch.bfloat16, device="cuda")
    o, lse = evo.evo_attn(q, q, q)
    assert o.numel() == 0 and lse.numel() == 0


def test_status_is_clear_after_parity_runs():
    assert evo.evo_attn_sync_status() == evo.EVO_OK


def test_buffers_on_another_device_are_rejected():
    """Every buffer must live on Q's device; a host (pinned) buffer is refused
    before anything is launched, and the caller's current device is kept."""
    case = W.random_case(1, 2, 128, 1, 32, torch.bfloat16, seed=8, mask="tail", pair=True)
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (case.q, case.k, case.v))
    o = torch.empty_like(q)
    lse_host = torch.empty((1, 2, 1, 128), dtype=torch.float32).pin_memory()
    before = torch.cuda.current_device()
    st = evo.evo_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), None, None, o.data_ptr(), lse_host.data_ptr(),
                          1, 2, 128, 1, 32, evo.EVO_DTYPE_BF16, None)
    assert st == evo.EVO_ERR_INVALID_ARG
    assert torch.cuda.current_device() == before


# fp16 inputs: the same kernels with fp16 loads, bias, mask and output (the
# score MMA runs fp16 x fp16; V needs no conversion).  The guide's mask
# 1e9 * (mask - 1) is -inf in fp16, so a fully masked n gives O = 0 and
# LSE = -inf.
FP16_SHAPES = [
    # B, N, S, H, D, pair, mask, fully_masked, spike_frac
    (1, 3, 200, 2, 32, True, "tail", 1, 0.0),
    (1, 4, 256, 2, 64, True, "bernoulli", 0, 0.01),
    (1, 2, 136, 1, 128, True, "head", 0, 0.0),
    (1, 5, 60, 2, 16, True, "tail", 0, 0.0),      # S % 8 != 0: bias read element by element
    (1, 3, 520, 2, 32, False, "neg_inf", 1, 0.0),  # no pair bias, five key blocks
    (1, 2, 96, 2, 24, True, "tail", 1, 0.0),      # D = 24: the SIMT kernel
]


@pytest.mark.parametrize("shape", FP16_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + f"-{s[6]}")
def test_fp16_random(shape):
    B, N, S, H, D, pair, mask, full, spike = shape
    case = W.random_case(B, N, S, H, D, torch.float16, seed=7, mask=mask, pair=pair,
                         fully_masked=full, spike_frac=spike)
    check_full(case, str(shape))
