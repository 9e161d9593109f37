"""The seeded input generators: determinism, shapes and the mask recipe."""
import numpy as np
import torch

from triangle_biased_attention_b200 import workloads as W


def test_deterministic_and_seed_dependent():
    a = W.random_case(1, 3, 40, 2, 16, torch.bfloat16, seed=5)
    b = W.random_case(1, 3, 40, 2, 16, torch.bfloat16, seed=5)
    c = W.random_case(1, 3, 40, 2, 16, torch.bfloat16, seed=6)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.mask, b.mask), (a.pair, b.pair)):
        assert torch.equal(x, y)
    assert not torch.equal(a.q, c.q)


def test_tiny_case_matches_its_description():
    c = W.make_case("tiny_fp32", 0)
    assert c.shape == (1, 4, 32, 2, 16) and c.dtype == torch.float32
    m = c.mask[0, :, 0, 0, :]
    assert torch.all(m[:, :28] == 0) and torch.all(m[:, 28:] == -1e9)
    assert c.pair.shape == (1, 1, 2, 32, 32)


def test_bf16_mask_value_is_rounded_minus_1e9():
    c = W.random_case(1, 2, 64, 1, 16, torch.bfloat16, seed=1, mask="tail", fully_masked=1)
    vals = set(c.mask.float().unique().tolist())
    assert vals <= {0.0, -998244352.0}
    n = c.meta["fully_masked_n"][0]
    assert torch.all(c.mask[0, n] == -998244352.0)


def test_named_workload_shapes_small_ones():
    for name in ("tri_start_384", "msa_row_512"):
        w = W.WORKLOADS[name]
        c = W.make_case(name, 1)
        assert c.shape == (w.B, w.N, w.S, w.H, w.D)
        assert c.pair is not None and c.pair.shape == (w.B, 1, w.H, w.S, w.S)
        assert c.mask.shape == (w.B, w.N, 1, 1, w.S)
    c = W.make_case("tri_start_384", 0)
    tail = c.meta["tail"]
    assert 0 <= tail <= 48
    keep = (c.mask[0, :, 0, 0, :] == 0)
    assert torch.all(keep[:, : 384 - tail]) and not torch.any(keep[:, 384 - tail:])
    r = W.make_case("msa_row_512", 0)
    frac = (r.mask != 0).float().mean().item()
    assert 0.03 < frac < 0.07
    assert abs(r.pair.float().std().item() - np.sqrt(2)) < 0.02


def test_flops():
    assert W.WORKLOADS["tri_1024"].flops == 4 * 1024 * 4 * 1024 * 1024 * 32


def test_sample_slices():
    s = W.sample_slices((1, 256, 2048, 8, 32), 64, 0, must_include_n=[3, 9])
    assert len(s) == 64 and len(set(s)) == 64
    assert all((0, n, h) in s for n in (3, 9) for h in range(8))


def test_half_spacing_bounds_bf16_rounding():
    """Every fp32 value lies within half_spacing_bf16(its bf16 rounding) of
    that rounding: the bound the parity check removes from |dO|."""
    from tests.parity import half_spacing_bf16
    assert np.allclose(half_spacing_bf16(np.array([1.0, 1.5, 2.0, 7.9, -4.0])), [2**-8, 2**-8, 2**-7, 2**-6, 2**-6])
    r = torch.from_numpy(np.random.default_rng(0).standard_normal(200000).astype(np.float32) * 8)
    rb = r.to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(rb - r.double().numpy()) <= half_spacing_bf16(rb))
    # ties go to the even significand: 1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    t = torch.tensor([1.0 + 2**-8, 1.0 + 3 * 2**-8], dtype=torch.float32).to(torch.bfloat16).double()
    assert t.tolist() == [1.0, 1.0 + 2**-6]
