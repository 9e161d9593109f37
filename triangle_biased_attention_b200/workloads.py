"""Seeded synthetic inputs for biased (Evoformer / Pairformer / triangle) attention.

This module only draws random numbers and lays them out; it performs none of
the attention arithmetic.  Both the float64 oracle and the CUDA path consume
exactly the bytes produced here, so a parity test compares the two on the same
inputs.

Layouts follow the DeepSpeed DS4Sci_EvoformerAttention guide (hmyw.cn, section
5.2 "unified tensor layout"): Q, K, V are ``[B, N, S, H, D]`` (``[*, L, Head,
Dim]``), the residue-mask bias is ``[B, N, 1, 1, S]`` and the pair bias is
``[B, 1, H, S, S]`` (shared across N).  The mask is built the way that guide
says its tests build it, as the additive ``1e9 * (mask - 1)``.

Recipe (one fixed draw order per case, numpy PCG64(seed), float32 normal draws,
then rounded to the case dtype round-to-nearest-even by torch):
  Q, K, V, pair (if present), then the mask parameters.

Named workloads (the shapes of the guide's four variants, section 5.3, at the
residue counts the other pages discuss):
  tiny_fp32     B=1 N=4    S=32   H=2 D=16 fp32, keys 28..31 masked
  tri_start_384 B=1 N=384  S=384  H=4 D=32 bf16, pair N(0,1), tail of 0..48 masked
  msa_row_512   B=1 N=512  S=256  H=8 D=32 bf16, pair N(0,2), ~5% of (n,j) masked
  msa_col_2048  B=1 N=256  S=2048 H=8 D=32 bf16, no pair, per-n tail of 0..512
                masked, plus 2 fully masked n
  tri_1024      B=1 N=1024 S=1024 H=4 D=32 bf16 (D=64 variant: tri_1024_d64),
                pair N(0,1) with 1% of entries set to +8, tail of 0..64 masked
Smaller cases of the same kernels, for single-launch profiler captures
(inputs still larger than the 126 MB L2):
  msa_col_512   B=1 N=256 S=512 H=8 D=32 bf16, no pair, per-n tail of 0..128
                masked, plus 1 fully masked n
  tri_512_d64   B=1 N=512 S=512 H=4 D=64 bf16, generated like tri_1024
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

# The guide's additive mask: 1e9 * (mask - 1), i.e. -1e9 on masked keys.
MASK_SCALE = 1.0e9


@dataclass
class Case:
    """One seeded input set. Tensors live on the host (CPU)."""
    name: str
    seed: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    mask: Optional[torch.Tensor]      # [B, N, 1, 1, S] or None
    pair: Optional[torch.Tensor]      # [B, 1, H, S, S] or None
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        return tuple(self.q.shape)  # (B, N, S, H, D)

    @property
    def dtype(self):
        return self.q.dtype


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    S: int
    H: int
    D: int
    dtype: torch.dtype
    description: str

    @property
    def flops(self) -> int:
        # two contractions of 2*S*S*D each per (b, n, h)
        return 4 * self.B * self.N * self.H * self.S * self.S * self.D


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 4, 32, 2, 16, torch.float32,
                          "tiny correctness case, fp32, keys 28..31 masked"),
    "tri_start_384": Workload("tri_start_384", 1, 384, 384, 4, 32, torch.bfloat16,
                              "triangle attention around the starting node, N_res=384"),
    "msa_row_512": Workload("msa_row_512", 1, 512, 256, 8, 32, torch.bfloat16,
                            "MSA row-wise attention with pair bias, 512 sequences x 256 residues"),
    "msa_col_2048": Workload("msa_col_2048", 1, 256, 2048, 8, 32, torch.bfloat16,
                             "MSA column-wise attention, mask only, 2048 sequences"),
    "tri_1024": Workload("tri_1024", 1, 1024, 1024, 4, 32, torch.bfloat16,
                         "large triangle attention, N_res=1024, D=32"),
    "tri_1024_d64": Workload("tri_1024_d64", 1, 1024, 1024, 4, 64, torch.bfloat16,
                             "large triangle attention, N_res=1024, D=64"),
    "tri_512_d128": Workload("tri_512_d128", 1, 512, 512, 4, 128, torch.bfloat16,
                             "triangle attention, N_res=512, D=128 (head-dim envelope)"),
    "msa_col_512": Workload("msa_col_512", 1, 256, 512, 8, 32, torch.bfloat16,
                            "MSA column-wise attention, mask only, 512 sequences (profiling size)"),
    "tri_512_d64": Workload("tri_512_d64", 1, 512, 512, 4, 64, torch.bfloat16,
                            "triangle attention, N_res=512, D=64 (profiling size)"),
}


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _to(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def _mask_from_keep(keep: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """keep: bool [B, N, S] (True = attend). Returns the guide's 1e9*(mask-1)."""
    m = keep.astype(np.float32)
    bias = np.float32(MASK_SCALE) * (m - np.float32(1.0))
    B, N, S = keep.shape
    return _to(bias.reshape(B, N, 1, 1, S), dtype)


def make_case(name: str, seed: int = 0) -> Case:
    """Build one of the named workloads for a seed."""
    w = WORKLOADS[name]
    B, N, S, H, D = w.B, w.N, w.S, w.H, w.D
    rng = _rng(seed)
    q = _normal(rng, (B, N, S, H, D))
    k = _normal(rng, (B, N, S, H, D))
    v = _normal(rng, (B, N, S, H, D))
    meta = {"workload": name}
    pair = None
    keep = np.ones((B, N, S), dtype=bool)
    if name == "tiny_fp32":
        pair = _normal(rng, (B, 1, H, S, S))
        keep[:, :, 28:] = False
    elif name == "tri_start_384":
        pair = _normal(rng, (B, 1, H, S, S))
        tail = int(rng.integers(0, 49))
        if tail:
            keep[:, :, S - tail:] = False
        meta["tail"] = tail
    elif name == "msa_row_512":
        pair = _normal(rng, (B, 1, H, S, S), std=float(np.sqrt(2.0)))
        keep = rng.random((B, N, S)) >= 0.05
    elif name in ("msa_col_2048", "msa_col_512"):
        tails = rng.integers(0, S // 4 + 1, size=(B, N))
        for b in range(B):
            for n in range(N):
                t = int(tails[b, n])
                if t:
                    keep[b, n, S - t:] = False
        full = rng.choice(N, size=2 if name == "msa_col_2048" else 1, replace=False)
        keep[:, full, :] = False
        meta["fully_masked_n"] = sorted(int(x) for x in full)
    elif name in ("tri_1024", "tri_1024_d64", "tri_512_d128", "tri_512_d64"):
        pair = _normal(rng, (B, 1, H, S, S))
        spikes = rng.random((B, 1, H, S, S)) < 0.01
        pair[spikes] = np.float32(8.0)
        tail = int(rng.integers(0, 65))
        if tail:
            keep[:, :, S - tail:] = False
        meta["tail"] = tail
    else:  # pragma: no cover
        raise KeyError(name)
    dt = w.dtype
    return Case(name=name, seed=seed, q=_to(q, dt), k=_to(k, dt), v=_to(v, dt),
                mask=_mask_from_keep(keep, dt),
                pair=None if pair is None else _to(pair, dt), meta=meta)


def random_case(B: int, N: int, S: int, H: int, D: int, dtype: torch.dtype, seed: int,
                mask: str = "tail", pair: bool = True, pair_std: float = 1.0,
                qkv_std: float = 1.0, spike_frac: float = 0.0, spike: float = 8.0,
                fully_masked: int = 0) -> Case:
    """A free-form seeded case for parity tests at arbitrary shapes.

    mask: "none" (no mask tensor), "zero" (all keys kept), "tail" (random tail of
    up to S//4 keys masked per n), "head" (a random head of S//4 .. S//2 keys
    masked per n, so leading key blocks can be fully masked), "bernoulli" (~5%
    of (n, j) masked), "neg_inf" (random ~10% of keys set to -inf instead of
    -1e9).
    fully_masked: how many n slices get every key masked with -1e9.
    """
    rng = _rng(seed)
    q = _normal(rng, (B, N, S, H, D), qkv_std)
    k = _normal(rng, (B, N, S, H, D), qkv_std)
    v = _normal(rng, (B, N, S, H, D), qkv_std)
    pr = None
    if pair:
        pr = _normal(rng, (B, 1, H, S, S), pair_std)
        if spike_frac > 0:
            pr[rng.random(pr.shape) < spike_frac] = np.float32(spike)
    meta = {"workload": f"random_{B}x{N}x{S}x{H}x{D}", "mask": mask}
    m = None
    if mask != "none":
        keep = np.ones((B, N, S), dtype=bool)
        neg_inf = np.zeros((B, N, S), dtype=bool)
        if mask == "tail":
            tails = rng.integers(0, S // 4 + 1, size=(B, N))
            for b in range(B):
                for n in range(N):
                    t = int(tails[b, n])
                    if t:
                        keep[b, n, S - t:] = False
        elif mask == "head":
            heads = rng.integers(S // 4, S // 2 + 1, size=(B, N))
            for b in range(B):
                for n in range(N):
                    keep[b, n, : int(heads[b, n])] = False
        elif mask == "bernoulli":
            keep = rng.random((B, N, S)) >= 0.05
        elif mask == "neg_inf":
            neg_inf = rng.random((B, N, S)) < 0.10
        elif mask != "zero":
            raise ValueError(mask)
        if fully_masked:
            full = rng.choice(N, size=min(fully_masked, N), replace=False)
            keep[:, full, :] = False
            meta["fully_masked_n"] = sorted(int(x) for x in full)
        bias = np.float32(MASK_SCALE) * (keep.astype(np.float32) - np.float32(1.0))
        bias[neg_inf] = -np.inf
        m = _to(bias.reshape(B, N, 1, 1, S), dtype)
    return Case(name=meta["workload"], seed=seed, q=_to(q, dtype), k=_to(k, dtype),
                v=_to(v, dtype), mask=m, pair=None if pr is None else _to(pr, dtype), meta=meta)


def sample_slices(case_or_shape, count: int, seed: int, must_include_n=()) -> list:
    """Pick (b, n, h) slices for a sampled comparison at full size.

    Slices whose n is in ``must_include_n`` come first (every b and h of those
    n), then distinct random slices up to ``count``.
    """
    if isinstance(case_or_shape, Case):
        B, N, S, H, D = case_or_shape.shape
    else:
        B, N, S, H, D = case_or_shape
    rng = _rng(10_000 + seed)
    chosen = []
    seen = set()
    for n in must_include_n:
        for b in range(B):
            for h in range(H):
                t = (b, int(n), h)
                if t not in seen:
                    seen.add(t)
                    chosen.append(t)
    total = B * N * H
    while len(chosen) < min(count, total):
        idx = int(rng.integers(0, total))
        b, rem = divmod(idx, N * H)
        n, h = divmod(rem, H)
        t = (b, n, h)
        if t not in seen:
            seen.add(t)
            chosen.append(t)
    return chosen


# Triangle multiplication: A, B [Bt, N, N, C] edge representations, standard
# normal draws (A then B) from PCG64(seed), rounded to the dtype.  Named
# sizes: the pair representation of an N-residue crop with the usual 128
# channels.
TRIMUL_WORKLOADS = {
    "trimul_768": (1, 768, 128),
    "trimul_1024": (1, 1024, 128),
    "trimul_512": (1, 512, 128),   # profiling size (inputs 2 x 67 MB, still larger than L2 together)
}


def trimul_case(Bt: int, N: int, C: int, dtype: torch.dtype, seed: int):
    """(A, B) host tensors for the triangle multiplication."""
    rng = _rng(seed)
    a = _normal(rng, (Bt, N, N, C))
    b = _normal(rng, (Bt, N, N, C))
    return _to(a, dtype), _to(b, dtype)
