"""Float64 oracle for the triangle-multiplication contraction (test
infrastructure only: only the test suite, the smoke check and the benchmark's
CPU-baseline leg use it; the CUDA path shares nothing with it).

What it computes.  The NVIDIA cuEquivariance blog (open-lab.net, "Accelerated
molecular modeling with NVIDIA cuEquivariance and NVIDIA NIM microservices",
the triangle-operations sections) names triangle multiplication beside
triangle attention as the two O(N^3) operations of these models, motivated by
"triangular relationships": if node i is close to k and k is close to j, then
i and j are related.  The page prints no formula.  Reading: the operation is
the contraction over the third node k of two edge representations, channel by
channel, in the two edge directions:

    outgoing:  Z[b, i, j, c] = sum_k A[b, i, k, c] * B[b, j, k, c]
    incoming:  Z[b, i, j, c] = sum_k A[b, k, i, c] * B[b, k, j, c]

with A, B, Z of shape [Bt, N, N, C] (the pair representation's layout: two
node axes, channels last).  The per-edge projections, gates and layer norms
that surround the contraction in a full model are plain per-edge linear
algebra, not part of this O(N^3) step.

The arithmetic: per (b, c), the N x N matrix product of the two channel
slices in float64 (numpy matmul as the library primitive the step is).
Pinned in tests/test_trimul_oracle.py by a pure-Python triple loop, closed
forms and symmetries.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def trimul(a, b, outgoing: bool = True) -> torch.Tensor:
    """Z of the contraction above, float64 torch tensor [Bt, N, N, C]."""
    A, Bm = _f64(a), _f64(b)
    if A.shape != Bm.shape or A.ndim != 4 or A.shape[1] != A.shape[2]:
        raise ValueError("a and b must both be [Bt, N, N, C]")
    Bt, N, _, C = A.shape
    Z = np.empty((Bt, N, N, C))
    for bi in range(Bt):
        for c in range(C):
            a_c = A[bi, :, :, c]
            b_c = Bm[bi, :, :, c]
            if outgoing:
                Z[bi, :, :, c] = a_c @ b_c.T      # sum_k a[i, k] b[j, k]
            else:
                Z[bi, :, :, c] = a_c.T @ b_c      # sum_k a[k, i] b[k, j]
    return torch.from_numpy(Z)


def trimul_entries(a, b, outgoing: bool, entries) -> np.ndarray:
    """Z at selected (b, i, j, c) entries only (each a dot product over k), for
    checks at sizes where the whole result is too slow to form."""
    out = np.empty(len(entries))
    for e, (bi, i, j, c) in enumerate(entries):
        if outgoing:
            x = _f64(a[bi, i, :, c])
            y = _f64(b[bi, j, :, c])
        else:
            x = _f64(a[bi, :, i, c])
            y = _f64(b[bi, :, j, c])
        out[e] = float(np.dot(x, y))
    return out
