"""Pins of the float64 triangle-multiplication oracle (CPU only), and planted
mistakes in copies of it that some pin must catch.

The contraction (oracle/trimul.py): outgoing Z_ij = sum_k A_ik B_jk,
incoming Z_ij = sum_k A_ki B_kj, channel by channel.  Each pin ties the
oracle to something other than itself: a pure-Python triple loop, closed
forms (all-ones and identity operands), the symmetry under exchanging A and
B, and the relation between the two directions.
"""
import importlib.util
import itertools
import os

import numpy as np
import pytest
import torch

from oracle import trimul as T

SOURCE = T.__file__


def _rand(seed, Bt=2, N=5, C=3, scale=1.0):
    rng = np.random.default_rng(seed)
    return (torch.from_numpy(rng.standard_normal((Bt, N, N, C)) * scale),
            torch.from_numpy(rng.standard_normal((Bt, N, N, C)) * scale))


def pin_triple_loop(f):
    """Every entry against a pure-Python triple loop (sums in index order)."""
    a, b = _rand(0)
    Bt, N, _, C = a.shape
    for outgoing in (True, False):
        Z = f(a, b, outgoing).numpy()
        for bi, i, j, c in itertools.product(range(Bt), range(N), range(N), range(C)):
            acc = 0.0
            for k in range(N):
                if outgoing:
                    acc += float(a[bi, i, k, c]) * float(b[bi, j, k, c])
                else:
                    acc += float(a[bi, k, i, c]) * float(b[bi, k, j, c])
            assert abs(Z[bi, i, j, c] - acc) <= 1e-12, (outgoing, bi, i, j, c)


def pin_closed_forms(f):
    """A = 1 everywhere: outgoing gives the row sums of B over k (sum_k B_jk),
    incoming the column sums (sum_k B_kj).  A = the identity in (i, k) for every
    channel: outgoing gives B transposed (Z_ij = B_ji), incoming B itself."""
    _, b = _rand(1)
    Bt, N, _, C = b.shape
    ones = torch.ones_like(b)
    Zo = f(ones, b, True).numpy()
    Zi = f(ones, b, False).numpy()
    rows = b.numpy().sum(axis=2)           # [Bt, j, C]: sum_k B[j, k]
    cols = b.numpy().sum(axis=1)           # [Bt, j, C]: sum_k B[k, j]
    assert np.allclose(Zo, np.broadcast_to(rows[:, None, :, :], Zo.shape), rtol=0, atol=1e-12)
    assert np.allclose(Zi, np.broadcast_to(cols[:, None, :, :], Zi.shape), rtol=0, atol=1e-12)
    eye = torch.zeros_like(b)
    for i in range(N):
        eye[:, i, i, :] = 1.0
    assert np.allclose(f(eye, b, True).numpy(), b.numpy().transpose(0, 2, 1, 3), rtol=0, atol=1e-12)
    assert np.allclose(f(eye, b, False).numpy(), b.numpy(), rtol=0, atol=1e-12)


def pin_exchange_symmetry(f):
    """Exchanging A and B transposes the result in (i, j), in both directions."""
    a, b = _rand(2, N=6)
    for outgoing in (True, False):
        Z1 = f(a, b, outgoing).numpy()
        Z2 = f(b, a, outgoing).numpy()
        assert np.allclose(Z1, Z2.transpose(0, 2, 1, 3), rtol=0, atol=1e-12)


def pin_direction_relation(f):
    """Incoming equals outgoing of the operands with their two node axes
    swapped (sum_k A_ki B_kj = sum_k A'_ik B'_jk with A' = A^T, B' = B^T)."""
    a, b = _rand(3, N=7)
    Zi = f(a, b, False).numpy()
    Zo = f(a.transpose(1, 2), b.transpose(1, 2), True).numpy()
    assert np.allclose(Zi, Zo, rtol=0, atol=1e-12)
    # and the two directions differ on general inputs (the relation is not vacuous)
    assert np.abs(Zi - f(a, b, True).numpy()).max() > 1e-3


PINS = [pin_triple_loop, pin_closed_forms, pin_exchange_symmetry, pin_direction_relation]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_trimul_oracle_pin(pin):
    pin(T.trimul)


def test_entries_match_the_whole_result():
    a, b = _rand(4, N=9, C=4)
    for outgoing in (True, False):
        Z = T.trimul(a, b, outgoing).numpy()
        entries = [(0, 0, 0, 0), (1, 8, 3, 2), (0, 4, 7, 3)]
        got = T.trimul_entries(a, b, outgoing, entries)
        assert np.allclose(got, [Z[e] for e in entries], rtol=0, atol=1e-12)


MUTANTS = [
    ("outgoing_without_transpose", "Z[bi, :, :, c] = a_c @ b_c.T      # sum_k a[i, k] b[j, k]",
     "Z[bi, :, :, c] = a_c @ b_c      # sum_k a[i, k] b[j, k]"),
    ("incoming_without_transpose", "Z[bi, :, :, c] = a_c.T @ b_c      # sum_k a[k, i] b[k, j]",
     "Z[bi, :, :, c] = a_c @ b_c      # sum_k a[k, i] b[k, j]"),
    ("directions_swapped", "            if outgoing:\n                Z[bi",
     "            if not outgoing:\n                Z[bi"),
    ("result_transposed", "Z[bi, :, :, c] = a_c @ b_c.T      # sum_k a[i, k] b[j, k]",
     "Z[bi, :, :, c] = (a_c @ b_c.T).T      # sum_k a[i, k] b[j, k]"),
    ("channel_mixed", "b_c = Bm[bi, :, :, c]", "b_c = Bm[bi, :, :, (c + 1) % C]"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_trimul_mutant_is_caught(tmp_path, name, old, new):
    src = open(SOURCE).read()
    assert old in src, f"mutation site for {name} not found"
    path = tmp_path / f"trimul_{name}.py"
    path.write_text(src.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location(f"trimul_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    caught = []
    for pin in PINS:
        try:
            pin(mod.trimul)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
