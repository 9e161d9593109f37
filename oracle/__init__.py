"""Float64 CPU oracle for biased attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may import this package.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

The arithmetic lives in ``evo_oracle.c`` (plain C, float64, OpenMP over
independent slices); this module only converts tensors exactly to float64,
gathers per-(b, n, h) slices and calls it.  The formula and the readings it
takes are stated in that file's header (DeepSpeed DS4Sci_EvoformerAttention
guide, hmyw.cn, sections 4, 5.2 and 5.4), together with the chain rule that
the backward entries (``attention_bwd``, ``attention_bwd_slices``,
``pair_grad_rows``) follow.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "evo_oracle.c")
_LIB = os.path.join(_HERE, "libevo_oracle.so")

C_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math"]


def compile_source(src: str, out: str) -> str:
    """Compile an oracle C source into a shared object (atomic replace)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *C_FLAGS, src, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if the shared object is missing or stale."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE)
    if force or stale:
        compile_source(SOURCE, _LIB)
    return _LIB


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """The oracle bound to one compiled shared object."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.evo_oracle_slices.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, p, p, ctypes.c_int]
        lib.evo_oracle_slices.restype = ctypes.c_int
        lib.evo_oracle_bwd_slices.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, i64, p,
                                              p, p, p, p, p, ctypes.c_int]
        lib.evo_oracle_bwd_slices.restype = ctypes.c_int
        lib.evo_oracle_bwd_rows.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, p, i64, p, p, p,
                                            ctypes.c_int]
        lib.evo_oracle_bwd_rows.restype = ctypes.c_int
        lib.evo_oracle_max_threads.argtypes = []
        lib.evo_oracle_max_threads.restype = ctypes.c_int
        self._lib = lib
        self.path = lib_path

    def max_threads(self) -> int:
        return int(self._lib.evo_oracle_max_threads())

    def _run(self, qs, ks, vs, mask_rows, mask_idx, pair_mats, pair_idx, S, D, nthreads):
        ns = qs.shape[0]
        o = np.empty((ns, S, D), dtype=np.float64)
        lse = np.empty((ns, S), dtype=np.float64)
        rc = self._lib.evo_oracle_slices(
            ns, S, D, _ptr(qs), _ptr(ks), _ptr(vs),
            _ptr(mask_rows), _ptr(mask_idx), _ptr(pair_mats), _ptr(pair_idx),
            _ptr(o), _ptr(lse), int(nthreads))
        if rc != 0:
            raise RuntimeError("evo_oracle_slices failed")
        return o, lse

    def attention(self, q, k, v, mask=None, pair=None, nthreads: int = 0):
        """Full forward on every (b, n, h) slice.

        q, k, v: [B, N, S, H, D]; mask: [B, N, 1, 1, S] or None; pair:
        [B, 1, H, S, S] or None.  Returns float64 torch tensors
        O [B, N, S, H, D] and LSE [B, N, H, S] (natural log).
        """
        B, N, S, H, D = q.shape
        qs = _f64(q).transpose(0, 1, 3, 2, 4).reshape(B * N * H, S, D).copy()
        ks = _f64(k).transpose(0, 1, 3, 2, 4).reshape(B * N * H, S, D).copy()
        vs = _f64(v).transpose(0, 1, 3, 2, 4).reshape(B * N * H, S, D).copy()
        b_idx, n_idx, h_idx = np.meshgrid(np.arange(B), np.arange(N), np.arange(H), indexing="ij")
        b_idx, n_idx, h_idx = b_idx.ravel(), n_idx.ravel(), h_idx.ravel()
        mask_rows = mask_idx = pair_mats = pair_idx = None
        if mask is not None:
            mask_rows = _f64(mask).reshape(B * N, S)
            mask_idx = np.ascontiguousarray((b_idx * N + n_idx).astype(np.int64))
        if pair is not None:
            pair_mats = _f64(pair).reshape(B * H, S, S)
            pair_idx = np.ascontiguousarray((b_idx * H + h_idx).astype(np.int64))
        o, lse = self._run(qs, ks, vs, mask_rows, mask_idx, pair_mats, pair_idx, S, D, nthreads)
        O = torch.from_numpy(o.reshape(B, N, H, S, D).transpose(0, 1, 3, 2, 4).copy())
        LSE = torch.from_numpy(lse.reshape(B, N, H, S))
        return O, LSE

    def attention_bwd(self, q, k, v, mask=None, pair=None, do=None, nthreads: int = 0):
        """Gradients of sum(dO * O) on every (b, n, h) slice (the backward pass).

        q, k, v, do: [B, N, S, H, D]; mask, pair as in ``attention``.  Returns a
        dict of float64 torch tensors: dq, dk, dv [B, N, S, H, D]; dmask
        [B, N, 1, 1, S] (the logit gradient summed over heads and query rows)
        when mask is given; dpair [B, 1, H, S, S] (summed over n) when pair is
        given.
        """
        B, N, S, H, D = q.shape
        tr = lambda x: _f64(x).transpose(0, 1, 3, 2, 4).reshape(B * N * H, S, D).copy()
        qs, ks, vs, dos = tr(q), tr(k), tr(v), tr(do)
        b_idx, n_idx, h_idx = np.meshgrid(np.arange(B), np.arange(N), np.arange(H), indexing="ij")
        b_idx, n_idx, h_idx = b_idx.ravel(), n_idx.ravel(), h_idx.ravel()
        mask_rows = mask_idx = pair_mats = pair_idx = dpair = None
        npair = 0
        if mask is not None:
            mask_rows = _f64(mask).reshape(B * N, S)
            mask_idx = np.ascontiguousarray((b_idx * N + n_idx).astype(np.int64))
        if pair is not None:
            pair_mats = _f64(pair).reshape(B * H, S, S)
            pair_idx = np.ascontiguousarray((b_idx * H + h_idx).astype(np.int64))
            npair = B * H
            dpair = np.empty((B * H, S, S))
        ns = B * N * H
        dq = np.empty((ns, S, D)); dk = np.empty((ns, S, D)); dv = np.empty((ns, S, D))
        colsum = np.empty((ns, S))
        rc = self._lib.evo_oracle_bwd_slices(
            ns, S, D, _ptr(qs), _ptr(ks), _ptr(vs), _ptr(mask_rows), _ptr(mask_idx),
            _ptr(pair_mats), _ptr(pair_idx), npair, _ptr(dos),
            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(colsum), _ptr(dpair), int(nthreads))
        if rc != 0:
            raise RuntimeError("evo_oracle_bwd_slices failed")
        back = lambda a: torch.from_numpy(a.reshape(B, N, H, S, D).transpose(0, 1, 3, 2, 4).copy())
        out = {"dq": back(dq), "dk": back(dk), "dv": back(dv)}
        if mask is not None:
            cs = colsum.reshape(B, N, H, S)
            acc = np.zeros((B, N, S))
            for h in range(H):          # heads added in index order
                acc += cs[:, :, h, :]
            out["dmask"] = torch.from_numpy(acc.reshape(B, N, 1, 1, S))
        if pair is not None:
            out["dpair"] = torch.from_numpy(dpair.reshape(B, 1, H, S, S))
        return out

    def _gather(self, q, k, v, mask, pair, do, slices):
        B, N, S, H, D = q.shape
        ns = len(slices)
        qs = np.empty((ns, S, D)); ks = np.empty((ns, S, D)); vs = np.empty((ns, S, D))
        dos = np.empty((ns, S, D))
        mask_rows = mask_idx = pair_mats = pair_idx = None
        if mask is not None:
            mask_rows = np.empty((ns, S)); mask_idx = np.arange(ns, dtype=np.int64)
        if pair is not None:
            keys = {}
            pair_idx = np.empty(ns, dtype=np.int64)
            for s, (b, n, h) in enumerate(slices):
                pair_idx[s] = keys.setdefault((b, h), len(keys))
            pair_mats = np.empty((len(keys), S, S))
            for (b, h), idx in keys.items():
                pair_mats[idx] = _f64(pair[b, 0, h])
        for s, (b, n, h) in enumerate(slices):
            qs[s] = _f64(q[b, n, :, h, :])
            ks[s] = _f64(k[b, n, :, h, :])
            vs[s] = _f64(v[b, n, :, h, :])
            dos[s] = _f64(do[b, n, :, h, :])
            if mask is not None:
                mask_rows[s] = _f64(mask[b, n, 0, 0, :])
        return qs, ks, vs, dos, mask_rows, mask_idx, pair_mats, pair_idx

    def attention_bwd_slices(self, q, k, v, mask, pair, do, slices: Sequence, nthreads: int = 0):
        """Backward on selected (b, n, h) slices only: float64 numpy arrays dq,
        dk, dv [len(slices), S, D] and the per-slice column sums of the logit
        gradient [len(slices), S] (one head's share of dmask)."""
        B, N, S, H, D = q.shape
        qs, ks, vs, dos, mr, mi, pm, pi = self._gather(q, k, v, mask, pair, do, slices)
        ns = len(slices)
        dq = np.empty((ns, S, D)); dk = np.empty((ns, S, D)); dv = np.empty((ns, S, D))
        colsum = np.empty((ns, S))
        npair = 0 if pm is None else pm.shape[0]
        rc = self._lib.evo_oracle_bwd_slices(
            ns, S, D, _ptr(qs), _ptr(ks), _ptr(vs), _ptr(mr), _ptr(mi), _ptr(pm), _ptr(pi), npair,
            _ptr(dos), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(colsum), None, int(nthreads))
        if rc != 0:
            raise RuntimeError("evo_oracle_bwd_slices failed")
        return dq, dk, dv, colsum

    def pair_grad_rows(self, q, k, v, mask, pair, do, rows: Sequence, chunk: int = 64,
                       nthreads: int = 0):
        """Rows of the pair-bias gradient, dpair[b, h, i, :] = sum over n of the
        logit gradient of query row i in slice (b, n, h), for each (b, h, i) in
        ``rows``; float64 numpy [len(rows), S].  Slices are gathered ``chunk``
        n at a time and the chunks added in order of n."""
        B, N, S, H, D = q.shape
        out = np.zeros((len(rows), S))
        for r, (b, h, i) in enumerate(rows):
            for n0 in range(0, N, chunk):
                slices = [(b, n, h) for n in range(n0, min(N, n0 + chunk))]
                qs, ks, vs, dos, mr, mi, pm, pi = self._gather(q, k, v, mask, pair, do, slices)
                nr = len(slices)
                rs = np.arange(nr, dtype=np.int64)
                ri = np.full(nr, i, dtype=np.int64)
                dt = np.empty((nr, S))
                rc = self._lib.evo_oracle_bwd_rows(
                    nr, S, D, _ptr(qs), _ptr(ks), _ptr(vs), _ptr(mr), _ptr(mi), _ptr(pm), _ptr(pi),
                    _ptr(dos), nr, _ptr(rs), _ptr(ri), _ptr(dt), int(nthreads))
                if rc != 0:
                    raise RuntimeError("evo_oracle_bwd_rows failed")
                for x in dt:            # n in index order
                    out[r] += x
        return out

    def attention_slices(self, q, k, v, mask, pair, slices: Sequence, nthreads: int = 0):
        """Forward on selected (b, n, h) slices only.

        Returns float64 numpy arrays O [len(slices), S, D] and LSE
        [len(slices), S] in the order of ``slices``.  Only the selected slices
        are converted to float64, so the tensors may be any size.
        """
        B, N, S, H, D = q.shape
        ns = len(slices)
        qs = np.empty((ns, S, D)); ks = np.empty((ns, S, D)); vs = np.empty((ns, S, D))
        mask_rows = mask_idx = pair_mats = pair_idx = None
        if mask is not None:
            mask_rows = np.empty((ns, S)); mask_idx = np.arange(ns, dtype=np.int64)
        if pair is not None:
            keys = {}
            pair_idx = np.empty(ns, dtype=np.int64)
            for s, (b, n, h) in enumerate(slices):
                pair_idx[s] = keys.setdefault((b, h), len(keys))
            pair_mats = np.empty((len(keys), S, S))
            for (b, h), idx in keys.items():
                pair_mats[idx] = _f64(pair[b, 0, h])
        for s, (b, n, h) in enumerate(slices):
            qs[s] = _f64(q[b, n, :, h, :])
            ks[s] = _f64(k[b, n, :, h, :])
            vs[s] = _f64(v[b, n, :, h, :])
            if mask is not None:
                mask_rows[s] = _f64(mask[b, n, 0, 0, :])
        return self._run(qs, ks, vs, mask_rows, mask_idx, pair_mats, pair_idx, S, D, nthreads)


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def attention(q, k, v, mask=None, pair=None, nthreads: int = 0):
    return default().attention(q, k, v, mask, pair, nthreads)


def attention_slices(q, k, v, mask, pair, slices, nthreads: int = 0):
    return default().attention_slices(q, k, v, mask, pair, slices, nthreads)


def attention_bwd(q, k, v, mask=None, pair=None, do=None, nthreads: int = 0):
    return default().attention_bwd(q, k, v, mask, pair, do, nthreads)


def max_threads() -> int:
    return default().max_threads()
