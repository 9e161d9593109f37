"""B200-native biased (Evoformer / Pairformer / triangle) attention.

The computation is the forward pass of the DeepSpeed DS4Sci_EvoformerAttention
guide (hmyw.cn, sections 4, 5.2-5.4):

    O   = softmax(Q K^T / sqrt(D) + mask_bias + pair_bias) V
    LSE = log sum exp of the same logits (natural log, fp32)

with Q, K, V, O of shape [B, N, S, H, D], mask_bias [B, N, 1, 1, S] and
pair_bias [B, 1, H, S, S] (shared by every n), and its backward pass (the
gradients of Q, K, V and of the biases, sections 1 and 5.4).  All arithmetic runs in the
CUDA library ``libevoattn.so`` (hand-written sm_100a kernels behind the C ABI
in ``include/evo_attn.h``); this module only marshals arguments through
ctypes.  PyTorch supplies device memory and the current stream.  There is no
fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "evo_attn", "evo_attn_fwd", "evo_attn_sync_status", "evo_attn_strerror", "evo_attn_version",
    "evo_attn_selftest_timeout", "evo_attn_bwd", "evo_attn_bwd_workspace_size", "evo_attn_backward",
    "EvoAttnError", "library_path", "load_library",
    "EVO_DTYPE_BF16", "EVO_DTYPE_FP32", "EVO_DTYPE_FP16",
    "EVO_OK", "EVO_ERR_INVALID_ARG", "EVO_ERR_UNSUPPORTED_DTYPE", "EVO_ERR_UNSUPPORTED_SHAPE",
    "EVO_ERR_MISALIGNED", "EVO_ERR_CUDA", "EVO_ERR_TIMEOUT", "EVO_ERR_RANGE", "EVO_ERR_SCRATCH",
    "evo_attn_bwd_noalloc", "NOALLOC_SCRATCH_BYTES", "evo_trimul", "evo_trimul_workspace_size", "trimul",
]

EVO_DTYPE_BF16 = 0
EVO_DTYPE_FP32 = 1
EVO_DTYPE_FP16 = 2

EVO_OK = 0
EVO_ERR_INVALID_ARG = -1
EVO_ERR_UNSUPPORTED_DTYPE = -2
EVO_ERR_UNSUPPORTED_SHAPE = -3
EVO_ERR_MISALIGNED = -4
EVO_ERR_CUDA = -5
EVO_ERR_TIMEOUT = -6
EVO_ERR_RANGE = -7
EVO_ERR_SCRATCH = -8

# size of the static scratch behind evo_attn_bwd_noalloc (EVO_ATTN_NOALLOC_SCRATCH_BYTES)
NOALLOC_SCRATCH_BYTES = 64 << 20

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libevoattn.so")
_lib = None

_DTYPES = {torch.bfloat16: EVO_DTYPE_BF16, torch.float32: EVO_DTYPE_FP32, torch.float16: EVO_DTYPE_FP16}


class EvoAttnError(RuntimeError):
    def __init__(self, status: int, what: str = "evo_attn_fwd"):
        self.status = status
        super().__init__(f"{what} failed with status {status}: {evo_attn_strerror(status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libevoattn.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m triangle_biased_attention_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.evo_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, vp]
    lib.evo_attn_fwd.restype = i32
    lib.evo_attn_fwd_host.argtypes = [vp] * 14 + [i64, i64, i64, i64, i64, i32, i64, vp]
    lib.evo_attn_fwd_host.restype = i32
    lib.evo_attn_sync_status.argtypes = [vp]
    lib.evo_attn_sync_status.restype = i32
    lib.evo_attn_strerror.argtypes = [i32]
    lib.evo_attn_strerror.restype = ctypes.c_char_p
    lib.evo_attn_version.argtypes = []
    lib.evo_attn_version.restype = i32
    lib.evo_attn_selftest_timeout.argtypes = [i64, vp, vp]
    lib.evo_attn_selftest_timeout.restype = i32
    lib.evo_attn_bwd_workspace_size.argtypes = [i64, i64, i64, i64, i64]
    lib.evo_attn_bwd_workspace_size.restype = i64
    lib.evo_attn_bwd.argtypes = [vp] * 14 + [i64, i64, i64, i64, i64, i64, i32, vp]
    lib.evo_attn_bwd.restype = i32
    lib.evo_attn_bwd_noalloc.argtypes = [vp] * 13 + [i64, i64, i64, i64, i64, i32, vp]
    lib.evo_attn_bwd_noalloc.restype = i32
    lib.evo_trimul_workspace_size.argtypes = [i64, i64, i64]
    lib.evo_trimul_workspace_size.restype = i64
    lib.evo_trimul.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, vp]
    lib.evo_trimul.restype = i32
    _lib = lib
    return lib


def evo_attn_fwd(Q: int, K: int, V: int, mask_bias: Optional[int], pair_bias: Optional[int], O: int, LSE: int,
                 B: int, N: int, S: int, H: int, D: int, dtype: int, stream: Optional[int]) -> int:
    """The C entry point with raw addresses (ints); returns the status code."""
    return int(load_library().evo_attn_fwd(Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, dtype, stream))


def evo_attn_fwd_host(Qh, Kh, Vh, mask_h, pair_h, Oh, LSEh, Qd, Kd, Vd, mask_d, pair_d, Od, LSEd,
                      B: int, N: int, S: int, H: int, D: int, dtype: int, chunk_n: int,
                      stream: Optional[int]) -> int:
    """The C entry point for host-memory inputs, raw addresses; returns the status code."""
    return int(load_library().evo_attn_fwd_host(Qh, Kh, Vh, mask_h, pair_h, Oh, LSEh, Qd, Kd, Vd, mask_d, pair_d,
                                                Od, LSEd, B, N, S, H, D, dtype, chunk_n, stream))


def evo_attn_sync_status(stream: Optional[int] = None) -> int:
    return int(load_library().evo_attn_sync_status(stream))


def evo_attn_strerror(status: int) -> str:
    return load_library().evo_attn_strerror(int(status)).decode()


def evo_attn_version() -> int:
    return int(load_library().evo_attn_version())


def evo_attn_selftest_timeout(limit_ns: int, result_ptr: int, stream: Optional[int] = None) -> int:
    """Launch the bounded-wait self-test (see include/evo_attn.h); returns the status code."""
    return int(load_library().evo_attn_selftest_timeout(limit_ns, result_ptr, stream))


def evo_attn_bwd_workspace_size(B: int, N: int, S: int, H: int, D: int) -> int:
    """Workspace bytes of evo_attn_bwd, or a negative status code."""
    return int(load_library().evo_attn_bwd_workspace_size(B, N, S, H, D))


def evo_attn_bwd(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, workspace,
                 workspace_bytes: int, B: int, N: int, S: int, H: int, D: int, dtype: int,
                 stream: Optional[int]) -> int:
    """The C backward entry point with raw addresses (ints); returns the status code."""
    return int(load_library().evo_attn_bwd(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair,
                                           workspace, workspace_bytes, B, N, S, H, D, dtype, stream))


def evo_attn_bwd_noalloc(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair,
                         B: int, N: int, S: int, H: int, D: int, dtype: int, stream: Optional[int]) -> int:
    """The C backward entry point that uses the library's static scratch (no
    workspace argument, no allocation); raw addresses; returns the status code."""
    return int(load_library().evo_attn_bwd_noalloc(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask,
                                                   dpair, B, N, S, H, D, dtype, stream))


def evo_trimul_workspace_size(Bt: int, N: int, C: int) -> int:
    """Workspace bytes of evo_trimul, or a negative status code."""
    return int(load_library().evo_trimul_workspace_size(Bt, N, C))


def evo_trimul(A, B, Z, workspace, workspace_bytes: int, Bt: int, N: int, C: int, outgoing: int, dtype: int,
               stream: Optional[int]) -> int:
    """The C triangle-multiplication entry point with raw addresses; returns the status code."""
    return int(load_library().evo_trimul(A, B, Z, workspace, workspace_bytes, Bt, N, C, outgoing, dtype, stream))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def evo_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             mask: Optional[torch.Tensor] = None, pair: Optional[torch.Tensor] = None,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Biased-attention forward on CUDA tensors; returns (O, LSE).

    q, k, v: [B, N, S, H, D] bf16, fp16 or fp32, contiguous, on one CUDA device.
    mask: [B, N, 1, 1, S] or None.  pair: [B, 1, H, S, S] or None (same dtype).
    out / lse: optional preallocated outputs ([B, N, S, H, D], [B, N, H, S] fp32).
    Runs on ``stream`` (default: the current stream) without synchronising.
    """
    if q.dim() != 5:
        raise ValueError("q must be [B, N, S, H, D]")
    B, N, S, H, D = q.shape
    if q.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for name, t, shape in (("k", k, q.shape), ("v", v, q.shape),
                           ("mask", mask, (B, N, 1, 1, S)), ("pair", pair, (B, 1, H, S, S))):
        if t is None:
            continue
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q dtype {q.dtype}")
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")
    for name, t in (("q", q), ("k", k), ("v", v), ("mask", mask), ("pair", pair)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.device.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, N, H, S), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    status = evo_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(mask), _ptr(pair),
                          out.data_ptr(), lse.data_ptr(), B, N, S, H, D, _DTYPES[q.dtype],
                          stream.cuda_stream)
    if status != EVO_OK:
        raise EvoAttnError(status)
    return out, lse


def evo_attn_from_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       mask: Optional[torch.Tensor] = None, pair: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       device_buffers: Optional[Tuple] = None, device=None, chunk_n: int = 0,
                       stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Biased-attention forward on page-locked host tensors; returns (O, LSE) on the host.

    Same shapes and dtypes as ``evo_attn``, all on the CPU and pinned.  The
    copies to and from the device overlap the computation (``evo_attn_fwd_host``
    in include/evo_attn.h).  ``device_buffers`` = (q, k, v, mask, pair, out,
    lse) device tensors of the full shapes (mask / pair None when absent);
    allocated on ``device`` (default: the current CUDA device) when not given.
    Asynchronous on ``stream``: synchronise it before reading the results, and
    keep the host inputs unchanged until then.  The returned O holds
    references to the inputs and device buffers, so that they are not freed
    (and their page-locked blocks not handed out again by PyTorch's host
    allocator, which does not see the library's copies) while O is alive.
    """
    if q.dim() != 5:
        raise ValueError("q must be [B, N, S, H, D]")
    B, N, S, H, D = q.shape
    if q.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for name, t, shape in (("k", k, q.shape), ("v", v, q.shape),
                           ("mask", mask, (B, N, 1, 1, S)), ("pair", pair, (B, 1, H, S, S))):
        if t is None:
            continue
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} differs from q dtype {q.dtype}")
    def host_ok(name, t):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous() or not t.is_pinned()):
            raise ValueError(f"{name} must be a contiguous page-locked host tensor")

    for name, t in (("q", q), ("k", k), ("v", v), ("mask", mask), ("pair", pair), ("out", out), ("lse", lse)):
        host_ok(name, t)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, N, H, S), dtype=torch.float32, pin_memory=True)
    if device_buffers is None:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        like = lambda t: None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev)
        device_buffers = (like(q), like(k), like(v), like(mask), like(pair), like(out), like(lse))
    qd, kd, vd, md, pd, od, ld = device_buffers
    if stream is None:
        stream = torch.cuda.current_stream(qd.device)
    # The copies and kernels run on `stream` (and on the library's copy
    # streams, which `stream` waits for before the call ends): tell PyTorch's
    # allocator, so that a buffer dropped early is not handed out again on
    # its allocation stream while the call still uses it.
    for t in device_buffers:
        if t is not None:
            t.record_stream(stream)
    status = evo_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(mask), _ptr(pair),
                               out.data_ptr(), lse.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                               _ptr(md), _ptr(pd), od.data_ptr(), ld.data_ptr(), B, N, S, H, D,
                               _DTYPES[q.dtype], int(chunk_n), stream.cuda_stream)
    if status != EVO_OK:
        raise EvoAttnError(status, "evo_attn_fwd_host")
    out._evo_keepalive = (q, k, v, mask, pair, device_buffers)
    return out, lse


def evo_attn_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      mask: Optional[torch.Tensor], pair: Optional[torch.Tensor],
                      o: torch.Tensor, lse: torch.Tensor, do: torch.Tensor,
                      need_dmask: Optional[bool] = None, need_dpair: Optional[bool] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None):
    """Backward pass on CUDA tensors; returns (dq, dk, dv, dmask, dpair).

    q, k, v, mask, pair: the forward's inputs; o, lse: its outputs (from
    ``evo_attn``); do: the gradient with respect to o ([B, N, S, H, D], q's
    dtype).  dmask ([B, N, 1, 1, S]) is computed when ``need_dmask`` (default:
    a mask was passed), dpair ([B, 1, H, S, S]) when ``need_dpair`` (default:
    a pair bias was passed); a gradient not computed comes back as None.
    ``workspace``: an optional uint8 CUDA tensor of at least
    ``evo_attn_bwd_workspace_size`` bytes (allocated here when not given).
    Runs on ``stream`` (default: the current stream) without synchronising.
    """
    if q.dim() != 5:
        raise ValueError("q must be [B, N, S, H, D]")
    B, N, S, H, D = q.shape
    if q.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {q.dtype}")
    need_dmask = (mask is not None) if need_dmask is None else bool(need_dmask)
    need_dpair = (pair is not None) if need_dpair is None else bool(need_dpair)
    if need_dmask and mask is None:
        raise ValueError("dmask requested without a mask")
    if need_dpair and pair is None:
        raise ValueError("dpair requested without a pair bias")
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, q.shape, q.dtype),
                               ("mask", mask, (B, N, 1, 1, S), q.dtype), ("pair", pair, (B, 1, H, S, S), q.dtype),
                               ("o", o, q.shape, q.dtype), ("lse", lse, (B, N, H, S), torch.float32),
                               ("do", do, q.shape, q.dtype)):
        if t is None:
            continue
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if t.dtype != dt:
            raise TypeError(f"{name} dtype {t.dtype}, expected {dt}")
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.device.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    need = evo_attn_bwd_workspace_size(B, N, S, H, D)
    if need < 0:
        raise EvoAttnError(need, "evo_attn_bwd_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dmask = torch.empty_like(mask) if need_dmask else None
    dpair = torch.empty_like(pair) if need_dpair else None
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    status = evo_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(mask), _ptr(pair), o.data_ptr(),
                          lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), _ptr(dmask),
                          _ptr(dpair), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          B, N, S, H, D, _DTYPES[q.dtype], stream.cuda_stream)
    if status != EVO_OK:
        raise EvoAttnError(status, "evo_attn_bwd")
    return dq, dk, dv, dmask, dpair


def trimul(a: torch.Tensor, b: torch.Tensor, outgoing: bool = True, out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Triangle multiplication on CUDA tensors: a, b [Bt, N, N, C] bf16 or fp16,
    contiguous; returns Z [Bt, N, N, C] with Z[:, i, j] = sum_k a[:, i, k] b[:, j, k]
    (outgoing) or sum_k a[:, k, i] b[:, k, j] (incoming), channel by channel.
    ``workspace``: optional uint8 CUDA tensor of ``evo_trimul_workspace_size``
    bytes (allocated here when not given).  Runs on ``stream`` (default: the
    current stream) without synchronising."""
    if a.dim() != 4 or a.shape[1] != a.shape[2]:
        raise ValueError("a must be [Bt, N, N, C]")
    if tuple(b.shape) != tuple(a.shape):
        raise ValueError(f"b has shape {tuple(b.shape)}, expected {tuple(a.shape)}")
    if a.dtype not in (torch.bfloat16, torch.float16) or b.dtype != a.dtype:
        raise TypeError("a and b must both be bf16 or both fp16")
    if a.device.type != "cuda" or b.device != a.device:
        raise ValueError("a and b must be on one CUDA device")
    if not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("a and b must be contiguous")
    Bt, N, _, C = a.shape
    need = evo_trimul_workspace_size(Bt, N, C)
    if need < 0:
        raise EvoAttnError(need, "evo_trimul_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=a.device)
    if out is None:
        out = torch.empty_like(a)
    if stream is None:
        stream = torch.cuda.current_stream(a.device)
    status = evo_trimul(a.data_ptr(), b.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                        workspace.numel() * workspace.element_size(), Bt, N, C, 1 if outgoing else 0,
                        _DTYPES[a.dtype], stream.cuda_stream)
    if status != EVO_OK:
        raise EvoAttnError(status, "evo_trimul")
    return out
