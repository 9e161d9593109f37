"""The C-ABI library loads, exports what include/*.h declares, and rejects bad
arguments with the documented status codes before touching the GPU."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import build as evo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    evo_build.build()
    return evo.load_library()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"EVO_API\s+[\w\s\*]*?\b(evo_\w+)\s*\(", text))
    return names


def test_exports_match_header(lib):
    declared = declared_symbols()
    assert {"evo_attn_fwd", "evo_attn_sync_status", "evo_attn_strerror", "evo_attn_version"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", evo.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert declared <= exported, f"declared but not exported: {declared - exported}"
    for name in declared:
        assert hasattr(lib, name)


def test_strerror_and_version(lib):
    for code in range(-8, 1):
        s = evo.evo_attn_strerror(code)
        assert s and s != "unknown status"
    assert evo.evo_attn_strerror(-99) == "unknown status"
    assert evo.evo_attn_version() >= 100


def call(Q=0x10000, K=0x20000, V=0x30000, M=None, P=None, O=0x100000, L=0x200000,
         B=1, N=2, S=64, H=2, D=32, dtype=evo.EVO_DTYPE_BF16):
    return evo.evo_attn_fwd(Q, K, V, M, P, O, L, B, N, S, H, D, dtype, None)


def test_zero_sizes_are_noops(lib):
    for dims in ({"B": 0}, {"N": 0}, {"S": 0}, {"H": 0}):
        assert call(Q=None, K=None, V=None, O=None, L=None, **dims) == evo.EVO_OK


def test_invalid_arguments(lib):
    assert call(Q=None) == evo.EVO_ERR_INVALID_ARG
    assert call(L=None) == evo.EVO_ERR_INVALID_ARG
    assert call(B=-1) == evo.EVO_ERR_INVALID_ARG
    assert call(S=-5) == evo.EVO_ERR_INVALID_ARG
    assert call(dtype=7) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert call(dtype=3) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert call(dtype=evo.EVO_DTYPE_FP16) == call()         # fp16: the bf16 envelope
    assert call(D=0) == evo.EVO_ERR_UNSUPPORTED_SHAPE


def test_overlapping_outputs_rejected(lib):
    # O overlaps Q
    assert call(Q=0x100000, O=0x100000 + 64) == evo.EVO_ERR_INVALID_ARG
    # LSE inside the mask bias
    assert call(M=0x400000, L=0x400000) == evo.EVO_ERR_INVALID_ARG
    # O overlaps LSE
    assert call(L=0x100000 + 16) == evo.EVO_ERR_INVALID_ARG


def test_bf16_envelope(lib):
    # A call that passes every argument check reaches the device lookup, which
    # refuses these made-up pointers as not device memory: on a host without a
    # GPU that status marks an accepted shape.
    accepted = call()
    assert accepted == evo.EVO_ERR_INVALID_ARG
    # head dims 16, 32, 64 and 128 go to the tensor-core kernel (a pair bias
    # whose rows are not whole 16-byte units read element by element); other
    # head dims up to 128 go to the SIMT kernel
    for d in (1, 8, 24, 48, 64, 128):
        assert call(D=d) == accepted
    assert call(S=60, P=0x800000) == accepted
    for d in (129, 256):
        assert call(D=d) == evo.EVO_ERR_UNSUPPORTED_SHAPE
    # the SIMT shapes need 2-byte alignment only
    assert call(D=48, Q=0x10008, O=0x100002) == accepted
    assert call(S=60, P=0x800002) == accepted
    assert call(D=48, Q=0x10001) == evo.EVO_ERR_MISALIGNED
    # the tensor-core shapes keep the 16-byte rule
    assert call(Q=0x10008) == evo.EVO_ERR_MISALIGNED
    assert call(D=128, Q=0x10008) == evo.EVO_ERR_MISALIGNED
    assert call(O=0x100002) == evo.EVO_ERR_MISALIGNED
    assert call(P=0x800008) == evo.EVO_ERR_MISALIGNED
    assert call(M=0x900001) == evo.EVO_ERR_MISALIGNED
    assert call(L=0x200002) == evo.EVO_ERR_MISALIGNED
    far = dict(Q=1 << 50, K=2 << 50, V=3 << 50, O=4 << 50, L=5 << 50)
    # tile count = query blocks x heads x n groups (3 slices at D = 16) x batch
    # beyond 2^31 - 1
    assert call(B=1 << 16, N=1 << 10, S=1 << 10, H=1 << 4, D=16, **far) == evo.EVO_ERR_UNSUPPORTED_SHAPE


def test_fp32_envelope(lib):
    f = evo.EVO_DTYPE_FP32
    assert call(D=129, dtype=f) == evo.EVO_ERR_UNSUPPORTED_SHAPE
    assert call(Q=0x10002, dtype=f) == evo.EVO_ERR_MISALIGNED
    assert call(M=0x900002, dtype=f) == evo.EVO_ERR_MISALIGNED


def test_size_overflow_rejected(lib):
    assert call(B=1 << 40, N=1 << 40) == evo.EVO_ERR_UNSUPPORTED_SHAPE


def test_python_wrapper_validates_before_calling():
    import torch
    q = torch.zeros(1, 2, 8, 1, 16)
    with pytest.raises(ValueError):
        evo.evo_attn(q, q, q)          # CPU tensors are refused
    with pytest.raises(ValueError):
        evo.evo_attn(q, q[:, :1], q)   # shape mismatch
    with pytest.raises(TypeError):
        evo.evo_attn(q.double(), q.double(), q.double())


def test_host_wrapper_validates_before_calling():
    import torch
    q = torch.zeros(1, 2, 8, 1, 16)
    with pytest.raises(ValueError, match="page-locked"):
        evo.evo_attn_from_host(q, q, q)           # pageable host tensors are refused
    with pytest.raises(ValueError):
        evo.evo_attn_from_host(q, q[:, :1], q)    # shape mismatch
    with pytest.raises(TypeError):
        evo.evo_attn_from_host(q.double(), q.double(), q.double())


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(evo, "_lib", None)
    monkeypatch.setattr(evo, "_LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        evo.load_library()


def test_selftest_timeout_rejects_bad_arguments(lib):
    assert evo.evo_attn_selftest_timeout(0, 0x1000, None) == evo.EVO_ERR_INVALID_ARG
    assert evo.evo_attn_selftest_timeout(2 * 10**9, 0x1000, None) == evo.EVO_ERR_INVALID_ARG
    assert evo.evo_attn_selftest_timeout(10**6, None, None) == evo.EVO_ERR_INVALID_ARG


def call_host(M=None, P=None, Md=None, Pd=None, chunk_n=0, **kw):
    """evo_attn_fwd_host with made-up host (0x1...) and device (0x9...) addresses."""
    d = dict(B=1, N=2, S=64, H=2, D=32, dtype=evo.EVO_DTYPE_BF16)
    d.update(kw)
    return evo.evo_attn_fwd_host(0x1000000, 0x2000000, 0x3000000, M, P, 0x4000000, 0x5000000,
                                 0x91000000, 0x92000000, 0x93000000, Md, Pd, 0x94000000, 0x95000000,
                                 d["B"], d["N"], d["S"], d["H"], d["D"], d["dtype"], chunk_n, None)


def test_host_entry_checks_arguments(lib):
    assert call_host(B=0) == evo.EVO_OK                       # nothing to do
    assert call_host(chunk_n=-1) == evo.EVO_ERR_INVALID_ARG
    assert call_host(M=0x6000000) == evo.EVO_ERR_INVALID_ARG   # host mask without a device mask
    assert call_host(Pd=0x96000000) == evo.EVO_ERR_INVALID_ARG  # device pair without a host pair
    assert call_host(D=256) == evo.EVO_ERR_UNSUPPORTED_SHAPE   # the device buffers get evo_attn_fwd's checks
    assert call_host(dtype=7) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    # made-up host addresses are not page-locked memory
    assert call_host() == evo.EVO_ERR_INVALID_ARG


def call_bwd(M=None, P=None, dM=None, dP=None, W=0x10000000, Wbytes=None, **kw):
    """evo_attn_bwd with made-up device addresses (far apart, so nothing overlaps)."""
    d = dict(B=1, N=2, S=64, H=2, D=32, dtype=evo.EVO_DTYPE_BF16)
    d.update(kw)
    if Wbytes is None:
        Wbytes = max(evo.evo_attn_bwd_workspace_size(d["B"], d["N"], d["S"], d["H"], d["D"]), 0)
    a = [0x1000000 * (i + 1) for i in range(9)]  # Q K V O LSE dO dQ dK dV
    for key in ("Q", "K", "V", "O", "L", "dO", "dQ", "dK", "dV"):
        if key in kw:
            a["Q K V O L dO dQ dK dV".split().index(key)] = kw.pop(key)
    return evo.evo_attn_bwd(a[0], a[1], a[2], M, P, a[3], a[4], a[5], a[6], a[7], a[8], dM, dP, W, Wbytes,
                            d["B"], d["N"], d["S"], d["H"], d["D"], d["dtype"], None)


def test_bwd_workspace_size(lib):
    B, N, S, H, D = 1, 2, 64, 2, 32
    size = evo.evo_attn_bwd_workspace_size(B, N, S, H, D)
    r = lambda b: (b + 255) // 256 * 256
    expect = (r(4 * B * N) + 2 * r(4 * B * N * H * S) + r(4 * B * N * S * H * D) + r(4 * B * N * S)
              + r(4 * B * H * S * S) + r(4 * (B * N + 1)))
    assert size == expect
    assert evo.evo_attn_bwd_workspace_size(-1, N, S, H, D) == evo.EVO_ERR_INVALID_ARG
    assert evo.evo_attn_bwd_workspace_size(1 << 40, 1 << 40, S, H, D) == evo.EVO_ERR_UNSUPPORTED_SHAPE


def test_bwd_checks_arguments(lib):
    accepted = call_bwd()          # passes every check, then the made-up pointers are refused
    assert accepted == evo.EVO_ERR_INVALID_ARG
    # (a rejected argument gives another status, or the same one earlier:
    # overlap tests below use addresses that pass every other check)
    assert call_bwd(W=0x10000010) != accepted
    assert call_bwd(B=0, W=None, Wbytes=0) == evo.EVO_OK
    assert call_bwd(dtype=9) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert call_bwd(D=129) == evo.EVO_ERR_UNSUPPORTED_SHAPE
    assert call_bwd(D=0) == evo.EVO_ERR_UNSUPPORTED_SHAPE
    assert call_bwd(W=None) == evo.EVO_ERR_INVALID_ARG
    # a workspace one byte short, or not on a 256-byte boundary
    full = evo.evo_attn_bwd_workspace_size(1, 2, 64, 2, 32)
    assert call_bwd(Wbytes=full - 1) == evo.EVO_ERR_INVALID_ARG
    assert call_bwd(W=0x10000010) == evo.EVO_ERR_MISALIGNED
    # a bias gradient needs its bias
    assert call_bwd(dM=0xA000000) == evo.EVO_ERR_INVALID_ARG
    assert call_bwd(dP=0xB000000) == evo.EVO_ERR_INVALID_ARG
    assert call_bwd(M=0xC000000, dM=0xA000000, P=0xD000000, dP=0xB000000) == accepted
    # outputs must not overlap inputs, each other or the workspace
    assert call_bwd(dQ=0x1000000 + 64) == evo.EVO_ERR_INVALID_ARG         # dQ inside Q
    assert call_bwd(dK=0x7000000 + 2) == evo.EVO_ERR_INVALID_ARG          # dK inside dQ
    assert call_bwd(W=0x9000000 - 256) == evo.EVO_ERR_INVALID_ARG         # workspace runs into dV
    # alignment to the element size
    assert call_bwd(dV=0x9000001) == evo.EVO_ERR_MISALIGNED
    assert call_bwd(L=0x5000002) == evo.EVO_ERR_MISALIGNED
    assert call_bwd(dtype=evo.EVO_DTYPE_FP32, dO=0x6000002) == evo.EVO_ERR_MISALIGNED
    assert call_bwd(D=48) == accepted and call_bwd(dtype=evo.EVO_DTYPE_FP32) == accepted


def test_backward_wrapper_validates_before_calling():
    import torch
    q = torch.zeros(1, 2, 8, 1, 16)
    lse = torch.zeros(1, 2, 1, 8)
    with pytest.raises(ValueError):
        evo.evo_attn_backward(q, q, q, None, None, q, lse, q)        # CPU tensors are refused
    with pytest.raises(ValueError, match="without a mask"):
        evo.evo_attn_backward(q, q, q, None, None, q, lse, q, need_dmask=True)
    with pytest.raises(TypeError):
        evo.evo_attn_backward(q, q, q, None, None, q, lse.double(), q)


def test_trimul_checks_arguments(lib):
    size = evo.evo_trimul_workspace_size(1, 37, 3)
    assert size == 3 * ((2 * 1 * 3 * 37 * 40 + 255) // 256 * 256)      # rows padded to 40
    assert evo.evo_trimul_workspace_size(-1, 4, 4) == evo.EVO_ERR_INVALID_ARG
    call = lambda **kw: evo.evo_trimul(kw.get("A", 0x1000000), kw.get("B", 0x2000000), kw.get("Z", 0x3000000),
                                       kw.get("W", 0x4000000), kw.get("Wb", 1 << 20), kw.get("Bt", 1),
                                       kw.get("N", 16), kw.get("C", 4), kw.get("out", 1),
                                       kw.get("dt", evo.EVO_DTYPE_BF16), None)
    assert call(Bt=0, A=None) == evo.EVO_OK
    assert call(dt=evo.EVO_DTYPE_FP32) == evo.EVO_ERR_UNSUPPORTED_DTYPE
    assert call(out=2) == evo.EVO_ERR_INVALID_ARG
    assert call(A=None) == evo.EVO_ERR_INVALID_ARG
    assert call(Wb=16) == evo.EVO_ERR_INVALID_ARG                       # workspace too small
    assert call(W=0x4000010) == evo.EVO_ERR_MISALIGNED
    assert call(A=0x1000001) == evo.EVO_ERR_MISALIGNED
    assert call(Z=0x1000000 + 64) == evo.EVO_ERR_INVALID_ARG            # Z over A
