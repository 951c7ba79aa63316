"""The C-ABI library loads, exports every function include/twell.h declares, and
rejects bad arguments on the host before touching the GPU.  No compute runs here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twell.h")


@pytest.fixture(scope="module")
def L():
    from activation_sparse_ffn_twell_b200 import build
    build.build()
    import activation_sparse_ffn_twell_b200 as T
    return T.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(twell_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_three_calls():
    names = _declared()
    for n in ("twell_pack", "twell_spmm", "twell_ffn_forward", "twell_up_pack",
              "twell_up_pack_stats", "twell_pack_noalloc",
              "twell_workspace_bytes", "twell_read_status", "twell_status_string", "twell_version"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    from activation_sparse_ffn_twell_b200 import library_path
    out = subprocess.run(["nm", "-D", "--defined-only", library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\S+)$", out, flags=re.M))
    for n in _declared():
        assert n in exported, n
        assert hasattr(L, n)


def test_library_has_no_cuda_runtime_dependency(L):
    from activation_sparse_ffn_twell_b200 import library_path
    deps = subprocess.run(["ldd", library_path()], capture_output=True, text=True).stdout
    assert "libcudart" not in deps and "libcuda.so" not in deps


def test_version_and_status_strings(L):
    assert L.twell_version() >= 100
    assert L.twell_status_string(0) == b"ok"
    assert b"capacity" in L.twell_status_string(3)
    assert L.twell_status_string(99) == b"unknown status"


def test_workspace_bytes_rules(L):
    ok = L.twell_workspace_bytes(4096, 2048, 8192, 128, 16, 0, 4096)
    assert ok > 0
    assert L.twell_workspace_bytes(4096, 2048, 8192, 96, 16, 0, 4096) == 0      # tile_w
    assert L.twell_workspace_bytes(4096, 2048, 8000, 128, 16, 0, 4096) == 0     # d_ff % tile_w
    assert L.twell_workspace_bytes(4096, 2000, 8192, 128, 16, 0, 4096) == 0     # d_model % 64
    assert L.twell_workspace_bytes(4096, 2048, 8192, 128, 0, 0, 4096) == 0      # ell_w < 1
    assert L.twell_workspace_bytes(4096, 2048, 8192, 128, 129, 0, 4096) == 0    # ell_w > tile_w
    assert L.twell_workspace_bytes(4096, 2048, 8192, 128, 16, 0, -1) == 0       # capacity
    bigger = L.twell_workspace_bytes(4096, 2048, 8192, 128, 16, 0, 8192)
    assert bigger >= ok + 4096 * (128 * 2 + 4)
    # the tensor-core down kernel's split schedules (M > 256 tokens, d_model > 256):
    # 160 arrival counters and 2 x 160 fp32 partial tiles of 128 x 512
    split = 2 * 160 * 128 * 512 * 4
    narrow = L.twell_workspace_bytes(4096, 256, 8192, 128, 16, 0, 4096)
    assert ok - narrow >= split
    small_m = L.twell_workspace_bytes(256, 2048, 8192, 128, 16, 0, 4096)
    assert small_m < split                      # decode-size batches use their own kernel


def _matrix(M=256, f=1024, tw=128, E=16, cap=64, base=0x10000):
    import activation_sparse_ffn_twell_b200 as T
    p = lambda k: base + 0x100000 * k
    return T._Matrix(M, f, tw, E, p(1), p(2), p(3), cap, p(4), p(5), p(6), p(7))


def test_argument_errors_are_synchronous(L):
    import activation_sparse_ffn_twell_b200 as T
    m = _matrix()
    ws, wsb = 0x9000000, 1 << 30
    h = 0x8000000
    bp = ctypes.byref
    assert L.twell_pack(None, 256, 1024, 1024, 128, 16, bp(m), ws, wsb, None) == 1
    assert L.twell_pack(h + 2, 256, 1024, 1024, 128, 16, bp(m), ws, wsb, None) == 1   # misaligned
    assert L.twell_pack(h, 256, 1024, 1000, 128, 16, bp(m), ws, wsb, None) == 1       # ld_h < d_ff
    assert L.twell_pack(h, 256, 1024, 1024, 100, 16, bp(m), ws, wsb, None) == 1       # tile_w
    assert L.twell_pack(h, 256, 1024, 1024, 128, 16, None, ws, wsb, None) == 1        # no matrix
    m2 = _matrix(M=128)
    assert L.twell_pack(h, 256, 1024, 1024, 128, 16, bp(m2), ws, wsb, None) == 1      # M mismatch
    assert L.twell_pack(h, 256, 1024, 1024, 128, 16, bp(m), None, wsb, None) == 6     # no workspace
    assert L.twell_pack(h, 256, 1024, 1024, 128, 16, bp(m), ws, 100, None) == 6       # too small
    # fused path limits
    x, w = 0x7000000, 0x6000000
    m3 = _matrix(E=72)
    assert L.twell_up_pack(x, w, None, None, 256, 256, 1024, 128, 72, bp(m3), None, ws, wsb, None) == 2
    m4 = _matrix(tw=256, E=16)
    assert L.twell_up_pack(x, w, w, None, 256, 256, 1024, 256, 16, bp(m4), None, ws, wsb, None) == 2
    assert L.twell_up_pack(x, w, None, None, 256, 100, 1024, 128, 16, bp(m), None, ws, wsb, None) == 1
    # statistics variant: same validation, plus its two output pointers
    assert L.twell_up_pack_stats(x, w, None, None, 256, 256, 1024, 128, 72, bp(m3), None, None, ws,
                                 wsb, None) == 2
    assert L.twell_up_pack_stats(x, w, None, None, 256, 256, 1024, 128, 16, bp(m), 0x5000004, None,
                                 ws, wsb, None) == 1                                    # misaligned l1
    assert L.twell_up_pack_stats(x, w, None, None, 256, 256, 1024, 128, 16, bp(m), None, None, ws,
                                 100, None) == 6                                        # workspace
    # backward: shape limits and workspace query
    assert L.twell_backward_workspace_bytes(200, 256, 1024, 128, 16, 100, 16, 100) == 0   # M % 128
    assert L.twell_backward_workspace_bytes(256, 256, 1024, 256, 16, 100, 16, 100) == 0   # tile_w
    assert L.twell_backward_workspace_bytes(256, 256, 1024, 128, 16, 100, 16, 100) > 0
    assert L.twell_ffn_backward(x, w, w, None, x, 256, 16, 100, x, x, x, x, ws, wsb, None) == 1
    # spmm
    assert L.twell_spmm(bp(m), None, 256, 0x5000000, 0, ws, wsb, None) == 1
    assert L.twell_spmm(bp(m), w, 256, 0x5000000, 7, ws, wsb, None) == 1               # mode
    assert L.twell_spmm(bp(m), w, 250, 0x5000000, 0, ws, wsb, None) == 1               # d_model
    assert L.twell_ffn_forward(x, w, None, None, w, 256, 256, 1024, 128, 16, bp(m), None, 0, ws,
                               wsb, None) == 1                                          # y missing
    # M == 0 is a no-op that touches nothing
    m0 = _matrix(M=0)
    assert L.twell_pack(h, 0, 1024, 1024, 128, 16, bp(m0), ws, wsb, None) == 0


def test_no_gpu_means_cuda_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("only meaningful where no GPU is present")
    m = _matrix()
    h = 0x8000000
    r = L.twell_pack(h, 256, 1024, 1024, 128, 16, ctypes.byref(m), 0x9000000, 1 << 30, None)
    assert r == 4


def test_pack_noalloc_argument_rules_match_pack(L):
    """twell_pack_noalloc shares twell_pack's validators: the same inputs are
    rejected on the host with the same status, before any launch."""
    import activation_sparse_ffn_twell_b200 as T
    bp = ctypes.byref
    ws, wsb = 0x9000000, 1 << 30
    h = 0x8000000

    def both(hh, M, f, ld, tw, E, m):
        a = L.twell_pack(hh, M, f, ld, tw, E, m, ws, wsb, None)
        b = L.twell_pack_noalloc(hh, M, f, ld, tw, E, m, None)
        assert a == b, (a, b)
        return b

    m = _matrix()
    assert both(h + 2, 256, 1024, 1024, 128, 16, bp(m)) == 1              # misaligned h
    assert both(h, 256, 1024, 1000, 128, 16, bp(m)) == 1                  # ld_h < d_ff
    assert both(h, 256, 1024, 1024, 100, 16, bp(m)) == 1                  # tile_w
    assert both(h, 256, 1024, 1024, 128, 16, None) == 1                   # no matrix
    assert both(h, 256, 1024, 1024, 128, 16, bp(_matrix(M=128))) == 1    # M mismatch
    # a misaligned device status word or overflow counter would be written by
    # the kernels as int32: both entry points reject it
    for field in ("n_ovf", "status"):
        bad = _matrix()
        setattr(bad, field, getattr(bad, field) + 2)
        assert both(h, 256, 1024, 1024, 128, 16, bp(bad)) == 1
    # M == 0 is a no-op for both, even without a destination
    assert both(h, 0, 1024, 1024, 128, 16, None) == 0
    assert both(None, 0, 1024, 1024, 128, 16, bp(_matrix(M=0))) == 0
