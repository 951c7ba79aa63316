"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Contract (each piece is tested below):
  (i)   twell_pack on a given h equals the oracle packer bitwise.
  (ii)  the fused producer's TwELL equals the oracle packer applied to h rebuilt
        from the GPU's own fp32 accumulators (z_debug), bitwise.
  (iii) the GPU accumulators are within the stated bound of the fp64 products.
  (iv)  integer-exact layers: TwELL and y equal the oracle bitwise.
  (v)   y is within rel-L2 2e-3 and max-abs 3e-2 of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import (assert_twell_equal, assert_twell_valid, assert_y_close, dev,
                              h_from_zdebug, twell_to_np, upload_twell, y_errors)

# accumulator bound: |z_gpu - z_fp64| <= 2^-16 * (sum_k |x_k W_jk| + |b_j|)
GEMM_REL_BOUND = 2.0 ** -16


def _layer(M, d, f, tw, E, rho, gated=False, seed=0):
    return S.small_random(M, d, f, tw, E, rho, gated=gated, seed=seed)


def _ref_h(L):
    return O.hidden(L.x, L.w_up, L.b, L.w_gate)


# ---------------------------------------------------------------- (i) packing
PACK_CASES = [
    # M, f, tw, E, rho
    (37, 256, 32, 4, 0.10),
    (300, 1024, 64, 16, 0.10),
    (300, 2048, 128, 16, 0.05),
    (129, 1024, 128, 40, 0.20),
    (70, 1024, 256, 24, 0.05),
    (257, 1024, 128, 8, 0.30),     # heavy overflow
    (100, 512, 128, 5, 0.05),      # ell_w not a multiple of 8
    (64, 512, 128, 128, 0.50),     # ell_w == tile_w: plain per-tile ELL
    (50, 512, 64, 8, 0.0),         # empty
]


@pytest.mark.parametrize("M,f,tw,E,rho", PACK_CASES)
def test_pack_bitexact(M, f, tw, E, rho):
    L = _layer(M, 64, f, tw, E, rho, seed=M + f)
    h = _ref_h(L)
    ref = O.twell_pack(h, tw, E)
    a = T.twell_pack(dev(O.f64_to_bits(h)), tw, E, ovf_capacity=max(ref.n_ovf, 1))
    code, n = T.read_status(a)
    assert code == 0 and n == ref.n_ovf
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)


def test_pack_full_density_and_strided_input():
    L = _layer(96, 64, 512, 64, 8, 1.0, seed=3)
    h = _ref_h(L)
    ref = O.twell_pack(h, 64, 8)
    wide = torch.zeros((96, 512 + 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :512] = dev(O.f64_to_bits(h))
    # a column slice is not contiguous: go through the C ABI with ld_h directly
    a = T.TwELL.allocate(96, 512, 64, 8, 96 * 8)
    nb = T.workspace_bytes(96, 64, 512, 64, 8, 0, a.ovf_capacity)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    import ctypes
    m = a.cstruct()
    code = T.lib().twell_pack(wide.data_ptr(), 96, 512, 576, 64, 8, ctypes.byref(m), ws.data_ptr(),
                              nb, torch.cuda.current_stream().cuda_stream)
    assert code == 0
    assert T.read_status(a) == (0, ref.n_ovf)
    assert ref.n_ovf == 96 * 8
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)


def test_pack_capacity_exhausted_is_reported():
    L = _layer(128, 64, 1024, 128, 8, 0.3, seed=9)
    h = _ref_h(L)
    ref = O.twell_pack(h, 128, 8)
    assert ref.n_ovf > 10
    a = T.twell_pack(dev(O.f64_to_bits(h)), 128, 8, ovf_capacity=5)
    code, n = T.read_status(a)
    assert code == 3 and n == ref.n_ovf
    got, _ = twell_to_np(a)
    assert np.array_equal(got.nnz, ref.nnz) and np.array_equal(got.vals, ref.vals)


def test_empty_batch_is_noop():
    a = T.TwELL.allocate(0, 1024, 128, 16, 0)
    h = torch.empty((0, 1024), dtype=torch.bfloat16, device="cuda")
    T.twell_pack(h, 128, 16, out=a)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1024, 256), dtype=torch.bfloat16, device="cuda")
    y, _ = T.twell_ffn_forward(x, w, None, w, tile_w=128, ell_w=16)
    assert y.shape == (0, 256)


# ---------------------------------------------------------------- (v) spmm
SPMM_CASES = [
    # M, d, f, tw, E, rho
    (37, 64, 256, 32, 4, 0.10),
    (300, 256, 1024, 64, 16, 0.10),
    (300, 320, 2048, 128, 16, 0.05),   # d not a multiple of 256
    (257, 512, 1024, 128, 8, 0.30),    # heavy overflow
    (130, 2048, 1024, 256, 24, 0.05),
    (200, 256, 512, 128, 5, 0.05),     # ell_w not a multiple of 8
    (96, 128, 512, 64, 8, 1.0),        # every pair overflows
    # more than 256 tokens: the token-major tensor-core kernel (fewer go to the
    # split-K decode kernel)
    (300, 256, 512, 128, 5, 0.05),     # ell_w not a multiple of 8
    (290, 128, 512, 64, 8, 1.0),       # every pair overflows
    (260, 1024, 1024, 32, 8, 0.10),
]


@pytest.mark.parametrize("mode", ["gather", "mma", "auto"])
@pytest.mark.parametrize("M,d,f,tw,E,rho", SPMM_CASES)
def test_spmm_modes(M, d, f, tw, E, rho, mode):
    L = _layer(M, d, f, tw, E, rho, seed=M * 7 + d)
    h = _ref_h(L)
    ref = O.twell_pack(h, tw, E)
    y_ref = O.twell_spmm(ref, L.w_down)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y = T.twell_spmm(a, dev(L.w_down), mode=mode)
    assert T.read_status(a)[0] == 0
    assert_y_close(y, y_ref)


@pytest.mark.parametrize("mode", ["gather", "mma"])
def test_spmm_zero_density_is_exact_zero(mode):
    L = _layer(150, 256, 1024, 128, 16, 0.0)
    ref = O.twell_pack(_ref_h(L), 128, 16)
    a = upload_twell(ref, cap=1)
    y = T.twell_spmm(a, dev(L.w_down), mode=mode)
    assert torch.count_nonzero(y.float()).item() == 0


# ---------------------------------------------------------------- (ii)/(iii) fused producer
UP_CASES = [
    # M, d, f, tw, E, rho, gated
    (200, 256, 1024, 128, 16, 0.05, False),
    (130, 192, 384, 128, 16, 0.10, False),     # f not a multiple of 256, ragged M
    (64, 256, 1024, 64, 16, 0.10, False),
    (100, 128, 512, 32, 8, 0.10, False),
    (90, 256, 1024, 256, 24, 0.05, False),
    (257, 128, 512, 128, 12, 0.20, False),     # E not a multiple of 8, overflow
    (200, 256, 1024, 128, 16, 0.05, True),
    (150, 128, 512, 64, 8, 0.10, True),
    (70, 128, 256, 32, 8, 0.15, True),
    # more than 256 tokens: the token-major producer (fewer go to the decode kernel)
    (300, 256, 1024, 128, 16, 0.05, False),
    (333, 128, 512, 32, 8, 0.10, False),
    (390, 128, 512, 64, 8, 0.10, True),
    (280, 128, 512, 128, 12, 0.20, True),
]


@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", UP_CASES)
def test_up_pack_epilogue_bitexact_and_gemm_bound(M, d, f, tw, E, rho, gated):
    L = _layer(M, d, f, tw, E, rho, gated=gated, seed=M + 13 * d)
    zcols = 2 * f if gated else f
    z = torch.zeros((M, zcols), dtype=torch.float32, device="cuda")
    a = T.twell_up_pack(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_gate), tile_w=tw, ell_w=E,
                        ovf_capacity=M * (f // tw), z_debug=z)
    code, n = T.read_status(a)
    assert code == 0
    zg = z.cpu().numpy()
    # (ii) epilogue exactness given the GPU's own accumulators
    h_gpu = h_from_zdebug(zg, L.b, gated, f)
    ref = O.twell_pack(h_gpu, tw, E)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    # (iii) accumulators against fp64 products
    x = O.bits_to_f64(L.x)
    for name, w in (("gate", L.w_gate), ("up", L.w_up)) if gated else (("up", L.w_up),):
        W = O.bits_to_f64(w)
        z64 = x @ W.T
        bound = GEMM_REL_BOUND * (np.abs(x) @ np.abs(W).T) + 1e-30
        zz = zg[:, :f] if (not gated or name == "gate") else zg[:, f:]
        ratio = np.abs(zz - z64) / bound
        assert ratio.max() <= 1.0, f"{name}: max |dz|/bound = {ratio.max():.3f}"
    # the GPU h differs from the oracle's only where fp32 vs fp64 rounding can flip it
    h64 = _ref_h(L)
    frac = np.mean(h_gpu != h64)
    assert frac < 2e-3, frac


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("mode", ["gather", "mma"])
def test_integer_family_forward_bitexact(gated, mode):
    L = S.integer_exact(M=300, d_model=512, d_ff=2048, tile_w=128, density=0.05, gated=gated)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=L.tile_w,
                               ell_w=L.ell_w, W_gate=dev(L.w_gate), mode=mode,
                               ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    y_bits = O.f64_to_bits(O.bf16_round(y64))
    from _gpu_helpers import host_bits
    assert np.array_equal(host_bits(y), y_bits)


# ---------------------------------------------------------------- (v) whole layer
FWD_CASES = [
    (300, 256, 1024, 128, 16, 0.05, False),
    (200, 512, 2048, 128, 24, 0.10, False),
    (129, 256, 1024, 64, 16, 0.10, False),
    (256, 256, 1024, 128, 16, 0.05, True),
    (100, 128, 512, 128, 8, 0.01, False),
]


@pytest.mark.parametrize("mode", ["gather", "mma", "auto"])
@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", FWD_CASES)
def test_forward_against_oracle(M, d, f, tw, E, rho, gated, mode):
    L = _layer(M, d, f, tw, E, rho, gated=gated, seed=5 * M + d)
    y_ref = O.dense_ffn(L.x, L.w_up, L.b, L.w_down, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=tw,
                               ell_w=E, W_gate=dev(L.w_gate), mode=mode,
                               ovf_capacity=M * (f // tw))
    assert T.read_status(a)[0] == 0
    got, _ = twell_to_np(a)
    assert_twell_valid(got)
    assert_y_close(y, y_ref)


def test_tiny_config_full():
    L = S.tiny_relu(0)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=L.tile_w,
                               ell_w=L.ell_w, ovf_capacity=L.M * L.n_tiles)
    assert T.read_status(a)[0] == 0
    got, _ = twell_to_np(a)
    assert_twell_valid(got)
    assert np.mean(got.nnz != ref.nnz) < 0.01
    assert_y_close(y, y64)
