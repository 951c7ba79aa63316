"""GPU parity of the decode-size kernels (M <= 256 tokens: tokens on the MMA's N
side, split-K clusters for the down-projection) against the CPU oracle.

Batches of at most 256 tokens are routed to these kernels by the library
(twell_up_pack when tile_w <= 128 and d_ff % 128 == 0; twell_spmm in the
tensor-core and automatic modes), so every case below runs them.  Cases cover
single-token and ragged batches, every tile width, the gated form, ell_w that is
not a multiple of 8 or above 32, heavy overflow, d_model that ends half-way into
a 128-column slice, and d_ff that ends inside a 64-column K step.
"""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import (assert_twell_equal, assert_y_close, dev, h_from_zdebug, host_bits,
                              twell_to_np, upload_twell)

GEMM_REL_BOUND = 2.0 ** -16

UP_CASES = [
    # M, d, f, tw, E, rho, gated
    (1, 256, 1024, 128, 16, 0.05, False),
    (5, 192, 512, 64, 8, 0.10, False),
    (16, 128, 256, 32, 8, 0.10, False),
    (33, 256, 1024, 128, 12, 0.20, False),     # E not a multiple of 8, overflow
    (100, 128, 512, 128, 40, 0.30, False),     # E > 32: two padding passes
    (256, 256, 2048, 128, 8, 0.15, False),     # largest decode batch, heavy overflow
    (7, 128, 512, 128, 16, 0.05, True),
    (64, 256, 512, 64, 8, 0.10, True),
    (250, 128, 256, 32, 8, 0.15, True),
    (40, 64, 256, 64, 64, 0.50, False),        # E == tile_w: no overflow possible
    (48, 128, 384, 64, 8, 1.0, False),         # every pair overflows
]


@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", UP_CASES)
def test_decode_up_pack_bitexact_given_accumulators(M, d, f, tw, E, rho, gated):
    L = S.small_random(M, d, f, tw, E, rho, gated=gated, seed=M * 31 + d + f)
    z = torch.zeros((M, 2 * f if gated else f), dtype=torch.float32, device="cuda")
    a = T.twell_up_pack(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_gate), tile_w=tw, ell_w=E,
                        ovf_capacity=M * (f // tw), z_debug=z)
    code, n = T.read_status(a)
    assert code == 0
    zg = z.cpu().numpy()
    h_gpu = h_from_zdebug(zg, L.b, gated, f)
    ref = O.twell_pack(h_gpu, tw, E)
    got, _ = twell_to_np(a)
    assert n == ref.n_ovf
    assert_twell_equal(got, ref)
    x = O.bits_to_f64(L.x)
    for name, w in (("gate", L.w_gate), ("up", L.w_up)) if gated else (("up", L.w_up),):
        W = O.bits_to_f64(w)
        bound = GEMM_REL_BOUND * (np.abs(x) @ np.abs(W).T) + 1e-30
        zz = zg[:, :f] if (not gated or name == "gate") else zg[:, f:]
        assert (np.abs(zz - x @ W.T) / bound).max() <= 1.0, name


DOWN_CASES = [
    # M, d, f, tw, E, rho
    (1, 256, 1024, 128, 16, 0.05),
    (17, 64, 512, 64, 8, 0.10),        # d_model = 64: half of one 128-column slice
    (64, 192, 1024, 128, 16, 0.10),    # second slice half outside d_model
    (200, 1024, 2048, 256, 24, 0.05),
    (256, 512, 1024, 128, 8, 0.30),    # heavy overflow
    (90, 256, 96, 32, 4, 0.10),        # d_ff = 96 ends inside a K step
    (120, 256, 512, 128, 5, 0.05),     # E not a multiple of 8
    (48, 128, 512, 64, 8, 1.0),        # every pair overflows
    (32, 4096, 2048, 128, 8, 0.02),    # 32 slices: split-K over 4-CTA clusters
]


@pytest.mark.parametrize("mode", ["mma", "auto"])
@pytest.mark.parametrize("M,d,f,tw,E,rho", DOWN_CASES)
def test_decode_spmm(M, d, f, tw, E, rho, mode):
    L = S.small_random(M, d, f, tw, E, rho, seed=M * 5 + d + 3 * f)
    h = O.hidden(L.x, L.w_up, L.b, L.w_gate)
    ref = O.twell_pack(h, tw, E)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y = T.twell_spmm(a, dev(L.w_down), mode=mode)
    assert T.read_status(a)[0] == 0
    assert_y_close(y, O.twell_spmm(ref, L.w_down))


def test_decode_spmm_zero_density_is_exact_zero():
    L = S.small_random(100, 512, 1024, 128, 16, 0.0)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), 128, 16)
    a = upload_twell(ref, cap=1)
    y = T.twell_spmm(a, dev(L.w_down), mode="mma")
    assert torch.count_nonzero(y.float()).item() == 0


@pytest.mark.parametrize("M", [1, 77, 256])
@pytest.mark.parametrize("gated", [False, True])
def test_decode_integer_family_forward_bitexact(M, gated):
    """Integer-valued layers: fp32 sums are exact in any order, so the fused
    decode forward (split-K partials included) must equal the oracle bitwise."""
    L = S.integer_exact(M=M, d_model=512, d_ff=2048, tile_w=128, density=0.05, gated=gated,
                        seed=M)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=L.tile_w,
                               ell_w=L.ell_w, W_gate=dev(L.w_gate), mode="auto",
                               ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))


def test_decode_and_gather_agree_on_the_same_twell():
    """The split-K kernel and the CUDA-core gather read the same TwELL; both are
    within tolerance of the oracle, and of each other."""
    L = S.small_random(128, 1024, 4096, 128, 16, 0.02, seed=11)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), 128, 16)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y_ref = O.twell_spmm(ref, L.w_down)
    y_mma = T.twell_spmm(a, dev(L.w_down), mode="mma")
    y_gat = T.twell_spmm(a, dev(L.w_down), mode="gather")
    assert_y_close(y_mma, y_ref)
    assert_y_close(y_gat, y_ref)


# Batches of at most 32 tokens take the touched-unit down kernel: a bitmap of
# the hidden units some token uses, compacted K, W_down rows gathered for those
# units only (or every row streamed when more than 3/4 of the units are touched).
TOUCHED_CASES = [
    # M, d, f, tw, E, rho
    (1, 256, 1024, 128, 16, 0.05),     # gather mode; most CTAs of a cluster get no K step
    (32, 4096, 2048, 128, 8, 0.02),    # gather mode over 32 column slices
    (2, 128, 4096, 128, 8, 0.20),      # every pair overflows: backup segments read by unit list
    (4, 128, 2048, 64, 5, 0.10),       # ell_w % 8 != 0: per-slot builder
    (3, 128, 1024, 32, 4, 0.05),       # tile_w 32
    (20, 128, 1024, 256, 24, 0.05),    # tile_w 256
    (17, 64, 512, 64, 8, 0.10),        # more than 3/4 touched: streaming inside the same kernel
    (32, 192, 1024, 128, 16, 0.01),    # largest batch of the kernel, a ragged column slice
    (64, 192, 1024, 128, 16, 0.01),    # above it: the streaming kernel
]


@pytest.mark.parametrize("M,d,f,tw,E,rho", TOUCHED_CASES)
def test_decode_touched_units_spmm(M, d, f, tw, E, rho):
    L = S.small_random(M, d, f, tw, E, rho, seed=M * 7 + f + tw)
    h = O.hidden(L.x, L.w_up, L.b, L.w_gate)
    ref = O.twell_pack(h, tw, E)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y = T.twell_spmm(a, dev(L.w_down), mode="mma")
    assert T.read_status(a)[0] == 0
    assert_y_close(y, O.twell_spmm(ref, L.w_down))


def test_decode_touched_zero_density_is_exact_zero():
    """No unit touched: compacted K is empty, every CTA stores a zero partial."""
    L = S.small_random(32, 512, 1024, 128, 16, 0.0)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), 128, 16)
    a = upload_twell(ref, cap=1)
    y = T.twell_spmm(a, dev(L.w_down), mode="mma")
    assert T.read_status(a)[0] == 0
    assert torch.count_nonzero(y.float()).item() == 0


def test_decode32_full_shape_integer_forward_bitexact():
    """The decode-size layer at its full shape (32 tokens, 4096 -> 16384, 2 %) on
    the integer-exact family: TwELL and every y bit through the touched-unit
    down kernel (about half of W_down's rows gathered)."""
    L = S.integer_exact(M=32, d_model=4096, d_ff=16384, tile_w=128, density=0.02, seed=32)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=128,
                               ell_w=L.ell_w, mode="auto", ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))


_CHILD = r"""
import sys, numpy as np
import activation_sparse_ffn_twell_b200 as T, oracle as O, twell_synth as S
sys.path.insert(0, 'tests')
from _gpu_helpers import dev, host_bits, upload_twell
out = {}
for i, (M, d, f, tw, E, rho) in enumerate(%r):
    L = S.small_random(M, d, f, tw, E, rho, seed=i + 3)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), tw, E)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y = T.twell_spmm(a, dev(L.w_down), mode="mma")
    assert T.read_status(a)[0] == 0
    out["y%%d" %% i] = host_bits(y)
np.savez(sys.argv[1], **out)
"""

FORCED_CASES = [(32, 256, 2048, 128, 8, 0.02), (128, 512, 2048, 128, 8, 0.005),
                (256, 256, 1024, 64, 8, 0.002), (8, 128, 1024, 128, 8, 0.05)]


@pytest.mark.parametrize("setting", ["0", "all"])
def test_decode_touched_switch(tmp_path, setting):
    """TWELL_DECODE_TOUCHED=0 keeps every batch on the streaming kernel, =all
    sends every decode-size batch whose stage ring allows it (gather mode where
    few units are touched) through the touched-unit kernel; y is within
    tolerance of the oracle either way."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = tmp_path / "y.npz"
    env = dict(os.environ, TWELL_DECODE_TOUCHED=setting, PYTHONPATH=root)
    subprocess.run([sys.executable, "-c", _CHILD % (FORCED_CASES,), str(out)], cwd=root, env=env,
                   check=True, timeout=600)
    got = np.load(out)
    for i, (M, d, f, tw, E, rho) in enumerate(FORCED_CASES):
        L = S.small_random(M, d, f, tw, E, rho, seed=i + 3)
        ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), tw, E)
        y = torch.from_numpy(got["y%d" % i].view(np.int16)).view(torch.bfloat16)
        assert_y_close(y, O.twell_spmm(ref, L.w_down))


@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", [
    (32, 256, 2048, 128, 8, 0.10, False),    # most pairs overflow: units found in backup segments
    (5, 192, 1024, 64, 8, 0.05, False),
    (24, 256, 1024, 128, 8, 0.10, True),
    (1, 128, 512, 128, 16, 0.0, False),      # no unit touched
])
def test_fused_decode_forward_touched_units(M, d, f, tw, E, rho, gated):
    """The fused decode forward up to 32 tokens (backup ordering in one kernel,
    then the bitmap pass and the touched-unit down kernel): y matches the oracle,
    including tokens whose hidden units appear only in backup segments, and a
    separate twell_spmm call on the same TwELL gives the same bits."""
    L = S.small_random(M, d, f, tw, E, rho, gated=gated, seed=M * 13 + f)
    y_ref = O.dense_ffn(L.x, L.w_up, L.b, L.w_down, L.w_gate)
    x, wu, b, wd, wg = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), dev(L.w_gate)
    y, a = T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=E, W_gate=wg, ovf_capacity=M * (f // tw))
    assert T.read_status(a)[0] == 0
    assert_y_close(y, y_ref)
    y2 = T.twell_spmm(a, wd)
    assert np.array_equal(host_bits(y), host_bits(y2))
