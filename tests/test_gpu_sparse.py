"""The 2:4 structured-sparse down path (twell_spmm mode "sparse", and AUTO where
it picks that path) against the oracle.

The path splits h per aligned group of 4 hidden units into the first two
nonzeros (run on the tensor cores' 2:4 sparse MMA) and the rest (added on CUDA
cores); y must equal h W_down exactly as the oracle defines it: bitwise on the
integer-exact family (every partial sum is an exact fp32 integer), within the
y tolerance on Gaussian layers.  Consumers are also fed TwELL matrices built
by the oracle packer from hand-shaped h (dense rows, heavy overflow, tokens
with many nonzeros per group of 4), so the backup compression and the
per-group fallback to the dense tensor-core path are exercised."""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import (assert_twell_equal, assert_twell_valid, assert_y_close, dev, host_bits,
                              twell_to_np, upload_twell)


INT_CASES = [
    # M, d_model, d_ff, tile_w, density, gated
    (512, 512, 2048, 128, 0.05, False),
    (300, 256, 1024, 128, 0.10, False),     # ragged token group
    (1024, 512, 4096, 64, 0.05, False),     # tile_w 64: two hidden tiles per operand stage
    (600, 384, 2048, 128, 0.05, True),      # gated; 384 columns: a ragged 256-column tile
    (777, 320, 3072, 128, 0.02, False),
]


@pytest.mark.parametrize("mode", ["sparse", "auto"])
@pytest.mark.parametrize("M,d,f,tw,rho,gated", INT_CASES)
def test_integer_family_bitexact(M, d, f, tw, rho, gated, mode):
    L = S.integer_exact(M=M, d_model=d, d_ff=f, tile_w=tw, density=rho, gated=gated, seed=M + d)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=tw, ell_w=L.ell_w,
                               W_gate=dev(L.w_gate), mode=mode, ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))


GAUSS_CASES = [
    (300, 256, 1024, 128, 16, 0.05, False),
    (520, 512, 2048, 128, 24, 0.10, False),
    (1000, 256, 2048, 64, 16, 0.10, False),
    (512, 256, 1024, 128, 16, 0.05, True),
    (400, 192, 1024, 128, 8, 0.01, False),     # 192 columns: one ragged tile
    (700, 1024, 4096, 128, 32, 0.20, False),
]


@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", GAUSS_CASES)
def test_gaussian_forward_sparse_mode(M, d, f, tw, E, rho, gated):
    L = S.small_random(M, d, f, tw, E, rho, gated=gated, seed=7 * M + d)
    y_ref = O.dense_ffn(L.x, L.w_up, L.b, L.w_down, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=tw, ell_w=E,
                               W_gate=dev(L.w_gate), mode="sparse", ovf_capacity=M * (f // tw))
    assert T.read_status(a)[0] == 0
    got, _ = twell_to_np(a)
    assert_twell_valid(got)
    assert_y_close(y, y_ref)


def _shaped_h(M, f, rho, rng, dense_rows=(), crowded_rows=(), crowd=3):
    """bf16-valued h [M, f]: each unit nonzero with probability rho; `dense_rows`
    fully nonzero; `crowded_rows` with `crowd` nonzeros in every group of 4."""
    mask = rng.random((M, f)) < rho
    for r in dense_rows:
        mask[r] = True
    for r in crowded_rows:
        m = np.zeros(f, dtype=bool)
        for g in range(f // 4):
            m[4 * g + rng.choice(4, size=crowd, replace=False)] = True
        mask[r] = m
    vals = rng.standard_normal((M, f))
    h = O.bf16_round(np.where(mask, vals, 0.0))
    return np.where(h == 0.0, 0.0, h)


@pytest.mark.parametrize("tw,E", [(128, 16), (128, 32), (64, 8)])
def test_consumer_mixed_groups_and_backup(tw, E):
    """TwELL from the oracle packer: group 0 ordinary (some overflowing pairs,
    whose backup segments are compressed in the operand build), group 1 with
    three tokens whose every group of 4 holds three nonzeros (more excess than
    the list holds: that group takes the dense tensor-core path), group 2 with
    dense tokens (overflow in every tile)."""
    rng = np.random.default_rng(tw + E)
    M, f, d = 700, 2048, 512
    h = _shaped_h(M, f, 0.06, rng, dense_rows=(600, 601), crowded_rows=(300, 301, 450))
    ref = O.twell_pack(h, tw, E)
    assert ref.n_ovf > 0
    wd = S.small_random(8, d, f, tw, E, 0.05, seed=3).w_down
    y_ref = h @ O.bits_to_f64(wd)
    a = upload_twell(ref)
    y = T.twell_spmm(a, dev(wd), mode="sparse")
    assert T.read_status(a)[0] == 0
    assert_y_close(y, y_ref)
    y2 = T.twell_spmm(a, dev(wd), mode="auto")
    assert_y_close(y2, y_ref)


def test_sparse_mode_is_deterministic():
    L = S.small_random(1100, 512, 4096, 128, 16, 0.05, seed=5)
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    ys = []
    for _ in range(3):
        y, a = T.twell_ffn_forward(x, wu, b, wd, tile_w=128, ell_w=16, mode="sparse")
        assert T.read_status(a)[0] == 0
        ys.append(host_bits(y))
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])


def test_full_shape_integer_layer_sparse_mode():
    """The 1.5B-shape layer (4096 x 2048 x 8192) on the integer-exact family:
    every y bit through the 2:4 path."""
    L = S.integer_exact(M=4096, d_model=2048, d_ff=8192, tile_w=128, density=0.05, seed=21)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=128, ell_w=L.ell_w,
                               mode="sparse", ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))
