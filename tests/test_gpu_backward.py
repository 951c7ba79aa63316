"""GPU parity of the backward pass through the hybrid sparse form
(twell_ffn_backward) against the CPU oracle.

* Integer-exact layers (x, weights, dY in {-1, 0, +1}, integer bias): every
  product and partial sum is an integer, so dX, dW_up, dW_down (bf16) and db
  (fp32) must equal the oracle bitwise.
* Gaussian layers: within rel-L2 2e-3 of the fp64 oracle evaluated on the GPU's
  own forward activations (so both sides use the same sparsity pattern).
Cases cover the decode-size dX path (M = 256) and the token-major one, every
tile width the backward supports, overflowing forward pairs, and overflowing
transposed pairs (a small ell_w_t).
"""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import dev, host_bits, twell_to_np


def _rel_l2(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    n = np.linalg.norm(ref)
    return np.linalg.norm(g - ref) / n if n > 0 else float(np.abs(g).max())


INT_CASES = [
    # M, d, f, tw, density, ell_w_t
    (256, 256, 1024, 128, 0.05, 16),
    (384, 128, 512, 64, 0.10, 16),
    (256, 128, 512, 32, 0.20, 8),      # overflowing transposed pairs
]


@pytest.mark.parametrize("M,d,f,tw,rho,et", INT_CASES)
def test_backward_integer_family_bitexact(M, d, f, tw, rho, et):
    L = S.integer_exact(M=M, d_model=d, d_ff=f, tile_w=tw, density=rho, seed=M + f)
    dy = S.integer_exact(M=M, d_model=d, d_ff=f, tile_w=tw, density=rho, seed=M + f + 1).x
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    y, h = T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=L.ell_w, ovf_capacity=M * (f // tw))
    assert T.read_status(h)[0] == 0
    dX, dWu, db, dWd = T.twell_ffn_backward(x, wu, wd, h, dev(dy), ell_w_t=et)
    assert T.read_status(h)[0] == 0
    g = O.ffn_backward(L.x, L.w_up, L.b, L.w_down, dy)
    assert np.array_equal(host_bits(dX), O.f64_to_bits(O.bf16_round(g["dx"])))
    assert np.array_equal(host_bits(dWu), O.f64_to_bits(O.bf16_round(g["dw_up"])))
    assert np.array_equal(host_bits(dWd), O.f64_to_bits(O.bf16_round(g["dw_down"])))
    assert np.array_equal(db.cpu().numpy().astype(np.float64), g["db"])


GAUSS_CASES = [
    # M, d, f, tw, E, rho
    (256, 256, 1024, 128, 16, 0.05),
    (512, 256, 1024, 128, 16, 0.05),
    (384, 128, 512, 64, 8, 0.20),      # overflowing forward pairs
    (256, 192, 384, 32, 8, 0.10),
]


@pytest.mark.parametrize("M,d,f,tw,E,rho", GAUSS_CASES)
def test_backward_gaussian_within_tolerance(M, d, f, tw, E, rho):
    L = S.small_random(M, d, f, tw, E, rho, seed=M * 7 + f)
    rng = np.random.default_rng(M)
    dy = S.bf16_bits_from_f32(rng.standard_normal((M, d)).astype(np.float32))
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    y, h = T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=E, ovf_capacity=M * (f // tw))
    assert T.read_status(h)[0] == 0
    dX, dWu, db, dWd = T.twell_ffn_backward(x, wu, wd, h, dev(dy))
    assert T.read_status(h)[0] == 0
    got, _ = twell_to_np(h)
    g = O.ffn_backward(L.x, L.w_up, L.b, L.w_down, dy, h=O.twell_unpack(got))
    for name, t in (("dx", dX), ("dw_up", dWu), ("dw_down", dWd)):
        assert _rel_l2(t, g[name]) <= 2e-3, name
    dbg = db.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(dbg - g["db"]) <= 2e-3 * np.linalg.norm(g["db"])


def test_backward_rejects_unsupported_shapes():
    L = S.small_random(200, 128, 512, 128, 16, 0.05, seed=1)    # M not a multiple of 128
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    y, h = T.twell_ffn_forward(x, wu, b, wd, tile_w=128, ell_w=16)
    with pytest.raises(T.TwellError):
        T.twell_ffn_backward(x, wu, wd, h, dev(L.x))


def test_backward_gaussian_full_shape_1_5b():
    """The backward pass at the 1.5B layer's full shape (4096 tokens, 2048 ->
    8192, 5 %), Gaussian weights and output gradient, through the same split
    schedules the bench times: every gradient within the y tolerance of the
    oracle's exact sums over the forward's own hidden activations."""
    L = S.relu_15b(0.05)
    rng = np.random.default_rng(15)
    dy = S.bf16_bits_from_f32(rng.standard_normal((L.M, L.d_model)).astype(np.float32))
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    y, h = T.twell_ffn_forward(x, wu, b, wd, tile_w=L.tile_w, ell_w=L.ell_w)
    assert T.read_status(h)[0] == 0
    dX, dWu, db, dWd = T.twell_ffn_backward(x, wu, wd, h, dev(dy))
    assert T.read_status(h)[0] == 0
    got, _ = twell_to_np(h)
    g = O.ffn_backward(L.x, L.w_up, L.b, L.w_down, dy, h=O.twell_unpack(got))
    for name, t in (("dx", dX), ("dw_up", dWu), ("dw_down", dWd)):
        assert _rel_l2(t, g[name]) <= 2e-3, name
    dbg = db.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(dbg - g["db"]) <= 2e-3 * np.linalg.norm(g["db"])
