"""The synthetic workloads have the densities and overflow rates they claim
(checked on oracle hidden activations of sampled tokens)."""
import numpy as np
import pytest

import oracle as O
import twell_synth as S


def _sample_density(L, rows):
    h = O.hidden(L.x[rows], L.w_up, L.b, L.w_gate)
    nnz = (h != 0).reshape(len(rows), L.n_tiles, L.tile_w).sum(axis=2)
    return float((h != 0).mean()), nnz


def test_bf16_generator_rounding_matches_torch():
    import torch
    a = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(S.bf16_bits_from_f32(a), ref)


def test_tiny_config():
    L = S.tiny_relu(0)
    assert (L.M, L.d_model, L.d_ff, L.tile_w, L.ell_w) == (64, 256, 1024, 64, 16)
    dens, _ = _sample_density(L, np.arange(64))
    assert 0.07 < dens < 0.13


@pytest.mark.parametrize("rho,E", [(0.20, 40), (0.10, 24), (0.05, 16), (0.01, 8)])
def test_15b_density_and_ell_rule(rho, E):
    L = S.relu_15b(rho, M=512)
    assert L.ell_w == E
    rows = np.arange(0, 512, 4)
    dens, nnz = _sample_density(L, rows)
    assert abs(dens - rho) < 0.15 * rho + 0.002
    assert (nnz > E).mean() < 0.02
    assert O.ell_width_p99(nnz, tile_w=128) <= E + 8


def test_gated_density():
    L = S.gated_2b(0.05, M=256, d_model=512, d_ff=2048)
    dens, nnz = _sample_density(L, np.arange(0, 256, 2))
    assert abs(dens - 0.05) < 0.01
    assert L.ell_w == 16


def test_heavy_tail_shape():
    L = S.heavy_tail(M=1024, d_model=512, d_ff=2048)
    rho = L.meta["token_density"]
    assert abs(L.meta["effective_density"] - rho.mean()) < 1e-12
    assert 0.03 < rho.mean() < 0.05
    dense_rows = L.meta["dense_rows"][:4]
    dens, nnz = _sample_density(L, dense_rows)
    assert dens > 0.99                      # forced tokens activate ~every neuron
    other = np.setdiff1d(np.arange(0, 1024, 8), L.meta["dense_rows"])
    d2, nnz2 = _sample_density(L, other)
    assert 0.02 < d2 < 0.05
    assert (nnz2 > L.ell_w).mean() < 0.03


def test_decode_and_integer_family():
    L = S.decode(M=32, d_model=512, d_ff=2048)
    dens, _ = _sample_density(L, np.arange(32))
    assert 0.01 < dens < 0.03
    I = S.integer_exact(64, 256, 1024, tile_w=64, density=0.1)
    for arr in (I.x, I.w_up, I.w_down):
        v = O.bits_to_f64(arr)
        assert set(np.unique(v)).issubset({-1.0, 0.0, 1.0})
    b = O.bits_to_f64(I.b)
    assert np.all(b == np.round(b))
    dens, _ = _sample_density(I, np.arange(64))
    assert 0.05 < dens < 0.15
