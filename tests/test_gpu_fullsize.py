"""Bit-exact TwELL at the full size of every workload.

The GPU accumulates the up-projection in fp32 in its own order, so its hidden
values can differ from an fp64 evaluation by a rounding flip.  What must agree
bit for bit is everything the epilogue does with those accumulators: bias add,
ReLU (and the gate product), the one bf16 rounding, the compaction into ELL
slots, the overflow decision and the ordered dense backup (the TwELL layout of
upppp.jp 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).

Each test runs the fused producer twice at the workload's full size, with the
backup capacity bench.py uses:
  * once with the z_debug hook, which also writes the fp32 accumulators;
  * once exactly as bench.py launches it (no hook).
Both packed matrices must be identical, and equal -- every field, every row --
to the oracle packer applied to h replayed from those accumulators with the
epilogue's fp32 arithmetic.  Beside it, sampled rows of the accumulators are
held to the fp32 summation bound of the fp64 products."""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import (assert_twell_equal, assert_twell_valid, dev, h_from_zdebug, host_bits,
                              twell_to_np)

GEMM_REL_BOUND = 2.0 ** -16


def _rows(M):
    rng = np.random.default_rng(7)
    rows = set(rng.choice(M, size=min(M, 64), replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(rows))


def _replay_exact(L):
    f, tw, E = L.d_ff, L.tile_w, L.ell_w
    cap = T.default_ovf_capacity(L.M, f // tw)
    x, wu, wg, b = dev(L.x), dev(L.w_up), dev(L.w_gate), dev(L.b)
    z = torch.empty((L.M, 2 * f if L.gated else f), dtype=torch.float32, device="cuda")
    a_dbg = T.twell_up_pack(x, wu, b, wg, tile_w=tw, ell_w=E, ovf_capacity=cap, z_debug=z)
    assert T.read_status(a_dbg)[0] == 0
    a = T.twell_up_pack(x, wu, b, wg, tile_w=tw, ell_w=E, ovf_capacity=cap)
    code, n = T.read_status(a)
    assert code == 0 and n <= cap
    got, _ = twell_to_np(a)
    got_dbg, _ = twell_to_np(a_dbg)
    assert_twell_equal(got, got_dbg)          # the hook does not change the packing
    zg = z.cpu().numpy()
    del z, a_dbg
    torch.cuda.empty_cache()
    ref = O.twell_pack(h_from_zdebug(zg, L.b, L.gated, f), tw, E)
    assert_twell_equal(got, ref)               # every row, every field
    assert_twell_valid(got)
    # the accumulators themselves: within the fp32 bound of fp64 products
    rows = _rows(L.M)
    xr = O.bits_to_f64(L.x[rows])
    parts = (("gate", L.w_gate, slice(0, f)), ("up", L.w_up, slice(f, 2 * f))) if L.gated else \
        (("up", L.w_up, slice(0, f)),)
    for name, w, cols in parts:
        W = O.bits_to_f64(w)
        err = np.abs(zg[rows][:, cols] - xr @ W.T)
        bound = GEMM_REL_BOUND * (np.abs(xr) @ np.abs(W).T) + 1e-30
        assert (err / bound).max() <= 1.0, name
    return got, ref


@pytest.mark.parametrize("rho", S.TARGET_DENSITIES_15B)
def test_15b_layer_twell_bitexact(rho):
    got, ref = _replay_exact(S.relu_15b(rho))
    assert ref.n_ovf > 0 or rho <= 0.01


def test_gated_2b_layer_twell_bitexact():
    _replay_exact(S.gated_2b(0.05))


def test_heavy_tail_twell_bitexact():
    L = S.heavy_tail()
    got, ref = _replay_exact(L)
    assert ref.n_ovf > 1000                    # the dense backup is exercised heavily


@pytest.mark.parametrize("M", [32, 128, 256])
def test_decode_twell_bitexact(M):
    _replay_exact(S.decode(M))


def test_tiny_twell_bitexact():
    _replay_exact(S.tiny_relu(0))


def test_integer_gated_many_tiles_per_cluster_bitexact():
    """Gated producer with 256 tiles on at most 74 CTA pairs: every pair works
    through several tiles, so both TMEM accumulators of the epilogue are used.
    Integer-exact inputs make the whole layer (TwELL and y) exact in fp32."""
    L = S.integer_exact(M=1024, d_model=512, d_ff=8192, tile_w=128, density=0.05, gated=True, seed=11)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=L.tile_w,
                               ell_w=L.ell_w, W_gate=dev(L.w_gate),
                               ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))
