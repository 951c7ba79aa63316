"""Parity at the full workload sizes, in the launch configuration bench.py times
(twell_up_pack then twell_spmm, AUTO down path, default backup capacity).

Gaussian layers: sampled tokens against the fp64 oracle (h, TwELL counts, y),
plus invariants of the whole packed matrix.  Integer-exact layer at the 1.5B
shape: every field and every y bit against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import (assert_twell_equal, assert_twell_valid, dev, host_bits, twell_to_np,
                              y_errors, Y_MAX_ABS, Y_REL_L2)

GEMM_REL_BOUND = 2.0 ** -16


def _run(L, mode="auto"):
    a = T.TwELL.allocate(L.M, L.d_ff, L.tile_w, L.ell_w,
                         T.default_ovf_capacity(L.M, L.d_ff // L.tile_w))
    x, wu, wg, b, wd = dev(L.x), dev(L.w_up), dev(L.w_gate), dev(L.b), dev(L.w_down)
    T.twell_up_pack(x, wu, b, wg, tile_w=L.tile_w, ell_w=L.ell_w, out=a)
    y = T.twell_spmm(a, wd, mode=mode)
    code, n = T.read_status(a)
    assert code == 0, T.STATUS[code]
    return a, y


def _sample_rows(M, extra=()):
    rng = np.random.default_rng(123)
    rows = set(rng.choice(M, size=min(M, 96), replace=False).tolist())
    rows |= {0, M - 1, min(127, M - 1), min(128, M - 1)} | set(int(r) for r in extra)
    return np.array(sorted(rows))


def _check_sampled(L, a, y, rows):
    got, n = twell_to_np(a)
    assert_twell_valid(got)
    h64, pre = O.hidden(L.x[rows], L.w_up, L.b, L.w_gate, return_preact=True)
    # GPU h of the sampled rows, decoded from its own TwELL
    sub = O.TwELL(len(rows), L.d_ff, L.tile_w, L.ell_w, got.vals[rows], got.idx[rows],
                  got.nnz[rows], np.zeros(0, np.int32), np.zeros((0, L.tile_w), np.uint16))
    Tn = L.d_ff // L.tile_w
    keep = {int(p): k for k, p in enumerate(got.ovf_pos)}
    pos, dense = [], []
    for i, r in enumerate(rows):
        for t in range(Tn):
            k = keep.get(int(r) * Tn + t)
            if k is not None:
                pos.append(i * Tn + t)
                dense.append(got.ovf_dense[k])
    sub.ovf_pos = np.array(pos, dtype=np.int32)
    sub.ovf_dense = np.array(dense, dtype=np.uint16).reshape(-1, L.tile_w)
    h_gpu = O.twell_unpack(sub)
    # every difference is a bf16 rounding flip or a ReLU flip of a pre-activation
    # within the accumulator bound of zero
    x = np.abs(O.bits_to_f64(L.x[rows]))
    wsrc = L.w_gate if L.gated else L.w_up
    delta = GEMM_REL_BOUND * (x @ np.abs(O.bits_to_f64(wsrc)).T)
    if L.b is not None:
        delta += GEMM_REL_BOUND * np.abs(O.bits_to_f64(L.b))[None, :]
    if L.gated:
        u = pre[1]
        delta = delta * np.abs(u) + np.maximum(pre[0] + 0.0, 0) * GEMM_REL_BOUND * (
            x @ np.abs(O.bits_to_f64(L.w_up)).T)
    diff = np.abs(h_gpu - h64)
    ok = (diff <= 2.0 ** -7 * np.abs(h64) + 1e-30) | (diff <= 4 * delta + 1e-30)
    assert ok.all(), f"{(~ok).sum()} hidden values beyond rounding/threshold flips"
    assert np.mean(h_gpu != h64) < 1e-3
    # y of the sampled rows against the fp64 oracle
    y_ref = h64 @ O.bits_to_f64(L.w_down)
    rel, mx = y_errors(y[torch.from_numpy(rows).cuda()], y_ref)
    assert rel <= Y_REL_L2 and mx <= Y_MAX_ABS, (rel, mx)
    return got


def test_config_tiny_full():
    L = S.tiny_relu(0)
    a, y = _run(L)
    _check_sampled(L, a, y, np.arange(L.M))


@pytest.mark.parametrize("rho", S.TARGET_DENSITIES_15B)
def test_config_15b(rho):
    L = S.relu_15b(rho)
    a, y = _run(L)
    got = _check_sampled(L, a, y, _sample_rows(L.M))
    assert abs(got.nnz.astype(np.int64).sum() / (L.M * L.d_ff) - rho) < 0.1 * rho


def test_config_gated_2b():
    L = S.gated_2b(0.05)
    a, y = _run(L)
    _check_sampled(L, a, y, _sample_rows(L.M))


def test_config_heavy_tail():
    L = S.heavy_tail()
    a, y = _run(L)
    got = _check_sampled(L, a, y, _sample_rows(L.M, extra=L.meta["dense_rows"][:8]))
    # forced-dense tokens overflow every tile
    Tn = L.d_ff // L.tile_w
    for r in L.meta["dense_rows"][:8]:
        assert np.all(got.nnz[r] > L.ell_w)


@pytest.mark.parametrize("M", [32, 128, 256])
def test_config_decode(M):
    L = S.decode(M)
    a, y = _run(L)
    _check_sampled(L, a, y, np.arange(M) if M <= 128 else _sample_rows(M))


@pytest.mark.parametrize("mode", ["auto", "gather", "mma"])
def test_integer_family_15b_shape_bitexact(mode):
    L = S.integer_exact(M=4096, d_model=2048, d_ff=8192, tile_w=128, density=0.05)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    a, y = _run(L, mode)
    got, n = twell_to_np(a)
    assert n == ref.n_ovf
    assert_twell_equal(got, ref)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))
