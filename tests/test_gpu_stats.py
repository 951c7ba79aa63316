"""GPU parity of the fused activation statistics (twell_up_pack_stats): per token
the L1 norm sum_j |h_rj| and the nonzero count, taken in the producer epilogues.

Reference: the oracle's activation_stats applied to h rebuilt from the GPU's own
TwELL output (so both sides see the same bf16 hidden values).  The count must
match exactly; the L1 norm is an fp32 sum of the token's n nonzero |h| values,
so it may differ from the exact sum by at most (n + 1) * 2^-24 * sum |h|
(the standard bound for recursive fp32 summation, plus the final rounding).
The sums are taken in a fixed order, so two runs give identical bits.
"""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import assert_twell_equal, dev, twell_to_np

CASES = [
    # M, d, f, tw, E, rho, gated   (M <= 256: decode-size producer; larger: token-major)
    (300, 256, 1024, 128, 16, 0.05, False),
    (520, 128, 512, 64, 8, 0.20, False),      # overflow
    (333, 128, 512, 32, 8, 0.10, True),       # gated: h can be negative
    (1, 256, 1024, 128, 16, 0.10, False),
    (100, 192, 512, 64, 8, 0.30, False),      # overflow
    (200, 128, 256, 32, 8, 0.15, True),
    (64, 256, 512, 128, 16, 0.0, False),      # zero density: l1 = 0, count = 0
]


def _check(a, l1, nnz_row):
    got, _ = twell_to_np(a)
    h = O.twell_unpack(got)
    l1_ref, nnz_ref = O.activation_stats(h)
    assert np.array_equal(nnz_row.cpu().numpy().astype(np.int64), nnz_ref)
    l1g = l1.cpu().numpy().astype(np.float64)
    bound = (nnz_ref + 1) * 2.0 ** -24 * l1_ref
    assert np.all(np.abs(l1g - l1_ref) <= bound), float(np.max(np.abs(l1g - l1_ref) - bound))


@pytest.mark.parametrize("M,d,f,tw,E,rho,gated", CASES)
def test_stats_match_oracle_and_packing_is_unchanged(M, d, f, tw, E, rho, gated):
    L = S.small_random(M, d, f, tw, E, rho, gated=gated, seed=M * 3 + f)
    args = (dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_gate))
    cap = M * (f // tw)
    a, l1, nnz_row = T.twell_up_pack_stats(*args, tile_w=tw, ell_w=E, ovf_capacity=cap)
    assert T.read_status(a)[0] == 0
    _check(a, l1, nnz_row)
    # the statistics do not perturb the packed output
    a2 = T.twell_up_pack(*args, tile_w=tw, ell_w=E, ovf_capacity=cap)
    assert T.read_status(a2)[0] == 0
    got2, _ = twell_to_np(a2)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, got2)
    # fixed summation order: identical bits on a second run
    _, l1b, nnzb = T.twell_up_pack_stats(*args, tile_w=tw, ell_w=E, ovf_capacity=cap)
    torch.cuda.synchronize()
    assert torch.equal(l1.view(torch.int32), l1b.view(torch.int32)) and torch.equal(nnz_row, nnzb)


def test_stats_15b_layer_full_size():
    L = S.relu_15b(0.05)
    a, l1, nnz_row = T.twell_up_pack_stats(dev(L.x), dev(L.w_up), dev(L.b), tile_w=L.tile_w,
                                           ell_w=L.ell_w)
    assert T.read_status(a)[0] == 0
    _check(a, l1, nnz_row)
    # every token's count is the sum of its packed per-tile counts
    nnz = a.nnz.view(torch.int16).to(torch.int32) & 0xFFFF
    assert torch.equal(nnz.sum(dim=1).to(torch.int32), nnz_row)
