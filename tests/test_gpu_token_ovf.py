"""GPU parity of the whole-token overflow form (twell_spmm_token_overflow)
against the oracle's token_overflow_split / token_overflow_spmm: the number of
overflowing tokens exactly, y within tolerance (bitwise on integer layers), and
the same y as the per-(token, tile) form computes."""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import assert_y_close, dev, host_bits, upload_twell

CASES = [
    # M, d, f, tw, E, rho
    (300, 256, 1024, 128, 8, 0.10),     # many overflowing tokens, token-major kernels
    (200, 128, 512, 64, 8, 0.15),       # decode-size kernels
    (130, 192, 512, 32, 4, 0.10),
    (64, 128, 512, 256, 24, 0.10),
    (100, 128, 256, 64, 64, 0.20),      # ell_w = tile_w: no overflow, no dense rows
]


@pytest.mark.parametrize("M,d,f,tw,E,rho", CASES)
def test_token_overflow_matches_oracle(M, d, f, tw, E, rho):
    L = S.small_random(M, d, f, tw, E, rho, seed=M + 2 * f)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), tw, E)
    main, tok, dense = O.token_overflow_split(ref)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y, n_tok = T.twell_spmm_token_overflow(a, dev(L.w_down), cap_tok=max(len(tok), 1))
    assert T.read_status(a)[0] == 0
    assert int(n_tok.item()) == len(tok)
    assert_y_close(y, O.token_overflow_spmm(main, tok, dense, L.w_down))
    y_pair = T.twell_spmm(a, dev(L.w_down))
    assert_y_close(y, O.twell_spmm(ref, L.w_down))
    assert_y_close(y_pair, O.twell_spmm(ref, L.w_down))


def test_token_overflow_integer_bitexact():
    L = S.integer_exact(M=256, d_model=256, d_ff=1024, tile_w=128, density=0.10, seed=3, ell_w=8)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    main, tok, dense = O.token_overflow_split(ref)
    assert len(tok) > 0
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y, n_tok = T.twell_spmm_token_overflow(a, dev(L.w_down), cap_tok=len(tok))
    assert int(n_tok.item()) == len(tok)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))


def test_token_overflow_capacity_is_reported():
    L = S.small_random(300, 128, 512, 128, 8, 0.10, seed=9)
    ref = O.twell_pack(O.hidden(L.x, L.w_up, L.b), 128, 8)
    _, tok, _ = O.token_overflow_split(ref)
    assert len(tok) > 2
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y, n_tok = T.twell_spmm_token_overflow(a, dev(L.w_down), cap_tok=2)
    code, _ = T.read_status(a)
    assert code == 3 and int(n_tok.item()) == len(tok)
