"""Pins for the CPU oracle, each against something other than the oracle itself:
a hand-computed example, brute force from the definition, invariants, closed
forms, and special cases that reduce to a library routine."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(v):
    return S.bf16_bits_from_f32(np.asarray(v, dtype=np.float32))


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------
def test_bf16_round_matches_torch_on_fp32_exact_values():
    rng = np.random.default_rng(1)
    a = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        # exact ties between two bf16 neighbours (low 16 bits == 0x8000)
        ((rng.integers(0x3000, 0x5000, 5000).astype(np.uint32) << 16) | 0x8000).view(np.float32),
        # fp32 subnormals, including ties
        (rng.integers(1, 1 << 16, 3000).astype(np.uint32)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0], dtype=np.float32),
    ])
    ours = O.bf16_round(a.astype(np.float64))
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_round_hand_values():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # just above a tie must round up; fp32 double rounding would get this wrong
    assert O.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    # integers: exact up to 256, then even spacing 2
    assert O.bf16_round(255.0) == 255.0 and O.bf16_round(257.0) == 256.0
    assert O.bf16_round(259.0) == 260.0
    # smallest subnormal step 2^-133: 1.5 steps ties to 2 steps
    assert O.bf16_round(1.5 * 2.0 ** -133) == 2.0 * 2.0 ** -133
    assert O.bf16_round(-3.140625) == -3.140625


def test_bits_roundtrip_all_finite_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]                       # finite only
    v = O.bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(v, ref)
    back = O.f64_to_bits(v)
    canon = np.where(bits == 0x8000, 0, bits)      # -0 stored as +0
    assert np.array_equal(back, canon.astype(np.uint16))


# ---------------------------------------------------------------------------
# Hand-computed example
# ---------------------------------------------------------------------------
def _hand():
    with open(os.path.join(GOLDEN, "hand_4x8.json")) as fh:
        return json.load(fh)


def test_hand_example_pack_and_y():
    g = _hand()
    x = _bits(g["x"])
    eye = _bits(np.eye(8))
    wd = _bits(g["w_down"])
    e = g["expected"]
    h = O.hidden(x, eye, None)
    assert np.array_equal(h, np.array(e["h"], dtype=np.float64))
    a = O.twell_pack(h, g["tile_w"], g["ell_w"])
    assert a.nnz.tolist() == e["nnz"]
    assert O.bits_to_f64(a.vals).tolist() == e["vals"]
    assert a.idx.tolist() == e["idx"]
    assert a.n_ovf == e["n_ovf"] and a.ovf_pos.tolist() == e["ovf_pos"]
    assert O.bits_to_f64(a.ovf_dense).tolist() == e["ovf_dense"]
    y = O.twell_spmm(a, wd)
    assert y.tolist() == e["y"]
    assert y.tolist() != e["y_if_truncated_ell_used_for_overflow"]
    a2, y2 = O.ffn_forward(x, eye, None, wd, g["tile_w"], g["ell_w"])
    assert y2.tolist() == e["y"]


# ---------------------------------------------------------------------------
# Brute force from the definition
# ---------------------------------------------------------------------------
def _pack_by_definition(hrow, tw, E):
    """Per-tile ELL of one token, written directly from the definition."""
    out = []
    for t in range(len(hrow) // tw):
        seg = hrow[t * tw:(t + 1) * tw]
        nzpos = [j for j in range(tw) if seg[j] != 0.0]
        vals = [seg[j] for j in nzpos[:E]] + [0.0] * (E - min(E, len(nzpos)))
        idx = nzpos[:E] + [0] * (E - min(E, len(nzpos)))
        out.append((len(nzpos), vals, idx, len(nzpos) > E, list(seg)))
    return out


@pytest.mark.parametrize("tw", [4, 8])
def test_pack_brute_force_all_patterns(tw):
    pats = np.array(list(itertools.product([0, 1], repeat=tw)), dtype=np.float64)
    # distinct small integers (bf16-exact), alternating sign
    base = np.array([(j + 1) * (-1) ** j for j in range(tw)], dtype=np.float64)
    h = np.concatenate([pats * base, pats[::-1] * (base + 0.5)], axis=1)  # 2 tiles per row
    for E in range(1, tw + 1):
        a = O.twell_pack(h, tw, E)
        T = 2
        ovf = []
        for r in range(h.shape[0]):
            for t, (n, vals, idx, over, seg) in enumerate(_pack_by_definition(list(h[r]), tw, E)):
                assert a.nnz[r, t] == n
                assert O.bits_to_f64(a.vals[r, t]).tolist() == vals
                assert a.idx[r, t].tolist() == idx
                if over:
                    ovf.append((r * T + t, seg))
        assert a.ovf_pos.tolist() == [p for p, _ in ovf]
        assert O.bits_to_f64(a.ovf_dense).tolist() == [s for _, s in ovf]
        assert np.array_equal(O.twell_unpack(a), h)


def test_hidden_brute_force_integers():
    """Small integer layers: z is computed here with exact Python integers;
    |z| and |g*u| stay below 256, so bf16 rounding is the identity."""
    rng = np.random.default_rng(7)
    M, d, f = 5, 6, 12     # f != d so a transposed weight cannot pass
    x = rng.integers(-2, 3, (M, d))
    wu = rng.integers(-2, 3, (f, d))
    wg = rng.integers(-2, 3, (f, d))
    b = rng.integers(-3, 4, f)
    h = O.hidden(_bits(x), _bits(wu), _bits(b))
    hg = O.hidden(_bits(x), _bits(wu), _bits(b), w_gate_bits=_bits(wg))
    for r in range(M):
        for j in range(f):
            z = sum(int(x[r, k]) * int(wu[j, k]) for k in range(d)) + int(b[j])
            assert h[r, j] == max(z, 0)
            g = sum(int(x[r, k]) * int(wg[j, k]) for k in range(d)) + int(b[j])
            u = sum(int(x[r, k]) * int(wu[j, k]) for k in range(d))
            assert hg[r, j] == max(g, 0) * u
    # the gated product is rounded once: 3 * 131 = 393 -> bf16 392
    hx = O.hidden(_bits([[1.0]]), _bits([[131.0]]), _bits([0.0]), w_gate_bits=_bits([[3.0]]))
    assert hx[0, 0] == 392.0


def test_spmm_brute_force_tiny():
    """y from explicit per-slot sums (math.fsum) over the TwELL slots."""
    rng = np.random.default_rng(3)
    for trial in range(6):
        M, d, f, tw = 7, 5, 32, 8
        E = int(rng.integers(1, tw + 1))
        h = O.bf16_round(rng.standard_normal((M, f)) * (rng.random((M, f)) < 0.4))
        wd = _bits(rng.standard_normal((f, d)))
        a = O.twell_pack(h, tw, E)
        y = O.twell_spmm(a, wd)
        W = O.bits_to_f64(wd)
        T = f // tw
        vals = O.bits_to_f64(a.vals)
        ovf = {int(p): k for k, p in enumerate(a.ovf_pos)}
        for r in range(M):
            for c in range(d):
                terms = []
                for t in range(T):
                    if a.nnz[r, t] <= E:
                        for s in range(int(a.nnz[r, t])):
                            terms.append(vals[r, t, s] * W[t * tw + a.idx[r, t, s], c])
                    else:
                        seg = O.bits_to_f64(a.ovf_dense[ovf[r * T + t]])
                        terms += [seg[j] * W[t * tw + j, c] for j in range(tw)]
                assert math.isclose(y[r, c], math.fsum(terms), rel_tol=1e-12, abs_tol=1e-12)


# ---------------------------------------------------------------------------
# Invariants and special cases
# ---------------------------------------------------------------------------
def _random_layer(seed, M=37, d=64, f=256, tw=32, E=4, rho=0.1, gated=False):
    return S.small_random(M, d, f, tw, E, rho, gated=gated, seed=seed)


@pytest.mark.parametrize("gated", [False, True])
def test_invariants_random(gated):
    L = _random_layer(11, gated=gated)
    h = O.hidden(L.x, L.w_up, L.b, L.w_gate)
    a = O.twell_pack(h, L.tile_w, L.ell_w)
    T = a.n_tiles
    assert np.array_equal(a.nnz.sum(axis=1), (h != 0).sum(axis=1))
    assert np.array_equal(O.twell_unpack(a), h)
    slot = np.arange(a.ell_w)[None, None, :]
    pad = slot >= a.nnz[:, :, None]
    assert np.all(a.vals[pad] == 0) and np.all(a.idx[pad] == 0)
    live = ~pad
    assert np.all(a.vals[live] != 0) and np.all((a.vals[live] & 0x7FFF) != 0)
    assert np.all(np.diff(a.ovf_pos) > 0)
    assert a.n_ovf == int((a.nnz > a.ell_w).sum())
    # ascending in-tile order inside each slot list
    for r in range(a.M):
        for t in range(T):
            n = min(int(a.nnz[r, t]), a.ell_w)
            assert np.all(np.diff(a.idx[r, t, :n].astype(int)) > 0)
    # sparse and dense down-projections agree
    y = O.twell_spmm(a, L.w_down)
    yd = O.dense_ffn(L.x, L.w_up, L.b, L.w_down, L.w_gate)
    assert np.allclose(y, yd, rtol=0, atol=1e-12)


def test_full_ell_width_is_plain_ell_and_textbook_matmul():
    L = _random_layer(5, tw=32, E=32, rho=0.3)
    h = O.hidden(L.x, L.w_up, L.b)
    a = O.twell_pack(h, 32, 32)
    assert a.n_ovf == 0
    y = O.twell_spmm(a, L.w_down)
    ref = np.matmul(h, O.bits_to_f64(L.w_down))
    assert np.array_equal(y, ref)


def test_zero_density_gives_zero():
    L = _random_layer(2, rho=0.0)
    a, y = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    assert int(a.nnz.sum()) == 0 and a.n_ovf == 0
    assert np.all(a.vals == 0) and np.all(a.idx == 0)
    assert np.all(y == 0)


def test_full_density_overflows_everywhere():
    L = _random_layer(4, rho=1.0, E=4, tw=32)
    a, y = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    assert a.n_ovf == a.M * a.n_tiles
    assert np.array_equal(a.ovf_pos, np.arange(a.M * a.n_tiles, dtype=np.int32))
    h = O.hidden(L.x, L.w_up, L.b)
    assert np.array_equal(y, h @ O.bits_to_f64(L.w_down))


def test_gated_zero_is_positive_zero():
    """max(g, 0) * u with u < 0 gives -0; it must count as zero and store as +0."""
    x = _bits([[1.0, 1.0]])
    wg = _bits([[-1.0, -1.0], [1.0, 1.0]])
    wu = _bits([[-1.0, 0.0], [-1.0, 0.0]])
    h = O.hidden(x, wu, None, w_gate_bits=wg)
    assert h[0, 0] == 0.0 and not np.signbit(h[0, 0])
    assert h[0, 1] == -2.0
    a = O.twell_pack(np.tile(h, (1, 16)), 32, 4)
    assert a.nnz[0, 0] == 16


def test_integer_family_exact():
    L = S.integer_exact(M=24, d_model=64, d_ff=256, tile_w=32, density=0.1, seed=1)
    h = O.hidden(L.x, L.w_up, L.b)
    assert np.all(h == np.round(h))
    x = O.bits_to_f64(L.x).astype(np.int64)
    wu = O.bits_to_f64(L.w_up).astype(np.int64)
    b = O.bits_to_f64(L.b).astype(np.int64)
    z = x @ wu.T + b
    assert np.array_equal(h, O.bf16_round(np.maximum(z, 0).astype(np.float64)))
    a, y = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    yi = h.astype(np.int64) @ O.bits_to_f64(L.w_down).astype(np.int64)
    assert np.array_equal(y, yi.astype(np.float64))


def test_ell_width_p99_closed_form():
    assert O.ell_width_p99(np.arange(1, 101)) == 104          # p99 = 99
    assert O.ell_width_p99(np.zeros(50)) == 8
    assert O.ell_width_p99(np.full(1000, 17)) == 24
    v = np.concatenate([np.full(99, 3), [200]])
    assert O.ell_width_p99(v) == 8                             # nearest rank 99 of 100 -> 3


# ---------------------------------------------------------------------------
# Per-token activation statistics (L1 norm, nonzero count)
# ---------------------------------------------------------------------------
def test_stats_hand_example():
    """The sums of |h| and the nonzero counts of the hand-computed example."""
    g = _hand()
    h = O.hidden(_bits(g["x"]), _bits(np.eye(8)), None)
    l1, nnz = O.activation_stats(h)
    assert l1.tolist() == g["expected"]["l1"]
    assert nnz.tolist() == g["expected"]["nnz_row"]


def test_stats_gated_negative_values_by_hand():
    """Gated layer whose h has negative entries (worked out by hand): x = [1, 2],
    W_gate = I, b = 0 -> ReLU(g) = [1, 2]; W_up rows [-1, 0] and [0, -3] ->
    u = [-1, -6]; h = [-1, -12]; a second token x = [-1, 5] -> ReLU(g) = [0, 5],
    u = [1, -15] -> h = [0, -75].  So l1 = [13, 75] and nnz = [2, 1]; a sum of
    signed values would give [-13, -75]."""
    x = _bits([[1, 2], [-1, 5]])
    wg = _bits(np.eye(2))
    wu = _bits([[-1, 0], [0, -3]])
    h = O.hidden(x, wu, None, wg)
    assert h.tolist() == [[-1.0, -12.0], [0.0, -75.0]]
    l1, nnz = O.activation_stats(h)
    assert l1.tolist() == [13.0, 75.0] and nnz.tolist() == [2, 1]


@pytest.mark.parametrize("tw,E", [(32, 4), (64, 8), (128, 16)])
def test_stats_agree_with_the_packed_form(tw, E):
    """nnz per token = the packed counts summed over tiles; l1 per token = the
    sum of |slot values| (pairs within the ELL width) plus |backup segments|."""
    L = S.small_random(37, 64, 512, tw, E, 0.15, seed=tw)
    h = O.hidden(L.x, L.w_up, L.b)
    l1, nnz = O.activation_stats(h)
    a = O.twell_pack(h, tw, E)
    assert np.array_equal(nnz, a.nnz.astype(np.int64).sum(axis=1))
    from_slots = np.zeros(h.shape[0])
    vals = np.abs(O.bits_to_f64(a.vals))
    seg = dict(zip(a.ovf_pos.tolist(), np.abs(O.bits_to_f64(a.ovf_dense))))
    T = a.nnz.shape[1]
    for r in range(h.shape[0]):
        parts = [seg[r * T + t].sum() if a.nnz[r, t] > E else vals[r, t].sum() for t in range(T)]
        from_slots[r] = math.fsum(parts)
    assert np.allclose(l1, from_slots, rtol=1e-13, atol=0)
    assert a.n_ovf > 0   # the backup branch is exercised


def test_stats_zero_density():
    L = S.small_random(8, 64, 256, 64, 8, 0.0)
    l1, nnz = O.activation_stats(O.hidden(L.x, L.w_up, L.b))
    assert np.all(l1 == 0) and np.all(nnz == 0)


# ---------------------------------------------------------------------------
# Backward pass (non-gated) and the transposed packed form
# ---------------------------------------------------------------------------
def test_backward_hand_example():
    """Worked out by hand: W_up = I, b = 0, W_down rows [1, 2] and [3, 4],
    x = [[1, -1], [2, 3]], dY = I.  h = [[1, 0], [2, 3]]; dY W_down^T =
    [[1, 3], [2, 4]]; masked dZ = [[1, 0], [2, 4]]; dX = dZ; dW_up = dZ^T x =
    [[5, 5], [8, 12]]; db = [3, 4]; dW_down = h^T dY = [[1, 2], [0, 3]]."""
    g = O.ffn_backward(_bits([[1, -1], [2, 3]]), _bits(np.eye(2)), None,
                       _bits([[1, 2], [3, 4]]), _bits(np.eye(2)))
    assert g["dz"].tolist() == [[1, 0], [2, 4]]
    assert g["dx"].tolist() == [[1, 0], [2, 4]]
    assert g["dw_up"].tolist() == [[5, 5], [8, 12]]
    assert g["db"].tolist() == [3, 4]
    assert g["dw_down"].tolist() == [[1, 2], [0, 3]]


def test_backward_matches_finite_differences():
    """Unrounded gradients against central differences of the fp64 layer
    L = sum(relu(x W_up^T + b) W_down * dY).  x W_up^T is a multiple of 1/8 and
    b = 1/16, so every pre-activation is at least 1/16 away from the ReLU kink: a
    step of 2^-12 never crosses it and the layer is exactly linear along each
    perturbed coordinate."""
    rng = np.random.default_rng(7)
    M, d, f = 5, 6, 9
    x = rng.integers(-3, 4, size=(M, d)).astype(np.float64) / 2
    wu = rng.integers(-3, 4, size=(f, d)).astype(np.float64) / 4
    b = np.full(f, 1.0 / 16)
    z = x @ wu.T + b
    assert np.min(np.abs(z)) >= 1.0 / 16 and np.any(z < 0) and np.any(z > 0)
    wd = rng.integers(-2, 3, size=(f, d)).astype(np.float64)
    dy = rng.integers(-2, 3, size=(M, d)).astype(np.float64)
    bits = [O.f64_to_bits(v) for v in (x, wu, b, wd, dy)]
    for v, bb in zip((x, wu, b, wd, dy), bits):
        assert np.array_equal(O.bits_to_f64(bb), v)            # all bf16-exact
    g = O.ffn_backward(*bits, round_bf16=False)

    def loss(x_, wu_, b_, wd_):
        return float(np.sum(np.maximum(x_ @ wu_.T + b_[None, :], 0.0) @ wd_ * dy))

    eps = 2.0 ** -12
    for name, arr, pos in (("dx", x, 0), ("dw_up", wu, 1), ("db", b, 2), ("dw_down", wd, 3)):
        for idx in np.ndindex(arr.shape):
            args_p = [x.copy(), wu.copy(), b.copy(), wd.copy()]
            args_m = [x.copy(), wu.copy(), b.copy(), wd.copy()]
            args_p[pos][idx] += eps
            args_m[pos][idx] -= eps
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[name][idx]) <= 1e-9 * max(1.0, abs(fd)), (name, idx, fd, g[name][idx])


def test_backward_dz_has_the_forward_pattern():
    L = S.small_random(20, 32, 128, 32, 8, 0.2, seed=5)
    dy = S.small_random(20, 32, 128, 32, 8, 0.2, seed=6).x
    g = O.ffn_backward(L.x, L.w_up, L.b, L.w_down, dy)
    h = O.hidden(L.x, L.w_up, L.b)
    assert np.all(g["dz"][h == 0] == 0)                        # zero where h is zero


@pytest.mark.parametrize("tw,E", [(32, 4), (64, 8)])
def test_transpose_matches_numpy_transpose(tw, E):
    L = S.small_random(128, 32, 256, 64, 8, 0.15, seed=tw)
    h = O.hidden(L.x, L.w_up, L.b)
    a = O.twell_pack(h, 64, 8)
    at = O.twell_transpose(a, tw, E)
    assert at.M == 256 and at.d_ff == 128
    assert np.array_equal(O.twell_unpack(at), h.T)
    assert at.n_ovf > 0 or E >= tw


# ---------------------------------------------------------------------------
# Whole-token overflow form (the alternative reading of the backup)
# ---------------------------------------------------------------------------
def test_token_overflow_hand_example():
    """In the hand example only token 2 has an over-full tile (tile 0, 3 > 2
    nonzeros): it becomes the one dense row, and y is unchanged."""
    g = _hand()
    e = g["expected"]
    h = O.hidden(_bits(g["x"]), _bits(np.eye(8)), None)
    a = O.twell_pack(h, g["tile_w"], g["ell_w"])
    main, tok, dense = O.token_overflow_split(a)
    assert tok.tolist() == [2]
    assert main.nnz.tolist() == [[2, 0], [1, 1], [0, 0], [0, 0]] and main.n_ovf == 0
    assert O.twell_unpack(dense).tolist() == [e["h"][2]]
    assert dense.n_ovf == 0
    y = O.token_overflow_spmm(main, tok, dense, _bits(g["w_down"]))
    assert y.tolist() == e["y"]


@pytest.mark.parametrize("tw,E,rho", [(32, 4, 0.15), (64, 8, 0.2), (128, 16, 0.1)])
def test_token_overflow_matches_dense_product(tw, E, rho):
    L = S.small_random(60, 48, 512, tw, E, rho, seed=tw + 3)
    h = O.hidden(L.x, L.w_up, L.b)
    a = O.twell_pack(h, tw, E)
    main, tok, dense = O.token_overflow_split(a)
    # the overflowing tokens, straight from h: any tile with more than E nonzeros
    per_tile = (h.reshape(h.shape[0], -1, tw) != 0).sum(axis=2)
    assert np.array_equal(tok, np.nonzero((per_tile > E).any(axis=1))[0])
    assert len(tok) > 0
    y = O.token_overflow_spmm(main, tok, dense, L.w_down)
    assert np.allclose(y, np.matmul(h, O.bits_to_f64(L.w_down)), rtol=1e-12, atol=1e-12)
