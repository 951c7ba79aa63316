"""CPU oracle for the activation-sparse ReLU FFN forward pass with TwELL packing.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module;
only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA library: inputs arrive as bf16 bit patterns and
every step below is written out plainly in float64 NumPy.

What is computed (sources are the news pages on "Sparser, Faster, Lighter
Transformer Language Models", Sakana AI / NVIDIA):

* FFN: up-projection to a wide hidden dimension, a ReLU, and a down-projection
  back to the model dimension; tokens are independent (upppp.jp 2026-05-11,
  section 「LLMフィードフォワード層の「無駄」とは何か」; innovatopia.jp,
  glossary entry フィードフォワード層).  Gated variant: h = ReLU(x W_g^T + b) * (x W_u^T)
  (the gated 2B-scale workload; the TwELL pages do not spell it out).
* TwELL: hidden columns are cut into fixed-width tiles and each token keeps an
  ELL-style list of its nonzeros (value, in-tile index) per tile (upppp.jp,
  section 「TwELLとカスタムCUDAカーネルが解決する課題」; innovatopia.jp glossary
  entry TwELL).
* Hybrid: a sparse main part plus a small dense backup (same upppp.jp section);
  here a (token, tile) pair whose nonzero count exceeds the ELL width keeps its
  whole dense tile segment in the backup.
* Down-projection consuming only the packed nonzeros (same section; innovatopia.jp
  editorial notes on tile alignment).

Readings where the pages are silent (each one is listed with its reason in the
design notes):
  R1  h is rounded once, fp64 -> bf16 round-to-nearest-even (gated: one rounding of
      the product).
  R2  "nonzero" means the bf16 value is not +-0; stored zeros are +0.
  R3  ELL slots hold nonzeros in ascending in-tile order; unused slots are
      (value +0, index 0); nnz holds the true count, which may exceed ell_w.
  R4  a (token, tile) pair overflows iff nnz > ell_w; overflow pairs are listed in
      ascending r*T + t with their full dense segment; their ELL slots still hold the
      first ell_w nonzeros and are ignored by consumers.
  R5  y is compared in fp64 before its final bf16 rounding.

Parity status: every function here is pinned by tests that do not call back into
the function under test (hand-computed example, brute force, invariants,
library special cases).  No function is "parity unpinned".
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "bf16_round",
    "bits_to_f64",
    "f64_to_bits",
    "hidden",
    "TwELL",
    "twell_pack",
    "twell_unpack",
    "twell_spmm",
    "ffn_forward",
    "dense_ffn",
    "ell_width_p99",
    "activation_stats",
    "ffn_backward",
    "twell_transpose",
    "token_overflow_split",
    "token_overflow_spmm",
]


# ---------------------------------------------------------------------------
# bf16 arithmetic
# ---------------------------------------------------------------------------
def bf16_round(a) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even (reading R1).

    bf16 keeps 8 significant bits and fp32's exponent range.  For a = m * 2**e with
    0.5 <= |m| < 1 the bf16 quantum is 2**(e - 8); below the smallest normal
    (2**-126, frexp exponent -125) the quantum stays 2**-133 (subnormals).
    Inputs are assumed finite and below the bf16 maximum.
    """
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)
    e = np.maximum(e, -125)
    q = np.ldexp(1.0, e - 8)
    return np.rint(a / q) * q


def bits_to_f64(bits) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bits(v) -> np.ndarray:
    """bf16 bit pattern of float64 values that are already bf16-exact; zeros -> +0."""
    v = np.asarray(v, dtype=np.float64)
    v = np.where(v == 0.0, 0.0, v)            # canonical +0 (reading R2)
    u = v.astype(np.float32).view(np.uint32)  # exact: v is a bf16 value
    assert np.all((u & np.uint32(0xFFFF)) == 0), "value is not bf16-exact"
    return (u >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Up-projection + activation
# ---------------------------------------------------------------------------
def hidden(x_bits, w_up_bits, b_bits=None, w_gate_bits=None, return_preact=False):
    """Hidden activations h (float64 holding bf16 values), shape [M, d_ff].

    Non-gated:  z = x W_up^T + b,            h = bf16(max(z, 0))
    Gated:      g = x W_gate^T + b, u = x W_up^T,  h = bf16(max(g, 0) * u)
    Products and sums are float64 (exact enough that only the final rounding
    matters at these sizes).  W_* are [d_ff, d_model] (row j = neuron j).
    """
    x = bits_to_f64(x_bits)
    wu = bits_to_f64(w_up_bits)
    b = bits_to_f64(b_bits) if b_bits is not None else 0.0
    if w_gate_bits is None:
        z = x @ wu.T + b
        h = bf16_round(np.maximum(z, 0.0))
        pre = (z,)
    else:
        g = x @ bits_to_f64(w_gate_bits).T + b
        u = x @ wu.T
        h = bf16_round(np.maximum(g, 0.0) * u)
        pre = (g, u)
    h = np.where(h == 0.0, 0.0, h)   # -0 -> +0 (reading R2)
    return (h, pre) if return_preact else h


# ---------------------------------------------------------------------------
# TwELL
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class TwELL:
    """Tile-wise ELLPACK matrix plus the dense backup for overflowing pairs."""

    M: int
    d_ff: int
    tile_w: int
    ell_w: int
    vals: np.ndarray       # [M, T, E] uint16 (bf16 bits)
    idx: np.ndarray        # [M, T, E] uint8  (in-tile column)
    nnz: np.ndarray        # [M, T]    uint16 (true count)
    ovf_pos: np.ndarray    # [n_ovf]   int32  (r*T + t, ascending)
    ovf_dense: np.ndarray  # [n_ovf, tile_w] uint16 (bf16 bits)

    @property
    def n_tiles(self) -> int:
        return self.d_ff // self.tile_w

    @property
    def n_ovf(self) -> int:
        return int(self.ovf_pos.shape[0])


def twell_pack(h, tile_w: int, ell_w: int) -> TwELL:
    """Pack dense h (float64 holding bf16 values, [M, d_ff]) into TwELL.

    For each token r and tile t: S = ascending in-tile positions of the nonzeros
    of h[r, t*tw:(t+1)*tw]; nnz = |S|; slot s < min(|S|, E) holds (h at S[s], S[s]);
    other slots hold (+0, 0).  A pair with |S| > E also appends its whole dense
    segment to the backup, pairs in ascending r*T + t (readings R3, R4).
    """
    h = np.asarray(h, dtype=np.float64)
    M, f = h.shape
    tw, E = int(tile_w), int(ell_w)
    assert f % tw == 0 and 1 <= E <= tw and tw <= 256
    T = f // tw
    vals = np.zeros((M, T, E), dtype=np.uint16)
    idx = np.zeros((M, T, E), dtype=np.uint8)
    nnz = np.zeros((M, T), dtype=np.uint16)
    for t in range(T):
        seg = h[:, t * tw:(t + 1) * tw]
        nz = seg != 0.0
        nnz[:, t] = nz.sum(axis=1)
        slot = np.cumsum(nz, axis=1) - 1          # slot of each nonzero, in column order
        rows, cols = np.nonzero(nz & (slot < E))
        s = slot[rows, cols]
        vals[rows, t, s] = f64_to_bits(seg[rows, cols])
        idx[rows, t, s] = cols
    ovf_r, ovf_t = np.nonzero(nnz.astype(np.int64) > E)   # row-major => ascending r*T+t
    ovf_pos = (ovf_r * T + ovf_t).astype(np.int32)
    ovf_dense = np.zeros((ovf_pos.size, tw), dtype=np.uint16)
    for k, (r, t) in enumerate(zip(ovf_r, ovf_t)):
        ovf_dense[k] = f64_to_bits(h[r, t * tw:(t + 1) * tw])
    return TwELL(M, f, tw, E, vals, idx, nnz, ovf_pos, ovf_dense)


def twell_unpack(a: TwELL) -> np.ndarray:
    """Rebuild dense h from TwELL: ELL slots for pairs with nnz <= E, the dense
    backup segment for overflowing pairs."""
    T, tw, E = a.n_tiles, a.tile_w, a.ell_w
    h = np.zeros((a.M, a.d_ff), dtype=np.float64)
    v = bits_to_f64(a.vals)
    for t in range(T):
        ok = a.nnz[:, t].astype(np.int64) <= E
        for s in range(E):
            live = ok & (s < a.nnz[:, t].astype(np.int64))
            r = np.nonzero(live)[0]
            h[r, t * tw + a.idx[r, t, s].astype(np.int64)] = v[r, t, s]
    for k, p in enumerate(a.ovf_pos):
        r, t = divmod(int(p), T)
        h[r, t * tw:(t + 1) * tw] = bits_to_f64(a.ovf_dense[k])
    return h


def twell_spmm(a: TwELL, w_down_bits) -> np.ndarray:
    """y = h W_down with h read only from the TwELL slots and the dense backup.

    y_r = sum_t [ nnz <= E ? sum_{s < nnz} vals * W_down[t*tw + idx]
                           : sum_j ovf_dense[j] * W_down[t*tw + j] ]
    evaluated as (decoded h) @ W_down in float64; returns fp64 y (reading R5).
    """
    return twell_unpack(a) @ bits_to_f64(w_down_bits)


def ffn_forward(x_bits, w_up_bits, b_bits, w_down_bits, tile_w, ell_w, w_gate_bits=None):
    """Full layer: hidden -> TwELL -> sparse down-projection.  Returns (TwELL, y_fp64)."""
    h = hidden(x_bits, w_up_bits, b_bits, w_gate_bits)
    a = twell_pack(h, tile_w, ell_w)
    return a, twell_spmm(a, w_down_bits)


def dense_ffn(x_bits, w_up_bits, b_bits, w_down_bits, w_gate_bits=None) -> np.ndarray:
    """The same layer with no packing at all: bf16(h) @ W_down in float64."""
    return hidden(x_bits, w_up_bits, b_bits, w_gate_bits) @ bits_to_f64(w_down_bits)


def activation_stats(h):
    """Per-token statistics of the hidden activations that an L1 activation
    regulariser works with (the pages pair ReLU sparsity with an L1 penalty:
    upppp.jp 2026-05-11, sections 「LLMフィードフォワード層の「無駄」とは何か」 and
    「実際の性能改善」): the L1 norm sum_j |h_rj| of the token's bf16 hidden
    values, and its number of nonzeros (bf16 value not +-0, reading R2).

    h: float64 [M, d_ff] holding bf16 values.  Returns (l1 float64 [M], nnz int64 [M]).
    """
    h = np.asarray(h, dtype=np.float64)
    return np.abs(h).sum(axis=1), np.count_nonzero(h, axis=1).astype(np.int64)


def ffn_backward(x_bits, w_up_bits, b_bits, w_down_bits, dy_bits, round_bf16: bool = True,
                 h=None):
    """Backward pass of the non-gated layer y = bf16(ReLU(x W_up^T + b)) W_down for
    a given output gradient dY, through the same sparsity pattern the forward packs
    (the pages' training kernel runs the whole backward pass on the hybrid sparse
    form: upppp.jp 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).

    Readings (the pages give no formulas):
      B1  the ReLU derivative is 1 where the stored h is nonzero, 0 elsewhere;
      B2  dZ = (dY W_down^T) masked by that pattern, stored in bf16 (one rounding);
      B3  dX = dZ W_up, dW_up = dZ^T x, db = column sums of dZ, dW_down = h^T dY,
          each an exact sum here (float64), rounded once to bf16 on the GPU.
    round_bf16=False keeps h and dZ unrounded: the exact gradient of the fp64
    piecewise-linear layer, used to pin this function against finite differences.
    h (float64 holding bf16 values), if given, is taken as the forward's hidden
    activations -- pattern and values -- instead of being recomputed from x.

    Returns dict(dz [M, d_ff], dx [M, d], dw_up [d_ff, d], db [d_ff], dw_down [d_ff, d]),
    all float64.
    """
    x = bits_to_f64(x_bits)
    w_up = bits_to_f64(w_up_bits)
    w_down = bits_to_f64(w_down_bits)
    dy = bits_to_f64(dy_bits)
    if h is None:
        z = x @ w_up.T
        if b_bits is not None:
            z = z + bits_to_f64(b_bits)[None, :]
        h = np.maximum(z, 0.0)
        if round_bf16:
            h = bf16_round(h)
    h = np.asarray(h, dtype=np.float64)
    mask = h != 0.0
    dz = np.where(mask, dy @ w_down.T, 0.0)
    if round_bf16:
        dz = bf16_round(dz)
    return dict(dz=dz, dx=dz @ w_up, dw_up=dz.T @ x, db=dz.sum(axis=0), dw_down=h.T @ dy)


def twell_transpose(a: TwELL, tile_w: int, ell_w: int) -> TwELL:
    """The same sparse matrix with rows and columns exchanged, packed as TwELL:
    rows = hidden units, columns = tokens cut into tiles of tile_w tokens (the
    layout the weight gradients h^T dY and dZ^T x are read from).  Requires
    a.M % tile_w == 0."""
    return twell_pack(twell_unpack(a).T.copy(), tile_w, ell_w)


def token_overflow_split(a: TwELL):
    """Whole-token reading of the backup (the alternative to R4): a token with any
    tile holding more than ell_w nonzeros keeps its whole hidden row, the rest keep
    only their ELL slots.

    Returns (main, tok_pos, dense): `main` is `a` with every overflowing token's
    counts set to 0 (its slots and backup no longer used; n_ovf = 0 since the
    remaining tokens have no overflowing pair); `tok_pos` the overflowing tokens in
    ascending order; `dense` their rows packed with ell_w = tile_w (every nonzero of
    a tile fits, so no backup exists)."""
    h = twell_unpack(a)
    tok = np.nonzero((a.nnz.astype(np.int64) > a.ell_w).any(axis=1))[0].astype(np.int32)
    nnz = a.nnz.copy()
    nnz[tok] = 0
    main = TwELL(a.M, a.d_ff, a.tile_w, a.ell_w, a.vals.copy(), a.idx.copy(), nnz,
                 np.zeros(0, np.int32), np.zeros((0, a.tile_w), np.uint16))
    dense = twell_pack(h[tok], a.tile_w, a.tile_w)
    return main, tok, dense


def token_overflow_spmm(main: TwELL, tok_pos, dense: TwELL, w_down_bits) -> np.ndarray:
    """y for the whole-token form: the ELL slots of the remaining tokens, and a
    small dense product for the overflowing tokens' rows."""
    y = twell_spmm(main, w_down_bits)
    if len(tok_pos):
        y[np.asarray(tok_pos)] = twell_unpack(dense) @ bits_to_f64(w_down_bits)
    return y


def ell_width_p99(nnz, multiple: int = 8, tile_w: Optional[int] = None) -> int:
    """Smallest multiple of 8 >= the nearest-rank 99th percentile of nnz values."""
    v = np.sort(np.asarray(nnz, dtype=np.int64).ravel())
    k = v[int(np.ceil(0.99 * v.size)) - 1]
    e = max(multiple, int(np.ceil(k / multiple)) * multiple)
    return min(e, tile_w) if tile_w else e
