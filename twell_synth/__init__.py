"""Seeded synthetic inputs for the activation-sparse ReLU FFN layer.

This module only *draws* inputs: activations x, weights W_up / W_gate / W_down,
the per-neuron bias b and the TwELL shape parameters (tile_w, ell_w).  It holds
none of the layer's arithmetic (no matmul, no ReLU, no packing); both the CUDA
path and the CPU oracle consume what it returns.

Everything is returned as bf16 *bit patterns* (``numpy.uint16``) so that both
sides see exactly the same values.  The draws follow the workloads described
in "Sparser, Faster, Lighter Transformer Language Models" (Sakana AI / NVIDIA,
news pages: upppp.jp 2026-05-11, section on real-world gains; innovatopia.jp,
editorial notes): ReLU FFN layers of 0.5B-2B models at 1-20 % activation
density, plus a heavy-tailed per-token density (a few tokens activate far more
neurons than the mean).  No trained weights or datasets are involved: weights
are N(0, 1/fan_in) and the density is set through the bias, using the normal
quantile of each neuron's exact pre-activation standard deviation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
from scipy.special import ndtri
from scipy.stats import binom

__all__ = [
    "FFNInputs",
    "bf16_bits_from_f32",
    "bf16_bits_to_f32",
    "ell_width_rule",
    "tiny_relu",
    "relu_15b",
    "gated_2b",
    "heavy_tail",
    "decode",
    "integer_exact",
    "small_random",
    "TARGET_DENSITIES_15B",
]

TARGET_DENSITIES_15B = (0.20, 0.10, 0.05, 0.01)


# ---------------------------------------------------------------------------
# bf16 bit helpers (input quantisation only)
# ---------------------------------------------------------------------------
def bf16_bits_from_f32(a) -> np.ndarray:
    """Round finite float32 values to bf16 (round-to-nearest-even); return bits."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
@dataclasses.dataclass
class FFNInputs:
    """One synthetic FFN layer problem (all arrays are bf16 bit patterns)."""

    name: str
    M: int
    d_model: int
    d_ff: int
    tile_w: int
    ell_w: int
    gated: bool
    x: np.ndarray                 # [M, d_model]
    w_up: np.ndarray              # [d_ff, d_model]  (nn.Linear(d_model, d_ff).weight layout)
    w_gate: Optional[np.ndarray]  # [d_ff, d_model] or None
    b: Optional[np.ndarray]       # [d_ff] (gate bias when gated) or None
    w_down: np.ndarray            # [d_ff, d_model]  row j = neuron j's output vector
    target_density: float
    meta: dict = dataclasses.field(default_factory=dict)

    @property
    def n_tiles(self) -> int:
        return self.d_ff // self.tile_w

    def describe(self) -> dict:
        d = dict(name=self.name, M=self.M, d_model=self.d_model, d_ff=self.d_ff,
                 tile_w=self.tile_w, ell_w=self.ell_w, gated=self.gated,
                 target_density=self.target_density)
        d.update({k: v for k, v in self.meta.items() if np.isscalar(v) or isinstance(v, (str, int, float))})
        return d


# ---------------------------------------------------------------------------
def ell_width_rule(tile_w: int, token_densities, pct: float = 0.99, multiple: int = 8) -> int:
    """ELL width: smallest multiple of 8 >= the nearest-rank 99th percentile of
    the per-(token, tile) nonzero count, modelled as Binomial(tile_w, rho_r) for
    a token of density rho_r (a mixture over tokens when densities differ).

    This is an input *parameter* computed from the target densities alone; it
    never looks at a computed hidden activation.
    """
    rho = np.atleast_1d(np.asarray(token_densities, dtype=np.float64))
    ks = np.arange(tile_w + 1)
    cdf = np.mean(binom.cdf(ks[None, :], tile_w, np.clip(rho, 0.0, 1.0)[:, None]), axis=0)
    k99 = int(np.argmax(cdf >= pct - 1e-12))
    e = max(multiple, int(math.ceil(k99 / multiple)) * multiple)
    return min(e, tile_w)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return bf16_bits_from_f32(a)


def _row_norms(w_bits: np.ndarray, cols: Optional[slice] = None) -> np.ndarray:
    """sigma_j = ||W[j, :]||_2 in fp64 over the bf16 weights: the exact standard
    deviation of x . W[j] for x ~ N(0, I)."""
    w = bf16_bits_to_f32(w_bits if cols is None else w_bits[:, cols]).astype(np.float64)
    return np.sqrt(np.einsum("ij,ij->i", w, w))


def _bias_for_density(sigma: np.ndarray, rho: float) -> np.ndarray:
    """b_j = bf16(-Phi^-1(1 - rho) * sigma_j): P(x.W_j + b_j > 0) = rho."""
    q = float(ndtri(1.0 - rho))
    return bf16_bits_from_f32((-q * sigma).astype(np.float32))


# ---------------------------------------------------------------------------
# The five workload families
# ---------------------------------------------------------------------------
def tiny_relu(seed: int = 0) -> FFNInputs:
    """Tiny non-gated layer: M=64, d_model=256, d_ff=1024, ~10 % density,
    tile_w=64, ell_w=16; x~N(0,1), W_up~N(0,1/256), W_down~N(0,1/1024)."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    M, d, f = 64, 256, 1024
    x = _normal_bf16(rng, (M, d), 1.0)
    w_up = _normal_bf16(rng, (f, d), 1.0 / math.sqrt(d))
    w_down = _normal_bf16(rng, (f, d), 1.0 / math.sqrt(f))
    b = _bias_for_density(_row_norms(w_up), 0.10)
    return FFNInputs("tiny_relu", M, d, f, 64, 16, False, x, w_up, None, b, w_down, 0.10,
                     dict(seed=seed))


def relu_15b(density: float = 0.05, M: int = 4096, d_model: int = 2048, d_ff: int = 8192,
             tile_w: int = 128, seed: int = 0, ell_w: Optional[int] = None) -> FFNInputs:
    """1.5B-scale non-gated ReLU FFN layer (M=4096, 2048 -> 8192), weights
    N(0, 1/fan_in), bias from the normal quantile for the target density."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    x = _normal_bf16(rng, (M, d_model), 1.0)
    w_up = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_model))
    w_down = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_ff))
    b = _bias_for_density(_row_norms(w_up), density)
    e = ell_w if ell_w is not None else ell_width_rule(tile_w, [density])
    return FFNInputs(f"relu_15b_rho{density:g}", M, d_model, d_ff, tile_w, e, False,
                     x, w_up, None, b, w_down, density, dict(seed=seed))


def gated_2b(density: float = 0.05, M: int = 8192, d_model: int = 2560, d_ff: int = 10240,
             tile_w: int = 128, seed: int = 0, ell_w: Optional[int] = None) -> FFNInputs:
    """2B-scale gated ReLU FFN: h = ReLU(x W_g^T + b) * (x W_u^T); the gate bias
    sets the density; the up branch has no bias."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    x = _normal_bf16(rng, (M, d_model), 1.0)
    w_gate = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_model))
    w_up = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_model))
    w_down = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_ff))
    b = _bias_for_density(_row_norms(w_gate), density)
    e = ell_w if ell_w is not None else ell_width_rule(tile_w, [density])
    return FFNInputs(f"gated_2b_rho{density:g}", M, d_model, d_ff, tile_w, e, True,
                     x, w_up, w_gate, b, w_down, density, dict(seed=seed))


def heavy_tail(M: int = 8192, d_model: int = 2048, d_ff: int = 8192, tile_w: int = 128,
               mean_density: float = 0.03, sigma_ln: float = 1.0, dense_frac: float = 0.01,
               dense_mult: float = 100.0, seed: int = 0, ell_w: Optional[int] = None) -> FFNInputs:
    """Heavy-tailed per-token density.

    Token r gets density rho_r ~ LogNormal(mean 3 %, sigma_ln) capped at 1, and
    1 % of tokens (chosen by the seed) get min(100 x mean, 1).  The per-token
    shift enters through a reserved input feature: W_up[j, d-1] = sigma'_j,
    x[r, d-1] = s_r, b_j = -c sigma'_j with c = Phi^-1(0.97), so that
    z_j / sigma'_j ~ N(s_r - c, 1) and s_r = c - Phi^-1(1 - rho_r) gives density
    rho_r (Phi^-1(0) is taken as -8: every neuron on).
    """
    rng = np.random.default_rng(np.random.PCG64(seed))
    d = d_model
    xg = rng.standard_normal(size=(M, d), dtype=np.float32)
    w = rng.standard_normal(size=(d_ff, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d))
    w_down = _normal_bf16(rng, (d_ff, d), 1.0 / math.sqrt(d_ff))
    mu = math.log(mean_density) - 0.5 * sigma_ln ** 2
    rho = np.minimum(np.exp(mu + sigma_ln * rng.standard_normal(M)), 1.0)
    n_dense = int(round(dense_frac * M))
    dense_rows = rng.choice(M, size=n_dense, replace=False)
    rho[dense_rows] = min(dense_mult * mean_density, 1.0)
    c = float(ndtri(0.97))
    q = np.where(rho >= 1.0, -8.0, ndtri(np.clip(1.0 - rho, 1e-300, 1.0)))
    s = c - q
    w_up = bf16_bits_from_f32(w)
    sig = _row_norms(w_up, slice(0, d - 1))
    w_up[:, d - 1] = bf16_bits_from_f32(sig.astype(np.float32))
    x = bf16_bits_from_f32(xg)
    x[:, d - 1] = bf16_bits_from_f32(s.astype(np.float32))
    b = bf16_bits_from_f32((-c * sig).astype(np.float32))
    mask = np.ones(M, dtype=bool)
    mask[dense_rows] = False
    e = ell_w if ell_w is not None else ell_width_rule(tile_w, rho[mask])
    meta = dict(seed=seed, sigma_ln=sigma_ln, mean_density=mean_density,
                effective_density=float(rho.mean()), n_dense_tokens=n_dense)
    out = FFNInputs("heavy_tail", M, d, d_ff, tile_w, e, False, x, w_up, None, b, w_down,
                    float(rho.mean()), meta)
    out.meta["token_density"] = rho
    out.meta["dense_rows"] = np.sort(dense_rows)
    return out


def decode(M: int = 128, d_model: int = 4096, d_ff: int = 16384, tile_w: int = 128,
           density: float = 0.02, seed: int = 0, ell_w: Optional[int] = None) -> FFNInputs:
    """Decode-like small batch (M in {32, 128, 256}), 4096 -> 16384, 2 % density."""
    r = relu_15b(density=density, M=M, d_model=d_model, d_ff=d_ff, tile_w=tile_w, seed=seed,
                 ell_w=ell_w)
    r.name = f"decode_M{M}"
    return r


def integer_exact(M: int, d_model: int, d_ff: int, tile_w: int = 128, density: float = 0.05,
                  gated: bool = False, seed: int = 0, ell_w: Optional[int] = None,
                  p_nonzero: float = 2.0 / 3.0) -> FFNInputs:
    """Integer-exact family: x, W in {-1, 0, +1}, integer bias.

    Every product and partial sum of the layer is an integer below 2^24, so
    fp32 accumulation in any order is exact and the whole layer (hidden bf16
    values, TwELL, and y) is bit-reproducible against an fp64 evaluation.
    """
    rng = np.random.default_rng(np.random.PCG64(seed))

    def tern(shape, p):
        v = rng.choice(np.array([-1.0, 0.0, 1.0], dtype=np.float32), size=shape,
                       p=[p / 2, 1.0 - p, p / 2])
        return bf16_bits_from_f32(v)

    pw = p_nonzero if not gated else p_nonzero / 2
    x = tern((M, d_model), p_nonzero)
    w_up = tern((d_ff, d_model), pw)
    w_gate = tern((d_ff, d_model), pw) if gated else None
    w_down = tern((d_ff, d_model), p_nonzero)
    sd = math.sqrt(d_model * p_nonzero * pw)
    q = float(ndtri(1.0 - density))
    b = bf16_bits_from_f32(np.full(d_ff, -round(q * sd), dtype=np.float32))
    e = ell_w if ell_w is not None else ell_width_rule(tile_w, [density])
    return FFNInputs(f"integer_M{M}_d{d_model}_f{d_ff}{'_gated' if gated else ''}", M, d_model,
                     d_ff, tile_w, e, gated, x, w_up, w_gate, b, w_down, density,
                     dict(seed=seed, integer=True))


def small_random(M: int, d_model: int, d_ff: int, tile_w: int, ell_w: int, density: float,
                 gated: bool = False, seed: int = 0, with_bias: bool = True) -> FFNInputs:
    """Gaussian layer of arbitrary (small) shape for ragged / edge-case tests."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    x = _normal_bf16(rng, (M, d_model), 1.0)
    w_up = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_model))
    w_gate = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_model)) if gated else None
    w_down = _normal_bf16(rng, (d_ff, d_model), 1.0 / math.sqrt(d_ff))
    src = w_gate if gated else w_up
    if not with_bias:
        b = None
    elif density <= 0.0:
        b = bf16_bits_from_f32(np.full(d_ff, -1.0e4, dtype=np.float32))
    elif density >= 1.0:
        # +6 sigma: every pre-activation is positive (P < 1e-9 otherwise) while h,
        # and therefore y, stay O(1)
        b = bf16_bits_from_f32((6.0 * _row_norms(src)).astype(np.float32))
    else:
        b = _bias_for_density(_row_norms(src), density)
    return FFNInputs(f"small_M{M}_d{d_model}_f{d_ff}_tw{tile_w}_E{ell_w}", M, d_model, d_ff,
                     tile_w, ell_w, gated, x, w_up, w_gate, b, w_down, density, dict(seed=seed))
