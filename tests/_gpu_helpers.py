"""Shared helpers for the GPU parity tests: moving bf16 bit patterns to and from
the device, turning the device TwELL into NumPy, and the comparison rules."""
import numpy as np
import torch

import oracle as O

Y_REL_L2 = 2e-3     # y tolerance against the fp64 oracle (before its bf16 rounding)
Y_MAX_ABS = 3e-2


def dev(bits):
    """np.uint16 bf16 bits -> CUDA bfloat16 tensor."""
    if bits is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def twell_to_np(a):
    """Device TwELL -> oracle.TwELL (n_ovf taken from the device word)."""
    n = int(a.n_ovf.item())
    n_keep = min(n, a.ovf_capacity)
    return O.TwELL(a.M, a.d_ff, a.tile_w, a.ell_w,
                   host_bits(a.vals), a.idx.cpu().numpy(),
                   a.nnz.view(torch.int16).cpu().numpy().view(np.uint16),
                   a.ovf_pos[:n_keep].cpu().numpy().astype(np.int32),
                   host_bits(a.ovf_dense[:n_keep])), n


def assert_twell_equal(got, ref, rows=None):
    """Bitwise equality of every TwELL field (optionally only for some rows)."""
    sel = slice(None) if rows is None else rows
    assert np.array_equal(got.nnz[sel], ref.nnz[sel]), "nnz differs"
    assert np.array_equal(got.idx[sel], ref.idx[sel]), "idx differs"
    assert np.array_equal(got.vals[sel], ref.vals[sel]), "vals differs"
    if rows is None:
        assert got.n_ovf == ref.n_ovf, f"n_ovf {got.n_ovf} != {ref.n_ovf}"
        assert np.array_equal(got.ovf_pos, ref.ovf_pos), "ovf_pos differs"
        assert np.array_equal(got.ovf_dense, ref.ovf_dense), "ovf_dense differs"


def assert_twell_valid(a):
    """Structural invariants of any TwELL (used where no oracle copy exists)."""
    M, T, E = a.vals.shape
    nnz = a.nnz.astype(np.int64)
    pad = np.arange(E)[None, None, :] >= np.minimum(nnz, E)[:, :, None]
    assert np.all(a.vals[pad] == 0) and np.all(a.idx[pad] == 0), "padding slots not (+0, 0)"
    assert np.all((a.vals[~pad] & 0x7FFF) != 0), "stored zero in a live slot"
    assert np.all(a.idx.astype(np.int64) < a.tile_w)
    both = ~pad[:, :, 1:] & ~pad[:, :, :-1]
    assert np.all(a.idx[:, :, 1:][both] > a.idx[:, :, :-1][both]), "slots not ascending"
    assert np.all(np.diff(a.ovf_pos) > 0), "backup not ascending"
    assert a.n_ovf == int((nnz > E).sum()), "n_ovf != #pairs over the ELL width"
    r, t = np.divmod(a.ovf_pos.astype(np.int64), T)
    assert np.all(nnz[r, t] > E)
    # the slots of an overflowing pair are the first E nonzeros of its segment
    seg = a.ovf_dense
    for k in range(min(a.n_ovf, 64)):
        nzp = np.nonzero(seg[k] & 0x7FFF)[0]
        assert len(nzp) == nnz[r[k], t[k]]
        assert np.array_equal(a.idx[r[k], t[k]], nzp[:E].astype(np.uint8))
        assert np.array_equal(a.vals[r[k], t[k]], seg[k][nzp[:E]])


def y_errors(y_gpu, y_ref):
    """(relative L2 error, max abs error beyond the output-rounding allowance).

    The absolute bound 3e-2 is met by any correct bf16 result only while |y| < 8
    (half a bf16 ulp is 2^-9 |y|); where |y_ref| is larger, one bf16 ulp of y_ref
    is allowed instead, so the bound never asks for more than bf16 can store."""
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    diff = np.abs(yg - y_ref)
    nrm = np.linalg.norm(y_ref)
    rel = np.linalg.norm(diff) / nrm if nrm > 0 else (0.0 if np.all(yg == 0) else np.inf)
    allow = np.maximum(Y_MAX_ABS, 2.0 ** -8 * np.abs(y_ref))
    excess = float(np.max(diff - allow + Y_MAX_ABS)) if diff.size else 0.0
    return rel, excess


def assert_y_close(y_gpu, y_ref):
    rel, mx = y_errors(y_gpu, y_ref)
    if np.linalg.norm(y_ref) == 0:
        assert np.all(y_gpu.float().cpu().numpy() == 0), "y must be exactly 0"
        return
    assert rel <= Y_REL_L2 and mx <= Y_MAX_ABS, f"rel_l2={rel:.3e} max_abs={mx:.3e}"


def upload_twell(ref, cap=None):
    """Oracle TwELL -> device TwELL (to test the consumer in isolation)."""
    import activation_sparse_ffn_twell_b200 as T
    cap = ref.n_ovf if cap is None else cap
    a = T.TwELL.allocate(ref.M, ref.d_ff, ref.tile_w, ref.ell_w, cap)
    a.vals.copy_(dev(ref.vals))
    a.idx.copy_(torch.from_numpy(ref.idx).cuda())
    a.nnz.copy_(torch.from_numpy(ref.nnz.view(np.int16)).cuda())
    a.n_ovf.fill_(ref.n_ovf)
    if ref.n_ovf:
        a.ovf_pos[:ref.n_ovf].copy_(torch.from_numpy(ref.ovf_pos).cuda())
        a.ovf_dense[:ref.n_ovf].copy_(dev(ref.ovf_dense))
    a.status.zero_()
    return a


def h_from_zdebug(z, b_bits, w_gate_present, f):
    """Replay the epilogue's fp32 arithmetic on the GPU's own accumulators:
    v = max(fp32(acc + b), 0) [ * up, one fp32 multiply ], then one bf16 rounding."""
    z = z.astype(np.float32)
    b = (O.bits_to_f64(b_bits).astype(np.float32) if b_bits is not None
         else np.zeros(f, dtype=np.float32))
    if w_gate_present:
        g, u = z[:, :f], z[:, f:]
        v = np.maximum(g + b[None, :], np.float32(0)) * u
    else:
        v = np.maximum(z + b[None, :], np.float32(0))
    h = O.bf16_round(v.astype(np.float64))
    return np.where(h == 0.0, 0.0, h)
