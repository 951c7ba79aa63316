"""twell_pack_noalloc: the packer for callers that cannot allocate device memory
when they pack (a runtime that reserved the whole GPU up front and forbids
cudaMalloc on its request path, or a plugin host that hands over only input and
output buffers).  It keeps its scratch in a fixed device array inside the
library instead of a caller workspace.

The test calls it through the C ABI twice in a row and checks each result
against twell_pack (which takes a workspace), bit for bit -- the tolerance every
packing test here uses.  The second call has fewer overflowing pairs than the
first, so scratch contents left over from the first call would show up.  This
file is collected last so a stop-at-first-failure run has already run the rest."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu


def _compare(a, b):
    n_a, n_b = int(a.n_ovf.item()), int(b.n_ovf.item())
    assert n_a == n_b
    assert torch.equal(a.nnz, b.nnz)
    assert torch.equal(a.vals.view(torch.int16), b.vals.view(torch.int16))
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.ovf_pos[:n_a], b.ovf_pos[:n_b])
    assert torch.equal(a.ovf_dense[:n_a].view(torch.int16), b.ovf_dense[:n_b].view(torch.int16))
    assert int(a.status.item()) == int(b.status.item()) == 0


def test_pack_noalloc_matches_pack_on_two_calls_in_a_row():
    import activation_sparse_ffn_twell_b200 as T
    L = T.lib()
    cases = [(300, 1024, 128, 8, 0.30, 1), (200, 1024, 128, 16, 0.05, 2)]   # many, then few overflows
    n_seen = []
    for M, f, tw, E, rho, seed in cases:
        lay = S.small_random(M, 64, f, tw, E, rho, seed=seed)
        h_bits = O.f64_to_bits(O.hidden(lay.x, lay.w_up, lay.b))
        h = torch.from_numpy(h_bits.view(np.int16)).view(torch.bfloat16).cuda()
        cap = M * (f // tw)          # room for every pair: the lists are fully defined
        ref = T.twell_pack(h, tw, E, ovf_capacity=cap)
        got = T.TwELL.allocate(M, f, tw, E, cap)
        m = got.cstruct()
        code = L.twell_pack_noalloc(h.data_ptr(), M, f, f, tw, E, ctypes.byref(m),
                                    torch.cuda.current_stream().cuda_stream)
        assert code == 0
        torch.cuda.synchronize()
        _compare(got, ref)
        n_seen.append(int(got.n_ovf.item()))
    assert n_seen[0] > n_seen[1]


def test_pack_noalloc_rejects_problems_beyond_its_scratch():
    import activation_sparse_ffn_twell_b200 as T
    L = T.lib()
    M, f, tw, E = 4096, 8192, 128, 16
    a = T.TwELL.allocate(M, f, tw, E, 20000)    # 20000 * 260 B > 4 MiB
    h = torch.zeros((M, f), dtype=torch.bfloat16, device="cuda")
    m = a.cstruct()
    code = L.twell_pack_noalloc(h.data_ptr(), M, f, f, tw, E, ctypes.byref(m),
                                torch.cuda.current_stream().cuda_stream)
    assert code == 6   # TWELL_ERR_WORKSPACE, nothing enqueued
