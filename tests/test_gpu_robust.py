"""Failure path and capture on the GPU.

* The bounded shared-memory-barrier wait used by every tensor-core kernel gives
  up by itself on a barrier nothing arrives on, reports TWELL_ERR_TIMEOUT, and
  leaves the context usable (no fault, no hang: the wait has a wall-clock limit).
* The whole forward (reset kernel, producer, backup ordering, down kernels, chained
  as dependent launches) captures into a CUDA graph and replays to the same
  bits as eager calls, for both the token-major and the decode-size kernels.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import assert_twell_equal, dev, twell_to_np


def test_bounded_wait_gives_up_and_context_survives():
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    code = T.lib().twell_selftest_bounded_wait(ctypes.c_void_p(status.data_ptr()),
                                               ctypes.c_void_p(elapsed.data_ptr()),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0
    torch.cuda.synchronize()
    assert int(status[0].item()) == 5          # TWELL_ERR_TIMEOUT
    ns = int(elapsed[0].item())
    assert 1.0e9 <= ns <= 30.0e9, ns           # gave up at its ~2 s limit
    # the context still works: a small pack is exact afterwards
    L = S.small_random(40, 64, 256, 64, 8, 0.1, seed=4)
    h = O.hidden(L.x, L.w_up, L.b)
    ref = O.twell_pack(h, 64, 8)
    a = T.twell_pack(dev(O.f64_to_bits(h)), 64, 8, ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    got, _ = twell_to_np(a)
    assert_twell_equal(got, ref)


@pytest.mark.parametrize("M", [300, 64])
def test_forward_replays_from_a_cuda_graph(M):
    L = S.small_random(M, 256, 1024, 128, 16, 0.05, seed=M)
    L2 = S.small_random(M, 256, 1024, 128, 16, 0.05, seed=M + 1)   # new tokens, same layer
    x = dev(L.x)
    wu, b, wd = dev(L.w_up), dev(L.b), dev(L.w_down)
    a = T.TwELL.allocate(M, 1024, 128, 16, M * 8)
    y = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")

    def fwd():
        T.twell_ffn_forward(x, wu, b, wd, tile_w=128, ell_w=16, out=a, y=y)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            fwd()                      # warm caches (workspace, attributes) before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    x.copy_(dev(L2.x))
    g.replay()
    torch.cuda.synchronize()
    y_graph = y.clone()
    tw_graph, _ = twell_to_np(a)
    fwd()                              # eager on the same new tokens
    assert T.read_status(a)[0] == 0
    assert torch.equal(y_graph.view(torch.int16), y.view(torch.int16))
    tw_eager, _ = twell_to_np(a)
    assert_twell_equal(tw_graph, tw_eager)
    # and it is the new tokens' layer, within the oracle tolerance
    from _gpu_helpers import assert_y_close
    ref, y64 = O.ffn_forward(L2.x, L.w_up, L.b, L.w_down, 128, 16)
    assert_y_close(y_graph, y64)
    del g
