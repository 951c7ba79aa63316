"""GPU parity of the split schedules of the tensor-core down-projection.

With 128-token x 512-column tiles the tile count rarely matches the SM count.
With fewer tiles than SMs each tile's K steps are cut into equal ranges taken
by different CTAs (split-K); with more (and not whole waves), every tile's K
steps, in hidden-tile chunks, are dealt out evenly over the SMs.  A
tile shared by several CTAs is summed from their fp32 partial tiles, in K
order, by the last one to finish.  The cases are chosen so that tiles really
are shared (checked on the host with the same rules), including four-way
splits, ragged M and d_model, every tile width, ell_w with and without the TMA
slot ring, overflowing pairs whose row starts a segment mid-row, more tiles
than SMs, and the AUTO path with blocks on both down kernels.

* Gaussian layers: y within the oracle tolerance (rel-L2 2e-3, max-abs 3e-2).
* Integer-exact layers: every partial sum is an integer below 2^24, so y must
  equal the oracle's bits whatever the split.
* Two runs give identical bits (the partials are added in a fixed order), and a
  CUDA-graph replay gives the eager call's bits (the arrival counters are reset
  inside the captured sequence).
"""
import numpy as np
import pytest
import torch

import oracle as O
import twell_synth as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import activation_sparse_ffn_twell_b200 as T
    from _gpu_helpers import assert_y_close, dev, host_bits, twell_to_np, upload_twell

MIN_SPLIT_STEPS = 32     # K steps per CTA at least
MAX_SPLIT_CTAS = 160
MIN_DEAL_STEPS = 128     # K steps per tile for the even deal


def _shared_tiles(M, d, f, tw):
    """{tile: contributing CTAs} for the shared tiles under the library's rules
    (a host restatement used only to confirm that a case exercises sharing)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    g = min(sms, MAX_SPLIT_CTAS)
    tiles = ((M + 127) // 128) * ((d + 511) // 512)
    num_kb = (f + 63) // 64
    ck = tw // 64 if tw > 64 else 1
    nc = (num_kb + ck - 1) // ck
    if tiles < g:
        parts = min(g // tiles, nc * ck // MIN_SPLIT_STEPS, nc)
        return {t: parts for t in range(tiles)} if parts >= 2 else {}
    if tiles % g == 0 or num_kb < MIN_DEAL_STEPS:
        return {}
    U = tiles * nc
    sk = max(1, min(g, U * ck // MIN_SPLIT_STEPS))
    owner = lambda q: ((q + 1) * sk + U - 1) // U - 1
    return {t: owner((t + 1) * nc - 1) - owner(t * nc) + 1 for t in range(tiles)
            if owner((t + 1) * nc - 1) > owner(t * nc)}


CASES = [
    # M, d, f, tw, E, rho
    (384, 512, 8192, 128, 16, 0.05),     # 3 tiles, split four ways
    (768, 1024, 8192, 128, 16, 0.05),    # 12 tiles, split four ways
    (700, 768, 4096, 64, 8, 0.15),       # ragged M and d_model; many overflowing pairs
    (520, 640, 4096, 32, 8, 0.10),       # tile_w 32: a chunk is one K step (two hidden tiles)
    (400, 1024, 4096, 256, 24, 0.05),    # tile_w 256: K steps claimed in groups of 3
    (600, 768, 4608, 128, 16, 0.05),     # T = 36 not a multiple of 8: slots fetched per thread
    (4864, 2048, 8192, 128, 16, 0.05),   # 152 tiles of 128 K steps: every tile's chunks dealt over 148 CTAs
]


@pytest.mark.parametrize("mode", ["mma", "auto"])
@pytest.mark.parametrize("M,d,f,tw,E,rho", CASES)
def test_split_spmm_against_oracle(M, d, f, tw, E, rho, mode):
    assert _shared_tiles(M, d, f, tw), "case does not share any tile"
    L = S.small_random(M, d, f, tw, E, rho, seed=M + d + f)
    h = O.hidden(L.x, L.w_up, L.b)
    ref = O.twell_pack(h, tw, E)
    y_ref = O.twell_spmm(ref, L.w_down)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    wd = dev(L.w_down)
    y = T.twell_spmm(a, wd, mode=mode)
    assert T.read_status(a)[0] == 0
    assert_y_close(y, y_ref)
    y2 = T.twell_spmm(a, wd, mode=mode)          # fixed summation order
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M,d,f", [(896, 1024, 4096), (4864, 2048, 8192)])
def test_split_mixed_paths_auto(M, d, f):
    """AUTO with some 128-token blocks below the gather crossover: the split
    schedules skip the gather-owned tiles and the shared ones still add up."""
    tw, E = 128, 16
    assert _shared_tiles(M, d, f, tw)
    L = S.small_random(M, d, f, tw, E, 0.05, seed=11)
    h = O.hidden(L.x, L.w_up, L.b)
    h[256:512] = 0.0                 # two blocks with no activations
    h[640:768] = 0.0
    h[640:768, ::509] = 1.0          # ~0.2 % density: below the crossover
    ref = O.twell_pack(h, tw, E)
    y_ref = O.twell_spmm(ref, L.w_down)
    a = upload_twell(ref, cap=max(ref.n_ovf, 1))
    y = T.twell_spmm(a, dev(L.w_down), mode="auto")
    assert T.read_status(a)[0] == 0
    assert_y_close(y, y_ref)


@pytest.mark.parametrize("M,d,f", [(384, 512, 8192), (4864, 2048, 8192)])
def test_split_integer_family_bitexact(M, d, f):
    assert _shared_tiles(M, d, f, 128)
    L = S.integer_exact(M=M, d_model=d, d_ff=f, tile_w=128, density=0.05, seed=M + f)
    ref, y64 = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    y, a = T.twell_ffn_forward(dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down), tile_w=L.tile_w,
                               ell_w=L.ell_w, mode="mma", ovf_capacity=max(ref.n_ovf, 1))
    assert T.read_status(a) == (0, ref.n_ovf)
    assert np.array_equal(host_bits(y), O.f64_to_bits(O.bf16_round(y64)))


def test_split_forward_replays_from_a_cuda_graph():
    M, d, f, tw, E = 384, 512, 8192, 128, 16
    assert _shared_tiles(M, d, f, tw)
    L = S.small_random(M, d, f, tw, E, 0.05, seed=3)
    L2 = S.small_random(M, d, f, tw, E, 0.05, seed=4)
    x = dev(L.x)
    wu, b, wd = dev(L.w_up), dev(L.b), dev(L.w_down)
    a = T.TwELL.allocate(M, f, tw, E, M * (f // tw))
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")

    def fwd():
        T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=E, out=a, y=y)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            fwd()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    x.copy_(dev(L2.x))
    for _ in range(3):                 # the counters must be back at zero every replay
        g.replay()
    torch.cuda.synchronize()
    y_graph = y.clone()
    fwd()
    assert T.read_status(a)[0] == 0
    assert torch.equal(y_graph.view(torch.int16), y.view(torch.int16))
    ref, y64 = O.ffn_forward(L2.x, L.w_up, L.b, L.w_down, tw, E)
    assert_y_close(y_graph, y64)
    del g


def test_split_backward_dx():
    """The backward's dX = dZ W_up runs through the same down kernels: at this
    shape its 8 tiles are split two ways (64 K steps each)."""
    M, d, f, tw, E = 512, 1024, 4096, 128, 16
    assert _shared_tiles(M, d, f, tw)
    L = S.small_random(M, d, f, tw, E, 0.05, seed=21)
    rng = np.random.default_rng(5)
    dy = S.bf16_bits_from_f32(rng.standard_normal((M, d)).astype(np.float32))
    x, wu, b, wd = dev(L.x), dev(L.w_up), dev(L.b), dev(L.w_down)
    y, h = T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=E, ovf_capacity=M * (f // tw))
    assert T.read_status(h)[0] == 0
    dX, dWu, db, dWd = T.twell_ffn_backward(x, wu, wd, h, dev(dy))
    assert T.read_status(h)[0] == 0
    got, _ = twell_to_np(h)
    g = O.ffn_backward(L.x, L.w_up, L.b, L.w_down, dy, h=O.twell_unpack(got))
    for name, t in (("dx", dX), ("dw_up", dWu), ("dw_down", dWd)):
        gg = t.float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(gg - g[name]) <= 2e-3 * np.linalg.norm(g[name]), name
