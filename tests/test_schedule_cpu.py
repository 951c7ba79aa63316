"""The work split of the token-major tensor-core down-projection, checked on the
host through the library's own planning and scheduling code
(twell_down_schedule compiles the kernel's schedule helpers for the host too).

For every shape and SM count below:
* every (tile, K step) is computed by exactly one CTA;
* a whole tile is one segment [0, K steps) with no sharing state;
* the segments of a shared tile agree on the number of sharers and on one
  arrival counter, no two shared tiles use the same counter, and every shared
  segment publishes its partial tile in a slot of its own, inside the
  workspace's 2 x 160 slots;
* the CTAs get the same number of K steps up to one chunk (whole tiles: up to
  one tile); a split never uses more than min(SMs, 160) CTAs;
* the choice of schedule: whole tiles when they fill whole waves, split-K when
  there are fewer tiles than SMs and enough K steps, an even deal when it is
  shorter than the whole-tile waves.
No GPU is needed and nothing is launched.
"""
import collections

import pytest

SHAPES = [
    # M, d_model, d_ff, tile_w, ell_w
    (4096, 2048, 8192, 128, 16),     # 1.5B layer: 128 tiles, whole
    (2048, 2048, 8192, 128, 16),     # 64 tiles: split-K two ways
    (384, 512, 8192, 128, 16),       # 3 tiles: split-K four ways
    (8192, 2560, 10240, 128, 16),    # gated 2B: 320 tiles, even deal
    (8192, 2048, 8192, 128, 24),     # heavy tail: 256 tiles, even deal
    (4736, 2048, 8192, 128, 16),     # 148 tiles: one whole wave
    (700, 768, 4096, 64, 8),         # ragged M and d_model
    (520, 640, 4096, 32, 8),         # tile_w 32
    (400, 1024, 4096, 256, 24),      # tile_w 256
    (4864, 2048, 3072, 128, 16),     # 152 tiles of 48 K steps: whole
    (8192, 2048, 4096, 128, 16),     # 256 tiles of 64 K steps: whole
    (16384, 4096, 16384, 128, 16),   # 1024 tiles
    (300, 320, 2048, 128, 16),       # few K steps: whole tiles
]
SMS = [148, 132, 160, 114, 200]


@pytest.fixture(scope="module")
def T():
    from activation_sparse_ffn_twell_b200 import build
    build.build()
    import activation_sparse_ffn_twell_b200 as T
    return T


@pytest.mark.parametrize("sms", SMS)
@pytest.mark.parametrize("M,d,f,tw,E", SHAPES)
def test_schedule_covers_each_k_step_once(T, M, d, f, tw, E, sms):
    s = T.down_schedule(M, d, f, tw, E, sms)
    assert s is not None
    tiles, K, ctas = s["tiles"], s["k_steps"], s["ctas"]
    assert tiles == ((M + 127) // 128) * ((d + 511) // 512)
    assert K == (f + 63) // 64
    assert 1 <= ctas <= (min(sms, 160) if s["split"] else sms)
    owner = {}
    steps = collections.Counter()
    by_tile = collections.defaultdict(list)
    for cta, tile, k0, k1, n, ctr, slot in s["segments"]:
        assert 0 <= cta < ctas and 0 <= tile < tiles and 0 <= k0 < k1 <= K
        for k in range(k0, k1):
            assert (tile, k) not in owner, (tile, k)
            owner[(tile, k)] = cta
        steps[cta] += k1 - k0
        by_tile[tile].append((cta, k0, k1, n, ctr, slot))
    assert len(owner) == tiles * K
    slots, ctrs = set(), set()
    for tile, segs in by_tile.items():
        if len(segs) == 1 and segs[0][1:3] == (0, K):
            assert segs[0][3:] == (1, -1, -1)
            continue
        ns = {g[3] for g in segs}
        cs = {g[4] for g in segs}
        assert ns == {len(segs)} and len(segs) >= 2
        assert len(cs) == 1 and 0 <= next(iter(cs)) < 160
        assert next(iter(cs)) not in ctrs
        ctrs |= cs
        assert len({g[0] for g in segs}) == len(segs)       # distinct CTAs
        for g in segs:
            assert 0 <= g[5] < 320 and g[5] not in slots
            slots.add(g[5])
    # balance: equal K steps per CTA up to one chunk (whole-tile schedules: up to one tile)
    ck = tw // 64 if tw > 64 else 1
    spread = max(steps.values()) - min(steps.values())
    if s["split"] == 0:
        assert spread in (0, K)
    else:
        assert spread <= ck * (2 if s["split"] == 1 else 1), (spread, ck)


def test_schedule_choice(T):
    assert T.down_schedule(4096, 2048, 8192, 128, 16, 148)["split"] == 0        # 128 tiles
    assert T.down_schedule(4736, 2048, 8192, 128, 16, 148)["split"] == 0        # a whole wave
    s = T.down_schedule(2048, 2048, 8192, 128, 16, 148)
    assert s["split"] == 1 and s["ctas"] == 128                                # 64 tiles x 2
    s = T.down_schedule(384, 512, 8192, 128, 16, 148)
    assert s["split"] == 1 and s["ctas"] == 12                                 # 3 tiles x 4
    assert T.down_schedule(8192, 2560, 10240, 128, 16, 148)["split"] == 2
    assert T.down_schedule(8192, 2048, 8192, 128, 24, 148)["split"] == 2        # heavy tail: 128 K steps
    # 256 tiles of 64 K steps (the backward's weight-gradient products): whole tiles
    assert T.down_schedule(8192, 2048, 4096, 128, 16, 148)["split"] == 0
    assert T.down_schedule(300, 320, 2048, 128, 16, 148)["split"] == 0          # 32 K steps
    assert T.down_schedule(8192, 2560, 10240, 128, 16, 160)["split"] == 0      # two whole waves
    assert T.down_schedule(21760, 1024, 4096, 128, 16, 200)["split"] == 0      # 340 tiles: deal not shorter
    assert T.down_schedule(256, 2048, 8192, 128, 16, 148) is None               # decode-size kernel
    assert T.down_schedule(4096, 2048, 8192, 96, 16, 148) is None               # invalid tile_w
