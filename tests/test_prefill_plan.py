"""Host-side checks of the tensor-core path's launch plan (no GPU needed).

bl_prefill_plan reports, for an explicit SM count, the tile geometry and how
many tiles run whole (one CTA each) and how many are shared out in k-stages in
a balanced last round.  These tests pin the decisions measured on a 148-SM
B200 and the invariants the kernel's unit partition relies on.
"""
import ctypes

import pytest


@pytest.fixture(scope="module")
def L():
    from bit_weight_linear_b200 import build as b
    b.build()
    import bit_weight_linear_b200 as blw
    return blw.lib()


def plan(L, form, M, K, N, sms=148):
    out = (ctypes.c_int * 5)()
    st = L.bl_prefill_plan(form, M, K, N, sms, out)
    assert st == 0, st
    return dict(bt=out[0], stages=out[1], tiles=out[2], whole=out[3], shared=out[4])


def test_70b_prefill_plans(L):
    # 128 tiles fill one round of 148 SMs with 20 idle: sharing them costs more
    # than it saves, so they run whole
    assert plan(L, 0, 512, 8192, 8192) == dict(bt=256, stages=64, tiles=128, whole=128, shared=0)
    assert plan(L, 0, 512, 28672, 8192) == dict(bt=256, stages=224, tiles=128, whole=128, shared=0)
    # 448 tiles = 3.03 rounds: two rounds whole, the last 152 tiles shared out
    assert plan(L, 0, 512, 8192, 28672) == dict(bt=256, stages=64, tiles=448, whole=296, shared=152)


def test_small_token_counts_share_few_tiles(L):
    # 13B-shaped 13824->5120: 40 tiles of 32 activation rows, four 128-k blocks
    # per stage; shared out over all SMs at any small M
    for M in (9, 16, 64):
        p = plan(L, 0, M, 13824, 5120)
        assert (p["bt"], p["stages"], p["tiles"], p["whole"], p["shared"]) == \
            ({9: 32, 16: 32, 64: 64}[M], 27, 40, 0, 40)
    # OneBit triples the activation rows (three limbs per token)
    assert plan(L, 1, 10, 13824, 5120)["bt"] == 32
    assert plan(L, 1, 16, 13824, 5120)["bt"] == 64
    assert plan(L, 1, 64, 13824, 5120)["bt"] == 192
    # 108 tiles of a 5120->13824 layer stay whole at M = 16
    assert plan(L, 0, 16, 5120, 13824)["shared"] == 0


def test_tile_geometry(L):
    # tokens cut into the fewest tiles of at most 256 activation rows, of
    # balanced size; activation rows per tile: the smallest multiple of 32
    # covering a tile's tokens; k-blocks per stage 4 / 2 / 1 for <= 64 / <= 128 / more
    for M, bt, kb in [(9, 32, 4), (33, 64, 4), (100, 128, 2), (129, 160, 1), (300, 160, 1),
                      (512, 256, 1), (513, 192, 1), (1024, 256, 1)]:
        p = plan(L, 0, M, 4096, 4096)
        assert p["bt"] == bt
        assert p["stages"] == (4096 // 128 + kb - 1) // kb
        assert p["tiles"] == (4096 // 128) * ((M + bt - 1) // bt)


def test_onebit_tile_geometry(L):
    # OneBit: three limb rows per token, at most 85 tokens (255 rows) per
    # tile, the token tiles balanced; a tile never splits a token's limbs
    for M, ttiles in [(5, 1), (10, 1), (11, 1), (85, 1), (86, 2), (256, 4), (512, 7), (1024, 13)]:
        tpt = -(-M // ttiles)
        assert tpt <= 85
        p = plan(L, 1, M, 5120, 13824)
        assert p["bt"] == min(256, -(-3 * tpt // 32) * 32), M
        assert p["tiles"] == (13824 // 128) * ttiles, M


@pytest.mark.parametrize("sms", [148, 132, 64, 7, 1])
def test_plan_invariants(L, sms):
    """Whole and shared tiles partition the tiles; the whole ones fill whole
    rounds; the balanced round has at least one SM's worth of tiles (fewer only
    when all tiles fit one round) and at least four stages per CTA, so no CTA
    of it is empty; a launch with tiles filling whole rounds is never split."""
    seen_split = False
    for form in (0, 1):
        for M in (9, 16, 40, 100, 256, 512, 1024):
            for K in (1024, 4096, 13824, 28672):
                for N in (1024, 5120, 8192, 13824, 28672):
                    p = plan(L, form, M, K, N, sms)
                    assert p["whole"] + p["shared"] == p["tiles"]
                    if p["tiles"] % sms == 0:
                        assert p["shared"] == 0
                    if p["shared"] == 0:
                        continue
                    seen_split = True
                    assert p["whole"] % sms == 0
                    assert p["shared"] >= sms or (p["whole"] == 0 and p["shared"] == p["tiles"])
                    assert p["shared"] < 2 * sms
                    assert p["shared"] * p["stages"] >= 4 * sms
    assert seen_split or sms == 1


def test_plan_rejects_bad_arguments(L):
    out = (ctypes.c_int * 5)()
    assert L.bl_prefill_plan(0, 16, 4096, 4096, 148, None) == 1      # BL_ERR_NULL
    assert L.bl_prefill_plan(2, 16, 4096, 4096, 148, out) == 2       # bad form
    assert L.bl_prefill_plan(0, 16, 100, 4096, 148, out) == 2        # bad K
    assert L.bl_prefill_plan(0, 16, 4096, 24, 148, out) == 2         # bad N
    assert L.bl_prefill_plan(0, 0, 4096, 4096, 148, out) == 2        # M = 0
    assert L.bl_prefill_plan(0, 16, 4096, 4096, 0, out) == 2         # no SMs
