"""The sampling calls' work plan (host code, queried through e2d2_attn_decoder_sample_plan, no
GPU) walked the way the kernels' schedulers walk it, checked for the invariants the kernels rely
on: every key tile of every unit is taken exactly once; a CTA of the split phase meets at most
two units and so needs at most its two partial slots of the workspace, never another CTA's; the
CTA that merges a unit (the ticket arithmetic: first and last owner of the unit's tiles) sees
exactly the CTAs that wrote partials; whole units come after the split phase and are spread
evenly over every launched CTA; split ranges keep at least six tiles (or a whole unit)."""
import itertools

import numpy as np
import pytest

from block_discrete_diffusion_tcgen05_b200 import _lib, attn

MAX_CTAS = 256          # grid bound the sampling workspace is sized for (two slots per CTA)
MIN_SPLIT_TILES = 6


def range_begin(c, T, ctas):
    return (c * T) // ctas


def owner_cta(x, T, ctas):
    return ((x + 1) * ctas - 1) // T


def walk(plan):
    """The tile ranges each CTA takes: split phase first (equal contiguous ranges of the split
    units' tile stream, cut at unit boundaries), then whole units k, k + grid, ... ."""
    U, Tu, R = plan["units"], plan["tiles_per_unit"], plan["split_units"]
    sc, W, grid = plan["split_ctas"], plan["whole_units"], plan["grid"]
    T = R * Tu
    taken = np.zeros(U * Tu, dtype=np.int64)
    partial_ctas = {u: set() for u in range(R)}
    slots = set()
    for c in range(grid):
        if c < sc:
            start, end = range_begin(c, T, sc), range_begin(c + 1, T, sc)
            pos, segments = start, 0
            while pos < end:
                u = pos // Tu
                ubeg = u * Tu
                seg_end = min(end, ubeg + Tu)
                taken[pos:seg_end] += 1
                if not (pos == ubeg and seg_end == ubeg + Tu):   # a piece: writes a partial
                    slot = 2 * c if start >= ubeg else 2 * c + 1
                    assert (c, slot) not in slots and slot // 2 == c
                    slots.add((c, slot))
                    partial_ctas[u].add(c)
                segments += 1
                pos = seg_end
            assert segments <= 2, (plan, c)
        k = c
        while k < W:
            u = R + k
            taken[u * Tu:(u + 1) * Tu] += 1
            k += grid
    return taken, partial_ctas


SHAPES = list(itertools.product(
    (1, 4, 32),            # batch
    (1, 8),                # kv heads
    (1, 2, 4),             # GQA group
    (64, 128),             # head dim
    (1, 16, 40, 130),      # S
    (0, 100, 2048, 8176),  # P
    (1, 13, 148),          # SMs
))


@pytest.mark.parametrize("B,Hkv,G,d,S,P,sms", SHAPES)
def test_sample_plan_covers_every_tile_once(B, Hkv, G, d, S, P, sms):
    plan = attn.sample_plan(B, Hkv * G, Hkv, d, S, P, sms)
    GS = G * S
    kernel = 0 if (d != 128 or GS > 64) else (16 if GS <= 16 else 32 if GS <= 32 else 64)
    assert plan["kernel"] == kernel
    qtiles = 1 if kernel else -(-GS // 128)
    assert plan["units"] == B * Hkv * qtiles
    assert plan["tiles_per_unit"] == -(-P // 128) + -(-S // 128)
    U, Tu, R = plan["units"], plan["tiles_per_unit"], plan["split_units"]
    sc, W, grid = plan["split_ctas"], plan["whole_units"], plan["grid"]
    assert 1 <= grid <= min(sms, MAX_CTAS) and R + W == U and sc <= grid
    if W:
        assert W % grid == 0, "every launched CTA takes the same number of whole units"
    else:
        assert grid == sc, "without whole units only the split phase's CTAs are launched"
    if R:
        assert sc >= R and sc <= min(grid, 5 * R) or sc == R
        assert (R * Tu) // sc >= min(MIN_SPLIT_TILES, Tu) or sc == R
    taken, partial_ctas = walk(plan)
    assert (taken == 1).all(), "a key tile taken twice or never"
    T = R * Tu
    for u, ctas in partial_ctas.items():
        c_first, c_last = owner_cta(u * Tu, T, sc), owner_cta(u * Tu + Tu - 1, T, sc)
        if ctas:
            assert ctas == set(range(c_first, c_last + 1)), "merge ticket count disagrees with the writers"
            assert len(ctas) <= 7
        else:
            assert c_first == c_last, "a split unit taken whole by one CTA"


def test_sample_plan_of_the_benchmark_shapes():
    # sampling step B32 P2048 S16 Hq16 Hkv8 d128 on 148 SMs: keys-on-lanes kernel, N = 32
    p = attn.sample_plan(32, 16, 8, 128, 16, 2048, 148)
    assert p == {"kernel": 32, "units": 256, "tiles_per_unit": 17, "split_units": 108, "split_ctas": 148,
                 "whole_units": 148, "grid": 148}
    # long-context loop at its largest prefix: 32 units split over every SM
    p = attn.sample_plan(4, 32, 8, 128, 16, 8176, 148)
    assert p["kernel"] == 64 and p["units"] == 32 and p["split_units"] == 32 and p["grid"] == 148


def test_sample_plan_argument_errors():
    lib = _lib.load()
    plan = _lib.SamplePlan()
    ref = _lib.ctypes.byref(plan)
    good = _lib.Dims(2, 4, 2, 128, 0.0)
    assert lib.e2d2_attn_decoder_sample_plan(good, 16, 64, 148, None) == 1
    assert lib.e2d2_attn_decoder_sample_plan(good, 0, 64, 148, ref) == 1
    assert lib.e2d2_attn_decoder_sample_plan(good, 16, -1, 148, ref) == 1
    assert lib.e2d2_attn_decoder_sample_plan(good, 16, 64, 0, ref) == 1
    assert lib.e2d2_attn_decoder_sample_plan(_lib.Dims(2, 4, 2, 96, 0.0), 16, 64, 148, ref) == 2
    assert lib.e2d2_attn_decoder_sample_plan(good, 16, 64, 148, ref) == 0


def test_sample_workspace_holds_two_slots_per_cta():
    for B, Hkv, G, d, S in [(32, 8, 2, 128, 16), (4, 8, 4, 128, 16), (2, 2, 8, 64, 40), (1, 1, 1, 32, 130)]:
        ws = attn.sample_workspace_bytes(B, Hkv * G, Hkv, d, S, 4096)
        rows = min(G * S, 128)
        assert ws >= 1024 + 2 * MAX_CTAS * rows * (d + 2) * 4
