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


# ---------------------------------------------------------------------------------------------
# Ragged prefixes (e2d2_attn_decoder_sample_ragged): one stream-K stream over every unit's tiles,
# entry b's units taking ceil(S/128) + ceil(P[b]/128) tiles each, cut into equal contiguous
# ranges over all launched CTAs.
# ---------------------------------------------------------------------------------------------
RAGGED_MIN_TILES = 3   # tiles per CTA the ragged split aims for (kMinRaggedTiles)


def ragged_stream_ctas(T, units, grid):
    return min(grid, T, max(units, T // RAGGED_MIN_TILES))


def ragged_walk(P, S, upe, cap, grid):
    """The schedule as the kernels walk it: per-entry prefix, binary search for a tile's entry,
    unit = entry's units in order, the stream cut over min(grid, tiles) CTAs.  Returns (taken per
    tile, partial writers per unit, prefix, tiles, CTAs of the stream)."""
    per_entry = [upe * (-(-S // 128) + -(-min(max(p, 0), cap) // 128)) for p in P]
    pre = np.concatenate([[0], np.cumsum(per_entry)]).astype(np.int64)
    T = int(pre[-1])
    grid = ragged_stream_ctas(T, len(P) * upe, grid)   # the stream's CTAs; the others take nothing
    taken = np.zeros(T, dtype=np.int64)
    writers = {}
    for c in range(grid):
        start, end = range_begin(c, T, grid), range_begin(c + 1, T, grid)
        pos, slots = start, set()
        while pos < end:
            b = int(np.searchsorted(pre, pos, side="right") - 1)   # pre[b] <= pos < pre[b+1]
            Tu = (int(pre[b + 1]) - int(pre[b])) // upe
            u_in = (pos - int(pre[b])) // Tu
            u, ubeg = b * upe + u_in, int(pre[b]) + u_in * Tu
            seg_end = min(end, ubeg + Tu)
            taken[pos:seg_end] += 1
            if not (pos == ubeg and seg_end == ubeg + Tu):
                slot = 2 * c if start >= ubeg else 2 * c + 1
                assert slot not in slots, "two partial units of one CTA share a slot"
                slots.add(slot)
                writers.setdefault(u, set()).add(c)
                # the merge ticket arithmetic of the kernels
                c_first, c_last = owner_cta(ubeg, T, grid), owner_cta(ubeg + Tu - 1, T, grid)
                assert c_first <= c <= c_last
            pos = seg_end
        assert len(slots) <= 2
    return taken, writers, pre, T, grid


RAGGED_CASES = [
    # B, Hq, Hkv, d, S, cap, P, sms
    (6, 16, 8, 128, 16, 1040, [0, 1040, 17, 128, 1000, 513], 148),
    (4, 8, 2, 64, 16, 600, [5, 600, 256, 0], 148),
    (2, 8, 1, 128, 16, 400, [300, 77], 148),
    (32, 16, 8, 128, 16, 2064, [(67 * b) % 2065 for b in range(32)], 148),
    (3, 4, 4, 32, 130, 5000, [4999, 1, 2560], 13),
    (1, 2, 1, 64, 1, 0, [0], 148),
    (256, 2, 1, 128, 16, 300, [(7 * b) % 301 for b in range(256)], 148),
    (5, 32, 8, 128, 16, 8192, [8192, 8176, 0, 16, 4000], 148),
]


@pytest.mark.parametrize("B,Hq,Hkv,d,S,cap,P,sms", RAGGED_CASES)
def test_ragged_plan_covers_every_tile_once(B, Hq, Hkv, d, S, cap, P, sms):
    plan = attn.sample_ragged_plan(B, Hq, Hkv, d, S, P, cap, sms)
    G = Hq // Hkv
    GS = G * S
    kernel = 0 if (d != 128 or GS > 64) else (16 if GS <= 16 else 32 if GS <= 32 else 64)
    qtiles = 1 if kernel else -(-GS // 128)
    assert plan["kernel"] == kernel
    assert plan["units_per_entry"] == Hkv * qtiles and plan["units"] == B * Hkv * qtiles
    assert plan["grid"] == min(sms, MAX_CTAS)
    taken, writers, pre, T, G = ragged_walk(P, S, plan["units_per_entry"], cap, plan["grid"])
    assert plan["total_tiles"] == T and plan["stream_ctas"] == G
    assert (taken == 1).all(), "a key tile taken twice or never"
    for u, ctas in writers.items():
        b, Tu = u // plan["units_per_entry"], None
        Tu = (int(pre[b + 1]) - int(pre[b])) // plan["units_per_entry"]
        ubeg = int(pre[b]) + (u % plan["units_per_entry"]) * Tu
        c_first, c_last = owner_cta(ubeg, T, G), owner_cta(ubeg + Tu - 1, T, G)
        assert ctas == set(range(c_first, c_last + 1)), "merge ticket count disagrees with the writers"


def test_ragged_plan_clamps_and_refuses():
    lib = _lib.load()
    # values outside [0, capacity] are clamped
    a = attn.sample_ragged_plan(2, 4, 2, 128, 16, [-5, 10_000], 300, 148)
    b = attn.sample_ragged_plan(2, 4, 2, 128, 16, [0, 300], 300, 148)
    assert a == b
    plan = _lib.RaggedPlan()
    ref = _lib.ctypes.byref(plan)
    arr = (_lib.ctypes.c_int * 2)(1, 2)
    good = _lib.Dims(2, 4, 2, 128, 0.0)
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 16, None, 64, 148, ref) == 1
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 16, arr, 64, 148, None) == 1
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 0, arr, 64, 148, ref) == 1
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 16, arr, -1, 148, ref) == 1
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 16, arr, 64, 0, ref) == 1
    big = (_lib.ctypes.c_int * 257)()
    assert lib.e2d2_attn_decoder_sample_ragged_plan(_lib.Dims(257, 4, 2, 128, 0.0), 16, big, 64, 148, ref) == 3
    assert lib.e2d2_attn_decoder_sample_ragged_plan(good, 16, arr, 64, 148, ref) == 0


_OVERRIDE = r"""
import sys
sys.path.insert(0, {root!r})
from block_discrete_diffusion_tcgen05_b200 import attn
for args in ((4, 32, 8, 128, 16, 2000, 148), (32, 16, 8, 128, 16, 2048, 148), (2, 8, 2, 64, 40, 5000, 13)):
    print(repr(attn.sample_plan(*args)))
"""


@pytest.mark.parametrize("splits", ["1", "7", "32", "100", "1000"])
def test_split_override_plans_stay_valid(splits):
    """E2D2_SPLITS=n (read once per process) sets the split phase's CTA count, clamped to what the
    schedule supports; every overridden plan still takes each tile once with correct merges."""
    import os
    import subprocess
    import sys
    from pathlib import Path

    root = Path(__file__).resolve().parents[1]
    res = subprocess.run([sys.executable, "-c", _OVERRIDE.format(root=str(root))], capture_output=True, text=True,
                         env=dict(os.environ, E2D2_SPLITS=splits), timeout=300)
    assert res.returncode == 0, res.stderr
    for line in res.stdout.splitlines():
        plan = eval(line)
        R, Tu = plan["split_units"], plan["tiles_per_unit"]
        if R:
            want = max(R, min(int(splits), min(148, 256)))
            assert plan["split_ctas"] == min(want, R * Tu, max(plan["grid"], R)), plan
        taken, partial_ctas = walk(plan)
        assert (taken == 1).all()
        T = R * Tu
        for u, ctas in partial_ctas.items():
            if ctas:
                c_first = owner_cta(u * Tu, T, plan["split_ctas"])
                c_last = owner_cta(u * Tu + Tu - 1, T, plan["split_ctas"])
                assert ctas == set(range(c_first, c_last + 1))
