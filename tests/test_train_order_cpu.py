"""Work order of the train calls (e2d2_attn_train_order, host only): every work item (a pair of
128-row query tiles of one head) is placed on exactly one CTA, and the placement is balanced the
way longest-processing-time-first guarantees: no CTA's work exceeds the mean by more than the
largest item.  Item work is recomputed here from the attention masks themselves (the key tiles
any row of the item may attend to, E2D2 encoder / decoder masks), not from the library's own
formula."""
import numpy as np
import pytest

from block_discrete_diffusion_tcgen05_b200 import attn


def item_tiles(decoder, L, S, pairs, BH, k):
    """Key tiles (128 keys) the item's rows may attend to, per key source, from the masks."""
    qp = pairs - 1 - k // BH
    rows = np.arange(qp * 256, min(L, qp * 256 + 256))
    blk0 = (rows // S) * S
    blk1 = np.minimum(L, blk0 + S)
    if not decoder:  # encoder: keys j < end of the row's block
        return len(set(int(t) for hi in blk1 for t in range(0, -(-hi // 128))))
    enc = set(int(t) for hi in blk0 for t in range(0, -(-hi // 128)))          # blocks strictly before
    dec = set(int(t) for lo, hi in zip(blk0, blk1) for t in range(lo // 128, -(-hi // 128)))  # own block
    return len(enc) + len(dec)


SHAPES = [
    (False, 8, 16, 1024, 16, 148),   # the train pass
    (True, 8, 16, 1024, 16, 148),
    (False, 16, 16, 512, 4, 148),    # translation-shaped pass
    (True, 16, 16, 512, 4, 148),
    (False, 2, 4, 1000, 7, 132),     # ragged last pair, odd block size
    (True, 3, 2, 300, 16, 20),
    (False, 1, 1, 64, 8, 148),       # fewer items than SMs
]


@pytest.mark.parametrize("decoder,B,H,L,S,sms", SHAPES)
def test_every_item_once_and_balanced(decoder, B, H, L, S, sms):
    r = attn.train_order(decoder, B, H, H, 64, L, S, sms)
    pairs = -(-L // 256)
    assert r["items"] == B * H * pairs
    assert r["grid"] == min(r["items"], sms)
    assert r["balanced"]
    cta = np.array(r["cta_of_item"])
    assert cta.min() >= 0 and cta.max() < r["grid"]
    assert len(set(np.unique(cta))) == r["grid"]  # every CTA has work
    cost = np.array([item_tiles(decoder, L, S, pairs, B * H, k) + 1 for k in range(r["items"])])
    load = np.bincount(cta, weights=cost, minlength=r["grid"])
    assert load.max() <= cost.sum() / r["grid"] + cost.max() + 1e-9
    # never worse than the plain round robin
    rr = np.bincount(np.arange(r["items"]) % r["grid"], weights=cost, minlength=r["grid"])
    assert load.max() <= rr.max()


def test_train_pass_order_is_tighter_than_round_robin():
    """On the train pass (512 items of 2-9 tile steps on 148 CTAs) the balanced order cuts the
    busiest CTA's work below round robin's."""
    B, H, L, S = 8, 16, 1024, 16
    r = attn.train_order(False, B, H, H, 64, L, S, 148)
    cost = np.array([item_tiles(False, L, S, 4, B * H, k) + 1 for k in range(r["items"])])
    load = np.bincount(np.array(r["cta_of_item"]), weights=cost)
    rr = np.bincount(np.arange(r["items"]) % 148, weights=cost)
    assert load.max() < rr.max()


def test_large_call_falls_back_to_round_robin():
    r = attn.train_order(False, 16, 32, 32, 64, 8192, 16, 148)   # 16384 items: over the table
    assert not r["balanced"]
    assert r["cta_of_item"][:300] == [k % 148 for k in range(300)]


@pytest.mark.parametrize("args", [(0, 0, 1024, 16, 148), (1, 8, 0, 16, 148), (0, 8, 1024, 0, 148),
                                  (0, 8, 1024, 16, 0)])
def test_bad_arguments_are_refused(args):
    dec, B, L, S, sms = args
    with pytest.raises(RuntimeError):
        attn.train_order(bool(dec), B, 16, 16, 64, L, S, sms)
