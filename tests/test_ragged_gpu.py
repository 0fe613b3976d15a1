"""GPU parity of the sampling step with ragged prefixes (e2d2_attn_decoder_sample_ragged): batch
entry b's S noised queries attend to rows 0..P[b]-1 of its own cache and to its own block
("Encoder-Decoder Diffusion Language Models for Efficient Training and Inference", paper notes,
sec. 3: the cache grows per decoded block; "Block Diffusion: Interpolating Between Autoregressive
and Diffusion Language Models", sec. 3: sequences of any length), checked element by element
against the oracle's decoder_sample_ragged.  Cache rows at or past each P[b] are NaN on the device
copy: they must never reach the result.  Bars as for every forward call: max |d out| <= 2e-2,
per-row |d lse| <= 1e-3."""
import numpy as np
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn
import gpu_helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, S, cap, d, P: P = 0, P = capacity, unaligned, short and long entries together
    (6, 16, 8, 16, 1040, 128, [0, 1040, 17, 128, 1000, 513]),   # keys-on-lanes kernel, N = 32
    (4, 32, 8, 16, 600, 128, [5, 600, 256, 0]),                  # keys-on-lanes kernel, N = 64
    (4, 8, 2, 16, 600, 64, [5, 600, 256, 0]),                    # generic kernel, head_dim 64
    (2, 8, 1, 16, 400, 128, [300, 77]),                          # generic kernel, G*S = 128
    (3, 4, 4, 7, 300, 32, [299, 1, 130]),                        # head_dim 32, S = 7
    (1, 2, 1, 16, 0, 128, [0]),                                  # empty cache
]


def run_ragged(orc, B, Hq, Hkv, S, cap, d, P, seed0=1400, sigma=1.0):
    q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, max(cap, 1), d, sigma, seed0)
    for b, pb in enumerate(P):
        for t in (kc[1], vc[1]):
            t[b, :, pb:, :] = float("nan")
    Pd = torch.tensor(P, dtype=torch.int32, device="cuda")
    out, lse = attn.decoder_sample_ragged(q[1], kc[1], vc[1], Pd, kb[1], vb[1])
    torch.cuda.synchronize()
    ref_o, ref_l = orc.decoder_sample_ragged(q[0].f32, kc[0].f32, vc[0].f32, P, kb[0].f32, vb[0].f32)
    return H.compare(out, lse, ref_o, ref_l, f"ragged B{B} Hq{Hq} Hkv{Hkv} S{S} d{d} P{P}")


@pytest.mark.parametrize("B,Hq,Hkv,S,cap,d,P", CASES)
def test_ragged_sample_matches_oracle(oracle, B, Hq, Hkv, S, cap, d, P):
    run_ragged(oracle, B, Hq, Hkv, S, cap, d, P)


def test_ragged_sample_sharp_softmax(oracle):
    run_ragged(oracle, 4, 16, 8, 16, 700, 128, [699, 3, 400, 64], seed0=1500, sigma=3.0)


def test_ragged_equal_prefixes_match_the_single_prefix_call():
    """With every P[b] equal, the ragged call is the single-prefix call (other split, same result
    within the fp32 merge)."""
    B, Hq, Hkv, S, cap, d, P = 8, 16, 8, 16, 1100, 128, 1024
    q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, 1600)
    o1, l1 = attn.decoder_sample(q[1], kc[1], vc[1], P, kb[1], vb[1])
    o2, l2 = attn.decoder_sample_ragged(q[1], kc[1], vc[1], torch.full((B,), P, dtype=torch.int32, device="cuda"),
                                        kb[1], vb[1])
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_ragged_sampling_workload_size_sampled_entries(oracle):
    """The sampling-step size (B32 Hq16 Hkv8 S16 d128, capacity 2064) with prefixes drawn from
    [0, 2064]; the oracle recomputes four entries (entries are independent)."""
    B, Hq, Hkv, S, cap, d = 32, 16, 8, 16, 2064, 128
    rng = np.random.default_rng(1700)
    P = [int(x) for x in rng.integers(0, cap + 1, size=B)]
    P[3], P[9] = 0, cap
    q, kc, vc, kb, vb = H.sample_inputs(B, Hq, Hkv, S, cap, d, 1.0, 1700)
    for b, pb in enumerate(P):
        for t in (kc[1], vc[1]):
            t[b, :, pb:, :] = float("nan")
    Pd = torch.tensor(P, dtype=torch.int32, device="cuda")
    out, lse = attn.decoder_sample_ragged(q[1], kc[1], vc[1], Pd, kb[1], vb[1])
    torch.cuda.synchronize()
    for b in (0, 3, 9, 31):
        sl = slice(b, b + 1)
        ref_o, ref_l = oracle.decoder_sample_ragged(q[0].f32[sl], kc[0].f32[sl], vc[0].f32[sl], [P[b]],
                                                    kb[0].f32[sl], vb[0].f32[sl])
        H.compare(out[sl], lse[sl], ref_o, ref_l, f"ragged sampling size entry {b} P {P[b]}")
    assert attn.last_device_error() == 0


def test_ragged_append_is_bitwise_per_entry(oracle):
    """e2d2_kv_cache_append_ragged: entry b's new rows land at rows P[b].. of its own caches, bit
    for bit (the oracle's append per entry); rows that would pass the capacity are not written; all
    other rows keep their bits."""
    from block_discrete_diffusion_tcgen05_b200 import synth

    B, Hkv, cap, d, S = 4, 2, 100, 128, 16
    P = [0, 84, 37, 90]   # the last entry's rows 100..105 fall past the capacity
    kc, vc = (synth.normal_bf16((B, Hkv, cap, d), 2100 + t) for t in range(2))
    kn, vn = (synth.normal_bf16((B, Hkv, S, d), 2102 + t) for t in range(2))
    kd, vd = synth.to_torch(kc, "cuda"), synth.to_torch(vc, "cuda")
    attn.kv_cache_append_ragged(kd, vd, torch.tensor(P, dtype=torch.int32, device="cuda"),
                                synth.to_torch(kn, "cuda"), synth.to_torch(vn, "cuda"))
    torch.cuda.synchronize()
    got_k = kd.cpu().view(torch.int16).numpy().view(np.uint16)
    got_v = vd.cpu().view(torch.int16).numpy().view(np.uint16)
    for b, pb in enumerate(P):
        kb, vb = kc.bits[b:b + 1].copy(), vc.bits[b:b + 1].copy()
        n = min(S, cap - pb)
        if n == S:
            oracle.kv_append(kb, vb, pb, kn.bits[b:b + 1], vn.bits[b:b + 1])
        else:
            kb[:, :, pb:pb + n], vb[:, :, pb:pb + n] = kn.bits[b:b + 1, :, :n], vn.bits[b:b + 1, :, :n]
        assert np.array_equal(got_k[b:b + 1], kb) and np.array_equal(got_v[b:b + 1], vb), f"entry {b}"
