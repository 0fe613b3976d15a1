"""The benchmark's roofline numerators (useful FLOPs and algorithmic bytes per call) checked on the
CPU: the pair count behind the train FLOPs equals the number of allowed pairs of the oracle's
explicit masks (themselves pinned to the FLOPs table of the E2D2 training algorithm, sec. 4), and
the per-call figures of the benchmark workloads equal their closed forms written out by hand."""
import pytest

from block_discrete_diffusion_tcgen05_b200 import workloads as W


@pytest.mark.parametrize("L,S", [(8, 1), (16, 4), (64, 8), (96, 32), (128, 128), (256, 16)])
def test_pair_count_equals_the_oracle_masks(oracle, L, S):
    pairs = W.unmasked_pairs(L, S)
    assert int(oracle.mask_encoder(L, S).sum()) == pairs
    assert int(oracle.mask_decoder(L, S).sum()) == pairs


def test_train_pass_figures():
    t = W.TRAIN  # B8 L1024 S16 H16 d64
    assert (t.batch, t.L, t.S, t.q_heads, t.kv_heads, t.head_dim) == (8, 1024, 16, 16, 16, 64)
    # 4 d Hq B (L^2 + L S) / 2
    assert W.useful_flops_train(t) == 4 * 64 * 16 * 8 * (1024 * 1024 + 1024 * 16) // 2 == 17_448_304_640
    q = 8 * 16 * 1024 * 64 * 2       # one [B, H, L, d] bf16 tensor
    lse = 8 * 16 * 1024 * 4
    assert W.bytes_train(t, decoder=False) == 4 * q + lse == 67_633_152       # Q, K, V, O
    assert W.bytes_train(t, decoder=True) == 6 * q + lse == 101_187_584       # Q, 2 K, 2 V, O
    assert W.bytes_train(t, decoder=False, with_lse=False) == 4 * q


def test_sampling_step_figures():
    s = W.SAMPLE  # B32 P2048 S16 Hq16 Hkv8 d128
    assert (s.batch, s.P, s.S, s.q_heads, s.kv_heads, s.head_dim) == (32, 2048, 16, 16, 8, 128)
    assert W.useful_flops_sample(s) == 4 * 128 * 16 * 32 * 16 * (2048 + 16) == 8_657_043_456
    q = 32 * 16 * 16 * 128 * 2
    kv = 32 * 8 * (2048 + 16) * 128 * 2
    assert W.bytes_sample(s) == 2 * q + 2 * kv + 32 * 16 * 16 * 4 == 274_759_680


def test_translation_chain_figures():
    c = W.TRAIN_CHAIN  # B16 L512 S4 H16 d64, 28 encoder + 4 decoder calls
    assert (c.batch, c.L, c.S, c.head_dim, c.enc_calls, c.dec_calls) == (16, 512, 4, 64, 28, 4)
    per_call = 4 * 64 * 16 * 16 * (512 * 512 + 512 * 4) // 2
    assert W.useful_flops_train(c) == per_call
    q = 16 * 16 * 512 * 64 * 2
    lse = 16 * 16 * 512 * 4
    step_bytes = 28 * (4 * q + lse) + 4 * (6 * q + lse)
    assert 28 * W.bytes_train(c, False) + 4 * W.bytes_train(c, True) == step_bytes
    assert round(step_bytes / 1e9, 3) == 2.298
