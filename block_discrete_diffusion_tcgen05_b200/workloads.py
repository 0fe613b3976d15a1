"""The five synthetic workloads of the E2D2 fused block-diffusion attention.

Shapes follow the E2D2 training and sampling algorithms ("Encoder-Decoder Diffusion
Language Models for Efficient Training and Inference", paper notes, sec. 3 and 4); the
sizes are synthetic stand-ins chosen to resemble the pages' settings (block sizes 4-16,
encoder/decoder layer splits such as 28/4, GQA heads of a pretrained decoder-only LLM for
the shared-KV-cache variant).  No dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass
import math


@dataclass(frozen=True)
class TrainShape:
    name: str
    batch: int
    L: int
    S: int
    q_heads: int
    kv_heads: int
    head_dim: int
    sigma: float
    enc_calls: int = 1
    dec_calls: int = 1


@dataclass(frozen=True)
class SampleShape:
    name: str
    batch: int
    P: int
    S: int
    q_heads: int
    kv_heads: int
    head_dim: int
    sigma: float = 1.0


# workload 1: tiny check, encoder + decoder-train over 2L keys.
TINY = TrainShape("tiny: B1 L64 S8 H2 d32", batch=1, L=64, S=8, q_heads=2, kv_heads=2,
                  head_dim=32, sigma=1.0)
# workload 2: E2D2 train pass, last-hidden-state variant.  "N(0, 1/sqrt(d))" read as
# variance 1/sqrt(d), i.e. sigma = d ** -0.25.
TRAIN = TrainShape("e2d2-train: B8 L1024 S16 H16 d64", batch=8, L=1024, S=16, q_heads=16,
                   kv_heads=16, head_dim=64, sigma=64 ** -0.25)
# workload 3: sampling step with the shared KV cache, GQA 16q/8kv, d128.
SAMPLE = SampleShape("e2d2-sample: B32 P2048 S16 Hq16 Hkv8 d128", batch=32, P=2048, S=16,
                     q_heads=16, kv_heads=8, head_dim=128)
# workload 4: translation-shaped train pass, 28 encoder + 4 decoder calls per step.
TRAIN_CHAIN = TrainShape("translation-train: B16 L512 S4 H16 d64 x(28 enc + 4 dec)", batch=16,
                         L=512, S=4, q_heads=16, kv_heads=16, head_dim=64, sigma=1.0,
                         enc_calls=28, dec_calls=4)
# workload 5: long-context sample loop, prefix 0..8192 in S=16 blocks, 8 decoder calls
# per denoise step x 16 steps per block, append after each block.
SAMPLE_LOOP = dict(name="long-sample-loop: B4 P0..8192 S16 Hq32 Hkv8 d128", batch=4,
                   P_max=8192, S=16, q_heads=32, kv_heads=8, head_dim=128, layers=8,
                   steps_per_block=16)


def unmasked_pairs(L: int, S: int) -> int:
    """(L^2 + L S) / 2: the attended (query, key) pairs of one E2D2 encoder or decoder pass
    with S | L (FLOPs table of the E2D2 training algorithm, sec. 4)."""
    assert L % S == 0
    return (L * L + L * S) // 2


def useful_flops_train(shape: TrainShape) -> int:
    """4 * d * Hq * batch * pairs: two matmuls of 2 FLOPs per multiply-add, masked pairs
    excluded -- the attention FLOPs term of the E2D2 FLOPs table with D = Hq * d."""
    return 4 * shape.head_dim * shape.q_heads * shape.batch * unmasked_pairs(shape.L, shape.S)


def useful_flops_sample(shape: SampleShape) -> int:
    return 4 * shape.head_dim * shape.q_heads * shape.batch * shape.S * (shape.P + shape.S)


def bytes_train(shape: TrainShape, decoder: bool, with_lse: bool = True) -> int:
    """Algorithmic HBM bytes of one call: Q, each K/V once, O, plus LSE."""
    n_q = shape.batch * shape.q_heads * shape.L * shape.head_dim * 2
    n_kv = shape.batch * shape.kv_heads * shape.L * shape.head_dim * 2
    kv_sets = 2 if decoder else 1
    lse = shape.batch * shape.q_heads * shape.L * 4 if with_lse else 0
    return n_q + 2 * kv_sets * n_kv + n_q + lse


def bytes_sample(shape: SampleShape, with_lse: bool = True) -> int:
    n_q = shape.batch * shape.q_heads * shape.S * shape.head_dim * 2
    n_kv = shape.batch * shape.kv_heads * (shape.P + shape.S) * shape.head_dim * 2
    lse = shape.batch * shape.q_heads * shape.S * 4 if with_lse else 0
    return n_q + 2 * n_kv + n_q + lse


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
