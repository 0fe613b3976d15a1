"""The Python binding on a machine without a GPU: every call refuses CPU tensors (there is no CPU
fallback), and the checks on caller-supplied buffers (out, lse, workspace) reject a wrong shape,
dtype or layout before anything reaches the C ABI -- the kernels write those buffers through
plain pointers, so a buffer that is too small must never get that far."""
import pytest
import torch

from block_discrete_diffusion_tcgen05_b200 import attn

B, Hq, Hkv, L, S, d = 1, 4, 2, 32, 8, 64


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


CALLS = [
    ("encoder_blockcausal", lambda: attn.encoder_blockcausal(bf16(B, Hq, L, d), bf16(B, Hkv, L, d),
                                                             bf16(B, Hkv, L, d), S)),
    ("decoder_train", lambda: attn.decoder_train(bf16(B, Hq, L, d), *(bf16(B, Hkv, L, d) for _ in range(4)), S)),
    ("encoder_backward", lambda: attn.encoder_backward(bf16(B, Hq, L, d), bf16(B, Hkv, L, d), bf16(B, Hkv, L, d),
                                                       bf16(B, Hq, L, d), torch.zeros(B, Hq, L), bf16(B, Hq, L, d),
                                                       S)),
    ("decoder_train_backward", lambda: attn.decoder_train_backward(
        bf16(B, Hq, L, d), *(bf16(B, Hkv, L, d) for _ in range(4)), bf16(B, Hq, L, d), torch.zeros(B, Hq, L),
        bf16(B, Hq, L, d), S)),
    ("decoder_sample", lambda: attn.decoder_sample(bf16(B, Hq, S, d), bf16(B, Hkv, 64, d), bf16(B, Hkv, 64, d), 16,
                                                   bf16(B, Hkv, S, d), bf16(B, Hkv, S, d))),
    ("encoder_block_step", lambda: attn.encoder_block_step(bf16(B, Hq, S, d), bf16(B, Hkv, 64, d),
                                                           bf16(B, Hkv, 64, d), 16, bf16(B, Hkv, S, d),
                                                           bf16(B, Hkv, S, d))),
    ("kv_cache_append", lambda: attn.kv_cache_append(bf16(B, Hkv, 64, d), bf16(B, Hkv, 64, d), 0,
                                                     bf16(B, Hkv, S, d), bf16(B, Hkv, S, d))),
]


@pytest.mark.parametrize("name,call", CALLS, ids=[c[0] for c in CALLS])
def test_every_call_refuses_cpu_tensors(name, call):
    with pytest.raises(ValueError, match="CUDA"):
        call()


@pytest.fixture
def cpu_need(monkeypatch):
    """attn._need without its CUDA-residency check, so the buffer checks can run on the CPU."""
    def need(t, name, dtype=torch.bfloat16, ndim=4):
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if t.dim() != ndim:
            raise ValueError(f"{name} must have {ndim} dimensions")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    monkeypatch.setattr(attn, "_need", need)


def test_out_buffer_is_checked(cpu_need):
    q = bf16(B, Hq, L, d)
    assert attn._out_tensor(None, q).shape == q.shape
    good = bf16(B, Hq, L, d)
    assert attn._out_tensor(good, q) is good
    with pytest.raises(ValueError, match="shape"):
        attn._out_tensor(bf16(B, Hq, L - 1, d), q)
    with pytest.raises(ValueError, match="bfloat16"):
        attn._out_tensor(torch.zeros(B, Hq, L, d), q)
    with pytest.raises(ValueError, match="contiguous"):
        attn._out_tensor(bf16(B, Hq, d, L).transpose(2, 3), q)


def test_lse_buffer_is_checked(cpu_need):
    shape = (B, Hq, L)
    assert attn._lse_tensor(None, shape, "cpu") is None and attn._lse_tensor(False, shape, "cpu") is None
    made = attn._lse_tensor(True, shape, "cpu")
    assert made.shape == shape and made.dtype == torch.float32
    good = torch.zeros(shape)
    assert attn._lse_tensor(good, shape, "cpu") is good
    with pytest.raises(ValueError, match="shape"):
        attn._lse_tensor(torch.zeros(B, Hq, L + 1), shape, "cpu")
    with pytest.raises(ValueError, match="float32"):
        attn._lse_tensor(torch.zeros(shape, dtype=torch.float64), shape, "cpu")


def test_workspace_must_be_a_contiguous_cuda_tensor():
    with pytest.raises(ValueError, match="workspace"):
        attn._need_workspace(torch.zeros(1024, dtype=torch.uint8))
    with pytest.raises(ValueError, match="workspace"):
        attn._need_workspace(b"not a tensor")
