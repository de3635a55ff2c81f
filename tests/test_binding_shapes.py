"""The Python binding checks every tensor's shape before a pointer reaches the library
(the kernels trust the sizes they are given).  CPU tensors are enough: the shape
checks come before the device checks, so a correctly shaped CPU call fails only on
the device."""
import pytest
import torch

from gated_delta_rule_126_b200 import _binding, build
from gated_delta_rule_126_b200 import (kda_backward, kda_decode_step, kda_decode_tokens, kda_prefill,
                                       kda_prefill_gated, kda_prologue)

T, H, DK, DV, N = 10, 2, 8, 12, 2
BF, F32 = torch.bfloat16, torch.float32


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return _binding.load()


def prefill_args(**over):
    a = dict(q=torch.zeros(T, H, DK, dtype=BF), k=torch.zeros(T, H, DK, dtype=BF),
             v=torch.zeros(T, H, DV, dtype=BF), log_alpha=torch.zeros(T, H, DK), beta=torch.zeros(T, H),
             cu_seqlens=torch.tensor([0, 4, T], dtype=torch.int32))
    a.update(over)
    return a


def test_prefill_shapes():
    with pytest.raises(ValueError, match="CUDA"):
        kda_prefill(**prefill_args())
    for name, bad in [("k", torch.zeros(T, H, DK + 1, dtype=BF)), ("v", torch.zeros(T - 1, H, DV, dtype=BF)),
                      ("log_alpha", torch.zeros(T, H, DV)), ("beta", torch.zeros(T, H, 1))]:
        with pytest.raises(ValueError, match="shape"):
            kda_prefill(**prefill_args(**{name: bad}))
    with pytest.raises(ValueError, match="dimensions"):
        kda_prefill(**prefill_args(q=torch.zeros(T, H * DK, dtype=BF)))
    with pytest.raises(ValueError, match="shape"):
        kda_prefill(**prefill_args(), S0=torch.zeros(N, H, DV, DK))
    with pytest.raises(ValueError, match="shape"):
        kda_prefill(**prefill_args(), o=torch.zeros(T, H, DK, dtype=BF))
    with pytest.raises(ValueError, match="shape"):
        kda_prefill(**prefill_args(), S_final=torch.zeros(N + 1, H, DK, DV))
    # offsets that run past the rows given
    with pytest.raises(ValueError, match="tokens"):
        kda_prefill(**prefill_args(cu_seqlens=torch.tensor([0, 4, T + 1], dtype=torch.int32)))
    with pytest.raises(ValueError, match="differ"):
        kda_prefill(**prefill_args(), cu_seqlens_host=[0, T])


def test_prefill_gated_shapes():
    gate, w = torch.zeros(T, H, DV, dtype=BF), torch.ones(DV)
    with pytest.raises(ValueError, match="CUDA"):
        kda_prefill_gated(**prefill_args(), gate=gate, norm_weight=w)
    with pytest.raises(ValueError, match="shape"):
        kda_prefill_gated(**prefill_args(), gate=torch.zeros(T, H, DK, dtype=BF), norm_weight=w)
    with pytest.raises(ValueError, match="shape"):
        kda_prefill_gated(**prefill_args(), gate=gate, norm_weight=torch.ones(DV + 1))


def test_backward_shapes():
    dO = torch.zeros(T, H, DV, dtype=BF)
    with pytest.raises(ValueError, match="CUDA"):
        kda_backward(**prefill_args(), dO=dO)
    with pytest.raises(ValueError, match="shape"):
        kda_backward(**prefill_args(), dO=torch.zeros(T, H, DK, dtype=BF))
    with pytest.raises(ValueError, match="shape"):
        kda_backward(**prefill_args(), dO=dO, dS_final=torch.zeros(N, H, DK, DK))


def test_prologue_shapes():
    W = 4
    a = dict(q_pre=torch.zeros(T, H, DK, dtype=BF), k_pre=torch.zeros(T, H, DK, dtype=BF),
             v_pre=torch.zeros(T, H, DV, dtype=BF), conv_q=torch.zeros(H, DK, W), conv_k=torch.zeros(H, DK, W),
             conv_v=torch.zeros(H, DV, W), a_gate=torch.zeros(T, H, DK), rate=torch.zeros(H),
             b_gate=torch.zeros(T, H), cu_seqlens=torch.tensor([0, T], dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        kda_prologue(**a)
    for name, bad in [("conv_k", torch.zeros(H, DK, W - 1)), ("conv_v", torch.zeros(H, DK, W)),
                      ("rate", torch.zeros(H + 1)), ("b_gate", torch.zeros(T, H, 1))]:
        with pytest.raises(ValueError, match="shape"):
            kda_prologue(**{**a, name: bad})
    with pytest.raises(ValueError, match="shape"):
        kda_prologue(**a, out={"v": torch.zeros(T, H, DK, dtype=BF)})


def test_decode_shapes():
    B = 3
    a = dict(q=torch.zeros(B, H, DK, dtype=BF), k=torch.zeros(B, H, DK, dtype=BF),
             v=torch.zeros(B, H, DV, dtype=BF), log_alpha=torch.zeros(B, H, DK), beta=torch.zeros(B, H),
             S=torch.zeros(B, H, DK, DV))
    with pytest.raises(ValueError, match="CUDA"):
        kda_decode_step(**a)
    with pytest.raises(ValueError, match="shape"):
        kda_decode_step(**{**a, "S": torch.zeros(B, H, DV, DK)})
    n = 2
    t = dict(q=torch.zeros(B, n, H, DK, dtype=BF), k=torch.zeros(B, n, H, DK, dtype=BF),
             v=torch.zeros(B, n, H, DV, dtype=BF), log_alpha=torch.zeros(B, n, H, DK), beta=torch.zeros(B, n, H),
             S_pool=torch.zeros(5, H, DK, DV))
    with pytest.raises(ValueError, match="CUDA"):
        kda_decode_tokens(**t)
    with pytest.raises(ValueError, match="shape"):
        kda_decode_tokens(**t, slot_idx=torch.zeros(B + 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="shape"):
        kda_decode_tokens(**{**t, "S_pool": torch.zeros(5, H + 1, DK, DV)})
