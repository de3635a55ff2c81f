"""Parity of the multi-token, slot-indexed decode with the fp64 oracle (needs a GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_126_b200 import inputs, kda_decode_step, kda_decode_tokens, kda_prefill
from tests.kda_check import TOL, host64, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tokens_inputs(B, n, H, dk, dv, dtype, num_slots, seed):
    """Inputs laid out [B, n, H, .] plus a state pool of ``num_slots`` slots."""
    d = inputs.decode_inputs(B * n, H, dk, dv, 1, dtype, seed=seed, device=DEV)
    shape = lambda t, last: t[0].reshape(B, n, H, last).contiguous()
    pool = inputs.decode_inputs(num_slots, H, dk, dv, 1, dtype, seed=seed + 1, device=DEV)["S0"]
    return dict(q=shape(d["q"], dk), k=shape(d["k"], dk), v=shape(d["v"], dv),
                log_alpha=shape(d["log_alpha"], dk), beta=d["beta"][0].reshape(B, n, H).contiguous(),
                S_pool=pool)


def _oracle(inp, b, h, slot, S_pool0):
    sl = lambda t: host64(t[b, :, h:h + 1])
    n = inp["q"].shape[1]
    o, S = oracle.prefill(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                          host64(inp["beta"][b, :, h:h + 1]), [0, n],
                          S0=host64(S_pool0[slot:slot + 1, h:h + 1]))
    return o[:, 0], S[0, 0]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (16, 8), (40, 44)])
def test_decode_tokens_slots(dtype, dk, dv):
    B, n, H, num_slots = 4, 5, 2, 7
    inp = _tokens_inputs(B, n, H, dk, dv, dtype, num_slots, seed=21)
    slots = torch.tensor([5, -1, 0, 9], dtype=torch.int32, device=DEV)  # -1 and 9 are skipped
    pool0 = inp["S_pool"].clone()
    sentinel = torch.full((B, n, H, dv), 7.0, dtype=inp["q"].dtype, device=DEV)
    o = kda_decode_tokens(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["S_pool"], slots, o=sentinel)
    torch.cuda.synchronize()
    worst_o = worst_S = 0.0
    for b, slot in enumerate([5, -1, 0, 9]):
        if not 0 <= slot < num_slots:
            assert torch.all(o[b] == 7.0), "a skipped sequence's outputs were written"
            continue
        for h in range(H):
            o_ref, S_ref = _oracle(inp, b, h, slot, pool0)
            worst_o = max(worst_o, rel_l2(host64(o[b, :, h]), o_ref))
            worst_S = max(worst_S, rel_l2(host64(inp["S_pool"][slot, h]), S_ref))
    assert worst_o <= TOL[dtype]["o"] and worst_S <= TOL[dtype]["S"], (worst_o, worst_S)
    untouched = [s for s in range(num_slots) if s not in (5, 0)]
    assert torch.equal(inp["S_pool"][untouched], pool0[untouched])


def test_decode_tokens_one_token_equals_decode_step():
    B, H = 6, 3
    inp = _tokens_inputs(B, 1, H, 128, 128, "bf16", B, seed=22)
    S = inp["S_pool"].clone()
    o1 = kda_decode_step(inp["q"][:, 0], inp["k"][:, 0], inp["v"][:, 0], inp["log_alpha"][:, 0],
                         inp["beta"][:, 0], S)
    o2 = kda_decode_tokens(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["S_pool"])
    torch.cuda.synchronize()
    assert rel_l2(host64(o2[:, 0]), host64(o1)) < 1e-5
    assert rel_l2(host64(inp["S_pool"]), host64(S)) < 1e-6


def test_decode_tokens_equals_prefill_of_the_same_tokens():
    B, n, H = 3, 9, 2
    inp = _tokens_inputs(B, n, H, 128, 128, "bf16", B, seed=23)
    pool0 = inp["S_pool"].clone()
    o = kda_decode_tokens(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["S_pool"])
    flat = lambda t: t.reshape(B * n, *t.shape[2:]).contiguous()
    cu = torch.arange(0, B * n + 1, n, dtype=torch.int32, device=DEV)
    o_p, S_p = kda_prefill(flat(inp["q"]), flat(inp["k"]), flat(inp["v"]), flat(inp["log_alpha"]),
                           flat(inp["beta"]), cu, cu.cpu().tolist(), S0=pool0, chunk=64)
    torch.cuda.synchronize()
    assert rel_l2(host64(o.reshape(B * n, H, 128)), host64(o_p)) < 2 * TOL["bf16"]["o"]
    assert rel_l2(host64(inp["S_pool"]), host64(S_p)) < 2 * TOL["bf16"]["S"]


def test_decode_tokens_full_shape_sampled():
    """256 sequences x 32 heads, d = 128, 4 tokens per call, slots permuted."""
    B, n, H, num_slots = 256, 4, 32, 300
    inp = _tokens_inputs(B, n, H, 128, 128, "bf16", num_slots, seed=24)
    perm = torch.randperm(num_slots, generator=torch.Generator().manual_seed(5))[:B]
    slots = perm.to(torch.int32).to(DEV)
    pool0 = inp["S_pool"].clone()
    o = kda_decode_tokens(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["S_pool"], slots)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    worst_o = worst_S = 0.0
    for _ in range(24):
        b, h = int(rng.integers(B)), int(rng.integers(H))
        slot = int(perm[b])
        o_ref, S_ref = _oracle(inp, b, h, slot, pool0)
        worst_o = max(worst_o, rel_l2(host64(o[b, :, h]), o_ref))
        worst_S = max(worst_S, rel_l2(host64(inp["S_pool"][slot, h]), S_ref))
    assert worst_o <= TOL["bf16"]["o"] and worst_S <= TOL["bf16"]["S"], (worst_o, worst_S)


def test_decode_tokens_unaligned_rows_take_the_other_kernel():
    """q/k/v/log alpha whose rows start 2 bytes past a 16-byte boundary (a contiguous view
    one element into a buffer) cannot use the column-slice kernel's 16-byte copies; the
    call must take the per-unit kernel and still match the oracle."""
    B, n, H, num_slots = 5, 3, 2, 5
    inp = _tokens_inputs(B, n, H, 128, 128, "bf16", num_slots, seed=25)

    def shifted(t):  # the same values, stored one element past an aligned start
        buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=DEV)
        view = buf[1:1 + t.numel()].view(t.shape)
        view.copy_(t)
        return view

    q, k, v = shifted(inp["q"]), shifted(inp["k"]), shifted(inp["v"])
    la = shifted(inp["log_alpha"])
    assert q.data_ptr() % 16 != 0
    pool0 = inp["S_pool"].clone()
    o = kda_decode_tokens(q, k, v, la, inp["beta"], inp["S_pool"])
    torch.cuda.synchronize()
    worst_o = worst_S = 0.0
    for b in range(B):
        for h in range(H):
            o_ref, S_ref = _oracle(inp, b, h, b, pool0)
            worst_o = max(worst_o, rel_l2(host64(o[b, :, h]), o_ref))
            worst_S = max(worst_S, rel_l2(host64(inp["S_pool"][b, h]), S_ref))
    assert worst_o <= TOL["bf16"]["o"] and worst_S <= TOL["bf16"]["S"], (worst_o, worst_S)
