"""A head's result must not depend on what else runs in the same call: how many
(batch, head) pairs there are, which cluster takes a head, or in which wave. A call with
more pairs than fit on the GPU at once (4 x 64 heads: several waves of clusters) is
compared bit for bit with calls of its batch elements alone (64 heads, one wave), and
sampled heads with the float64 oracle. The forward, the snapshot variant, the fused
normalisation and gate, and the backward are all covered."""
import pytest
import torch

import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import inputs

from parity import TOL, oracle_prefill, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF = torch.bfloat16


def _inputs(batch, seq, seed):
    # 4 x 64 heads: more than the 74 clusters of two CTAs that fit on a B200 at once
    return inputs.prefill_inputs(batch, 64, seq, 128, BF, True, seed=seed, device=DEV)


def _one(inp, b):
    return {n: (t[b:b + 1].contiguous() if t is not None and n != "slopes" else t) for n, t in inp.items()}


def test_forward_heads_match_their_own_batch_element():
    inp = _inputs(4, 1000, 71)
    o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, inp["state_in"], variant="pair")
    torch.cuda.synchronize()
    for b in range(4):
        one = _one(inp, b)
        ob, sb = la.prefill(one["q"], one["k"], one["v"], one["slopes"], 256, one["state_in"], variant="pair")
        torch.cuda.synchronize()
        assert torch.equal(o[b:b + 1], ob), b
        assert torch.equal(s[b:b + 1], sb), b
    # and against the oracle on heads of the last wave
    ref_o, ref_s = oracle_prefill(inp, batch_idx=[3], heads_idx=[5, 40, 63])
    assert rel_err(to_f64(o[3:4, [5, 40, 63]]), ref_o, bf16_out=1) <= TOL[BF]
    assert rel_err(to_f64(s[3:4, [5, 40, 63]]), ref_s) <= TOL[BF]
    assert la.abi.lightning_last_device_status(torch.cuda.current_stream().cuda_stream) == la.abi.LA_OK


def test_snapshots_match_their_own_batch_element():
    inp = _inputs(3, 1024, 72)
    o, s, sn = la.prefill_snapshots(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, 256, inp["state_in"],
                                    variant="pair")
    torch.cuda.synchronize()
    for b in (0, 2):
        one = _one(inp, b)
        ob, sb, snb = la.prefill_snapshots(one["q"], one["k"], one["v"], one["slopes"], 256, 256, one["state_in"],
                                           variant="pair")
        torch.cuda.synchronize()
        assert torch.equal(o[b:b + 1], ob) and torch.equal(s[b:b + 1], sb) and torch.equal(sn[b:b + 1], snb), b


def test_fused_norm_gate_matches_its_own_batch_element():
    inp = _inputs(3, 700, 73)
    g = torch.Generator(device=DEV).manual_seed(173)
    gate = torch.randn((3, 700, 64 * 128), generator=g, device=DEV).to(BF)
    gamma = 1.0 + 0.1 * torch.randn((64 * 128,), generator=g, device=DEV)
    y, s = la.prefill_norm_gate(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, gate, gamma,
                                state_in=inp["state_in"])
    torch.cuda.synchronize()
    for b in (1, 2):
        one = _one(inp, b)
        yb, sb = la.prefill_norm_gate(one["q"], one["k"], one["v"], one["slopes"], 256,
                                      gate[b:b + 1].contiguous(), gamma, state_in=one["state_in"])
        torch.cuda.synchronize()
        assert torch.equal(y[b:b + 1], yb) and torch.equal(s[b:b + 1], sb), b


def test_backward_matches_its_own_batch_element():
    inp = _inputs(2, 600, 74)
    g = torch.Generator(device=DEV).manual_seed(174)
    d_o = torch.randn(inp["q"].shape, generator=g, device=DEV).to(BF)
    d_so = torch.randn((2, 64, 128, 128), generator=g, device=DEV) * 0.1
    full = la.prefill_backward(inp["q"], inp["k"], inp["v"], d_o, inp["slopes"], 256, inp["state_in"], d_so,
                               variant="pair")
    torch.cuda.synchronize()
    for b in range(2):
        one = _one(inp, b)
        part = la.prefill_backward(one["q"], one["k"], one["v"], d_o[b:b + 1].contiguous(), one["slopes"], 256,
                                   one["state_in"], d_so[b:b + 1].contiguous(), variant="pair")
        torch.cuda.synchronize()
        for name, x, y in zip(("dq", "dk", "dv", "d_state_in"), full, part):
            assert torch.equal(x[b:b + 1], y), (name, b)
