"""GPU parity of the prefix-cache snapshots (lightning_prefill_snapshots)
against the oracle's snapshot form, through the C ABI, for every kernel.

A snapshot is the state after the first (n+1)*interval tokens; the oracle
computes it by the token recurrence, and its own pin ties that to the
definition on each prefix.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import inputs

from parity import TOL, guarded_empty, guards_intact, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (batch, heads, seq, dim, block, interval, dtype, variant, with_state)
CASES = [
    (1, 2, 512, 64, 64, 128, torch.float32, "simt", False),
    (2, 3, 700, 128, 100, 200, torch.bfloat16, "simt", True),
    (1, 3, 1024, 128, 128, 256, torch.bfloat16, "tcgen05", True),
    (1, 2, 1000, 128, 256, 256, torch.bfloat16, "tcgen05", False),
    (2, 3, 1536, 128, 256, 512, torch.bfloat16, "pair", True),
    (1, 4, 1300, 128, 256, 256, torch.bfloat16, "pair", False),
    (1, 2, 768, 128, 256, 768, torch.bfloat16, "pair", True),   # one snapshot: the last block
    (1, 2, 200, 128, 256, 256, torch.bfloat16, "pair", True),   # shorter than the interval: none
]


def _oracle_snapshots(inp, interval, heads_idx=None):
    k, v, s0, sl = inp["k"], inp["v"], inp["state_in"], inp["slopes"]
    if heads_idx is not None:
        k, v, sl = k[:, heads_idx], v[:, heads_idx], sl[heads_idx]
        s0 = None if s0 is None else s0[:, heads_idx]
    return oracle.snapshots(inputs.to_oracle(k), inputs.to_oracle(v), sl.cpu().numpy(), interval,
                            None if s0 is None else s0.cpu().numpy())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_L%d_d%d_B%d_I%d_%s_%s_%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "bf16" if c[6] == torch.bfloat16 else "f32", c[7],
    "state" if c[8] else "zero"))
def test_snapshots_match_the_oracle(case):
    b, h, L, d, block, interval, dtype, variant, with_state = case
    inp = inputs.prefill_inputs(b, h, L, d, dtype, with_state, seed=21, device=DEV)
    n = L // interval
    snaps, back = guarded_empty((b, h, n, d, d), torch.float32, DEV)
    o, s_out, snaps = la.prefill_snapshots(inp["q"], inp["k"], inp["v"], inp["slopes"], block, interval,
                                           inp["state_in"], snapshots=snaps, variant=variant)
    o_ref, s_ref = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], block, inp["state_in"],
                              variant=variant)
    torch.cuda.synchronize()
    assert guards_intact(back, snaps.numel()), "snapshots written outside their buffer"
    # the snapshots change nothing else the kernel writes
    assert torch.equal(o, o_ref)
    assert torch.equal(s_out, s_ref)
    ref = _oracle_snapshots(inp, interval)
    assert ref.shape == tuple(snaps.shape)
    if n:
        e = rel_err(to_f64(snaps), ref)
        assert e <= TOL[dtype], "snapshot error %.3g rms > %.3g" % (e, TOL[dtype])
    if L % interval == 0 and n:
        # the last snapshot is the state the call returns
        assert torch.equal(snaps[:, :, -1], s_out)


def test_long_context_snapshots_sampled_heads():
    # the long-context workload in the bench's launch configuration, a snapshot every
    # 16384 tokens, checked on sampled heads
    w = inputs.WORKLOADS["m1_prefill_128k"]
    inp = inputs.workload_inputs(w, device=DEV)
    interval = 16384
    o, s_out, snaps = la.prefill_snapshots(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, interval,
                                           inp["state_in"])
    torch.cuda.synchronize()
    heads = [0, 21, 63]
    ref = _oracle_snapshots(inp, interval, heads_idx=heads)
    e = rel_err(to_f64(snaps[:, heads]), ref)
    assert e <= TOL[torch.bfloat16], "snapshot error %.3g rms" % e
    assert torch.equal(snaps[:, :, -1], s_out)
