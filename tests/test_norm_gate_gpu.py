"""GPU parity of the normalisation-and-gating epilogue (lightning_norm_gate)
against the oracle's norm_gate, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import inputs

from parity import TOL, guarded_empty, guards_intact, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case_inputs(b, h, L, d, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    o = (torch.randn((b, h, L, d), generator=g, device=DEV) * 0.05).to(dtype)
    gate = torch.randn((b, L, h * d), generator=g, device=DEV).to(dtype)
    gamma = 1.0 + 0.1 * torch.randn((h * d,), generator=g, device=DEV)
    return o, gate, gamma


def _oracle(o, gate, gamma, eps, per_head):
    return oracle.norm_gate(inputs.to_oracle(o), inputs.to_oracle(gate), gamma.cpu().numpy(), eps, per_head)


# (batch, heads, seq, dim, dtype)
CASES = [
    (2, 3, 5, 64, torch.float32),
    (1, 2, 300, 128, torch.float32),
    (1, 64, 8, 128, torch.float32),     # 8192 channels: the f32 maximum
    (2, 3, 5, 64, torch.bfloat16),
    (1, 64, 37, 128, torch.bfloat16),
    (1, 128, 4, 128, torch.bfloat16),   # 16384 channels: the bf16 maximum
    (3, 1, 1, 64, torch.bfloat16),
]


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_L%d_d%d_%s" % (
    c[0], c[1], c[2], c[3], "bf16" if c[4] == torch.bfloat16 else "f32"))
def test_norm_gate_matches_the_oracle(case, per_head):
    b, h, L, d, dtype = case
    o, gate, gamma = _case_inputs(b, h, L, d, dtype, seed=50)
    y, back = guarded_empty((b, L, h * d), dtype, DEV)
    la.norm_gate(o, gate, gamma, 1e-6, per_head, y=y)
    torch.cuda.synchronize()
    assert guards_intact(back, y.numel()), "norm_gate wrote outside y"
    e = rel_err(to_f64(y), _oracle(o, gate, gamma, 1e-6, per_head), bf16_out=int(dtype == torch.bfloat16))
    assert e <= TOL[dtype], "y error %.3g rms > %.3g" % (e, TOL[dtype])


def test_norm_gate_after_the_8k_prefill():
    # the epilogue on a real prefill output of the 8k workload
    w = inputs.WORKLOADS["m1_prefill_8k"]
    inp = inputs.workload_inputs(w, device=DEV)
    o, _ = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, inp["state_in"])
    g = torch.Generator(device=DEV).manual_seed(51)
    gate = torch.randn((w.batch, w.seq, w.heads * w.dim), generator=g, device=DEV).to(w.dtype)
    gamma = torch.ones(w.heads * w.dim, device=DEV)
    for per_head in (False, True):
        y = la.norm_gate(o, gate, gamma, 1e-6, per_head)
        torch.cuda.synchronize()
        e = rel_err(to_f64(y), _oracle(o, gate, gamma, 1e-6, per_head), bf16_out=1)
        assert e <= TOL[w.dtype], "y error %.3g rms (per_head=%s)" % (e, per_head)
