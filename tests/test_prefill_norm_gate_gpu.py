"""GPU parity of the prefill with the per-head normalisation and gate fused into
its epilogue (lightning_prefill_norm_gate) against the oracle's prefill followed
by the oracle's norm_gate, through the C ABI. y's error is measured through
dy/do against the prefill's bound on o (parity.norm_gate_y_err_in_o_units)."""
import pytest
import torch

import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

from parity import (NG_EPS, TOL, guarded_empty, guards_intact, norm_gate_y_err_in_o_units as _y_err_in_o_units,
                    oracle_norm_gate_of as _oracle_y, oracle_prefill, rel_err, to_f64, y_err_per_head)

pytestmark = pytest.mark.gpu

DEV = "cuda"
EPS = NG_EPS


def _gate_gamma(b, h, L, d, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    gate = torch.randn((b, L, h * d), generator=g, device=DEV).to(torch.bfloat16)
    gamma = 1.0 + 0.1 * torch.randn((h * d,), generator=g, device=DEV)
    return gate, gamma


def _run(b, h, L, state_in, seed):
    inp = inputs.prefill_inputs(b, h, L, 128, torch.bfloat16, state_in, seed=seed, device=DEV)
    gate, gamma = _gate_gamma(b, h, L, 128, seed + 1000)
    y, back = guarded_empty((b, L, h * 128), torch.bfloat16, DEV)
    _, s_out = la.prefill_norm_gate(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, gate, gamma, EPS,
                                    state_in=inp["state_in"], y=y)
    torch.cuda.synchronize()
    assert guards_intact(back, y.numel()), "prefill_norm_gate wrote outside y"
    o64, s64 = oracle_prefill(inp)
    if L > 0:
        ref = _oracle_y(o64, gate, gamma)
        e = _y_err_in_o_units(to_f64(y), ref, o64, gate, gamma)
        ep = y_err_per_head(to_f64(y), ref, h)
        print("prefill_norm_gate b%d h%d L%d: error %.3g rms(o) through dy/do, %.3g rms(y) per head as is"
              % (b, h, L, e, ep))
        assert e <= TOL[torch.bfloat16], "y error %.3g rms(o) through dy/do > %.3g" % (e, TOL[torch.bfloat16])
        assert ep <= TOL[torch.bfloat16], "y error %.3g rms(y) per head > %.3g" % (ep, TOL[torch.bfloat16])
    es = rel_err(to_f64(s_out), s64)
    assert es <= TOL[torch.bfloat16], "state_out error %.3g rms" % es
    return inp, gate, gamma, y, s_out


CASES = [
    # (batch, heads, seq, state_in)
    (1, 2, 1, False),
    (1, 2, 255, False),
    (2, 4, 700, True),
    (1, 8, 1000, False),
    (1, 64, 300, True),
    (3, 2, 513, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_L%d%s" % (c[0], c[1], c[2], "_s" if c[3] else ""))
def test_prefill_norm_gate_matches_the_oracle(case):
    b, h, L, s0 = case
    _run(b, h, L, s0, seed=70 + L)


def test_prefill_norm_gate_equals_prefill_then_norm_gate():
    # the fused call against the two calls it replaces: the same bf16 o, the mean of
    # squares from fp32 (fused) or bf16 (two calls) values, then one rounding of y each
    inp, gate, gamma, y, s_out = _run(2, 8, 600, True, seed=80)
    o, s2 = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, inp["state_in"])
    y2 = la.norm_gate(o, gate, gamma, EPS, True)
    torch.cuda.synchronize()
    assert torch.equal(s_out, s2), "state_out differs from the plain prefill's"
    e = rel_err(to_f64(y), to_f64(y2), bf16_out=2)
    assert e <= 4e-3, "fused and two-call y differ by %.3g rms" % e


def test_prefill_norm_gate_empty_sequence_passes_the_state_through():
    b, h = 2, 4
    inp = inputs.prefill_inputs(b, h, 0, 128, torch.bfloat16, True, seed=81, device=DEV)
    gate, gamma = _gate_gamma(b, h, 0, 128, 82)
    y = torch.empty((b, 0, h * 128), dtype=torch.bfloat16, device=DEV)
    _, s_out = la.prefill_norm_gate(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, gate, gamma, EPS,
                                    state_in=inp["state_in"], y=y)
    torch.cuda.synchronize()
    assert torch.equal(s_out, inp["state_in"])


def test_prefill_norm_gate_8k_workload_sampled_heads():
    # the 8192-token workload in the fused call; the per-head mean makes each head's
    # 128 channels of y depend on that head alone, so the oracle runs on sampled heads
    w = inputs.WORKLOADS["m1_prefill_8k"]
    inp = inputs.workload_inputs(w, device=DEV)
    gate, gamma = _gate_gamma(w.batch, w.heads, w.seq, w.dim, 83)
    y, s_out = la.prefill_norm_gate(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, gate, gamma, EPS,
                                    state_in=inp["state_in"])
    torch.cuda.synchronize()
    heads = [0, 17, 40, 63]
    o64, s64 = oracle_prefill(inp, heads_idx=heads)
    ref = _oracle_y(o64, gate, gamma, heads_idx=heads)
    got = to_f64(y).reshape(w.batch, w.seq, w.heads, w.dim)[:, :, heads].reshape(ref.shape)
    e = _y_err_in_o_units(got, ref, o64, gate, gamma, heads_idx=heads)
    ep = y_err_per_head(got, ref, len(heads))
    print("prefill_norm_gate 8k sampled heads: error %.3g rms(o) through dy/do, %.3g rms(y) per head as is"
          % (e, ep))
    assert e <= TOL[torch.bfloat16]
    assert ep <= TOL[torch.bfloat16], "y error %.3g rms(y) per head" % ep
    assert rel_err(to_f64(s_out[:, heads]), s64) <= TOL[torch.bfloat16]


def test_prefill_norm_gate_rejects_what_the_pair_kernel_does_not_take():
    stream = torch.cuda.current_stream().cuda_stream
    for dtype, block in ((torch.float32, 256), (torch.bfloat16, 128)):
        inp = inputs.prefill_inputs(1, 2, 64, 128, dtype, False, seed=84, device=DEV)
        gate = torch.zeros((1, 64, 256), dtype=dtype, device=DEV)
        gamma = torch.ones((256,), dtype=torch.float32, device=DEV)
        y = torch.empty_like(gate)
        rc = abi.lightning_prefill_norm_gate(
            inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(), 0 if dtype == torch.float32 else 1,
            inp["slopes"].data_ptr(), 1, 2, 64, 128, block, None, gate.data_ptr(), gamma.data_ptr(), EPS,
            y.data_ptr(), None, None, 0, stream)
        assert rc == abi.LA_ERR_UNSUPPORTED
    assert abi.lightning_device_status(stream) == abi.LA_OK
