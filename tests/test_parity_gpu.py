"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances: max |err| <= 1e-4 rms(o) for float32 inputs and <= 2e-2 rms(o)
for bfloat16 inputs (fp32 accumulation and state), the same rule for the
state against rms(state). A bfloat16 o is compared after its own final
rounding: half a bf16 ulp per element is excluded from |err|, since no
bf16-valued output can be closer than that to the float64 result. Inputs
come from the seeded generators in linear_attention_lightning_b200.inputs.
"""
import numpy as np
import pytest
import torch

import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import inputs

from parity import TOL, guarded_empty, guards_intact, oracle_prefill, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
VARIANTS = ["simt", "tcgen05", "pair"]


def _skip_unsupported(variant, dtype, b, h, L, d, block):
    if variant != "simt":
        try:
            la.prefill_variant(dtype, b, h, L, d, block, variant)
        except ValueError:
            pytest.skip("%s kernel does not take dtype=%s dim=%d block=%d" % (variant, dtype, d, block))


def _check_prefill(inp, block, variant, tol=None, heads_idx=None, batch_idx=None, form="recurrence"):
    q = inp["q"]
    b, h, L, d = q.shape
    o, back = guarded_empty(q.shape, q.dtype, DEV)
    s_out, s_back = guarded_empty((b, h, d, d), torch.float32, DEV)
    o, s_out = la.prefill(q, inp["k"], inp["v"], inp["slopes"], block, inp["state_in"], o=o,
                          state_out=s_out, variant=variant)
    torch.cuda.synchronize()
    assert guards_intact(back, o.numel()), "prefill wrote outside o"
    assert guards_intact(s_back, s_out.numel()), "prefill wrote outside state_out"
    ref_o, ref_s = oracle_prefill(inp, heads_idx=heads_idx, batch_idx=batch_idx, form=form)
    go, gs = o, s_out
    if batch_idx is not None:
        go, gs = go[batch_idx], gs[batch_idx]
    if heads_idx is not None:
        go, gs = go[:, heads_idx], gs[:, heads_idx]
    tol = TOL[q.dtype] if tol is None else tol
    e_o = rel_err(to_f64(go), ref_o, bf16_out=int(q.dtype == torch.bfloat16))
    e_s = rel_err(to_f64(gs), ref_s)
    assert e_o <= tol, "o error %.3g rms > %.3g" % (e_o, tol)
    assert e_s <= tol, "state error %.3g rms > %.3g" % (e_s, tol)
    return e_o, e_s


# ---- the named workloads -------------------------------------------------

def test_tiny_prefill_f32():
    w = inputs.WORKLOADS["tiny_prefill_f32"]
    inp = inputs.workload_inputs(w, DEV)
    _check_prefill(inp, w.block, "simt", form="definition")


@pytest.mark.parametrize("variant", VARIANTS)
def test_m1_prefill_8k(variant):
    w = inputs.WORKLOADS["m1_prefill_8k"]
    _skip_unsupported(variant, w.dtype, w.batch, w.heads, w.seq, w.dim, w.block)
    inp = inputs.workload_inputs(w, DEV)
    _check_prefill(inp, w.block, variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_m1_prefill_128k_sampled_heads(variant):
    # full size, in the bench's launch configuration; the oracle checks every
    # output of heads spanning fast to slow decay
    w = inputs.WORKLOADS["m1_prefill_128k"]
    _skip_unsupported(variant, w.dtype, w.batch, w.heads, w.seq, w.dim, w.block)
    if variant == "simt":
        pytest.skip("the CUDA-core kernel is checked at this size through the 8k case only")
    inp = inputs.workload_inputs(w, DEV)
    _check_prefill(inp, w.block, variant, heads_idx=[0, 9, 31, 63])


@pytest.mark.parametrize("variant", VARIANTS)
def test_batched_prefill_with_state_sampled(variant):
    w = inputs.WORKLOADS["batched_prefill_state"]
    _skip_unsupported(variant, w.dtype, w.batch, w.heads, w.seq, w.dim, w.block)
    inp = inputs.workload_inputs(w, DEV)
    _check_prefill(inp, w.block, variant, batch_idx=[0, 7, 15], heads_idx=[0, 5, 17, 40, 63])


def test_batched_decode_1000_steps_sampled():
    w = inputs.WORKLOADS["batched_decode"]
    inp = inputs.workload_inputs(w, DEV)
    state = inp["state"].clone()
    steps = w.steps
    outs = torch.empty_like(inp["q"])
    for t in range(steps):
        la.decode(inp["q"][t], inp["k"][t], inp["v"][t], inp["slopes"], state, o=outs[t])
    torch.cuda.synchronize()
    import oracle
    bsel, hsel = [0, 21, 63], [0, 8, 33, 63]
    sub = lambda x: x[:, bsel][:, :, hsel] if x.dim() == 4 else x[bsel][:, hsel]
    ref_state = inp["state"][bsel][:, hsel].cpu().numpy().astype(np.float64)
    sl = inp["slopes"][hsel].cpu().numpy()
    ref_outs = []
    for t in range(steps):
        o_t, ref_state = oracle.decode(inputs.to_oracle(sub(inp["q"][t:t + 1])[0]),
                                       inputs.to_oracle(sub(inp["k"][t:t + 1])[0]),
                                       inputs.to_oracle(sub(inp["v"][t:t + 1])[0]), sl, ref_state)
        ref_outs.append(o_t)
    ref_outs = np.stack(ref_outs)
    got = to_f64(outs[:, bsel][:, :, hsel])
    assert rel_err(got, ref_outs, bf16_out=1) <= TOL[torch.bfloat16]
    assert rel_err(to_f64(state[bsel][:, hsel]), ref_state) <= TOL[torch.bfloat16]


# ---- edge cases ----------------------------------------------------------

EDGE = [
    # (batch, heads, seq, dim, block, dtype, state_in)
    (1, 2, 1, 128, 256, torch.bfloat16, False),
    (2, 3, 7, 64, 64, torch.float32, True),
    (1, 4, 255, 128, 128, torch.bfloat16, True),
    (1, 4, 257, 128, 256, torch.bfloat16, False),
    (3, 2, 300, 64, 100, torch.bfloat16, True),
    (1, 2, 1000, 128, 256, torch.float32, True),
    (2, 5, 640, 128, 128, torch.bfloat16, True),
    (1, 3, 129, 128, 256, torch.bfloat16, True),
    (1, 2, 513, 128, 1, torch.float32, False),
]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("case", EDGE, ids=lambda c: "b%d_h%d_L%d_d%d_B%d_%s_%s" % (
    c[0], c[1], c[2], c[3], c[4], str(c[5]).split(".")[-1], "s" if c[6] else "z"))
def test_edge_shapes(case, variant):
    b, h, L, d, block, dtype, st = case
    _skip_unsupported(variant, dtype, b, h, L, d, block)
    inp = inputs.prefill_inputs(b, h, L, d, dtype, st, seed=100 + L, device=DEV)
    _check_prefill(inp, block, variant, form="definition" if L <= 300 else "recurrence")


@pytest.mark.parametrize("variant", VARIANTS)
def test_extreme_slopes(variant):
    b, h, L, d, block = 1, 4, 600, 128, 256
    _skip_unsupported(variant, torch.bfloat16, b, h, L, d, block)
    inp = inputs.prefill_inputs(b, h, L, d, torch.bfloat16, True, seed=7, device=DEV)
    inp["slopes"] = torch.tensor([0.0, 1e-6, 5.0, 60.0], dtype=torch.float32, device=DEV)
    _check_prefill(inp, block, variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_chunked_prefill_and_decode_continue(variant):
    b, h, L, d, block = 2, 4, 513, 128, 256
    _skip_unsupported(variant, torch.bfloat16, b, h, L, d, block)
    inp = inputs.prefill_inputs(b, h, L + 1, d, torch.bfloat16, True, seed=11, device=DEV)
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    o_full, s_full = la.prefill(q, k, v, sl, block, s0, variant=variant)
    cut = 256
    oa, sa = la.prefill(q[:, :, :cut].contiguous(), k[:, :, :cut].contiguous(),
                        v[:, :, :cut].contiguous(), sl, block, s0, variant=variant)
    ob, sb = la.prefill(q[:, :, cut:].contiguous(), k[:, :, cut:].contiguous(),
                        v[:, :, cut:].contiguous(), sl, block, sa, variant=variant)
    tol = TOL[torch.bfloat16]
    assert rel_err(to_f64(torch.cat([oa, ob], dim=2)), to_f64(o_full), bf16_out=2) <= tol
    assert rel_err(to_f64(sb), to_f64(s_full)) <= tol
    # decode of the last token after prefilling L tokens == prefill of L+1 tokens
    op, sp = la.prefill(q[:, :, :L].contiguous(), k[:, :, :L].contiguous(),
                        v[:, :, :L].contiguous(), sl, block, s0, variant=variant)
    od = la.decode(q[:, :, L].contiguous(), k[:, :, L].contiguous(), v[:, :, L].contiguous(), sl, sp)
    torch.cuda.synchronize()
    assert rel_err(to_f64(od), to_f64(o_full[:, :, L]), bf16_out=2) <= tol
    assert rel_err(to_f64(sp), to_f64(s_full)) <= tol


@pytest.mark.parametrize("variant", VARIANTS)
def test_in_place_state_carry(variant):
    b, h, L, d, block = 1, 3, 384, 128, 128
    _skip_unsupported(variant, torch.bfloat16, b, h, L, d, block)
    inp = inputs.prefill_inputs(b, h, L, d, torch.bfloat16, True, seed=13, device=DEV)
    ref_o, ref_s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], block, inp["state_in"],
                              variant=variant)
    st = inp["state_in"].clone()
    o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], block, st, state_out=st,
                      variant=variant)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o)
    assert torch.equal(st, ref_s)


def test_empty_sequence_passes_the_state_through():
    b, h, d = 2, 3, 64
    z = torch.empty((b, h, 0, d), dtype=torch.bfloat16, device=DEV)
    sl = inputs.slopes(h, DEV)
    s0 = torch.randn((b, h, d, d), device=DEV)
    _, s = la.prefill(z, z, z, sl, 64, s0)
    _, s_zero = la.prefill(z, z, z, sl, 64, None)
    torch.cuda.synchronize()
    assert torch.equal(s, s0)
    assert torch.count_nonzero(s_zero) == 0


def test_no_device_timeouts_recorded():
    assert la.abi.lightning_device_status(torch.cuda.current_stream().cuda_stream) == la.abi.LA_OK


def test_kernels_agree_under_full_concurrency():
    # Races between the warp roles show up only with every SM busy; repeat the
    # 64-head workload and compare the tensor-core kernels with each other.
    inp = inputs.prefill_inputs(1, 64, 8192, 128, torch.bfloat16, True, seed=21, device=DEV)
    ref_o, ref_s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, inp["state_in"],
                              variant="tcgen05")
    for _ in range(4):
        o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, inp["state_in"],
                          variant="pair")
        torch.cuda.synchronize()
        assert rel_err(to_f64(o), to_f64(ref_o), bf16_out=2) <= 1e-3
        assert rel_err(to_f64(s), to_f64(ref_s)) <= 1e-4
    assert la.abi.lightning_device_status(torch.cuda.current_stream().cuda_stream) == la.abi.LA_OK
