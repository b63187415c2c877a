"""GPU parity of the tensor-core prefill away from the workloads' input scale.

The tensor-core kernels round the operands they form to fp16 (range 2^-24 ..
65504) while bf16 inputs span fp32's range; the pages put no normalisation on
q or k before Q_t K_t^T ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention).
Both tensor-core kernels (the CTA pair and the single-CTA kernel) carry a
range guard: they measure every (batch, head) while they run and recompute,
with power-of-two operand scales, the heads whose operands would leave fp16's
range. These tests scale q, k, v and the carried
state by powers of two (exact in bf16), put |q . k| above 65504 on a few rows,
and hold every result to the bound of the workloads (max |err| <= 2e-2 rms).
The guard's records (48 bytes per (batch, head) in the workspace) show which
heads took the second pass."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

from parity import TOL, oracle_prefill, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
HEADS = [0, 9, 31, 63]     # fast to slow decay
BF = torch.bfloat16
# (variant, block): the CTA pair, and the single-CTA kernel at both of its block sizes
KERNELS = [("pair", 256), ("tcgen05", 256), ("tcgen05", 128)]


def _scaled(inp, eq=0, ek=0, ev=0, es=0):
    out = dict(inp)
    for name, e in (("q", eq), ("k", ek), ("v", ev)):
        out[name] = (inp[name].float() * 2.0 ** e).to(inp[name].dtype) if e else inp[name]
    if inp["state_in"] is not None and es:
        out["state_in"] = inp["state_in"] * 2.0 ** es
    return out


def _prefill_with_records(inp, block=256, variant="pair", state_out=None, in_place=False):
    q = inp["q"]
    b, h, L, d = q.shape
    need = abi.lightning_prefill_workspace_size(b, h, L, d, block)
    ws = torch.full((max(need, 16),), 0xAB, dtype=torch.uint8, device=DEV)  # stale contents on purpose
    s_in = inp["state_in"]
    if in_place:
        state_out = s_in
    o, s = la.prefill(q, inp["k"], inp["v"], inp["slopes"], block, s_in, state_out=state_out, variant=variant,
                      workspace=ws)
    torch.cuda.synchronize()
    flags = ws[:need].view(torch.int32).view(b * h, 12)[:, 8].cpu().numpy() if need else None
    return o, s, flags


def _check(inp, o, s, tol=None, heads=HEADS, ref=None):
    ref_o, ref_s = oracle_prefill(inp, heads_idx=heads) if ref is None else ref
    tol = TOL[BF] if tol is None else tol
    e_o = rel_err(to_f64(o[:, heads]), ref_o, bf16_out=1)
    e_s = rel_err(to_f64(s[:, heads]), ref_s)
    assert np.all(np.isfinite(to_f64(o[:, heads]))), "non-finite o"
    assert e_o <= tol, "o error %.3g rms > %.3g" % (e_o, tol)
    assert e_s <= tol, "state error %.3g rms > %.3g" % (e_s, tol)
    return e_o, e_s


# q, k, v scaled one at a time by 2^-10, 2^-6, 2^4 and 2^8 (below and above fp16's range for
# the products the kernels form), on the 8192-token workload
SCALES = [(t, e) for e in (-10, -6, 4, 8) for t in "qkv"]


@pytest.mark.parametrize("variant", ["pair", "tcgen05"])
@pytest.mark.parametrize("which,e", SCALES, ids=lambda x: str(x))
def test_one_input_scaled_8k(variant, which, e):
    w = inputs.WORKLOADS["m1_prefill_8k"]
    inp = _scaled(inputs.workload_inputs(w, DEV), **{"e" + which: e})
    o, s, flags = _prefill_with_records(inp, variant=variant)
    e_o, e_s = _check(inp, o, s)
    print("%s %s x 2^%d: o %.2e, state %.2e rms; %d of 64 heads took the scaled pass" % (
        variant, which, e, e_o, e_s, int(flags.sum())))


@pytest.mark.parametrize("variant,block", KERNELS)
def test_the_workload_itself_takes_no_second_pass(variant, block):
    # at the workloads' own scale every head passes the guard: the plain kernel's result stands
    for name in ("m1_prefill_8k", "batched_prefill_state"):
        w = inputs.WORKLOADS[name]
        inp = inputs.workload_inputs(w, DEV)
        _, _, flags = _prefill_with_records(inp, block=block, variant=variant)
        assert flags.sum() == 0, name


@pytest.mark.parametrize("eq,ek,ev,es", [
    (8, 8, 0, 0),        # |q . k| ~ 2^16 on average: P overflows fp16 without the guard
    (-12, -12, 0, 0),    # P deep in fp16's subnormals
    (0, 10, 10, 20),     # a large state
    (0, -12, -12, -24),  # a tiny state
    (-20, 0, 12, 0),
    (16, -16, 0, 0),
])
@pytest.mark.parametrize("variant,block", KERNELS)
def test_joint_scales_with_a_carried_state(variant, block, eq, ek, ev, es):
    inp = inputs.prefill_inputs(2, 64, 1000, 128, BF, True, seed=61, device=DEV)
    inp = _scaled(inp, eq, ek, ev, es)
    o, s, flags = _prefill_with_records(inp, block=block, variant=variant)
    _check(inp, o, s, heads=[0, 17, 40, 63])
    assert flags.sum() == 2 * 64, "every head is outside fp16's window and must take the scaled pass"


def _outlier_rows(inp, rows, mag=2.0 ** 8.5):
    """|q_r . k_r| = mag^2 = 2^17 > 65504 on the given rows (where each row meets its
    own key), with o kept homogeneous: those rows' q and k point along dim 0, which
    every other q, k and the carried state leave empty, and their v is scaled down
    by mag^2."""
    q, k, v = (inp[n].float().clone() for n in ("q", "k", "v"))
    q[..., 0] = 0
    k[..., 0] = 0
    for r in rows:
        q[:, :, r] = 0
        k[:, :, r] = 0
        q[:, :, r, 0] = mag
        k[:, :, r, 0] = mag
        v[:, :, r] *= 1.0 / (mag * mag)
    out = dict(inp, q=q.to(BF), k=k.to(BF), v=v.to(BF))
    if inp["state_in"] is not None:
        s0 = inp["state_in"].clone()
        s0[:, :, 0, :] = 0
        out["state_in"] = s0
    return out


@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("variant,block", KERNELS)
def test_q_dot_k_above_65504_on_a_few_rows(variant, block, with_state):
    inp = inputs.prefill_inputs(1, 64, 8192, 128, BF, with_state, seed=62, device=DEV)
    inp = _outlier_rows(inp, rows=[5, 3000, 8000])
    qk = (inp["q"][0, :, [5, 3000, 8000]].float() * inp["k"][0, :, [5, 3000, 8000]].float()).sum(-1)
    assert float(qk.abs().min()) > 65504.0
    o, s, flags = _prefill_with_records(inp, block=block, variant=variant)
    e_o, e_s = _check(inp, o, s)
    assert flags.sum() == 64
    print("%s B%d |q.k| = %.0f on 3 rows: o %.2e, state %.2e rms" % (variant, block, float(qk.abs().max()), e_o, e_s))


@pytest.mark.parametrize("variant,block", KERNELS)
def test_a_flagged_head_keeps_an_in_place_state_carry_intact(variant, block):
    # pass 1 must not overwrite state_in (== state_out) for a head it hands to pass 2;
    # heads 0-3 are scaled out of fp16's window, heads 4-7 stay in it (their state is
    # carried by pass 1 alone)
    inp = inputs.prefill_inputs(1, 8, 700, 128, BF, True, seed=63, device=DEV)
    for name in ("q", "k"):
        x = inp[name].float()
        x[:, :4] *= 2.0 ** 9
        inp[name] = x.to(BF)
    ref = oracle_prefill(inp, heads_idx=list(range(8)))
    s_carry = inp["state_in"].clone()
    o, s, flags = _prefill_with_records(dict(inp, state_in=s_carry), block=block, variant=variant, in_place=True)
    assert list(flags) == [1, 1, 1, 1, 0, 0, 0, 0]
    _check(inp, o, s, heads=list(range(8)), ref=ref)


@pytest.mark.parametrize("variant,block", KERNELS)
def test_snapshots_of_a_scaled_input(variant, block):
    inp = _scaled(inputs.prefill_inputs(1, 4, 1024, 128, BF, True, seed=64, device=DEV), 8, 8, -8, 0)
    o, s, snaps = la.prefill_snapshots(inp["q"], inp["k"], inp["v"], inp["slopes"], block, 512, inp["state_in"],
                                       variant=variant)
    torch.cuda.synchronize()
    conv = inputs.to_oracle
    ref = oracle.snapshots(conv(inp["k"]), conv(inp["v"]), inp["slopes"].cpu().numpy(), 512,
                           inp["state_in"].cpu().numpy())
    assert rel_err(to_f64(snaps), ref) <= TOL[BF]
    _check(inp, o, s, heads=[0, 1, 2, 3])


def test_backward_of_scaled_inputs():
    b, h, L, d = 1, 4, 1000, 128
    inp = _scaled(inputs.prefill_inputs(b, h, L, d, BF, True, seed=65, device=DEV), 8, 8, 0, 0)
    g = torch.Generator(device=DEV).manual_seed(165)
    d_o = torch.randn((b, h, L, d), generator=g, device=DEV).to(BF)
    d_so = torch.randn((b, h, d, d), generator=g, device=DEV) * 0.1
    got = la.prefill_backward(inp["q"], inp["k"], inp["v"], d_o, inp["slopes"], 256, inp["state_in"], d_so,
                              variant="pair")
    torch.cuda.synchronize()
    conv = inputs.to_oracle
    ref = oracle.backward(conv(inp["q"]), conv(inp["k"]), conv(inp["v"]), conv(d_o), inp["slopes"].cpu().numpy(),
                          inp["state_in"].cpu().numpy(), d_so.cpu().numpy())
    for name, x, r in zip(("dq", "dk", "dv", "d_state_in"), got, ref):
        e = rel_err(to_f64(x), r, bf16_out=int(name != "d_state_in"))
        assert e <= TOL[BF], "%s error %.3g rms" % (name, e)


def test_fused_norm_gate_of_scaled_inputs():
    from parity import norm_gate_y_err_in_o_units, oracle_norm_gate_of
    b, h, L = 1, 4, 700
    inp = _scaled(inputs.prefill_inputs(b, h, L, 128, BF, False, seed=66, device=DEV), 8, 8, 0, 0)
    g = torch.Generator(device=DEV).manual_seed(166)
    gate = torch.randn((b, L, h * 128), generator=g, device=DEV).to(BF)
    gamma = 1.0 + 0.1 * torch.randn((h * 128,), generator=g, device=DEV)
    y, s = la.prefill_norm_gate(inp["q"], inp["k"], inp["v"], inp["slopes"], 256, gate, gamma)
    torch.cuda.synchronize()
    o64, s64 = oracle_prefill(inp)
    ref = oracle_norm_gate_of(o64, gate, gamma)
    assert norm_gate_y_err_in_o_units(to_f64(y), ref, o64, gate, gamma) <= TOL[BF]
    assert rel_err(to_f64(s), s64) <= TOL[BF]
