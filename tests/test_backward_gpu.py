"""GPU parity of the prefill gradients (lightning_prefill_backward) against
the oracle's backward form, through the C ABI. The oracle's backward is pinned
by exact central differences of the definition (tests/test_oracle_pins.py)."""
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

from parity import TOL, guarded_empty, guards_intact, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _grads_inputs(b, h, L, d, dtype, with_state, with_dstate, seed):
    inp = inputs.prefill_inputs(b, h, L, d, dtype, with_state, seed=seed, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(seed + 1000)
    inp["d_o"] = torch.randn((b, h, L, d), generator=g, device=DEV).to(dtype)
    inp["d_state_out"] = (torch.randn((b, h, d, d), generator=g, device=DEV) * 0.1) if with_dstate else None
    return inp


def _oracle_backward(inp, heads_idx=None):
    sel = (lambda t: t) if heads_idx is None else (lambda t: None if t is None else t[:, heads_idx])
    conv = inputs.to_oracle
    sl = inp["slopes"] if heads_idx is None else inp["slopes"][heads_idx]
    s0, dso = sel(inp["state_in"]), sel(inp["d_state_out"])
    return oracle.backward(conv(sel(inp["q"])), conv(sel(inp["k"])), conv(sel(inp["v"])), conv(sel(inp["d_o"])),
                           sl.cpu().numpy(), None if s0 is None else s0.cpu().numpy(),
                           None if dso is None else dso.cpu().numpy())


def _check(got, ref, dtype):
    names = ("dq", "dk", "dv", "d_state_in")
    for name, g, r in zip(names, got, ref):
        bf = int(dtype == torch.bfloat16 and name != "d_state_in")
        e = rel_err(to_f64(g), r, bf16_out=bf)
        assert e <= TOL[dtype], "%s error %.3g rms > %.3g" % (name, e, TOL[dtype])


# (batch, heads, seq, dim, block, dtype, with_state, with_dstate, variant)
CASES = [
    (1, 2, 256, 64, 64, torch.float32, False, False, "simt"),
    (2, 3, 300, 64, 100, torch.float32, True, True, "simt"),
    (1, 2, 129, 128, 1, torch.float32, True, False, "simt"),
    (1, 2, 513, 128, 256, torch.float32, False, True, "simt"),
    (1, 4, 1000, 128, 256, torch.bfloat16, True, True, "simt"),
    (2, 2, 640, 128, 128, torch.bfloat16, False, False, "simt"),
    (1, 1, 1, 128, 256, torch.bfloat16, True, True, "simt"),
    (1, 4, 1000, 128, 256, torch.bfloat16, True, True, "pair"),
    (2, 3, 512, 128, 256, torch.bfloat16, False, False, "pair"),
    (1, 2, 1300, 128, 256, torch.bfloat16, False, True, "pair"),
    (1, 2, 257, 128, 256, torch.bfloat16, True, False, "pair"),
    (1, 1, 1, 128, 256, torch.bfloat16, True, True, "pair"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_L%d_d%d_B%d_%s_%s_%s_%s" % (
    c[0], c[1], c[2], c[3], c[4], "bf16" if c[5] == torch.bfloat16 else "f32",
    "state" if c[6] else "zero", "dstate" if c[7] else "nodstate", c[8]))
def test_backward_matches_the_oracle(case):
    b, h, L, d, block, dtype, with_state, with_dstate, variant = case
    inp = _grads_inputs(b, h, L, d, dtype, with_state, with_dstate, seed=31)
    got = la.prefill_backward(inp["q"], inp["k"], inp["v"], inp["d_o"], inp["slopes"], block, inp["state_in"],
                              inp["d_state_out"], variant=variant)
    torch.cuda.synchronize()
    _check(got, _oracle_backward(inp), dtype)


@pytest.mark.parametrize("variant,block", [(abi.LA_VARIANT_SIMT, 64), (abi.LA_VARIANT_TCGEN05_PAIR, 256)])
def test_backward_writes_only_its_outputs(variant, block):
    b, h, L, d = 1, 2, 300, 128
    inp = _grads_inputs(b, h, L, d, torch.bfloat16, True, True, seed=32)
    outs = [guarded_empty((b, h, L, d), torch.bfloat16, DEV) for _ in range(3)]
    ds, ds_back = guarded_empty((b, h, d, d), torch.float32, DEV)
    need = abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, b, h, L, d, block, variant)
    ws, ws_back = guarded_empty((max(need, 4) // 4,), torch.float32, DEV)  # need is a multiple of 4
    st = abi.lightning_prefill_backward(
        inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(), inp["d_o"].data_ptr(), abi.LA_DTYPE_BF16,
        inp["slopes"].data_ptr(), b, h, L, d, block, inp["state_in"].data_ptr(), inp["d_state_out"].data_ptr(),
        outs[0][0].data_ptr(), outs[1][0].data_ptr(), outs[2][0].data_ptr(), ds.data_ptr(), ws.data_ptr(), need,
        torch.cuda.current_stream().cuda_stream, variant)
    assert st == abi.LA_OK, abi.last_error_message()
    torch.cuda.synchronize()
    for view, back in outs:
        assert guards_intact(back, view.numel())
    assert guards_intact(ds_back, ds.numel())
    assert guards_intact(ws_back, ws.numel())
    _check([outs[0][0], outs[1][0], outs[2][0], ds], _oracle_backward(inp), torch.bfloat16)


def test_backward_of_an_empty_sequence_passes_the_state_gradient():
    b, h, d = 1, 2, 64
    z = torch.empty((b, h, 0, d), dtype=torch.bfloat16, device=DEV)
    dso = torch.randn((b, h, d, d), device=DEV)
    dq, dk, dv, ds_in = la.prefill_backward(z, z, z, z, inputs.slopes(h, DEV), 64, None, dso)
    torch.cuda.synchronize()
    assert torch.equal(ds_in, dso)


@pytest.mark.parametrize("variant", ["simt", "pair"])
def test_m1_prefill_8k_backward_sampled_heads(variant):
    w = inputs.WORKLOADS["m1_prefill_8k"]
    inp = _grads_inputs(w.batch, w.heads, w.seq, w.dim, w.dtype, w.state_in, True, seed=w.seed)
    got = la.prefill_backward(inp["q"], inp["k"], inp["v"], inp["d_o"], inp["slopes"], w.block, inp["state_in"],
                              inp["d_state_out"], variant=variant)
    torch.cuda.synchronize()
    heads = [0, 40, 63]
    _check([t[:, heads] for t in got], _oracle_backward(inp, heads_idx=heads), w.dtype)


def test_backward_captures_into_a_cuda_graph():
    # the tensor-core passes fork onto the library's side streams and join back with events;
    # captured into a graph and replayed, they give the same gradients as the direct call
    import linear_attention_lightning_b200 as la
    torch.manual_seed(0)
    b, h, L, d, block = 1, 4, 700, 128, 256
    dev = torch.device("cuda")
    mk = lambda: (torch.randn(b, h, L, d, device=dev) / d ** 0.5).to(torch.bfloat16)
    q, k, v, d_o = mk(), mk(), mk(), mk()
    sl = torch.rand(h, device=dev) * 0.05 + 0.001
    s0 = torch.randn(b, h, d, d, device=dev) * 0.1
    dso = torch.randn(b, h, d, d, device=dev) * 0.1
    ref = la.prefill_backward(q, k, v, d_o, sl, block, s0, dso)
    torch.cuda.synchronize()
    outs = [torch.empty_like(q) for _ in range(3)] + [torch.empty_like(dso)]
    from linear_attention_lightning_b200 import abi
    need = abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, b, h, L, d, block, abi.LA_VARIANT_AUTO)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            abi.check(abi.lightning_prefill_backward(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), d_o.data_ptr(), abi.LA_DTYPE_BF16, sl.data_ptr(), b, h, L,
                d, block, s0.data_ptr(), dso.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(),
                outs[3].data_ptr(), ws.data_ptr(), need, side.cuda_stream, abi.LA_VARIANT_AUTO))
    for x in outs:
        x.zero_()
    g.replay()
    torch.cuda.synchronize()
    for got, want in zip(outs, ref):
        assert torch.equal(got, want)
    assert abi.lightning_device_status(torch.cuda.current_stream().cuda_stream) == abi.LA_OK
