"""The library's calls capture into CUDA graphs: a serving loop replays one prefill
and a run of decode steps without host work per launch. A tensor-core prefill call is
two launches, the second one the first's programmatic dependent, and a range-guarded
call may also run a cluster launch. Captured and replayed, each call gives exactly what
the direct call gives."""
import pytest
import torch

import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF = torch.bfloat16


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn(side.cuda_stream)
    torch.cuda.current_stream().wait_stream(side)
    return g


@pytest.mark.parametrize("variant,block,in_place", [("pair", 256, False), ("tcgen05", 128, False),
                                                    ("tcgen05", 256, True)])
def test_prefill_replays_like_the_direct_call(variant, block, in_place):
    b, h, L, d = 2, 8, 1000, 128
    inp = inputs.prefill_inputs(b, h, L, d, BF, True, seed=81, device=DEV)
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["slopes"]
    s0 = inp["state_in"]
    ref_o, ref_s = la.prefill(q, k, v, sl, block, s0.clone(), variant=variant)
    torch.cuda.synchronize()
    o = torch.empty_like(q)
    s_io = s0.clone()
    s_out = s_io if in_place else torch.empty_like(s0)
    need = abi.lightning_prefill_workspace_size(b, h, L, d, block)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=DEV)
    vcode = {"pair": abi.LA_VARIANT_TCGEN05_PAIR, "tcgen05": abi.LA_VARIANT_TCGEN05}[variant]
    g = _capture(lambda st: abi.check(abi.lightning_prefill_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), abi.LA_DTYPE_BF16, sl.data_ptr(), b, h, L, d, block,
        s_io.data_ptr(), o.data_ptr(), s_out.data_ptr(), ws.data_ptr(), need, st, vcode)))
    for _ in range(2):
        s_io.copy_(s0)  # an in-place carry consumes its state: start each replay from the same one
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o)
        assert torch.equal(s_out, ref_s)
    assert abi.lightning_last_device_status(torch.cuda.current_stream().cuda_stream) == abi.LA_OK


def test_decode_steps_replay_like_direct_steps():
    b, h, d, steps = 8, 64, 128, 16
    w = inputs.WORKLOADS["batched_decode"]
    inp = inputs.workload_inputs(w, DEV, batch=b, steps=steps)  # q, k, v: [steps, b, H, d]
    state0 = inp["state"].clone()
    qs, ks, vs, sl = inp["q"], inp["k"], inp["v"], inp["slopes"]
    # direct
    st = state0.clone()
    ref = []
    for i in range(steps):
        ref.append(la.decode(qs[i], ks[i], vs[i], sl, st))
    torch.cuda.synchronize()
    # captured: the whole run of steps as one graph
    st2 = state0.clone()
    outs = [torch.empty_like(r) for r in ref]

    def run(stream):
        for i in range(steps):
            abi.check(abi.lightning_decode(qs[i].data_ptr(), ks[i].data_ptr(), vs[i].data_ptr(), abi.LA_DTYPE_BF16,
                                           sl.data_ptr(), b, h, d, st2.data_ptr(), outs[i].data_ptr(), stream))
    g = _capture(run)
    st2.copy_(state0)
    g.replay()
    torch.cuda.synchronize()
    for a, r in zip(outs, ref):
        assert torch.equal(a, r)
    assert torch.equal(st2, st)
