"""The failure-detection path on the GPU, without a fault: a bounded device-side
wait that is never satisfied runs out, the kernel records LA_ERR_TIMEOUT in the
status word and returns, and the context stays usable. The failure is reported
on demand (lightning_last_device_status) and by the next call that would
launch work, which then launches nothing."""
import time

import pytest
import torch

from linear_attention_lightning_b200 import abi, inputs

from parity import TOL, oracle_prefill, rel_err, to_f64
import linear_attention_lightning_b200 as la

pytestmark = pytest.mark.gpu


def _tiny():
    w = inputs.WORKLOADS["tiny_prefill_f32"]
    return w, inputs.workload_inputs(w, torch.device("cuda"))


def _prefill_call(w, inp, o, s_out, stream):
    # the float32 workload runs on CUDA cores: no workspace
    return abi.lightning_prefill_ex(
        inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(), abi.LA_DTYPE_F32, inp["slopes"].data_ptr(),
        w.batch, w.heads, w.seq, w.dim, w.block, None, o.data_ptr(), s_out.data_ptr(), None, 0, stream,
        abi.LA_VARIANT_AUTO)


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
    t0 = time.time()
    abi.check(abi.lightning_selftest_wait_timeout(stream))
    assert abi.lightning_last_device_status(stream) == abi.LA_ERR_TIMEOUT
    assert "gave up" in abi.last_error_message()
    assert time.time() - t0 < 60.0                       # the wait is bounded
    assert abi.lightning_last_device_status(stream) == abi.LA_OK  # the word was cleared
    assert abi.lightning_device_status(stream) == abi.LA_OK       # the earlier name reads the same word
    # the context still runs a prefill correctly
    w, inp = _tiny()
    o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, inp["state_in"])
    torch.cuda.synchronize()
    ref_o, _ = oracle_prefill(inp)
    assert rel_err(to_f64(o), ref_o) <= TOL[w.dtype]
    assert abi.lightning_last_device_status(stream) == abi.LA_OK


def test_a_timeout_is_returned_by_the_next_launching_call_which_launches_nothing():
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
    w, inp = _tiny()
    o = torch.full_like(inp["q"], float("nan"))
    s_out = torch.full((w.batch, w.heads, w.dim, w.dim), float("nan"), device="cuda")
    abi.check(abi.lightning_selftest_wait_timeout(stream))
    torch.cuda.synchronize()  # the wait has run out by now (no status query in between)
    assert _prefill_call(w, inp, o, s_out, stream) == abi.LA_ERR_TIMEOUT
    assert "gave up" in abi.last_error_message()
    torch.cuda.synchronize()
    assert torch.isnan(o).all() and torch.isnan(s_out).all()   # nothing was launched
    # the word was cleared by that call: the next one runs, to parity
    assert _prefill_call(w, inp, o, s_out, stream) == abi.LA_OK
    torch.cuda.synchronize()
    ref_o, ref_s = oracle_prefill(inp)
    assert rel_err(to_f64(o), ref_o) <= TOL[w.dtype]
    assert rel_err(to_f64(s_out), ref_s) <= TOL[w.dtype]
    assert abi.lightning_last_device_status(stream) == abi.LA_OK


def test_a_timeout_reaches_a_decode_call_too():
    stream = torch.cuda.current_stream().cuda_stream
    b, h, d = 2, 3, 128
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v = (torch.randn((b, h, d), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    sl = torch.full((h,), 0.1, device="cuda")
    state = torch.zeros((b, h, d, d), device="cuda")
    abi.check(abi.lightning_selftest_wait_timeout(stream))
    torch.cuda.synchronize()
    with pytest.raises(abi.LightningError) as info:
        la.decode(q, k, v, sl, state)
    assert info.value.status == abi.LA_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert torch.count_nonzero(state) == 0     # the state was not touched
    la.decode(q, k, v, sl, state)
    torch.cuda.synchronize()
    assert torch.count_nonzero(state) > 0
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
