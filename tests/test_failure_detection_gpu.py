"""The failure-detection path on the GPU, without a fault: a bounded device-side
wait that is never satisfied runs out, the kernel records LA_ERR_TIMEOUT in the
device status word and returns, and the context stays usable."""
import time

import pytest
import torch

from linear_attention_lightning_b200 import abi, inputs

from parity import TOL, oracle_prefill, rel_err, to_f64
import linear_attention_lightning_b200 as la

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_device_status(stream) == abi.LA_OK
    t0 = time.time()
    abi.check(abi.lightning_selftest_wait_timeout(stream))
    assert abi.lightning_device_status(stream) == abi.LA_ERR_TIMEOUT
    assert "gave up" in abi.last_error_message()
    assert time.time() - t0 < 60.0                       # the wait is bounded
    assert abi.lightning_device_status(stream) == abi.LA_OK  # the word was cleared
    # the context still runs a prefill correctly
    w = inputs.WORKLOADS["tiny_prefill_f32"]
    inp = inputs.workload_inputs(w, torch.device("cuda"))
    o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, inp["state_in"])
    torch.cuda.synchronize()
    ref_o, _ = oracle_prefill(inp)
    assert rel_err(to_f64(o), ref_o) <= TOL[w.dtype]
    assert abi.lightning_device_status(stream) == abi.LA_OK
