"""The longest sequences: 2^20 tokens of two heads (4096 blocks of 256), eight times the
long-context workload, with a carried-in state, against the float64 oracle's token
recurrence. Positions, offsets and block counts run past what the workloads reach; o is
compared on a seeded sample of rows spread over the whole sequence and on the last rows,
the state after the last token in full."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import inputs

from parity import TOL, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
L = 1 << 20


@pytest.fixture(scope="module")
def case():
    inp = inputs.prefill_inputs(1, 2, L, 128, torch.bfloat16, True, seed=91, device=DEV)
    conv = inputs.to_oracle
    ref_o, ref_s = oracle.prefill(conv(inp["q"]), conv(inp["k"]), conv(inp["v"]), inp["slopes"].cpu().numpy(),
                                  inp["state_in"].cpu().numpy())
    rows = np.sort(np.random.default_rng(91).choice(L, 4096, replace=False))
    rows = np.unique(np.concatenate([rows, np.arange(L - 1024, L)]))
    return inp, ref_o[:, :, rows], ref_s, rows


@pytest.mark.parametrize("variant,block", [("pair", 256), ("tcgen05", 256), ("tcgen05", 128)])
def test_two_to_the_twenty_tokens(case, variant, block):
    inp, ref_o, ref_s, rows = case
    o, s = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], block, inp["state_in"], variant=variant)
    torch.cuda.synchronize()
    got = to_f64(o[:, :, torch.as_tensor(rows, device=DEV)])
    # the tolerance is relative to the rms of the sampled rows (the whole o is not kept)
    assert rel_err(got, ref_o, bf16_out=1) <= TOL[torch.bfloat16]
    assert rel_err(to_f64(s), ref_s) <= TOL[torch.bfloat16]
    assert la.abi.lightning_last_device_status(torch.cuda.current_stream().cuda_stream) == la.abi.LA_OK
