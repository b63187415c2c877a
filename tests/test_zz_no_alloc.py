"""lightning_prefill_backward_noalloc: the backward entry point that takes its
scratch from a fixed array inside the library instead of a caller workspace.
Its results must equal lightning_prefill_backward's on the same inputs."""
import pytest
import torch

from linear_attention_lightning_b200 import abi, inputs
from linear_attention_lightning_b200.build import build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()
    abi.load()


def test_capacity_and_bad_requests_are_rejected_before_any_launch():
    assert abi.lightning_prefill_backward_noalloc_capacity() == 64 << 20
    # argument checks run on the host, before the scratch is looked up or anything launches
    fake = [0x10000000 * (i + 1) for i in range(8)]
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                1, 64, 131072, 96, 256, None, None, fake[5], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_AUTO)
    assert st == abi.LA_ERR_UNSUPPORTED
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                1, 64, 131072, 128, 256, None, None, fake[0], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_AUTO)
    assert st == abi.LA_ERR_INVALID_ARG  # dq overlaps q


@pytest.mark.gpu
@pytest.mark.parametrize("variant", [abi.LA_VARIANT_TCGEN05_PAIR, abi.LA_VARIANT_SIMT])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(variant):
    dev = "cuda"
    b, h, L, d, block = 1, 4, 1000, 128, 256
    need = abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, b, h, L, d, block, variant)
    assert need <= abi.lightning_prefill_backward_noalloc_capacity()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        inp = inputs.prefill_inputs(b, h, L, d, torch.bfloat16, True, seed=40 + call, device=dev)
        g = torch.Generator(device=dev).manual_seed(140 + call)
        d_o = torch.randn((b, h, L, d), generator=g, device=dev).to(torch.bfloat16)
        d_so = torch.randn((b, h, d, d), generator=g, device=dev) * 0.1
        ptrs = (inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(), d_o.data_ptr(), abi.LA_DTYPE_BF16,
                inp["slopes"].data_ptr(), b, h, L, d, block, inp["state_in"].data_ptr(), d_so.data_ptr())
        ref = [torch.empty_like(inp["q"]) for _ in range(3)] + [torch.empty_like(d_so)]
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        st = abi.lightning_prefill_backward(*ptrs, *(t.data_ptr() for t in ref), ws.data_ptr(), need, stream,
                                            variant)
        assert st == abi.LA_OK, abi.last_error_message()
        got = [torch.empty_like(t) for t in ref]
        st = abi.lightning_prefill_backward_noalloc(*ptrs, *(t.data_ptr() for t in got), stream, variant)
        assert st == abi.LA_OK, abi.last_error_message()
        torch.cuda.synchronize()
        for r, g_ in zip(ref, got):
            assert torch.equal(r, g_)
