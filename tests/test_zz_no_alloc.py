"""lightning_prefill_backward_noalloc: the backward entry point for callers that
cannot allocate device memory themselves (a runtime whose allocator owns all
of the device's memory, or a plugin that may not call cudaMalloc). It takes the
scratch the tensor-core passes need (their range-guard records) from a fixed
array inside the library instead of a caller workspace, and its results must
equal lightning_prefill_backward's on the same inputs.

This file is collected last, so that a run stopping at the first failure has
run every other test before it."""
import pytest
import torch

from linear_attention_lightning_b200 import abi, inputs
from linear_attention_lightning_b200.build import build

CAPACITY = 4 << 20


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()
    abi.load()


def test_capacity_and_bad_requests_are_rejected_before_any_launch():
    assert abi.lightning_prefill_backward_noalloc_capacity() == CAPACITY
    # argument checks run on the host, in lightning_prefill_backward's order, before
    # the scratch is looked up or anything launches
    fake = [0x10000000 * (i + 1) for i in range(8)]
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                1, 64, 131072, 96, 256, None, None, fake[5], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_AUTO)
    assert st == abi.LA_ERR_UNSUPPORTED and "dim 96" in abi.last_error_message()  # the shape check
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                1, 64, 131072, 128, 256, None, None, fake[0], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_AUTO)
    assert st == abi.LA_ERR_INVALID_ARG  # dq overlaps q
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                1, 64, 16, 128, 256, None, None, fake[5], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_TCGEN05)
    assert st == abi.LA_ERR_INVALID_ARG  # not a backward variant
    # more (batch, head) pairs than the array holds records for: 3 x 456 x 64 x 48 bytes > 4 MiB
    st = abi.lightning_prefill_backward_noalloc(fake[0], fake[1], fake[2], fake[3], abi.LA_DTYPE_BF16, fake[4],
                                                456, 64, 16, 128, 256, None, None, fake[5], fake[6], fake[7],
                                                None, None, abi.LA_VARIANT_AUTO)
    assert st == abi.LA_ERR_UNSUPPORTED and "scratch" in abi.last_error_message()
    assert abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, 456, 64, 16, 128, 256,
                                                         abi.LA_VARIANT_AUTO) > CAPACITY
    assert abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, 455, 64, 16, 128, 256,
                                                         abi.LA_VARIANT_AUTO) <= CAPACITY


@pytest.mark.gpu
@pytest.mark.parametrize("variant", [abi.LA_VARIANT_TCGEN05_PAIR, abi.LA_VARIANT_SIMT])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(variant):
    dev = "cuda"
    b, h, L, d, block = 1, 4, 1000, 128, 256
    need = abi.lightning_prefill_backward_workspace_size(abi.LA_DTYPE_BF16, b, h, L, d, block, variant)
    assert need <= abi.lightning_prefill_backward_noalloc_capacity()
    if variant == abi.LA_VARIANT_TCGEN05_PAIR:
        assert need > 0  # the tensor-core passes keep their records in the library's array
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
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
