"""Host-only checks of the C ABI: the library loads, exports everything the
header declares, and rejects bad arguments before launching anything.

No call here reaches a kernel launch, so these run without a GPU.
"""
import ctypes

import pytest

from linear_attention_lightning_b200 import abi
from linear_attention_lightning_b200.build import build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()
    abi.load()


def test_every_declared_function_is_exported():
    lib = ctypes.CDLL(abi.LIBRARY)
    declared = abi.declared_functions()
    assert "lightning_prefill" in declared and "lightning_decode" in declared
    for name in declared:
        assert hasattr(lib, name), name
        assert name in abi._SIGNATURES, "binding lacks " + name


def test_version_and_status_strings():
    assert abi.lightning_abi_version() == 2
    for st in range(5):
        assert abi.status_string(st).startswith("LA_")
    assert abi.status_string(99) == "unknown status"


def test_prefill_workspace_holds_the_range_guard_records():
    # 48 bytes per (batch, head) for the tensor-core kernels (dim 128: the CTA pair at
    # block 256, the single-CTA kernel at block 128); none for the CUDA-core kernel
    assert abi.lightning_prefill_workspace_size(16, 64, 4096, 128, 256) == 16 * 64 * 48
    assert abi.lightning_prefill_workspace_size(1, 64, 131072, 128, 256) == 64 * 48
    assert abi.lightning_prefill_workspace_size(1, 2, 256, 64, 64) == 0
    assert abi.lightning_prefill_workspace_size(1, 2, 256, 128, 128) == 2 * 48
    assert abi.lightning_prefill_workspace_size(-1, 2, 256, 128, 256) == 0


# Fake, well-aligned, non-overlapping "device" addresses: every call below must
# be rejected (or finish trivially) before any CUDA call is made.
Q, K, V, O, SL, S0, S1 = (0x10000000 * (i + 1) for i in range(7))
PWS = 0x10000000 * 40  # fake prefill workspace
GOOD = dict(q=Q, k=K, v=V, dtype=abi.LA_DTYPE_BF16, slopes=SL, batch=1, heads=2, seq=16, dim=128,
            block=256, state_in=S0, o=O, state_out=S1, pws=PWS, pws_bytes=4096)


def _prefill(variant=abi.LA_VARIANT_AUTO, **kw):
    a = dict(GOOD)
    a.update(kw)
    return abi.lightning_prefill_ex(a["q"], a["k"], a["v"], a["dtype"], a["slopes"], a["batch"],
                                    a["heads"], a["seq"], a["dim"], a["block"], a["state_in"], a["o"],
                                    a["state_out"], a["pws"], a["pws_bytes"], None, variant)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=7), abi.LA_ERR_INVALID_ARG),
    (dict(batch=-1), abi.LA_ERR_INVALID_ARG),
    (dict(heads=0), abi.LA_ERR_INVALID_ARG),
    (dict(seq=-3), abi.LA_ERR_INVALID_ARG),
    (dict(block=0), abi.LA_ERR_INVALID_ARG),
    (dict(dim=96), abi.LA_ERR_UNSUPPORTED),
    (dict(q=None), abi.LA_ERR_INVALID_ARG),
    (dict(o=None), abi.LA_ERR_INVALID_ARG),
    (dict(slopes=None), abi.LA_ERR_INVALID_ARG),
    (dict(k=K + 8), abi.LA_ERR_INVALID_ARG),            # misaligned
    (dict(state_out=S1 + 4), abi.LA_ERR_INVALID_ARG),   # misaligned
    (dict(o=Q + 256), abi.LA_ERR_INVALID_ARG),          # o overlaps q
    (dict(state_out=V), abi.LA_ERR_INVALID_ARG),        # state overlaps v
    (dict(state_out=S0 + 4096), abi.LA_ERR_INVALID_ARG),  # partial overlap with state_in
    (dict(pws=None, pws_bytes=0), abi.LA_ERR_INVALID_ARG),  # the CTA-pair kernel needs its workspace
    (dict(pws_bytes=48), abi.LA_ERR_INVALID_ARG),           # 2 heads need 96 bytes (48 each)
    (dict(pws=PWS + 8), abi.LA_ERR_INVALID_ARG),            # misaligned workspace
    (dict(pws=V + 64), abi.LA_ERR_INVALID_ARG),             # workspace overlaps v
])
def test_prefill_argument_errors(kw, status):
    assert _prefill(**kw) == status
    assert abi.last_error_message() != ""


def test_prefill_trivial_calls_need_no_gpu():
    assert _prefill(batch=0) == abi.LA_OK
    assert _prefill(seq=0, state_out=None) == abi.LA_OK


@pytest.mark.parametrize("block", [128, 256])
def test_single_cta_kernel_needs_its_workspace(block):
    tc = abi.LA_VARIANT_TCGEN05
    assert _prefill(variant=tc, block=block, pws=None, pws_bytes=0) == abi.LA_ERR_INVALID_ARG
    assert "workspace" in abi.last_error_message()
    assert _prefill(variant=tc, block=block, pws_bytes=48) == abi.LA_ERR_INVALID_ARG  # 2 heads need 96
    # the CUDA-core kernel takes none
    assert _prefill(variant=abi.LA_VARIANT_SIMT, block=block, pws=None, pws_bytes=0, batch=0) == abi.LA_OK


def test_unknown_variant_and_unsupported_tensor_core_requests():
    assert _prefill(variant=9) == abi.LA_ERR_INVALID_ARG
    assert _prefill(variant=abi.LA_VARIANT_TCGEN05, dtype=abi.LA_DTYPE_F32) == abi.LA_ERR_UNSUPPORTED
    assert _prefill(variant=abi.LA_VARIANT_TCGEN05, dim=64) == abi.LA_ERR_UNSUPPORTED
    assert _prefill(variant=abi.LA_VARIANT_TCGEN05, block=192) == abi.LA_ERR_UNSUPPORTED
    assert _prefill(variant=abi.LA_VARIANT_TCGEN05_PAIR, block=128) == abi.LA_ERR_UNSUPPORTED


def test_variant_selection():
    sel = abi.lightning_prefill_selected_variant
    assert sel(abi.LA_DTYPE_F32, 1, 2, 256, 64, 64, abi.LA_VARIANT_AUTO) == abi.LA_VARIANT_SIMT
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 8192, 128, 256, abi.LA_VARIANT_SIMT) == abi.LA_VARIANT_SIMT
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 8192, 96, 256, abi.LA_VARIANT_AUTO) == -1
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 131072, 128, 256, abi.LA_VARIANT_AUTO) == abi.LA_VARIANT_TCGEN05_PAIR
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 131072, 128, 128, abi.LA_VARIANT_AUTO) == abi.LA_VARIANT_TCGEN05
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 131072, 128, 128, abi.LA_VARIANT_TCGEN05_PAIR) == -1
    assert sel(abi.LA_DTYPE_BF16, 1, 64, 4096, 128, 256, abi.LA_VARIANT_TCGEN05) == abi.LA_VARIANT_TCGEN05


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=5), abi.LA_ERR_INVALID_ARG),
    (dict(dim=32), abi.LA_ERR_UNSUPPORTED),
    (dict(state=None), abi.LA_ERR_INVALID_ARG),
    (dict(o=S1 + 8), abi.LA_ERR_INVALID_ARG),
    (dict(o=S1 + 1024), abi.LA_ERR_INVALID_ARG),   # o inside the state
    (dict(state=Q), abi.LA_ERR_INVALID_ARG),       # state overlaps q
])
def test_decode_argument_errors(kw, status):
    a = dict(q=Q, k=K, v=V, dtype=abi.LA_DTYPE_BF16, slopes=SL, batch=2, heads=4, dim=128, state=S1, o=O)
    a.update(kw)
    st = abi.lightning_decode(a["q"], a["k"], a["v"], a["dtype"], a["slopes"], a["batch"], a["heads"],
                              a["dim"], a["state"], a["o"], None)
    assert st == status


def test_decode_empty_batch_is_a_no_op():
    assert abi.lightning_decode(Q, K, V, abi.LA_DTYPE_BF16, SL, 0, 4, 128, S1, O, None) == abi.LA_OK


SN = 0x10000000 * 9  # fake snapshot buffer address, clear of the others


def _prefill_snapshots(interval=256, snapshots=SN, variant=abi.LA_VARIANT_AUTO, **kw):
    a = dict(GOOD, seq=1024)
    a.update(kw)
    return abi.lightning_prefill_snapshots(a["q"], a["k"], a["v"], a["dtype"], a["slopes"], a["batch"],
                                           a["heads"], a["seq"], a["dim"], a["block"], a["state_in"], a["o"],
                                           a["state_out"], interval, snapshots, a["pws"], a["pws_bytes"], None,
                                           variant)


def test_snapshot_count():
    assert abi.lightning_prefill_snapshot_count(1024, 256) == 4
    assert abi.lightning_prefill_snapshot_count(1000, 256) == 3
    assert abi.lightning_prefill_snapshot_count(100, 256) == 0
    assert abi.lightning_prefill_snapshot_count(0, 256) == 0
    assert abi.lightning_prefill_snapshot_count(-1, 256) == -1
    assert abi.lightning_prefill_snapshot_count(16, 0) == -1


@pytest.mark.parametrize("kw,status", [
    (dict(interval=0), abi.LA_ERR_INVALID_ARG),
    (dict(interval=-256), abi.LA_ERR_INVALID_ARG),
    (dict(interval=128), abi.LA_ERR_INVALID_ARG),           # shorter than the block
    (dict(interval=384), abi.LA_ERR_INVALID_ARG),           # not a multiple of the block
    (dict(snapshots=None), abi.LA_ERR_INVALID_ARG),         # 4 snapshots but no buffer
    (dict(snapshots=SN + 8), abi.LA_ERR_INVALID_ARG),       # misaligned
    (dict(snapshots=Q + 4096), abi.LA_ERR_INVALID_ARG),     # overlaps q
    (dict(snapshots=O), abi.LA_ERR_INVALID_ARG),            # overlaps o
    (dict(snapshots=S1 - 4096), abi.LA_ERR_INVALID_ARG),    # runs into state_out
    (dict(dim=96), abi.LA_ERR_UNSUPPORTED),
    (dict(variant=abi.LA_VARIANT_TCGEN05_PAIR, block=128, interval=128), abi.LA_ERR_UNSUPPORTED),
])
def test_snapshot_argument_errors(kw, status):
    assert _prefill_snapshots(**kw) == status
    assert abi.last_error_message() != ""


def test_snapshot_trivial_calls_need_no_gpu():
    assert _prefill_snapshots(batch=0) == abi.LA_OK
    # an empty sequence takes no snapshot, so the buffer may be NULL
    assert _prefill_snapshots(seq=0, state_out=None, snapshots=None) == abi.LA_OK


DO, DQ, DK, DV, DSI, DSO, WS = (0x10000000 * (i + 10) for i in range(7))
WS_BYTES = 1 << 26


def _backward(variant=abi.LA_VARIANT_AUTO, **kw):
    a = dict(GOOD, d_o=DO, d_state_out=DSO, dq=DQ, dk=DK, dv=DV, d_state_in=DSI, ws=WS, ws_bytes=WS_BYTES)
    a.update(kw)
    return abi.lightning_prefill_backward(a["q"], a["k"], a["v"], a["d_o"], a["dtype"], a["slopes"], a["batch"],
                                          a["heads"], a["seq"], a["dim"], a["block"], a["state_in"],
                                          a["d_state_out"], a["dq"], a["dk"], a["dv"], a["d_state_in"],
                                          a["ws"], a["ws_bytes"], None, variant)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=5), abi.LA_ERR_INVALID_ARG),
    (dict(block=0), abi.LA_ERR_INVALID_ARG),
    (dict(dim=48), abi.LA_ERR_UNSUPPORTED),
    (dict(d_o=None), abi.LA_ERR_INVALID_ARG),
    (dict(dk=None), abi.LA_ERR_INVALID_ARG),
    (dict(slopes=None), abi.LA_ERR_INVALID_ARG),
    (dict(dv=DV + 4), abi.LA_ERR_INVALID_ARG),           # misaligned
    (dict(dq=Q + 512), abi.LA_ERR_INVALID_ARG),          # output overlaps q
    (dict(dk=DO), abi.LA_ERR_INVALID_ARG),               # output overlaps d_o
    (dict(dv=DQ + 1024), abi.LA_ERR_INVALID_ARG),        # two outputs overlap
    (dict(d_state_in=DSO), abi.LA_ERR_INVALID_ARG),      # overlaps d_state_out
    (dict(d_state_in=S0 + 16), abi.LA_ERR_INVALID_ARG),  # overlaps state_in
    (dict(variant=abi.LA_VARIANT_TCGEN05), abi.LA_ERR_INVALID_ARG),
    (dict(variant=7), abi.LA_ERR_INVALID_ARG),
    (dict(variant=abi.LA_VARIANT_TCGEN05_PAIR, block=128), abi.LA_ERR_UNSUPPORTED),
])
def test_backward_argument_errors(kw, status):
    assert _backward(**kw) == status
    assert abi.last_error_message() != ""


def test_backward_workspace_size():
    ws = abi.lightning_prefill_backward_workspace_size
    # the three tensor-core passes keep one range-guard record (48 bytes) per (batch, head)
    # each; the CUDA-core passes need no workspace
    assert ws(abi.LA_DTYPE_BF16, 1, 64, 131072, 128, 256, abi.LA_VARIANT_AUTO) == 3 * 64 * 48
    assert ws(abi.LA_DTYPE_BF16, 2, 64, 131072, 128, 256, abi.LA_VARIANT_TCGEN05_PAIR) == 3 * 2 * 64 * 48
    for dt, blk, var in ((abi.LA_DTYPE_BF16, 256, abi.LA_VARIANT_SIMT), (abi.LA_DTYPE_F32, 64, abi.LA_VARIANT_AUTO)):
        assert ws(dt, 1, 64, 131072, 128, blk, var) == 0
    assert _backward(ws=None, ws_bytes=0, batch=0) == abi.LA_OK
    assert _backward(ws=None, ws_bytes=0) == abi.LA_ERR_INVALID_ARG          # the tensor-core passes need it
    assert _backward(ws_bytes=3 * 2 * 48 - 16) == abi.LA_ERR_INVALID_ARG     # 2 heads need 288 bytes


def test_backward_trivial_calls_need_no_gpu():
    assert _backward(batch=0) == abi.LA_OK
    assert _backward(seq=0, d_state_in=None) == abi.LA_OK


G_, GM, Y_ = (0x10000000 * (i + 20) for i in range(3))


def _norm_gate(**kw):
    a = dict(o=O, gate=G_, dtype=abi.LA_DTYPE_BF16, gamma=GM, eps=1e-6, batch=1, heads=64, seq=16, dim=128,
             per_head=0, y=Y_)
    a.update(kw)
    return abi.lightning_norm_gate(a["o"], a["gate"], a["dtype"], a["gamma"], a["eps"], a["batch"], a["heads"],
                                   a["seq"], a["dim"], a["per_head"], a["y"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=3), abi.LA_ERR_INVALID_ARG),
    (dict(heads=0), abi.LA_ERR_INVALID_ARG),
    (dict(seq=-1), abi.LA_ERR_INVALID_ARG),
    (dict(eps=-1.0), abi.LA_ERR_INVALID_ARG),
    (dict(eps=float("nan")), abi.LA_ERR_INVALID_ARG),
    (dict(dim=32), abi.LA_ERR_UNSUPPORTED),
    (dict(heads=129), abi.LA_ERR_UNSUPPORTED),                           # 16512 bf16 channels per token
    (dict(heads=65, dtype=abi.LA_DTYPE_F32), abi.LA_ERR_UNSUPPORTED),    # 8320 f32 channels
    (dict(gate=None), abi.LA_ERR_INVALID_ARG),
    (dict(gate=G_ + 8), abi.LA_ERR_INVALID_ARG),  # the kernel reads the gate by 16-byte loads and a bulk L2 prefetch
    (dict(y=Y_ + 4), abi.LA_ERR_INVALID_ARG),
    (dict(y=O + 1024), abi.LA_ERR_INVALID_ARG),                          # overlaps o
    (dict(y=G_ + 1024), abi.LA_ERR_INVALID_ARG),                         # overlaps the gate
])
def test_norm_gate_argument_errors(kw, status):
    assert _norm_gate(**kw) == status
    assert abi.last_error_message() != ""


def test_norm_gate_empty_needs_no_gpu():
    assert _norm_gate(batch=0) == abi.LA_OK
    assert _norm_gate(seq=0, o=None, y=None) == abi.LA_OK


def _prefill_norm_gate(**kw):
    a = dict(GOOD, gate=G_, gamma=GM, eps=1e-6, y=Y_)
    a.update(kw)
    return abi.lightning_prefill_norm_gate(a["q"], a["k"], a["v"], a["dtype"], a["slopes"], a["batch"], a["heads"],
                                           a["seq"], a["dim"], a["block"], a["state_in"], a["gate"], a["gamma"],
                                           a["eps"], a["y"], a["state_out"], a["pws"], a["pws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=5), abi.LA_ERR_INVALID_ARG),
    (dict(heads=0), abi.LA_ERR_INVALID_ARG),
    (dict(seq=-2), abi.LA_ERR_INVALID_ARG),
    (dict(dtype=abi.LA_DTYPE_F32), abi.LA_ERR_UNSUPPORTED),      # the CTA-pair kernel only
    (dict(block=128), abi.LA_ERR_UNSUPPORTED),
    (dict(dim=64), abi.LA_ERR_UNSUPPORTED),
    (dict(eps=-1.0), abi.LA_ERR_INVALID_ARG),
    (dict(eps=float("inf")), abi.LA_ERR_INVALID_ARG),
    (dict(y=None), abi.LA_ERR_INVALID_ARG),
    (dict(gate=None), abi.LA_ERR_INVALID_ARG),
    (dict(gamma=None), abi.LA_ERR_INVALID_ARG),
    (dict(gate=G_ + 2), abi.LA_ERR_INVALID_ARG),                  # misaligned
    (dict(y=Q + 512), abi.LA_ERR_INVALID_ARG),                    # y overlaps q
    (dict(y=G_ + 1024), abi.LA_ERR_INVALID_ARG),                  # y overlaps the gate
    (dict(gamma=Y_ + 64), abi.LA_ERR_INVALID_ARG),                # y overlaps gamma
    (dict(state_out=G_ + 256), abi.LA_ERR_INVALID_ARG),           # state_out overlaps the gate
])
def test_prefill_norm_gate_argument_errors(kw, status):
    assert _prefill_norm_gate(**kw) == status
    assert abi.last_error_message() != ""


def test_prefill_norm_gate_trivial_calls_need_no_gpu():
    assert _prefill_norm_gate(batch=0) == abi.LA_OK
    assert _prefill_norm_gate(seq=0, state_out=None, y=None, gate=None, gamma=None) == abi.LA_OK


def _gqa(**kw):
    a = dict(q=Q, kn=K, vn=V, kc=0x10000000 * 30, vc=0x10000000 * 40, dtype=abi.LA_DTYPE_BF16, pos=SL, batch=2,
             heads=64, kv=8, dim=128, cap=1024, rot=64, base=1e4, scale=0.088, o=O, ws=WS, ws_bytes=1 << 26)
    a.update(kw)
    return abi.lightning_gqa_decode(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["dtype"], a["pos"], a["batch"],
                                    a["heads"], a["kv"], a["dim"], a["cap"], a["rot"], a["base"], a["scale"], a["o"],
                                    a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=9), abi.LA_ERR_INVALID_ARG),
    (dict(kv=7), abi.LA_ERR_INVALID_ARG),               # does not divide 64
    (dict(cap=0), abi.LA_ERR_INVALID_ARG),
    (dict(dim=64), abi.LA_ERR_UNSUPPORTED),
    (dict(kv=4, dtype=abi.LA_DTYPE_F32), abi.LA_ERR_UNSUPPORTED),  # 16 query heads per KV head, float32
    (dict(kv=1), abi.LA_ERR_UNSUPPORTED),               # 64 query heads per KV head
    (dict(rot=63), abi.LA_ERR_INVALID_ARG),
    (dict(rot=130), abi.LA_ERR_INVALID_ARG),
    (dict(base=0.0), abi.LA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), abi.LA_ERR_INVALID_ARG),
    (dict(pos=None), abi.LA_ERR_INVALID_ARG),
    (dict(ws_bytes=64), abi.LA_ERR_INVALID_ARG),        # workspace too small
    (dict(o=Q), abi.LA_ERR_INVALID_ARG),                # o is q
    (dict(kc=0x10000000 * 40), abi.LA_ERR_INVALID_ARG), # k_cache is v_cache
    (dict(vc=0x10000000 * 40 + 8), abi.LA_ERR_INVALID_ARG),
])
def test_gqa_decode_argument_errors(kw, status):
    assert _gqa(**kw) == status
    assert abi.last_error_message() != ""


def test_gqa_workspace_size_and_empty_batch():
    # per (sequence, query head, 2048-position chunk): max, sum, 128 weighted values;
    # per (sequence, query head): the rotated, scaled query
    n = 2 * 64 * 1
    assert abi.lightning_gqa_decode_workspace_size(2, 64, 1024) == n * 4 + n * 4 + n * 128 * 4 + 2 * 64 * 128 * 4
    assert abi.lightning_gqa_decode_workspace_size(0, 64, 1024) == 0
    assert _gqa(batch=0) == abi.LA_OK


ST = 0x10000000 * 50  # fake device start[batch] array


def _gqp(**kw):
    # sizes: q, o 2 x 64 x 512 x 128 bf16 = 16 MiB; caches 2 x 8 x 1024 x 128 bf16 = 4 MiB (fake addresses 256 MiB apart)
    a = dict(q=Q, kn=K, vn=V, kc=0x10000000 * 30, vc=0x10000000 * 40, dtype=abi.LA_DTYPE_BF16, start=ST, batch=2,
             heads=64, kv=8, seq=512, dim=128, cap=1024, rot=64, base=1e4, scale=0.088, o=O, ws=WS, ws_bytes=1 << 26)
    a.update(kw)
    return abi.lightning_gqa_prefill(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["dtype"], a["start"], a["batch"],
                                     a["heads"], a["kv"], a["seq"], a["dim"], a["cap"], a["rot"], a["base"],
                                     a["scale"], a["o"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype=9), abi.LA_ERR_INVALID_ARG),
    (dict(kv=7), abi.LA_ERR_INVALID_ARG),                     # does not divide 64
    (dict(start=None), abi.LA_ERR_INVALID_ARG),               # the device start array is required
    (dict(start=ST + 4), abi.LA_ERR_INVALID_ARG),             # not 16-byte aligned
    (dict(o=ST), abi.LA_ERR_INVALID_ARG),                     # o overlaps start
    (dict(seq=-3), abi.LA_ERR_INVALID_ARG),
    (dict(seq=1025), abi.LA_ERR_INVALID_ARG),                 # seq > cap
    (dict(dim=64), abi.LA_ERR_UNSUPPORTED),
    (dict(rot=62), abi.LA_ERR_INVALID_ARG),                   # not a multiple of 4
    (dict(rot=132), abi.LA_ERR_INVALID_ARG),
    (dict(base=-1.0), abi.LA_ERR_INVALID_ARG),
    (dict(scale=0.0), abi.LA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), abi.LA_ERR_INVALID_ARG),
    (dict(batch=70000, seq=1, cap=2), abi.LA_ERR_UNSUPPORTED),
    (dict(kn=None), abi.LA_ERR_INVALID_ARG),
    (dict(q=Q + 8), abi.LA_ERR_INVALID_ARG),                  # not 16-byte aligned
    (dict(ws_bytes=1 << 20), abi.LA_ERR_INVALID_ARG),         # workspace too small
    (dict(o=Q + (1 << 20)), abi.LA_ERR_INVALID_ARG),          # o overlaps q
    (dict(ws=0x10000000 * 30 + 4096), abi.LA_ERR_INVALID_ARG),  # workspace overlaps k_cache
    (dict(vc=0x10000000 * 30 + 1024), abi.LA_ERR_INVALID_ARG),  # caches overlap
])
def test_gqa_prefill_argument_errors(kw, status):
    assert _gqp(**kw) == status
    assert abi.last_error_message() != ""


def test_gqa_prefill_workspace_size_and_empty_calls():
    # the rotated queries, bf16, q's shape
    bf, f32 = abi.LA_DTYPE_BF16, abi.LA_DTYPE_F32
    assert abi.lightning_gqa_prefill_workspace_size(bf, 2, 64, 512, 128) == 2 * 64 * 512 * 128 * 2
    assert abi.lightning_gqa_prefill_workspace_size(f32, 2, 64, 512, 128) == 2 * 64 * 512 * 128 * 4
    assert abi.lightning_gqa_prefill_workspace_size(bf, 2, 64, 512, 64) == 0
    assert abi.lightning_gqa_prefill_workspace_size(bf, -1, 64, 512, 128) == 0
    assert abi.lightning_gqa_prefill_workspace_size(7, 2, 64, 512, 128) == 0
    assert _gqp(batch=0) == abi.LA_OK
    assert _gqp(seq=0, q=None, o=None, ws=None) == abi.LA_OK


def test_the_header_is_c_and_matches_the_library(tmp_path):
    # a plain C program against include/lightning.h, linked with the library
    import os
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    libdir = os.path.dirname(abi.LIBRARY)
    exe = str(tmp_path / "abi_from_c")
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                    os.path.join(here, "c", "abi_from_c.c"), "-o", exe, "-L", libdir, "-llightning",
                    "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_the_binding_has_no_cpu_path():
    # every entry point refuses host tensors instead of computing on the CPU
    import torch
    import linear_attention_lightning_b200 as la
    x = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    sl = torch.ones(2)
    calls = [
        lambda: la.prefill(x, x, x, sl, 256),
        lambda: la.prefill_snapshots(x, x, x, sl, 256, 256),
        lambda: la.prefill_backward(x, x, x, x, sl, 256),
        lambda: la.prefill_norm_gate(x, x, x, sl, 256, torch.zeros((1, 8, 256), dtype=torch.bfloat16),
                                     torch.ones(256)),
        lambda: la.norm_gate(x, torch.zeros((1, 8, 256), dtype=torch.bfloat16), torch.ones(256)),
        lambda: la.decode(x[:, :, 0], x[:, :, 0], x[:, :, 0], sl, torch.zeros((1, 2, 128, 128))),
        lambda: la.gqa_decode(x[:, :, 0], x[:, :1, 0], x[:, :1, 0], x[:, :1], x[:, :1],
                              torch.zeros(1, dtype=torch.int32)),
        lambda: la.gqa_prefill(x, x[:, :1], x[:, :1], x[:, :1], x[:, :1]),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_a_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(abi, "LIBRARY", str(tmp_path / "absent.so"))
    monkeypatch.setattr(abi, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        abi.load()


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU: the binding's checks
    read only shape, dtype, device and contiguity, and must reject a bad argument
    before anything is allocated or called."""

    def __init__(self, shape, dtype, index=0):
        import torch
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def data_ptr(self):  # pragma: no cover - never reached: the checks raise first
        raise AssertionError("a pointer was taken before the arguments were checked")


def _fake_args():
    import torch
    b, h, L, d = 1, 2, 8, 128
    bf = torch.bfloat16
    return {
        "q": _FakeCuda((b, h, L, d), bf), "k": _FakeCuda((b, h, L, d), bf), "v": _FakeCuda((b, h, L, d), bf),
        "slopes": _FakeCuda((h,), torch.float32), "state": _FakeCuda((b, h, d, d), torch.float32),
        "o": _FakeCuda((b, h, L, d), bf), "gate": _FakeCuda((b, L, h * d), bf),
        "gamma": _FakeCuda((h * d,), torch.float32), "y": _FakeCuda((b, L, h * d), bf),
    }


@pytest.mark.parametrize("case", [
    "short_slopes", "long_slopes", "o_shape", "o_dtype", "state_out_shape", "state_in_other_gpu",
    "q_other_gpu", "o_other_gpu", "snapshots_shape", "y_shape", "decode_o_shape", "decode_state_shape",
    "decode_slopes",
])
def test_the_binding_checks_every_tensor_before_calling(monkeypatch, case):
    # a short slopes vector, an undersized output, or a tensor on another GPU would let
    # the kernel read or write out of bounds or touch a peer's memory: the binding
    # must refuse them, since the C layer sees raw pointers only
    import torch
    import linear_attention_lightning_b200.api as api
    monkeypatch.setattr(api, "_current_device", lambda: 0)
    a = _fake_args()
    q, k, v, sl, st, o = a["q"], a["k"], a["v"], a["slopes"], a["state"], a["o"]
    bad_st = _FakeCuda((1, 2, 128, 64), torch.float32)
    calls = {
        "short_slopes": lambda: api.prefill(q, k, v, _FakeCuda((1,), torch.float32), 256, o=o, state_out=st),
        "long_slopes": lambda: api.prefill(q, k, v, _FakeCuda((3,), torch.float32), 256, o=o, state_out=st),
        "o_shape": lambda: api.prefill(q, k, v, sl, 256, o=_FakeCuda((1, 2, 4, 128), torch.bfloat16)),
        "o_dtype": lambda: api.prefill(q, k, v, sl, 256, o=_FakeCuda((1, 2, 8, 128), torch.float32)),
        "state_out_shape": lambda: api.prefill(q, k, v, sl, 256, o=o, state_out=bad_st),
        "state_in_other_gpu": lambda: api.prefill(q, k, v, sl, 256, state_in=_FakeCuda(st.shape, torch.float32, 1)),
        "q_other_gpu": lambda: api.prefill(_FakeCuda(q.shape, torch.bfloat16, 1), k, v, sl, 256),
        "o_other_gpu": lambda: api.prefill(q, k, v, sl, 256, o=_FakeCuda(o.shape, torch.bfloat16, 1)),
        "snapshots_shape": lambda: api.prefill_snapshots(q, k, v, sl, 256, 4, o=o, state_out=st,
                                                         snapshots=_FakeCuda((1, 2, 1, 128, 128), torch.float32)),
        "y_shape": lambda: api.prefill_norm_gate(q, k, v, sl, 256, a["gate"], a["gamma"],
                                                 y=_FakeCuda((1, 8, 128), torch.bfloat16)),
        "decode_o_shape": lambda: api.decode(_FakeCuda((1, 2, 128), torch.bfloat16),
                                             _FakeCuda((1, 2, 128), torch.bfloat16),
                                             _FakeCuda((1, 2, 128), torch.bfloat16), sl, st,
                                             o=_FakeCuda((1, 1, 128), torch.bfloat16)),
        "decode_state_shape": lambda: api.decode(_FakeCuda((1, 2, 128), torch.bfloat16),
                                                 _FakeCuda((1, 2, 128), torch.bfloat16),
                                                 _FakeCuda((1, 2, 128), torch.bfloat16), sl, bad_st),
        "decode_slopes": lambda: api.decode(_FakeCuda((1, 2, 128), torch.bfloat16),
                                            _FakeCuda((1, 2, 128), torch.bfloat16),
                                            _FakeCuda((1, 2, 128), torch.bfloat16),
                                            _FakeCuda((1,), torch.float32), st),
    }
    with pytest.raises(ValueError):
        calls[case]()
