"""GPU parity of one decode step of the softmax GQA layer (lightning_gqa_decode)
against the oracle's gqa_decode, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

from parity import TOL, rel_err, to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(b, h, hk, cap, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    d = 128
    mk = lambda *shape: (torch.randn(shape, generator=g, device=DEV)).to(dtype)
    return mk(b, h, d), mk(b, hk, d), mk(b, hk, d), mk(b, hk, cap, d), mk(b, hk, cap, d)


def _run_and_check(b, h, hk, cap, positions, rot, dtype, seed=80, base=10000.0):
    q, kn, vn, kc, vc = _inputs(b, h, hk, cap, dtype, seed)
    pos = torch.tensor(positions, dtype=torch.int32, device=DEV)
    kc0, vc0 = kc.clone(), vc.clone()
    conv = inputs.to_oracle
    ref = oracle.gqa_decode(conv(q), conv(kn), conv(vn), conv(kc0), conv(vc0), np.array(positions, np.int32), rot,
                            base, 1.0 / np.sqrt(128.0))
    o = la.gqa_decode(q, kn, vn, kc, vc, pos, rot=rot, rope_base=base)
    torch.cuda.synchronize()
    e = rel_err(to_f64(o), ref, bf16_out=int(dtype == torch.bfloat16))
    assert e <= TOL[dtype], "o error %.3g rms > %.3g" % (e, TOL[dtype])
    # the new rotated key and value sit at pos[b]; every other slot is untouched
    for bb, p in enumerate(positions):
        want_k = oracle.rope(to_f64(kn[bb]), p, rot, base)
        ek = np.max(np.abs(to_f64(kc[bb, :, p]) - want_k)) / max(np.sqrt(np.mean(want_k ** 2)), 1e-30)
        assert ek <= (1e-5 if dtype == torch.float32 else 1e-2), ek
        assert torch.equal(vc[bb, :, p], vn[bb])
        keep = torch.ones(cap, dtype=torch.bool, device=DEV)
        keep[p] = False
        assert torch.equal(kc[bb][:, keep], kc0[bb][:, keep]) and torch.equal(vc[bb][:, keep], vc0[bb][:, keep])


CASES = [
    # (batch, heads, kv_heads, cap, positions, rot)
    (2, 8, 2, 100, [0, 57], 64),
    (3, 64, 8, 1500, [1499, 513, 511], 64),
    (1, 16, 8, 40, [39], 128),
    (2, 8, 8, 700, [600, 3], 0),
    (1, 64, 8, 2048, [1024], 64),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_kv%d_cap%d_rot%d" % (c[0], c[1], c[2], c[3], c[5]))
def test_gqa_decode_matches_the_oracle(case, dtype):
    b, h, hk, cap, positions, rot = case
    _run_and_check(b, h, hk, cap, positions, rot, dtype)


def test_gqa_decode_long_context():
    # the serving shape: 64 query heads over 8 KV heads, a context of 131071 tokens
    _run_and_check(2, 64, 8, 131072, [131071, 70000], 64, torch.bfloat16, seed=81)


def test_gqa_decode_rejects_an_out_of_range_position_on_the_device():
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_device_status(stream) == abi.LA_OK
    q, kn, vn, kc, vc = _inputs(2, 8, 2, 64, torch.bfloat16, 82)
    kc0, vc0 = kc.clone(), vc.clone()
    pos = torch.tensor([64, 5], dtype=torch.int32, device=DEV)  # 64 == cap: outside the cache
    o = la.gqa_decode(q, kn, vn, kc, vc, pos)
    assert abi.lightning_device_status(stream) == abi.LA_ERR_INVALID_ARG
    assert torch.equal(kc[0], kc0[0]) and torch.equal(vc[0], vc0[0])  # nothing written for it
    assert torch.count_nonzero(o[0]) == 0
    assert abi.lightning_device_status(stream) == abi.LA_OK          # the word was cleared


def test_gqa_decode_never_lets_cache_rows_past_pos_into_the_result():
    # rows past pos[b] hold NaN: masked weights are 0, and 0 x NaN would still be NaN, so the
    # kernel must keep those rows out of every sum (the tensor-core path zeroes them in shared
    # memory before P V)
    b, h, hk, cap = 3, 16, 2, 2500
    positions = [300, 2047, 2100]          # inside the first chunk, its last slot, the second chunk
    q, kn, vn, kc, vc = _inputs(b, h, hk, cap, torch.bfloat16, 83)
    for bb, p in enumerate(positions):
        kc[bb, :, p + 1:] = float("nan")
        vc[bb, :, p + 1:] = float("nan")
    kc0, vc0 = kc.clone(), vc.clone()
    conv = inputs.to_oracle
    ref = oracle.gqa_decode(conv(q), conv(kn), conv(vn), conv(kc0), conv(vc0), np.array(positions, np.int32), 64,
                            10000.0, 1.0 / np.sqrt(128.0))
    o = la.gqa_decode(q, kn, vn, kc, vc, torch.tensor(positions, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    got = to_f64(o)
    assert np.all(np.isfinite(got))
    e = rel_err(got, ref, bf16_out=1)
    assert e <= TOL[torch.bfloat16], e


@pytest.mark.parametrize("case", [(1, 32, 2, 1500, [1499]), (2, 64, 2, 2100, [2099, 700])],
                         ids=["group16", "group32"])
def test_gqa_decode_bf16_groups_up_to_32(case):
    # the tensor-core path takes a KV head's query group as the rows of its tile, one softmax
    # lane per head: groups up to 32
    b, h, hk, cap, positions = case
    _run_and_check(b, h, hk, cap, positions, 64, torch.bfloat16, seed=84)
