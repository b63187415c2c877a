"""GPU parity of the softmax GQA layer's prefill (lightning_gqa_prefill) against
the oracle's gqa_prefill, through the C ABI: outputs, the cache writes, the
rows of the cache that must stay untouched, and guard bands around o."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_lightning_b200 as la
from linear_attention_lightning_b200 import abi, inputs

from parity import half_ulp_bf16, rel_err, to_f64

pytestmark = pytest.mark.gpu

# o_i is a weighted mean of value rows, so its error is stated against the values' rms:
# with bf16 q, keys and weights P, each weight carries a relative error of about 2^-8,
# moving o_i by at most ~2^-8 max_j |v_j - o_i|. Bound: max |err| <= 2e-2 rms(v) (after
# the output's own bf16 rounding), and rms(err) <= 1e-2 rms(o) for systematic drift.
TOL_V = 2e-2
TOL_RMS = 1e-2


# float32 inputs: fp32 throughout (rotation, scores, exact softmax, accumulation)
TOL_V_F32 = 1e-4
TOL_RMS_F32 = 1e-4


def check(got, ref, v_rms, dtype=torch.bfloat16):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    if dtype == torch.bfloat16:
        diff = np.maximum(diff - half_ulp_bf16(np.maximum(np.abs(got), np.abs(ref))), 0.0)
    tv, tr = (TOL_V, TOL_RMS) if dtype == torch.bfloat16 else (TOL_V_F32, TOL_RMS_F32)
    e = float(diff.max()) / v_rms
    assert e <= tv, "max error %.3g rms(v) > %.3g" % (e, tv)
    er = float(np.sqrt(np.mean((got - ref) ** 2)) / np.sqrt(np.mean(ref ** 2)))
    assert er <= tr, "rms error %.3g rms(o) > %.3g" % (er, tr)
    return e


DEV = "cuda"
GUARD = 1024          # bf16 elements of guard band on each side of o (16-byte multiple)
SENTINEL = -77.0


def _inputs(b, h, hk, L, cap, seed, q_scale=1.0, dtype=torch.bfloat16):
    g = torch.Generator(device=DEV).manual_seed(seed)
    d = 128
    mk = lambda *shape: torch.randn(shape, generator=g, device=DEV).to(dtype)
    q = (torch.randn((b, h, L, d), generator=g, device=DEV) * q_scale).to(dtype)
    return q, mk(b, hk, L, d), mk(b, hk, L, d), mk(b, hk, cap, d), mk(b, hk, cap, d)


def _guarded_o(shape, dtype=torch.bfloat16):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), SENTINEL, dtype=dtype, device=DEV)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _run(b, h, hk, L, start, cap, rot, seed, scale=None, q_scale=1.0, poison_tail=False, base=10000.0,
         rows=None, dtype=torch.bfloat16):
    q, kn, vn, kc, vc = _inputs(b, h, hk, L, cap, seed, q_scale, dtype)
    if poison_tail and start + L < cap:
        # rows past the sequence hold NaN: the kernel must never read them
        kc[:, :, start + L:] = float("nan")
        vc[:, :, start + L:] = float("nan")
    kc0, vc0 = kc.clone(), vc.clone()
    conv = inputs.to_oracle
    sc = 1.0 / np.sqrt(128.0) if scale is None else scale
    ref = oracle.gqa_prefill(conv(q), conv(kn), conv(vn), conv(kc0), conv(vc0), start, rot, base, sc, rows=rows)
    buf, o = _guarded_o(q.shape, dtype)
    la.gqa_prefill(q, kn, vn, kc, vc, start=start, rot=rot, rope_base=base, scale=sc, o=o)
    torch.cuda.synchronize()
    assert torch.all(buf[:GUARD] == SENTINEL) and torch.all(buf[-GUARD:] == SENTINEL), "o guard band written"
    got = to_f64(o).reshape(-1, 128)
    if rows is not None:
        got = got[np.asarray(rows)]
    else:
        ref = ref.reshape(-1, 128)
    assert np.all(np.isfinite(got))
    v_rms = float(torch.sqrt(torch.mean(torch.cat([vn.float().flatten(), vc0[:, :, :start].float().flatten()]) ** 2)))
    e = check(got, ref, v_rms, dtype)
    print("gqa_prefill %s b%d h%d kv%d L%d start%d rot%d: max error %.3g rms(v)" % (str(dtype)[6:], b, h, hk, L, start, rot, e))
    # cache rows start .. start+L-1 hold the rotated keys and the values; the rest is untouched
    span = slice(start, start + L)
    for bb in range(b):
        for g in range(hk):
            pos = np.arange(start, start + L)
            want = np.stack([oracle.rope(x, p, rot, base) for x, p in zip(to_f64(kn[bb, g]), pos)]) if L <= 2048 \
                else None
            if want is not None:
                # the rotated key within the bf16 rounding of the cache (plus fp32 rotation noise)
                got_k = to_f64(kc[bb, g, span])
                slack = np.abs(got_k - want)
                if dtype == torch.bfloat16:
                    slack = slack - half_ulp_bf16(np.maximum(np.abs(got_k), np.abs(want)))
                assert slack.max() <= 1e-5 * np.sqrt(np.mean(want ** 2)), slack.max()
    assert torch.equal(vc[:, :, span], vn)
    keep = torch.ones(cap, dtype=torch.bool, device=DEV)
    keep[span] = False
    iv = torch.int16 if dtype == torch.bfloat16 else torch.int32
    assert torch.equal(kc[:, :, keep].view(iv), kc0[:, :, keep].view(iv))
    assert torch.equal(vc[:, :, keep].view(iv), vc0[:, :, keep].view(iv))
    return e


CASES = [
    # (batch, heads, kv_heads, seq, start, cap, rot)
    (1, 8, 2, 1, 0, 1, 64),            # one token, empty prefix
    (1, 8, 1, 100, 0, 128, 64),        # one ragged tile
    (2, 8, 8, 256, 0, 300, 64),        # exactly one CTA's rows
    (1, 16, 2, 257, 0, 257, 128),      # one row into the second CTA
    (2, 8, 4, 700, 37, 1000, 64),      # an unaligned prefix
    (1, 8, 8, 129, 300, 429, 0),       # no rotation, prefix of 300
    (1, 64, 8, 1000, 0, 1024, 64),     # the model's 64 over 8 heads
    (3, 16, 2, 511, 1, 600, 64),       # prefix of one token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_h%d_kv%d_L%d_s%d_rot%d" % (c[0], c[1], c[2], c[3], c[4],
                                                                                         c[6]))
def test_gqa_prefill_matches_the_oracle(case):
    b, h, hk, L, start, cap, rot = case
    _run(b, h, hk, L, start, cap, rot, seed=90 + L)


def test_gqa_prefill_never_reads_cache_rows_past_the_sequence():
    _run(1, 8, 2, 300, 50, 1000, 64, seed=91, poison_tail=True)
    _run(2, 8, 8, 128, 0, 512, 64, seed=92, poison_tail=True)


def test_gqa_prefill_peaked_softmax_raises_the_running_max():
    # scale 1 instead of 1/sqrt(128): scores spread over tens of units, so the running max
    # is raised (and O rescaled) many times along the keys. No rotation, so that q and the
    # keys reach the tensor cores exactly and only the rounding of P is left: the same bound
    # holds however peaked the softmax is.
    _run(1, 8, 2, 600, 0, 600, 0, seed=93, scale=1.0)
    _run(1, 8, 2, 600, 200, 800, 0, seed=94, scale=0.5, q_scale=3.0)


def test_gqa_prefill_long_context_sampled_rows():
    # 16384 new tokens after a 16384-token prefix, 64 query heads over 8 KV heads; rows sampled
    # across heads and positions (the first and last of each tile edge among them)
    b, h, hk, L, start = 1, 64, 8, 16384, 16384
    rng = np.random.default_rng(95)
    heads = rng.choice(h, 6, replace=False)
    pos = np.concatenate([[0, 127, 128, 255, 256, L - 1], rng.integers(0, L, 10)])
    rows = np.array([hh * L + p for hh in heads for p in pos])
    _run(b, h, hk, L, start, start + L, 64, seed=96, rows=rows)


def test_gqa_prefill_chunked_equals_one_call():
    # two calls (the second continuing from the cache the first wrote) give the one-call result
    b, h, hk, L, cap = 1, 8, 2, 640, 700
    q, kn, vn, kc, vc = _inputs(b, h, hk, L, cap, 97)
    kc2, vc2 = kc.clone(), vc.clone()
    o = la.gqa_prefill(q, kn, vn, kc, vc, start=0)
    cut = 300
    o1 = la.gqa_prefill(q[:, :, :cut].contiguous(), kn[:, :, :cut].contiguous(), vn[:, :, :cut].contiguous(), kc2,
                        vc2, start=0)
    o2 = la.gqa_prefill(q[:, :, cut:].contiguous(), kn[:, :, cut:].contiguous(), vn[:, :, cut:].contiguous(), kc2,
                        vc2, start=cut)
    torch.cuda.synchronize()
    assert torch.equal(kc2.view(torch.int16), kc.view(torch.int16)) and torch.equal(vc2, vc)
    both = torch.cat([o1, o2], 2)
    e = rel_err(to_f64(both), to_f64(o), bf16_out=2)
    assert e <= 2 * TOL_V * float(torch.sqrt(torch.mean(vn.float() ** 2))) / float(torch.sqrt(torch.mean(o.float() ** 2)))


def test_gqa_prefill_then_decode_continues_the_cache():
    # the decode step after a prefill of L tokens sees what the prefill wrote
    b, h, hk, L, cap = 2, 8, 2, 300, 400
    q, kn, vn, kc, vc = _inputs(b, h, hk, L + 1, cap, 98)
    la.gqa_prefill(q[:, :, :L].contiguous(), kn[:, :, :L].contiguous(), vn[:, :, :L].contiguous(), kc, vc, start=0)
    pos = torch.full((b,), L, dtype=torch.int32, device=DEV)
    od = la.gqa_decode(q[:, :, L].contiguous(), kn[:, :, L].contiguous(), vn[:, :, L].contiguous(), kc, vc, pos)
    torch.cuda.synchronize()
    conv = inputs.to_oracle
    ref = oracle.gqa_prefill(conv(q), conv(kn), conv(vn), conv(kc), conv(vc), 0, 64, 10000.0, 1.0 / np.sqrt(128.0),
                             rows=[(bb * h + hh) * (L + 1) + L for bb in range(b) for hh in range(h)])
    check(to_f64(od).reshape(-1, 128), ref, float(torch.sqrt(torch.mean(vn.float() ** 2))))


def test_gqa_prefill_leaves_the_device_status_clean():
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_device_status(stream) == abi.LA_OK
    _run(1, 8, 2, 64, 10, 80, 64, seed=99)
    assert abi.lightning_device_status(stream) == abi.LA_OK


F32_CASES = [
    # (batch, heads, kv_heads, seq, start, cap, rot)
    (1, 8, 2, 1, 0, 1, 64),
    (2, 8, 4, 300, 37, 400, 64),
    (1, 16, 2, 257, 0, 257, 128),
    (1, 8, 8, 129, 200, 400, 0),
]


@pytest.mark.parametrize("case", F32_CASES, ids=lambda c: "b%d_h%d_kv%d_L%d_s%d_rot%d" % (c[0], c[1], c[2], c[3], c[4],
                                                                                             c[6]))
def test_gqa_prefill_float32_matches_the_oracle(case):
    b, h, hk, L, start, cap, rot = case
    _run(b, h, hk, L, start, cap, rot, seed=190 + L, dtype=torch.float32)


def test_gqa_prefill_float32_never_reads_cache_rows_past_the_sequence():
    _run(1, 8, 2, 100, 20, 400, 64, seed=191, poison_tail=True, dtype=torch.float32)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gqa_prefill_sequences_with_unequal_prefixes(dtype):
    # each sequence continues its own cached prefix (start[b] on the device): the pages'
    # KV cache grows per sequence ("MINIMAX SIGNAL LAB · M1", §04). Cache rows past each
    # sequence's end hold NaN: the last key tile a query reads may reach them, and they
    # must enter no result.
    b, h, hk, L, cap, rot, base = 4, 16, 4, 300, 1500, 64, 10000.0
    starts = [0, 37, 1000, 1200]
    q, kn, vn, kc, vc = _inputs(b, h, hk, L, cap, 301, dtype=dtype)
    for bb, st in enumerate(starts):
        kc[bb, :, st + L:] = float("nan")
        vc[bb, :, st + L:] = float("nan")
    kc0, vc0 = kc.clone(), vc.clone()
    sc = 1.0 / np.sqrt(128.0)
    buf, o = _guarded_o(q.shape, dtype)
    la.gqa_prefill(q, kn, vn, kc, vc, start=torch.tensor(starts, dtype=torch.int32, device=DEV), rot=rot,
                   rope_base=base, scale=sc, o=o)
    torch.cuda.synchronize()
    assert torch.all(buf[:GUARD] == SENTINEL) and torch.all(buf[-GUARD:] == SENTINEL), "o guard band written"
    conv = inputs.to_oracle
    iv = torch.int16 if dtype == torch.bfloat16 else torch.int32
    for bb, st in enumerate(starts):
        sl = slice(bb, bb + 1)
        ref = oracle.gqa_prefill(conv(q[sl]), conv(kn[sl]), conv(vn[sl]), conv(kc0[sl]), conv(vc0[sl]), st, rot,
                                 base, sc)
        got = to_f64(o[sl])
        assert np.all(np.isfinite(got)), "sequence %d" % bb
        v_rms = float(torch.sqrt(torch.mean(torch.cat([vn[sl].float().flatten(),
                                                       vc0[sl, :, :st].float().flatten()]) ** 2)))
        e = check(got.reshape(-1, 128), ref.reshape(-1, 128), v_rms, dtype)
        print("gqa_prefill %s, sequence %d at start %d: max error %.3g rms(v)" % (str(dtype)[6:], bb, st, e))
        # this sequence's new rows are written; every other row keeps its contents (NaN included)
        assert torch.equal(vc[bb, :, st:st + L], vn[bb])
        keep = torch.ones(cap, dtype=torch.bool, device=DEV)
        keep[st:st + L] = False
        assert torch.equal(kc[bb][:, keep].view(iv), kc0[bb][:, keep].view(iv))
        assert torch.equal(vc[bb][:, keep].view(iv), vc0[bb][:, keep].view(iv))
    assert abi.lightning_last_device_status(torch.cuda.current_stream().cuda_stream) == abi.LA_OK


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gqa_prefill_skips_and_reports_a_start_outside_the_cache(dtype):
    b, h, hk, L, cap = 3, 8, 2, 200, 600
    starts = [5, 450, 100]            # 450 + 200 > 600: sequence 1 does not fit
    q, kn, vn, kc, vc = _inputs(b, h, hk, L, cap, 302, dtype=dtype)
    kc0, vc0 = kc.clone(), vc.clone()
    o = torch.full_like(q, SENTINEL)
    stream = torch.cuda.current_stream().cuda_stream
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
    la.gqa_prefill(q, kn, vn, kc, vc, start=torch.tensor(starts, dtype=torch.int32, device=DEV), rot=64, o=o)
    assert abi.lightning_last_device_status(stream) == abi.LA_ERR_INVALID_ARG
    iv = torch.int16 if dtype == torch.bfloat16 else torch.int32
    assert torch.equal(kc[1].view(iv), kc0[1].view(iv)) and torch.equal(vc[1].view(iv), vc0[1].view(iv))
    assert torch.all(o[1] == SENTINEL)       # nothing written for the sequence that does not fit
    conv = inputs.to_oracle
    for bb in (0, 2):
        sl = slice(bb, bb + 1)
        ref = oracle.gqa_prefill(conv(q[sl]), conv(kn[sl]), conv(vn[sl]), conv(kc0[sl]), conv(vc0[sl]), starts[bb],
                                 64, 10000.0, 1.0 / np.sqrt(128.0))
        v_rms = float(torch.sqrt(torch.mean(torch.cat([vn[sl].float().flatten(),
                                                       vc0[sl, :, :starts[bb]].float().flatten()]) ** 2)))
        check(to_f64(o[sl]).reshape(-1, 128), ref.reshape(-1, 128), v_rms, dtype)
    assert abi.lightning_last_device_status(stream) == abi.LA_OK
