"""CPU checks of the error measures the GPU parity tests state their bounds in,
on oracle outputs with errors planted in them: a measure must see a planted
error at its size and must read zero for what it is meant to exclude."""
import numpy as np
import torch

from parity import half_ulp_bf16, norm_gate_y_err_in_o_units, oracle_norm_gate_of, rel_err


def _case(seed=0, b=1, h=2, L=40, d=128):
    rng = np.random.default_rng(seed)
    # rows of very different size, as the prefill's output has (small rows are where the
    # per-row normalisation magnifies o's error)
    o64 = rng.standard_normal((b, h, L, d)) * np.exp(rng.standard_normal((1, 1, L, 1)))
    g = torch.Generator().manual_seed(seed)
    gate = (3.0 * torch.randn((b, L, h * d), generator=g)).to(torch.bfloat16)
    gamma = 1.0 + 0.1 * torch.randn((h * d,), generator=g)
    return o64, gate, gamma


def test_half_ulp_of_bf16():
    # 8 significant bits: half an ulp at 1 is 2^-8, at 3 is 2^-7, at 0 nothing
    assert np.allclose(half_ulp_bf16(np.array([1.0, 3.0, -0.5, 0.0])), [2.0 ** -8, 2.0 ** -7, 2.0 ** -9, 0.0])


def test_planted_o_error_is_seen_at_its_size_through_the_normalisation():
    o64, gate, gamma = _case()
    y_ref = oracle_norm_gate_of(o64, gate, gamma)
    rms = float(np.sqrt(np.mean(o64 ** 2)))
    # on the smallest row of head 1, an element of ordinary size within that row
    row = int(np.argmin(np.sqrt(np.mean(o64[0, 1] ** 2, axis=-1))))
    c = int(np.argmin(np.abs(np.abs(o64[0, 1, row]) - np.sqrt(np.mean(o64[0, 1, row] ** 2)))))
    for size in (0.05, 0.2):
        o_bad = o64.copy()
        o_bad[0, 1, row, c] += size * rms
        e = norm_gate_y_err_in_o_units(oracle_norm_gate_of(o_bad, gate, gamma), y_ref, o64, gate, gamma)
        assert 0.8 * size <= e <= 1.05 * size, (size, e)
        # the same error read against y as is: magnified on this small row
        assert rel_err(oracle_norm_gate_of(o_bad, gate, gamma), y_ref) > 2 * size


def test_format_rounding_and_the_sigmoid_allowance_read_zero():
    o64, gate, gamma = _case(1)
    y_ref = oracle_norm_gate_of(o64, gate, gamma)
    # o rounded to bf16 before the normalisation, y rounded to bf16 after it
    ob = torch.tensor(o64).to(torch.bfloat16).double().numpy()
    yb = torch.tensor(oracle_norm_gate_of(ob, gate, gamma)).to(torch.bfloat16).double().numpy()
    assert norm_gate_y_err_in_o_units(yb, y_ref, o64, gate, gamma) == 0.0
    # a sigmoid off by the documented bound of the SFU approximation everywhere is allowed
    # (2^-12 + 2^-24: tanh.approx.f32's relative error of at most 2^-11, halved, plus the
    # fma's rounding); off by 5e-3, not
    b, h, L, d = o64.shape
    gf = gate.float().numpy().reshape(b, L, h, d)
    o = np.transpose(o64, (0, 2, 1, 3))
    rstd = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + 1e-6)
    gm = gamma.numpy().reshape(h, d)[None, None]
    for off, ok in ((2.0 ** -12, True), (5e-3, False)):
        y_off = (gm * o * rstd * (1.0 / (1.0 + np.exp(-gf)) + off)).reshape(b, L, h * d)
        e = norm_gate_y_err_in_o_units(y_off, y_ref, o64, gate, gamma)
        assert (e == 0.0) == ok, (off, e)


def test_the_per_head_reading_sees_an_error_in_one_head_against_that_head():
    from parity import y_err_per_head
    o64, gate, gamma = _case(2)
    y_ref = oracle_norm_gate_of(o64, gate, gamma)
    b, L, hd = y_ref.shape
    y_bad = y_ref.copy().reshape(b, L, 2, hd // 2)
    rms1 = float(np.sqrt(np.mean(y_bad[:, :, 1] ** 2)))
    y_bad[0, 3, 1, 5] += 0.1 * rms1
    e = y_err_per_head(y_bad.reshape(b, L, hd), y_ref, 2)
    assert 0.09 <= e <= 0.101, e
    assert y_err_per_head(y_ref, y_ref, 2) == 0.0
