"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and measure the error the
way the tolerances are stated (max |err| relative to the oracle's rms)."""
import numpy as np
import torch

import oracle
from linear_attention_lightning_b200 import inputs

# max |err| <= TOL * rms(reference)
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bfloat16 ulp at |x| (8 significant bits): the most that rounding a
    value of that size to bfloat16 can move it."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8.0), 0.0)


def rel_err(got, ref, bf16_out: int = 0) -> float:
    """max |got - ref| / rms(ref). For bfloat16 outputs the unavoidable final
    rounding of each element (half an ulp at max(|got|, |ref|)) is excluded,
    so that the bound measures the computation, not the output format;
    bf16_out counts how many bf16-rounded operands the comparison has (1 for
    GPU against oracle, 2 for two GPU results)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    diff = np.abs(got - ref)
    if bf16_out:
        allow = int(bf16_out) * half_ulp_bf16(np.maximum(np.abs(got), np.abs(ref)))
        diff = np.maximum(diff - allow, 0.0)
    err = float(np.max(diff))
    return err / rms if rms > 0 else err


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_prefill(inp, heads_idx=None, batch_idx=None, form="recurrence", block=None):
    """Oracle on (optionally) a subset of batches / heads of a prefill input dict."""
    q, k, v, s0 = inp["q"], inp["k"], inp["v"], inp["state_in"]
    sl = inp["slopes"]
    if batch_idx is not None:
        q, k, v = q[batch_idx], k[batch_idx], v[batch_idx]
        s0 = None if s0 is None else s0[batch_idx]
    if heads_idx is not None:
        q, k, v = q[:, heads_idx], k[:, heads_idx], v[:, heads_idx]
        s0 = None if s0 is None else s0[:, heads_idx]
        sl = sl[heads_idx]
    conv = inputs.to_oracle
    return oracle.prefill(conv(q), conv(k), conv(v), sl.cpu().numpy(),
                          None if s0 is None else s0.cpu().numpy(), form=form, block=block)


def guarded_empty(shape, dtype, device, guard=4096):
    """Tensor with sentinel-filled guard bands on both sides; returns (view, backing)."""
    n = int(np.prod(shape))
    back = torch.empty(n + 2 * guard, dtype=dtype, device=device)
    back.fill_(-1234.5)
    view = back[guard:guard + n].view(shape)
    return view, back


def guards_intact(back, n, guard=4096) -> bool:
    sentinel = torch.tensor(-1234.5, dtype=back.dtype)
    head = back[:guard].cpu()
    tail = back[guard + n:].cpu()
    return bool(torch.all(head == sentinel)) and bool(torch.all(tail == sentinel))


# The per-head normalisation and gate after a prefill (the fused call's reference).
NG_EPS = 1e-6


def oracle_norm_gate_of(o64, gate, gamma, heads_idx=None):
    """norm_gate of the oracle's float64 prefill output (per-head mean), on the
    heads heads_idx (all when None). The oracle's norm_gate reads float32: o is
    rounded once to float32 (relative 2^-24, far below the bound) and the bf16
    gate widens exactly."""
    b, h, L, d = o64.shape
    g = gate.float().cpu().numpy().reshape(b, L, -1, d)
    gm = gamma.cpu().numpy().reshape(-1, d)
    if heads_idx is not None:
        g, gm = g[:, :, heads_idx], gm[heads_idx]
    g = np.ascontiguousarray(g.reshape(b, L, h * d))
    return oracle.norm_gate(o64.astype(np.float32), g, np.ascontiguousarray(gm.reshape(-1)), NG_EPS, True)


# Absolute error allowed for sigmoid(g) = 1/2 + tanh(g/2)/2 as the fused kernel forms it:
# tanh.approx.f32, whose relative error the PTX ISA documents as at most 2^-11 over its
# whole range, so |error of tanh| <= 2^-11 |tanh| <= 2^-11; halved by the 1/2 factor, plus
# the fp32 rounding of the fma that adds 1/2 (half an ulp of a value below 1: 2^-24). g/2
# is exact (g is bf16). Bound: 2^-12 + 2^-24.
SIGMOID_ABS_ERR = 2.0 ** -12 + 2.0 ** -24


def norm_gate_y_err_in_o_units(y, y_ref, o64, gate, gamma, heads_idx=None):
    """The error of y carried back to o, over rms(o): (|y - y_ref| - allowance) / dy/do,
    dy/do = |gamma| sigmoid(g) / sqrt(mean o^2 + eps) at the reference.

    y normalises each head's row to unit rms, so an error of o that is small against
    rms(o) (the prefill's bound, 2e-2 rms(o) for bf16 inputs) becomes large against y
    on rows whose own rms is small; the fused kernel's y is held to the prefill's bound
    on o through the exact normalisation. The allowance excludes, as the bound on o
    does, the rounding of the formats (half a bf16 ulp of y, and half a bf16 ulp of o
    through dy/do: y is formed from o rounded to bf16, as in the two-call path), and
    the sigmoid's absolute error times |gamma o / rms(o_row)|, which dividing by
    sigmoid(g) would otherwise magnify where g is very negative."""
    b, h, L, d = o64.shape
    g = gate.float().cpu().numpy().reshape(b, L, -1, d)
    gm = gamma.cpu().numpy().reshape(-1, d)
    if heads_idx is not None:
        g, gm = g[:, :, heads_idx], gm[heads_idx]
    o = np.transpose(o64, (0, 2, 1, 3))                           # [b, L, h, d]
    rstd = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + NG_EPS)
    sig = 1.0 / (1.0 + np.exp(-g.astype(np.float64)))
    dydo = np.abs(gm)[None, None] * sig * rstd
    got = np.asarray(y, np.float64).reshape(b, L, h, d)
    ref = np.asarray(y_ref, np.float64).reshape(b, L, h, d)
    allow = (half_ulp_bf16(np.maximum(np.abs(got), np.abs(ref))) + dydo * half_ulp_bf16(o)
             + np.abs(gm)[None, None] * np.abs(o) * rstd * SIGMOID_ABS_ERR)
    diff = np.maximum(np.abs(got - ref) - allow, 0.0)
    return float(np.max(diff / dydo)) / float(np.sqrt(np.mean(o64 * o64)))


def y_err_per_head(y, y_ref, heads: int) -> float:
    """The plain reading of the fused call's error: per head (its 128 channels over
    every token), max |y - y_ref| / rms(y_ref of that head), with half a bf16 ulp of
    y excluded as rel_err does; the largest over the heads."""
    got = np.asarray(y, np.float64)
    ref = np.asarray(y_ref, np.float64)
    got = got.reshape(got.shape[0], got.shape[1], heads, -1)
    ref = ref.reshape(got.shape)
    worst = 0.0
    for h in range(heads):
        worst = max(worst, rel_err(got[:, :, h], ref[:, :, h], bf16_out=1))
    return worst
