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
