"""Seeded synthetic inputs for Lightning Attention workloads.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and distributions of the workloads, and the per-head slope
schedule s_h = 2^(-8(h+1)/H) (h 0-based) that the workloads fix as an input.
Both the CUDA path and the oracle are fed from here; neither imports the other.

Shapes follow MiniMax-M1's Lightning layers: 64 heads of 128 dims ("MINIMAX
SIGNAL LAB · M1", §02 architecture, attention projection 64 heads × 128) and a
float32 128×128 state per head (same page, §04 context cache).

Recipe, per workload: a torch.Generator on the target device seeded with the
workload's seed; draw order q, k, v (float32 N(0,1) scaled by 1/sqrt(dim),
then rounded to the workload dtype), then the initial state (float32
N(0,1) × 0.1, i.e. variance 0.01) when the workload carries one in. Decode
workloads draw the state first, then q, k, v for all steps at once.
"""
import math
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    batch: int
    heads: int
    seq: int             # tokens per sequence (1 for decode)
    dim: int
    block: int           # prefill block size B (unused for decode)
    dtype: torch.dtype   # q, k, v, o element type
    state_in: bool       # carried-in state drawn (True) or zeros (False)
    seed: int
    steps: int = 1       # decode steps


WORKLOADS = {
    w.name: w for w in (
        Workload("tiny_prefill_f32", "prefill", 1, 2, 256, 64, 64, torch.float32, False, 0),
        Workload("m1_prefill_8k", "prefill", 1, 64, 8192, 128, 256, torch.bfloat16, False, 1),
        Workload("m1_prefill_128k", "prefill", 1, 64, 131072, 128, 256, torch.bfloat16, False, 2),
        Workload("batched_prefill_state", "prefill", 16, 64, 4096, 128, 256, torch.bfloat16, True, 3),
        Workload("batched_decode", "decode", 64, 64, 1, 128, 0, torch.bfloat16, True, 4, 1000),
    )
}


def slopes(heads: int, device="cpu") -> torch.Tensor:
    """Per-head decay slopes s_h = 2^(-8(h+1)/heads), rounded once to float32."""
    vals = [2.0 ** (-8.0 * (h + 1) / heads) for h in range(heads)]
    return torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(device)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, scale: float, dtype, g, device) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype) if dtype != torch.float32 else x


def prefill_inputs(batch, heads, seq, dim, dtype=torch.bfloat16, state_in=False,
                   seed=0, device="cpu"):
    """Return dict(q, k, v [b,H,L,d] dtype; slopes [H] f32; state_in [b,H,d,d] f32 or None)."""
    g = _gen(device, seed)
    shape = (batch, heads, seq, dim)
    scale = 1.0 / math.sqrt(dim)
    q = _normal(shape, scale, dtype, g, device)
    k = _normal(shape, scale, dtype, g, device)
    v = _normal(shape, scale, dtype, g, device)
    s0: Optional[torch.Tensor] = None
    if state_in:
        s0 = _normal((batch, heads, dim, dim), 0.1, torch.float32, g, device)
    return {"q": q, "k": k, "v": v, "slopes": slopes(heads, device), "state_in": s0}


def decode_inputs(batch, heads, dim, steps, dtype=torch.bfloat16, seed=0, device="cpu"):
    """Return dict(state [b,H,d,d] f32; q, k, v [steps,b,H,d] dtype; slopes [H] f32)."""
    g = _gen(device, seed)
    state = _normal((batch, heads, dim, dim), 0.1, torch.float32, g, device)
    shape = (steps, batch, heads, dim)
    scale = 1.0 / math.sqrt(dim)
    q = _normal(shape, scale, dtype, g, device)
    k = _normal(shape, scale, dtype, g, device)
    v = _normal(shape, scale, dtype, g, device)
    return {"state": state, "q": q, "k": k, "v": v, "slopes": slopes(heads, device)}


def workload_inputs(w: Workload, device="cpu", seq: Optional[int] = None,
                    batch: Optional[int] = None, steps: Optional[int] = None):
    """Inputs of a named workload, optionally cut to a smaller seq/batch/steps."""
    b = w.batch if batch is None else batch
    if w.kind == "decode":
        return decode_inputs(b, w.heads, w.dim, w.steps if steps is None else steps,
                             w.dtype, w.seed, device)
    return prefill_inputs(b, w.heads, w.seq if seq is None else seq, w.dim, w.dtype,
                          w.state_in, w.seed, device)


def to_oracle(t: torch.Tensor):
    """Host numpy view the oracle reads: float32 as is, bfloat16 as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError("unsupported dtype %s" % t.dtype)
