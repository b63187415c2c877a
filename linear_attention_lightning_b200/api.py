"""torch-facing wrappers over the C ABI: argument marshalling only.

Tensors must be CUDA, contiguous, on the current device. Outputs are
allocated with torch when not supplied. Nothing here computes anything of
the method; a missing library raises instead of falling back.
"""
from typing import Optional, Tuple

import torch

from . import abi

_DTYPES = {torch.float32: abi.LA_DTYPE_F32, torch.bfloat16: abi.LA_DTYPE_BF16}
_VARIANTS = {"auto": abi.LA_VARIANT_AUTO, "simt": abi.LA_VARIANT_SIMT, "tcgen05": abi.LA_VARIANT_TCGEN05,
             "pair": abi.LA_VARIANT_TCGEN05_PAIR}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need_cuda(name, t, dtype=None):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
            state_in: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
            state_out: Optional[torch.Tensor] = None, want_state: bool = True,
            variant: str = "auto", stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill on [batch, heads, seq, dim] tensors; returns (o, state_out)."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [batch, heads, seq, dim] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    b, h, L, d = q.shape
    _need_cuda("slopes", slopes, torch.float32)
    if state_in is not None:
        _need_cuda("state_in", state_in, torch.float32)
        if tuple(state_in.shape) != (b, h, d, d):
            raise ValueError("state_in must be [batch, heads, dim, dim]")
    if o is None:
        o = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    abi.check(abi.lightning_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(o), _ptr(state_out), None, 0, _stream(stream), _VARIANTS[variant]))
    return o, state_out


def prefill_snapshots(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
                      interval: int, state_in: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
                      state_out: Optional[torch.Tensor] = None, snapshots: Optional[torch.Tensor] = None,
                      want_state: bool = True, variant: str = "auto",
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor], torch.Tensor]:
    """lightning_prefill_snapshots: returns (o, state_out, snapshots); snapshots is
    [batch, heads, seq // interval, dim, dim] float32, the state after each
    interval tokens."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [batch, heads, seq, dim] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    b, h, L, d = q.shape
    _need_cuda("slopes", slopes, torch.float32)
    if state_in is not None:
        _need_cuda("state_in", state_in, torch.float32)
        if tuple(state_in.shape) != (b, h, d, d):
            raise ValueError("state_in must be [batch, heads, dim, dim]")
    n = abi.lightning_prefill_snapshot_count(L, int(interval))
    if n < 0:
        raise ValueError("interval must be >= 1")
    if o is None:
        o = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    if snapshots is None:
        snapshots = torch.empty((b, h, n, d, d), dtype=torch.float32, device=q.device)
    else:
        _need_cuda("snapshots", snapshots, torch.float32)
        if tuple(snapshots.shape) != (b, h, n, d, d):
            raise ValueError("snapshots must be [batch, heads, seq // interval, dim, dim]")
    abi.check(abi.lightning_prefill_snapshots(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(o), _ptr(state_out), int(interval), _ptr(snapshots) if n > 0 else None,
        _stream(stream), _VARIANTS[variant]))
    return o, state_out, snapshots


def prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, d_o: torch.Tensor, slopes: torch.Tensor,
                     block: int, state_in: Optional[torch.Tensor] = None,
                     d_state_out: Optional[torch.Tensor] = None, want_state_grad: bool = True,
                     variant: str = "auto", workspace: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill_backward: returns (dq, dk, dv, d_state_in) for the loss
    sum(d_o * o) + sum(d_state_out * state_out). The workspace the tensor-core
    kernels need is allocated with torch unless a uint8 tensor is passed."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or any(t.shape != q.shape for t in (k, v, d_o)):
        raise ValueError("q, k, v, d_o must share one [batch, heads, seq, dim] shape")
    if variant not in ("auto", "simt", "pair"):
        raise ValueError("backward variant must be auto, simt or pair")
    for name, t in (("q", q), ("k", k), ("v", v), ("d_o", d_o)):
        _need_cuda(name, t, q.dtype)
    b, h, L, d = q.shape
    _need_cuda("slopes", slopes, torch.float32)
    for name, t in (("state_in", state_in), ("d_state_out", d_state_out)):
        if t is not None:
            _need_cuda(name, t, torch.float32)
            if tuple(t.shape) != (b, h, d, d):
                raise ValueError("%s must be [batch, heads, dim, dim]" % name)
    need = abi.lightning_prefill_backward_workspace_size(_DTYPES[q.dtype], b, h, L, d, int(block),
                                                          _VARIANTS[variant])
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ds_in = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device) if want_state_grad else None
    abi.check(abi.lightning_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(d_o), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(d_state_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds_in), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream),
        _VARIANTS[variant]))
    return dq, dk, dv, ds_in


def norm_gate(o: torch.Tensor, gate: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
              per_head: bool = False, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lightning_norm_gate: RMS-normalise the attention output o [batch, heads,
    seq, dim] per token (or per head) and gate it with sigmoid(gate); returns y
    [batch, seq, heads*dim]."""
    if o.dtype not in _DTYPES:
        raise ValueError("o must be float32 or bfloat16")
    if o.dim() != 4:
        raise ValueError("o must be [batch, heads, seq, dim]")
    b, h, L, d = o.shape
    _need_cuda("o", o, o.dtype)
    _need_cuda("gate", gate, o.dtype)
    if tuple(gate.shape) != (b, L, h * d):
        raise ValueError("gate must be [batch, seq, heads*dim]")
    _need_cuda("gamma", gamma, torch.float32)
    if tuple(gamma.shape) != (h * d,):
        raise ValueError("gamma must be [heads*dim]")
    if y is None:
        y = torch.empty((b, L, h * d), dtype=o.dtype, device=o.device)
    abi.check(abi.lightning_norm_gate(_ptr(o), _ptr(gate), _DTYPES[o.dtype], _ptr(gamma), float(eps), b, h, L, d,
                                      1 if per_head else 0, _ptr(y), _stream(stream)))
    return y


def prefill_norm_gate(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
                      gate: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                      state_in: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                      state_out: Optional[torch.Tensor] = None, want_state: bool = True,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill_norm_gate: the prefill with the per-head normalisation and
    gate fused into its epilogue; returns (y [batch, seq, heads*dim], state_out)."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [batch, heads, seq, dim] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    b, h, L, d = q.shape
    _need_cuda("slopes", slopes, torch.float32)
    _need_cuda("gate", gate, q.dtype)
    if tuple(gate.shape) != (b, L, h * d):
        raise ValueError("gate must be [batch, seq, heads*dim]")
    _need_cuda("gamma", gamma, torch.float32)
    if tuple(gamma.shape) != (h * d,):
        raise ValueError("gamma must be [heads*dim]")
    if state_in is not None:
        _need_cuda("state_in", state_in, torch.float32)
        if tuple(state_in.shape) != (b, h, d, d):
            raise ValueError("state_in must be [batch, heads, dim, dim]")
    if y is None:
        y = torch.empty((b, L, h * d), dtype=q.dtype, device=q.device)
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    abi.check(abi.lightning_prefill_norm_gate(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block), _ptr(state_in),
        _ptr(gate), _ptr(gamma), float(eps), _ptr(y), _ptr(state_out), _stream(stream)))
    return y, state_out


def gqa_decode(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
               v_cache: torch.Tensor, pos: torch.Tensor, rot: int = 64, rope_base: float = 10000.0,
               scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lightning_gqa_decode: one decode step of the softmax GQA layer. Writes the
    new rotated key and value into the caches at pos[b] and returns o
    [batch, heads, dim]. scale defaults to 1/sqrt(dim)."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    b, h, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or tuple(k_new.shape) != (b, hk, d) or tuple(v_new.shape) != (b, hk, d) \
            or v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent shapes: q [b, heads, dim], k/v_new [b, kv_heads, dim], caches [b, kv_heads, cap, dim]")
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda(name, t, q.dtype)
    _need_cuda("pos", pos, torch.int32)
    if tuple(pos.shape) != (b,):
        raise ValueError("pos must be [batch]")
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty_like(q)
    need = abi.lightning_gqa_decode_workspace_size(b, h, cap)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    abi.check(abi.lightning_gqa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                       _DTYPES[q.dtype], _ptr(pos), b, h, hk, d, cap, int(rot), float(rope_base),
                                       float(scale), _ptr(o), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def gqa_prefill(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, start: int = 0, rot: int = 64, rope_base: float = 10000.0,
                scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lightning_gqa_prefill: the softmax GQA layer over seq new tokens at
    positions start .. start+seq-1. Writes their rotated keys and values into
    the caches and returns o [batch, heads, seq, dim]. bf16 (tensor cores) or
    float32 (CUDA cores); scale defaults to 1/sqrt(dim)."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    b, h, L, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or tuple(k_new.shape) != (b, hk, L, d) or tuple(v_new.shape) != (b, hk, L, d) \
            or v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent shapes: q [b, heads, seq, dim], k/v_new [b, kv_heads, seq, dim], "
                         "caches [b, kv_heads, cap, dim]")
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda(name, t, q.dtype)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty_like(q)
    need = abi.lightning_gqa_prefill_workspace_size(_DTYPES[q.dtype], b, h, L, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    abi.check(abi.lightning_gqa_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                        _DTYPES[q.dtype], int(start), b, h, hk, L, d, cap, int(rot),
                                        float(rope_base), float(scale), _ptr(o), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def prefill_variant(dtype: torch.dtype, batch: int, heads: int, seq: int, dim: int, block: int,
                    variant: str = "auto") -> str:
    """Which kernel lightning_prefill would run: "simt", "tcgen05" or "pair"."""
    r = abi.lightning_prefill_selected_variant(_DTYPES[dtype], batch, heads, seq, dim, block,
                                               _VARIANTS[variant])
    if r < 0:
        raise ValueError(abi.last_error_message() or "unsupported request")
    return {abi.LA_VARIANT_SIMT: "simt", abi.LA_VARIANT_TCGEN05: "tcgen05",
            abi.LA_VARIANT_TCGEN05_PAIR: "pair"}[r]


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor,
           state: torch.Tensor, o: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lightning_decode on [batch, heads, dim] tensors; updates `state` in place, returns o."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [batch, heads, dim] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    b, h, d = q.shape
    _need_cuda("slopes", slopes, torch.float32)
    _need_cuda("state", state, torch.float32)
    if tuple(state.shape) != (b, h, d, d):
        raise ValueError("state must be [batch, heads, dim, dim]")
    if o is None:
        o = torch.empty_like(q)
    abi.check(abi.lightning_decode(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, d,
                                   _ptr(state), _ptr(o), _stream(stream)))
    return o
