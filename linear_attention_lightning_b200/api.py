"""torch-facing wrappers over the C ABI: argument marshalling only.

Tensors must be CUDA, contiguous, on the current device. Outputs are
allocated with torch when not supplied; a supplied output, like every input,
is checked for its shape, dtype and device before the call, because the C
layer sees raw pointers only and could not tell a short buffer or another
GPU's memory from a good one. Nothing here computes anything of the method;
a missing library raises instead of falling back.
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


def _current_device() -> int:
    return torch.cuda.current_device()


def _need_cuda(name, t, dtype=None, shape=None):
    """A CUDA tensor, contiguous, of `dtype` and `shape` (when given), on the current device."""
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    cur = _current_device()
    if t.device.index != cur:
        raise ValueError("%s is on %s, not on the current device cuda:%d" % (name, t.device, cur))


def _qkv(q, k, v, extra=()):
    """q, k, v (and `extra`) share one [batch, heads, seq, dim] shape and a supported dtype."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or any(t.shape != q.shape for _, t in extra):
        raise ValueError("q, k, v%s must share one [batch, heads, seq, dim] shape"
                         % "".join(", " + n for n, _ in extra))
    for name, t in (("q", q), ("k", k), ("v", v)) + tuple(extra):
        _need_cuda(name, t, q.dtype)
    return q.shape


def _state(name, t, b, h, d):
    if t is not None:
        _need_cuda(name, t, torch.float32, (b, h, d, d))


def _workspace(need, workspace, device):
    """The caller's uint8 workspace (checked), or one allocated with torch when the call needs any."""
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=device) if need > 0 else None
    _need_cuda("workspace", workspace, torch.uint8)
    return workspace


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
            state_in: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
            state_out: Optional[torch.Tensor] = None, want_state: bool = True,
            variant: str = "auto", workspace: Optional[torch.Tensor] = None,
            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill on [batch, heads, seq, dim] tensors; returns (o, state_out).
    The workspace the kernel needs is allocated with torch unless a uint8
    tensor is passed."""
    b, h, L, d = _qkv(q, k, v)
    _need_cuda("slopes", slopes, torch.float32, (h,))
    _state("state_in", state_in, b, h, d)
    if o is None:
        o = torch.empty_like(q)
    else:
        _need_cuda("o", o, q.dtype, q.shape)
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    else:
        _state("state_out", state_out, b, h, d)
    workspace = _workspace(abi.lightning_prefill_workspace_size(b, h, L, d, int(block)), workspace, q.device)
    abi.check(abi.lightning_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(o), _ptr(state_out), _ptr(workspace), _nbytes(workspace), _stream(stream),
        _VARIANTS[variant]))
    return o, state_out


def prefill_snapshots(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
                      interval: int, state_in: Optional[torch.Tensor] = None, o: Optional[torch.Tensor] = None,
                      state_out: Optional[torch.Tensor] = None, snapshots: Optional[torch.Tensor] = None,
                      want_state: bool = True, variant: str = "auto", workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor], torch.Tensor]:
    """lightning_prefill_snapshots: returns (o, state_out, snapshots); snapshots is
    [batch, heads, seq // interval, dim, dim] float32, the state after each
    interval tokens. The workspace is allocated with torch unless given."""
    b, h, L, d = _qkv(q, k, v)
    _need_cuda("slopes", slopes, torch.float32, (h,))
    _state("state_in", state_in, b, h, d)
    n = abi.lightning_prefill_snapshot_count(L, int(interval))
    if n < 0:
        raise ValueError("interval must be >= 1")
    if o is None:
        o = torch.empty_like(q)
    else:
        _need_cuda("o", o, q.dtype, q.shape)
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    else:
        _state("state_out", state_out, b, h, d)
    if snapshots is None:
        snapshots = torch.empty((b, h, n, d, d), dtype=torch.float32, device=q.device)
    else:
        _need_cuda("snapshots", snapshots, torch.float32, (b, h, n, d, d))
    workspace = _workspace(abi.lightning_prefill_workspace_size(b, h, L, d, int(block)), workspace, q.device)
    abi.check(abi.lightning_prefill_snapshots(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(o), _ptr(state_out), int(interval), _ptr(snapshots) if n > 0 else None,
        _ptr(workspace), _nbytes(workspace), _stream(stream), _VARIANTS[variant]))
    return o, state_out, snapshots


def prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, d_o: torch.Tensor, slopes: torch.Tensor,
                     block: int, state_in: Optional[torch.Tensor] = None,
                     d_state_out: Optional[torch.Tensor] = None, want_state_grad: bool = True,
                     variant: str = "auto", workspace: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill_backward: returns (dq, dk, dv, d_state_in) for the loss
    sum(d_o * o) + sum(d_state_out * state_out). The workspace the tensor-core
    kernels need is allocated with torch unless a uint8 tensor is passed."""
    if variant not in ("auto", "simt", "pair"):
        raise ValueError("backward variant must be auto, simt or pair")
    b, h, L, d = _qkv(q, k, v, (("d_o", d_o),))
    _need_cuda("slopes", slopes, torch.float32, (h,))
    _state("state_in", state_in, b, h, d)
    _state("d_state_out", d_state_out, b, h, d)
    need = abi.lightning_prefill_backward_workspace_size(_DTYPES[q.dtype], b, h, L, d, int(block),
                                                          _VARIANTS[variant])
    workspace = _workspace(need, workspace, q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ds_in = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device) if want_state_grad else None
    abi.check(abi.lightning_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(d_o), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block),
        _ptr(state_in), _ptr(d_state_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds_in), _ptr(workspace),
        _nbytes(workspace), _stream(stream), _VARIANTS[variant]))
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
    _need_cuda("gate", gate, o.dtype, (b, L, h * d))
    _need_cuda("gamma", gamma, torch.float32, (h * d,))
    if y is None:
        y = torch.empty((b, L, h * d), dtype=o.dtype, device=o.device)
    else:
        _need_cuda("y", y, o.dtype, (b, L, h * d))
    abi.check(abi.lightning_norm_gate(_ptr(o), _ptr(gate), _DTYPES[o.dtype], _ptr(gamma), float(eps), b, h, L, d,
                                      1 if per_head else 0, _ptr(y), _stream(stream)))
    return y


def prefill_norm_gate(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, slopes: torch.Tensor, block: int,
                      gate: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                      state_in: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                      state_out: Optional[torch.Tensor] = None, want_state: bool = True,
                      workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """lightning_prefill_norm_gate: the prefill with the per-head normalisation and
    gate fused into its epilogue; returns (y [batch, seq, heads*dim], state_out).
    The workspace is allocated with torch unless given."""
    b, h, L, d = _qkv(q, k, v)
    _need_cuda("slopes", slopes, torch.float32, (h,))
    _need_cuda("gate", gate, q.dtype, (b, L, h * d))
    _need_cuda("gamma", gamma, torch.float32, (h * d,))
    _state("state_in", state_in, b, h, d)
    if y is None:
        y = torch.empty((b, L, h * d), dtype=q.dtype, device=q.device)
    else:
        _need_cuda("y", y, q.dtype, (b, L, h * d))
    if state_out is None and want_state:
        state_out = torch.empty((b, h, d, d), dtype=torch.float32, device=q.device)
    else:
        _state("state_out", state_out, b, h, d)
    workspace = _workspace(abi.lightning_prefill_workspace_size(b, h, L, d, int(block)), workspace, q.device)
    abi.check(abi.lightning_prefill_norm_gate(
        _ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, L, d, int(block), _ptr(state_in),
        _ptr(gate), _ptr(gamma), float(eps), _ptr(y), _ptr(state_out), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))
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
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [batch, heads, dim] and the caches [batch, kv_heads, cap, dim]")
    b, h, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or tuple(k_new.shape) != (b, hk, d) or tuple(v_new.shape) != (b, hk, d) \
            or v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent shapes: q [b, heads, dim], k/v_new [b, kv_heads, dim], caches [b, kv_heads, cap, dim]")
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda(name, t, q.dtype)
    _need_cuda("pos", pos, torch.int32, (b,))
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty_like(q)
    else:
        _need_cuda("o", o, q.dtype, q.shape)
    need = abi.lightning_gqa_decode_workspace_size(b, h, cap)
    workspace = _workspace(max(need, 16), workspace, q.device)
    abi.check(abi.lightning_gqa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                       _DTYPES[q.dtype], _ptr(pos), b, h, hk, d, cap, int(rot), float(rope_base),
                                       float(scale), _ptr(o), _ptr(workspace), _nbytes(workspace), _stream(stream)))
    return o


def gqa_prefill(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, start=0, rot: int = 64, rope_base: float = 10000.0,
                scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lightning_gqa_prefill: the softmax GQA layer over seq new tokens of each
    sequence b at positions start[b] .. start[b]+seq-1. Writes their rotated keys
    and values into the caches and returns o [batch, heads, seq, dim]. `start` is
    an int (the same for every sequence) or a CUDA int32 tensor [batch]. bf16
    (tensor cores) or float32 (CUDA cores); scale defaults to 1/sqrt(dim)."""
    if q.dtype not in _DTYPES:
        raise ValueError("q must be float32 or bfloat16")
    if q.dim() != 4 or k_cache.dim() != 4:
        raise ValueError("q must be [batch, heads, seq, dim] and the caches [batch, kv_heads, cap, dim]")
    b, h, L, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or tuple(k_new.shape) != (b, hk, L, d) or tuple(v_new.shape) != (b, hk, L, d) \
            or v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent shapes: q [b, heads, seq, dim], k/v_new [b, kv_heads, seq, dim], "
                         "caches [b, kv_heads, cap, dim]")
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda(name, t, q.dtype)
    if isinstance(start, torch.Tensor):
        _need_cuda("start", start, torch.int32, (b,))
    else:
        start = torch.full((b,), int(start), dtype=torch.int32, device=q.device)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty_like(q)
    else:
        _need_cuda("o", o, q.dtype, q.shape)
    need = abi.lightning_gqa_prefill_workspace_size(_DTYPES[q.dtype], b, h, L, d)
    workspace = _workspace(max(need, 16), workspace, q.device)
    abi.check(abi.lightning_gqa_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                        _DTYPES[q.dtype], _ptr(start), b, h, hk, L, d, cap, int(rot),
                                        float(rope_base), float(scale), _ptr(o), _ptr(workspace),
                                        _nbytes(workspace), _stream(stream)))
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
    _need_cuda("slopes", slopes, torch.float32, (h,))
    _need_cuda("state", state, torch.float32, (b, h, d, d))
    if o is None:
        o = torch.empty_like(q)
    else:
        _need_cuda("o", o, q.dtype, q.shape)
    abi.check(abi.lightning_decode(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(slopes), b, h, d,
                                   _ptr(state), _ptr(o), _stream(stream)))
    return o
