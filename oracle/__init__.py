"""float64 CPU oracle for Lightning Attention — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never calls it and
shares no code with it.

The arithmetic lives in ``lightning_oracle.c`` (three forms of the same
result: F1 definition, F2 token recurrence, F3 blockwise, plus one decode
step, the state snapshots of a prefix cache, the gradients of one prefill,
the normalisation and gating of the output, and one decode step and one
prefill of the softmax GQA layer; see that file's header for
the formulas and their sources on the "MINIMAX SIGNAL LAB · M1" page, §03
Lightning Attention). This module only
marshals numpy arrays into it.

Inputs are numpy arrays: float32, or uint16 holding bfloat16 bit patterns.
Outputs are float64.

LA_ORACLE_LIBRARY, when set, names a compiled oracle to load instead of building
this one: the mutation tests point it at copies with a planted mistake, to show
that the pins reject them.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_F32, _BF16 = 0, 1
_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(os.environ.get("LA_ORACLE_LIBRARY") or _build())
        vp, ip, fp, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
        for name in ("la_oracle_definition", "la_oracle_recurrence"):
            fn = getattr(lib, name)
            fn.argtypes = [vp, vp, vp, ip, fp, ip, ip, ip, ip, fp, dp, dp]
            fn.restype = ctypes.c_int
        lib.la_oracle_blockwise.argtypes = [vp, vp, vp, ip, fp, ip, ip, ip, ip, ip, fp, dp, dp]
        lib.la_oracle_blockwise.restype = ctypes.c_int
        lib.la_oracle_decode.argtypes = [vp, vp, vp, ip, fp, ip, ip, ip, dp, dp]
        lib.la_oracle_decode.restype = ctypes.c_int
        lib.la_oracle_snapshots.argtypes = [vp, vp, ip, fp, ip, ip, ip, ip, fp, ip, dp]
        lib.la_oracle_snapshots.restype = ctypes.c_int
        lib.la_oracle_backward.argtypes = [vp, vp, vp, vp, ip, fp, ip, ip, ip, ip, fp, fp, dp, dp, dp, dp]
        lib.la_oracle_backward.restype = ctypes.c_int
        lib.la_oracle_norm_gate.argtypes = [vp, vp, ip, fp, ctypes.c_double, ip, ip, ip, ip, ip, dp]
        lib.la_oracle_norm_gate.restype = ctypes.c_int
        lib.la_oracle_gqa_decode.argtypes = [vp, vp, vp, vp, vp, ip, vp, ip, ip, ip, ip, ip, ip, ctypes.c_double,
                                             ctypes.c_double, dp]
        lib.la_oracle_gqa_decode.restype = ctypes.c_int
        lib.la_oracle_gqa_prefill.argtypes = [vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, ip, ip, ip,
                                              ctypes.c_double, ctypes.c_double, vp, ctypes.c_longlong, dp]
        lib.la_oracle_gqa_prefill.restype = ctypes.c_int
        lib.la_oracle_max_threads.restype = ctypes.c_int
        lib.la_oracle_set_threads.argtypes = [ip]
        _lib = lib
    return _lib


def threads() -> int:
    """Number of OpenMP threads the oracle uses."""
    return _load().la_oracle_max_threads()


def set_threads(n: int) -> None:
    _load().la_oracle_set_threads(int(n))


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return _F32
    if a.dtype == np.uint16:
        return _BF16
    raise TypeError("oracle inputs must be float32 or uint16 (bfloat16 bits), got %s" % a.dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prepare(q, k, v, slopes, state_in):
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    if not (q.shape == k.shape == v.shape) or q.ndim != 4:
        raise ValueError("q, k, v must share one [batch, heads, seq, dim] shape")
    code = _dtype_code(q)
    if _dtype_code(k) != code or _dtype_code(v) != code:
        raise TypeError("q, k, v must share a dtype")
    b, h, L, d = q.shape
    slopes = np.ascontiguousarray(slopes, dtype=np.float32)
    if slopes.shape != (h,):
        raise ValueError("slopes must have shape [heads]")
    if state_in is not None:
        state_in = np.ascontiguousarray(state_in, dtype=np.float32)
        if state_in.shape != (b, h, d, d):
            raise ValueError("state_in must have shape [batch, heads, dim, dim]")
    return q, k, v, code, slopes, state_in, (b, h, L, d)


def prefill(q, k, v, slopes, state_in=None, form="recurrence", block=None):
    """Return (o, state_out) in float64 for one prefill.

    form: "definition" (F1), "recurrence" (F2) or "blockwise" (F3, needs block).
    """
    q, k, v, code, slopes, state_in, (b, h, L, d) = _prepare(q, k, v, slopes, state_in)
    o = np.empty((b, h, L, d), dtype=np.float64)
    s_out = np.empty((b, h, d, d), dtype=np.float64)
    lib = _load()
    args_head = (_ptr(q), _ptr(k), _ptr(v), code, _ptr(slopes), b, h, L, d)
    if form == "definition":
        rc = lib.la_oracle_definition(*args_head, _ptr(state_in), _ptr(o), _ptr(s_out))
    elif form == "recurrence":
        rc = lib.la_oracle_recurrence(*args_head, _ptr(state_in), _ptr(o), _ptr(s_out))
    elif form == "blockwise":
        if block is None or int(block) <= 0:
            raise ValueError("the blockwise form needs a positive block size")
        rc = lib.la_oracle_blockwise(*args_head, int(block), _ptr(state_in), _ptr(o), _ptr(s_out))
    else:
        raise ValueError("unknown form %r" % (form,))
    if rc != 0:
        raise RuntimeError("oracle %s failed (rc=%d)" % (form, rc))
    return o, s_out


def snapshots(k, v, slopes, interval, state_in=None):
    """States after the first (n+1)*interval tokens, n = 0 .. seq//interval - 1.

    Returns float64 [batch, heads, seq//interval, dim, dim] (token recurrence)."""
    k, v, _, code, slopes, state_in, (b, h, L, d) = _prepare(k, v, v, slopes, state_in)
    interval = int(interval)
    if interval <= 0:
        raise ValueError("interval must be positive")
    out = np.empty((b, h, L // interval, d, d), dtype=np.float64)
    if out.size == 0:
        return out
    rc = _load().la_oracle_snapshots(_ptr(k), _ptr(v), code, _ptr(slopes), b, h, L, d, _ptr(state_in),
                                     interval, _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle snapshots failed (rc=%d)" % rc)
    return out


def backward(q, k, v, d_o, slopes, state_in=None, d_state_out=None):
    """Gradients of one prefill for the loss sum(d_o * o) + sum(d_state_out * state_out).

    Returns float64 (dq, dk, dv, d_state_in)."""
    q, k, v, code, slopes, state_in, (b, h, L, d) = _prepare(q, k, v, slopes, state_in)
    d_o = np.ascontiguousarray(d_o)
    if d_o.shape != q.shape or _dtype_code(d_o) != code:
        raise ValueError("d_o must match q in shape and dtype")
    if d_state_out is not None:
        d_state_out = np.ascontiguousarray(d_state_out, dtype=np.float32)
        if d_state_out.shape != (b, h, d, d):
            raise ValueError("d_state_out must have shape [batch, heads, dim, dim]")
    dq, dk, dv = (np.empty((b, h, L, d), dtype=np.float64) for _ in range(3))
    ds_in = np.empty((b, h, d, d), dtype=np.float64)
    rc = _load().la_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(d_o), code, _ptr(slopes), b, h, L, d,
                                    _ptr(state_in), _ptr(d_state_out), _ptr(dq), _ptr(dk), _ptr(dv),
                                    _ptr(ds_in))
    if rc != 0:
        raise RuntimeError("oracle backward failed (rc=%d)" % rc)
    return dq, dk, dv, ds_in


def norm_gate(o, g, gamma, eps, per_head):
    """RMS normalisation then sigmoid gating of an attention output.

    o: [batch, heads, seq, dim]; g: [batch, seq, heads*dim] (same dtype);
    gamma: [heads*dim]. Returns y float64 [batch, seq, heads*dim]."""
    o = np.ascontiguousarray(o)
    g = np.ascontiguousarray(g)
    code = _dtype_code(o)
    if _dtype_code(g) != code:
        raise TypeError("o and g must share a dtype")
    b, h, L, d = o.shape
    if g.shape != (b, L, h * d):
        raise ValueError("g must have shape [batch, seq, heads*dim]")
    gamma = np.ascontiguousarray(gamma, dtype=np.float32)
    if gamma.shape != (h * d,):
        raise ValueError("gamma must have shape [heads*dim]")
    y = np.empty((b, L, h * d), dtype=np.float64)
    rc = _load().la_oracle_norm_gate(_ptr(o), _ptr(g), code, _ptr(gamma), float(eps), b, h, L, d,
                                     1 if per_head else 0, _ptr(y))
    if rc != 0:
        raise RuntimeError("oracle norm_gate failed (rc=%d)" % rc)
    return y


def gqa_decode(q, k_new, v_new, k_cache, v_cache, pos, rot, base, scale):
    """One decode step of the softmax GQA layer (RoPE on the first `rot` dims).

    q: [batch, heads, dim]; k_new, v_new: [batch, kv_heads, dim]; caches:
    [batch, kv_heads, cap, dim] (rotated keys; positions < pos[b] filled);
    pos: [batch] int. Returns o float64 [batch, heads, dim]."""
    q, k_new, v_new, k_cache, v_cache = (np.ascontiguousarray(x) for x in (q, k_new, v_new, k_cache, v_cache))
    code = _dtype_code(q)
    for x in (k_new, v_new, k_cache, v_cache):
        if _dtype_code(x) != code:
            raise TypeError("all gqa inputs must share a dtype")
    b, h, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or k_new.shape != (b, hk, d) or v_new.shape != (b, hk, d) or v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent gqa shapes")
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    if pos.shape != (b,):
        raise ValueError("pos must have shape [batch]")
    o = np.empty((b, h, d), dtype=np.float64)
    rc = _load().la_oracle_gqa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), code,
                                      _ptr(pos), b, h, hk, d, cap, int(rot), float(base), float(scale), _ptr(o))
    if rc != 0:
        raise RuntimeError("oracle gqa_decode failed (rc=%d)" % rc)
    return o


def gqa_prefill(q, k_new, v_new, k_cache, v_cache, start, rot, base, scale, rows=None):
    """The softmax GQA layer over `seq` new tokens at positions start ..
    start+seq-1 (RoPE on the first `rot` dims, causal).

    q: [batch, heads, seq, dim]; k_new, v_new: [batch, kv_heads, seq, dim];
    caches: [batch, kv_heads, cap, dim] (rotated keys; positions < start
    filled). rows: None for every output (returns o float64 [batch, heads,
    seq, dim]) or indices (b*heads + h)*seq + i (returns [len(rows), dim])."""
    q, k_new, v_new, k_cache, v_cache = (np.ascontiguousarray(x) for x in (q, k_new, v_new, k_cache, v_cache))
    code = _dtype_code(q)
    for x in (k_new, v_new, k_cache, v_cache):
        if _dtype_code(x) != code:
            raise TypeError("all gqa inputs must share a dtype")
    b, h, L, d = q.shape
    bk, hk, cap, dk = k_cache.shape
    if (bk, dk) != (b, d) or k_new.shape != (b, hk, L, d) or v_new.shape != k_new.shape or \
            v_cache.shape != k_cache.shape:
        raise ValueError("inconsistent gqa shapes")
    if rows is None:
        o = np.empty((b, h, L, d), dtype=np.float64)
        rp, n = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
        o = np.empty((rows.size, d), dtype=np.float64)
        rp, n = _ptr(rows), rows.size
    rc = _load().la_oracle_gqa_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), code,
                                       int(start), b, h, hk, L, d, cap, int(rot), float(base), float(scale), rp, n,
                                       _ptr(o))
    if rc != 0:
        raise RuntimeError("oracle gqa_prefill failed (rc=%d)" % rc)
    return o


def rope(x, pos, rot, base):
    """RoPE of the last axis of x (float64 reference of the oracle's rotation,
    used by tests to fill key caches): x [..., dim] at position pos."""
    x = np.asarray(x, dtype=np.float64)
    half = rot // 2
    i = np.arange(half, dtype=np.float64)
    ang = float(pos) * np.power(float(base), -2.0 * i / rot)
    out = x.copy()
    cs, sn = np.cos(ang), np.sin(ang)
    out[..., :half] = x[..., :half] * cs - x[..., half:rot] * sn
    out[..., half:rot] = x[..., half:rot] * cs + x[..., :half] * sn
    return out


def decode(q, k, v, slopes, state):
    """One decode step. q, k, v: [batch, heads, dim]; state: [batch, heads, dim, dim].

    Returns (o float64 [batch, heads, dim], new state float64)."""
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    if not (q.shape == k.shape == v.shape) or q.ndim != 3:
        raise ValueError("q, k, v must share one [batch, heads, dim] shape")
    code = _dtype_code(q)
    b, h, d = q.shape
    slopes = np.ascontiguousarray(slopes, dtype=np.float32)
    S = np.array(state, dtype=np.float64, copy=True, order="C")
    if S.shape != (b, h, d, d):
        raise ValueError("state must have shape [batch, heads, dim, dim]")
    o = np.empty((b, h, d), dtype=np.float64)
    rc = _load().la_oracle_decode(_ptr(q), _ptr(k), _ptr(v), code, _ptr(slopes), b, h, d,
                                  _ptr(S), _ptr(o))
    if rc != 0:
        raise RuntimeError("oracle decode failed (rc=%d)" % rc)
    return o, S


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float64 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
