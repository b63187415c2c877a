"""ctypes binding of liblightning.so — argument marshalling only.

Every entry point of include/lightning.h is exposed under the same name with
the same arguments (device pointers as ints, sizes, a cudaStream_t as int).
The library is loaded from this package directory; if it has not been built
the first call raises, so a missing CUDA extension can never be mistaken for
a result.
"""
import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(PKG, "liblightning.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "lightning.h")

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT = range(5)
LA_DTYPE_F32, LA_DTYPE_BF16 = 0, 1
LA_VARIANT_AUTO, LA_VARIANT_SIMT, LA_VARIANT_TCGEN05, LA_VARIANT_TCGEN05_PAIR = 0, 1, 2, 3

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

_SIGNATURES = {
    "lightning_abi_version": ([], _i),
    "lightning_prefill": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "lightning_prefill_ex": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp,
                              _i], _i),
    "lightning_prefill_selected_variant": ([_i, _i, _i, _i, _i, _i, _i], _i),
    "lightning_prefill_workspace_size": ([_i, _i, _i, _i, _i], _sz),
    "lightning_prefill_snapshots": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp,
                                     _sz, _vp, _i], _i),
    "lightning_prefill_snapshot_count": ([_i, _i], _i),
    "lightning_norm_gate": ([_vp, _vp, _i, _vp, ctypes.c_float, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "lightning_prefill_norm_gate": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, ctypes.c_float,
                                     _vp, _vp, _vp, _sz, _vp], _i),
    "lightning_gqa_decode": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_double,
                              ctypes.c_float, _vp, _vp, _sz, _vp], _i),
    "lightning_gqa_decode_workspace_size": ([_i, _i, _i], _sz),
    "lightning_gqa_prefill": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, ctypes.c_double,
                               ctypes.c_float, _vp, _vp, _sz, _vp], _i),
    "lightning_gqa_prefill_workspace_size": ([_i, _i, _i, _i, _i], _sz),
    "lightning_prefill_backward": ([_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _sz, _vp, _i], _i),
    "lightning_prefill_backward_workspace_size": ([_i, _i, _i, _i, _i, _i, _i], _sz),
    "lightning_prefill_backward_noalloc": ([_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp,
                                            _vp, _vp, _vp, _i], _i),
    "lightning_prefill_backward_noalloc_capacity": ([], _sz),
    "lightning_decode": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _vp, _vp, _vp], _i),
    "lightning_device_status": ([_vp], _i),
    "lightning_last_device_status": ([_vp], _i),
    "lightning_selftest_wait_timeout": ([_vp], _i),
    "lightning_status_string": ([_i], ctypes.c_char_p),
    "lightning_last_error_message": ([], ctypes.c_char_p),
}

_lib = None


class LightningError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s (%s)" % (message, status_string(status)) if _lib else message)
        self.status = status


def declared_functions():
    """Names of the functions include/lightning.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lightning_\w+)\s*\(", text)))


def load():
    """Load liblightning.so once; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY):
            raise RuntimeError("liblightning.so is not built: run __graft_entry__.build() "
                               "(or python -m linear_attention_lightning_b200.build)")
        lib = ctypes.CDLL(LIBRARY)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def status_string(status):
    return load().lightning_status_string(int(status)).decode()


def last_error_message():
    return load().lightning_last_error_message().decode()


def check(status):
    if status != LA_OK:
        raise LightningError(status, last_error_message() or status_string(status))
    return status


def lightning_abi_version():
    return load().lightning_abi_version()


def lightning_prefill(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o, state_out,
                      workspace, workspace_bytes, stream):
    return load().lightning_prefill(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o,
                                    state_out, workspace, workspace_bytes, stream)


def lightning_prefill_ex(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o, state_out,
                         workspace, workspace_bytes, stream, variant):
    return load().lightning_prefill_ex(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                       o, state_out, workspace, workspace_bytes, stream, variant)


def lightning_prefill_selected_variant(dtype, batch, heads, seq, dim, block, variant):
    return load().lightning_prefill_selected_variant(dtype, batch, heads, seq, dim, block, variant)


def lightning_prefill_workspace_size(batch, heads, seq, dim, block):
    return load().lightning_prefill_workspace_size(batch, heads, seq, dim, block)


def lightning_prefill_snapshots(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o, state_out,
                                interval, snapshots, workspace, workspace_bytes, stream, variant):
    return load().lightning_prefill_snapshots(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                              o, state_out, interval, snapshots, workspace, workspace_bytes, stream,
                                              variant)


def lightning_prefill_backward(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in,
                               d_state_out, dq, dk, dv, d_state_in, workspace, workspace_bytes, stream, variant):
    return load().lightning_prefill_backward(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block,
                                             state_in, d_state_out, dq, dk, dv, d_state_in, workspace,
                                             workspace_bytes, stream, variant)


def lightning_prefill_backward_noalloc(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                       d_state_out, dq, dk, dv, d_state_in, stream, variant):
    return load().lightning_prefill_backward_noalloc(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block,
                                                     state_in, d_state_out, dq, dk, dv, d_state_in, stream, variant)


def lightning_prefill_backward_noalloc_capacity():
    return load().lightning_prefill_backward_noalloc_capacity()


def lightning_prefill_backward_workspace_size(dtype, batch, heads, seq, dim, block, variant):
    return load().lightning_prefill_backward_workspace_size(dtype, batch, heads, seq, dim, block, variant)


def lightning_norm_gate(o, gate, dtype, gamma, eps, batch, heads, seq, dim, per_head, y, stream):
    return load().lightning_norm_gate(o, gate, dtype, gamma, eps, batch, heads, seq, dim, per_head, y, stream)


def lightning_prefill_norm_gate(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, gate, gamma, eps,
                                y, state_out, workspace, workspace_bytes, stream):
    return load().lightning_prefill_norm_gate(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                              gate, gamma, eps, y, state_out, workspace, workspace_bytes, stream)


def lightning_gqa_decode(q, k_new, v_new, k_cache, v_cache, dtype, pos, batch, heads, kv_heads, dim, cap, rot,
                         rope_base, scale, o, workspace, workspace_bytes, stream):
    return load().lightning_gqa_decode(q, k_new, v_new, k_cache, v_cache, dtype, pos, batch, heads, kv_heads, dim,
                                       cap, rot, rope_base, scale, o, workspace, workspace_bytes, stream)


def lightning_gqa_decode_workspace_size(batch, heads, cap):
    return load().lightning_gqa_decode_workspace_size(batch, heads, cap)


def lightning_gqa_prefill(q, k_new, v_new, k_cache, v_cache, dtype, start, batch, heads, kv_heads, seq, dim, cap,
                          rot, rope_base, scale, o, workspace, workspace_bytes, stream):
    return load().lightning_gqa_prefill(q, k_new, v_new, k_cache, v_cache, dtype, start, batch, heads, kv_heads, seq,
                                        dim, cap, rot, rope_base, scale, o, workspace, workspace_bytes, stream)


def lightning_gqa_prefill_workspace_size(dtype, batch, heads, seq, dim):
    return load().lightning_gqa_prefill_workspace_size(dtype, batch, heads, seq, dim)


def lightning_prefill_snapshot_count(seq, interval):
    return load().lightning_prefill_snapshot_count(seq, interval)


def lightning_decode(q, k, v, dtype, slopes, batch, heads, dim, state, o, stream):
    return load().lightning_decode(q, k, v, dtype, slopes, batch, heads, dim, state, o, stream)


def lightning_device_status(stream):
    return load().lightning_device_status(stream)


def lightning_last_device_status(stream):
    return load().lightning_last_device_status(stream)


def lightning_selftest_wait_timeout(stream):
    return load().lightning_selftest_wait_timeout(stream)
