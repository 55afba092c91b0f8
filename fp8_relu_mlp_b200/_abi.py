"""ctypes binding of libfp8mlp.so (include/fp8mlp.h), same names as the C ABI.

Argument marshalling only: torch tensors are passed as their device pointers
(after a contiguity/device check), streams as their CUDA handles, and a
non-zero return code raises :class:`Fp8MlpError` with the library's detail
text.  Every step of the computation runs in the library's CUDA kernels;
there is no fallback: if the library cannot be loaded, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8mlp.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "fp8mlp.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fp8_relu_mlp_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_CUDA = 3
ERR_TIMEOUT = 4
ERR_NO_DEVICE = 5
STATUS_TIMEOUT = 1
STATUS_NONFINITE_AMAX = 2
STATUS_W2_DEGENERATE = 4
STATE_KEPT_SCALE = 1
FWD_EVAL_BF16 = 1
FWD_CALIBRATE = 2
CE_SUM = 0
CE_MEAN = 1
LAUNCH_OVERLAP_PREVIOUS = 1
DEBUG_STALL_PRODUCER = 1
DEBUG_STALL_AUX = 2
E4M3_MAX = 448.0


class Fp8MlpError(RuntimeError):
    def __init__(self, code, fn):
        self.code = code
        detail = lib.fp8mlp_last_error_detail().decode()
        msg = lib.fp8mlp_error_string(code).decode()
        super().__init__(f"{fn}: {msg} ({code}){': ' + detail if detail else ''}")


_i, _u64, _f, _p, _sz = ctypes.c_int, ctypes.c_ulonglong, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

_SIGS = {
    "fp8mlp_up_proj_fused": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _i, _p],
    "fp8mlp_down_proj_fp8": [_i, _i, _i, _p, _p, _p, _p, _p, _p],
    "fp8mlp_down_proj_bf16": [_i, _i, _i, _p, _p, _p, _p],
    "fp8mlp_mlp_fwd": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _p],
    "fp8mlp_partial_amax_shape": [_i, _i, _p, _p, _p, _p],
    "fp8mlp_partial_amax_count": [_i, _i],
    "fp8mlp_mlp_train_step": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p],
    "fp8mlp_scale_state_init": [_p, _f, _f, _p],
    "fp8mlp_amax_reduce_update_scale": [_p, _i, _p, _p],
    "fp8mlp_w2_fp8_cache_refresh": [_i, _i, _p, _p, _p, _p, _p],
    "fp8mlp_w2_fp8_cache_refresh_noalloc": [_i, _i, _p, _p, _p, _p],
    "fp8mlp_bwd_dpre": [_i, _i, _i, _p, _p, _p, _p, _i, _p],
    "fp8mlp_quantize_x": [_i, _i, _p, _p, _p, _p, _p],
    "fp8mlp_x_partial_amax_count": [_i, _i],
    "fp8mlp_w1_fp8_cache_refresh": [_i, _i, _p, _p, _p, _p, _p],
    "fp8mlp_up_proj_fused_fp8": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _p],
    "fp8mlp_linear_fwd_fp8": [_i, _i, _i, _p, _p, _p, _p, _p, _p],
    "fp8mlp_weight_fp8_cache_refresh": [_i, _i, _p, _p, _p, _p, _p],
    "fp8mlp_linear_bwd": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _i, _p],
    "fp8mlp_ce_fwd": [_i, _i, _i, _i, _p, _p, _p, _p, _f, _p, _p, _p, _p, _p],
    "fp8mlp_ce_fwd_fp8": [_i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _f, _p, _p, _p, _p, _p],
    "fp8mlp_ce_bwd_dlogits": [_i, _i, _i, _i, _p, _p, _p, _p, _f, _p, _p, _p, _i, _p, _p],
    "fp8mlp_ce_bwd_dlogits_fp8": [_i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _f, _p, _p, _p, _i, _p, _p],
    "fp8mlp_bwd_dx": [_i, _i, _i, _p, _p, _p, _p],
    "fp8mlp_bwd_dw": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _i, _p],
    "fp8mlp_mlp_bwd": [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p],
    "fp8mlp_rmsnorm_fwd": [_i, _i, _p, _p, _p, _p],
    "fp8mlp_rmsnorm_fwd_quant": [_i, _i, _p, _p, _p, _p, _p, _p, _p],
    "fp8mlp_rmsnorm_bwd": [_i, _i, _p, _p, _p, _p, _p, _p],
    "fp8mlp_residual_add": [_i, _i, _p, _p, _p, _p],
    "fp8mlp_get_device_status": [_p, _p],
    "fp8mlp_clear_device_status": [_p],
    "fp8mlp_set_wait_timeout_ns": [_u64],
    "fp8mlp_set_debug_flags": [_i],
    "fp8mlp_set_programmatic_launch": [_i],
}
for _n, _a in _SIGS.items():
    _fn = getattr(lib, _n)
    _fn.argtypes = _a
    _fn.restype = ctypes.c_int
lib.fp8mlp_workspace_size.argtypes = [_i, _i, _i]
lib.fp8mlp_workspace_size.restype = _sz
lib.fp8mlp_ce_workspace_size.argtypes = [_i, _i, _i]
lib.fp8mlp_ce_workspace_size.restype = _sz
lib.fp8mlp_linear_bwd_workspace_size.argtypes = [_i, _i, _i]
lib.fp8mlp_linear_bwd_workspace_size.restype = _sz
lib.fp8mlp_kernel_launch_count.argtypes = []
lib.fp8mlp_kernel_launch_count.restype = ctypes.c_ulonglong
for _n in ("fp8mlp_error_string",):
    getattr(lib, _n).argtypes = [_i]
    getattr(lib, _n).restype = ctypes.c_char_p
for _n in ("fp8mlp_last_error_detail", "fp8mlp_version"):
    getattr(lib, _n).argtypes = []
    getattr(lib, _n).restype = ctypes.c_char_p


def header_symbols() -> list[str]:
    """Every function the public header declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(fp8mlp_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return t.data_ptr()
    raise TypeError(f"cannot pass {type(t)} as a pointer")


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name, *args):
    rc = getattr(lib, name)(*args)
    if rc != OK:
        raise Fp8MlpError(rc, name)
    return rc


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def fp8mlp_up_proj_fused(M, d, h, x, W1, st, post, post_fp8, partial_amax, pre_debug=None, flags=0, stream=None):
    return _call("fp8mlp_up_proj_fused", M, d, h, _ptr(x), _ptr(W1), _ptr(st), _ptr(post), _ptr(post_fp8),
                 _ptr(partial_amax), _ptr(pre_debug), flags, _stream(stream))


def fp8mlp_down_proj_fp8(M, d, h, post_fp8, W2q_t, w2_scale_inv, st, out, stream=None):
    return _call("fp8mlp_down_proj_fp8", M, d, h, _ptr(post_fp8), _ptr(W2q_t), _ptr(w2_scale_inv), _ptr(st),
                 _ptr(out), _stream(stream))


def fp8mlp_down_proj_bf16(M, d, h, post, W2, out, stream=None):
    return _call("fp8mlp_down_proj_bf16", M, d, h, _ptr(post), _ptr(W2), _ptr(out), _stream(stream))


def fp8mlp_mlp_fwd(M, d, h, x, W1, W2q_t, w2_scale_inv, W2, st, post, post_fp8, partial_amax, out,
                   pre_debug=None, flags=0, stream=None):
    return _call("fp8mlp_mlp_fwd", M, d, h, _ptr(x), _ptr(W1), _ptr(W2q_t), _ptr(w2_scale_inv), _ptr(W2),
                 _ptr(st), _ptr(post), _ptr(post_fp8), _ptr(partial_amax), _ptr(out), _ptr(pre_debug), flags,
                 _stream(stream))


def fp8mlp_partial_amax_shape(M, h):
    """-> (row_blocks, col_blocks, block_rows, block_cols)"""
    v = [ctypes.c_int() for _ in range(4)]
    _call("fp8mlp_partial_amax_shape", M, h, *[ctypes.addressof(x) for x in v])
    return tuple(x.value for x in v)


def fp8mlp_mlp_train_step(M, d, h, x, W1, W2, dOut, W2q_t, w2_scale_inv, st, post, post_fp8, partial_amax, out,
                          dPre, dX, dW1, dW2, workspace, stream=None):
    return _call("fp8mlp_mlp_train_step", M, d, h, _ptr(x), _ptr(W1), _ptr(W2), _ptr(dOut), _ptr(W2q_t),
                 _ptr(w2_scale_inv), _ptr(st), _ptr(post), _ptr(post_fp8), _ptr(partial_amax), _ptr(out), _ptr(dPre),
                 _ptr(dX), _ptr(dW1), _ptr(dW2), _ptr(workspace), _stream(stream))


def fp8mlp_partial_amax_count(M, h):
    return int(lib.fp8mlp_partial_amax_count(M, h))


def fp8mlp_scale_state_init(st, margin, initial_scale, stream=None):
    return _call("fp8mlp_scale_state_init", _ptr(st), margin, initial_scale, _stream(stream))


def fp8mlp_amax_reduce_update_scale(partial_amax, n, st, stream=None):
    return _call("fp8mlp_amax_reduce_update_scale", _ptr(partial_amax), n, _ptr(st), _stream(stream))


def fp8mlp_w2_fp8_cache_refresh(h, d, W2, W2q_t, w2_scale_inv, workspace, stream=None):
    return _call("fp8mlp_w2_fp8_cache_refresh", h, d, _ptr(W2), _ptr(W2q_t), _ptr(w2_scale_inv), _ptr(workspace),
                 _stream(stream))


def fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, W2q_t, w2_scale_inv, stream=None):
    """W2 cache refresh without a workspace: for callers that cannot hand the
    library device memory (see include/fp8mlp.h)."""
    return _call("fp8mlp_w2_fp8_cache_refresh_noalloc", h, d, _ptr(W2), _ptr(W2q_t), _ptr(w2_scale_inv),
                 _stream(stream))


def fp8mlp_workspace_size(M, d, h):
    return int(lib.fp8mlp_workspace_size(M, d, h))


def fp8mlp_quantize_x(M, d, x, st_x, x_fp8, partial_amax_x, stream=None):
    return _call("fp8mlp_quantize_x", M, d, _ptr(x), _ptr(st_x), _ptr(x_fp8), _ptr(partial_amax_x), _stream(stream))


def fp8mlp_x_partial_amax_count(M, d):
    return int(lib.fp8mlp_x_partial_amax_count(M, d))


def fp8mlp_w1_fp8_cache_refresh(h, d, W1, W1q, w1_scale_inv, workspace, stream=None):
    return _call("fp8mlp_w1_fp8_cache_refresh", h, d, _ptr(W1), _ptr(W1q), _ptr(w1_scale_inv), _ptr(workspace),
                 _stream(stream))


def fp8mlp_up_proj_fused_fp8(M, d, h, x_fp8, W1q, w1_scale_inv, st_x, st, post, post_fp8, partial_amax,
                             pre_debug=None, flags=0, stream=None):
    return _call("fp8mlp_up_proj_fused_fp8", M, d, h, _ptr(x_fp8), _ptr(W1q), _ptr(w1_scale_inv), _ptr(st_x),
                 _ptr(st), _ptr(post), _ptr(post_fp8), _ptr(partial_amax), _ptr(pre_debug), flags, _stream(stream))


def fp8mlp_linear_fwd_fp8(M, K, N, x_fp8, Wq, w_scale_inv, st_x, y, stream=None):
    return _call("fp8mlp_linear_fwd_fp8", M, K, N, _ptr(x_fp8), _ptr(Wq), _ptr(w_scale_inv), _ptr(st_x), _ptr(y),
                 _stream(stream))


def fp8mlp_weight_fp8_cache_refresh(N, K, W, Wq, w_scale_inv, workspace, stream=None):
    return _call("fp8mlp_weight_fp8_cache_refresh", N, K, _ptr(W), _ptr(Wq), _ptr(w_scale_inv), _ptr(workspace),
                 _stream(stream))


def fp8mlp_linear_bwd_workspace_size(M, K, N):
    return int(lib.fp8mlp_linear_bwd_workspace_size(M, K, N))


def fp8mlp_linear_bwd(M, K, N, x, W, dY, dX, dW, flags=0, stream=None, workspace=None):
    return _call("fp8mlp_linear_bwd", M, K, N, _ptr(x), _ptr(W), _ptr(dY), _ptr(dX), _ptr(dW), _ptr(workspace), flags,
                 _stream(stream))


def _host_floats(seq):
    """A host float array for a C `const float*` (None stays NULL); the
    returned object must stay alive for the call."""
    if seq is None:
        return None
    vals = [float(v) for v in seq]
    return (ctypes.c_float * len(vals))(*vals)


def fp8mlp_ce_workspace_size(M, V, T):
    return int(lib.fp8mlp_ce_workspace_size(M, V, T))


def fp8mlp_ce_fwd(M, d, V, T, x, W, targets, target_weights, softcap, lse, row_loss, loss, workspace, stream=None):
    w = _host_floats(target_weights)
    return _call("fp8mlp_ce_fwd", M, d, V, T, _ptr(x), _ptr(W), _ptr(targets), ctypes.cast(w, _p) if w else None,
                 softcap, _ptr(lse), _ptr(row_loss), _ptr(loss), _ptr(workspace), _stream(stream))


def fp8mlp_ce_fwd_fp8(M, d, V, T, x_fp8, st_x, Wq, w_scale_inv, targets, target_weights, softcap, lse, row_loss,
                      loss, workspace, stream=None):
    w = _host_floats(target_weights)
    return _call("fp8mlp_ce_fwd_fp8", M, d, V, T, _ptr(x_fp8), _ptr(st_x), _ptr(Wq), _ptr(w_scale_inv),
                 _ptr(targets), ctypes.cast(w, _p) if w else None, softcap, _ptr(lse), _ptr(row_loss), _ptr(loss),
                 _ptr(workspace), _stream(stream))


def fp8mlp_ce_bwd_dlogits(M, d, V, T, x, W, targets, target_weights, softcap, lse, loss, dloss, reduction, dlogits,
                          stream=None):
    w = _host_floats(target_weights)
    return _call("fp8mlp_ce_bwd_dlogits", M, d, V, T, _ptr(x), _ptr(W), _ptr(targets),
                 ctypes.cast(w, _p) if w else None, softcap, _ptr(lse), _ptr(loss), _ptr(dloss), reduction,
                 _ptr(dlogits), _stream(stream))


def fp8mlp_ce_bwd_dlogits_fp8(M, d, V, T, x_fp8, st_x, Wq, w_scale_inv, targets, target_weights, softcap, lse, loss,
                              dloss, reduction, dlogits, stream=None):
    w = _host_floats(target_weights)
    return _call("fp8mlp_ce_bwd_dlogits_fp8", M, d, V, T, _ptr(x_fp8), _ptr(st_x), _ptr(Wq), _ptr(w_scale_inv),
                 _ptr(targets), ctypes.cast(w, _p) if w else None, softcap, _ptr(lse), _ptr(loss), _ptr(dloss),
                 reduction, _ptr(dlogits), _stream(stream))


def fp8mlp_bwd_dpre(M, d, h, dOut, W2, post, dPre, flags=0, stream=None):
    return _call("fp8mlp_bwd_dpre", M, d, h, _ptr(dOut), _ptr(W2), _ptr(post), _ptr(dPre), flags, _stream(stream))


def fp8mlp_bwd_dx(M, d, h, dPre, W1, dX, stream=None):
    return _call("fp8mlp_bwd_dx", M, d, h, _ptr(dPre), _ptr(W1), _ptr(dX), _stream(stream))


def fp8mlp_bwd_dw(M, d, h, x, dPre, post, dOut, dW1, dW2, flags=0, stream=None):
    return _call("fp8mlp_bwd_dw", M, d, h, _ptr(x), _ptr(dPre), _ptr(post), _ptr(dOut), _ptr(dW1), _ptr(dW2),
                 flags, _stream(stream))


def fp8mlp_mlp_bwd(M, d, h, x, W1, W2, post, dOut, dPre, dX, dW1, dW2, stream=None):
    return _call("fp8mlp_mlp_bwd", M, d, h, _ptr(x), _ptr(W1), _ptr(W2), _ptr(post), _ptr(dOut), _ptr(dPre),
                 _ptr(dX), _ptr(dW1), _ptr(dW2), _stream(stream))


def fp8mlp_rmsnorm_fwd_quant(M, d, r, x, rstd, st_x, x_fp8, row_amax, stream=None):
    return _call("fp8mlp_rmsnorm_fwd_quant", M, d, _ptr(r), _ptr(x), _ptr(rstd), _ptr(st_x), _ptr(x_fp8),
                 _ptr(row_amax), _stream(stream))


def fp8mlp_rmsnorm_fwd(M, d, r, x, rstd, stream=None):
    return _call("fp8mlp_rmsnorm_fwd", M, d, _ptr(r), _ptr(x), _ptr(rstd), _stream(stream))


def fp8mlp_rmsnorm_bwd(M, d, r, rstd, dx, dr_in, dr_out, stream=None):
    return _call("fp8mlp_rmsnorm_bwd", M, d, _ptr(r), _ptr(rstd), _ptr(dx), _ptr(dr_in), _ptr(dr_out),
                 _stream(stream))


def fp8mlp_residual_add(M, d, r, out, r_next, stream=None):
    return _call("fp8mlp_residual_add", M, d, _ptr(r), _ptr(out), _ptr(r_next), _stream(stream))


def fp8mlp_get_device_status(stream=None):
    v = ctypes.c_uint()
    _call("fp8mlp_get_device_status", ctypes.addressof(v), _stream(stream))
    return v.value


def fp8mlp_clear_device_status(stream=None):
    return _call("fp8mlp_clear_device_status", _stream(stream))


def fp8mlp_set_wait_timeout_ns(ns):
    return _call("fp8mlp_set_wait_timeout_ns", int(ns))


def fp8mlp_set_programmatic_launch(enable):
    return _call("fp8mlp_set_programmatic_launch", int(bool(enable)))


def fp8mlp_set_debug_flags(flags):
    return _call("fp8mlp_set_debug_flags", int(flags))


def fp8mlp_error_string(code):
    return lib.fp8mlp_error_string(code).decode()


def fp8mlp_last_error_detail():
    return lib.fp8mlp_last_error_detail().decode()


def fp8mlp_kernel_launch_count():
    return int(lib.fp8mlp_kernel_launch_count())


def fp8mlp_version():
    return lib.fp8mlp_version().decode()
