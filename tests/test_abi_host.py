"""Host-side checks of the C-ABI library (no GPU needed, no compute calls).

The library must load, export every function the public header declares, and
reject bad arguments on the host before touching CUDA.  With valid arguments
and no GPU present it must say so (FP8MLP_ERR_NO_DEVICE) rather than fall back.
"""
import ctypes
import re

import pytest

from fp8_relu_mlp_b200 import _abi as A

FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced on the host


def test_library_exports_every_header_symbol():
    syms = A.header_symbols()
    assert len(syms) >= 20
    for s in syms:
        assert hasattr(A.lib, s), s
        assert hasattr(A, s), f"binding lacks {s}"


# the calls the boundary of the block is specified with (forward, backward,
# W2 cache refresh, amax reduction with the scale update, and their helpers)
BOUNDARY = ["fp8mlp_mlp_fwd", "fp8mlp_mlp_bwd", "fp8mlp_w2_fp8_cache_refresh", "fp8mlp_amax_reduce_update_scale",
            "fp8mlp_scale_state_init", "fp8mlp_workspace_size", "fp8mlp_partial_amax_count",
            "fp8mlp_get_device_status", "fp8mlp_error_string"]


def test_header_declares_the_boundary_calls():
    syms = set(A.header_symbols())
    for s in BOUNDARY + ["fp8mlp_up_proj_fused", "fp8mlp_down_proj_fp8", "fp8mlp_bwd_dpre", "fp8mlp_bwd_dx",
                         "fp8mlp_bwd_dw", "fp8mlp_partial_amax_shape"]:
        assert s in syms, s
        assert hasattr(A.lib, s), s


def test_partial_amax_count_is_the_shape_product():
    for M, h in [(0, 3072), (1, 16), (300, 272), (16384, 3072), (49152, 3072), (65536, 4096)]:
        rb, cb, br, bc = A.fp8mlp_partial_amax_shape(M, h)
        assert A.fp8mlp_partial_amax_count(M, h) == rb * cb
        # every block of post is covered
        assert rb * br >= M and cb * bc >= h
    assert A.fp8mlp_partial_amax_count(16384, 3072) == 512 * 48
    assert A.fp8mlp_partial_amax_count(-1, 16) == 0


def test_scale_state_layout_is_32_bytes():
    text = open(A.HEADER).read()
    body = re.search(r"typedef struct fp8mlp_scale_state \{(.*?)\} fp8mlp_scale_state;", text, re.S).group(1)
    fields = re.findall(r"(float|int32_t)\s+(\w+)(\[(\d+)\])?;", body)
    assert [f[1] for f in fields] == ["amax_prev", "scale", "scale_inv", "margin", "step", "flags", "pad"]
    assert sum(4 * (int(f[3]) if f[3] else 1) for f in fields) == 32


def test_version_and_error_strings():
    assert "sm_100a" in A.fp8mlp_version()
    assert A.fp8mlp_error_string(0) == "ok"
    assert A.fp8mlp_error_string(A.ERR_NO_DEVICE) == "no sm_100a device"
    assert A.fp8mlp_error_string(99) == "unknown error code"


def _rc(name, *args):
    return getattr(A.lib, name)(*args)


@pytest.mark.parametrize("M,d,h,code", [(-1, 64, 256, A.ERR_INVALID_ARG), (16, 8, 256, A.ERR_UNSUPPORTED_SHAPE),
                                        (16, 64, 250, A.ERR_UNSUPPORTED_SHAPE), (16, 72, 0, A.ERR_UNSUPPORTED_SHAPE)])
def test_shape_checks(M, d, h, code):
    assert _rc("fp8mlp_up_proj_fused", M, d, h, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None) == code
    assert _rc("fp8mlp_bwd_dpre", M, d, h, FAKE, FAKE, FAKE, FAKE, 0, None) == code


def test_null_and_misaligned_pointers_rejected():
    args = [256, 64, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None]
    for pos in (3, 4, 6, 7):          # x, W1, post, post_fp8
        a = list(args)
        a[pos] = None
        assert _rc("fp8mlp_up_proj_fused", *a) == A.ERR_INVALID_ARG
        a[pos] = FAKE + 8
        assert _rc("fp8mlp_up_proj_fused", *a) == A.ERR_INVALID_ARG
        assert "aligned" in A.fp8mlp_last_error_detail()
    # state is needed only when the FP8 copy is written
    a = list(args)
    a[5] = None
    assert _rc("fp8mlp_up_proj_fused", *a) == A.ERR_INVALID_ARG
    a[10] = A.FWD_CALIBRATE
    a[7] = None
    assert _rc("fp8mlp_up_proj_fused", *a) in (A.ERR_NO_DEVICE, A.OK)


def test_flag_checks():
    assert _rc("fp8mlp_up_proj_fused", 16, 64, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 8, None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_mlp_fwd", 16, 64, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
               A.FWD_EVAL_BF16 | A.FWD_CALIBRATE, None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_set_debug_flags", 4) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_set_debug_flags", A.DEBUG_STALL_AUX) == 0 and _rc("fp8mlp_set_debug_flags", 0) == 0
    assert _rc("fp8mlp_set_wait_timeout_ns", 0) == A.ERR_INVALID_ARG


def test_launch_flag_checks():
    assert _rc("fp8mlp_bwd_dpre", 16, 64, 256, FAKE, FAKE, FAKE, FAKE, 2, None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_bwd_dw", 16, 64, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, None) == A.ERR_INVALID_ARG


def test_linear_bwd_checks_before_enqueueing():
    # host-side checks (pointers, dX alignment, workspace alignment) come
    # before the device query, so they answer without a GPU
    args = [300, 768, 2304, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None]
    for pos, bad in ((3, None), (4, FAKE + 8), (5, None), (6, FAKE + 4), (8, FAKE + 8)):
        a = list(args)
        a[pos] = bad
        assert _rc("fp8mlp_linear_bwd", *a) == A.ERR_INVALID_ARG, pos
    assert A.fp8mlp_linear_bwd_workspace_size(300, 768, 2304) == 4 * 768 * 2304
    assert A.fp8mlp_linear_bwd_workspace_size(100, 768, 2304) == 0


def test_train_step_checks_before_enqueueing():
    # M, d, h, x, W1, W2, dOut, W2q_t, w2_scale_inv, st, post, post_fp8, pa, out, dPre, dX, dW1, dW2, ws, stream
    args = [256, 64, 256] + [FAKE] * 16 + [None]
    for pos in range(3, 19):
        a = list(args)
        a[pos] = None
        assert _rc("fp8mlp_mlp_train_step", *a) == A.ERR_INVALID_ARG, pos
    a = list(args)
    a[4] = FAKE + 8          # W1 misaligned
    assert _rc("fp8mlp_mlp_train_step", *a) == A.ERR_INVALID_ARG
    a = list(args)
    a[1] = 72                # d not a multiple of 16
    assert _rc("fp8mlp_mlp_train_step", *a) == A.ERR_UNSUPPORTED_SHAPE


def test_scale_state_init_checks():
    assert _rc("fp8mlp_scale_state_init", FAKE, ctypes.c_float(0.0), ctypes.c_float(1.0), None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_scale_state_init", FAKE, ctypes.c_float(2.0), ctypes.c_float(-1.0), None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_scale_state_init", FAKE, ctypes.c_float(float("nan")), ctypes.c_float(1.0), None) == A.ERR_INVALID_ARG
    assert _rc("fp8mlp_amax_reduce_update_scale", FAKE, -1, FAKE, None) == A.ERR_INVALID_ARG


def test_empty_batch_is_a_no_op():
    # M = 0: nothing to do, nothing enqueued, no device needed
    assert _rc("fp8mlp_up_proj_fused", 0, 64, 256, None, None, None, None, None, None, None, 0, None) == A.OK
    assert _rc("fp8mlp_down_proj_fp8", 0, 64, 256, None, None, None, None, None, None) == A.OK
    assert _rc("fp8mlp_bwd_dx", 0, 64, 256, None, None, None, None) == A.OK


def test_partial_amax_shape():
    assert A.fp8mlp_partial_amax_shape(16384, 3072) == (512, 48, 32, 64)
    assert A.fp8mlp_partial_amax_shape(129, 256) == (8, 4, 32, 64)
    assert A.fp8mlp_partial_amax_shape(300, 272) == (16, 8, 32, 64)
    assert A.fp8mlp_partial_amax_shape(0, 256) == (0, 4, 32, 64)
    assert A.fp8mlp_workspace_size(16384, 768, 3072) >= 4


def test_valid_call_without_gpu_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = _rc("fp8mlp_up_proj_fused", 256, 64, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None)
    assert rc == A.ERR_NO_DEVICE
    with pytest.raises(A.Fp8MlpError):
        A.fp8mlp_bwd_dx(128, 64, 256, FAKE, FAKE, FAKE, stream=0)


def test_python_binding_rejects_non_contiguous():
    import torch
    t = torch.zeros(4, 4)[:, ::2]
    with pytest.raises(ValueError):
        A.fp8mlp_bwd_dx(4, 16, 16, t, t, t, stream=0)


def _ce_rc(**kw):
    a = dict(M=256, d=64, V=512, T=1, x=FAKE, W=FAKE, targets=FAKE, w=None, cap=15.0, lse=FAKE, row=None,
             loss=FAKE, ws=FAKE)
    a.update(kw)
    return _rc("fp8mlp_ce_fwd", a["M"], a["d"], a["V"], a["T"], a["x"], a["W"], a["targets"], a["w"],
               ctypes.c_float(a["cap"]), a["lse"], a["row"], a["loss"], a["ws"], None)


def test_ce_argument_checks():
    assert _ce_rc(T=0) == A.ERR_INVALID_ARG
    assert _ce_rc(T=5) == A.ERR_INVALID_ARG
    assert _ce_rc(cap=0.0) == A.ERR_INVALID_ARG
    assert _ce_rc(cap=41.0) == A.ERR_INVALID_ARG            # exp(-2c) would leave fp32's normal range
    assert _ce_rc(cap=float("nan")) == A.ERR_INVALID_ARG
    assert _ce_rc(V=500) == A.ERR_UNSUPPORTED_SHAPE         # vocabulary not a multiple of 16
    assert _ce_rc(targets=None) == A.ERR_INVALID_ARG
    assert _ce_rc(targets=FAKE + 2) == A.ERR_INVALID_ARG     # int32 targets need 4-byte alignment
    assert _ce_rc(loss=None) == A.ERR_INVALID_ARG
    bad_w = (ctypes.c_float * 1)(float("inf"))
    assert _ce_rc(w=ctypes.cast(bad_w, ctypes.c_void_p)) == A.ERR_INVALID_ARG
    # the backward's reduction selector
    rc = _rc("fp8mlp_ce_bwd_dlogits", 256, 64, 512, 1, FAKE, FAKE, FAKE, None, ctypes.c_float(15.0), FAKE, FAKE,
             None, 2, FAKE, None)
    assert rc == A.ERR_INVALID_ARG


def test_ce_workspace_layout():
    # [block sums][partials: 4 per 256-column tile (one per epilogue warp's
    # 64 columns) x M][z at targets: M x T], 256-byte aligned pieces
    M, V, T = 16384, 50304, 1
    nparts = 4 * -(-V // 256)
    want = (2 * 8 * (M // 32)) + 4 * nparts * M + 4 * M * T
    got = A.fp8mlp_ce_workspace_size(M, V, T)
    assert want <= got < want + 3 * 256
    assert A.fp8mlp_ce_workspace_size(0, V, T) == 0


def test_ce_valid_call_without_gpu_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _ce_rc() == A.ERR_NO_DEVICE
