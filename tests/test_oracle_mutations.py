"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Every mutation below is a plausible slip in writing the oracle: a dropped
term, a wrong rounding mode, a transposed operand, a missing factor.  The
test patches the oracle function, runs the pins that should catch it, and
requires that at least one of them fails.
"""
import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import ref


def _trunc_bf16(v):
    u = np.asarray(v, np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def _e4m3_half_away(v):
    v = np.asarray(v, np.float32).astype(np.float64)
    a = np.abs(v)
    _, E = np.frexp(np.where(a > 0, a, 1.0))
    q = np.ldexp(1.0, np.maximum(E.astype(np.int64) - 1, -6) - 3)
    r = np.minimum(np.floor(a / q + 0.5) * q, 448.0)
    return ref._orig_e4m3((np.sign(v) * r).astype(np.float32))


def _e4m3_no_sat(v):
    v = np.asarray(v, np.float32)
    out = ref._orig_e4m3(v)
    return np.where(np.abs(v) > 448, np.uint8(0x7F), out).astype(np.uint8)


MUTATIONS = {
    # name: (oracle attribute, mutated version, pins expected to catch it)
    "bf16_truncates": ("bf16_bits_from_f32", lambda orig: _trunc_bf16,
                       ["test_bf16_matches_torch_and_ml_dtypes"]),
    "e4m3_half_away": ("e4m3_bits_from_f32", lambda orig: _e4m3_half_away,
                       ["test_e4m3_hand_cases", "test_e4m3_random_fp32"]),
    "e4m3_no_saturation": ("e4m3_bits_from_f32", lambda orig: _e4m3_no_sat,
                           ["test_e4m3_hand_cases", "test_worked_example_golden"]),
    "up_proj_operand_swapped": ("up_proj", lambda orig: (lambda x, W1: ref.bf16_to_f64(x) @ ref.bf16_to_f64(W1).T[:, ::-1]),
                                ["test_up_proj_bruteforce"]),
    "relu_dropped": ("relu2_post", lambda orig: (lambda pre: ref.bf16_bits_from_f32((ref.f32(pre) * ref.f32(pre)).astype(np.float32))),
                     ["test_relu2_invariants"]),
    "square_dropped": ("relu2_post", lambda orig: (lambda pre: ref.bf16_bits_from_f32(np.maximum(ref.f32(pre), np.float32(0)))),
                       ["test_relu2_invariants", "test_worked_example_golden"]),
    "margin_dropped": ("scale_update", lambda orig: (lambda st, A: orig(dict(st, margin=np.float32(1.0)), A) | {"margin": st["margin"]}),
                       ["test_scale_exact_values"]),
    "scale_inv_not_reciprocal": ("scale_update", lambda orig: (lambda st, A: (lambda o: o | {"scale_inv": o["scale"]})(orig(st, A))),
                                 ["test_scale_exact_values", "test_worked_example_golden", "test_scale_keeps_previous_on_degenerate_amax"]),
    "w2_cache_not_transposed": ("w2_cache", lambda orig: (lambda W2: (lambda r: (r[0].T.copy(), r[1], r[2]))(orig(W2))),
                                ["test_w2_cache_matches_library", "test_worked_example_golden"]),
    "dpre_factor_two_dropped": ("bwd_dpre", lambda orig: (lambda post, dOut, W2: ref.bf16_bits_from_f32(ref.f32(np.sqrt(ref.bf16_to_f64(post)) * (ref.bf16_to_f64(dOut) @ ref.bf16_to_f64(W2).T)))),
                                ["test_backward_vs_torch_autograd"]),
    "dpre_uses_post_not_sqrt": ("bwd_dpre", lambda orig: (lambda post, dOut, W2: ref.bf16_bits_from_f32(ref.f32(2 * ref.bf16_to_f64(post) * (ref.bf16_to_f64(dOut) @ ref.bf16_to_f64(W2).T)))),
                                ["test_backward_vs_torch_autograd"]),
    "dw2_scaled": ("bwd_dw2", lambda orig: (lambda post, dOut: ref.f32(ref.bf16_to_f64(post).T @ (ref.bf16_to_f64(dOut) * 0.5))),
                   ["test_backward_vs_torch_autograd", "test_backward_gemms_bruteforce"]),
    "dx_wrong_operand": ("bwd_dx", lambda orig: (lambda dPre, W1: ref.bf16_bits_from_f32(ref.f32(ref.bf16_to_f64(dPre) @ ref.bf16_to_f64(W1)[::-1]))),
                         ["test_backward_gemms_bruteforce"]),
    "rmsnorm_bwd_sign": ("rmsnorm_bwd", lambda orig: (lambda r, dx: -orig(r, dx)),
                         ["test_rmsnorm_constant_rows_and_autograd"]),
    "amax_drops_last_block": ("partial_amax", lambda orig: (lambda post, rows, cols: orig(post, rows, cols)[:-1]),
                              ["test_amax_partials_equal_brute_max"]),
    "ce_softcap_derivative_dropped": ("ce_backward_dlogits",
                                      lambda orig: (lambda y, tg, w, c, lse, g: orig(y, tg, w, c, lse, g) / (1.0 - np.tanh(np.asarray(y) / c) ** 2)),
                                      ["test_ce_bruteforce_with_ignored_targets", "test_ce_softcapped_vs_torch_autograd",
                                       "test_ce_closed_form_at_exact_tanh_points"]),
    "ce_onehot_dropped": ("ce_backward_dlogits", lambda orig: _ce_grad_no_onehot,
                          ["test_ce_zero_logits_closed_form", "test_ce_softcapped_vs_torch_autograd"]),
    "ce_target_reads_raw_logit": ("ce_forward", lambda orig: _ce_fwd_raw_target,
                                  ["test_ce_bruteforce_with_ignored_targets", "test_ce_softcapped_vs_torch_autograd"]),
    "ce_weights_ignored": ("ce_forward", lambda orig: (lambda y, tg, w, c: orig(y, tg, np.ones(np.shape(tg)[1]), c)),
                           ["test_ce_bruteforce_with_ignored_targets", "test_ce_multi_target_is_sum_of_single_targets"]),
    "ce_out_of_range_target_clipped": ("_ce_targets", lambda orig: _ce_targets_clipped,
                                       ["test_ce_bruteforce_with_ignored_targets", "test_ce_zero_logits_closed_form"]),
    "stack_fp8up_x_dequant_dropped": ("stack_forward_fp8up",
                                      lambda orig: (lambda r0, ly, sc, xs: orig(r0, ly, sc, [(a, np.float32(1.0)) for a, _ in xs])),
                                      ["test_stack_fp8up_close_to_bf16_stack"]),
    "ce_fp8_scale_dropped": ("head_logits_fp8", lambda orig: (lambda xq, Wq, a, b: orig(xq, Wq, 1.0, 1.0)),
                             ["test_ce_head_logits_fp8_bruteforce_and_exact_grid"]),
    "quantise_x_scale_dropped": ("quantise_x", lambda orig: (lambda x, s: orig(x, 1.0)),
                                 ["test_quantise_x_matches_library_and_amax"]),
    "w1_cache_scales_swapped": ("w1_cache", lambda orig: (lambda W1: (lambda r: (r[0], r[2], r[1]))(orig(W1))),
                                ["test_w1_cache_matches_library"]),
    "up_proj_fp8_dequant_dropped": ("up_proj_fp8", lambda orig: (lambda xq, Wq, a, b: orig(xq, Wq, 1.0, 1.0)),
                                    ["test_up_proj_fp8_bruteforce_and_exact_grid"]),
    "linear_bwd_dw_transposed": ("linear_bwd", lambda orig: (lambda x, W, dY: (lambda r: (r[0], r[1].T.copy()))(orig(x, W, dY))),
                                 ["test_linear_fp8_and_bwd_bruteforce"]),
    "rmsnorm_eps_dropped": ("rmsnorm_fwd", lambda orig: _rmsnorm_no_eps,
                            ["test_rmsnorm_constant_rows_and_autograd"]),
    "residual_add_drops_out": ("residual_add", lambda orig: (lambda r, out: np.asarray(r).copy()),
                               ["test_residual_add_rounds_the_fp32_sum"]),
    "residual_add_truncates": ("residual_add", lambda orig: (lambda r, out: _trunc_bf16(ref.f32(ref.bf16_to_f64(r) + ref.bf16_to_f64(out)))),
                               ["test_residual_add_rounds_the_fp32_sum"]),
    "reduce_partials_skips_nan": ("reduce_partials", lambda orig: (lambda pa: np.float32(np.nanmax(pa)) if np.size(pa) else np.float32(0.0)),
                                  ["test_reduce_partials_nan_and_empty"]),
    # the sampled evaluators of the full-size GPU tests
    "forward_rows_takes_leading_rows": ("forward_rows",
                                        lambda orig: (lambda rows, *a: orig(np.arange(len(rows)), *a)),
                                        ["test_forward_rows_equal_whole_batch"]),
    "dx_rows_dout_not_sliced": ("dx_rows", lambda orig: _dx_rows_dout_prefix,
                                ["test_dx_rows_equal_whole_batch"]),
    "dpre_column_reads_w2_column": ("dpre_column",
                                    lambda orig: (lambda i, pc, dOut, W2: orig(i, pc, dOut, np.asarray(W2).T.copy())),
                                    ["test_post_and_dpre_columns_equal_whole_batch"]),
    "dpre_column_factor_two_dropped": ("dpre_column", lambda orig: _dpre_column_no_two,
                                       ["test_post_and_dpre_columns_equal_whole_batch"]),
    "post_column_off_by_one": ("post_column",
                               lambda orig: (lambda i, x, W1: orig((i + 1) % np.shape(W1)[0], x, W1)),
                               ["test_post_and_dpre_columns_equal_whole_batch"]),
    "dw_entries_dw2_from_dpre": ("dw_entries", lambda orig: _dw_entries_mut("dw2_dpre"),
                                 ["test_dw_entries_equal_whole_batch"]),
    "dw_entries_dw1_reads_dout": ("dw_entries", lambda orig: _dw_entries_mut("dw1_dout"),
                                  ["test_dw_entries_equal_whole_batch"]),
    "down_proj_bf16_w2_reversed": ("down_proj_bf16", lambda orig: (lambda post, W2: orig(post, np.asarray(W2)[::-1].copy())),
                                   ["test_down_proj_bf16_bruteforce"]),
}


def _dx_rows_dout_prefix(rows, x, W1, W2, dOut):
    post = ref.relu2_post(ref.up_proj(x[rows], W1))
    dPre = ref.bwd_dpre(post, dOut[:len(rows)], W2)
    return dPre, ref.bwd_dx(dPre, W1)


def _dpre_column_no_two(i, post_col, dOut, W2):
    dPost = ref.bf16_to_f64(dOut) @ ref.bf16_to_f64(W2[i])
    return ref.bf16_bits_from_f32(ref.f32(np.sqrt(ref.bf16_to_f64(post_col)) * dPost))


def _dw_entries_mut(kind):
    def f(pairs, x, W1, W2, dOut):
        X, G = ref.bf16_to_f64(x), ref.bf16_to_f64(dOut)
        o1, o2 = [], []
        for i, j in pairs:
            pc = ref.post_column(i, x, W1)
            dc = ref.dpre_column(i, pc, dOut, W2)
            o1.append(np.float32(ref.bf16_to_f64(dc) @ (G if kind == "dw1_dout" else X)[:, j]))
            o2.append(np.float32(ref.bf16_to_f64(dc if kind == "dw2_dpre" else pc) @ G[:, j]))
        return np.array(o1, np.float32), np.array(o2, np.float32)
    return f


def _rmsnorm_no_eps(r):
    R = ref.bf16_to_f64(r)
    rstd = 1.0 / np.sqrt(np.mean(R * R, axis=1))
    return ref.bf16_bits_from_f32(ref.f32(R * rstd[:, None])), ref.f32(rstd)


def _ce_grad_no_onehot(y, tg, w, c, lse, g):
    th = np.tanh(np.asarray(y) / c)
    _, we = ref._ce_targets(tg, w, np.shape(y)[1])
    return g * we.sum(axis=1)[:, None] * np.exp(c * th - np.asarray(lse)[:, None]) * (1.0 - th * th)


def _ce_fwd_raw_target(y, tg, w, c):
    y = np.asarray(y, np.float64)
    z = ref.softcap(y, c)
    zmax = z.max(axis=1)
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
    t, we = ref._ce_targets(tg, w, y.shape[1])
    row = (we * (lse[:, None] - np.take_along_axis(y, t, axis=1))).sum(axis=1)
    ws = float(we.sum())
    return dict(lse=lse, row_loss=row, loss_sum=float(row.sum()), weight_sum=ws, mean=float(row.sum()) / ws)


def _ce_targets_clipped(targets, weights, V):
    tg = np.clip(np.asarray(targets, np.int64), 0, V - 1)
    return tg, np.broadcast_to(np.asarray(weights, np.float64), tg.shape).copy()


PARAMS = {"test_e4m3_exhaustive_over_bf16": dict(s=3.7),
          "test_scale_update_closed_form": dict(A=3.0, margin=2.0),
          "test_scale_keeps_previous_on_degenerate_amax": dict(A=0.0),
          # the square case: a transposed operand has the right shape
          "test_forward_rows_equal_whole_batch": dict(M=130, d=96, h=96),
          "test_dx_rows_equal_whole_batch": dict(M=130, d=96, h=96),
          "test_post_and_dpre_columns_equal_whole_batch": dict(M=130, d=96, h=96),
          "test_dw_entries_equal_whole_batch": dict(M=130, d=96, h=96)}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, make, catchers = MUTATIONS[name]
    orig = getattr(ref, attr)
    monkeypatch.setattr(ref, "_orig_e4m3", ref.e4m3_bits_from_f32, raising=False)
    monkeypatch.setattr(ref, attr, make(orig))
    failed = []
    for pin in catchers:
        fn = getattr(pins, pin)
        try:
            fn(**PARAMS.get(pin, {}))
        except Exception:
            failed.append(pin)
    assert failed, f"mutation {name} passed the pins {catchers}"
