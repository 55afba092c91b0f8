"""Pins of the CPU oracle against things other than itself.

Each pin checks one oracle function against a library routine that computes
the same rounding, a closed form, a brute-force evaluation, an invariant the
method fixes, or the hand-derived worked example in tests/golden.  None of
them calls the CUDA library.
"""
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _rand_f32(n, seed):
    g = np.random.default_rng(seed)
    # wide exponent spread, both signs
    return (g.standard_normal(n) * np.exp2(g.integers(-30, 30, n))).astype(np.float32)


# ---------------------------------------------------------------------------
# BF16 rounding
# ---------------------------------------------------------------------------

def test_bf16_matches_torch_and_ml_dtypes():
    v = _rand_f32(1_000_000, 1)
    ours = ref.bf16_bits_from_f32(v)
    assert np.array_equal(ours, _bf16(v))
    assert np.array_equal(ours, v.astype(ml_dtypes.bfloat16).view(np.uint16))


def test_bf16_ties_to_even():
    hi = np.arange(0x3F80, 0x3F80 + 512, dtype=np.uint32)
    u = (hi << 16) | 0x8000                       # exactly halfway
    v = u.view(np.float32)
    ours = ref.bf16_bits_from_f32(v).astype(np.uint32)
    want = np.where(hi & 1, hi + 1, hi)           # to even
    assert np.array_equal(ours, want)
    assert np.array_equal(ours.astype(np.uint16), _bf16(v))


def test_bf16_specials():
    v = np.array([np.inf, -np.inf, 0.0, -0.0, np.finfo(np.float32).max,
                  1e-40, -1e-42, 3.3895314e38], np.float32)
    assert np.array_equal(ref.bf16_bits_from_f32(v), _bf16(v))
    n = ref.bf16_bits_from_f32(np.array([np.nan], np.float32))
    assert np.isnan(ref.bf16_to_f64(n)).all()


def test_bf16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        want = bits.view(ml_dtypes.bfloat16).astype(np.float64)
        got = ref.bf16_to_f64(bits)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


# ---------------------------------------------------------------------------
# e4m3
# ---------------------------------------------------------------------------

def _e4m3_lib(v32):
    c = np.clip(v32, -448.0, 448.0).astype(np.float32)
    a = c.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    b = torch.from_numpy(c).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(a, b)
    return a


@pytest.mark.parametrize("s", [1.0, 2.0 ** -3, 448.0 / 37.0, 3.7])
def test_e4m3_exhaustive_over_bf16(s):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = ref.bf16_to_f64(bits)
    v = v[np.isfinite(v)].astype(np.float32)
    with np.errstate(over="ignore"):
        prod = (v * np.float32(s)).astype(np.float32)
    prod = prod[np.isfinite(prod)]
    assert np.array_equal(ref.e4m3_bits_from_f32(prod), _e4m3_lib(prod))


def test_e4m3_random_fp32():
    v = _rand_f32(500_000, 2)
    v = np.clip(v, -1e4, 1e4).astype(np.float32)
    assert np.array_equal(ref.e4m3_bits_from_f32(v), _e4m3_lib(v))


def test_e4m3_hand_cases():
    cases = [
        (448.0, 0x7E),            # largest finite
        (464.0, 0x7E),            # halfway 448/480: even mantissa (448)
        (465.0, 0x7E),            # rounds to 480 -> saturates
        (1e6, 0x7E), (np.inf, 0x7E), (-np.inf, 0xFE), (-500.0, 0xFE),
        (2.0 ** -9, 0x01),        # smallest subnormal
        (2.0 ** -10, 0x00),       # halfway 0 / 2^-9 -> even (0)
        (3 * 2.0 ** -10, 0x02),   # halfway 2^-9 / 2^-8 -> even (2^-8)
        (2.0 ** -6, 0x08),        # smallest normal
        (1.0, 0x38), (1.0625, 0x38), (1.1875, 0x3A), (-1.0, 0xB8),
        (0.0, 0x00), (-0.0, 0x80),
    ]
    for v, code in cases:
        got = int(ref.e4m3_bits_from_f32(np.array([v], np.float32))[0])
        assert got == code, (v, hex(got), hex(code))
    assert int(ref.e4m3_bits_from_f32(np.array([np.nan], np.float32))[0]) == 0x7F


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    want = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = ref.e4m3_to_f64(codes)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x7E] == 448.0


# ---------------------------------------------------------------------------
# GEMMs: brute force on tiny, non-square shapes (a transposed operand fails)
# ---------------------------------------------------------------------------

def _brute(A, B):          # A [m,k] . B[n,k]^T
    m, k = A.shape
    n = B.shape[0]
    out = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            s = 0.0
            for t in range(k):
                s += float(A[i, t]) * float(B[j, t])
            out[i, j] = s
    return out


def test_up_proj_bruteforce():
    g = np.random.default_rng(3)
    x = _bf16(g.standard_normal((5, 4)))
    W1 = _bf16(g.standard_normal((8, 4)))
    got = ref.up_proj(x, W1)
    want = _brute(ref.bf16_to_f64(x), ref.bf16_to_f64(W1))
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)


def test_down_proj_fp8_bruteforce():
    g = np.random.default_rng(4)
    q = g.integers(0, 0x7E, (5, 8)).astype(np.uint8)
    Wq = g.integers(0, 0xFE, (4, 8)).astype(np.uint8)
    Wq[Wq == 0x7F] = 0x10
    si, swi = np.float32(1 / 3), np.float32(1 / 7)
    got = ref.bf16_to_f64(ref.down_proj_fp8(q, Wq, si, swi))
    acc = _brute(ref.e4m3_to_f64(q), ref.e4m3_to_f64(Wq))
    comb = float(np.float32(si * swi))
    want = acc * comb
    np.testing.assert_allclose(got, want, rtol=2 ** -8)


def test_backward_gemms_bruteforce():
    g = np.random.default_rng(5)
    M, d, h = 6, 4, 8
    x = _bf16(g.standard_normal((M, d)))
    W1 = _bf16(g.standard_normal((h, d)))
    dPre = _bf16(g.standard_normal((M, h)))
    post = _bf16(np.abs(g.standard_normal((M, h))))
    dOut = _bf16(g.standard_normal((M, d)))
    X, W, D = ref.bf16_to_f64(x), ref.bf16_to_f64(W1), ref.bf16_to_f64(dPre)
    P, G = ref.bf16_to_f64(post), ref.bf16_to_f64(dOut)
    np.testing.assert_allclose(ref.bf16_to_f64(ref.bwd_dx(dPre, W1)), _brute(D, W.T), rtol=2 ** -8)
    np.testing.assert_allclose(ref.bwd_dw1(dPre, x), _brute(D.T, X.T), rtol=1e-6)
    np.testing.assert_allclose(ref.bwd_dw2(post, dOut), _brute(P.T, G.T), rtol=1e-6)


# ---------------------------------------------------------------------------
# ReLU^2 and sqrt(post) invariants
# ---------------------------------------------------------------------------

def test_relu2_invariants():
    g = np.random.default_rng(6)
    pre = g.standard_normal((64, 512)) * np.exp2(g.integers(-12, 12, (64, 512)))
    post = ref.relu2_post(pre)
    P = ref.bf16_to_f64(post)
    assert (P >= 0).all()
    assert (P[pre <= 0] == 0).all()
    r = np.maximum(pre, 0)
    # BF16 keeps 8 significant bits (unit roundoff 2^-8): post = r^2 (1+delta),
    # |delta| <= 2^-8 + 2^-23 (two fp32 steps) => |sqrt(post) - r| <= (2^-9 + 2^-20) r
    assert (np.abs(np.sqrt(P) - r) <= (2.0 ** -9 + 2.0 ** -20) * r).all()
    # and the bound is tight: some element uses more than half of it
    assert (np.abs(np.sqrt(P) - r) > 2.0 ** -10 * r).any()
    # invariant: post == bf16(fp32 square) element-wise via a library cast
    r32 = np.maximum(pre.astype(np.float32), np.float32(0))
    assert np.array_equal(post, _bf16(r32 * r32))


def test_amax_partials_equal_brute_max():
    g = np.random.default_rng(7)
    pre = g.standard_normal((300, 200)) * 3
    post = ref.relu2_post(pre)
    A = ref.amax(post)
    assert A == np.float32(ref.bf16_to_f64(post).max())
    for rows, cols in [(32, 256), (128, 64), (7, 13), (300, 200), (1, 1)]:
        pa = ref.partial_amax(post, rows, cols)
        assert pa.shape == (-(-300 // rows), -(-200 // cols))
        assert ref.reduce_partials(pa) == A
    # RNE is monotone: max of rounded == rounded max of the fp32 squares
    r32 = np.maximum(pre.astype(np.float32), np.float32(0))
    sq = (r32 * r32).astype(np.float32)
    assert A == np.float32(ref.bf16_to_f64(_bf16(np.array([sq.max()])))[0])


def test_quantise_post_matches_library():
    g = np.random.default_rng(8)
    post = ref.relu2_post(g.standard_normal((128, 256)) * 2)
    for s in [1.0, 17.5, 448.0 / 9.0, 1000.0]:
        q = ref.quantise_post(post, s)
        v = (ref.bf16_to_f64(post).astype(np.float32) * np.float32(s)).astype(np.float32)
        assert np.array_equal(q, _e4m3_lib(v))


# ---------------------------------------------------------------------------
# Delayed scale: closed form with exact rational arithmetic
# ---------------------------------------------------------------------------

def _nearest_f32(fr):
    x = np.float32(float(fr))
    cands = [np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))]
    errs = [abs(Fraction(float(c)) - fr) for c in cands]
    best = min(errs)
    winners = [c for c, e in zip(cands, errs) if e == best]
    if len(winners) > 1:      # tie: even mantissa
        winners = [c for c in winners if (np.array(c).view(np.uint32) & 1) == 0]
    return np.float32(winners[0])


@pytest.mark.parametrize("A,margin", [(7.0, 2.0), (4.0, 2.0), (3.0, 2.0), (0.123, 1.5),
                                      (1e-30, 2.0), (2.0e4, 2.0), (5.5, 1.0)])
def test_scale_update_closed_form(A, margin):
    st = ref.scale_state_init(margin, 1.0)
    out = ref.scale_update(st, A)
    A32, m32 = np.float32(A), np.float32(margin)
    den = _nearest_f32(Fraction(float(A32)) * Fraction(float(m32)))
    s = _nearest_f32(Fraction(448) / Fraction(float(den)))
    assert out["scale"] == s
    assert out["scale_inv"] == _nearest_f32(Fraction(1) / Fraction(float(s)))
    assert out["step"] == 1 and out["flags"] == 0 and out["amax_prev"] == A32


def test_scale_exact_values():
    st = ref.scale_state_init(2.0, 1.0)
    assert ref.scale_update(st, 7.0)["scale"] == 32.0
    assert ref.scale_update(st, 4.0)["scale"] == 56.0
    assert ref.scale_update(st, 1.75)["scale"] == 128.0
    assert ref.scale_update(ref.scale_state_init(1.0, 1.0), 448.0)["scale"] == 1.0


@pytest.mark.parametrize("A", [0.0, np.nan, np.inf, -1.0])
def test_scale_keeps_previous_on_degenerate_amax(A):
    st = ref.scale_update(ref.scale_state_init(2.0, 1.0), 7.0)
    out = ref.scale_update(st, A)
    assert out["scale"] == st["scale"] and out["scale_inv"] == st["scale_inv"]
    assert out["flags"] & ref.FLAG_KEPT_SCALE and out["step"] == 2
    out2 = ref.scale_update(out, 4.0)
    assert out2["scale"] == 56.0 and not (out2["flags"] & ref.FLAG_KEPT_SCALE)


def test_scale_resume_mid_sequence():
    amaxes = [3.0, 5.25, 0.0, 17.0, 2.5]
    st = ref.scale_state_init(2.0, 1.0)
    seq = []
    for a in amaxes:
        st = ref.scale_update(st, a)
        seq.append(st)
    resumed = dict(seq[1])
    for a, want in zip(amaxes[2:], seq[2:]):
        resumed = ref.scale_update(resumed, a)
        assert resumed == want


def test_reduce_partials_nan_and_empty():
    assert np.isnan(ref.reduce_partials(np.array([1.0, np.nan], np.float32)))
    assert ref.reduce_partials(np.zeros(0, np.float32)) == 0.0


# ---------------------------------------------------------------------------
# W2 cache
# ---------------------------------------------------------------------------

def test_w2_cache_matches_library():
    g = np.random.default_rng(9)
    W2 = _bf16(g.standard_normal((96, 64)) / 10)
    q, s_w, s_wi = ref.w2_cache(W2)
    W = ref.bf16_to_f64(W2)
    assert q.shape == (64, 96)
    a = np.abs(W).max()
    assert s_w == _nearest_f32(Fraction(448) / Fraction(float(a)))
    assert s_wi == _nearest_f32(Fraction(1) / Fraction(float(s_w)))
    v = (W.T.astype(np.float32) * s_w).astype(np.float32)
    assert np.array_equal(q, _e4m3_lib(v))
    # the max-magnitude entry lands exactly on +-448
    assert np.abs(ref.e4m3_to_f64(q)).max() == 448.0


def test_w2_cache_zero_weights():
    q, s_w, s_wi = ref.w2_cache(np.zeros((16, 16), np.uint16))
    assert s_w == 1.0 and s_wi == 1.0 and not q.any()


# ---------------------------------------------------------------------------
# Backward: library autograd in fp64 and central finite differences
# ---------------------------------------------------------------------------

def _rel(a, b):
    return np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-300)


def test_backward_vs_torch_autograd():
    g = np.random.default_rng(10)
    M, d, h = 48, 32, 96
    x = _bf16(g.standard_normal((M, d)))
    W1 = _bf16(g.standard_normal((h, d)) / np.sqrt(d))
    W2 = _bf16(g.standard_normal((h, d)) / np.sqrt(h))
    dOut = _bf16(g.standard_normal((M, d)))
    post = ref.relu2_post(ref.up_proj(x, W1))
    b = ref.backward(x, W1, W2, post, dOut)
    X = torch.tensor(ref.bf16_to_f64(x), requires_grad=True)
    A = torch.tensor(ref.bf16_to_f64(W1), requires_grad=True)
    B = torch.tensor(ref.bf16_to_f64(W2), requires_grad=True)
    out = torch.relu(X @ A.T).pow(2) @ B
    out.backward(torch.tensor(ref.bf16_to_f64(dOut)))
    assert _rel(ref.bf16_to_f64(b["dX"]), X.grad.numpy()) < 1e-2
    assert _rel(b["dW1"], A.grad.numpy()) < 1e-2
    assert _rel(b["dW2"], B.grad.numpy()) < 1e-2
    assert _rel(ref.bf16_to_f64(b["dPre"]),
                (2 * torch.relu(X @ A.T) * (torch.tensor(ref.bf16_to_f64(dOut)) @ B.T)).detach().numpy()) < 1e-2


def test_backward_exact_integers_and_finite_differences():
    # integer operands keep every BF16 rounding exact, so the oracle's backward
    # must equal the finite-difference gradient of the plain fp64 function
    g = np.random.default_rng(11)
    M, d, h = 5, 4, 8
    while True:
        xf = g.integers(-2, 3, (M, d)).astype(np.float32) + 0.5
        W1f = g.integers(-1, 2, (h, d)).astype(np.float32)
        if np.all(np.abs(xf @ W1f.T) > 0.1):
            break
    W2f = g.integers(-1, 2, (h, d)).astype(np.float32)
    dOf = g.integers(-2, 3, (M, d)).astype(np.float32)
    x, W1, W2, dOut = _bf16(xf), _bf16(W1f), _bf16(W2f), _bf16(dOf)
    post = ref.relu2_post(ref.up_proj(x, W1))
    assert np.array_equal(ref.bf16_to_f64(post), np.maximum(xf @ W1f.T, 0) ** 2)
    b = ref.backward(x, W1, W2, post, dOut)

    def loss(X, A, B):
        return float(np.sum(dOf * (np.maximum(X @ A.T, 0) ** 2 @ B)))

    eps = 1e-6
    for name, arr, got in [("x", xf.astype(np.float64), ref.bf16_to_f64(b["dX"])),
                           ("W1", W1f.astype(np.float64), b["dW1"]),
                           ("W2", W2f.astype(np.float64), b["dW2"])]:
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            args = {"x": xf, "W1": W1f, "W2": W2f}
            ap, am = dict(args), dict(args)
            ap[name], am[name] = p, m
            fd[idx] = (loss(ap["x"], ap["W1"], ap["W2"]) - loss(am["x"], am["W1"], am["W2"])) / (2 * eps)
        np.testing.assert_allclose(got, fd, rtol=2 ** -8, atol=1e-5)


# ---------------------------------------------------------------------------
# RMSNorm of the layer stack
# ---------------------------------------------------------------------------

def test_rmsnorm_constant_rows_and_autograd():
    # a constant row c normalises to c / sqrt(c^2 + eps); at c ~ 1e-3 the
    # eps = 1e-6 term halves the mean square's reciprocal
    r = _bf16(np.array([[3.0] * 8, [-0.5] * 8, [1e-3] * 8], np.float32))
    x, _ = ref.rmsnorm_fwd(r)
    X = ref.bf16_to_f64(x)
    np.testing.assert_allclose(X[0], 3 / np.sqrt(9 + 1e-6), rtol=2 ** -8)
    np.testing.assert_allclose(X[1], -0.5 / np.sqrt(0.25 + 1e-6), rtol=2 ** -8)
    c = ref.bf16_to_f64(r)[2, 0]
    np.testing.assert_allclose(X[2], c / np.sqrt(c * c + 1e-6), rtol=2 ** -8)
    g = np.random.default_rng(12)
    r = _bf16(g.standard_normal((6, 16)))
    dx = _bf16(g.standard_normal((6, 16)))
    R = torch.tensor(ref.bf16_to_f64(r), requires_grad=True)
    y = R * torch.rsqrt(R.pow(2).mean(dim=1, keepdim=True) + 1e-6)
    y.backward(torch.tensor(ref.bf16_to_f64(dx)))
    np.testing.assert_allclose(ref.rmsnorm_bwd(r, dx), R.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_residual_add_rounds_the_fp32_sum():
    # BF16 has 7 stored mantissa bits: next to 1.0 a step is 2^-7
    r = _bf16(np.array([[1.0, 1.0, 1.0, -2.0]], np.float32))
    o = _bf16(np.array([[2.0 ** -9, 2.0 ** -8, 3 * 2.0 ** -8, 2.0 ** -7]], np.float32))
    got = ref.bf16_to_f64(ref.residual_add(r, o))[0]
    # below half a step: down; a tie: to even (1.0); 1.5 steps: the tie goes
    # to the even neighbour 1 + 2^-6; -2 + 2^-7 = -1.9921875 is representable
    assert list(got) == [1.0, 1.0, 1.0 + 2.0 ** -6, -2.0 + 2.0 ** -7]
    g = np.random.default_rng(14)
    a, b = _bf16(g.standard_normal((32, 40))), _bf16(g.standard_normal((32, 40)) * 0.01)
    want = (torch.tensor(ref.bf16_to_f64(a), dtype=torch.float32) + torch.tensor(ref.bf16_to_f64(b), dtype=torch.float32))
    want = want.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ref.residual_add(a, b), want)


def test_down_proj_bf16_bruteforce():
    g = np.random.default_rng(15)
    post = _bf16(np.abs(g.standard_normal((5, 12))))
    W2 = _bf16(g.standard_normal((12, 7)))
    got = ref.bf16_to_f64(ref.down_proj_bf16(post, W2))
    want = _brute(ref.bf16_to_f64(post), ref.bf16_to_f64(W2).T)
    np.testing.assert_allclose(got, want, rtol=2 ** -8)


# ---------------------------------------------------------------------------
# Hand-derived worked example (tests/golden/worked_example_2x2.json)
# ---------------------------------------------------------------------------

def test_worked_example_golden():
    G = json.load(open(os.path.join(GOLDEN, "worked_example_2x2.json")))
    x, W1, W2, dOut = (_bf16(np.array(G[k], np.float32)) for k in ("x", "W1", "W2", "dOut"))
    st = ref.scale_state_init(G["margin"], G["initial_scale"])
    # step 0: calibration
    post = ref.relu2_post(ref.up_proj(x, W1))
    assert np.array_equal(ref.bf16_to_f64(post), G["step0_calibration"]["post"])
    A0 = ref.reduce_partials(ref.partial_amax(post, 1, 1))
    assert A0 == G["step0_calibration"]["amax"]
    st = ref.scale_update(st, A0)
    assert st["scale"] == G["step0_calibration"]["scale_after"]
    # W2 cache
    W2q_t, s_w, s_wi = ref.w2_cache(W2)
    assert s_w == G["w2_cache"]["s_w"]
    assert np.array_equal(W2q_t, np.array(G["w2_cache"]["W2q_t"], np.uint8))
    # step 1
    f = ref.forward(x, W1, W2q_t, s_wi, st["scale"], st["scale_inv"])
    assert st["scale"] == G["step1"]["scale"]
    assert np.array_equal(f["q"], np.array(G["step1"]["q"], np.uint8))
    assert np.array_equal(ref.bf16_to_f64(f["out"]), G["step1"]["out"])
    assert f["amax"] == G["step1"]["amax"]
    st = ref.scale_update(st, f["amax"])
    assert st["scale"] == G["step1"]["scale_after"]
    b = ref.backward(x, W1, W2, f["post"], dOut)
    for k in ("dPre", "dX"):
        assert np.array_equal(ref.bf16_to_f64(b[k]), G["step1_backward"][k]), k
    for k in ("dW1", "dW2"):
        assert np.array_equal(b[k], np.array(G["step1_backward"][k], np.float32)), k
    # step 2: 2x input spike, delayed scale saturates
    x2 = _bf16(np.array(G["x"], np.float32) * G["step2_spike"]["x_factor"])
    f2 = ref.forward(x2, W1, W2q_t, s_wi, st["scale"], st["scale_inv"])
    assert np.array_equal(ref.bf16_to_f64(f2["post"]), G["step2_spike"]["post"])
    assert np.array_equal(f2["q"], np.array(G["step2_spike"]["q"], np.uint8))
    st = ref.scale_update(st, f2["amax"])
    assert st["scale"] == G["step2_spike"]["scale_after"]


# ---------------------------------------------------------------------------
# Layer stack: straight-through autograd in torch fp64
# ---------------------------------------------------------------------------

def test_stack_backward_vs_straight_through_autograd():
    g = np.random.default_rng(13)
    M, d, h, L = 24, 16, 64, 3
    r0 = _bf16(g.standard_normal((M, d)))
    layers = []
    for _ in range(L):
        W1 = _bf16(g.standard_normal((h, d)) / np.sqrt(d))
        W2 = _bf16(g.standard_normal((h, d)) / np.sqrt(h))
        W2q_t, s_w, s_wi = ref.w2_cache(W2)
        layers.append(dict(W1=W1, W2=W2, W2q_t=W2q_t, w2_scale_inv=s_wi))
    scales = [(np.float32(40.0), np.float32(1 / 40.0))] * L
    saved, rL = ref.stack_forward(r0, layers, scales)
    dtop = _bf16(g.standard_normal((M, d)))
    dr0, grads = ref.stack_backward(saved, layers, dtop)

    # torch: same forward values, gradient straight through the FP8 step
    R = torch.tensor(ref.bf16_to_f64(r0), requires_grad=True)
    Ws = [(torch.tensor(ref.bf16_to_f64(Ly["W1"]), requires_grad=True),
           torch.tensor(ref.bf16_to_f64(Ly["W2"]), requires_grad=True)) for Ly in layers]
    r = R
    for l, (A, B) in enumerate(Ws):
        x = r * torch.rsqrt(r.pow(2).mean(dim=1, keepdim=True) + 1e-6)
        y = torch.relu(x @ A.T).pow(2) @ B
        r_next = torch.tensor(ref.bf16_to_f64(saved[l + 1]["r"] if l + 1 < L else rL))
        r = r + y + (r_next - r - y).detach()     # value: the oracle's residual
    r.backward(torch.tensor(ref.bf16_to_f64(dtop)))
    assert _rel(ref.bf16_to_f64(dr0), R.grad.numpy()) < 2e-2
    for (dW1, dW2), (A, B) in zip(grads, Ws):
        assert _rel(dW1, A.grad.numpy()) < 2e-2
        assert _rel(dW2, B.grad.numpy()) < 2e-2


def test_synth_is_deterministic():
    from fp8_relu_mlp_b200 import synth
    a = synth.make_problem(64, 32, 128, seed=5)
    b = synth.make_problem(64, 32, 128, seed=5)
    c = synth.make_problem(64, 32, 128, seed=6)
    for k in a:
        assert np.array_equal(a[k], b[k])
    assert not np.array_equal(a["x"], c["x"])
    gx = synth.make_problem(64, 32, 128, seed=5, x_dist="grid", w_dist="grid")
    X = ref.bf16_to_f64(gx["x"])
    assert np.array_equal(X * 4, np.round(X * 4)) and np.abs(X).max() <= 2


# ---------------------------------------------------------------------------
# FP8 up-projection
# ---------------------------------------------------------------------------

def test_quantise_x_matches_library_and_amax():
    g = np.random.default_rng(21)
    x = _bf16(g.standard_normal((64, 48)) * 3)
    for s in [1.0, 37.25, 448.0 / 11.0]:
        q, a = ref.quantise_x(x, s)
        v = (ref.bf16_to_f64(x).astype(np.float32) * np.float32(s)).astype(np.float32)
        assert np.array_equal(q, _e4m3_lib(v))
        assert a == np.float32(np.abs(ref.bf16_to_f64(x)).max())
    # negative values keep their sign bit
    q, _ = ref.quantise_x(_bf16(np.array([[-1.0, 1.0]], np.float32)), 1.0)
    assert list(q[0]) == [0xB8, 0x38]


def test_w1_cache_matches_library():
    g = np.random.default_rng(22)
    W1 = _bf16(g.standard_normal((96, 64)) / 8)
    q, s, si = ref.w1_cache(W1)
    W = ref.bf16_to_f64(W1)
    assert q.shape == W1.shape
    assert s == _nearest_f32(Fraction(448) / Fraction(float(np.abs(W).max())))
    assert np.array_equal(q, _e4m3_lib((W.astype(np.float32) * s).astype(np.float32)))
    assert si == _nearest_f32(Fraction(1) / Fraction(float(s)))


def test_up_proj_fp8_bruteforce_and_exact_grid():
    g = np.random.default_rng(23)
    xq = g.integers(0, 256, (5, 8)).astype(np.uint8)
    Wq = g.integers(0, 256, (7, 8)).astype(np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x21
    Wq[(Wq & 0x7F) == 0x7F] = 0x22
    sxi, swi = np.float32(1 / 5), np.float32(1 / 9)
    got = ref.up_proj_fp8(xq, Wq, sxi, swi)
    want = _brute(ref.e4m3_to_f64(xq), ref.e4m3_to_f64(Wq)) * float(np.float32(sxi * swi))
    np.testing.assert_allclose(got, want, rtol=2e-7)
    # power-of-two scales on grid values: quantisation and dequantisation are
    # exact, so the FP8 up-projection equals the BF16 one
    x = _bf16(g.integers(-8, 9, (6, 16)) / 4.0)
    W1 = _bf16(g.integers(-16, 17, (10, 16)) / 256.0)
    xq2, _ = ref.quantise_x(x, 16.0)
    W1q = ref.e4m3_bits_from_f32((ref.bf16_to_f64(W1) * 1024.0).astype(np.float32))
    assert np.array_equal(ref.up_proj_fp8(xq2, W1q, 1 / 16.0, 1 / 1024.0), ref.up_proj(x, W1))


def test_linear_fp8_and_bwd_bruteforce():
    g = np.random.default_rng(31)
    xq = g.integers(0, 256, (5, 8)).astype(np.uint8)
    Wq = g.integers(0, 256, (6, 8)).astype(np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x30
    Wq[(Wq & 0x7F) == 0x7F] = 0x31
    y = ref.bf16_to_f64(ref.linear_fp8(xq, Wq, np.float32(1 / 3), np.float32(1 / 5)))
    want = _brute(ref.e4m3_to_f64(xq), ref.e4m3_to_f64(Wq)) * float(np.float32(np.float32(1 / 3) * np.float32(1 / 5)))
    np.testing.assert_allclose(y, want, rtol=2 ** -8)
    x = _bf16(g.standard_normal((7, 8)))
    W = _bf16(g.standard_normal((6, 8)))
    dY = _bf16(g.standard_normal((7, 6)))
    dX, dW = ref.linear_bwd(x, W, dY)
    X, Wm, G = ref.bf16_to_f64(x), ref.bf16_to_f64(W), ref.bf16_to_f64(dY)
    np.testing.assert_allclose(ref.bf16_to_f64(dX), _brute(G, Wm.T), rtol=2 ** -8)
    np.testing.assert_allclose(dW, _brute(G.T, X.T), rtol=1e-6)
    # torch autograd of the unquantised layer
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(Wm, requires_grad=True)
    (Xt @ Wt.T).backward(torch.tensor(G))
    assert _rel(ref.bf16_to_f64(dX), Xt.grad.numpy()) < 1e-2 and _rel(dW, Wt.grad.numpy()) < 1e-6


# ---------------------------------------------------------------------------
# Softcapped cross-entropy over the LM head
# ---------------------------------------------------------------------------

def _ce_brute(y, targets, weights, c):
    """Pure-Python loops over the math module: per-row loss and dL/dy of the
    summed loss."""
    import math
    loss, grad = [], []
    for m in range(len(y)):
        V = len(y[m])
        z = [c * math.tanh(y[m][v] / c) for v in range(V)]
        mx = max(z)
        s = 0.0
        for v in range(V):
            s += math.exp(z[v] - mx)
        lse = mx + math.log(s)
        row, wsum = 0.0, 0.0
        for t, tg in enumerate(targets[m]):
            if 0 <= tg < V:
                row += weights[t] * (lse - z[tg])
                wsum += weights[t]
        gr = []
        for v in range(V):
            dz = wsum * math.exp(z[v] - lse)
            for t, tg in enumerate(targets[m]):
                if tg == v:
                    dz -= weights[t]
            th = math.tanh(y[m][v] / c)
            gr.append(dz * (1.0 - th * th))
        loss.append(row)
        grad.append(gr)
    return loss, grad


def test_ce_bruteforce_with_ignored_targets():
    g = np.random.default_rng(41)
    y = g.standard_normal((3, 6)) * 8.0
    tg = np.array([[2, 5, -1], [0, 0, 3], [6, 1, 4]])  # -1 and 6 (= V) are ignored
    w = [1.0, 0.5, 0.25]
    c = 5.0
    f = ref.ce_forward(y, tg, w, c)
    loss, grad = _ce_brute(y.tolist(), tg.tolist(), w, c)
    np.testing.assert_allclose(f["row_loss"], loss, rtol=1e-12)
    assert f["weight_sum"] == 1.5 + 1.75 + 0.75
    np.testing.assert_allclose(f["mean"], sum(loss) / 4.0, rtol=1e-12)
    np.testing.assert_allclose(ref.ce_backward_dlogits(y, tg, w, c, f["lse"], 1.0), grad, rtol=1e-10, atol=1e-14)


def test_ce_uncapped_limit_matches_torch():
    # c -> infinity: z = y, and the loss is the library's cross-entropy
    g = np.random.default_rng(43)
    y = g.standard_normal((16, 50)) * 3.0
    tg = g.integers(0, 50, (16, 1))
    f = ref.ce_forward(y, tg, [1.0], 1e9)
    Y = torch.tensor(y)
    want = torch.nn.functional.cross_entropy(Y, torch.tensor(tg[:, 0]), reduction="none")
    np.testing.assert_allclose(f["row_loss"], want.numpy(), rtol=1e-12)
    np.testing.assert_allclose(f["lse"], torch.logsumexp(Y, 1).numpy(), rtol=1e-12)


def test_ce_softcapped_vs_torch_autograd():
    g = np.random.default_rng(47)
    M, V, c = 8, 40, 15.0
    y = g.standard_normal((M, V)) * 10.0
    tg = g.integers(0, V, (M, 3))
    tg[1, 2] = -1
    tg[5, 0] = -1
    w = [1.0, 0.5, 0.25]
    Y = torch.tensor(y, requires_grad=True)
    Z = c * torch.tanh(Y / c)
    Tg = torch.tensor(tg)
    loss_sum = sum(w[t] * torch.nn.functional.cross_entropy(Z, Tg[:, t], ignore_index=-1, reduction="sum")
                   for t in range(3))
    wsum = sum(w[t] * float((tg[:, t] >= 0).sum()) for t in range(3))
    (loss_sum / wsum).backward()
    f = ref.ce_forward(y, tg, w, c)
    np.testing.assert_allclose(f["loss_sum"], float(loss_sum.detach()), rtol=1e-12)
    np.testing.assert_allclose(f["mean"], float(loss_sum.detach()) / wsum, rtol=1e-12)
    gs = ref.ce_grad_scale(1.0, f["weight_sum"], mean=True)
    np.testing.assert_allclose(ref.ce_backward_dlogits(y, tg, w, c, f["lse"], gs), Y.grad.numpy(),
                               rtol=1e-9, atol=1e-15)


def test_ce_zero_logits_closed_form():
    # z = 0 everywhere: every valid target costs ln V; softmax is uniform and
    # tanh'(0) = 1, so dL/dy = 1/V - onehot
    M, V = 4, 37
    tg = np.array([[0], [36], [5], [-3]])
    f = ref.ce_forward(np.zeros((M, V)), tg, [1.0], 15.0)
    np.testing.assert_allclose(f["row_loss"], [np.log(V)] * 3 + [0.0], rtol=1e-15)
    dy = ref.ce_backward_dlogits(np.zeros((M, V)), tg, [1.0], 15.0, f["lse"], 1.0)
    want = np.full((M, V), 1.0 / V)
    want[3] = 0.0
    for m in range(3):
        want[m, tg[m, 0]] -= 1.0
    np.testing.assert_allclose(dy, want, rtol=1e-13, atol=1e-16)


def test_ce_multi_target_is_sum_of_single_targets():
    g = np.random.default_rng(53)
    y = g.standard_normal((6, 20)) * 20.0
    tg = g.integers(-2, 22, (6, 3))
    w = [1.0, 0.75, 0.5]
    f = ref.ce_forward(y, tg, w, 15.0)
    singles = [ref.ce_forward(y, tg[:, t:t + 1], [w[t]], 15.0) for t in range(3)]
    np.testing.assert_allclose(f["row_loss"], sum(s["row_loss"] for s in singles), rtol=1e-12)
    assert f["weight_sum"] == sum(s["weight_sum"] for s in singles)
    dy = ref.ce_backward_dlogits(y, tg, w, 15.0, f["lse"], 1.0)
    dys = sum(ref.ce_backward_dlogits(y, tg[:, t:t + 1], [w[t]], 15.0, f["lse"], 1.0) for t in range(3))
    np.testing.assert_allclose(dy, dys, rtol=1e-12, atol=1e-15)


def test_ce_head_logits_fp8_bruteforce_and_exact_grid():
    g = np.random.default_rng(59)
    xq = g.integers(0, 256, (5, 16)).astype(np.uint8)
    Wq = g.integers(0, 256, (9, 16)).astype(np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x25
    Wq[(Wq & 0x7F) == 0x7F] = 0x26
    sxi, swi = np.float32(1 / 7), np.float32(1 / 3)
    want = _brute(ref.e4m3_to_f64(xq), ref.e4m3_to_f64(Wq)) * float(np.float32(sxi * swi))
    np.testing.assert_allclose(ref.head_logits_fp8(xq, Wq, sxi, swi), want, rtol=2e-7)
    x = _bf16(g.integers(-8, 9, (6, 32)) / 4.0)
    W = _bf16(g.integers(-16, 17, (11, 32)) / 256.0)
    np.testing.assert_array_equal(ref.head_logits(x, W), _brute(ref.bf16_to_f64(x), ref.bf16_to_f64(W)))
    xq2, _ = ref.quantise_x(x, 16.0)
    Wq2 = ref.e4m3_bits_from_f32((ref.bf16_to_f64(W) * 1024.0).astype(np.float32))
    assert np.array_equal(ref.head_logits_fp8(xq2, Wq2, 1 / 16.0, 1 / 1024.0), ref.head_logits(x, W))


def test_ce_backward_through_head_vs_torch_autograd():
    g = np.random.default_rng(61)
    M, d, V, c = 12, 16, 48, 15.0
    x = _bf16(g.standard_normal((M, d)))
    W = _bf16(g.standard_normal((V, d)) * 2.0)
    tg = g.integers(0, V, (M, 1))
    y = ref.head_logits(x, W)
    f = ref.ce_forward(y, tg, [1.0], c)
    dl, dX, dW = ref.ce_backward(x, W, ref.ce_backward_dlogits(y, tg, [1.0], c, f["lse"], 1.0))
    Xt = torch.tensor(ref.bf16_to_f64(x), requires_grad=True)
    Wt = torch.tensor(ref.bf16_to_f64(W), requires_grad=True)
    torch.nn.functional.cross_entropy(c * torch.tanh((Xt @ Wt.T) / c), torch.tensor(tg[:, 0]),
                                      reduction="sum").backward()
    # dlogits is rounded to BF16 (relative error <= 2^-9 per element)
    assert _rel(ref.bf16_to_f64(dX), Xt.grad.numpy()) < 1e-2
    assert _rel(dW, Wt.grad.numpy()) < 1e-2


def test_stack_fp8up_close_to_bf16_stack():
    # the e4m3 up-projection perturbs each layer's pre by the e4m3 rounding
    # of x and W1 (round to nearest: relative error uniform within 2^-4, RMS
    # 2^-4/sqrt(3) per operand, so about 5% RMS on pre and twice that on
    # post = pre^2); the residual stream carries r as well, so the two
    # stacks stay within 10% of each other.  A missing or inverted
    # dequantising scale (a factor 8 to 56 here), a transposed operand or a
    # skipped layer would not
    g = np.random.default_rng(71)
    M, d, h, Lyr = 24, 32, 64, 3
    r0 = _bf16(g.standard_normal((M, d)) * 2.0)
    layers, scales, xs = [], [], []
    for l in range(Lyr):
        W1 = _bf16(g.standard_normal((h, d)) / np.sqrt(d))
        W2 = _bf16(g.standard_normal((h, d)) / np.sqrt(h))
        W2q_t, _, s_wi = ref.w2_cache(W2)
        W1q, _, s1i = ref.w1_cache(W1)
        layers.append(dict(W1=W1, W2=W2, W2q_t=W2q_t, w2_scale_inv=s_wi, W1q=W1q, w1_scale_inv=s1i))
        scales.append((np.float32(448.0 / 40), np.float32(40 / 448.0)))
        xs.append((np.float32(448.0 / 8), np.float32(8 / 448.0)))
    sv8, r8 = ref.stack_forward_fp8up(r0, layers, scales, xs)
    sv, r = ref.stack_forward(r0, layers, scales)
    for l in range(Lyr):
        d_out = ref.bf16_to_f64(sv8[l]["r"]) - ref.bf16_to_f64(sv[l]["r"])
        assert _rel(ref.bf16_to_f64(sv8[l]["post"]), ref.bf16_to_f64(sv[l]["post"])) < 0.2
        assert np.abs(d_out).max() <= 0.2 * np.abs(ref.bf16_to_f64(sv[l]["r"])).max()
        assert sv8[l]["x_amax"] == np.float32(np.abs(ref.bf16_to_f64(sv8[l]["x"])).max())
    assert _rel(ref.bf16_to_f64(r8), ref.bf16_to_f64(r)) < 0.1


def test_ce_closed_form_at_exact_tanh_points():
    # c = 2 and y = +-ln 3: tanh(ln(3)/2) = (3-1)/(3+1) = 1/2 exactly, so the
    # softcapped logits are z = [1, 0, -1] (and 0 for y = 0), and everything
    # downstream has a closed form:
    #   lse(row 0) = ln(e + 1 + 1/e) = ln(1 + 2 cosh 1),  lse(row 1) = ln 3
    #   losses with w = (1, 0.5), targets row 0 = (0, 2), row 1 = (1, ignored):
    #   row 0 = (lse0 - 1) + 0.5 (lse0 + 1),  row 1 = ln 3,  weight 2.5
    #   dL/dy = (W_m softmax(z) - sum_t w_t onehot) (1 - tanh^2), with
    #   1 - tanh^2 = 3/4 at +-ln 3 and 1 at 0; W_0 = 1.5, W_1 = 1
    import math
    ln3 = math.log(3.0)
    y = np.array([[ln3, 0.0, -ln3], [0.0, 0.0, 0.0]])
    tg = np.array([[0, 2], [1, -1]])
    w = [1.0, 0.5]
    np.testing.assert_allclose(ref.softcap(y, 2.0), [[1.0, 0.0, -1.0], [0.0, 0.0, 0.0]], atol=1e-15)
    f = ref.ce_forward(y, tg, w, 2.0)
    lse0 = math.log(1.0 + 2.0 * math.cosh(1.0))
    np.testing.assert_allclose(f["lse"], [lse0, ln3], rtol=1e-14)
    np.testing.assert_allclose(f["row_loss"], [(lse0 - 1.0) + 0.5 * (lse0 + 1.0), ln3], rtol=1e-14)
    assert f["weight_sum"] == 2.5
    np.testing.assert_allclose(f["mean"], ((lse0 - 1.0) + 0.5 * (lse0 + 1.0) + ln3) / 2.5, rtol=1e-14)
    e = math.e
    p0 = np.array([e, 1.0, 1.0 / e]) / (e + 1.0 + 1.0 / e)
    want = np.array([[(1.5 * p0[0] - 1.0) * 0.75, 1.5 * p0[1], (1.5 * p0[2] - 0.5) * 0.75],
                     [1 / 3, 1 / 3 - 1.0, 1 / 3]])
    np.testing.assert_allclose(ref.ce_backward_dlogits(y, tg, w, 2.0, f["lse"], 1.0), want, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------------------
# Sampled evaluators.  The full-size GPU tests take their expected values from
# forward_rows, dx_rows, post_column, dpre_column and dw_entries, which
# evaluate the block's definitions at chosen rows, columns or entries.  Here
# they are held, bit for bit, to the whole-batch functions above (forward,
# backward, relu2_post of up_proj), which the pins in this file tie to
# libraries, brute force and closed forms.  A square case (d == h) makes a
# transposed operand shape-compatible, so only the values can catch it.
# ---------------------------------------------------------------------------

SAMPLED_SHAPES = [(300, 64, 256), (130, 96, 96)]


def _whole_batch(M, d, h, seed):
    from fp8_relu_mlp_b200 import synth
    P = synth.make_problem(M, d, h, seed=seed)
    W2q, _, s_wi = ref.w2_cache(P["W2"])
    post = ref.relu2_post(ref.up_proj(P["x"], P["W1"]))
    st = ref.scale_update(ref.scale_state_init(2.0, 1.0), ref.amax(post))
    f = ref.forward(P["x"], P["W1"], W2q, s_wi, st["scale"], st["scale_inv"])
    b = ref.backward(P["x"], P["W1"], P["W2"], f["post"], P["dOut"])
    return P, W2q, s_wi, st, f, b


def _rows(M):
    # unsorted, with both ends and a repeat-free middle
    return np.array([M - 1, 0, 7, M // 2, 3, M - 2])


@pytest.mark.parametrize("M,d,h", SAMPLED_SHAPES)
def test_forward_rows_equal_whole_batch(M, d, h):
    P, W2q, s_wi, st, f, _ = _whole_batch(M, d, h, seed=31)
    rows = _rows(M)
    fr = ref.forward_rows(rows, P["x"], P["W1"], W2q, s_wi, st["scale"], st["scale_inv"])
    for k in ("post", "q", "out"):
        assert np.array_equal(fr[k], f[k][rows]), k


@pytest.mark.parametrize("M,d,h", SAMPLED_SHAPES)
def test_dx_rows_equal_whole_batch(M, d, h):
    P, _, _, _, f, b = _whole_batch(M, d, h, seed=32)
    rows = _rows(M)
    dPre, dX = ref.dx_rows(rows, P["x"], P["W1"], P["W2"], P["dOut"])
    assert np.array_equal(dPre, b["dPre"][rows])
    assert np.array_equal(dX, b["dX"][rows])


@pytest.mark.parametrize("M,d,h", SAMPLED_SHAPES)
def test_post_and_dpre_columns_equal_whole_batch(M, d, h):
    P, _, _, _, f, b = _whole_batch(M, d, h, seed=33)
    for i in (0, 5, h // 2, h - 1):
        pc = ref.post_column(i, P["x"], P["W1"])
        assert np.array_equal(pc, f["post"][:, i]), i
        assert np.array_equal(ref.dpre_column(i, pc, P["dOut"], P["W2"]), b["dPre"][:, i]), i


@pytest.mark.parametrize("M,d,h", SAMPLED_SHAPES)
def test_dw_entries_equal_whole_batch(M, d, h):
    P, _, _, _, _, b = _whole_batch(M, d, h, seed=34)
    pairs = [(0, 0), (h - 1, d - 1), (5, d - 1), (h // 2, 3), (h - 1, 0), (7, 11)]
    w1, w2 = ref.dw_entries(pairs, P["x"], P["W1"], P["W2"], P["dOut"])
    assert np.array_equal(w1, np.array([b["dW1"][i, j] for i, j in pairs]))
    assert np.array_equal(w2, np.array([b["dW2"][i, j] for i, j in pairs]))
