"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact where the result is unique: post, the FP8 codes, the partial amax,
the scale sequence, the W2 cache.  For those the up-projection inputs are
drawn on a grid (small integers times powers of two) so that the fp32
accumulation is exact in any order.  Within the stated tolerances elsewhere:
relative Frobenius error <= 2e-2 for the FP8 forward output, <= 1e-2 for
the BF16 gradients.  Every output buffer is surrounded by canaries.
"""
import numpy as np
import pytest
import torch

from fp8_relu_mlp_b200 import _abi as A
from fp8_relu_mlp_b200 import synth
from oracle import ref
from tests.gpu_util import (Guarded, bf16_ulps, dev_bf16, dev_f32, dev_u8, host_bits, rel_fro,
                            stack_errors_given_layer_inputs)

pytestmark = pytest.mark.gpu

TOL_OUT = 2e-2
TOL_GRAD = 1e-2

SHAPES = [  # (M, d, h): several tiles, ragged tails in every dimension
    (256, 64, 256),
    (300, 80, 272),
    (1, 64, 256),
    (129, 128, 512),
    (1000, 768, 3072),
    (17, 16, 16),     # the smallest d and h: K and N inside one partial block
    (260, 48, 144),   # K under one k-block, N ending inside a 32-column chunk
    (1700, 64, 2800),  # 77 tiles on 74 CTA pairs: the last 3 run as half-width units
]


def _state(margin=2.0, s0=1.0):
    st = torch.zeros(8, dtype=torch.float32, device="cuda")
    A.fp8mlp_scale_state_init(st, margin, s0)
    return st


def _read_state(st):
    s = st.cpu()
    i = s.view(torch.int32)
    return dict(amax_prev=np.float32(s[0]), scale=np.float32(s[1]), scale_inv=np.float32(s[2]),
                margin=np.float32(s[3]), step=int(i[4]), flags=int(i[5]))


def _pa_oracle(post, M, h):
    rb, cb, br, bc = A.fp8mlp_partial_amax_shape(M, h)
    pa = ref.partial_amax(post, br, bc)
    full = np.zeros((rb, cb), np.float32)
    full[:pa.shape[0], :pa.shape[1]] = pa
    return full


def _up(M, d, h, x, W1, st, flags=0, pre=False):
    post = Guarded((M, h), torch.bfloat16)
    q = Guarded((M, h), torch.uint8)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    pa = Guarded((rb, cb), torch.float32)
    pre_t = Guarded((M, h), torch.float32) if pre else None
    A.fp8mlp_up_proj_fused(M, d, h, x, W1, st, post.t, q.t, pa.t, pre_t.t if pre else None, flags)
    torch.cuda.synchronize()
    for g in (post, q, pa) + ((pre_t,) if pre else ()):
        assert g.intact(), "write outside an output buffer"
    return post, q, pa, pre_t


# ---------------------------------------------------------------------------
# K1: fused up-projection epilogue, bit-exact on grid inputs
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,d,h", SHAPES)
def test_up_proj_fused_bit_exact_grid(M, d, h):
    P = synth.make_problem(M, d, h, seed=M + d, x_dist="grid", w_dist="grid")
    s = np.float32(448.0 / 37.0)
    st = _state(2.0, float(s))
    post, q, pa, pre = _up(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), st, pre=True)
    pre_o = ref.up_proj(P["x"], P["W1"])
    # grid inputs: every partial sum is exact in fp32, so pre must match exactly
    assert np.array_equal(host_bits(pre.t), pre_o.astype(np.float32))
    post_o = ref.relu2_post(pre_o)
    assert np.array_equal(host_bits(post.t), post_o)
    assert np.array_equal(host_bits(q.t), ref.quantise_post(post_o, s))
    assert np.array_equal(host_bits(pa.t), _pa_oracle(post_o, M, h))


@pytest.mark.parametrize("flags", [A.FWD_CALIBRATE, A.FWD_EVAL_BF16])
def test_up_proj_without_fp8_copy(flags):
    M, d, h = 300, 64, 256
    P = synth.make_problem(M, d, h, seed=3, x_dist="grid", w_dist="grid")
    post = Guarded((M, h), torch.bfloat16)
    q = Guarded((M, h), torch.uint8, fill=7)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    pa = Guarded((rb, cb), torch.float32)
    A.fp8mlp_up_proj_fused(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), None, post.t, q.t, pa.t, None, flags)
    torch.cuda.synchronize()
    post_o = ref.relu2_post(ref.up_proj(P["x"], P["W1"]))
    assert np.array_equal(host_bits(post.t), post_o)
    assert (host_bits(q.t) == 7).all(), "the FP8 copy must not be written"
    assert np.array_equal(host_bits(pa.t), _pa_oracle(post_o, M, h))
    assert post.intact() and q.intact() and pa.intact()


def post_within_accumulation_bound(post_gpu, x, W1, rows=None):
    """post_gpu may differ from the oracle's post only through the fp32
    accumulation of pre: with |fl(pre) - pre| <= K 2^-24 sum_k |x_k w_k|
    (the usual recursive-summation bound), post = r^2 moves by at most
    2 r delta + delta^2, plus one BF16 rounding step on each side."""
    X = ref.bf16_to_f64(x if rows is None else x[rows])
    W = ref.bf16_to_f64(W1)
    pre = X @ W.T
    delta = X.shape[1] * 2.0 ** -24 * (np.abs(X) @ np.abs(W).T)
    r = np.maximum(pre, 0)
    post_o = ref.relu2_post(pre)
    g = ref.bf16_to_f64(post_gpu)
    o = ref.bf16_to_f64(post_o)
    bound = 2 * (r + delta) * delta + 2.0 ** -7 * np.maximum(g, o) + 1e-30
    ok = np.abs(g - o) <= bound
    return bool(ok.all()), float((post_gpu != post_o).mean())


def within_accumulation_bound(got, exact, absprod, K, bf16_out, extra=0.0):
    """Element by element: a result accumulated in fp32 over K products, in
    any order, lies within K 2^-24 sum_k |a_k b_k| of the exact sum (the
    recursive-summation bound); a BF16 output adds half a BF16 step (2^-8
    relative); `extra` covers a scaling applied after the sum."""
    g = np.asarray(got, np.float64)
    e = np.asarray(exact, np.float64)
    bound = K * 2.0 ** -24 * absprod * (1 + extra) + extra * np.abs(e) + 1e-30
    if bf16_out:
        bound = bound + 2.0 ** -8 * np.maximum(np.abs(g), np.abs(e))
    bad = np.abs(g - e) > bound
    return (not bad.any()), int(bad.sum())


def pre_within_accumulation_bound(pre_gpu, x, W1):
    """The kernel's fp32 pre against the exact product: within the
    recursive-summation bound K 2^-24 sum_k |x_k w_k| element by element."""
    X = ref.bf16_to_f64(x)
    W = ref.bf16_to_f64(W1)
    exact = X @ W.T
    bound = X.shape[1] * 2.0 ** -24 * (np.abs(X) @ np.abs(W).T) + 1e-30
    return bool((np.abs(np.asarray(pre_gpu, np.float64) - exact) <= bound).all())


@pytest.mark.parametrize("M,d,h,seed", [(256, 64, 256, 11), (1000, 768, 3072, 11), (16384, 768, 3072, 0)])
def test_up_proj_fused_normal_inputs(M, d, h, seed):
    """Normal inputs: the order of the fp32 accumulation makes pre unique only
    up to rounding, so the kernel exports its pre, which is held to the exact
    product within the accumulation bound.  Given that pre, post, the FP8
    codes and the partial amax must equal the oracle's bit for bit: the
    epilogue's fp32 square, its BF16 rounding and the e4m3 rounding on values
    that are not exact (grid inputs never produce those).  The scale
    saturates the top of the distribution.  At M=16384 the inputs are the
    benchmark's own (seed 0), in the kernel configuration it times."""
    P = synth.make_problem(M, d, h, seed=seed)
    s = np.float32(20.0)
    st = _state(2.0, float(s))
    post, q, pa, pre = _up(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), st, pre=True)
    pre_g = host_bits(pre.t)
    assert pre_within_accumulation_bound(pre_g, P["x"], P["W1"])
    pg = host_bits(post.t)
    assert np.array_equal(pg, ref.relu2_post(pre_g))
    qg = host_bits(q.t)
    assert np.array_equal(qg, ref.quantise_post(pg, s))
    assert np.array_equal(host_bits(pa.t), _pa_oracle(pg, M, h))
    # the square is not exact in fp32 here, and some codes saturate
    assert (pre_g.astype(np.float64) ** 2 != (pre_g * pre_g).astype(np.float64)).any()
    if M >= 1000:
        assert ((qg & 0x7F) == 0x7E).any()


# ---------------------------------------------------------------------------
# K3: amax reduction + delayed scale, bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [0, 1, 7, 1000, 6144, 65537])
def test_amax_reduce_update_scale_bit_exact(n):
    pa = synth.make_partials(n, seed=n, scale=37.0)
    st = _state(2.0, 1.0)
    o = ref.scale_state_init(2.0, 1.0)
    pa_d = dev_f32(pa) if n else torch.zeros(1, device="cuda")
    for _ in range(2):
        A.fp8mlp_amax_reduce_update_scale(pa_d, n, st)
        o = ref.scale_update(o, ref.reduce_partials(pa))
    g = _read_state(st)
    for k in ("amax_prev", "scale", "scale_inv", "margin"):
        assert g[k] == o[k], k
    assert g["step"] == o["step"] == 2 and g["flags"] == o["flags"]


def test_forward_of_zero_activations_keeps_the_scale():
    """x = 0: post, its FP8 copy, every partial amax and out are zero; the
    reduced amax is 0, so the update keeps the previous scale and sets the
    kept-scale flag (no device status: 0 is finite), as the oracle does."""
    M, d, h = 300, 128, 512
    P = synth.make_problem(M, d, h, seed=9)
    x = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    W2q_o, _, s_wi = ref.w2_cache(P["W2"])
    st = _state(2.0, 37.0)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    post = Guarded((M, h), torch.bfloat16, fill=1.0)
    q = Guarded((M, h), torch.uint8, fill=7)
    pa = Guarded((rb, cb), torch.float32, fill=1.0)
    out = Guarded((M, d), torch.bfloat16, fill=1.0)
    A.fp8mlp_clear_device_status()
    A.fp8mlp_mlp_fwd(M, d, h, x, dev_bf16(P["W1"]), dev_u8(W2q_o), dev_f32(np.array([s_wi, 0, 0, 0], np.float32)),
                     None, st, post.t, q.t, pa.t, out.t, None, 0)
    A.fp8mlp_amax_reduce_update_scale(pa.t, A.fp8mlp_partial_amax_count(M, h), st)
    g = _read_state(st)
    assert A.fp8mlp_get_device_status() == 0
    assert not host_bits(post.t).any() and not host_bits(q.t).any() and not host_bits(pa.t).any()
    assert not host_bits(out.t).any()
    o = ref.scale_update(ref.scale_state_init(2.0, 37.0), ref.reduce_partials(host_bits(pa.t)))
    for k in ("amax_prev", "scale", "scale_inv"):
        assert g[k] == o[k], k
    assert g["flags"] == o["flags"] == ref.FLAG_KEPT_SCALE and g["step"] == o["step"] == 1
    for t in (post, q, pa, out):
        assert t.intact()


def test_scale_keeps_previous_on_nonfinite_amax():
    A.fp8mlp_clear_device_status()
    st = _state(1.5, 1.0)
    A.fp8mlp_amax_reduce_update_scale(dev_f32(np.array([3.0, 9.0], np.float32)), 2, st)
    before = _read_state(st)
    A.fp8mlp_amax_reduce_update_scale(dev_f32(np.array([3.0, np.nan], np.float32)), 2, st)
    after = _read_state(st)
    assert after["scale"] == before["scale"] and after["flags"] & A.STATE_KEPT_SCALE
    assert A.fp8mlp_get_device_status() & A.STATUS_NONFINITE_AMAX
    A.fp8mlp_amax_reduce_update_scale(dev_f32(np.zeros(4, np.float32)), 4, st)
    assert _read_state(st)["flags"] & A.STATE_KEPT_SCALE
    A.fp8mlp_clear_device_status()
    assert A.fp8mlp_get_device_status() == 0


def test_scale_state_checkpoint_resume():
    seq = [synth.make_partials(50, seed=i, scale=1.0 + i) for i in range(5)]
    st = _state(2.0, 1.0)
    saved = None
    for i, pa in enumerate(seq):
        A.fp8mlp_amax_reduce_update_scale(dev_f32(pa), 50, st)
        if i == 1:
            saved = st.clone()
    final = st.clone()
    st2 = saved.clone()
    for pa in seq[2:]:
        A.fp8mlp_amax_reduce_update_scale(dev_f32(pa), 50, st2)
    assert torch.equal(st2, final)


# ---------------------------------------------------------------------------
# K4: transposed FP8 W2 cache, bit-exact on any input
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("h,d", [(256, 64), (272, 80), (3072, 768), (4096, 1024), (16, 16)])
def test_w2_cache_bit_exact(h, d):
    W2 = synth.make_problem(1, d, h, seed=h)["W2"]
    Wq = Guarded((d, h), torch.uint8)
    inv = Guarded((4,), torch.float32)
    ws = torch.empty(A.fp8mlp_workspace_size(0, d, h), dtype=torch.uint8, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh(h, d, dev_bf16(W2), Wq.t, inv.t, ws)
    torch.cuda.synchronize()
    q_o, s_w, s_wi = ref.w2_cache(W2)
    assert np.array_equal(host_bits(Wq.t), q_o)
    assert host_bits(inv.t)[0] == s_wi
    assert Wq.intact() and inv.intact()


def test_w2_cache_zero_weights_flagged():
    A.fp8mlp_clear_device_status()
    h, d = 64, 32
    Wq = torch.full((d, h), 9, dtype=torch.uint8, device="cuda")
    inv = torch.zeros(4, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh(h, d, torch.zeros(h, d, dtype=torch.bfloat16, device="cuda"), Wq, inv, ws)
    assert (Wq == 0).all() and float(inv[0]) == 1.0
    assert A.fp8mlp_get_device_status() & A.STATUS_W2_DEGENERATE
    A.fp8mlp_clear_device_status()


# ---------------------------------------------------------------------------
# K2: FP8 down-projection
# ---------------------------------------------------------------------------

def _rand_codes(g, shape):
    c = g.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x30   # no NaN codes
    return c


# more e4m3 down-projections: ragged M with an N ending a quarter into its
# second tile (320 = 256 + 64), K ending inside a partial k-block (1040 =
# 8 x 128 + 16) over several waves, and the benchmark's M = 16384 (2.59 waves)
EXTRA_DOWN_SHAPES = [(1000, 320, 512), (4100, 768, 1040), (16384, 768, 3072)]


@pytest.mark.parametrize("M,d,h", SHAPES + EXTRA_DOWN_SHAPES)
def test_down_proj_fp8(M, d, h):
    g = np.random.default_rng(M * 7 + h)
    q = _rand_codes(g, (M, h))
    Wq = _rand_codes(g, (d, h))
    sinv, swinv = np.float32(1 / 37.0), np.float32(1 / 150.0)
    st = _state(2.0, float(np.float32(1) / sinv))
    A.fp8mlp_amax_reduce_update_scale(torch.zeros(1, device="cuda"), 0, st)  # keeps scale; exercises the state
    s_now = _read_state(st)
    out = Guarded((M, d), torch.bfloat16)
    A.fp8mlp_down_proj_fp8(M, d, h, dev_u8(q), dev_u8(Wq), dev_f32(np.array([swinv, 0, 0, 0], np.float32)), st, out.t)
    torch.cuda.synchronize()
    want = ref.down_proj_fp8(q, Wq, s_now["scale_inv"], swinv)
    got = host_bits(out.t)
    # only the fp32 accumulation order and the final BF16 rounding differ
    assert rel_fro(ref.bf16_to_f64(got), ref.bf16_to_f64(want)) < 4e-3
    Q, Wd = ref.e4m3_to_f64(q), ref.e4m3_to_f64(Wq)
    comb = float(np.float32(np.float32(s_now["scale_inv"]) * swinv))
    ok, nbad = within_accumulation_bound(ref.bf16_to_f64(got), (Q @ Wd.T) * comb,
                                         (np.abs(Q) @ np.abs(Wd).T) * comb, h, True, extra=2.0 ** -23)
    assert ok, nbad
    assert out.intact()


@pytest.mark.parametrize("M,d,h", [(256, 64, 256), (300, 80, 272), (1000, 768, 3072)])
def test_down_proj_bf16_eval(M, d, h):
    P = synth.make_problem(M, d, h, seed=5)
    post = ref.relu2_post(ref.up_proj(P["x"], P["W1"]))
    out = Guarded((M, d), torch.bfloat16)
    A.fp8mlp_down_proj_bf16(M, d, h, dev_bf16(post), dev_bf16(P["W2"]), out.t)
    torch.cuda.synchronize()
    want = ref.down_proj_bf16(post, P["W2"])
    assert rel_fro(ref.bf16_to_f64(host_bits(out.t)), ref.bf16_to_f64(want)) < 4e-3
    assert out.intact()


# ---------------------------------------------------------------------------
# whole forward, FP8 path, vs the oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,d,h", SHAPES + EXTRA_DOWN_SHAPES[:1])
def test_mlp_fwd_fp8(M, d, h):
    P = synth.make_problem(M, d, h, seed=21)
    W2q_t, s_w, s_wi = ref.w2_cache(P["W2"])
    st = _state(2.0, 1.0)
    x, W1 = dev_bf16(P["x"]), dev_bf16(P["W1"])
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    post = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    pa = torch.empty(rb, cb, device="cuda")
    # step 0: calibration, then the first scale
    A.fp8mlp_mlp_fwd(M, d, h, x, W1, None, None, None, st, post, None, pa, None, None, A.FWD_CALIBRATE)
    A.fp8mlp_amax_reduce_update_scale(pa, pa.numel(), st)
    s1 = _read_state(st)
    q = torch.empty(M, h, dtype=torch.uint8, device="cuda")
    out = Guarded((M, d), torch.bfloat16)
    inv = dev_f32(np.array([s_wi, 0, 0, 0], np.float32))
    A.fp8mlp_mlp_fwd(M, d, h, x, W1, dev_u8(W2q_t), inv, None, st, post, q, pa, out.t, None, 0)
    torch.cuda.synchronize()
    o_st = ref.scale_update(ref.scale_state_init(2.0, 1.0),
                            ref.amax(ref.relu2_post(ref.up_proj(P["x"], P["W1"]))))
    assert abs(float(s1["scale"]) / float(o_st["scale"]) - 1) < 1e-2
    f = ref.forward(P["x"], P["W1"], W2q_t, s_wi, s1["scale"], s1["scale_inv"])
    assert rel_fro(ref.bf16_to_f64(host_bits(out.t)), ref.bf16_to_f64(f["out"])) < TOL_OUT
    # and the FP8 forward stays close to the exact BF16 network
    exact = ref.bf16_to_f64(ref.down_proj_bf16(f["post"], P["W2"]))
    assert rel_fro(ref.bf16_to_f64(host_bits(out.t)), exact) < 6e-2
    assert out.intact()


# ---------------------------------------------------------------------------
# backward kernels
# ---------------------------------------------------------------------------

def _post_like(g, M, h):
    v = np.maximum(g.standard_normal((M, h)), 0).astype(np.float32) ** 2
    return synth.to_bf16_bits(v)


@pytest.mark.parametrize("M,d,h", SHAPES)
def test_bwd_dpre(M, d, h):
    P = synth.make_problem(M, d, h, seed=31)
    post = _post_like(np.random.default_rng(M), M, h)
    dPre = Guarded((M, h), torch.bfloat16)
    A.fp8mlp_bwd_dpre(M, d, h, dev_bf16(P["dOut"]), dev_bf16(P["W2"]), dev_bf16(post), dPre.t)
    torch.cuda.synchronize()
    want = ref.bwd_dpre(post, P["dOut"], P["W2"])
    got = host_bits(dPre.t)
    assert rel_fro(ref.bf16_to_f64(got), ref.bf16_to_f64(want)) < 4e-3
    # dPre = 2 sqrt(post) dPost: the accumulation bound of dPost times
    # 2 sqrt(post), plus the approximate square root (relative 2^-21 allowed)
    G, W2 = ref.bf16_to_f64(P["dOut"]), ref.bf16_to_f64(P["W2"])
    r2 = 2.0 * np.sqrt(ref.bf16_to_f64(post))
    ok, nbad = within_accumulation_bound(ref.bf16_to_f64(got), r2 * (G @ W2.T), r2 * (np.abs(G) @ np.abs(W2).T),
                                         d, True, extra=2.0 ** -21)
    assert ok, nbad
    # zero post gives exactly zero dPre (relu'(pre) = 0 there)
    assert (ref.bf16_to_f64(got)[ref.bf16_to_f64(post) == 0] == 0).all()
    assert dPre.intact()


@pytest.mark.parametrize("M,d,h", [(300, 80, 272), (1000, 768, 3072)])
def test_bwd_dpre_post_16_byte_aligned(M, d, h):
    """post, and then dPre too, at an address that is 16-byte but not 32-byte
    aligned (the boundary allows any 16-byte aligned pointer): the same bits
    as from aligned buffers holding the same values."""
    P = synth.make_problem(M, d, h, seed=33)
    post = _post_like(np.random.default_rng(M + 1), M, h)
    dOut, W2 = dev_bf16(P["dOut"]), dev_bf16(P["W2"])
    base = torch.zeros(M * h + 64, dtype=torch.bfloat16, device="cuda")
    off = next(k for k in range(8, 64, 8) if (base.data_ptr() + 2 * k) % 32 == 16)
    post_u = base[off:off + M * h].view(M, h)
    post_u.copy_(dev_bf16(post))
    assert post_u.data_ptr() % 32 == 16
    got_u = Guarded((M, h), torch.bfloat16)
    got_a = Guarded((M, h), torch.bfloat16)
    A.fp8mlp_bwd_dpre(M, d, h, dOut, W2, post_u, got_u.t)
    A.fp8mlp_bwd_dpre(M, d, h, dOut, W2, dev_bf16(post), got_a.t)
    # and dPre itself at such an address, the bytes around it untouched
    out_base = torch.full((M * h + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    off2 = next(k for k in range(8, 64, 8) if (out_base.data_ptr() + 2 * k) % 32 == 16)
    out_u = out_base[off2:off2 + M * h].view(M, h)
    assert out_u.data_ptr() % 32 == 16
    A.fp8mlp_bwd_dpre(M, d, h, dOut, W2, post_u, out_u)
    torch.cuda.synchronize()
    assert torch.equal(got_u.t, got_a.t)
    assert torch.equal(out_u, got_a.t)
    assert bool((out_base[:off2] == 7.0).all()) and bool((out_base[off2 + M * h:] == 7.0).all())
    want = ref.bwd_dpre(post, P["dOut"], P["W2"])
    assert rel_fro(ref.bf16_to_f64(host_bits(got_u.t)), ref.bf16_to_f64(want)) < 4e-3
    assert got_u.intact() and got_a.intact()


@pytest.mark.parametrize("M,d,h", SHAPES)
def test_bwd_dx(M, d, h):
    P = synth.make_problem(M, d, h, seed=41)
    g = np.random.default_rng(M + 1)
    dPre = synth.to_bf16_bits(g.standard_normal((M, h)).astype(np.float32))
    dX = Guarded((M, d), torch.bfloat16)
    A.fp8mlp_bwd_dx(M, d, h, dev_bf16(dPre), dev_bf16(P["W1"]), dX.t)
    torch.cuda.synchronize()
    want = ref.bwd_dx(dPre, P["W1"])
    assert rel_fro(ref.bf16_to_f64(host_bits(dX.t)), ref.bf16_to_f64(want)) < 4e-3
    D, W1 = ref.bf16_to_f64(dPre), ref.bf16_to_f64(P["W1"])
    ok, nbad = within_accumulation_bound(ref.bf16_to_f64(host_bits(dX.t)), D @ W1, np.abs(D) @ np.abs(W1), h, True)
    assert ok, nbad
    assert dX.intact()


@pytest.mark.parametrize("M,d,h", SHAPES)
def test_bwd_dw(M, d, h):
    P = synth.make_problem(M, d, h, seed=51)
    g = np.random.default_rng(M + 2)
    dPre = synth.to_bf16_bits(g.standard_normal((M, h)).astype(np.float32))
    post = _post_like(g, M, h)
    dW1, dW2 = Guarded((h, d), torch.float32), Guarded((h, d), torch.float32)
    A.fp8mlp_bwd_dw(M, d, h, dev_bf16(P["x"]), dev_bf16(dPre), dev_bf16(post), dev_bf16(P["dOut"]), dW1.t, dW2.t)
    torch.cuda.synchronize()
    assert rel_fro(host_bits(dW1.t), ref.bwd_dw1(dPre, P["x"])) < 1e-4
    assert rel_fro(host_bits(dW2.t), ref.bwd_dw2(post, P["dOut"])) < 1e-4
    D, X = ref.bf16_to_f64(dPre), ref.bf16_to_f64(P["x"])
    Pp, G = ref.bf16_to_f64(post), ref.bf16_to_f64(P["dOut"])
    ok1, n1 = within_accumulation_bound(host_bits(dW1.t), D.T @ X, np.abs(D).T @ np.abs(X), M, False)
    ok2, n2 = within_accumulation_bound(host_bits(dW2.t), Pp.T @ G, np.abs(Pp).T @ np.abs(G), M, False)
    assert ok1 and ok2, (n1, n2)
    assert dW1.intact() and dW2.intact()


@pytest.mark.parametrize("M,d,h", SHAPES)
def test_mlp_bwd_vs_oracle(M, d, h):
    P = synth.make_problem(M, d, h, seed=61)
    post = ref.relu2_post(ref.up_proj(P["x"], P["W1"]))
    dPre = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    dW1 = torch.empty(h, d, device="cuda")
    dW2 = torch.empty(h, d, device="cuda")
    A.fp8mlp_mlp_bwd(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), dev_bf16(P["W2"]), dev_bf16(post),
                     dev_bf16(P["dOut"]), dPre, dX, dW1, dW2)
    torch.cuda.synchronize()
    b = ref.backward(P["x"], P["W1"], P["W2"], post, P["dOut"])
    assert rel_fro(ref.bf16_to_f64(host_bits(dX)), ref.bf16_to_f64(b["dX"])) < TOL_GRAD
    assert rel_fro(host_bits(dW1), b["dW1"]) < TOL_GRAD
    assert rel_fro(host_bits(dW2), b["dW2"]) < TOL_GRAD


def test_bwd_dw_empty_batch_zeroes():
    h, d = 256, 64
    dW1 = torch.full((h, d), 3.0, device="cuda")
    dW2 = torch.full((h, d), 3.0, device="cuda")
    A.fp8mlp_bwd_dw(0, d, h, None, None, None, None, dW1, dW2)
    assert (dW1 == 0).all() and (dW2 == 0).all()


def test_empty_batch_every_entry_point():
    """M = 0 through every call that takes a batch: nothing is written, except
    the results an empty batch defines (zero weight gradients, zero
    cross-entropy totals)."""
    d, h, V, T = 64, 256, 512, 1

    def buf(nbytes, dtype=torch.uint8):  # a sentinel byte pattern
        return torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda").view(dtype)

    x, W1, W2, post, dOut, dPre, dX, out = (buf(8192, torch.bfloat16) for _ in range(8))
    q, W2q, W1q, xq = (buf(4096) for _ in range(4))
    pa, rstd, ramax, lse, rowl, ws = (buf(4096, torch.float32) for _ in range(6))
    inv = torch.ones(4, dtype=torch.float32, device="cuda")
    st, st_x = _state(), _state()
    tg = torch.zeros(16, dtype=torch.int32, device="cuda")
    untouched = [x, W1, W2, post, dOut, dPre, dX, out, q, W2q, W1q, xq, pa, rstd, ramax, lse, rowl, ws]
    before = [t.clone() for t in untouched]
    dW1 = torch.full((h * d,), 3.0, device="cuda")
    dW2 = torch.full((h * d,), 3.0, device="cuda")
    dW = torch.full((h * d,), 3.0, device="cuda")
    loss = torch.full((4,), 3.0, device="cuda")
    loss8 = torch.full((4,), 3.0, device="cuda")
    st_before = st.clone()

    A.fp8mlp_up_proj_fused(0, d, h, x, W1, st, post, q, pa)
    A.fp8mlp_up_proj_fused_fp8(0, d, h, xq, W1q, inv, st_x, st, post, q, pa)
    A.fp8mlp_down_proj_fp8(0, d, h, q, W2q, inv, st, out)
    A.fp8mlp_down_proj_bf16(0, d, h, post, W2, out)
    A.fp8mlp_mlp_fwd(0, d, h, x, W1, W2q, inv, W2, st, post, q, pa, out)
    A.fp8mlp_quantize_x(0, d, x, st_x, xq, pa)
    A.fp8mlp_linear_fwd_fp8(0, d, h, xq, W1q, inv, st_x, out)
    A.fp8mlp_linear_bwd(0, d, h, x, W1, dPre, dX, dW)
    A.fp8mlp_bwd_dpre(0, d, h, dOut, W2, post, dPre)
    A.fp8mlp_bwd_dx(0, d, h, dPre, W1, dX)
    A.fp8mlp_bwd_dw(0, d, h, x, dPre, post, dOut, dW1, dW2)
    A.fp8mlp_rmsnorm_fwd(0, d, x, out, rstd)
    A.fp8mlp_rmsnorm_fwd_quant(0, d, x, out, rstd, st_x, xq, ramax)
    A.fp8mlp_rmsnorm_bwd(0, d, x, rstd, dX, dOut, out)
    A.fp8mlp_residual_add(0, d, x, out, dPre)
    A.fp8mlp_ce_fwd(0, d, V, T, x, W1, tg, None, 15.0, lse, rowl, loss, ws)
    A.fp8mlp_ce_fwd_fp8(0, d, V, T, xq, st_x, W1q, inv, tg, None, 15.0, lse, rowl, loss8, ws)
    A.fp8mlp_ce_bwd_dlogits(0, d, V, T, x, W1, tg, None, 15.0, lse, loss, None, A.CE_MEAN, dPre)
    A.fp8mlp_ce_bwd_dlogits_fp8(0, d, V, T, xq, st_x, W1q, inv, tg, None, 15.0, lse, loss, None, A.CE_MEAN, dPre)
    torch.cuda.synchronize()
    for t, b in zip(untouched, before):
        assert torch.equal(t.view(torch.uint8), b.view(torch.uint8)), "a call with M = 0 wrote an output"
    assert torch.equal(st, st_before)
    assert (dW1 == 0).all() and (dW2 == 0).all() and (dW == 0).all()
    assert (loss[:3] == 0).all() and loss[3] == 3.0 and (loss8[:3] == 0).all()
    A.fp8mlp_mlp_bwd(0, d, h, x, W1, W2, post, dOut, dPre, dX, dW1.fill_(3.0), dW2.fill_(3.0))
    torch.cuda.synchronize()
    assert (dW1 == 0).all() and (dW2 == 0).all()
    assert A.fp8mlp_get_device_status() == 0


# ---------------------------------------------------------------------------
# delayed scaling over steps (the tiny workload), bit-exact on grid inputs
# ---------------------------------------------------------------------------

def _grid_perturb(W, seed):
    g = np.random.default_rng(seed)
    v = ref.bf16_to_f64(W) + g.integers(-2, 3, W.shape) / 256.0
    return synth.to_bf16_bits(np.clip(v, -0.25, 0.25).astype(np.float32))


def test_tiny_three_steps_bit_exact_grid():
    W = synth.WORKLOADS["tiny"]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0, x_dist="grid", w_dist="grid")
    W1, W2 = P["W1"], P["W2"]
    st = _state(W.margin, 1.0)
    o = ref.scale_state_init(W.margin, 1.0)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    x = dev_bf16(P["x"])
    post = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(M, h, dtype=torch.uint8, device="cuda")
    pa = torch.empty(rb, cb, device="cuda")
    out = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    Wq = torch.empty(d, h, dtype=torch.uint8, device="cuda")
    inv = torch.empty(4, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    # calibration step
    A.fp8mlp_mlp_fwd(M, d, h, x, dev_bf16(W1), None, None, None, st, post, None, pa, None, None, A.FWD_CALIBRATE)
    A.fp8mlp_amax_reduce_update_scale(pa, pa.numel(), st)
    o = ref.scale_update(o, ref.amax(ref.relu2_post(ref.up_proj(P["x"], W1))))
    for step in range(W.steps):
        A.fp8mlp_w2_fp8_cache_refresh(h, d, dev_bf16(W2), Wq, inv, ws)
        W2q_o, _, s_wi_o = ref.w2_cache(W2)
        A.fp8mlp_mlp_fwd(M, d, h, x, dev_bf16(W1), Wq, inv, None, st, post, q, pa, out, None, 0)
        A.fp8mlp_amax_reduce_update_scale(pa, pa.numel(), st)
        f = ref.forward(P["x"], W1, W2q_o, s_wi_o, o["scale"], o["scale_inv"])
        assert np.array_equal(host_bits(Wq), W2q_o)
        assert np.array_equal(host_bits(post), f["post"])
        assert np.array_equal(host_bits(q), f["q"])
        assert rel_fro(ref.bf16_to_f64(host_bits(out)), ref.bf16_to_f64(f["out"])) < 4e-3
        o = ref.scale_update(o, f["amax"])
        g = _read_state(st)
        assert g["scale"] == o["scale"] and g["scale_inv"] == o["scale_inv"] and g["amax_prev"] == o["amax_prev"]
        W1 = _grid_perturb(W1, 1000 * step)
        W2 = _grid_perturb(W2, 1000 * step + 1)


def test_tiny_three_steps_normal_perturbed():
    W = synth.WORKLOADS["tiny"]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0)
    W1, W2 = P["W1"], P["W2"]
    st = _state(W.margin, 1.0)
    o = ref.scale_state_init(W.margin, 1.0)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    x = dev_bf16(P["x"])
    post = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(M, h, dtype=torch.uint8, device="cuda")
    pa = torch.empty(rb, cb, device="cuda")
    out = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    Wq = torch.empty(d, h, dtype=torch.uint8, device="cuda")
    inv = torch.empty(4, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    A.fp8mlp_mlp_fwd(M, d, h, x, dev_bf16(W1), None, None, None, st, post, None, pa, None, None, A.FWD_CALIBRATE)
    A.fp8mlp_amax_reduce_update_scale(pa, pa.numel(), st)
    o = ref.scale_update(o, ref.amax(ref.relu2_post(ref.up_proj(P["x"], W1))))
    for step in range(W.steps):
        A.fp8mlp_w2_fp8_cache_refresh(h, d, dev_bf16(W2), Wq, inv, ws)
        W2q_o, _, s_wi_o = ref.w2_cache(W2)
        assert np.array_equal(host_bits(Wq), W2q_o)
        A.fp8mlp_mlp_fwd(M, d, h, x, dev_bf16(W1), Wq, inv, None, st, post, q, pa, out, None, 0)
        A.fp8mlp_amax_reduce_update_scale(pa, pa.numel(), st)
        f = ref.forward(P["x"], W1, W2q_o, s_wi_o, o["scale"], o["scale_inv"])
        assert rel_fro(ref.bf16_to_f64(host_bits(out)), ref.bf16_to_f64(f["out"])) < TOL_OUT
        o = ref.scale_update(o, f["amax"])
        g = _read_state(st)
        assert abs(float(g["scale"]) / float(o["scale"]) - 1) < 1e-2
        W1 = synth.perturb(W1, 0, step, W.perturb_var, "W1")
        W2 = synth.perturb(W2, 0, step, W.perturb_var, "W2")


_THREADS_SCRIPT = r"""
import threading, torch
from fp8_relu_mlp_b200 import _abi as A
M, d, h, n = 1000, 128, 512, 8
g = torch.Generator(device="cpu").manual_seed(7)
W1 = (torch.randn(h, d, generator=g) / d ** 0.5).bfloat16().cuda()
W2 = (torch.randn(h, d, generator=g) / h ** 0.5).bfloat16().cuda()
xs = [torch.randn(M, d, generator=g).bfloat16().cuda() for _ in range(n)]
rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
bufs = [dict(st=torch.zeros(8, device="cuda"), post=torch.empty(M, h, dtype=torch.bfloat16, device="cuda"),
             q=torch.empty(M, h, dtype=torch.uint8, device="cuda"), pa=torch.empty(rb, cb, device="cuda"),
             out=torch.empty(M, d, dtype=torch.bfloat16, device="cuda"), s=torch.cuda.Stream()) for _ in range(n)]
torch.cuda.synchronize()
go = threading.Barrier(n)
errs = []
def work(i):
    b = bufs[i]
    try:
        go.wait()   # every thread's first library call at once
        A.fp8mlp_scale_state_init(b["st"], 2.0, 4.0, stream=b["s"])
        A.fp8mlp_up_proj_fused(M, d, h, xs[i], W1, b["st"], b["post"], b["q"], b["pa"], stream=b["s"])
        A.fp8mlp_down_proj_bf16(M, d, h, b["post"], W2, b["out"], stream=b["s"])
    except Exception as e:
        errs.append(repr(e))
ts = [threading.Thread(target=work, args=(i,)) for i in range(n)]
[t.start() for t in ts]
[t.join() for t in ts]
torch.cuda.synchronize()
assert not errs, errs
for i in range(n):   # the same calls again, one at a time, must agree bit for bit
    b = bufs[i]
    post, q, out = b["post"].clone(), b["q"].clone(), b["out"].clone()
    A.fp8mlp_up_proj_fused(M, d, h, xs[i], W1, b["st"], b["post"], b["q"], b["pa"])
    A.fp8mlp_down_proj_bf16(M, d, h, b["post"], W2, b["out"])
    torch.cuda.synchronize()
    assert torch.equal(post.view(torch.int16), b["post"].view(torch.int16)), i
    assert torch.equal(q, b["q"]), i
    assert torch.equal(out.view(torch.int16), b["out"].view(torch.int16)), i
assert A.fp8mlp_get_device_status() == 0
print("ok")
"""


def test_first_calls_from_many_threads_at_once():
    """A fresh process whose first library calls come from 8 host threads at
    once, each on its own stream: the per-device set-up is done once and every
    thread's results equal the same calls made one at a time."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _THREADS_SCRIPT], cwd=root, capture_output=True, text=True,
                       timeout=300, env=dict(os.environ, PYTHONPATH=root))
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


# ---------------------------------------------------------------------------
# failure detection: a bounded wait runs out, the context stays usable
# ---------------------------------------------------------------------------

def test_bounded_wait_times_out_and_reports():
    M, d, h = 256, 64, 256
    P = synth.make_problem(M, d, h, seed=1, x_dist="grid", w_dist="grid")
    st = _state(2.0, 4.0)
    A.fp8mlp_clear_device_status()
    A.fp8mlp_set_wait_timeout_ns(50_000_000)
    A.fp8mlp_set_debug_flags(A.DEBUG_STALL_PRODUCER)
    try:
        post, q, pa, _ = _up(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), st)
        status = A.fp8mlp_get_device_status()
    finally:
        A.fp8mlp_set_debug_flags(0)
        A.fp8mlp_set_wait_timeout_ns(2_000_000_000)
    assert status & A.STATUS_TIMEOUT
    A.fp8mlp_clear_device_status()
    # the same call now runs normally and is correct
    post, q, pa, _ = _up(M, d, h, dev_bf16(P["x"]), dev_bf16(P["W1"]), st)
    assert A.fp8mlp_get_device_status() == 0
    assert np.array_equal(host_bits(post.t), ref.relu2_post(ref.up_proj(P["x"], P["W1"])))


def test_bounded_wait_of_the_dpre_post_ring_times_out_and_reports():
    """dPre's epilogue streams post through a ring of its own; with the hook
    that stops those loads its waits run out, then the MMA warp's wait for a
    free accumulator (256 tiles on 74 CTA pairs: every pair has more tiles
    than accumulators); the kernel returns with the timeout status and the
    next call on the context is correct."""
    M, d, h = 16384, 256, 1024
    P = synth.make_problem(M, d, h, seed=2)
    post_in = dev_bf16(ref.relu2_post(ref.up_proj(P["x"], P["W1"])))
    dOut, W2 = dev_bf16(P["dOut"]), dev_bf16(P["W2"])
    dPre = Guarded((M, h), torch.bfloat16)
    A.fp8mlp_clear_device_status()
    A.fp8mlp_set_wait_timeout_ns(50_000_000)
    A.fp8mlp_set_debug_flags(A.DEBUG_STALL_AUX)
    try:
        A.fp8mlp_bwd_dpre(M, d, h, dOut, W2, post_in, dPre.t)
        status = A.fp8mlp_get_device_status()
    finally:
        A.fp8mlp_set_debug_flags(0)
        A.fp8mlp_set_wait_timeout_ns(2_000_000_000)
    assert status & A.STATUS_TIMEOUT
    assert dPre.intact()
    A.fp8mlp_clear_device_status()
    A.fp8mlp_bwd_dpre(M, d, h, dOut, W2, post_in, dPre.t)
    assert A.fp8mlp_get_device_status() == 0
    assert dPre.intact()
    want = ref.bwd_dpre(host_bits(post_in), P["dOut"], P["W2"])
    assert rel_fro(ref.bf16_to_f64(host_bits(dPre.t)), ref.bf16_to_f64(want)) < 4e-3


# ---------------------------------------------------------------------------
# RMSNorm / residual helpers of the layer stack
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,d", [(1, 768), (300, 64), (4096, 768), (77, 1024)])
def test_rmsnorm_and_residual(M, d):
    g = np.random.default_rng(M + d)
    r = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32) * 3)
    dx = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    dr = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    o = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    x = Guarded((M, d), torch.bfloat16)
    rstd = Guarded((M,), torch.float32)
    A.fp8mlp_rmsnorm_fwd(M, d, dev_bf16(r), x.t, rstd.t)
    xo, rso = ref.rmsnorm_fwd(r)
    torch.cuda.synchronize()
    xg, xw = ref.bf16_to_f64(host_bits(x.t)), ref.bf16_to_f64(xo)
    assert (np.abs(xg - xw) <= 2.0 ** -7 * np.abs(xw) + 1e-30).all()   # at most one BF16 step
    np.testing.assert_allclose(host_bits(rstd.t), rso, rtol=1e-5)
    dro = Guarded((M, d), torch.bfloat16)
    A.fp8mlp_rmsnorm_bwd(M, d, dev_bf16(r), rstd.t, dev_bf16(dx), dev_bf16(dr), dro.t)
    want = ref.bf16_to_f64(dr) + ref.rmsnorm_bwd(r, dx)
    assert rel_fro(ref.bf16_to_f64(host_bits(dro.t)), want) < 4e-3
    rn = Guarded((M, d), torch.bfloat16)
    A.fp8mlp_residual_add(M, d, dev_bf16(r), dev_bf16(o), rn.t)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(rn.t), ref.residual_add(r, o))
    assert x.intact() and rstd.intact() and dro.intact() and rn.intact()


@pytest.mark.parametrize("M,d", [(300, 768), (1, 64), (1000, 1024)])
def test_rmsnorm_fwd_quant(M, d):
    g = np.random.default_rng(3 * M + d)
    r = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32) * 3)
    s_x = np.float32(448.0 / 9.0)
    st = _state(2.0, float(s_x))
    x, rstd = Guarded((M, d), torch.bfloat16), Guarded((M,), torch.float32)
    xq, ra = Guarded((M, d), torch.uint8), Guarded((M,), torch.float32)
    A.fp8mlp_rmsnorm_fwd_quant(M, d, dev_bf16(r), x.t, rstd.t, st, xq.t, ra.t)
    x2, rstd2 = torch.empty(M, d, dtype=torch.bfloat16, device="cuda"), torch.empty(M, device="cuda")
    A.fp8mlp_rmsnorm_fwd(M, d, dev_bf16(r), x2, rstd2)
    torch.cuda.synchronize()
    # x and rstd are those of the plain RMSNorm kernel
    assert torch.equal(x.t, x2) and torch.equal(rstd.t, rstd2)
    xg, qg = host_bits(x.t), host_bits(xq.t)
    xo, _ = ref.rmsnorm_fwd(r)
    qo, _ = ref.quantise_x(xo, s_x)
    same = xg == xo
    assert same.mean() > 0.9
    assert np.array_equal(qg[same], qo[same])
    # where the BF16 x is one step away from the oracle's, the code is at most
    # one e4m3 step away (rounding is monotone)
    signed = lambda c: (c & 0x7F).astype(np.int64) * np.where(c & 0x80, -1, 1)
    assert (np.abs(signed(qg[~same]) - signed(qo[~same])) <= 1).all()
    # the codes are RNE-satfinite e4m3 of the kernel's own x * s_x (torch's cast)
    want = (x.t.float() * float(s_x)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(xq.t, want)
    # per-row max |x| of the kernel's own x, exactly
    assert torch.equal(ra.t, x.t.float().abs().amax(dim=1))
    assert x.intact() and rstd.intact() and xq.intact() and ra.intact()


@pytest.mark.parametrize("L,M,d,h", [(3, 300, 128, 512), (2, 1024, 768, 3072)])
def test_stack_fp8_up_vs_oracle(L, M, d, h):
    from fp8_relu_mlp_b200.block import MLPBlock, MLPStack
    g = np.random.default_rng(L * 100 + M + 7)
    r0 = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    dtop = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    layers, scales, xsc = [], [], []
    S = MLPStack(L, M, d, h, fp8_up=True)
    for l in range(L):
        P = synth.make_problem(1, d, h, seed=600 + l)
        W2q_t, _, s_wi = ref.w2_cache(P["W2"])
        W1q, _, s1i = ref.w1_cache(P["W1"])
        layers.append(dict(W1=P["W1"], W2=P["W2"], W2q_t=W2q_t, w2_scale_inv=s_wi, W1q=W1q, w1_scale_inv=s1i))
        s = np.float32(30.0 + 5 * l)
        sx = np.float32(448.0 / (9.0 + l))
        scales.append((s, np.float32(np.float32(1) / s)))
        xsc.append((sx, np.float32(np.float32(1) / sx)))
        b = S.blocks[l]
        b.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], b.device))
        b.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], b.device))
        A.fp8mlp_scale_state_init(b.state, 2.0, float(s))
        A.fp8mlp_scale_state_init(b.state_x, 2.0, float(sx))
    S.refresh_w2_caches()
    S.r[0].copy_(MLPBlock.bits_to_bf16(r0, S.device))
    S.forward()
    S.dr.copy_(MLPBlock.bits_to_bf16(dtop, S.device))
    S.backward()
    torch.cuda.synchronize()
    for l in range(L):
        assert np.array_equal(host_bits(S.blocks[l].W1q), layers[l]["W1q"]), l
    saved, rL = ref.stack_forward_fp8up(r0, layers, scales, xsc)
    dr0, grads = ref.stack_backward(saved, layers, dtop)
    # each layer against the oracle given that layer's inputs: the FP8
    # forward's codes bit for bit, the gradients within 1e-2
    e = stack_errors_given_layer_inputs(S, layers, scales, dtop)
    assert e["q_mismatch"] == 0 and e["out"] < 4e-3, e
    assert e["dX"] < TOL_GRAD and e["dW1"] < TOL_GRAD and e["dW2"] < TOL_GRAD and e["dr0"] < TOL_GRAD, e
    # end to end against the oracle's own stack (two FP8 forwards whose codes
    # part where post differs by a rounding step): the FP8 forward's bound
    assert rel_fro(ref.bf16_to_f64(host_bits(S.r[L])), ref.bf16_to_f64(rL)) < TOL_OUT
    assert rel_fro(ref.bf16_to_f64(host_bits(S.dr)), ref.bf16_to_f64(dr0)) < TOL_OUT
    for l in range(L):
        assert rel_fro(host_bits(S.blocks[l].dW1), grads[l][0]) < TOL_OUT, l
        assert rel_fro(host_bits(S.blocks[l].dW2), grads[l][1]) < TOL_OUT, l
        # the x amax that drives the next x-scale: within one BF16 step
        ga = float(host_bits(S.row_amax[l]).max())
        assert abs(ga - float(saved[l]["x_amax"])) <= 2.0 ** -7 * float(saved[l]["x_amax"]), l
    S.update_scales()
    torch.cuda.synchronize()
    assert A.fp8mlp_get_device_status() == 0


# ---------------------------------------------------------------------------
# a CUDA-graph replay of the step gives the same bits as the eager calls
# ---------------------------------------------------------------------------

def test_graph_replay_matches_eager():
    from fp8_relu_mlp_b200.block import MLPBlock
    M, d, h = 1000, 768, 3072
    P = synth.make_problem(M, d, h, seed=77)

    def make():
        b = MLPBlock(M, d, h)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        b.calibrate()
        return b

    def step(b):
        b.forward()
        b.backward()
        b.update_scale()
        b.refresh_w2_cache()

    e = make()
    step(e)
    step(e)
    g = make()
    step(g)                      # eager first step, then capture the second
    graph = g.capture(lambda: step(g))
    # capture only records: the state is still after one step; replay runs step 2
    graph.replay()
    torch.cuda.synchronize()
    for k in ("post", "post_fp8", "out", "dPre", "dX", "dW1", "dW2", "W2q_t", "state", "partial_amax"):
        assert torch.equal(getattr(e, k), getattr(g, k)), k


@pytest.mark.parametrize("M,fp8_up", [(1000, False), (1000, True), (16384, False), (16384, True)])
def test_overlapped_step_matches_serial(M, fp8_up):
    # the scale update and the W2 cache refresh on a second stream beside the
    # GEMMs, dPre and dW launched to overlap the previous GEMM's last wave:
    # the same calls in a dependency-respecting order, so every output is
    # bit-identical to the serial step's, eagerly and replayed as a graph.
    # M = 16384 is the benchmark's step: there the N = 768 GEMMs run 2.59
    # waves of tiles, so dPre and dW really start inside their tails.
    from fp8_relu_mlp_b200.block import MLPBlock
    d, h = 768, 3072
    P = synth.make_problem(M, d, h, seed=78)

    def make():
        b = MLPBlock(M, d, h, fp8_up=fp8_up)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        if fp8_up:
            b.refresh_w1_cache()
        b.calibrate()
        return b

    def serial(b):
        if fp8_up:
            b.refresh_w1_cache()
        b.refresh_w2_cache()
        b.train_step()

    keys = ["post", "post_fp8", "out", "dPre", "dX", "dW1", "dW2", "W2q_t", "state", "partial_amax"]
    if fp8_up:
        keys += ["x_fp8", "W1q", "state_x"]
    side = torch.cuda.Stream()
    e, o, g = make(), make(), make()
    for _ in range(3):
        serial(e)
        o.train_step_overlapped(side)
    g.train_step_overlapped(side)
    graph = g.capture(lambda: g.train_step_overlapped(side))
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for k in keys:
        assert torch.equal(getattr(e, k), getattr(o, k)), k
        assert torch.equal(getattr(e, k), getattr(g, k)), k


@pytest.mark.parametrize("M,d,h", [(17, 16, 16), (300, 80, 272), (1000, 768, 3072), (16384, 768, 3072)])
def test_native_train_step_matches_serial(M, d, h):
    """fp8mlp_mlp_train_step (the library's own scheduled step: second
    stream, launch overlap) against refresh_w2_cache + train_step, bit for
    bit, three steps, eagerly and replayed as a CUDA graph; ragged shapes
    down to the smallest d and h."""
    from fp8_relu_mlp_b200.block import MLPBlock
    P = synth.make_problem(M, d, h, seed=81)

    def make():
        b = MLPBlock(M, d, h)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        b.calibrate()
        return b

    keys = ["post", "post_fp8", "out", "dPre", "dX", "dW1", "dW2", "W2q_t", "w2_scale_inv", "state", "partial_amax"]
    e, n, g = make(), make(), make()
    for _ in range(3):
        e.refresh_w2_cache()
        e.train_step()
        n.train_step_native()
    g.train_step_native()
    graph = g.capture(g.train_step_native)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for k in keys:
        assert torch.equal(getattr(e, k), getattr(n, k)), k
        assert torch.equal(getattr(e, k), getattr(g, k)), k
    assert A.fp8mlp_get_device_status() == 0


def test_native_train_step_empty_batch():
    from fp8_relu_mlp_b200.block import MLPBlock
    d, h = 128, 512
    P = synth.make_problem(1, d, h, seed=82)
    b = MLPBlock(0, d, h)
    for k in ("W1", "W2"):
        getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
    b.dW1.fill_(1.0)
    b.dW2.fill_(1.0)
    before = b.read_state()
    b.train_step_native()
    torch.cuda.synchronize()
    assert not b.dW1.any() and not b.dW2.any()
    W2q_o, _, s_wi = ref.w2_cache(P["W2"])
    assert np.array_equal(host_bits(b.W2q_t), W2q_o) and np.float32(b.w2_scale_inv[0].item()) == s_wi
    after = b.read_state()
    assert after["scale"] == before["scale"] and after["flags"] & ref.FLAG_KEPT_SCALE and after["step"] == 1


def test_host_pipeline_matches_in_place_steps():
    # inputs from pinned host memory and results back to it, with the copies
    # overlapped across two buffer sets: the same step sequence as stepping
    # the block in place, so the host copies of the last step's results, the
    # scale state and the weight gradients are bit-identical
    from fp8_relu_mlp_b200.block import MLPBlock
    from fp8_relu_mlp_b200.hostio import block_pipeline
    M, d, h = 1000, 768, 3072
    P = synth.make_problem(M, d, h, seed=79)

    def make():
        b = MLPBlock(M, d, h)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        b.calibrate()
        return b

    side = torch.cuda.Stream()
    ref_b, pipe_b = make(), make()
    pipe = block_pipeline(pipe_b, side)          # one warm-up step per buffer set
    host_in = [MLPBlock.bits_to_bf16(P[k], "cpu").pin_memory() for k in ("x", "dOut")]
    host_out = [torch.empty(M, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe.run(host_in, host_out, steps=5)
    for _ in range(2 + 5):
        ref_b.refresh_w2_cache()
        ref_b.train_step()
    torch.cuda.synchronize()
    assert torch.equal(host_out[0], ref_b.out.cpu())
    assert torch.equal(host_out[1], ref_b.dX.cpu())
    for k in ("state", "dW1", "dW2", "W2q_t", "partial_amax"):
        assert torch.equal(getattr(ref_b, k), getattr(pipe_b, k)), k


# ---------------------------------------------------------------------------
# layer stack: RMSNorm + block + residual, forward and backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,M,d,h", [(3, 300, 128, 512), (2, 1024, 768, 3072)])
def test_stack_vs_oracle(L, M, d, h):
    from fp8_relu_mlp_b200.block import MLPBlock, MLPStack
    g = np.random.default_rng(L * 100 + M)
    r0 = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    dtop = synth.to_bf16_bits(g.standard_normal((M, d)).astype(np.float32))
    layers, scales = [], []
    S = MLPStack(L, M, d, h)
    for l in range(L):
        P = synth.make_problem(1, d, h, seed=500 + l)
        W2q_t, s_w, s_wi = ref.w2_cache(P["W2"])
        layers.append(dict(W1=P["W1"], W2=P["W2"], W2q_t=W2q_t, w2_scale_inv=s_wi))
        s = np.float32(30.0 + 5 * l)
        scales.append((s, np.float32(np.float32(1) / s)))
        b = S.blocks[l]
        b.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], b.device))
        b.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], b.device))
        A.fp8mlp_scale_state_init(b.state, 2.0, float(s))
    S.refresh_w2_caches()
    S.r[0].copy_(MLPBlock.bits_to_bf16(r0, S.device))
    S.forward()
    S.dr.copy_(MLPBlock.bits_to_bf16(dtop, S.device))
    S.backward()
    torch.cuda.synchronize()
    saved, rL = ref.stack_forward(r0, layers, scales)
    dr0, grads = ref.stack_backward(saved, layers, dtop)
    # each layer against the oracle given that layer's inputs: the FP8
    # forward's codes bit for bit, the gradients within 1e-2
    e = stack_errors_given_layer_inputs(S, layers, scales, dtop)
    assert e["q_mismatch"] == 0 and e["out"] < 4e-3, e
    assert e["dX"] < TOL_GRAD and e["dW1"] < TOL_GRAD and e["dW2"] < TOL_GRAD and e["dr0"] < TOL_GRAD, e
    # end to end against the oracle's own stack (two FP8 forwards whose codes
    # part where post differs by a rounding step): the FP8 forward's bound
    assert rel_fro(ref.bf16_to_f64(host_bits(S.r[L])), ref.bf16_to_f64(rL)) < TOL_OUT
    assert rel_fro(ref.bf16_to_f64(host_bits(S.dr)), ref.bf16_to_f64(dr0)) < TOL_OUT
    for l in range(L):
        assert rel_fro(host_bits(S.blocks[l].dW1), grads[l][0]) < TOL_OUT, l
        assert rel_fro(host_bits(S.blocks[l].dW2), grads[l][1]) < TOL_OUT, l
    assert A.fp8mlp_get_device_status() == 0


# ---------------------------------------------------------------------------
# the data-parallel step on a one-rank NCCL group equals the plain step
# ---------------------------------------------------------------------------

def test_data_parallel_step_single_rank():
    import os
    import socket
    import torch.distributed as dist
    from fp8_relu_mlp_b200.block import MLPBlock
    from fp8_relu_mlp_b200.dp import DataParallelStep
    M, d, h = 1000, 768, 3072
    P = synth.make_problem(M, d, h, seed=91)

    def make():
        b = MLPBlock(M, d, h)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        b.calibrate()
        return b

    plain = make()
    plain.forward()
    plain.backward()
    plain.update_scale()
    plain.refresh_w2_cache()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        b = make()
        DataParallelStep(b)()
        bs = make()
        sharded = DataParallelStep(bs, shard_grads=True)
        sharded()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for k in ("post", "post_fp8", "out", "dPre", "dX", "dW1", "dW2", "state", "W2q_t"):
        assert torch.equal(getattr(plain, k), getattr(b, k)), k
    # one rank owns every row: the reduce-scattered shards are the whole gradients
    assert torch.equal(sharded.dW1_shard, plain.dW1) and torch.equal(sharded.dW2_shard, plain.dW2)


def test_token_sharding_on_two_blocks_reproduces_the_whole_batch():
    """The data-parallel partition on one GPU, without ranks that wait on one
    another: two blocks hold the two halves of the tokens and run the
    library's kernels in turn; the two exchanges of the data-parallel step
    are done between them with plain tensor ops (MAX over the two
    partial-amax tensors, SUM of the weight gradients).  Against the block
    that holds the whole batch: the delayed scale after calibration and after
    the step bit for bit, the rows of post, its FP8 copy, out, dPre and dX
    bit for bit (each output element's accumulation does not depend on which
    tile holds its row), and dW = dW(half 0) + dW(half 1) within the fp32
    rounding of the two partial sums and of their sum."""
    from fp8_relu_mlp_b200.block import MLPBlock
    M, d, h = 2048, 768, 3072
    half = M // 2
    P = synth.make_problem(M, d, h, seed=92)

    def make(rows):
        b = MLPBlock(len(range(*rows.indices(M))), d, h)
        for k in ("x", "W1", "W2", "dOut"):
            a = P[k][rows] if k in ("x", "dOut") else P[k]
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(a, b.device))
        b.refresh_w2_cache()
        return b

    def calibrate_shared(blocks):
        for b in blocks:
            A.fp8mlp_mlp_fwd(b.M, d, h, b.x, b.W1, None, None, None, b.state, b.post, None, b.partial_amax, None,
                             None, A.FWD_CALIBRATE)
        exchange_amax(blocks)

    def exchange_amax(blocks):
        m = blocks[0].partial_amax.clone()
        for b in blocks[1:]:
            m = torch.maximum(m, b.partial_amax)
        for b in blocks:
            b.partial_amax.copy_(m)
            b.update_scale()

    whole = make(slice(0, M))
    whole.calibrate()
    parts = [make(slice(0, half)), make(slice(half, M))]
    calibrate_shared(parts)
    torch.cuda.synchronize()
    for b in parts:
        assert torch.equal(b.state, whole.state)
    whole.forward()
    whole.backward()
    whole.update_scale()
    for b in parts:
        b.forward()
        b.backward()
    exchange_amax(parts)
    torch.cuda.synchronize()
    for b in parts:
        assert torch.equal(b.state, whole.state)
    for i, b in enumerate(parts):
        sl = slice(i * half, (i + 1) * half)
        for k in ("post", "post_fp8", "out", "dPre", "dX"):
            assert torch.equal(getattr(b, k), getattr(whole, k)[sl]), (i, k)
    # dW1 = dPre^T x and dW2 = post^T dOut from the kernels' own (identical)
    # dPre and post: the whole batch's fp32 accumulation and the sum of the
    # two halves' are each within the recursive-summation bound of the exact
    # product (the halves' sum adds one rounding, relative 2^-24)
    X, G = ref.bf16_to_f64(P["x"]), ref.bf16_to_f64(P["dOut"])
    for k, left in (("dW1", whole.dPre), ("dW2", whole.post)):
        L = ref.bf16_to_f64(host_bits(left))
        exact, absprod = L.T @ (X if k == "dW1" else G), np.abs(L).T @ np.abs(X if k == "dW1" else G)
        got = host_bits(getattr(parts[0], k) + getattr(parts[1], k))
        for val in (got, host_bits(getattr(whole, k))):
            ok, nbad = within_accumulation_bound(val, exact, absprod, M, False, extra=2.0 ** -23)
            assert ok, (k, nbad)
        assert rel_fro(got, host_bits(getattr(whole, k))) < 1e-5
    assert A.fp8mlp_get_device_status() == 0


# ---------------------------------------------------------------------------
# FP8 up-projection: x quantiser, W1 cache, e4m3 up-projection
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,d", [(1, 64), (300, 80), (16384, 768)])
def test_quantize_x_bit_exact(M, d):
    x = synth.make_problem(M, d, 16, seed=M, x_dist="student_t3" if M > 1000 else "normal")["x"]
    s = np.float32(448.0 / 29.0)
    st = _state(2.0, float(s))
    n = A.fp8mlp_x_partial_amax_count(M, d)
    xq = Guarded((M, d), torch.uint8)
    pa = Guarded((n,), torch.float32)
    A.fp8mlp_quantize_x(M, d, dev_bf16(x), st, xq.t, pa.t)
    torch.cuda.synchronize()
    q_o, a_o = ref.quantise_x(x, s)
    assert np.array_equal(host_bits(xq.t), q_o)
    flat = np.abs(ref.bf16_to_f64(x)).reshape(-1)
    want = [np.float32(flat[i * 8192:(i + 1) * 8192].max()) for i in range(n)]
    assert np.array_equal(host_bits(pa.t), np.array(want, np.float32))
    assert host_bits(pa.t).max() == a_o
    assert xq.intact() and pa.intact()


@pytest.mark.parametrize("h,d", [(256, 64), (272, 80), (3072, 768)])
def test_w1_cache_bit_exact(h, d):
    W1 = synth.make_problem(1, d, h, seed=h + 1)["W1"]
    Wq = Guarded((h, d), torch.uint8)
    inv = Guarded((4,), torch.float32)
    ws = torch.empty(A.fp8mlp_workspace_size(0, d, h), dtype=torch.uint8, device="cuda")
    A.fp8mlp_w1_fp8_cache_refresh(h, d, dev_bf16(W1), Wq.t, inv.t, ws)
    torch.cuda.synchronize()
    q_o, s_o, si_o = ref.w1_cache(W1)
    assert np.array_equal(host_bits(Wq.t), q_o)
    assert host_bits(inv.t)[0] == si_o
    assert Wq.intact() and inv.intact()


@pytest.mark.parametrize("M,d,h", SHAPES)
def test_up_proj_fp8_bit_exact_grid(M, d, h):
    # grid inputs with power-of-two scales: both quantisations and the fp32
    # accumulation are exact, so pre, post, the FP8 copy and the partial amax
    # are unique
    P = synth.make_problem(M, d, h, seed=M + 3, x_dist="grid", w_dist="grid")
    st_x = _state(2.0, 16.0)
    st = _state(2.0, float(np.float32(448.0 / 37.0)))
    xq_o, _ = ref.quantise_x(P["x"], 16.0)
    W1q_o = ref.e4m3_bits_from_f32((ref.bf16_to_f64(P["W1"]) * 1024.0).astype(np.float32))
    n = A.fp8mlp_x_partial_amax_count(M, d)
    xq = torch.empty(M, d, dtype=torch.uint8, device="cuda")
    pax = torch.empty(n, device="cuda")
    A.fp8mlp_quantize_x(M, d, dev_bf16(P["x"]), st_x, xq, pax)
    post = Guarded((M, h), torch.bfloat16)
    q = Guarded((M, h), torch.uint8)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    pa = Guarded((rb, cb), torch.float32)
    pre = Guarded((M, h), torch.float32)
    A.fp8mlp_up_proj_fused_fp8(M, d, h, xq, dev_u8(W1q_o), dev_f32(np.array([1 / 1024.0, 0, 0, 0], np.float32)),
                               st_x, st, post.t, q.t, pa.t, pre.t, 0)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(xq), xq_o)
    pre_o = ref.up_proj_fp8(xq_o, W1q_o, np.float32(1 / 16.0), np.float32(1 / 1024.0))
    assert np.array_equal(host_bits(pre.t), pre_o.astype(np.float32))
    assert np.array_equal(pre_o, ref.up_proj(P["x"], P["W1"]))   # exact: equals the BF16 up-projection
    post_o = ref.relu2_post(pre_o)
    assert np.array_equal(host_bits(post.t), post_o)
    assert np.array_equal(host_bits(q.t), ref.quantise_post(post_o, np.float32(448.0 / 37.0)))
    assert np.array_equal(host_bits(pa.t), _pa_oracle(post_o, M, h))
    assert post.intact() and q.intact() and pa.intact() and pre.intact()


@pytest.mark.parametrize("M,d,h", [(256, 64, 256), (1000, 768, 3072)])
def test_fp8_up_forward_normal_inputs(M, d, h):
    from fp8_relu_mlp_b200.block import MLPBlock
    P = synth.make_problem(M, d, h, seed=123)
    b = MLPBlock(M, d, h, fp8_up=True)
    for k in ("x", "W1", "W2"):
        getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
    b.refresh_w2_cache()
    b.refresh_w1_cache()
    b.calibrate()
    b.forward()
    torch.cuda.synchronize()
    sx = b.read_state(b.state_x)
    sp = b.read_state()
    # the oracle runs the same FP8 pipeline with the GPU's calibrated scales
    # taken from the oracle's own calibration on the same inputs
    xq_cal, ax = ref.quantise_x(P["x"], 1.0)
    st_x = ref.scale_update(ref.scale_state_init(2.0, 1.0), ax)
    assert np.float32(sx["scale"]) == st_x["scale"]          # amax of x is exact, so the x-scale is bit-exact
    W1q_o, _, s_w1i = ref.w1_cache(P["W1"])
    xq_o, _ = ref.quantise_x(P["x"], st_x["scale"])
    pre_o = ref.up_proj_fp8(xq_o, W1q_o, st_x["scale_inv"], s_w1i)
    st_p = ref.scale_update(ref.scale_state_init(2.0, 1.0), ref.amax(ref.relu2_post(pre_o)))
    assert abs(sp["scale"] / float(st_p["scale"]) - 1) <= 2.0 ** -7
    W2q_o, _, s_w2i = ref.w2_cache(P["W2"])
    A.fp8mlp_scale_state_init(b.state, 2.0, float(st_p["scale"]))
    b.forward()
    torch.cuda.synchronize()
    post_o = ref.relu2_post(pre_o)
    out_o = ref.down_proj_fp8(ref.quantise_post(post_o, st_p["scale"]), W2q_o, st_p["scale_inv"], s_w2i)
    assert rel_fro(ref.bf16_to_f64(host_bits(b.post)), ref.bf16_to_f64(post_o)) < 1e-2
    assert rel_fro(ref.bf16_to_f64(host_bits(b.out)), ref.bf16_to_f64(out_o)) < TOL_OUT
    # against the exact BF16 network: the FP8 up- and down-projection error
    exact = ref.bf16_to_f64(ref.down_proj_bf16(ref.relu2_post(ref.up_proj(P["x"], P["W1"])), P["W2"]))
    assert rel_fro(ref.bf16_to_f64(host_bits(b.out)), exact) < 8e-2


@pytest.mark.parametrize("M,d,h,seed", [(1000, 768, 3072, 124), (16384, 768, 3072, 0)])
def test_up_proj_fp8_normal_inputs_bit_exact_given_pre(M, d, h, seed):
    """The e4m3 up-projection on normal inputs.  The x codes and the W1 cache
    equal the oracle's bit for bit; the kernel's exported pre (the fp32
    accumulator times fp32(s_x^-1 s_w1^-1)) lies within the fp32 accumulation
    bound of the exact e4m3 product (itself exact in fp64) plus the rounding
    of the scaling; given that pre, post, the FP8 copy and the partial amax
    equal the oracle's bit for bit.  At M=16384 the inputs are the
    benchmark's own (seed 0)."""
    P = synth.make_problem(M, d, h, seed=seed)
    s_x = np.float32(448.0 / 10.0)
    st_x = _state(2.0, float(s_x))
    st = _state(2.0, 20.0)
    x, W1 = dev_bf16(P["x"]), dev_bf16(P["W1"])
    xq = Guarded((M, d), torch.uint8)
    pax = torch.zeros(max(1, A.fp8mlp_x_partial_amax_count(M, d)), device="cuda")
    A.fp8mlp_quantize_x(M, d, x, st_x, xq.t, pax)
    W1q = Guarded((h, d), torch.uint8)
    w1inv = torch.zeros(4, device="cuda")
    ws = torch.empty(A.fp8mlp_workspace_size(0, d, h), dtype=torch.uint8, device="cuda")
    A.fp8mlp_w1_fp8_cache_refresh(h, d, W1, W1q.t, w1inv, ws)
    post = Guarded((M, h), torch.bfloat16)
    q = Guarded((M, h), torch.uint8)
    rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
    pa = Guarded((rb, cb), torch.float32)
    pre = Guarded((M, h), torch.float32)
    A.fp8mlp_up_proj_fused_fp8(M, d, h, xq.t, W1q.t, w1inv, st_x, st, post.t, q.t, pa.t, pre.t, 0)
    torch.cuda.synchronize()
    for g in (xq, W1q, post, q, pa, pre):
        assert g.intact()
    xq_o, _ = ref.quantise_x(P["x"], s_x)
    W1q_o, _, s_w1i = ref.w1_cache(P["W1"])
    assert np.array_equal(host_bits(xq.t), xq_o)
    assert np.array_equal(host_bits(W1q.t), W1q_o)
    assert np.float32(w1inv[0].item()) == s_w1i
    comb = np.float32(np.float32(np.float32(1) / s_x) * s_w1i)
    X, Wd = ref.e4m3_to_f64(xq_o), ref.e4m3_to_f64(W1q_o)
    exact = (X @ Wd.T) * np.float64(comb)
    pre_g = host_bits(pre.t).astype(np.float64)
    bound = d * 2.0 ** -24 * (np.abs(X) @ np.abs(Wd).T) * np.float64(comb) + 2.0 ** -24 * np.abs(pre_g) + 1e-30
    assert bool((np.abs(pre_g - exact) <= bound).all())
    pg = host_bits(post.t)
    assert np.array_equal(pg, ref.relu2_post(host_bits(pre.t)))
    assert np.array_equal(host_bits(q.t), ref.quantise_post(pg, np.float32(20.0)))
    assert np.array_equal(host_bits(pa.t), _pa_oracle(pg, M, h))


# ---------------------------------------------------------------------------
# generic FP8 linear layer (attention projections)
# ---------------------------------------------------------------------------

LINEAR_SHAPES = [(300, 768, 2304), (1000, 768, 768), (129, 512, 768), (33, 16, 48), (16384, 768, 2304)]


@pytest.mark.parametrize("M,K,N", LINEAR_SHAPES[:4])
def test_linear_fwd_fp8_bit_exact_grid(M, K, N):
    P = synth.make_problem(M, K, N, seed=M + N, x_dist="grid", w_dist="grid")   # W1 is [N,K]
    st_x = _state(2.0, 16.0)
    xq_o, _ = ref.quantise_x(P["x"], 16.0)
    Wq_o = ref.e4m3_bits_from_f32((ref.bf16_to_f64(P["W1"]) * 1024.0).astype(np.float32))
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    pax = torch.empty(A.fp8mlp_x_partial_amax_count(M, K), device="cuda")
    A.fp8mlp_quantize_x(M, K, dev_bf16(P["x"]), st_x, xq, pax)
    y = Guarded((M, N), torch.bfloat16)
    A.fp8mlp_linear_fwd_fp8(M, K, N, xq, dev_u8(Wq_o), dev_f32(np.array([1 / 1024.0, 0, 0, 0], np.float32)), st_x, y.t)
    torch.cuda.synchronize()
    want = ref.linear_fp8(xq_o, Wq_o, np.float32(1 / 16.0), np.float32(1 / 1024.0))
    assert np.array_equal(host_bits(y.t), want)
    assert y.intact()


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("M,K,N", LINEAR_SHAPES)
def test_linear_fp8_fwd_bwd_normal(M, K, N, split):
    """With a workspace (split) dW of the shapes with few output tiles is
    summed in two halves over the tokens: (300, 768, 2304) at row 192,
    (1000, 768, 768) at 512, (129, 512, 768) at 128 (one row in the second
    half), 16384 x 768 -> 2304 at 8192; M = 33 is below the split size."""
    P = synth.make_problem(M, K, N, seed=7 * M + N)
    s_x = np.float32(448.0 / 9.0)
    st_x = _state(2.0, float(s_x))
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    pax = torch.empty(A.fp8mlp_x_partial_amax_count(M, K), device="cuda")
    A.fp8mlp_quantize_x(M, K, dev_bf16(P["x"]), st_x, xq, pax)
    Wq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    inv = torch.empty(4, device="cuda")
    ws = torch.empty(A.fp8mlp_workspace_size(0, K, N), dtype=torch.uint8, device="cuda")
    A.fp8mlp_weight_fp8_cache_refresh(N, K, dev_bf16(P["W1"]), Wq, inv, ws)
    y = Guarded((M, N), torch.bfloat16)
    A.fp8mlp_linear_fwd_fp8(M, K, N, xq, Wq, inv, st_x, y.t)
    g = np.random.default_rng(M)
    dY = synth.to_bf16_bits(g.standard_normal((M, N)).astype(np.float32))
    dX = Guarded((M, K), torch.bfloat16)
    dW = Guarded((N, K), torch.float32)
    wsl = Guarded((max(1, A.fp8mlp_linear_bwd_workspace_size(M, K, N)),), torch.uint8) if split else None
    A.fp8mlp_linear_bwd(M, K, N, dev_bf16(P["x"]), dev_bf16(P["W1"]), dev_bf16(dY), dX.t, dW.t,
                        workspace=wsl.t if split else None)
    torch.cuda.synchronize()
    if split:
        assert wsl.intact()
    rows = np.arange(M) if M <= 1000 else np.unique(np.r_[0, M - 1, np.random.default_rng(1).integers(0, M, 64)])
    xq_o, _ = ref.quantise_x(P["x"][rows], s_x)
    Wq_o, _, swi = ref.w1_cache(P["W1"])
    assert np.array_equal(host_bits(Wq), Wq_o)
    y_o = ref.linear_fp8(xq_o, Wq_o, np.float32(np.float32(1) / s_x), swi)
    assert rel_fro(ref.bf16_to_f64(host_bits(y.t)[rows]), ref.bf16_to_f64(y_o)) < 4e-3
    # element by element: the exact product of the e4m3 operands, scaled
    Xq, Wqd = ref.e4m3_to_f64(xq_o), ref.e4m3_to_f64(Wq_o)
    comb = float(np.float32(np.float32(np.float32(1) / s_x) * np.float32(swi[0] if np.ndim(swi) else swi)))
    ok, nbad = within_accumulation_bound(ref.bf16_to_f64(host_bits(y.t)[rows]), (Xq @ Wqd.T) * comb,
                                         (np.abs(Xq) @ np.abs(Wqd).T) * comb, K, True, extra=2.0 ** -23)
    assert ok, nbad
    exact = ref.bf16_to_f64(P["x"][rows]) @ ref.bf16_to_f64(P["W1"]).T
    assert rel_fro(ref.bf16_to_f64(host_bits(y.t)[rows]), exact) < 6e-2
    dX_o = ref.bf16_bits_from_f32(ref.f32(ref.bf16_to_f64(dY[rows]) @ ref.bf16_to_f64(P["W1"])))
    assert rel_fro(ref.bf16_to_f64(host_bits(dX.t)[rows]), ref.bf16_to_f64(dX_o)) < TOL_GRAD
    Gr, Wd = ref.bf16_to_f64(dY[rows]), ref.bf16_to_f64(P["W1"])
    ok, nbad = within_accumulation_bound(ref.bf16_to_f64(host_bits(dX.t)[rows]), Gr @ Wd, np.abs(Gr) @ np.abs(Wd), N,
                                         True)
    assert ok, nbad
    if M <= 1000:
        _, dW_o = ref.linear_bwd(P["x"], P["W1"], dY)
        assert rel_fro(host_bits(dW.t), dW_o) < TOL_GRAD
        # with the token split, each half is within its own bound and the
        # final add rounds once more (relative 2^-24)
        G, X = ref.bf16_to_f64(dY), ref.bf16_to_f64(P["x"])
        ok, nbad = within_accumulation_bound(host_bits(dW.t), G.T @ X, np.abs(G).T @ np.abs(X), M, False,
                                             extra=2.0 ** -23)
        assert ok, nbad
    else:
        G, X = ref.bf16_to_f64(dY), ref.bf16_to_f64(P["x"])
        pairs = [(0, 0), (N - 1, K - 1), (N // 2, 17), (5, K // 3)]
        got = np.array([host_bits(dW.t)[i, j] for i, j in pairs])
        want = np.array([G[:, i] @ X[:, j] for i, j in pairs])
        assert rel_fro(got, want) < TOL_GRAD
    assert y.intact() and dX.intact() and dW.intact()


def test_smoke_entry_point():
    """The entry point the driver runs: one small training step through the
    C ABI on cuda:0, checked against the oracle inside."""
    import __graft_entry__
    __graft_entry__.smoke()
    assert A.fp8mlp_get_device_status() == 0


# ---------------------------------------------------------------------------
# a seeded sweep of shapes: ragged tails at every position
# ---------------------------------------------------------------------------

def _random_shapes(n, seed):
    g = np.random.default_rng(seed)
    shapes = []
    for _ in range(n):
        M = int(g.integers(1, 2049))
        d = 16 * int(g.integers(1, 65))    # 16 .. 1024
        h = 16 * int(g.integers(1, 257))   # 16 .. 4096
        shapes.append((M, d, h))
    return shapes


@pytest.mark.parametrize("M,d,h", _random_shapes(16, 2026))
def test_random_shapes_up_projection_and_step(M, d, h):
    """On grid inputs (every partial sum exact in fp32) the fused
    up-projection's post, FP8 copy and partial amax equal the oracle's bit
    for bit; the library's scheduled training step equals the serial calls
    bit for bit on normal inputs."""
    from fp8_relu_mlp_b200.block import MLPBlock
    G = synth.make_problem(M, d, h, seed=M + 7 * d + h, x_dist="grid", w_dist="grid")
    s = np.float32(448.0 / 37.0)
    st = _state(2.0, float(s))
    post, q, pa, _ = _up(M, d, h, dev_bf16(G["x"]), dev_bf16(G["W1"]), st)
    post_o = ref.relu2_post(ref.up_proj(G["x"], G["W1"]))
    assert np.array_equal(host_bits(post.t), post_o)
    assert np.array_equal(host_bits(q.t), ref.quantise_post(post_o, s))
    assert np.array_equal(host_bits(pa.t), _pa_oracle(post_o, M, h))
    P = synth.make_problem(M, d, h, seed=M + d + h)

    def make():
        b = MLPBlock(M, d, h)
        for k in ("x", "W1", "W2", "dOut"):
            getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
        b.refresh_w2_cache()
        b.calibrate()
        return b

    e, n = make(), make()
    for _ in range(2):
        e.refresh_w2_cache()
        e.train_step()
        n.train_step_native()
    torch.cuda.synchronize()
    for k in ("post", "post_fp8", "out", "dPre", "dX", "dW1", "dW2", "W2q_t", "state", "partial_amax"):
        assert torch.equal(getattr(e, k), getattr(n, k)), k
    assert A.fp8mlp_get_device_status() == 0
