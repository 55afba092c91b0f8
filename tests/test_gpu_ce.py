"""Parity of the softcapped cross-entropy head (CUDA path, through the C ABI)
against the CPU oracle.

Tolerances follow from the arithmetic of the kernels:
  * logits: exact on grid inputs (x = k/4, W = k/256: every partial sum is
    exact in fp32); otherwise within eps_y = d 2^-24 max_v sum_k |x_k W_vk|
    (fp32 accumulation in any order; 2^-14 per add for the e4m3 GEMM, whose
    accumulation need not round to full fp32);
  * lse, z - c: the hardware 2^x (relative error ~2^-22), the Newton
    reciprocal (< 1.4e-7) and the fp32 sum of 128 terms per thread give
    |error| < 3e-5; tested at 5e-5 + eps_y;
  * dlogits: BF16 rounding (2^-9 relative) plus, where the one-hot cancels
    against the softmax, an absolute part 1e-4 g W_m p (1 - t^2).
"""
import numpy as np
import pytest
import torch

from fp8_relu_mlp_b200 import _abi as A
from fp8_relu_mlp_b200 import synth
from oracle import ref
from tests.gpu_util import Guarded, dev_bf16, dev_f32, dev_u8, host_bits, rel_fro

pytestmark = pytest.mark.gpu

CAP = 15.0
TOL_TR = 5e-5  # transcendental + summation part of the lse / z - c error

SHAPES = [  # (M, d, V, T): ragged rows, columns and vocabulary tiles
    (300, 128, 1040, 3),
    (256, 64, 256, 1),
    (1, 64, 16, 1),
    (513, 768, 4096, 2),
    (200, 96, 528, 4),    # the most targets per row; d and V end inside a block
]
WEIGHTS = [1.0, 0.5, 0.25, 0.125]


def _state(margin=2.0, s0=1.0):
    st = torch.zeros(8, dtype=torch.float32, device="cuda")
    A.fp8mlp_scale_state_init(st, margin, s0)
    return st


class Head:
    """Device buffers of one head problem and the calls on them."""

    def __init__(self, P, T, weights, cap=CAP):
        self.x_bits, self.W_bits, self.tg = P["x"], P["W"], P["targets"]
        self.M, self.d = self.x_bits.shape
        self.V = self.W_bits.shape[0]
        self.T = T
        self.w = list(weights[:T])
        self.cap = cap
        self.x = dev_bf16(self.x_bits)
        self.W = dev_bf16(self.W_bits)
        self.targets = torch.from_numpy(np.ascontiguousarray(self.tg, np.int32)).cuda()
        self.lse = Guarded((self.M,), torch.float32)
        self.row = Guarded((self.M,), torch.float32)
        self.loss = Guarded((3,), torch.float32)
        self.ws = torch.empty(max(A.fp8mlp_ce_workspace_size(self.M, self.V, T), 16), dtype=torch.uint8,
                              device="cuda")

    def fwd(self):
        A.fp8mlp_ce_fwd(self.M, self.d, self.V, self.T, self.x, self.W, self.targets, self.w, self.cap,
                        self.lse.t, self.row.t, self.loss.t, self.ws)

    def fp8_operands(self, s_x, w_cache=None):
        """e4m3 copies: x under the delayed scale s_x; W either from the
        library's cache refresh (w_cache None) or given (codes, scale_inv)."""
        self.st_x = _state(2.0, float(s_x))
        self.xq = torch.empty(self.M, self.d, dtype=torch.uint8, device="cuda")
        pax = torch.empty(max(A.fp8mlp_x_partial_amax_count(self.M, self.d), 1), device="cuda")
        A.fp8mlp_quantize_x(self.M, self.d, self.x, self.st_x, self.xq, pax)
        if w_cache is None:
            self.Wq = torch.empty(self.V, self.d, dtype=torch.uint8, device="cuda")
            self.w_inv = torch.empty(4, device="cuda")
            ws = torch.empty(A.fp8mlp_workspace_size(0, self.d, self.V), dtype=torch.uint8, device="cuda")
            A.fp8mlp_weight_fp8_cache_refresh(self.V, self.d, self.W, self.Wq, self.w_inv, ws)
        else:
            self.Wq = dev_u8(w_cache[0])
            self.w_inv = dev_f32(np.array([w_cache[1], 0, 0, 0], np.float32))

    def fwd_fp8(self):
        A.fp8mlp_ce_fwd_fp8(self.M, self.d, self.V, self.T, self.xq, self.st_x, self.Wq, self.w_inv, self.targets,
                            self.w, self.cap, self.lse.t, self.row.t, self.loss.t, self.ws)

    def bwd(self, dloss=None, reduction=A.CE_SUM, fp8=False):
        dl = Guarded((self.M, self.V), torch.bfloat16)
        dls = None if dloss is None else torch.tensor([dloss], dtype=torch.float32, device="cuda")
        if fp8:
            A.fp8mlp_ce_bwd_dlogits_fp8(self.M, self.d, self.V, self.T, self.xq, self.st_x, self.Wq, self.w_inv,
                                        self.targets, self.w, self.cap, self.lse.t, self.loss.t, dls, reduction,
                                        dl.t)
        else:
            A.fp8mlp_ce_bwd_dlogits(self.M, self.d, self.V, self.T, self.x, self.W, self.targets, self.w, self.cap,
                                    self.lse.t, self.loss.t, dls, reduction, dl.t)
        return dl

    def intact(self):
        return self.lse.intact() and self.row.intact() and self.loss.intact()


def _eps_y(X, Wm, unit=2.0 ** -24):
    """Per-row bound on the fp32 accumulation error of the logits."""
    d = X.shape[1]
    return d * unit * (np.abs(X) @ np.abs(Wm).T).max(axis=1)


def _check_fwd(h, y, eps):
    """GPU lse, row loss and totals against the oracle on logits y (fp64)."""
    f = ref.ce_forward(y, h.tg, h.w, h.cap)
    lse = host_bits(h.lse.t).astype(np.float64)
    row = host_bits(h.row.t).astype(np.float64)
    tot = host_bits(h.loss.t).astype(np.float64)
    np.testing.assert_array_less(np.abs(lse - f["lse"]), TOL_TR + eps + 1e-6 * np.abs(f["lse"]))
    _, we = ref._ce_targets(h.tg, h.w, h.V)
    wrow = we.sum(axis=1)
    np.testing.assert_array_less(np.abs(row - f["row_loss"]), wrow * (2 * TOL_TR + 2 * eps) + 1e-6 * np.abs(f["row_loss"]) + 1e-12)
    assert tot[1] == np.float32(f["weight_sum"])
    np.testing.assert_allclose(tot[0], f["loss_sum"], rtol=1e-6, atol=float((wrow * (2 * TOL_TR + 2 * eps)).sum()) + 1e-12)
    np.testing.assert_allclose(tot[2], f["mean"], rtol=1e-6, atol=float((wrow * (2 * TOL_TR + 2 * eps)).sum() / max(f["weight_sum"], 1.0)) + 1e-12)
    return f


def _check_dlogits(h, dl, y, f, g, eps):
    """GPU dlogits (BF16) elementwise against the oracle's fp64 gradient."""
    want = ref.ce_backward_dlogits(y, h.tg, h.w, h.cap, f["lse"], g)
    got = ref.bf16_to_f64(host_bits(dl.t))
    th = np.tanh(y / h.cap)
    p = np.exp(h.cap * th - f["lse"][:, None])
    _, we = ref._ce_targets(h.tg, h.w, h.V)
    scale = abs(g) * we.sum(axis=1)[:, None] * p * (1 - th * th)
    tol = 2.0 ** -8 * np.abs(want) + (1e-4 + 4 * eps[:, None]) * scale + 1e-30
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{bad.sum()} dlogits outside tolerance, worst at {np.unravel_index(np.argmax(np.abs(got - want) - tol), got.shape)}"
    assert rel_fro(got, want) < 4e-3
    return want


@pytest.mark.parametrize("M,d,V,T", SHAPES)
def test_ce_bf16_grid(M, d, V, T):
    P = synth.make_head_problem(M, d, V, T=T, seed=M + V, x_dist="grid", ignore_frac=0.1 if T > 1 else 0.0)
    h = Head(P, T, WEIGHTS)
    h.fwd()
    torch.cuda.synchronize()
    y = ref.head_logits(h.x_bits, h.W_bits)
    zero = np.zeros(M)
    f = _check_fwd(h, y, zero)
    dl = h.bwd(reduction=A.CE_MEAN)
    torch.cuda.synchronize()
    _check_dlogits(h, dl, y, f, ref.ce_grad_scale(1.0, f["weight_sum"], True), zero)
    assert h.intact() and dl.intact()


@pytest.mark.parametrize("M,d,V,T", SHAPES)
@pytest.mark.parametrize("logit_std", [4.0, 12.0])
def test_ce_bf16_normal(M, d, V, T, logit_std):
    # logit std 12 against the cap 15 drives many logits into the tanh's flat part
    P = synth.make_head_problem(M, d, V, T=T, seed=3 * M + V, logit_std=logit_std, ignore_frac=0.05)
    h = Head(P, T, WEIGHTS)
    h.fwd()
    torch.cuda.synchronize()
    X, Wm = ref.bf16_to_f64(h.x_bits), ref.bf16_to_f64(h.W_bits)
    y = X @ Wm.T
    eps = _eps_y(X, Wm)
    f = _check_fwd(h, y, eps)
    dl = h.bwd()
    torch.cuda.synchronize()
    want = _check_dlogits(h, dl, y, f, 1.0, eps)
    # the BF16 backward through the head on the GPU's dlogits, against the
    # oracle's chain from its own dlogits
    dX = Guarded((M, d), torch.bfloat16)
    dW = Guarded((V, d), torch.float32)
    A.fp8mlp_linear_bwd(M, d, V, h.x, h.W, dl.t, dX.t, dW.t)
    torch.cuda.synchronize()
    _, dX_o, dW_o = ref.ce_backward(h.x_bits, h.W_bits, want)
    assert rel_fro(ref.bf16_to_f64(host_bits(dX.t)), ref.bf16_to_f64(dX_o)) < 1e-2
    assert rel_fro(host_bits(dW.t), dW_o) < 1e-2
    assert h.intact() and dl.intact() and dX.intact() and dW.intact()


@pytest.mark.parametrize("M,d,V,T", SHAPES)
def test_ce_fp8_grid(M, d, V, T):
    # power-of-two scales on grid inputs: both e4m3 copies are exact, so the
    # FP8 logits equal the BF16 ones and both are exact
    P = synth.make_head_problem(M, d, V, T=T, seed=5 * M + V, x_dist="grid")
    h = Head(P, T, WEIGHTS)
    Wq_o = ref.e4m3_bits_from_f32((ref.bf16_to_f64(h.W_bits) * 1024.0).astype(np.float32))
    h.fp8_operands(16.0, (Wq_o, np.float32(1 / 1024.0)))
    h.fwd_fp8()
    torch.cuda.synchronize()
    xq_o, _ = ref.quantise_x(h.x_bits, 16.0)
    y = ref.head_logits_fp8(xq_o, Wq_o, np.float32(1 / 16.0), np.float32(1 / 1024.0))
    assert np.array_equal(y, ref.head_logits(h.x_bits, h.W_bits))
    zero = np.zeros(M)
    f = _check_fwd(h, y, zero)
    dl = h.bwd(fp8=True)
    torch.cuda.synchronize()
    _check_dlogits(h, dl, y, f, 1.0, zero)
    assert h.intact() and dl.intact()


@pytest.mark.parametrize("M,d,V,T", SHAPES)
def test_ce_fp8_normal(M, d, V, T):
    P = synth.make_head_problem(M, d, V, T=T, seed=7 * M + V, logit_std=6.0)
    h = Head(P, T, WEIGHTS)
    s_x = np.float32(448.0 / 9.0)
    h.fp8_operands(s_x)
    h.fwd_fp8()
    torch.cuda.synchronize()
    xq_o, _ = ref.quantise_x(h.x_bits, s_x)
    Wq_o, _, swi = ref.w1_cache(h.W_bits)
    assert np.array_equal(host_bits(h.Wq), Wq_o)
    sxi = np.float32(np.float32(1.0) / s_x)
    y = ref.head_logits_fp8(xq_o, Wq_o, sxi, swi)
    comb = float(np.float32(sxi * swi))
    eps = _eps_y(ref.e4m3_to_f64(xq_o), ref.e4m3_to_f64(Wq_o), unit=2.0 ** -14) * comb
    f = _check_fwd(h, y, eps)
    dl = h.bwd(fp8=True, reduction=A.CE_MEAN)
    torch.cuda.synchronize()
    _check_dlogits(h, dl, y, f, ref.ce_grad_scale(1.0, f["weight_sum"], True), eps)
    assert h.intact() and dl.intact()


def test_ce_dloss_scales_gradient_exactly():
    # g = 0.5 scales every fp32 product by a power of two: BF16 halves exactly
    P = synth.make_head_problem(300, 128, 1040, T=2, seed=11)
    h = Head(P, 2, WEIGHTS)
    h.fwd()
    a = h.bwd()
    b = h.bwd(dloss=0.5)
    torch.cuda.synchronize()
    A_, B_ = ref.bf16_to_f64(host_bits(a.t)), ref.bf16_to_f64(host_bits(b.t))
    assert np.array_equal(B_, 0.5 * A_)


def test_ce_all_targets_ignored_and_empty_batch():
    P = synth.make_head_problem(70, 64, 512, T=2, seed=13)
    P["targets"][:] = -1
    P["targets"][3, 1] = 512  # == V: ignored as well
    h = Head(P, 2, WEIGHTS)
    h.fwd()
    dl = h.bwd(reduction=A.CE_MEAN)
    dl_sum = h.bwd(reduction=A.CE_SUM)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(h.loss.t), np.zeros(3, np.float32))
    assert np.array_equal(host_bits(h.row.t), np.zeros(70, np.float32))
    f = ref.ce_forward(ref.head_logits(h.x_bits, h.W_bits), h.tg, h.w, CAP)
    np.testing.assert_array_less(np.abs(host_bits(h.lse.t) - f["lse"]), TOL_TR + _eps_y(ref.bf16_to_f64(h.x_bits), ref.bf16_to_f64(h.W_bits)))
    assert not host_bits(dl.t).any() and not host_bits(dl_sum.t).any()
    # M = 0: nothing launched, the totals are zero
    loss = torch.full((3,), 7.0, device="cuda")
    A.fp8mlp_ce_fwd(0, 64, 512, 1, None, None, None, None, CAP, None, None, loss, None)
    torch.cuda.synchronize()
    assert loss.tolist() == [0.0, 0.0, 0.0]


def test_ce_forward_is_deterministic():
    P = synth.make_head_problem(513, 768, 4096, T=1, seed=17)
    h = Head(P, 1, WEIGHTS)
    h.fwd()
    torch.cuda.synchronize()
    first = (host_bits(h.lse.t).copy(), host_bits(h.loss.t).copy())
    for _ in range(3):
        h.fwd()
    torch.cuda.synchronize()
    assert np.array_equal(first[0], host_bits(h.lse.t)) and np.array_equal(first[1], host_bits(h.loss.t))


@pytest.mark.parametrize("fp8", [False, True])
def test_ce_fullsize_sampled_rows(fp8):
    # the benchmark's workload: 16384 tokens, d = 768, V = 50304; the oracle
    # evaluates sampled rows one by one
    W = synth.WORKLOADS["ce16k"]
    M, d, V = W.M, W.d, W.h
    P = synth.make_head_problem(M, d, V, T=1, seed=0, logit_std=4.0)
    h = Head(P, 1, WEIGHTS)
    if fp8:
        s_x = np.float32(448.0 / 10.0)
        h.fp8_operands(s_x)
        h.fwd_fp8()
    else:
        h.fwd()
    dl = h.bwd(fp8=fp8, reduction=A.CE_MEAN)
    torch.cuda.synchronize()
    rows = np.unique(np.r_[0, 1, 255, 256, M - 1, np.random.default_rng(2).integers(0, M, 40)])
    sub = Head.__new__(Head)
    sub.tg, sub.w, sub.cap, sub.V = h.tg[rows], h.w, h.cap, V
    if fp8:
        xq_o, _ = ref.quantise_x(h.x_bits[rows], s_x)
        Wq_o, _, swi = ref.w1_cache(h.W_bits)
        sxi = np.float32(np.float32(1.0) / s_x)
        y = ref.head_logits_fp8(xq_o, Wq_o, sxi, swi)
        eps = _eps_y(ref.e4m3_to_f64(xq_o), ref.e4m3_to_f64(Wq_o), unit=2.0 ** -14) * float(np.float32(sxi * swi))
    else:
        X, Wm = ref.bf16_to_f64(h.x_bits[rows]), ref.bf16_to_f64(h.W_bits)
        y = X @ Wm.T
        eps = _eps_y(X, Wm)
    f = ref.ce_forward(y, sub.tg, sub.w, CAP)
    lse = host_bits(h.lse.t)[rows].astype(np.float64)
    row = host_bits(h.row.t)[rows].astype(np.float64)
    np.testing.assert_array_less(np.abs(lse - f["lse"]), TOL_TR + eps + 1e-6 * np.abs(f["lse"]))
    np.testing.assert_array_less(np.abs(row - f["row_loss"]), 2 * TOL_TR + 2 * eps + 1e-6 * np.abs(f["row_loss"]))
    tot = host_bits(h.loss.t).astype(np.float64)
    assert tot[1] == M  # every target valid, weight 1
    np.testing.assert_allclose(tot[0], host_bits(h.row.t).astype(np.float64).sum(), rtol=1e-5)
    np.testing.assert_allclose(tot[2], tot[0] / M, rtol=1e-6)
    # dlogits of the sampled rows (g = 1 / M for the mean)
    g = 1.0 / M
    want = ref.ce_backward_dlogits(y, sub.tg, sub.w, CAP, f["lse"], g)
    got = ref.bf16_to_f64(host_bits(dl.t)[rows])
    th = np.tanh(y / CAP)
    scale = g * np.exp(CAP * th - f["lse"][:, None]) * (1 - th * th)
    tol = 2.0 ** -8 * np.abs(want) + (1e-4 + 4 * eps[:, None]) * scale + 1e-30
    assert not (np.abs(got - want) > tol).any()
    assert h.intact() and dl.intact()


@pytest.mark.parametrize("cap", [1.0, 40.0])
def test_ce_cap_extremes(cap):
    # logits far beyond the cap: with c = 40 the smallest terms exp(z - c)
    # reach e^-80 (still normal fp32), with c = 1 every z is within [-1, 1].
    # The exponent arguments grow with c (|c log2(e) (t - 1)| <= 2c log2(e)),
    # so the transcendental part of the tolerance scales with c / 15.
    M, d, V, T = 257, 64, 1040, 2
    P = synth.make_head_problem(M, d, V, T=T, seed=int(cap) + 29, logit_std=100.0)
    h = Head(P, T, WEIGHTS, cap=cap)
    h.fwd()
    dl = h.bwd(reduction=A.CE_MEAN)
    torch.cuda.synchronize()
    X, Wm = ref.bf16_to_f64(h.x_bits), ref.bf16_to_f64(h.W_bits)
    y = X @ Wm.T
    eps = _eps_y(X, Wm)
    f = ref.ce_forward(y, h.tg, h.w, cap)
    tol = TOL_TR * max(1.0, cap / 15.0) + eps
    lse = host_bits(h.lse.t).astype(np.float64)
    np.testing.assert_array_less(np.abs(lse - f["lse"]), tol + 1e-6 * np.abs(f["lse"]))
    row = host_bits(h.row.t).astype(np.float64)
    _, we = ref._ce_targets(h.tg, h.w, V)
    np.testing.assert_array_less(np.abs(row - f["row_loss"]), we.sum(axis=1) * 2 * tol + 1e-6 * np.abs(f["row_loss"]) + 1e-12)
    want = ref.ce_backward_dlogits(y, h.tg, h.w, cap, f["lse"], ref.ce_grad_scale(1.0, f["weight_sum"], True))
    got = ref.bf16_to_f64(host_bits(dl.t))
    assert rel_fro(got, want) < 4e-3
    assert np.isfinite(lse).all() and np.isfinite(got).all()
    assert h.intact() and dl.intact()
