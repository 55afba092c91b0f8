"""Plain, slow, obviously-correct CPU oracle of the fused FP8 ReLU^2 MLP block.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs, never by the product path.
It shares no code with the CUDA library and does not import it.

Everything is numpy.  Arithmetic that the method leaves in full precision is
done in fp64.  The rounding points that the method fixes (BF16 storage of
``post``, the FP8 e4m3 copy, the fp32 epilogue registers and the fp32 scale
arithmetic) are emulated on bit patterns written out here, not borrowed from
a library.  Library primitives used as steps: ``numpy.matmul`` in fp64,
``numpy.float32`` scalar/array arithmetic (IEEE round-to-nearest-even),
``numpy.rint`` (round-half-even), ``numpy.frexp``.

Sources, cited by page title and section:
  [R83]  "NanoGPT Speedrun (Track 1)" (Recursive), section "Changes vs Record
         #83", item 4: the ReLU^2 MLP kernel stores only post = relu(pre)^2 and
         the backward rebuilds relu(pre) = sqrt(post).
  [RUO]  same page, section "From Unoptimized / Approach", item 5: FP8 e4m3 MLP
         GEMMs in the training forward, BF16 backward, BF16 at evaluation.
  [PAR]  "A Retrospective on Our World Records" (paradigma.inc), Modded-NanoGPT
         Main Track section: fused up-projection writes BF16 post, an FP8 copy
         and a tiny partial-amax tensor; delayed scaling from amax(t-1) times a
         safety margin; transposed FP8 cache of W2 refreshed after optimizer
         updates; BF16 backward unchanged.
  [PAR-N] same page, "A few implementation notes": exact non-delayed W2
         refresh is viable; BF16 post is kept for backward; amax(t-1) with a
         margin instead of a rolling window.

Readings where the pages are silent:
  * scale s = 448 / (margin * amax), 448 being the largest finite e4m3 value;
  * the FP8 copy quantises the BF16-rounded post;
  * amax/scale keep the previous value when amax is zero or not finite;
  * W2 cache scale: exact (current-step) amax of |W2|, no margin; a zero or
    non-finite amax gives s_w = 1;
  * backward uses BF16 post and BF16 W2 (straight-through over the FP8 step);
  * out, dX and dPre are BF16; dW1 and dW2 are fp32;
  * RMSNorm of the layer stack has no gain, eps = 1e-6.

Tensors are passed as numpy arrays of raw bit patterns: BF16 as ``uint16``,
e4m3 as ``uint8``; fp32 quantities as ``float32``.

Layouts (row-major):  x [M,d]  W1 [h,d]  W2 [h,d]  post [M,h]  q [M,h]
W2q_t [d,h]  out [M,d]  dOut [M,d]  dPre [M,h]  dX [M,d]  dW1 [h,d]  dW2 [h,d].
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0          # largest finite OCP e4m3fn value: 1.75 * 2**8
E4M3_NAN = 0x7F           # the code satfinite conversion gives for NaN input

# ----------------------------------------------------------------------------
# Rounding primitives on bit patterns
# ----------------------------------------------------------------------------


def f32(x):
    """Round to fp32 (IEEE binary32, round-to-nearest-even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_bits_from_f32(v):
    """BF16 bit pattern of fp32 values, round-to-nearest-even; NaN stays NaN.

    BF16 is the upper half of a binary32.  RNE on the dropped 16 bits: add
    0x7FFF plus the lowest kept bit, then truncate.  Infinity and overflow come
    out right because the carry walks into the exponent field.
    """
    v = np.asarray(v, dtype=np.float32)
    u = v.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(v)
    if nan.any():
        sign = ((u >> 16) & 0x8000).astype(np.uint16)
        r = np.where(nan, sign | np.uint16(0x7FC0), r)
    return r


def bf16_to_f64(bits):
    """Exact value of BF16 bit patterns (as fp64)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def e4m3_bits_from_f32(v):
    """OCP e4m3fn code of fp32 values: round-to-nearest-even, saturating.

    Format: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
    infinities; 0x7F / 0xFF are NaN.  Normal values (1+m/8)*2**(e-7) for
    e=1..15 (e=15,m=7 excluded), subnormals m*2**-9.  Saturating conversion:
    every magnitude that does not round to a value <= 448 becomes 448 (this
    includes infinity); NaN becomes 0x7F.
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    sign = np.signbit(v)
    a = np.abs(v)
    nan = np.isnan(v)
    a = np.where(nan, 0.0, a)
    with np.errstate(invalid="ignore", over="ignore"):
        # exponent of the leading bit: a = f * 2**E, f in [0.5, 1)
        _, E = np.frexp(np.where(a > 0, a, 1.0))
        e_unb = E.astype(np.int64) - 1                   # floor(log2 a)
        # quantum: 2**(e_unb-3) in the normal range, 2**-9 below 2**-6
        qexp = np.maximum(e_unb, -6) - 3
        quantum = np.ldexp(1.0, qexp)
        n = np.rint(np.where(np.isfinite(a), a / quantum, 0.0))   # ties to even
        r = n * quantum                                   # rounded magnitude
        r = np.where(np.isinf(a), np.inf, r)
    r = np.where(r > E4M3_MAX, E4M3_MAX, r)               # satfinite
    # encode r (exact grid value) into bits
    code = np.zeros(r.shape, dtype=np.int64)
    sub = r < 2.0 ** -6
    code = np.where(sub, np.rint(r / 2.0 ** -9).astype(np.int64), code)
    _, E2 = np.frexp(np.where(r > 0, r, 1.0))
    e2 = E2.astype(np.int64) - 1
    mant = np.rint((r / np.ldexp(1.0, e2) - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, code, ((e2 + 7) << 3) | mant)
    code = np.where(sign, code | 0x80, code)
    code = np.where(nan, E4M3_NAN, code)
    return code.astype(np.uint8)


def e4m3_to_f64(bits):
    """Exact value of e4m3fn codes (NaN for 0x7F / 0xFF)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


# ----------------------------------------------------------------------------
# Forward
# ----------------------------------------------------------------------------


def up_proj(x, W1):
    """pre = x . W1^T, [M,h], in fp64 from the BF16 operands ([R83] item 4;
    [PAR] "fused up-projection kernel")."""
    return bf16_to_f64(x) @ bf16_to_f64(W1).T


def relu2_post(pre):
    """post = relu(pre)^2 as stored: BF16 of the fp32 square of the fp32 relu.

    [R83] item 4 (post = relu(pre)^2 is the one stored tensor); [PAR] (BF16
    post written for the backward).  The epilogue holds pre in fp32 registers,
    so relu and the square are taken in fp32, then rounded to BF16 (RNE).
    """
    r = np.maximum(f32(pre), np.float32(0.0))
    p = (r * r).astype(np.float32)           # fp32 multiply, RNE
    return bf16_bits_from_f32(p)


def quantise_post(post, s):
    """FP8 copy q = e4m3(fp32(post * s)) of the BF16 post ([PAR]: emitted while
    post is in registers, scaled by the delayed scale)."""
    p = bf16_to_f64(post).astype(np.float32)
    return e4m3_bits_from_f32(p * np.float32(s))


def partial_amax(post, rows, cols):
    """Partial amax: max of post over each [rows x cols] block, fp32, laid out
    [ceil(M/rows), ceil(h/cols)] ([PAR]: "a tiny partial-amax tensor")."""
    P = bf16_to_f64(post)
    M, H = P.shape
    ti, tj = -(-M // rows), -(-H // cols)
    out = np.zeros((ti, tj), dtype=np.float32)
    for i in range(ti):
        for j in range(tj):
            blk = P[i * rows:(i + 1) * rows, j * cols:(j + 1) * cols]
            out[i, j] = np.float32(blk.max()) if blk.size else np.float32(0.0)
    return out


def amax(post):
    """Exact amax of post (post >= 0, so max == max |post|)."""
    P = bf16_to_f64(post)
    return np.float32(P.max()) if P.size else np.float32(0.0)


def down_proj_fp8(q, W2q_t, scale_inv, w2_scale_inv):
    """out = bf16( fp32( sum_k dec(q[m,k]) dec(W2q_t[j,k]) * fp32(s^-1 s_w^-1) ) )

    [PAR]: the down-projection runs as an FP8 scaled matmul on both operands.
    The dequantising factor is formed in fp32 as the kernel forms it.
    """
    comb = np.float32(np.float32(scale_inv) * np.float32(w2_scale_inv))
    acc = e4m3_to_f64(q) @ e4m3_to_f64(W2q_t).T
    return bf16_bits_from_f32(f32(acc * np.float64(comb)))


def down_proj_bf16(post, W2):
    """Evaluation forward: out = bf16(post . W2) with BF16 post and W2 ([RUO]:
    "bf16 at eval")."""
    acc = bf16_to_f64(post) @ bf16_to_f64(W2)
    return bf16_bits_from_f32(f32(acc))


def forward(x, W1, W2q_t, w2_scale_inv, scale, scale_inv):
    """Training forward at step t with the delayed scale s_t ([PAR]).

    Returns dict(pre, post, q, amax, out)."""
    pre = up_proj(x, W1)
    post = relu2_post(pre)
    q = quantise_post(post, scale)
    out = down_proj_fp8(q, W2q_t, scale_inv, w2_scale_inv)
    return dict(pre=pre, post=post, q=q, amax=amax(post), out=out)


# ----------------------------------------------------------------------------
# Delayed scaling state ([PAR], [PAR-N])
# ----------------------------------------------------------------------------

FLAG_KEPT_SCALE = 1     # the last update kept the previous scale


def scale_state_init(margin, initial_scale):
    s = np.float32(initial_scale)
    return dict(amax_prev=np.float32(0.0), scale=s,
                scale_inv=np.float32(np.float32(1.0) / s),
                margin=np.float32(margin), step=0, flags=0)


def scale_update(state, A):
    """s_{t+1} = fp32(448 / fp32(margin * A_t)), s^-1 = fp32(1/s).

    [PAR]: the scale used at step t comes from the amax measured at step t-1
    multiplied by a safety margin; no rolling window ([PAR-N]).  The constant
    448 makes margin * amax land on the largest e4m3 value.  A zero or
    non-finite amax keeps the previous scale and sets FLAG_KEPT_SCALE.
    """
    st = dict(state)
    A = np.float32(A)
    st["amax_prev"] = A
    st["step"] = state["step"] + 1
    if np.isfinite(A) and A > 0:
        den = np.float32(st["margin"] * A)
        s = np.float32(np.float32(E4M3_MAX) / den)
        if np.isfinite(s) and s > 0:
            st["scale"] = s
            st["scale_inv"] = np.float32(np.float32(1.0) / s)
            st["flags"] = state["flags"] & ~FLAG_KEPT_SCALE
            return st
    st["flags"] = state["flags"] | FLAG_KEPT_SCALE
    return st


def reduce_partials(pa):
    """A_t = max over the partial-amax tensor; NaN partials make A_t NaN
    (so that the update keeps the scale)."""
    pa = np.asarray(pa, dtype=np.float32)
    if pa.size == 0:
        return np.float32(0.0)
    if np.isnan(pa).any():
        return np.float32(np.nan)
    return np.float32(pa.max())


# ----------------------------------------------------------------------------
# Transposed FP8 W2 cache ([PAR], [PAR-N] first note)
# ----------------------------------------------------------------------------


def w2_cache(W2):
    """Exact, non-delayed refresh: s_w = fp32(448 / max|W2|),
    W2q_t[j,k] = e4m3(fp32(W2[k,j] * s_w)), s_w^-1 = fp32(1/s_w).

    Returns (W2q_t [d,h] uint8, s_w, s_w_inv)."""
    W = bf16_to_f64(W2)
    a = np.float32(np.abs(W).max()) if W.size else np.float32(0.0)
    if np.isfinite(a) and a > 0:
        s_w = np.float32(np.float32(E4M3_MAX) / a)
    else:
        s_w = np.float32(1.0)
    Wt = W.T.astype(np.float32)                           # exact (BF16 -> fp32)
    q = e4m3_bits_from_f32((Wt * s_w).astype(np.float32))
    return q, s_w, np.float32(np.float32(1.0) / s_w)


# ----------------------------------------------------------------------------
# Backward ([R83] item 4, [PAR] "existing BF16 backward path", [RUO])
# ----------------------------------------------------------------------------


def bwd_dpre(post, dOut, W2):
    """dPost = dOut . W2^T;  dPre = bf16(fp32(2 sqrt(post) dPost)).

    relu(pre) is rebuilt as sqrt(post) of the stored BF16 post ([R83] item 4):
    d(relu(pre)^2)/dpre = 2 relu(pre)."""
    dPost = bf16_to_f64(dOut) @ bf16_to_f64(W2).T
    r = np.sqrt(bf16_to_f64(post))
    return bf16_bits_from_f32(f32(2.0 * r * dPost))


def bwd_dx(dPre, W1):
    """dX = bf16(dPre . W1)."""
    return bf16_bits_from_f32(f32(bf16_to_f64(dPre) @ bf16_to_f64(W1)))


def bwd_dw1(dPre, x):
    """dW1 = fp32(dPre^T . x), [h,d]."""
    return f32(bf16_to_f64(dPre).T @ bf16_to_f64(x))


def bwd_dw2(post, dOut):
    """dW2 = fp32(post^T . dOut), [h,d] (BF16 post, [PAR-N] second note)."""
    return f32(bf16_to_f64(post).T @ bf16_to_f64(dOut))


def backward(x, W1, W2, post, dOut):
    dPre = bwd_dpre(post, dOut, W2)
    return dict(dPre=dPre, dX=bwd_dx(dPre, W1), dW1=bwd_dw1(dPre, x),
                dW2=bwd_dw2(post, dOut))


# ----------------------------------------------------------------------------
# Sampled evaluation at full size: single rows of the forward, single columns
# of the backward.  These evaluate the same definitions at chosen indices.
# ----------------------------------------------------------------------------


def forward_rows(rows, x, W1, W2q_t, w2_scale_inv, scale, scale_inv):
    """Forward of the selected token rows (the MLP is row-wise independent)."""
    return forward(x[rows], W1, W2q_t, w2_scale_inv, scale, scale_inv)


def dpre_column(i, post_col, dOut, W2):
    """Column i of dPre over all M tokens, from column i of the BF16 post."""
    dPost = bf16_to_f64(dOut) @ bf16_to_f64(W2[i])
    r = np.sqrt(bf16_to_f64(post_col))
    return bf16_bits_from_f32(f32(2.0 * r * dPost))


def post_column(i, x, W1):
    """Column i of post over all M tokens."""
    pre = bf16_to_f64(x) @ bf16_to_f64(W1[i])
    return relu2_post(pre)


def dw_entries(pairs, x, W1, W2, dOut):
    """Sampled entries (i, j) of dW1 and dW2 (each needs a full column of post
    and dPre over all tokens)."""
    out1, out2 = [], []
    X = bf16_to_f64(x)
    G = bf16_to_f64(dOut)
    cache = {}
    for i, j in pairs:
        if i not in cache:
            pc = post_column(i, x, W1)
            cache[i] = (pc, dpre_column(i, pc, dOut, W2))
        pc, dc = cache[i]
        out1.append(np.float32(bf16_to_f64(dc) @ X[:, j]))
        out2.append(np.float32(bf16_to_f64(pc) @ G[:, j]))
    return np.array(out1, np.float32), np.array(out2, np.float32)


def dx_rows(rows, x, W1, W2, dOut):
    """Rows of dPre and dX for the selected tokens."""
    pre = up_proj(x[rows], W1)
    post = relu2_post(pre)
    dPre = bwd_dpre(post, dOut[rows], W2)
    return dPre, bwd_dx(dPre, W1)


# ----------------------------------------------------------------------------
# Layer stack with RMSNorm and residual (no counterpart on the pages; the
# block is the 768-dim ReLU^2 MLP of the 9-layer models the pages train)
# ----------------------------------------------------------------------------

RMS_EPS = 1e-6


def rmsnorm_fwd(r):
    """x = bf16(r / sqrt(mean(r^2) + eps)) per row, no gain.  Returns
    (x bits, rstd fp32 per row)."""
    R = bf16_to_f64(r)
    ms = np.mean(R * R, axis=1)
    rstd = 1.0 / np.sqrt(ms + RMS_EPS)
    return bf16_bits_from_f32(f32(R * rstd[:, None])), f32(rstd)


def rmsnorm_bwd(r, dx):
    """dr = rstd * (dx - xhat * mean(dx * xhat)), xhat = r * rstd (unrounded)."""
    R = bf16_to_f64(r)
    G = bf16_to_f64(dx)
    rstd = 1.0 / np.sqrt(np.mean(R * R, axis=1) + RMS_EPS)
    xh = R * rstd[:, None]
    dot = np.mean(G * xh, axis=1)
    return rstd[:, None] * (G - xh * dot[:, None])


def residual_add(r, out):
    """r' = bf16(r + out)."""
    return bf16_bits_from_f32(f32(bf16_to_f64(r) + bf16_to_f64(out)))


def stack_forward(r0, layers, scales):
    """layers: list of dict(W1, W2, W2q_t, w2_scale_inv); scales: list of
    (s, s_inv).  Returns per-layer dicts and the final residual."""
    r = r0
    saved = []
    for L, (s, si) in zip(layers, scales):
        xb, _ = rmsnorm_fwd(r)
        f = forward(xb, L["W1"], L["W2q_t"], L["w2_scale_inv"], s, si)
        saved.append(dict(r=r, x=xb, post=f["post"], amax=f["amax"]))
        r = residual_add(r, f["out"])
    return saved, r


def stack_forward_fp8up(r0, layers, scales, x_scales):
    """The stack with every up-projection on e4m3 copies ("NanoGPT Speedrun
    (Track 1)", From Unoptimized, item 5): per layer x = rmsnorm(r),
    x_q = e4m3(fp32(x s_x)) under the layer's delayed x-scale, pre from the
    e4m3 up-projection against the W1 cache, then post, its FP8 copy and the
    FP8 down-projection as in stack_forward.  layers: dicts with W1q and
    w1_scale_inv as well; x_scales: list of (s_x, s_x_inv).  The saved dicts
    also hold x_amax = max |x| (the next x-scale's amax); the backward is
    stack_backward (BF16 x and W1)."""
    r = r0
    saved = []
    for L, (s, si), (sx, sxi) in zip(layers, scales, x_scales):
        xb, _ = rmsnorm_fwd(r)
        xq, ax = quantise_x(xb, sx)
        post = relu2_post(up_proj_fp8(xq, L["W1q"], sxi, L["w1_scale_inv"]))
        out = down_proj_fp8(quantise_post(post, s), L["W2q_t"], si, L["w2_scale_inv"])
        saved.append(dict(r=r, x=xb, post=post, amax=amax(post), x_amax=ax))
        r = residual_add(r, out)
    return saved, r


def stack_backward(saved, layers, dr_top):
    """Backward through the stack; the residual gradient is carried as BF16.
    Returns (dr0 bits, list of (dW1, dW2))."""
    dr = dr_top
    grads = [None] * len(layers)
    for l in range(len(layers) - 1, -1, -1):
        S, L = saved[l], layers[l]
        g = backward(S["x"], L["W1"], L["W2"], S["post"], dr)
        grads[l] = (g["dW1"], g["dW2"])
        drn = rmsnorm_bwd(S["r"], g["dX"])
        dr = bf16_bits_from_f32(f32(bf16_to_f64(dr) + drn))
    return dr, grads


# ----------------------------------------------------------------------------
# FP8 up-projection ("NanoGPT Speedrun (Track 1)", From Unoptimized, item 5:
# the MLP GEMMs in e4m3 in the training forward, BF16 backward).  Both inputs
# of the up-projection are e4m3 copies: x under its own delayed scale s_x (the
# same recurrence as post's, over max |x|), W1 under an exact cache scale.
# ----------------------------------------------------------------------------


def quantise_x(x, s_x):
    """x_q = e4m3(fp32(x * s_x)) of the BF16 x, and max |x| (the amax that
    drives the next step's s_x)."""
    X = bf16_to_f64(x).astype(np.float32)
    q = e4m3_bits_from_f32((X * np.float32(s_x)).astype(np.float32))
    a = np.float32(np.abs(X).max()) if X.size else np.float32(0.0)
    return q, a


def w1_cache(W1):
    """Exact FP8 copy of W1 (not transposed: W1 [h,d] is already K-major for
    the up-projection): s_w1 = fp32(448 / max|W1|), W1q = e4m3(fp32(W1 s_w1)).
    Returns (W1q [h,d] uint8, s_w1, s_w1_inv)."""
    W = bf16_to_f64(W1)
    a = np.float32(np.abs(W).max()) if W.size else np.float32(0.0)
    s = np.float32(np.float32(E4M3_MAX) / a) if (np.isfinite(a) and a > 0) else np.float32(1.0)
    q = e4m3_bits_from_f32((W.astype(np.float32) * s).astype(np.float32))
    return q, s, np.float32(np.float32(1.0) / s)


def up_proj_fp8(x_q, W1q, s_x_inv, s_w1_inv):
    """pre = fp32( fp32(sum_k dec(x_q[m,k]) dec(W1q[i,k])) * fp32(s_x^-1 s_w1^-1) ).

    The accumulator is fp32 in the kernel; the dequantising factor is applied
    to it in the epilogue, before relu and the square."""
    comb = np.float32(np.float32(s_x_inv) * np.float32(s_w1_inv))
    acc = f32(e4m3_to_f64(x_q) @ e4m3_to_f64(W1q).T)
    return (acc * comb).astype(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# Generic FP8 linear layer (attention QKV / output projections in e4m3 in the
# forward, BF16 backward: "NanoGPT Speedrun (Track 1)", Changes vs Record #83,
# item 1).  y = x . W^T with W [N,K] (nn.Linear weight layout).
# ----------------------------------------------------------------------------


def linear_fp8(x_q, Wq, s_x_inv, s_w_inv):
    """y = bf16( fp32( fp32(sum_k dec(x_q[m,k]) dec(Wq[n,k])) * fp32(s_x^-1 s_w^-1) ) )."""
    comb = np.float32(np.float32(s_x_inv) * np.float32(s_w_inv))
    acc = f32(e4m3_to_f64(x_q) @ e4m3_to_f64(Wq).T)
    return bf16_bits_from_f32((acc * comb).astype(np.float32))


def linear_bwd(x, W, dY):
    """BF16 backward of y = x . W^T: dX = bf16(dY . W), dW = fp32(dY^T . x)."""
    G = bf16_to_f64(dY)
    return (bf16_bits_from_f32(f32(G @ bf16_to_f64(W))), f32(G.T @ bf16_to_f64(x)))


# ----------------------------------------------------------------------------
# Softcapped cross-entropy over a language-model head.
#   [RUO] item 5: a fused softcapped cross-entropy that never materialises
#         the [M,V] logits in fp32.
#   [SLOW] "A Retrospective on Our World Records", SlowRun section: one LM
#         head scored against several successive targets at each position,
#         through an FP8 soft-capped cross-entropy kernel.
#   [R83-1] "NanoGPT Speedrun (Track 1)", Changes vs Record #83, item 1: the
#         earlier record ran FP8 only in the LM head.
# Readings where the pages are silent:
#   * softcap z = c * tanh(y / c), c > 0 (a cap of the form 2c * sigmoid(y/c')
#     differs from it by a per-row constant, which cross-entropy ignores);
#   * T targets per position, weights w_t; a target outside [0, V) is ignored;
#     loss_m = sum over valid t of w_t * (logsumexp_v z[m,v] - z[m, tgt[m,t]]);
#   * reductions: the sum over rows, and the mean = sum / (sum of the valid
#     weights), 0 when no target is valid;
#   * FP8 head: y = fp32( fp32(sum_k dec(x_q) dec(Wq)) * fp32(s_x^-1 s_w^-1) ),
#     BF16 backward (straight-through over the quantisation, like the MLP);
#   * dlogits = dL/dy rounded to BF16; dX = bf16(dlogits . W),
#     dW = fp32(dlogits^T . x).
# ----------------------------------------------------------------------------


def head_logits(x, W):
    """y = x . W^T in fp64 from BF16 x [M,d] and W [V,d]."""
    return bf16_to_f64(x) @ bf16_to_f64(W).T


def head_logits_fp8(x_q, Wq, s_x_inv, s_w_inv):
    """y = fp32( fp32(sum_k dec(x_q[m,k]) dec(Wq[v,k])) * fp32(s_x^-1 s_w^-1) ), as fp64."""
    comb = np.float32(np.float32(s_x_inv) * np.float32(s_w_inv))
    acc = f32(e4m3_to_f64(x_q) @ e4m3_to_f64(Wq).T)
    return (acc * comb).astype(np.float32).astype(np.float64)


def softcap(y, c):
    """z = c tanh(y / c)."""
    return c * np.tanh(np.asarray(y, dtype=np.float64) / c)


def _ce_targets(targets, weights, V):
    """(clipped target indices [M,T], effective weights [M,T]: w_t where the
    target is in [0, V), else 0)."""
    tg = np.asarray(targets, dtype=np.int64)
    w = np.broadcast_to(np.asarray(weights, dtype=np.float64), tg.shape)
    valid = (tg >= 0) & (tg < V)
    return np.where(valid, tg, 0), np.where(valid, w, 0.0)


def ce_forward(y, targets, weights, c):
    """Loss of the softcapped logits y [M,V] (fp64) against targets [M,T].

    Returns dict(lse [M], row_loss [M], loss_sum, weight_sum, mean)."""
    y = np.asarray(y, dtype=np.float64)
    M, V = y.shape
    z = softcap(y, c)
    zmax = z.max(axis=1) if V else np.zeros(M)
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
    tg, w = _ce_targets(targets, weights, V)
    zt = np.take_along_axis(z, tg, axis=1)
    row = (w * (lse[:, None] - zt)).sum(axis=1)
    ws = float(w.sum())
    s = float(row.sum())
    return dict(lse=lse, row_loss=row, loss_sum=s, weight_sum=ws, mean=s / ws if ws > 0 else 0.0)


def ce_grad_scale(dloss, weight_sum, mean):
    """g: the factor that multiplies every row's gradient -- dloss for the
    summed loss, dloss / weight_sum for the mean (0 when no weight)."""
    if not mean:
        return float(dloss)
    return float(dloss) / weight_sum if weight_sum > 0 else 0.0


def ce_backward_dlogits(y, targets, weights, c, lse, g):
    """dL/dy [M,V] in fp64 for the loss sum_m loss_m scaled by g:
    g * (W_m softmax(z_m) - sum_t w_t onehot(tgt_t)) * (1 - tanh(y/c)^2),
    W_m = sum of row m's valid weights."""
    y = np.asarray(y, dtype=np.float64)
    M, V = y.shape
    th = np.tanh(y / c)
    p = np.exp(c * th - np.asarray(lse, dtype=np.float64)[:, None])
    tg, w = _ce_targets(targets, weights, V)
    dz = w.sum(axis=1)[:, None] * p
    for t in range(tg.shape[1]):
        np.subtract.at(dz, (np.arange(M), tg[:, t]), w[:, t])
    return g * dz * (1.0 - th * th)


def ce_backward(x, W, dlogits_f64):
    """BF16 backward through the head: dlogits = bf16(dL/dy), dX, dW."""
    dl = bf16_bits_from_f32(f32(dlogits_f64))
    dX, dW = linear_bwd(x, W, dl)
    return dl, dX, dW
