"""Parity at the full benchmark sizes, in the launch configuration bench.py
times (MLPBlock, one call per kernel), on outputs the oracle can compute one
by one: sampled token rows of the forward and of dX, sampled entries of dW1
and dW2, the full W2 cache, and properties that hold at any size.

The oracle computes its own amax and scale over the whole batch (in row
chunks); the GPU state is then set to the oracle's scale so that both sides
quantise with the same s_t.  No oracle input comes from the GPU.
"""
import numpy as np
import pytest
import torch

from fp8_relu_mlp_b200 import _abi as A
from fp8_relu_mlp_b200 import synth
from fp8_relu_mlp_b200.block import MLPBlock
from oracle import ref
from tests.gpu_util import host_bits, rel_fro, stack_errors_given_layer_inputs
from tests.test_gpu_parity import post_within_accumulation_bound

pytestmark = pytest.mark.gpu


def _oracle_amax(x, W1, chunk=2048):
    A_ = np.float32(0.0)
    for i in range(0, x.shape[0], chunk):
        A_ = max(A_, ref.amax(ref.relu2_post(ref.up_proj(x[i:i + chunk], W1))))
    return np.float32(A_)


def _sample_rows(M, n, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(M, size=n, replace=False).tolist())
    rows |= {0, M - 1, M - 128, M // 2}
    return np.array(sorted(rows))


def _load(blk, P):
    dev = blk.device
    blk.x.copy_(MLPBlock.bits_to_bf16(P["x"], dev))
    blk.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], dev))
    blk.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], dev))
    if hasattr(blk, "dOut"):
        blk.dOut.copy_(MLPBlock.bits_to_bf16(P["dOut"], dev))


def _forward_checks(blk, P, W, rows, s_o):
    """GPU forward at the oracle's scale s_o vs oracle rows."""
    A.fp8mlp_scale_state_init(blk.state, W.margin, float(s_o))
    blk.forward()
    torch.cuda.synchronize()
    W2q_o, _, s_wi = ref.w2_cache(P["W2"])
    assert np.array_equal(host_bits(blk.W2q_t), W2q_o)
    s_inv = np.float32(np.float32(1) / s_o)
    f = ref.forward_rows(rows, P["x"], P["W1"], W2q_o, s_wi, s_o, s_inv)
    idx = torch.as_tensor(rows, device=blk.post.device)
    post_g = host_bits(blk.post.index_select(0, idx))
    ok, frac = post_within_accumulation_bound(post_g, P["x"], P["W1"], rows=rows)
    assert ok and frac < 1e-2, frac
    q_g = host_bits(blk.post_fp8.index_select(0, idx))
    # the FP8 copy is the oracle's quantisation of the kernel's own post
    assert np.array_equal(q_g, ref.quantise_post(post_g, s_o))
    same = post_g == f["post"]
    assert np.array_equal(q_g[same], f["q"][same])
    out_g = ref.bf16_to_f64(host_bits(blk.out.index_select(0, idx)))
    assert rel_fro(out_g, ref.bf16_to_f64(f["out"])) < 2e-2
    # partial amax: block max of the GPU's own post, and its max is the global max
    pa = blk.partial_amax
    assert float(pa.max()) == float(blk.post.max())
    return f


@pytest.mark.parametrize("name", ["fwd16k", "step16k"])
def test_fullsize_forward_backward_sampled(name):
    W = synth.WORKLOADS[name]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0)
    blk = MLPBlock(M, d, h, margin=W.margin, with_backward=W.backward)
    _load(blk, P)
    blk.refresh_w2_cache()
    # GPU calibration vs the oracle's own amax over the whole batch
    blk.calibrate()
    torch.cuda.synchronize()
    A_o = _oracle_amax(P["x"], P["W1"])
    st_o = ref.scale_update(ref.scale_state_init(W.margin, 1.0), A_o)
    g = blk.read_state()
    assert abs(g["amax_prev"] / float(A_o) - 1) <= 2.0 ** -7
    assert abs(g["scale"] / float(st_o["scale"]) - 1) <= 2.0 ** -7
    rows = _sample_rows(M, 48, seed=1)
    _forward_checks(blk, P, W, rows, st_o["scale"])
    assert A.fp8mlp_get_device_status() == 0
    if not W.backward:
        return
    blk.backward()
    torch.cuda.synchronize()
    dPre_o, dX_o = ref.dx_rows(rows, P["x"], P["W1"], P["W2"], P["dOut"])
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dPre)[rows]), ref.bf16_to_f64(dPre_o)) < 1e-2
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dX)[rows]), ref.bf16_to_f64(dX_o)) < 1e-2
    gen = np.random.default_rng(2)
    pairs = [(int(i), int(j)) for i, j in zip(gen.integers(0, h, 12), gen.integers(0, d, 12))]
    pairs += [(h - 1, d - 1), (0, 0)]
    w1_o, w2_o = ref.dw_entries(pairs, P["x"], P["W1"], P["W2"], P["dOut"])
    dW1, dW2 = host_bits(blk.dW1), host_bits(blk.dW2)
    w1_g = np.array([dW1[i, j] for i, j in pairs])
    w2_g = np.array([dW2[i, j] for i, j in pairs])
    assert rel_fro(w1_g, w1_o) < 1e-2
    assert rel_fro(w2_g, w2_o) < 1e-2
    assert A.fp8mlp_get_device_status() == 0


def test_train49k_steps_sampled():
    """Three steps of the M=49152 train workload: perturbed weights, W2 cache
    refreshed per step, delayed scale tracked against the oracle's."""
    W = synth.WORKLOADS["train49k"]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0)
    blk = MLPBlock(M, d, h, margin=W.margin)
    _load(blk, P)
    blk.refresh_w2_cache()
    blk.calibrate()
    o = ref.scale_update(ref.scale_state_init(W.margin, 1.0), _oracle_amax(P["x"], P["W1"]))
    steps = 3
    for step in range(steps):
        blk.train_step()
        A_o = _oracle_amax(P["x"], P["W1"])
        o = ref.scale_update(o, A_o)
        g = blk.read_state()
        assert abs(g["scale"] / float(o["scale"]) - 1) <= 2.0 ** -7
        # optimizer stand-in: perturb the weights, refresh the W2 cache
        P["W1"] = synth.perturb(P["W1"], 0, step, W.perturb_var, "W1")
        P["W2"] = synth.perturb(P["W2"], 0, step, W.perturb_var, "W2")
        _load(blk, P)
        blk.refresh_w2_cache()
    rows = _sample_rows(M, 32, seed=3)
    _forward_checks(blk, P, W, rows, o["scale"])
    blk.backward()
    torch.cuda.synchronize()
    _, dX_o = ref.dx_rows(rows, P["x"], P["W1"], P["W2"], P["dOut"])
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dX)[rows]), ref.bf16_to_f64(dX_o)) < 1e-2
    pairs = [(5, 7), (h - 1, 3), (1000, d - 1), (2048, 100)]
    w1_o, w2_o = ref.dw_entries(pairs, P["x"], P["W1"], P["W2"], P["dOut"])
    dW1, dW2 = host_bits(blk.dW1), host_bits(blk.dW2)
    assert rel_fro(np.array([dW1[i, j] for i, j in pairs]), w1_o) < 1e-2
    assert rel_fro(np.array([dW2[i, j] for i, j in pairs]), w2_o) < 1e-2
    assert A.fp8mlp_get_device_status() == 0


def test_heavytail_spike_saturates_and_matches():
    """M=65536, d=1024, h=4096, Student-t(3) inputs: with the delayed scale of
    the previous (normal) step, the 2x spike step saturates the FP8 copy; both
    sides saturate the same elements."""
    W = synth.WORKLOADS["heavytail"]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0, x_dist=W.x_dist)
    blk = MLPBlock(M, d, h, margin=W.margin)
    _load(blk, P)
    blk.refresh_w2_cache()
    blk.calibrate()
    torch.cuda.synchronize()
    A_o = _oracle_amax(P["x"], P["W1"])
    s_o = ref.scale_update(ref.scale_state_init(W.margin, 1.0), A_o)["scale"]
    assert abs(blk.read_state()["scale"] / float(s_o) - 1) <= 2.0 ** -7
    # spike step: x * 2 (post * 4) quantised with the scale of the normal step
    xs = synth.to_bf16_bits(ref.bf16_to_f64(P["x"]).astype(np.float32) * W.spike_factor)
    P2 = dict(P, x=xs)
    _load(blk, P2)
    rows = _sample_rows(M, 32, seed=4)
    f = _forward_checks(blk, P2, W, rows, s_o)
    sat_g = float(((blk.post_fp8 & 0x7F) == 0x7E).float().mean())
    assert sat_g > 0
    assert np.array_equal((f["q"] & 0x7F) == 0x7E, (host_bits(blk.post_fp8)[rows] & 0x7F) == 0x7E) or \
        np.mean(((f["q"] & 0x7F) == 0x7E) != ((host_bits(blk.post_fp8)[rows] & 0x7F) == 0x7E)) < 1e-4
    # the next scale follows the spike's amax
    blk.update_scale()
    A_spike = _oracle_amax(xs, P["W1"])
    assert abs(blk.read_state()["amax_prev"] / float(A_spike) - 1) <= 2.0 ** -7


def test_fullsize_fp8_up_overlapped_step_sampled():
    """The e4m3 up-projection at the benchmark's size (bench.py --fp8-up,
    M=16384), through the overlapped training step the benchmark times: the
    x-scale bit-exact from the oracle's own max |x|, the W1 cache and the x
    codes bit-exact, sampled rows of post, out and dX against the oracle's
    same FP8 pipeline (the BF16 backward of its own post)."""
    W = synth.WORKLOADS["step16k"]
    M, d, h = W.M, W.d, W.h
    P = synth.make_problem(M, d, h, seed=0)
    blk = MLPBlock(M, d, h, margin=W.margin, fp8_up=True)
    _load(blk, P)
    blk.refresh_w2_cache()
    blk.refresh_w1_cache()
    blk.calibrate()
    torch.cuda.synchronize()
    ax = np.float32(np.abs(ref.bf16_to_f64(P["x"])).max())
    st_x = ref.scale_update(ref.scale_state_init(W.margin, 1.0), ax)
    assert np.float32(blk.read_state(blk.state_x)["scale"]) == st_x["scale"]
    W1q_o, _, s_w1i = ref.w1_cache(P["W1"])
    assert np.array_equal(host_bits(blk.W1q), W1q_o)
    # the step at a known post scale
    s_o = np.float32(448.0 / 50.0)
    A.fp8mlp_scale_state_init(blk.state, W.margin, float(s_o))
    side = torch.cuda.Stream()
    blk.train_step_overlapped(side)
    torch.cuda.synchronize()
    rows = _sample_rows(M, 48, seed=3)
    xq_o, _ = ref.quantise_x(P["x"][rows], st_x["scale"])
    assert np.array_equal(host_bits(blk.x_fp8)[rows], xq_o)
    post_o = ref.relu2_post(ref.up_proj_fp8(xq_o, W1q_o, st_x["scale_inv"], s_w1i))
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.post)[rows]), ref.bf16_to_f64(post_o)) < 1e-2
    W2q_o, _, s_w2i = ref.w2_cache(P["W2"])
    out_o = ref.down_proj_fp8(ref.quantise_post(post_o, s_o), W2q_o, np.float32(np.float32(1) / s_o), s_w2i)
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.out)[rows]), ref.bf16_to_f64(out_o)) < 2e-2
    # the BF16 backward of the kernel's own post (the straight-through
    # gradient of this layer given its inputs) within the gradient bound
    post_g = host_bits(blk.post)[rows]
    dPre_g = ref.bwd_dpre(post_g, P["dOut"][rows], P["W2"])
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dX)[rows]), ref.bf16_to_f64(ref.bwd_dx(dPre_g, P["W1"]))) < 1e-2
    # end to end, the oracle's backward of its own post (from its e4m3
    # up-projection): the FP8 forward's bound
    dPre_o = ref.bwd_dpre(post_o, P["dOut"][rows], P["W2"])
    dX_o = ref.bwd_dx(dPre_o, P["W1"])
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dX)[rows]), ref.bf16_to_f64(dX_o)) < 2e-2
    assert A.fp8mlp_get_device_status() == 0


@pytest.mark.parametrize("fp8_up", [False, True])
def test_stack9_fullsize_sampled_rows(fp8_up):
    """The 9-layer stack at the benchmark's size (M=131072), in the launch
    configuration bench.py times.  With every layer's delayed scales fixed
    the stack is row-wise independent (RMSNorm, the MLP and the residual act
    per token), so the oracle runs sampled rows through all nine layers,
    forward (r_L) and backward (dL/dr_0)."""
    from fp8_relu_mlp_b200.block import MLPStack
    W = synth.WORKLOADS["stack9"]
    L, M, d, h = W.layers, W.M, W.d, W.h
    g = synth.rng(1000)
    r0 = synth.to_bf16_bits(synth.make_x(g, M, d, "normal"))
    dtop = synth.to_bf16_bits(synth.make_x(g, M, d, "normal"))
    S = MLPStack(L, M, d, h, margin=W.margin, fp8_up=fp8_up)
    layers, scales, xsc = [], [], []
    for l, b in enumerate(S.blocks):
        P = synth.make_problem(1, d, h, seed=100 + l)
        b.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], b.device))
        b.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], b.device))
        W2q_t, _, s_wi = ref.w2_cache(P["W2"])
        lay = dict(W1=P["W1"], W2=P["W2"], W2q_t=W2q_t, w2_scale_inv=s_wi)
        s = np.float32(448.0 / (2.0 * (20.0 + 3 * l)))
        A.fp8mlp_scale_state_init(b.state, W.margin, float(s))
        scales.append((s, np.float32(np.float32(1) / s)))
        if fp8_up:
            lay["W1q"], _, lay["w1_scale_inv"] = ref.w1_cache(P["W1"])
            sx = np.float32(448.0 / (2.0 * 5.0))
            A.fp8mlp_scale_state_init(b.state_x, W.margin, float(sx))
            xsc.append((sx, np.float32(np.float32(1) / sx)))
        layers.append(lay)
    S.refresh_w2_caches()
    S.r[0].copy_(MLPBlock.bits_to_bf16(r0, S.device))
    S.forward()
    S.dr.copy_(MLPBlock.bits_to_bf16(dtop, S.device))
    S.backward()
    torch.cuda.synchronize()
    rows = _sample_rows(M, 24, seed=5)
    if fp8_up:
        saved, rL = ref.stack_forward_fp8up(r0[rows], layers, scales, xsc)
    else:
        saved, rL = ref.stack_forward(r0[rows], layers, scales)
    dr0, _ = ref.stack_backward(saved, layers, dtop[rows])
    # each layer given its own inputs: FP8 codes bit for bit, out and the
    # gradients within the single-kernel bounds
    e = stack_errors_given_layer_inputs(S, layers, scales, dtop, rows=rows)
    assert e["q_mismatch"] == 0 and e["out"] < 4e-3, e
    assert e["dX"] < 1e-2 and e["dr0"] < 1e-2, e
    # end to end against the oracle's own stack: the FP8 forward's bound
    assert rel_fro(ref.bf16_to_f64(host_bits(S.r[L])[rows]), ref.bf16_to_f64(rL)) < 2e-2
    assert rel_fro(ref.bf16_to_f64(host_bits(S.dr)[rows]), ref.bf16_to_f64(dr0)) < 2e-2
    assert A.fp8mlp_get_device_status() == 0


def test_batch_past_2_31_elements_sampled():
    """M = 704512 tokens at d = 768, h = 3072: post and dPre hold 2.16e9
    elements, so the rows from 699051 on sit past element 2^31 and every
    offset into them needs 64-bit arithmetic.  Forward rows (at a scale the
    oracle takes from the sampled rows; any s_t serves when both sides use
    it) and backward rows against the oracle; dX and out past 2^31 bytes too.

    The token rows repeat with a period of 16381 rows (a prime: no tile
    boundary and no 2^32-byte wrap maps a row onto a copy of itself), so the
    inputs are drawn in seconds; the oracle takes the sampled rows' own
    values.  post and dPre are filled with NaN first, so an element left
    unwritten shows."""
    M, d, h = 704512, 768, 3072
    assert M * h > 2 ** 31
    period = 16381
    P = synth.make_problem(period, d, h, seed=5)
    reps = -(-M // period)
    for k in ("x", "dOut"):
        P[k] = np.ascontiguousarray(np.tile(P[k], (reps, 1))[:M])
    blk = MLPBlock(M, d, h, margin=2.0, with_backward=True)
    _load(blk, P)
    blk.refresh_w2_cache()
    rows = np.array(sorted(set(_sample_rows(M, 24, seed=3).tolist()) | {699050, 699051, 699052}))
    A_rows = ref.amax(ref.relu2_post(ref.up_proj(P["x"][rows], P["W1"])))
    st_o = ref.scale_update(ref.scale_state_init(2.0, 1.0), A_rows)

    class _W:
        margin = 2.0

    blk.post.fill_(float("nan"))
    blk.dPre.fill_(float("nan"))
    _forward_checks(blk, P, _W, rows, st_o["scale"])
    assert A.fp8mlp_get_device_status() == 0
    blk.backward()
    torch.cuda.synchronize()
    idx = torch.as_tensor(rows, device=blk.dPre.device)
    dPre_o, dX_o = ref.dx_rows(rows, P["x"], P["W1"], P["W2"], P["dOut"])
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dPre.index_select(0, idx))), ref.bf16_to_f64(dPre_o)) < 1e-2
    assert rel_fro(ref.bf16_to_f64(host_bits(blk.dX.index_select(0, idx))), ref.bf16_to_f64(dX_o)) < 1e-2
    # every element past 2^31 was written
    assert not bool(blk.post[699050:].isnan().any())
    assert not bool(blk.dPre[699050:].isnan().any())
    assert A.fp8mlp_get_device_status() == 0
