"""Helpers for the GPU parity tests: device transfers of bit patterns, guarded
output buffers (canaries around every output), and error norms."""
import numpy as np
import torch

CANARY_BYTES = 4096


def dev_bf16(bits):
    """numpy uint16 BF16 bits -> contiguous torch.bfloat16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_bits(t):
    """torch bf16 / uint8 / fp32 tensor -> numpy (uint16 bits for bf16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class Guarded:
    """An output tensor with CANARY_BYTES of a fixed pattern on both sides."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) if len(shape) else 1
        esz = torch.empty(0, dtype=dtype).element_size()
        nbytes = n * esz
        self.raw = torch.empty(2 * CANARY_BYTES + ((nbytes + 255) // 256) * 256, dtype=torch.uint8, device="cuda")
        self.raw.fill_(0xA5)
        self.lo = CANARY_BYTES
        self.hi = CANARY_BYTES + nbytes
        self.t = self.raw[self.lo:self.hi].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool((r[:self.lo] == 0xA5).all() and (r[self.hi:] == 0xA5).all())


def rel_fro(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def bf16_ulps(a_bits, b_bits):
    """Distance in representable BF16 steps between two arrays of
    non-negative BF16 bit patterns (ordering of the bit patterns)."""
    return np.abs(a_bits.astype(np.int64) - b_bits.astype(np.int64))


def stack_errors_given_layer_inputs(S, layers, scales, dtop, rows=None):
    """Relative errors of each layer of a layer stack (``MLPStack`` after its
    forward and backward) against the oracle given that layer's own inputs.

    For layer l the inputs are the GPU's x_l and post_l and the residual
    gradient dL/dr_{l+1} that reached it.  The GPU updates that gradient in
    place, so it is rebuilt here from the top gradient ``dtop`` and the GPU's
    dX of the layers above with the oracle's residual step (dr_l = bf16(dr_{l+1}
    + rmsnorm_bwd(r_l, dX_l))).  Then:
      out_l  vs the oracle's FP8 down-projection of the GPU's post_l (its codes
             bit for bit, the product within accumulation);
      dX_l, dW1_l, dW2_l vs the oracle's backward of (x_l, post_l, dr_{l+1});
      dL/dr_0 vs the oracle's residual step on the GPU's dX_0.
    ``rows`` restricts everything to sampled token rows (then dW, which needs
    every token, is not compared).  Returns {name: max over layers}."""
    from oracle import ref
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])

    def g(t):
        if rows is None:
            return host_bits(t)
        return host_bits(t.index_select(0, torch.as_tensor(rows, device=t.device)))

    L = len(layers)
    err = {"out": 0.0, "q_mismatch": 0, "dX": 0.0, "dW1": 0.0, "dW2": 0.0, "dr0": 0.0}
    dr = sel(dtop)
    for l in range(L - 1, -1, -1):
        b, lay = S.blocks[l], layers[l]
        s, si = scales[l]
        x_l, post_l = g(b.x), g(b.post)
        q_o = ref.quantise_post(post_l, s)
        err["q_mismatch"] += int((g(b.post_fp8) != q_o).sum())
        out_o = ref.down_proj_fp8(q_o, lay["W2q_t"], si, lay["w2_scale_inv"])
        err["out"] = max(err["out"], rel_fro(ref.bf16_to_f64(g(b.out)), ref.bf16_to_f64(out_o)))
        dPre_o = ref.bwd_dpre(post_l, dr, lay["W2"])
        dX_o = ref.bwd_dx(dPre_o, lay["W1"])
        dX_g = g(b.dX)
        err["dX"] = max(err["dX"], rel_fro(ref.bf16_to_f64(dX_g), ref.bf16_to_f64(dX_o)))
        if rows is None:
            err["dW1"] = max(err["dW1"], rel_fro(host_bits(b.dW1), ref.bwd_dw1(dPre_o, x_l)))
            err["dW2"] = max(err["dW2"], rel_fro(host_bits(b.dW2), ref.bwd_dw2(post_l, dr)))
        drn = ref.rmsnorm_bwd(g(S.r[l]), dX_g)
        dr = ref.bf16_bits_from_f32(ref.f32(ref.bf16_to_f64(dr) + drn))
    err["dr0"] = rel_fro(ref.bf16_to_f64(g(S.dr)), ref.bf16_to_f64(dr))
    return err
