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
