"""One fused FP8 ReLU^2 MLP block: device buffers plus the call sequence.

Torch is used only to allocate device memory and to name the stream; every
step runs in libfp8mlp's kernels through the C ABI (:mod:`._abi`).

Training step at step t ("A Retrospective on Our World Records", Modded-NanoGPT
Main Track):
    forward      fused up-projection (post, FP8 copy under s_t, partial amax)
                 + FP8 down-projection against the transposed W2 cache
    backward     dPre = 2 sqrt(post) dPost, then dX, dW1, dW2 (BF16)
    scale        reduce the partial amax -> s_{t+1}
    (optimizer)  caller updates W1 / W2
    W2 cache     refreshed after the update
"""
from __future__ import annotations

import torch

from . import _abi as A


class MLPBlock:
    def __init__(self, M: int, d: int, h: int, device="cuda", margin: float = 2.0, initial_scale: float = 1.0,
                 with_backward: bool = True, stream=None, fp8_up: bool = False):
        """``fp8_up``: run the up-projection on e4m3 copies of x (delayed scale
        of its own) and W1 (exact cache scale) as well; the backward keeps the
        BF16 x and W1."""
        self.M, self.d, self.h = M, d, h
        self.fp8_up = fp8_up
        self.device = torch.device(device)
        self.stream = stream
        dev = self.device
        bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
        self.x = torch.zeros(M, d, dtype=bf, device=dev)
        self.W1 = torch.zeros(h, d, dtype=bf, device=dev)
        self.W2 = torch.zeros(h, d, dtype=bf, device=dev)
        self.W2q_t = torch.zeros(d, h, dtype=u8, device=dev)
        self.w2_scale_inv = torch.ones(4, dtype=f32, device=dev)
        self.state = torch.zeros(8, dtype=f32, device=dev)  # fp8mlp_scale_state (32 bytes)
        self.post = torch.empty(M, h, dtype=bf, device=dev)
        self.post_fp8 = torch.empty(M, h, dtype=u8, device=dev)
        rb, cb, _, _ = A.fp8mlp_partial_amax_shape(M, h)
        self.partial_amax = torch.zeros(rb, cb, dtype=f32, device=dev)
        self.out = torch.empty(M, d, dtype=bf, device=dev)
        self.workspace = torch.zeros(max(256, A.fp8mlp_workspace_size(M, d, h)), dtype=u8, device=dev)
        if with_backward:
            self.dOut = torch.zeros(M, d, dtype=bf, device=dev)
            self.dPre = torch.empty(M, h, dtype=bf, device=dev)
            self.dX = torch.empty(M, d, dtype=bf, device=dev)
            self.dW1 = torch.empty(h, d, dtype=f32, device=dev)
            self.dW2 = torch.empty(h, d, dtype=f32, device=dev)
        A.fp8mlp_scale_state_init(self.state, margin, initial_scale, self.stream)
        if fp8_up:
            self.x_fp8 = torch.empty(M, d, dtype=u8, device=dev)
            self.W1q = torch.zeros(h, d, dtype=u8, device=dev)
            self.w1_scale_inv = torch.ones(4, dtype=f32, device=dev)
            self.state_x = torch.zeros(8, dtype=f32, device=dev)
            self.partial_amax_x = torch.zeros(max(1, A.fp8mlp_x_partial_amax_count(M, d)), dtype=f32, device=dev)
            A.fp8mlp_scale_state_init(self.state_x, margin, initial_scale, self.stream)

    # ------------------------------------------------------------------ calls
    def refresh_w1_cache(self):
        A.fp8mlp_w1_fp8_cache_refresh(self.h, self.d, self.W1, self.W1q, self.w1_scale_inv, self.workspace,
                                      self.stream)

    def _quantize_x(self):
        A.fp8mlp_quantize_x(self.M, self.d, self.x, self.state_x, self.x_fp8, self.partial_amax_x, self.stream)

    def _update_x_scale(self):
        A.fp8mlp_amax_reduce_update_scale(self.partial_amax_x, A.fp8mlp_x_partial_amax_count(self.M, self.d),
                                          self.state_x, self.stream)

    def _up_fp8(self, flags):
        A.fp8mlp_up_proj_fused_fp8(self.M, self.d, self.h, self.x_fp8, self.W1q, self.w1_scale_inv, self.state_x,
                                   self.state, self.post, self.post_fp8 if flags == 0 else None,
                                   self.partial_amax, None, flags, self.stream)
    def refresh_w2_cache(self):
        A.fp8mlp_w2_fp8_cache_refresh(self.h, self.d, self.W2, self.W2q_t, self.w2_scale_inv, self.workspace,
                                      self.stream)

    def calibrate(self):
        """Step 0: post and partial amax only, then the first scale (with the
        FP8 up-projection, first the x-scale from x's own amax)."""
        if self.fp8_up:
            self._quantize_x()
            self._update_x_scale()
            self._quantize_x()
            self._up_fp8(A.FWD_CALIBRATE)
            A.fp8mlp_amax_reduce_update_scale(self.partial_amax, self.partial_amax.numel(), self.state, self.stream)
            return
        A.fp8mlp_mlp_fwd(self.M, self.d, self.h, self.x, self.W1, None, None, None, self.state, self.post, None,
                         self.partial_amax, None, None, A.FWD_CALIBRATE, self.stream)
        self.update_scale()

    def forward(self, eval_bf16: bool = False, pre_debug=None):
        if self.fp8_up and not eval_bf16:
            self._quantize_x()
            self._up_fp8(0)
            A.fp8mlp_down_proj_fp8(self.M, self.d, self.h, self.post_fp8, self.W2q_t, self.w2_scale_inv, self.state,
                                   self.out, self.stream)
            return
        flags = A.FWD_EVAL_BF16 if eval_bf16 else 0
        A.fp8mlp_mlp_fwd(self.M, self.d, self.h, self.x, self.W1, self.W2q_t, self.w2_scale_inv, self.W2,
                         self.state, self.post, None if eval_bf16 else self.post_fp8, self.partial_amax, self.out,
                         pre_debug, flags, self.stream)

    def update_scale(self):
        A.fp8mlp_amax_reduce_update_scale(self.partial_amax, self.partial_amax.numel(), self.state, self.stream)
        if self.fp8_up:
            self._update_x_scale()

    def backward(self):
        A.fp8mlp_mlp_bwd(self.M, self.d, self.h, self.x, self.W1, self.W2, self.post, self.dOut, self.dPre,
                         self.dX, self.dW1, self.dW2, self.stream)

    def train_step(self):
        """forward at s_t, backward, s_{t+1}; the caller's optimizer then
        updates W1/W2 and calls refresh_w2_cache()."""
        self.forward()
        self.backward()
        self.update_scale()

    def train_step_overlapped(self, side, refresh_w2: bool = True, mark=None):
        """One training step with the small launches off the critical path.

        ``side`` is a second CUDA stream.  The W2 cache refresh (from the
        current W2: call this after the optimizer's update) runs on ``side``
        beside the up-projection, which does not read the cache, and is joined
        before the down-projection; the delayed-scale update runs on ``side``
        beside the dX and dW GEMMs, which do not read the scale, and is joined
        at the end.  dPre and dW are launched with
        ``LAUNCH_OVERLAP_PREVIOUS`` (each reads nothing the GEMM before it
        writes).  The calls and their results are those of
        ``refresh_w2_cache(); train_step()``.  With the FP8 up-projection the
        W1 cache refresh (the same workspace) stays on the main stream, first.
        ``mark(i)``, if given, is called on the main stream at 0 (start), after
        the up-projection (1), the down-projection (2), dPre (3), dX (4), dW
        (5), and at the end (7)."""
        mark = mark or (lambda i: None)
        M, d, h = self.M, self.d, self.h
        main = torch.cuda.current_stream(self.device) if self.stream is None else self.stream
        mark(0)
        if self.fp8_up:
            self.refresh_w1_cache()
        if refresh_w2:
            side.wait_stream(main)
            with torch.cuda.stream(side):
                A.fp8mlp_w2_fp8_cache_refresh(h, d, self.W2, self.W2q_t, self.w2_scale_inv, self.workspace, side)
        if self.fp8_up:
            self._quantize_x()
            self._up_fp8(0)
        else:
            A.fp8mlp_up_proj_fused(M, d, h, self.x, self.W1, self.state, self.post, self.post_fp8, self.partial_amax,
                                   None, 0, self.stream)
        mark(1)
        if refresh_w2:
            main.wait_stream(side)
        A.fp8mlp_down_proj_fp8(M, d, h, self.post_fp8, self.W2q_t, self.w2_scale_inv, self.state, self.out,
                               self.stream)
        mark(2)
        # dPre does not read the down-projection's output: it may start while
        # that GEMM finishes its last wave (likewise dW after dX)
        A.fp8mlp_bwd_dpre(M, d, h, self.dOut, self.W2, self.post, self.dPre, A.LAUNCH_OVERLAP_PREVIOUS, self.stream)
        mark(3)
        side.wait_stream(main)
        with torch.cuda.stream(side):
            A.fp8mlp_amax_reduce_update_scale(self.partial_amax, self.partial_amax.numel(), self.state, side)
            if self.fp8_up:
                A.fp8mlp_amax_reduce_update_scale(self.partial_amax_x, A.fp8mlp_x_partial_amax_count(M, d),
                                                  self.state_x, side)
        A.fp8mlp_bwd_dx(M, d, h, self.dPre, self.W1, self.dX, self.stream)
        mark(4)
        A.fp8mlp_bwd_dw(M, d, h, self.x, self.dPre, self.post, self.dOut, self.dW1, self.dW2,
                        A.LAUNCH_OVERLAP_PREVIOUS, self.stream)
        mark(5)
        main.wait_stream(side)
        mark(7)

    def train_step_native(self):
        """``refresh_w2_cache(); train_step()`` as one library call with the
        schedule of ``train_step_overlapped`` built into the library
        (``fp8mlp_mlp_train_step``: its own second stream for the cache
        refresh and the scale update, dPre and dW started in the previous
        GEMM's last wave); the same results, bit for bit.  BF16 up-projection
        only."""
        if self.fp8_up:
            raise ValueError("the library's training step runs the BF16 up-projection; use train_step_overlapped")
        A.fp8mlp_mlp_train_step(self.M, self.d, self.h, self.x, self.W1, self.W2, self.dOut, self.W2q_t,
                                self.w2_scale_inv, self.state, self.post, self.post_fp8, self.partial_amax, self.out,
                                self.dPre, self.dX, self.dW1, self.dW2, self.workspace, self.stream)

    # ------------------------------------------------------------ CUDA graph
    def capture(self, fn):
        """Record the library calls made by ``fn()`` into a CUDA graph and return
        it (``torch.cuda.CUDAGraph``; ``.replay()`` re-issues them).  The calls
        bake this block's buffer addresses into the graph, so the buffers must
        stay alive and in place.  Run ``fn()`` once eagerly before capturing."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    # --------------------------------------------------------------- helpers
    def read_state(self, state=None) -> dict:
        s = (self.state if state is None else state).cpu()
        i = s.view(torch.int32)
        return dict(amax_prev=float(s[0]), scale=float(s[1]), scale_inv=float(s[2]), margin=float(s[3]),
                    step=int(i[4]), flags=int(i[5]))

    @staticmethod
    def bits_to_bf16(a, device):
        """numpy uint16 BF16 bit patterns -> torch bf16 device tensor."""
        import numpy as np
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


class MLPStack:
    """L residual layers of ``r_{l+1} = r_l + MLP_l(RMSNorm(r_l))`` (the 9-layer,
    768-dim ReLU^2 stacks of the nanochat runs), forward and backward, all
    through the C ABI.  Each layer keeps its own block buffers (post, x, its
    delayed-scale state and W2 cache); the residual stream r_l and the RMSNorm
    statistics are kept per layer for the backward.

    ``fp8_up``: every up-projection runs on e4m3 copies of x and W1; the
    RMSNorm kernel writes x's copy under the layer's delayed x-scale and the
    per-row max |x| that drives the next one (fp8mlp_rmsnorm_fwd_quant), so
    x is read once.  The backward keeps the BF16 x and W1."""

    def __init__(self, L: int, M: int, d: int, h: int, device="cuda", margin: float = 2.0,
                 initial_scale: float = 1.0, stream=None, fp8_up: bool = False):
        self.L, self.M, self.d, self.h = L, M, d, h
        self.fp8_up = fp8_up
        self.device = torch.device(device)
        self.stream = stream
        self.blocks = [MLPBlock(M, d, h, device, margin, initial_scale, stream=stream, fp8_up=fp8_up)
                       for _ in range(L)]
        self.r = [torch.zeros(M, d, dtype=torch.bfloat16, device=self.device) for _ in range(L + 1)]
        self.rstd = [torch.empty(M, dtype=torch.float32, device=self.device) for _ in range(L)]
        self.dr = torch.zeros(M, d, dtype=torch.bfloat16, device=self.device)
        if fp8_up:
            self.row_amax = [torch.zeros(max(M, 1), dtype=torch.float32, device=self.device) for _ in range(L)]

    def refresh_w2_caches(self):
        """The FP8 weight caches from the current weights (after the optimizer):
        W2 of every layer, and W1 with ``fp8_up``."""
        for b in self.blocks:
            b.refresh_w2_cache()
            if self.fp8_up:
                b.refresh_w1_cache()

    def _norm(self, l):
        b = self.blocks[l]
        if self.fp8_up:
            A.fp8mlp_rmsnorm_fwd_quant(self.M, self.d, self.r[l], b.x, self.rstd[l], b.state_x, b.x_fp8,
                                       self.row_amax[l], self.stream)
        else:
            A.fp8mlp_rmsnorm_fwd(self.M, self.d, self.r[l], b.x, self.rstd[l], self.stream)

    def _update_x_scale(self, l):
        A.fp8mlp_amax_reduce_update_scale(self.row_amax[l], self.M, self.blocks[l].state_x, self.stream)

    def _block_forward(self, b):
        if self.fp8_up:
            b._up_fp8(0)
            A.fp8mlp_down_proj_fp8(self.M, self.d, self.h, b.post_fp8, b.W2q_t, b.w2_scale_inv, b.state, b.out,
                                   self.stream)
        else:
            b.forward()

    def calibrate(self):
        for l, b in enumerate(self.blocks):
            self._norm(l)
            if self.fp8_up:
                # first the x-scale from x's own amax, then post's scale
                self._update_x_scale(l)
                self._norm(l)
                b._up_fp8(A.FWD_CALIBRATE)
                A.fp8mlp_amax_reduce_update_scale(b.partial_amax, b.partial_amax.numel(), b.state, self.stream)
            else:
                b.calibrate()
            self._block_forward(b)
            A.fp8mlp_residual_add(self.M, self.d, self.r[l], b.out, self.r[l + 1], self.stream)

    def forward(self):
        for l, b in enumerate(self.blocks):
            self._norm(l)
            self._block_forward(b)
            A.fp8mlp_residual_add(self.M, self.d, self.r[l], b.out, self.r[l + 1], self.stream)

    def backward(self):
        """``self.dr`` holds dL/dr_L on entry and dL/dr_0 on exit."""
        M, d, h = self.M, self.d, self.h
        for l in range(self.L - 1, -1, -1):
            b = self.blocks[l]
            A.fp8mlp_mlp_bwd(M, d, h, b.x, b.W1, b.W2, b.post, self.dr, b.dPre, b.dX, b.dW1, b.dW2, self.stream)
            A.fp8mlp_rmsnorm_bwd(M, d, self.r[l], self.rstd[l], b.dX, self.dr, self.dr, self.stream)

    def update_scales(self):
        for l, b in enumerate(self.blocks):
            A.fp8mlp_amax_reduce_update_scale(b.partial_amax, b.partial_amax.numel(), b.state, self.stream)
            if self.fp8_up:
                self._update_x_scale(l)
