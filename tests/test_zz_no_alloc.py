"""The workspace-free W2 cache refresh against the workspace version.

fp8mlp_w2_fp8_cache_refresh_noalloc serves callers that cannot give the
library any device memory of its own -- for example an operator hook inside
another framework that owns every allocation through its own pool and offers
no workspace, or a runtime that forbids cudaMalloc/cudaFree on its hot path
because those calls can synchronise the device.  Its scratch lives in a fixed
array inside the library, shared by all calls.  This file runs last so that a
failure here does not hide the other tests; it also passes on its own.
"""
import numpy as np
import pytest
import torch

from fp8_relu_mlp_b200 import _abi as A
from fp8_relu_mlp_b200 import synth
from oracle import ref

pytestmark = pytest.mark.gpu


def _dev(W2_bits):
    return torch.from_numpy(np.ascontiguousarray(W2_bits).view(np.int16)).view(torch.bfloat16).cuda()


def _refresh_both(W2_bits, h, d):
    W2 = _dev(W2_bits)
    ref_q = torch.full((d, h), 0x55, dtype=torch.uint8, device="cuda")
    ref_inv = torch.zeros(4, device="cuda")
    ws = torch.empty(A.fp8mlp_workspace_size(0, d, h), dtype=torch.uint8, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh(h, d, W2, ref_q, ref_inv, ws)
    q = torch.full((d, h), 0xAA, dtype=torch.uint8, device="cuda")
    inv = torch.zeros(4, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, q, inv)
    torch.cuda.synchronize()
    return ref_q, ref_inv, q, inv


def _weights(h, d, seed, scale=1.0):
    W2 = synth.make_problem(1, d, h, seed=seed)["W2"]
    return synth.to_bf16_bits(ref.bf16_to_f64(W2).astype(np.float32) * np.float32(scale))


def _check(W2, h, d, call):
    ref_q, ref_inv, q, inv = _refresh_both(W2, h, d)
    # the W2 cache is compared bit for bit in every test of this suite
    assert torch.equal(q, ref_q), f"call {call}: FP8 codes differ from the workspace version"
    assert float(inv[0]) == float(ref_inv[0]), f"call {call}: scale differs from the workspace version"
    q_o, _, s_wi_o = ref.w2_cache(W2)
    assert np.array_equal(q.cpu().numpy(), q_o), f"call {call}: FP8 codes differ from the oracle"
    assert np.float32(inv[0].item()) == s_wi_o, f"call {call}: scale differs from the oracle"


@pytest.mark.parametrize("h,d", [(3072, 768), (4096, 1024), (272, 80)])
def test_noalloc_refresh_matches_workspace_version_twice(h, d):
    # two calls in a row with different weights: the shared scratch keeps the
    # first call's contents, which must not leak into the second result
    for call, scale in enumerate([1.0, 1e-3]):
        _check(_weights(h, d, 100 + call, scale), h, d, call)


def test_noalloc_smaller_call_after_a_larger_one():
    # the large call fills 512 scratch entries with maxima of order 0.1; the
    # small one (3 entries) must reduce only its own, much smaller maxima
    _check(_weights(4096, 1024, 7), 4096, 1024, 0)
    _check(_weights(272, 80, 8, 1e-3), 272, 80, 1)


def test_noalloc_zero_weights_are_flagged_like_the_workspace_version():
    h, d = 272, 80
    _check(_weights(h, d, 9), h, d, 0)  # leaves non-zero maxima in the scratch
    zeros = np.zeros((h, d), np.uint16)
    W2 = _dev(zeros)
    q = torch.full((d, h), 0xAA, dtype=torch.uint8, device="cuda")
    inv = torch.zeros(4, device="cuda")
    A.fp8mlp_clear_device_status()
    A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, q, inv)
    status = A.fp8mlp_get_device_status()
    A.fp8mlp_clear_device_status()
    assert status & A.STATUS_W2_DEGENERATE
    ref_q, ref_inv, q2, inv2 = _refresh_both(zeros, h, d)
    assert A.fp8mlp_get_device_status() & A.STATUS_W2_DEGENERATE
    A.fp8mlp_clear_device_status()
    assert float(inv[0]) == float(ref_inv[0]) == 1.0
    assert not q.any() and torch.equal(q, ref_q) and torch.equal(q2, ref_q)


def test_noalloc_refresh_allocates_nothing():
    # after a first call (which looks up the scratch's address and loads the
    # kernels), further calls change neither torch's allocator nor the
    # device's free memory
    h, d = 3072, 768
    W2 = _dev(_weights(h, d, 11))
    q = torch.empty((d, h), dtype=torch.uint8, device="cuda")
    inv = torch.zeros(4, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, q, inv)
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    reserved0 = torch.cuda.memory_reserved()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, q, inv)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert free1 == free0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    h, d = 8192, 4096  # 33.5M elements > the 16,777,216 the fixed scratch covers
    with pytest.raises(A.Fp8MlpError) as ei:
        A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, 0x10000, 0x10000, 0x10000)
    assert ei.value.code == A.ERR_UNSUPPORTED_SHAPE
    assert "scratch limit" in A.fp8mlp_last_error_detail()
