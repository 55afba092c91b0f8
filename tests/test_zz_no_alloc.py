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

pytestmark = pytest.mark.gpu


def _refresh_both(W2_bits, h, d):
    W2 = torch.from_numpy(W2_bits.view(np.int16)).view(torch.bfloat16).cuda()
    ref_q = torch.full((d, h), 0x55, dtype=torch.uint8, device="cuda")
    ref_inv = torch.zeros(4, device="cuda")
    ws = torch.empty(A.fp8mlp_workspace_size(0, d, h), dtype=torch.uint8, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh(h, d, W2, ref_q, ref_inv, ws)
    q = torch.full((d, h), 0xAA, dtype=torch.uint8, device="cuda")
    inv = torch.zeros(4, device="cuda")
    A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, W2, q, inv)
    torch.cuda.synchronize()
    return ref_q, ref_inv, q, inv


@pytest.mark.parametrize("h,d", [(3072, 768), (4096, 1024), (272, 80)])
def test_noalloc_refresh_matches_workspace_version_twice(h, d):
    # two calls in a row with different weights: the shared scratch keeps the
    # first call's contents, which must not leak into the second result
    for call, scale in enumerate([1.0, 1e-3]):
        W2 = synth.make_problem(1, d, h, seed=100 + call)["W2"]
        W2 = synth.to_bf16_bits(torch.from_numpy(W2.view(np.int16)).view(torch.bfloat16).float().numpy() * scale)
        ref_q, ref_inv, q, inv = _refresh_both(W2, h, d)
        # the W2 cache is compared bit for bit in every test of this suite
        assert torch.equal(q, ref_q), f"call {call}: FP8 codes differ"
        assert float(inv[0]) == float(ref_inv[0]), f"call {call}: scale differs"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    h, d = 8192, 4096  # 33.5M elements > the 16,777,216 the fixed scratch covers
    with pytest.raises(A.Fp8MlpError) as ei:
        A.fp8mlp_w2_fp8_cache_refresh_noalloc(h, d, 0x10000, 0x10000, 0x10000)
    assert ei.value.code == A.ERR_UNSUPPORTED_SHAPE
    assert "scratch limit" in A.fp8mlp_last_error_detail()
