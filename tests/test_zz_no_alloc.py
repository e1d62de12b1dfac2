"""svdq_linear_forward_noalloc: the forward pass for callers that cannot
allocate device memory when they run the layer (hosts that hand a kernel only
its inputs and outputs, and loops where a cudaMalloc, which can block on work
already queued, is not allowed).  It keeps its intermediates in one fixed
library-owned array per device instead of a caller workspace.

Checked through the C ABI against svdq_linear_forward (caller workspace) on the
same layer and inputs, for two calls in a row: the second call has a different
x and a smaller M, so any stale contents the first call leaves in the shared
array would show up in its result.  Both entry points run the same kernels with
the same M (the same kernel choice and summation order), so the outputs must be
bit-identical; the first call is also held to the CPU oracle's tolerance.  This
file is named to be collected last and also passes when run alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import bit_quantized_linear_svdq_b200 as S
from bit_quantized_linear_svdq_b200 import synthetic as syn
from oracle import svdq_oracle as O

pytestmark = pytest.mark.gpu

# Output tolerance used by the GPU parity tests.
Y_REL_FRO = 5e-3
Y_MAX_REL = 1e-2


def _layer(ck):
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.uint8)).cuda()
    bf = _bf16
    return S.SVDQLinear(u8(ck.qweight), u8(ck.wscales), bf(ck.proj_down), bf(ck.proj_up), bf(ck.smooth_factor),
                        bf(ck.wcscales), bf(ck.wtscale), rotate_block=ck.rotate_block)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _x(ck):
    return _bf16(ck.x)


def _assert_y_close(y, y_ref, what):
    y = y.float().cpu().numpy().astype(np.float64)
    err = y - y_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-30)
    mx = np.max(np.abs(err)) / max(np.max(np.abs(y_ref)), 1e-30)
    assert rel <= Y_REL_FRO, f"{what}: rel-Frobenius {rel:.3e}"
    assert mx <= Y_MAX_REL, f"{what}: max-abs/max|y| {mx:.3e}"


def test_noalloc_matches_workspace_forward_two_calls():
    K, N, R = 3072, 640, 32
    first = syn.make_checkpoint(333, K, N, R, seed=71, wcscales="uniform", wtscale=0.75)
    second = syn.make_checkpoint(130, K, N, R, seed=72, wcscales="uniform", wtscale=0.75)
    # Same weights for both calls: the second checkpoint only supplies a new x.
    layer = _layer(first)
    try:
        stream = torch.cuda.current_stream()
        for i, ck in enumerate((first, second)):
            x = _x(ck)
            M = x.shape[0]
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            S.svdq_linear_forward_noalloc(layer.handle, x.data_ptr(), M, y.data_ptr(), stream)
            y_ref = layer.forward(x)
            torch.cuda.synchronize()
            assert torch.isfinite(y.float()).all(), f"call {i}: output not fully written"
            assert torch.equal(y, y_ref), f"call {i} (M={M}): differs from svdq_linear_forward"
            if i == 0:
                _assert_y_close(y, O.linear_forward(ck), f"call {i} (M={M}) against the oracle")
        assert layer.device_status() == 0
    finally:
        layer.close()


def test_noalloc_rejects_m_beyond_scratch():
    K, N, R = 3072, 256, 32
    ck = syn.make_checkpoint(16, K, N, R, seed=73)
    layer = _layer(ck)
    try:
        per_row = S.svdq_workspace_bytes(layer.handle, 1280) / 1280
        M = int(S.NOALLOC_SCRATCH_BYTES / per_row) + 1280
        assert S.svdq_workspace_bytes(layer.handle, M) > S.NOALLOC_SCRATCH_BYTES
        # Real buffers of the right size, so only the scratch is too small; the
        # size check returns before anything is looked up or launched.
        x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(S.SvdqError) as ei:
            S.svdq_linear_forward_noalloc(layer.handle, x.data_ptr(), M, y.data_ptr())
        assert ei.value.status == S.SVDQ_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert layer.device_status() == 0
    finally:
        layer.close()
