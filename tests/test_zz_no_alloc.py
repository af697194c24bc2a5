"""smuon_ns_static: the Newton-Schulz entry point for callers that cannot
allocate device memory at the call site. It must produce what smuon_ns
produces with a caller-provided workspace, call after call, although every
call reuses the same fixed scratch array and finds the previous call's
contents in it. Collected last so that a failure here never hides the rest."""
import ctypes

import numpy as np
import pytest
import torch

import matrix_aware_sign_b200 as S
import workloads as WL
from tests.gpu_util import dev, rel_fro

pytestmark = pytest.mark.gpu

SHAPES = [(64, 147), (256, 64), (256, 256), (130, 300)]


def _inputs(seed):
    rng = np.random.default_rng(seed)
    M0 = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
    G = [rng.standard_normal(s).astype(np.float32) for s in SHAPES]
    return M0, G


def _static_call(Md, Ud, Gd, coeffs, iters, flags):
    """Calls smuon_ns_static through the C ABI (ctypes), on the current stream."""
    L = S.lib()
    n = len(Md)
    mats = lambda ts: (S.SmuonMat * n)(*[S.mat(t) for t in ts])
    return L.smuon_ns_static(mats(Md), mats(Ud), n, mats(Gd), 0.9, *coeffs, iters, 1e-7, flags, None, None, None,
                             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("flags", [0, S.NS_FP32_REF])
def test_static_scratch_matches_workspace_entry_on_two_calls(flags):
    for seed, (coeffs, iters) in ((1, (WL.QUINTIC, 2)), (2, (WL.CUBIC, 3))):
        M0, G = _inputs(seed)
        # the existing entry point, with a workspace
        Ma = [dev(m) for m in M0]
        Ua = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in SHAPES]
        S.smuon_ns(Ma, Ua, *coeffs, iters, G=[dev(g) for g in G], beta=0.9, flags=flags)
        # the no-allocation entry point on fresh copies of the same inputs
        Mb = [dev(m) for m in M0]
        Ub = [torch.full(s, 3.0, dtype=torch.bfloat16, device="cuda") for s in SHAPES]
        rc = _static_call(Mb, Ub, [dev(g) for g in G], coeffs, iters, flags)
        assert rc == 0, S.lib().smuon_last_error()
        torch.cuda.synchronize()
        for a, b in zip(Ua, Ub):
            assert rel_fro(b.float().cpu().numpy(), a.float().cpu().numpy()) <= 1e-6
        for a, b in zip(Ma, Mb):
            np.testing.assert_allclose(b.cpu().numpy(), a.cpu().numpy(), rtol=1e-6, atol=0)


def test_static_scratch_rejects_a_batch_beyond_its_size():
    big = [torch.zeros((4096, 4096), device="cuda")]
    out = [torch.zeros((4096, 4096), dtype=torch.bfloat16, device="cuda")]
    assert S.smuon_ns_workspace_bytes(big, 5) > S.NS_STATIC_SCRATCH_BYTES
    L = S.lib()
    rc = L.smuon_ns_static((S.SmuonMat * 1)(S.mat(big[0])), (S.SmuonMat * 1)(S.mat(out[0])), 1, None, 0.0,
                           *WL.QUINTIC, 5, 1e-7, 0, None, None, None, torch.cuda.current_stream().cuda_stream)
    assert rc == -5
    assert b"smuon_ns_static holds at most" in L.smuon_last_error()
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0)
