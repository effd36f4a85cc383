"""The workspace-free Q4_0 GEMV (bw_gemv_q4_0_noalloc), for callers that
cannot allocate device memory (a host framework that owns every device
allocation, or a path where cudaMalloc's implicit synchronization is not
acceptable).  It runs the same kernel with the same split plan as
bw_gemv_q4_0, its scratch living in the library's fixed device array, so its
outputs must be bit-identical to the workspace entry point's, call after
call, and within the GEMV tolerance of the oracle.  Kept in a file of its own
that pytest collects last, so that a run stopping at the first failure has
run every other test before it."""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


@pytest.mark.parametrize("N,K,M,flags", [
    (3584, 18944, 1, bw.GEMV_RESIDUAL),          # split-K: partial sums and counters in the scratch
    (4608, 3584, 3, bw.GEMV_RMSNORM),
    (8192, 3584, 2, bw.GEMV_RMSNORM | bw.GEMV_ARGMAX),
])
def test_noalloc_gemv_matches_workspace_entry_point_twice(N, K, M, flags):
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 11, f"na{N}x{K}"), synth.FMT_Q4_0)
    qw, keep = runtime._gpu_layout(m)
    om = oracle.QMat(m)
    gamma = 1 + 0.02 * torch.randn(K, device="cuda")
    ws = bw.workspace(bw.gemv_workspace_bytes(N, K, M, flags))
    assert bw.read_error(None) == 0          # the fixed scratch's error word starts clear
    tol = 2e-7 * np.sqrt(K)                  # the GEMV parity tolerance against the oracle
    for call in range(2):
        x = torch.randn((M, K), device="cuda") * (1 + call)
        res = torch.randn((M, N), device="cuda")
        y_ref, y_na = res.clone(), res.clone()
        a_ref = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        a_na = a_ref.clone()
        want_am = bool(flags & bw.GEMV_ARGMAX)
        bw.gemv_q4_0(qw.q, qw.s, N, K, x, M, y_ref, ws, gamma=gamma,
                     residual=y_ref if flags & bw.GEMV_RESIDUAL else None,
                     argmax_out=a_ref if want_am else None, flags=flags)
        bw.gemv_q4_0_noalloc(qw.q, qw.s, N, K, x, M, y_na, gamma=gamma,
                             residual=y_na if flags & bw.GEMV_RESIDUAL else None,
                             argmax_out=a_na if want_am else None, flags=flags)
        torch.cuda.synchronize()
        # same kernel, same plan: bit for bit
        assert torch.equal(y_na, y_ref)
        if want_am:
            assert torch.equal(a_na, a_ref)
        # and the oracle's matrix-vector product
        xh, rh, yh = x.cpu().numpy(), res.cpu().numpy(), y_na.cpu().numpy()
        for r in range(M):
            xr = oracle.rmsnorm(xh[r], gamma.cpu().numpy(), 1e-6) if flags & bw.GEMV_RMSNORM else xh[r]
            want = oracle.matvec(om, xr)
            got = yh[r] - rh[r] if flags & bw.GEMV_RESIDUAL else yh[r]
            assert rel_err(got, want) <= tol, (call, r, rel_err(got, want))
    assert bw.read_error(None) == 0
