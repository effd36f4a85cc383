"""The workspace-free Q4_0 GEMV (bw_gemv_q4_0_noalloc), for callers that
cannot allocate device memory: it must give the same results as the regular
entry point, call after call, with its scratch living in the library's fixed
device array.  Kept in a file of its own so it runs after every other test."""
import numpy as np
import pytest
import torch

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
    gamma = 1 + 0.02 * torch.randn(K, device="cuda")
    ws = bw.workspace(bw.gemv_workspace_bytes(N, K, M, flags))
    tol = 2e-7 * np.sqrt(K)          # the GEMV parity tolerance
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
        for r in range(M):
            assert rel_err(y_na[r].cpu().numpy(), y_ref[r].cpu().numpy()) <= tol
        if want_am:
            assert torch.equal(a_na, a_ref)
