"""GPU parity of the tensor-core (tcgen05) GEMM that bw_gemv_nvfp4 uses for
more than 4 activation rows.

The A operand carries the block-scaled NVFP4 weights e2m1 * e4m3, exact in
fp16; the activations are rounded to fp16 for the B operand.  So:
  - one-hot activation rows reproduce the dequantized weight columns
    BIT-EXACTLY (one exact product, times the fp32 tensor scale -- the
    oracle's own rounding);
  - against the oracle evaluated on the same fp16-rounded activations the
    only difference left is fp32 accumulation order;
  - against the plain fp32 oracle the difference is the activation rounding,
    within the graded 2e-3 normwise tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, synth
from gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


def _pack(m, up=None):
    rows = m.N * (2 if up is not None else 1)
    qb, sb = bw.repack_bytes(rows, m.K)
    q = torch.empty((qb,), dtype=torch.uint8, device="cuda")
    s = torch.empty((sb,), dtype=torch.uint8, device="cuda")
    bw.repack_nvfp4(m.q, m.s, m.N, m.K, q, s, q_up=None if up is None else up.q,
                    s_up=None if up is None else up.s)
    return q, s, rows


def _run(m, x, M, flags=0, gamma=None, up=None, residual=None, want_argmax=False, eps=1e-6):
    q, s, N = _pack(m, up)
    ncols = N // 2 if flags & bw.GEMV_SILU_GATE else N
    y = torch.full((M, ncols), float("nan"), device="cuda")
    if residual is not None:
        y.copy_(residual)
    am = torch.full((M,), -1, dtype=torch.int32, device="cuda") if want_argmax else None
    ws = bw.workspace(bw.gemv_workspace_bytes(N, m.K, M, flags))
    bw.gemv_nvfp4(q, s, m.ts, N, m.K, x, M, y, ws, ts_up=(up.ts if up is not None else m.ts),
                  gamma=gamma, eps=eps, residual=y if residual is not None else None,
                  argmax_out=am, flags=flags)
    torch.cuda.synchronize()
    assert bw.read_error(ws) == 0
    return y.cpu().numpy(), (am.cpu().numpy() if am is not None else None)


def _f16(v):
    return np.asarray(v, np.float32).astype(np.float16).astype(np.float32)


@pytest.mark.parametrize("shape", [(128, 512), (640, 704), (4608, 3584)])
@pytest.mark.parametrize("M", [5, 16, 32])
def test_mma_one_hot_columns_bit_exact(shape, M):
    N, K = shape
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 11, f"mo{N}x{K}"), synth.FMT_NVFP4)
    rng = np.random.default_rng(N + K + M)
    cols = rng.choice(K, size=M, replace=False)
    cols[0], cols[-1] = 0, K - 1
    x = torch.zeros((M, K), device="cuda")
    for i, c in enumerate(cols):
        x[i, int(c)] = 1.0
    y, _ = _run(m, x, M)
    deq = oracle.dequant(m)
    for i, c in enumerate(cols):
        assert np.array_equal(y[i], deq[:, int(c)]), (i, int(c))


@pytest.mark.parametrize("shape", [(256, 256), (640, 704), (4608, 3584), (1024, 18944)])
@pytest.mark.parametrize("M", [5, 8, 17, 32, 40])
def test_mma_matches_oracle(shape, M):
    N, K = shape
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 12, f"mg{N}x{K}"), synth.FMT_NVFP4)
    x = torch.randn((M, K), device="cuda")
    y, _ = _run(m, x, M)
    om = oracle.QMat(m)
    xh = x.cpu().numpy()
    for r in range(M):
        # same fp16 activations: fp32 accumulation order is the only difference
        assert rel_err(y[r], oracle.matvec(om, _f16(xh[r]))) < 1e-5
        # plain fp32 oracle: the graded tolerance
        assert rel_err(y[r], oracle.matvec(om, xh[r])) < TOL


@pytest.mark.parametrize("M", [6, 32])
def test_mma_fused_rmsnorm_silu_and_residual(M):
    H, F = 3584, 1024
    fmt = synth.FMT_NVFP4
    wg = synth.quantize(synth.randn((F, H), 0.02, "cuda", 13, "mwg"), fmt)
    wu = synth.quantize(synth.randn((F, H), 0.02, "cuda", 13, "mwu"), fmt)
    wd = synth.quantize(synth.randn((H, F), 0.02, "cuda", 13, "mwd"), fmt)
    x = torch.randn((M, H), device="cuda") * 3
    gamma = 1 + 0.02 * torch.randn(H, device="cuda")
    eps = 1e-6
    a, _ = _run(wg, x, M, flags=bw.GEMV_RMSNORM | bw.GEMV_SILU_GATE, gamma=gamma, up=wu, eps=eps)
    xh, gh = x.cpu().numpy(), gamma.cpu().numpy()
    og, ou, od = oracle.QMat(wg), oracle.QMat(wu), oracle.QMat(wd)
    for r in range(M):
        yn = oracle.rmsnorm(xh[r], gh, eps)
        # against fp16(y) of the oracle: the GPU's RMSNorm factor comes from a
        # tree-ordered sum, so a few elements of y round to the other fp16
        # neighbour (2^-11 relative each); the gated product roughly doubles
        # the relative error of g and u -- 1e-4 leaves room for both
        for y_in, tol in ((_f16(yn), 1e-4), (yn, TOL)):
            g = oracle.matvec(og, y_in)
            u = oracle.matvec(ou, y_in)
            want = np.array([oracle.silu(float(v)) for v in g], np.float32) * u
            assert rel_err(a[r], want) < tol, (r, tol, rel_err(a[r], want))
    act = torch.from_numpy(a).cuda()
    res = torch.randn((M, H), device="cuda")
    y, _ = _run(wd, act, M, flags=bw.GEMV_RESIDUAL, residual=res)
    for r in range(M):
        base = res[r].cpu().numpy()
        assert rel_err(y[r], base + oracle.matvec(od, _f16(a[r]))) < 1e-5
        assert rel_err(y[r], base + oracle.matvec(od, a[r])) < TOL


def test_mma_argmax_lm_head_rows():
    V, H, M = 151936, 4096, 8
    m = synth.quantize(synth.randn((V, H), 0.02, "cuda", 14, "mlm"), synth.FMT_NVFP4)
    x = torch.randn((M, H), device="cuda")
    gamma = 1 + 0.02 * torch.randn(H, device="cuda")
    y, am = _run(m, x, M, flags=bw.GEMV_RMSNORM | bw.GEMV_ARGMAX, gamma=gamma, want_argmax=True)
    om = oracle.QMat(m)
    for r in range(M):
        yn = oracle.rmsnorm(x[r].cpu().numpy(), gamma.cpu().numpy(), 1e-6)
        want = oracle.matvec(om, yn)
        assert rel_err(y[r], want) < TOL
        # the argmax is exact over the kernel's own logits
        assert am[r] == int(np.argmax(y[r]))
        i, margin = oracle.argmax(want)
        if margin > 1e-2:
            assert am[r] == i
