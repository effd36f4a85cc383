"""GPU parity of the individual libbw kernels against the CPU oracle, called
through the C ABI (token_decode_b200.bw)."""
import os

import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import bits, rel_err

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()
    torch.manual_seed(0)


def _ws(nbytes=1 << 26):
    return bw.workspace(nbytes)


# ------------------------------------------------------------- dequantize

@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_dequant_bit_exact_full_table(fmt):
    N, K = 1024, 256
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 0, "deq"), fmt)
    qw, keep = runtime._gpu_layout(m)
    toks = torch.arange(N, dtype=torch.int32, device="cuda")
    x = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ws = _ws(1 << 18)
    bw.embed(fmt, qw.q, qw.s, qw.ts, N, K, toks, N, x, ws)
    assert bw.read_error(ws) == 0
    want = oracle.dequant(m)
    assert np.array_equal(bits(x.cpu().numpy()), bits(want))


def _golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return [l.strip() for l in f if l.strip() and not l.startswith("#")]


def test_dequant_golden_blocks_on_gpu():
    """The hand-computed Q4_0 / NVFP4 blocks decode to the printed values on the GPU."""
    rows = [np.frombuffer(bytes.fromhex(l.split("|")[0].strip()), np.uint8) for l in _golden("q4_0_blocks.txt")]
    want = [np.array([float(v) for v in l.split("|")[1].split()], np.float32) for l in _golden("q4_0_blocks.txt")]
    N = 8
    blocks = np.zeros((N, 18), np.uint8)
    for i, r in enumerate(rows):
        blocks[i] = r
    m = synth.QMat(synth.FMT_Q4_0, N, 32, torch.from_numpy(blocks).cuda())
    qw, keep = runtime._gpu_layout(m)
    x = torch.empty((N, 32), dtype=torch.float32, device="cuda")
    bw.embed(0, qw.q, qw.s, 1.0, N, 32, torch.arange(N, dtype=torch.int32, device="cuda"), N, x)
    got = x.cpu().numpy()
    for i, w in enumerate(want):
        assert np.array_equal(got[i], w), (i, got[i], w)
    # NVFP4 (two 16-element blocks per 32-element row; the second block repeats the first)
    lines = _golden("nvfp4_blocks.txt")
    for l in lines:
        lhs, vals = l.split("|")
        codes, sc, ts = lhs.split()
        q = np.frombuffer(bytes.fromhex(codes), np.uint8)
        qq = np.zeros((8, 16), np.uint8)
        ss = np.zeros((8, 2), np.uint8)
        qq[:, :8] = q
        qq[:, 8:] = q
        ss[:] = int(sc, 16)
        m = synth.QMat(synth.FMT_NVFP4, 8, 32, torch.from_numpy(qq).cuda(), torch.from_numpy(ss).cuda(), float(ts))
        qw, keep = runtime._gpu_layout(m)
        bw.embed(1, qw.q, qw.s, float(ts), 8, 32, torch.arange(8, dtype=torch.int32, device="cuda"), 8, x)
        w = np.array([float(v) for v in vals.split()], np.float32)
        got = x.cpu().numpy()
        assert np.array_equal(bits(got[3, :16]), bits(w)) and np.array_equal(bits(got[3, 16:]), bits(w))


def test_embed_bad_token_sets_error_word():
    m = synth.quantize(synth.randn((64, 64), 0.02, "cuda", 0, "e"), synth.FMT_Q4_0)
    qw, keep = runtime._gpu_layout(m)
    ws = _ws(1 << 18)
    x = torch.full((2, 64), 7.0, device="cuda")
    bw.embed(0, qw.q, qw.s, 1.0, 64, 64, torch.tensor([3, 64], dtype=torch.int32, device="cuda"), 2, x, ws)
    assert bw.read_error(ws) == bw.DEVERR_BAD_TOKEN
    assert torch.all(x[1] == 0)
    assert bw.read_error(ws) == 0


# ------------------------------------------------------------------- GEMV

def _gemv(m, x, M, flags=0, gamma=None, residual=None, up=None, want_argmax=False, eps=1e-6):
    qw, keep = runtime._gpu_layout(m, up)
    N = qw.N
    ncols = N // 2 if flags & bw.GEMV_SILU_GATE else N
    y = torch.full((M, ncols), float("nan"), device="cuda")
    if residual is not None:
        y.copy_(residual)
    am = torch.full((M,), -1, dtype=torch.int32, device="cuda") if want_argmax else None
    ws = _ws(bw.gemv_workspace_bytes(N, m.K, M, flags))
    if m.fmt == synth.FMT_Q4_0:
        bw.gemv_q4_0(qw.q, qw.s, N, m.K, x, M, y, ws, gamma=gamma, eps=eps,
                     residual=y if residual is not None else None, argmax_out=am, flags=flags)
    else:
        bw.gemv_nvfp4(qw.q, qw.s, qw.ts, N, m.K, x, M, y, ws, ts_up=qw.ts_up, gamma=gamma, eps=eps,
                      residual=y if residual is not None else None, argmax_out=am, flags=flags)
    torch.cuda.synchronize()
    return y.cpu().numpy(), (am.cpu().numpy() if am is not None else None)


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
@pytest.mark.parametrize("shape", [(64, 256), (512, 704), (4608, 3584), (1024, 18944)])
def test_gemv_one_hot_columns_bit_exact(fmt, shape):
    N, K = shape
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 1, f"oh{N}x{K}"), fmt)
    cols = [0, 33, K // 2 + 5, K - 1]
    x = torch.zeros((4, K), device="cuda")
    for i, c in enumerate(cols):
        x[i, c] = 1.0
    y, _ = _gemv(m, x, 4)
    deq = oracle.dequant(m)
    for i, c in enumerate(cols):
        # exact equality of values: a zero weight may come out as +0 where the
        # plain product d*(q-8) gives -0 (same value, different sign bit)
        assert np.array_equal(y[i], deq[:, c]), (i, c)


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
@pytest.mark.parametrize("shape", [(8, 32), (256, 256), (512, 704), (4608, 3584), (3584, 18944)])
@pytest.mark.parametrize("M", [1, 3])
def test_gemv_matches_oracle(fmt, shape, M):
    N, K = shape
    m = synth.quantize(synth.randn((N, K), 0.02, "cuda", 2, f"g{N}x{K}"), fmt)
    x = torch.randn((M, K), device="cuda")
    y, _ = _gemv(m, x, M)
    om = oracle.QMat(m)
    xh = x.cpu().numpy()
    # both sides accumulate K fp32 products in different orders: a normwise
    # difference of a few sqrt(K) * 2^-24 is rounding, nothing more
    tol = 2e-7 * np.sqrt(K)
    for r in range(M):
        want = oracle.matvec(om, xh[r])
        assert rel_err(y[r], want) < tol, rel_err(y[r], want)


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
@pytest.mark.parametrize("M", [1, 2, 4, 6])
def test_gemv_fused_rmsnorm_residual_silu(fmt, M):
    H, F = 3584, 1024
    # NVFP4 with more than 4 rows runs on the tensor cores with fp16
    # activations (tests/test_gpu_mma.py checks that path tightly); here it
    # gets the graded tolerance, the CUDA-core path the fp32-reordering one
    tol = 2e-3 if (fmt == synth.FMT_NVFP4 and M > 4) else 1e-5
    wg = synth.quantize(synth.randn((F, H), 0.02, "cuda", 3, "wg"), fmt)
    wu = synth.quantize(synth.randn((F, H), 0.02, "cuda", 3, "wu"), fmt)
    wd = synth.quantize(synth.randn((H, F), 0.02, "cuda", 3, "wd"), fmt)
    x = torch.randn((M, H), device="cuda") * 3
    gamma = 1 + 0.02 * torch.randn(H, device="cuda")
    eps = 1e-6
    # gate/up with the RMSNorm prologue and SiLU-gate epilogue
    a, _ = _gemv(wg, x, M, flags=bw.GEMV_RMSNORM | bw.GEMV_SILU_GATE, gamma=gamma, up=wu, eps=eps)
    xh, gh = x.cpu().numpy(), gamma.cpu().numpy()
    ogu = [oracle.QMat(wg), oracle.QMat(wu)]
    for r in range(M):
        yn = oracle.rmsnorm(xh[r], gh, eps)
        g = oracle.matvec(ogu[0], yn)
        u = oracle.matvec(ogu[1], yn)
        want = np.array([oracle.silu(float(v)) for v in g], np.float32) * u
        assert rel_err(a[r], want) < tol, rel_err(a[r], want)
    # down with the residual epilogue (in place)
    act = torch.from_numpy(a).cuda()
    res = torch.randn((M, H), device="cuda")
    y, _ = _gemv(wd, act, M, flags=bw.GEMV_RESIDUAL, residual=res)
    od = oracle.QMat(wd)
    for r in range(M):
        want = res[r].cpu().numpy() + oracle.matvec(od, a[r])
        assert rel_err(y[r], want) < tol


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_gemv_argmax_lm_head(fmt):
    V, H, M = 151936, 4096, 2
    m = synth.quantize(synth.randn((V, H), 0.02, "cuda", 4, "lm"), fmt)
    x = torch.randn((M, H), device="cuda")
    gamma = 1 + 0.02 * torch.randn(H, device="cuda")
    y, am = _gemv(m, x, M, flags=bw.GEMV_RMSNORM | bw.GEMV_ARGMAX, gamma=gamma, want_argmax=True)
    om = oracle.QMat(m)
    for r in range(M):
        yn = oracle.rmsnorm(x[r].cpu().numpy(), gamma.cpu().numpy(), 1e-6)
        want = oracle.matvec(om, yn)
        assert rel_err(y[r], want) < 2e-7 * np.sqrt(H)
        i, margin = oracle.argmax(want)
        # the GPU's argmax is exact over its own logits
        assert am[r] == int(np.argmax(y[r]))
        if margin > 1e-3:
            assert am[r] == i


def test_gemv_argmax_ties_lowest_index():
    """Two identical rows: equal logits, the lower index wins."""
    N, K = 2048, 256
    x0 = synth.randn((N, K), 0.02, "cuda", 5, "tie")
    x0[1500] = x0[37] * 0 + 1.0    # rows 37 and 1500 become identical large rows
    x0[37] = 1.0
    m = synth.quantize(x0, synth.FMT_Q4_0)
    x = torch.ones((1, K), device="cuda")
    y, am = _gemv(m, x, 1, flags=bw.GEMV_ARGMAX, want_argmax=True)
    assert y[0, 37] == y[0, 1500] == y[0].max()
    assert am[0] == 37


# -------------------------------------------------------------- RMSNorm, argmax

def test_rmsnorm_fused_kernel():
    M, H = 3, 4096
    x = torch.randn((M, H), device="cuda")
    add = torch.randn((M, H), device="cuda")
    gamma = 1 + 0.02 * torch.randn(H, device="cuda")
    y = torch.empty((M, H), device="cuda")
    x0 = x.cpu().numpy() + add.cpu().numpy()
    bw.rmsnorm_fused(x, gamma, M, H, 1e-6, y=y, add=add)
    torch.cuda.synchronize()
    assert np.array_equal(x.cpu().numpy(), x0.astype(np.float32))
    for r in range(M):
        assert rel_err(y[r].cpu().numpy(), oracle.rmsnorm(x0[r], gamma.cpu().numpy(), 1e-6)) < 1e-6
    y16 = torch.empty((M, H), dtype=torch.float16, device="cuda")
    bw.rmsnorm_fused(x, gamma, M, H, 1e-6, y=y16, y_fp16=True)
    assert torch.equal(y16, y.half())


def test_argmax_kernel_planted_ties_margin():
    M, V = 3, 152064
    lg = torch.randn((M, V), device="cuda")
    lg[0, 100000] = 50.0
    lg[1, 7] = 50.0
    lg[1, 9000] = 50.0
    lg[2, V - 1] = 60.0
    lg[2, 3] = 59.5
    idx = torch.empty(M, dtype=torch.int32, device="cuda")
    mg = torch.empty(M, device="cuda")
    bw.argmax(lg, M, V, idx, mg)
    assert idx.tolist() == [100000, 7, V - 1]
    assert mg[1].item() == 0.0 and mg[2].item() == 0.5


def test_rope_table_matches_double_precision():
    hd, P = 128, 8400
    c = torch.empty((P, hd // 2), device="cuda")
    s = torch.empty_like(c)
    bw.rope_table(1e6, hd, P, c, s)
    p = np.arange(P, dtype=np.float64)[:, None]
    inv = 1e6 ** (-2.0 * np.arange(hd // 2) / hd)
    ang = p * inv
    wc, ws_ = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    gc, gs = c.cpu().numpy(), s.cpu().numpy()
    # fp64 evaluation rounded once to fp32: equal except (rarely) one ulp at a rounding boundary
    assert np.max(np.abs(gc.view(np.int32).astype(np.int64) - wc.view(np.int32))) <= 1
    assert np.max(np.abs(gs.view(np.int32).astype(np.int64) - ws_.view(np.int32))) <= 1
    assert np.mean(gc == wc) > 0.999 and np.mean(gs == ws_) > 0.999


# -------------------------------------------------------------- attention

def _attn_case(B, R, nq, nkv, hd, ctxs, seed=0, n_pages=None, perm=True):
    P = 16
    max_pages = -(-(max(ctxs) + R) // P)
    n_pages = B * max_pages if n_pages is None else n_pages
    g = torch.Generator(device="cpu").manual_seed(seed)
    kp = torch.randn((n_pages, nkv, P, hd), generator=g).half().cuda()
    vp = torch.randn((n_pages, nkv, P, hd), generator=g).half().cuda()
    table = (torch.randperm(n_pages, generator=g) if perm else torch.arange(n_pages))[: B * max_pages]
    table = table.reshape(B, max_pages).to(torch.int32).cuda()
    qkv = (torch.randn((B * R, (nq + 2 * nkv) * hd), generator=g) * 1.5).cuda()
    pos = torch.tensor(ctxs, dtype=torch.int32, device="cuda")
    return kp, vp, table, qkv, pos, max_pages, n_pages


def _attn_oracle(kp, vp, table, qkv, pos, B, R, nq, nkv, hd, n_pages, theta=1e6):
    class _KV:
        pass
    kv = _KV()
    kv.k = [kp.cpu().view(torch.int16)]
    kv.v = [vp.cpu().view(torch.int16)]
    kv.page_table = table.cpu()
    kv.n_pages = n_pages
    kv.page_tokens = 16
    okv = oracle.KV(kv)
    q_all = qkv.cpu().numpy()
    out = np.zeros((B * R, nq * hd), np.float32)
    for b in range(B):
        for r in range(R):
            p = int(pos[b]) + r
            row = q_all[b * R + r]
            q = row[: nq * hd].reshape(nq, hd)
            k = row[nq * hd:(nq + nkv) * hd].reshape(nkv, hd)
            v = row[(nq + nkv) * hd:].reshape(nkv, hd)
            P = 16
            page = int(okv.page_table[b, p // P])
            for h in range(nkv):
                kr = oracle.rope(k[h], p, theta)
                okv.k[0][page, h, p % P] = [oracle.f32_to_fp16(float(t)) for t in kr]
                okv.v[0][page, h, p % P] = [oracle.f32_to_fp16(float(t)) for t in v[h]]
            for h in range(nq):
                qr = oracle.rope(q[h], p, theta)
                out[b * R + r, h * hd:(h + 1) * hd] = oracle.attend_head(qr, okv, 0, b, nkv, h // (nq // nkv), p + 1)
    return out, okv


@pytest.mark.parametrize("case", [
    dict(B=1, R=1, nq=4, nkv=2, hd=64, ctxs=[128]),           # tiny shape
    dict(B=1, R=1, nq=28, nkv=4, hd=128, ctxs=[2000]),        # 7B shape
    dict(B=1, R=1, nq=28, nkv=4, hd=128, ctxs=[0]),           # first position only
    dict(B=1, R=4, nq=64, nkv=8, hd=128, ctxs=[8190]),        # verify rows across a page boundary
    dict(B=3, R=1, nq=32, nkv=8, hd=128, ctxs=[15, 16, 333]), # ragged lengths
    dict(B=2, R=4, nq=16, nkv=2, hd=128, ctxs=[5, 47]),
    dict(B=1, R=1, nq=4, nkv=2, hd=64, ctxs=[8000]),          # long splits: the 4-stage ring wraps
    dict(B=40, R=1, nq=8, nkv=4, hd=64,                       # >= one group per SM: one split, 2-stage ring
         ctxs=[17 + 7 * i for i in range(40)]),
    dict(B=3, R=1, nq=8, nkv=4, hd=64, ctxs=[9300, 40, 5000]),  # page-table rows too wide to load with the
                                                               # position; cluster merge of ragged lengths
])
def test_paged_attention_matches_oracle(case):
    B, R, nq, nkv, hd, ctxs = case["B"], case["R"], case["nq"], case["nkv"], case["hd"], case["ctxs"]
    kp, vp, table, qkv, pos, max_pages, n_pages = _attn_case(B, R, nq, nkv, hd, ctxs)
    maxpos = max_pages * 16
    cos = torch.empty((maxpos, hd // 2), device="cuda")
    sin = torch.empty_like(cos)
    bw.rope_table(1e6, hd, maxpos, cos, sin)
    out = torch.empty((B * R, nq * hd), device="cuda")
    ws = _ws(bw.attn_workspace_bytes(B, R, nq, nkv, hd, max_pages))
    kp_gpu, vp_gpu = kp.clone(), vp.clone()
    bw.paged_attn_decode(qkv, cos, sin, maxpos, kp_gpu, vp_gpu, table, max_pages, n_pages, pos, B, R,
                         nq, nkv, hd, out, ws)
    assert bw.read_error(ws) == 0
    want, okv = _attn_oracle(kp, vp, table, qkv, pos, B, R, nq, nkv, hd, n_pages)
    assert rel_err(out.cpu().numpy(), want) < 2e-5, rel_err(out.cpu().numpy(), want)
    # every slot the call did not write is untouched, bit for bit; the rows it
    # wrote are the oracle's fp16 roundings: V exactly, RoPE'd K within one fp16
    # step (the rotation's cos/sin come from a table rounded once from fp64)
    kg = kp_gpu.cpu().view(torch.int16).numpy().view(np.uint16)
    vg = vp_gpu.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(vg, okv.v[0])
    written = np.zeros(kg.shape[0:1] + kg.shape[2:3], dtype=bool)          # [page][slot]
    tab = table.cpu().numpy()
    for b in range(B):
        for p in range(ctxs[b], ctxs[b] + R):
            written[tab[b, p // 16], p % 16] = True
    g = kg.transpose(0, 2, 1, 3)
    o = okv.k[0].transpose(0, 2, 1, 3)
    assert np.array_equal(g[~written], o[~written])

    def ordered(h):     # fp16 bit patterns -> integers in value order (adjacent values differ by 1)
        h = h.astype(np.int64)
        return np.where(h & 0x8000, -(h & 0x7FFF), h)
    assert np.max(np.abs(ordered(g[written]) - ordered(o[written]))) <= 1


def test_paged_attention_page_order_invariant_and_deterministic():
    B, R, nq, nkv, hd = 2, 1, 28, 4, 128
    kp, vp, table, qkv, pos, max_pages, n_pages = _attn_case(B, R, nq, nkv, hd, [700, 1234], seed=3)
    # same logical content under the identity page table
    ident = torch.arange(B * max_pages, dtype=torch.int32, device="cuda").reshape(B, max_pages)
    kp2, vp2 = torch.empty_like(kp), torch.empty_like(vp)
    for b in range(B):
        kp2[ident[b].long()] = kp[table[b].long()]
        vp2[ident[b].long()] = vp[table[b].long()]
    maxpos = max_pages * 16
    cos = torch.empty((maxpos, hd // 2), device="cuda")
    sin = torch.empty_like(cos)
    bw.rope_table(1e6, hd, maxpos, cos, sin)
    ws = _ws(bw.attn_workspace_bytes(B, R, nq, nkv, hd, max_pages))
    outs = []
    for (k_, v_, t_) in ((kp.clone(), vp.clone(), table), (kp2.clone(), vp2.clone(), ident), (kp.clone(), vp.clone(), table)):
        o = torch.empty((B * R, nq * hd), device="cuda")
        bw.paged_attn_decode(qkv, cos, sin, maxpos, k_, v_, t_, max_pages, n_pages, pos, B, R, nq, nkv, hd, o, ws)
        outs.append(o.cpu())
    assert torch.equal(outs[0], outs[1])      # paged == contiguous, bit for bit
    assert torch.equal(outs[0], outs[2])      # run-to-run deterministic


def test_paged_attention_bad_page_sets_error_and_skips():
    B, R, nq, nkv, hd = 1, 1, 8, 2, 128
    kp, vp, table, qkv, pos, max_pages, n_pages = _attn_case(B, R, nq, nkv, hd, [100], seed=4)
    table[0, 2] = n_pages + 5         # poisoned entry inside the context
    table[0, 3] = -1
    maxpos = max_pages * 16
    cos = torch.empty((maxpos, hd // 2), device="cuda")
    sin = torch.empty_like(cos)
    bw.rope_table(1e6, hd, maxpos, cos, sin)
    ws = _ws(bw.attn_workspace_bytes(B, R, nq, nkv, hd, max_pages))
    out = torch.empty((B * R, nq * hd), device="cuda")
    bw.paged_attn_decode(qkv, cos, sin, maxpos, kp, vp, table, max_pages, n_pages, pos, B, R, nq, nkv, hd, out, ws)
    assert bw.read_error(ws) & bw.DEVERR_BAD_PAGE
    assert torch.isfinite(out).all()
    # a position beyond the page table is reported too
    pos2 = torch.tensor([max_pages * 16 + 3], dtype=torch.int32, device="cuda")
    bw.paged_attn_decode(qkv, cos, sin, maxpos, kp, vp, table, max_pages, n_pages, pos2, B, R, nq, nkv, hd, out, ws)
    assert bw.read_error(ws) & bw.DEVERR_BAD_POS


# ------------------------------------------------------ FP8 (E4M3) attention

def _attn_fp8_oracle(kp8, vp8, ks, vs, table, qkv, pos, B, R, nq, nkv, hd, n_pages, theta=1e6):
    """The oracle over an E4M3 cache: the new rows encoded as E4M3 of value /
    scale, then each query head attends (oracle.attend_head_e4m3)."""
    class _KV:
        pass
    kv = _KV()
    kv.k = [kp8.cpu()]
    kv.v = [vp8.cpu()]
    kv.page_table = table.cpu()
    kv.n_pages = n_pages
    kv.page_tokens = 16
    okv = oracle.KV(kv)      # byte pools read as uint16 pairs are not used: attend_head_e4m3 takes the bytes
    kb = kp8.cpu().numpy().copy()
    vb = vp8.cpu().numpy().copy()
    q_all = qkv.cpu().numpy()
    out = np.zeros((B * R, nq * hd), np.float32)
    for b in range(B):
        for r in range(R):
            p = int(pos[b]) + r
            row = q_all[b * R + r]
            q = row[: nq * hd].reshape(nq, hd)
            k = row[nq * hd:(nq + nkv) * hd].reshape(nkv, hd)
            v = row[(nq + nkv) * hd:].reshape(nkv, hd)
            page = int(okv.page_table[b, p // 16])
            for h in range(nkv):
                kr = oracle.rope(k[h], p, theta)
                kb[page, h, p % 16] = [oracle.f32_to_e4m3(float(np.float32(t) / np.float32(ks))) for t in kr]
                vb[page, h, p % 16] = [oracle.f32_to_e4m3(float(np.float32(t) / np.float32(vs))) for t in v[h]]
            for h in range(nq):
                qr = oracle.rope(q[h], p, theta)
                out[b * R + r, h * hd:(h + 1) * hd] = oracle.attend_head_e4m3(qr, kb, vb, ks, vs, okv, b, nkv,
                                                                              h // (nq // nkv), p + 1)
    return out, kb, vb


@pytest.mark.parametrize("case", [
    dict(B=1, R=1, nq=4, nkv=2, hd=64, ctxs=[128]),
    dict(B=1, R=1, nq=28, nkv=4, hd=128, ctxs=[2000]),
    dict(B=1, R=4, nq=64, nkv=8, hd=128, ctxs=[8190]),        # verify rows across a page boundary
    dict(B=3, R=1, nq=32, nkv=8, hd=128, ctxs=[15, 16, 333]),
    dict(B=40, R=1, nq=8, nkv=4, hd=64, ctxs=[17 + 7 * i for i in range(40)]),
])
def test_paged_attention_fp8_matches_oracle(case):
    """Attention over an E4M3 cache with per-layer scales against the oracle's
    E4M3 attention: outputs within 2e-5; the written codes are the oracle's
    (V exactly; RoPE'd K within one code), every other byte untouched."""
    B, R, nq, nkv, hd, ctxs = case["B"], case["R"], case["nq"], case["nkv"], case["hd"], case["ctxs"]
    kp, vp, table, qkv, pos, max_pages, n_pages = _attn_case(B, R, nq, nkv, hd, ctxs, seed=7)
    ks, vs = 1.0 / 16 + 3.0 / 256, 1.0 / 20 + 3.0 / 256
    kp8 = (kp.float() / ks).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    vp8 = (vp.float() / vs).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    maxpos = max_pages * 16
    cos = torch.empty((maxpos, hd // 2), device="cuda")
    sin = torch.empty_like(cos)
    bw.rope_table(1e6, hd, maxpos, cos, sin)
    out = torch.empty((B * R, nq * hd), device="cuda")
    ws = _ws(bw.attn_workspace_bytes(B, R, nq, nkv, hd, max_pages))
    kg, vg = kp8.clone(), vp8.clone()
    bw.paged_attn_decode_fp8(qkv, cos, sin, maxpos, kg, vg, ks, vs, table, max_pages, n_pages, pos, B, R,
                             nq, nkv, hd, out, ws)
    assert bw.read_error(ws) == 0
    want, kb, vb = _attn_fp8_oracle(kp8, vp8, ks, vs, table, qkv, pos, B, R, nq, nkv, hd, n_pages)
    assert rel_err(out.cpu().numpy(), want) < 2e-5, rel_err(out.cpu().numpy(), want)
    assert np.array_equal(vg.cpu().numpy(), vb)
    kgn = kg.cpu().numpy()
    diff = kgn != kb
    if diff.any():
        # a RoPE'd k may land one code away (its cos/sin come from a table rounded once from fp64)
        a = kgn[diff].astype(np.int64)
        o = kb[diff].astype(np.int64)
        oa = np.where(a & 0x80, -(a & 0x7F), a)
        oo = np.where(o & 0x80, -(o & 0x7F), o)
        assert np.max(np.abs(oa - oo)) <= 1
        assert diff.sum() <= B * R * nkv * hd // 8


def test_paged_attention_fp8_rejects_bad_scales():
    kp, vp, table, qkv, pos, max_pages, n_pages = _attn_case(1, 1, 4, 2, 64, [40], seed=8)
    kp8 = torch.zeros_like(kp, dtype=torch.uint8)
    cos = torch.zeros((max_pages * 16, 32), device="cuda")
    out = torch.empty((1, 4 * 64), device="cuda")
    ws = _ws(bw.attn_workspace_bytes(1, 1, 4, 2, 64, max_pages))
    for ks in (0.0, -1.0, float("inf")):
        with pytest.raises(bw.BWError):
            bw.paged_attn_decode_fp8(qkv, cos, cos, max_pages * 16, kp8, kp8.clone(), ks, 0.05, table, max_pages,
                                     n_pages, pos, 1, 1, 4, 2, 64, out, ws)


def test_drain_error_moves_the_word_without_a_sync_and_in_a_graph():
    """bw_drain_error ORs a workspace's device error word into a device
    accumulator and clears it, queued on the stream (eagerly and inside a
    captured graph)."""
    ws = bw.workspace(1 << 18)
    word = ws[:4].view(torch.int32)
    dst = torch.full((1,), 2, dtype=torch.int32, device="cuda")
    word.fill_(5)                      # a planted error word: bits 0 and 2
    bw.drain_error(ws, dst)
    torch.cuda.synchronize()
    assert int(dst.item()) == 7 and int(word.item()) == 0
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            bw.drain_error(ws, dst, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    dst.zero_()
    word.fill_(8)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert int(dst.item()) == 8 and int(word.item()) == 0
    g.replay()                         # nothing planted: the accumulator keeps its bits
    torch.cuda.synchronize()
    assert int(dst.item()) == 8
    assert bw.read_error(ws) == 0
