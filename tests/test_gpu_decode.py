"""GPU parity of the whole decode step (bw_decode_step) against the CPU oracle:
greedy tokens under the margin rule, logits within the stated tolerance,
the KV cache written by the step, graph replay with on-device advance,
determinism, paging and batch invariance, and full-size layer shapes."""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import MARGIN, TOL, rel_err
from gpu_util import check_kv as check_kv_pools

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


def _setup(cfg, seed=0, n_layers=None, permute=True):
    model = synth.make_model(cfg, "cuda", seed=seed, n_layers=n_layers)
    kv = synth.make_kv(cfg, "cuda", seed=seed, permute=permute, n_layers=n_layers)
    om = oracle.Model(model)
    okv = oracle.KV(kv)
    max_pos = cfg.max_pages * synth.PAGE_TOKENS
    dm = runtime.DeviceModel(model, max_pos)
    dkv = runtime.DeviceKV(kv)
    return model, kv, om, okv, dm, dkv


def _run_steps(cfg, steps, seed=0, n_layers=None, B=None, check_kv=True):
    """Greedy decode on the GPU with the oracle teacher-forced on the GPU's
    tokens; returns the worst normwise logit error."""
    B = cfg.B if B is None else B
    model, kv, om, okv, dm, dkv = _setup(cfg, seed, n_layers)
    dec = runtime.Decoder(dm, dkv, B)
    toks = synth.start_tokens(cfg, seed)[:B]
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    logits = torch.empty((B, cfg.V), device="cuda")
    worst = 0.0
    cur = toks.tolist()
    for step in range(steps):
        dec.tokens_in.copy_(torch.tensor(cur, dtype=torch.int32))
        dec.step(logits=logits)
        assert bw.read_error(dec.ws) == 0
        got_tok = dec.tokens_out.cpu().tolist()
        got_lg = logits.cpu().numpy()
        for b in range(B):
            res = oracle.decode_token(om, okv, b, cur[b], cfg.ctx + step)
            err = rel_err(got_lg[b], res["logits"])
            worst = max(worst, err)
            assert err < TOL, (step, b, err)
            assert got_tok[b] == int(np.argmax(got_lg[b]))
            if res["margin"] > MARGIN:
                assert got_tok[b] == res["token"], (step, b, res["margin"])
        cur = got_tok
        dec.pos += 1
    if check_kv:
        check_kv_pools(list(dkv.k) + list(dkv.v), list(okv.k) + list(okv.v), dkv.page_table, B,
                       cfg.ctx, steps)
    return worst


def test_tiny_decode_8_steps():
    cfg = synth.CONFIGS["tiny"]
    _run_steps(cfg, cfg.steps)


def test_tiny_nvfp4_two_layers_batch2():
    cfg = synth.CONFIGS["tiny"].with_(fmt=synth.FMT_NVFP4, L=2, B=2)
    _run_steps(cfg, 4)


def test_tiny_nvfp4_batch8_tensor_core_path():
    """8 rows of NVFP4: every projection runs on the tcgen05 GEMM."""
    cfg = synth.CONFIGS["tiny"].with_(fmt=synth.FMT_NVFP4, B=8)
    _run_steps(cfg, 3)


def test_tiny_batch5_rows_above_gemv_block():
    cfg = synth.CONFIGS["tiny"].with_(B=5)
    _run_steps(cfg, 3)


def _tiny_moe(**kw):
    return synth.CONFIGS["tiny"].with_(name="tiny-moe", fmt=synth.FMT_NVFP4, F=0, n_experts=16,
                                       topk=4, F_exp=64, B=4, L=2, **kw)


def test_tiny_moe_decode_and_router_topk():
    """MoE decode vs the oracle: logits, tokens and the selected experts."""
    cfg = _tiny_moe()
    model, kv, om, okv, dm, dkv = _setup(cfg, seed=3)
    dec = runtime.Decoder(dm, dkv, cfg.B)
    toks = synth.start_tokens(cfg, 3)[: cfg.B]
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    logits = torch.empty((cfg.B, cfg.V), device="cuda")
    dec.step(logits=logits)
    assert bw.read_error(dec.ws) == 0
    for b in range(cfg.B):
        res = oracle.decode_token(om, okv, b, int(toks[b]), cfg.ctx)
        assert rel_err(logits[b].cpu().numpy(), res["logits"]) < TOL
        if res["margin"] > MARGIN:
            assert int(dec.tokens_out[b]) == res["token"]
    # the routing kernel alone: same inputs -> same expert choice as the oracle's
    x = torch.randn((cfg.B, cfg.H), device="cuda")
    ly = dm.layers[0]
    idx = torch.empty((cfg.B, cfg.topk), dtype=torch.int32, device="cuda")
    wts = torch.empty((cfg.B, cfg.topk), device="cuda")
    ws = bw.workspace(bw.moe_workspace_bytes(dm.c, cfg.B))
    x0 = x.clone()
    bw.moe_route_gemv(dm.c, ly, x, cfg.B, ws, topk_idx=idx, topk_w=wts)
    torch.cuda.synchronize()
    g = model.layers[0]
    for b in range(cfg.B):
        y = oracle.rmsnorm(x0[b].cpu().numpy(), g.ffn_norm.cpu().numpy(), cfg.eps)
        r = (g.router.cpu().numpy().astype(np.float64) @ y.astype(np.float64))
        order = np.lexsort((np.arange(cfg.n_experts), -r))
        gap = r[order[cfg.topk - 1]] - r[order[cfg.topk]]
        if gap > 1e-3:
            assert sorted(idx[b].tolist()) == sorted(order[: cfg.topk].tolist())
        assert abs(float(wts[b].sum()) - 1.0) < 1e-5
    assert torch.isfinite(x).all() and not torch.equal(x, x0)


def test_step_hidden_state_matches_oracle():
    """The residual stream bw_decode_hidden exposes after a step is each row's
    hidden state after the last layer, as the oracle computes it."""
    cfg = synth.CONFIGS["tiny"].with_(B=2, L=2)
    model, kv, om, okv, dm, dkv = _setup(cfg, seed=9)
    dec = runtime.Decoder(dm, dkv, cfg.B)
    toks = synth.start_tokens(cfg, 9)[: cfg.B]
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    dec.step()
    assert bw.read_error(dec.ws) == 0
    hid = bw.decode_hidden(dm.c, dkv.c, cfg.B, 1, dec.ws).cpu().numpy()
    for b in range(cfg.B):
        res = oracle.decode_token(om, okv, b, int(toks[b]), cfg.ctx, want_logits=False, want_hidden=True)
        assert rel_err(hid[b], res["hidden"][cfg.L]) < TOL


def test_graph_replay_with_device_advance_matches_eager():
    cfg = synth.CONFIGS["tiny"].with_(B=2)
    model, kv, om, okv, dm, dkv = _setup(cfg, seed=5)
    kv0 = [t.clone() for t in kv.k], [t.clone() for t in kv.v]
    dec = runtime.Decoder(dm, dkv, cfg.B)
    toks = synth.start_tokens(cfg, 5)[: cfg.B]
    # eager, host-driven
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    eager = []
    for _ in range(6):
        dec.step(advance=True)
        eager.append(dec.tokens_out.cpu().clone())
    # restore the cache, capture 6 steps in one graph, replay
    for l in range(cfg.L):
        dkv.k[l].copy_(kv0[0][l])
        dkv.v[l].copy_(kv0[1][l])
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    outs = torch.empty((6, cfg.B), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(6):
                dec.step(advance=True, stream=s)
                outs[i].copy_(dec.tokens_out)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(outs.cpu(), torch.stack(eager))
    assert dec.pos.tolist() == [cfg.ctx + 6] * cfg.B
    assert bw.read_error(dec.ws) == 0


def test_decode_deterministic_and_page_order_invariant():
    cfg = synth.CONFIGS["tiny"].with_(B=2, L=2)
    model = synth.make_model(cfg, "cuda", seed=7)
    kv_a = synth.make_kv(cfg, "cuda", seed=7, permute=True)
    # same logical content under the identity page table
    kv_b = kv_a.clone()
    kv_b.page_table = synth.page_table(cfg, "cuda", 7, permute=False)
    for l in range(cfg.L):
        for b in range(cfg.B):
            src = kv_a.page_table[b].long()
            dst = kv_b.page_table[b].long()
            kv_b.k[l][dst] = kv_a.k[l][src]
            kv_b.v[l][dst] = kv_a.v[l][src]
    dm = runtime.DeviceModel(model, cfg.max_pages * 16)
    toks = synth.start_tokens(cfg, 7)[: cfg.B]
    res = []
    for kv in (kv_a, kv_b, kv_a.clone()):
        dkv = runtime.DeviceKV(kv)
        dec = runtime.Decoder(dm, dkv, cfg.B)
        lg = torch.empty((cfg.B, cfg.V), device="cuda")
        dec.tokens_in.copy_(toks)
        dec.pos.fill_(cfg.ctx)
        dec.step(logits=lg)
        res.append(lg.cpu())
    assert torch.equal(res[0], res[1])
    # kv_a was advanced by the first run; the clone started from the advanced cache,
    # so compare the third run with a fresh copy instead
    kv_c = synth.make_kv(cfg, "cuda", seed=7, permute=True)
    dkv = runtime.DeviceKV(kv_c)
    dec = runtime.Decoder(dm, dkv, cfg.B)
    lg = torch.empty((cfg.B, cfg.V), device="cuda")
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    dec.step(logits=lg)
    assert torch.equal(res[0], lg.cpu())


def test_batch_rows_equal_single_sequence_runs():
    cfg = synth.CONFIGS["tiny"].with_(B=3)
    model = synth.make_model(cfg, "cuda", seed=8)
    kv = synth.make_kv(cfg, "cuda", seed=8)
    dm = runtime.DeviceModel(model, cfg.max_pages * 16)
    toks = synth.start_tokens(cfg, 8)[: cfg.B]
    dkv = runtime.DeviceKV(kv.clone())
    dec = runtime.Decoder(dm, dkv, cfg.B)
    lg = torch.empty((cfg.B, cfg.V), device="cuda")
    dec.tokens_in.copy_(toks)
    dec.pos.fill_(cfg.ctx)
    dec.step(logits=lg)
    for b in range(cfg.B):
        one = kv.clone()
        one.page_table = kv.page_table[b:b + 1].contiguous()
        dkv1 = runtime.DeviceKV(one)
        d1 = runtime.Decoder(dm, dkv1, 1)
        l1 = torch.empty((1, cfg.V), device="cuda")
        d1.tokens_in.copy_(toks[b:b + 1])
        d1.pos.fill_(cfg.ctx)
        d1.step(logits=l1)
        assert rel_err(lg[b].cpu().numpy(), l1[0].cpu().numpy()) < TOL
        assert int(dec.tokens_out[b]) == int(d1.tokens_out[0]) or \
            oracle.argmax(l1[0].cpu().numpy())[1] <= MARGIN


@pytest.mark.slow
def test_7b_full_model_two_steps():
    """The benchmark workload itself: all 28 layers at full size, two steps."""
    cfg = synth.CONFIGS["7b"]
    _run_steps(cfg, 2, check_kv=False)


@pytest.mark.slow
def test_moe_full_size_layers_batch32():
    """35B-A3B-class shapes (256 experts, top-8, shared expert), B = 32, two layers."""
    cfg = synth.CONFIGS["moe"].with_(L=2)
    _run_steps(cfg, 1, n_layers=2, check_kv=False)


@pytest.mark.slow
@pytest.mark.parametrize("name,layers", [("9b", 3), ("27b", 2), ("9b_b32", 2)])
def test_full_size_layers_nvfp4(name, layers):
    """Full-size layer shapes of the NVFP4 models (a few layers, one step)."""
    cfg = synth.CONFIGS[name].with_(L=layers)
    _run_steps(cfg, 1, n_layers=layers, check_kv=False)
