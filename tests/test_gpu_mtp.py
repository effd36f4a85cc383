"""GPU speculative decoding with the MTP draft head (bw_mtp_draft, bw_decode_step
with K + 1 rows, bw_spec_accept) against the CPU oracle.

"bw24" deep-dive page (10100.com): section 7 (a light draft head sharing the
main model's embedding, its vocabulary pruned to the first ids), section 5,
stage 4 (the drafts become the rows of one verify pass) and section 1 (the
speculative output is token for token the plain greedy output)."""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import MARGIN

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


def _setup(cfg, seed):
    model = synth.make_model(cfg, "cuda", seed=seed)
    kv = synth.make_kv(cfg, "cuda", seed=seed)
    head = synth.make_draft_head(cfg, "cuda", seed=seed)
    dm = runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS)
    return model, kv, head, dm


def _margin(z):
    s = np.sort(np.asarray(z, np.float64))
    return float(s[-1] - s[-2])


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_draft_head_matches_oracle(fmt):
    """K drafts from one hidden row: every draft equals the oracle's draft chain
    (z = W_draft rmsnorm(h + E[t]) * norm) until a draft whose oracle top-2
    margin is under the margin rule (either token is then correct)."""
    cfg = synth.CONFIGS["tiny"].with_(fmt=fmt, L=1)
    model, kv, head, dm = _setup(cfg, 41)
    ddh = runtime.DeviceDraftHead(head)
    K = 7
    H = cfg.H
    g = torch.Generator(device="cuda").manual_seed(3)
    hidden = torch.randn((3, H), device="cuda", generator=g)
    row = torch.tensor([2], dtype=torch.int32, device="cuda")
    tokens = torch.zeros(K + 1, dtype=torch.int32, device="cuda")
    tokens[0] = 77
    ws = bw.workspace(bw.mtp_workspace_bytes(dm.c, ddh.c))
    bw.mtp_draft(dm.c, ddh.c, hidden, 3, tokens, K, ws, row=row)
    assert bw.read_error(ws) == 0
    got = tokens.cpu().tolist()
    odh = oracle.DraftHead(head, model.embed, cfg.eps)
    h, t = hidden[2].cpu().numpy(), 77
    for i in range(K):
        t, h, z = oracle.draft_token(odh, h, t)
        assert 0 <= got[i + 1] < cfg.draft_vocab
        if _margin(z) <= MARGIN:
            break
        assert got[i + 1] == t, (i, got, t)
    # a row outside the hidden rows is reported
    bad = torch.tensor([3], dtype=torch.int32, device="cuda")
    bw.mtp_draft(dm.c, ddh.c, hidden, 3, tokens, K, ws, row=bad)
    assert bw.read_error(ws) & bw.DEVERR_BAD_TOKEN


def _greedy_gpu(dm, kv, token, pos, n):
    """Plain greedy GPU decoding of n tokens (logits margins kept)."""
    dkv = runtime.DeviceKV(kv)
    dec = runtime.Decoder(dm, dkv, 1)
    lg = torch.empty((1, dm.cfg.V), device="cuda")
    out, margins = [], []
    for i in range(n):
        dec.tokens_in.fill_(int(token))
        dec.pos.fill_(pos + i)
        dec.step(logits=lg)
        token = int(dec.tokens_out[0])
        out.append(token)
        margins.append(_margin(lg[0].cpu().numpy()))
    return out, margins


def _spec_gpu(dm, kv, ddh, token, pos, n, K, drafts_from=None):
    """GPU speculative loop: emitted tokens and accepted drafts per pass.
    drafts_from: a token list to draft from instead of the draft head."""
    sd = runtime.SpecDecoder(dm, runtime.DeviceKV(kv), ddh, K)
    sd.start(token, pos)
    out = [int(sd.ver.tokens_in[0])]
    accepted = []
    while len(out) < n:
        if drafts_from is None:
            sd.draft()
        else:
            d = (drafts_from[len(out):len(out) + K] + [0] * K)[:K]
            sd.ver.tokens_in[1:].copy_(torch.tensor(d, dtype=torch.int32))
        sd.verify_accept()
        row = sd.ver.tokens_in.cpu().tolist()
        nacc = int(sd.n_acc[0])
        accepted.append(nacc)
        out.extend(row[1:1 + nacc] + [row[0]])
        assert int(sd.ver.pos[0]) == pos + len(out)
    assert bw.read_error(sd.ver.ws) == 0 and bw.read_error(sd.mws) == 0
    return out[:n], accepted


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_speculative_loop_is_greedy(fmt):
    """The speculative loop with the draft head emits the plain greedy sequence
    (up to the first token whose greedy margin is under the margin rule), and
    the oracle's own speculative loop with the same head emits it too."""
    cfg = synth.CONFIGS["tiny"].with_(fmt=fmt, L=2, steps=48)   # cache room for the passes' rows
    model, kv, head, dm = _setup(cfg, 42)
    ddh = runtime.DeviceDraftHead(head)
    tok, pos, n, K = int(synth.start_tokens(cfg, 42)[0]), cfg.ctx, 14, 3
    greedy, margins = _greedy_gpu(dm, kv.clone(), tok, pos, n)
    spec, accepted = _spec_gpu(dm, kv.clone(), ddh, tok, pos, n, K)
    for i in range(n):
        if spec[i] != greedy[i]:
            assert margins[i] <= MARGIN, (i, spec, greedy)
            break
    om, okv = oracle.Model(model), oracle.KV(kv)
    ref = oracle.mtp_generate(om, okv, oracle.DraftHead(head, model.embed, cfg.eps), 0, tok, pos, n, K)
    for i in range(n):
        if ref["tokens"][i] != spec[i]:
            assert margins[i] <= MARGIN, (i, spec, ref["tokens"])
            break
    assert all(0 <= a <= K for a in accepted)


def test_speculative_loop_accepts_correct_drafts():
    """Drafts that are the greedy continuation are all accepted: K + 1 tokens
    per pass, the greedy sequence, positions advanced by K + 1."""
    cfg = synth.CONFIGS["tiny"].with_(L=2, steps=48)
    model, kv, head, dm = _setup(cfg, 43)
    ddh = runtime.DeviceDraftHead(head)
    tok, pos, n, K = int(synth.start_tokens(cfg, 43)[0]), cfg.ctx, 17, 3
    greedy, margins = _greedy_gpu(dm, kv.clone(), tok, pos, n + K)
    spec, accepted = _spec_gpu(dm, kv.clone(), ddh, tok, pos, n, K, drafts_from=greedy)
    clear = all(m > MARGIN for m in margins[:n])
    if clear:
        assert spec == greedy[:n]
        assert accepted == [K] * len(accepted)


def test_speculative_pass_in_cuda_graph():
    """One pass (draft, verify, accept) captured in a CUDA graph and replayed
    gives the same tokens as the eager passes."""
    cfg = synth.CONFIGS["tiny"].with_(L=2, steps=48)
    model, kv, head, dm = _setup(cfg, 44)
    ddh = runtime.DeviceDraftHead(head)
    tok, pos, K, P = int(synth.start_tokens(cfg, 44)[0]), cfg.ctx, 3, 5
    eager = []
    sd = runtime.SpecDecoder(dm, runtime.DeviceKV(kv.clone()), ddh, K)
    sd.start(tok, pos)
    sd.step_pass()
    for _ in range(P):
        sd.step_pass()
        eager.append((sd.ver.tokens_in.cpu().tolist(), int(sd.n_acc[0])))
    sd2 = runtime.SpecDecoder(dm, runtime.DeviceKV(kv.clone()), ddh, K)
    sd2.start(tok, pos)
    sd2.step_pass()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    rows = torch.empty((P, K + 1), dtype=torch.int32, device="cuda")
    nacc = torch.empty(P, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(P):
                sd2.step_pass(stream=s)
                rows[i].copy_(sd2.ver.tokens_in)
                nacc[i].copy_(sd2.n_acc[0])
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    assert [(rows[i].tolist(), int(nacc[i])) for i in range(P)] == eager
