"""GPU parity of the speculative verify pass (bw_decode_step with n_rows = K+1)
and its acceptance step (bw_spec_accept) against the CPU oracle.

The oracle of a verify pass is plain sequential decoding: row r of the pass
(token rows[r] at position pos + r) must give the logits of the oracle's
single-token step on the same token after rows 0..r-1 were decoded one by one
("bw24" deep-dive page, section 1: speculative output equals greedy output;
section 5, stage 4: the drafts run as rows over one shared cache)."""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import MARGIN, TOL, check_kv, parallel_rows, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


def _setup(cfg, seed, n_layers=None):
    model = synth.make_model(cfg, "cuda", seed=seed, n_layers=n_layers)
    kv = synth.make_kv(cfg, "cuda", seed=seed, n_layers=n_layers)
    om = oracle.Model(model)
    okv = oracle.KV(kv)
    dm = runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS)
    dkv = runtime.DeviceKV(kv)
    return model, kv, om, okv, dm, dkv


def _verify_vs_oracle(cfg, K, seed, n_layers=None, drafts=None):
    """One verify pass of K drafts for every sequence; returns GPU tokens_out,
    oracle margins and the rows that ran."""
    B, R = cfg.B, K + 1
    model, kv, om, okv, dm, dkv = _setup(cfg, seed, n_layers)
    dec = runtime.Decoder(dm, dkv, B, n_rows=R)
    t0 = synth.start_tokens(cfg, seed)[:B].tolist()
    if drafts is None:
        drafts = synth.draft_tokens(cfg, K, seed)[:B].tolist()
    rows = [[t0[b]] + list(drafts[b]) for b in range(B)]
    dec.tokens_in.copy_(torch.tensor(sum(rows, []), dtype=torch.int32))
    dec.pos.fill_(cfg.ctx)
    logits = torch.empty((B * R, cfg.V), device="cuda")
    dec.step(logits=logits)
    assert bw.read_error(dec.ws) == 0
    lg = logits.cpu().numpy()
    got = dec.tokens_out.cpu().tolist()
    def seq_rows(b):
        # the rows of one sequence run in order: row r reads the K/V rows 0..r-1 wrote
        return [oracle.decode_token(om, okv, b, rows[b][r], cfg.ctx + r) for r in range(R)]

    margins = []
    for b, ress in enumerate(parallel_rows(seq_rows, range(B))):
        for r, res in enumerate(ress):
            err = rel_err(lg[b * R + r], res["logits"])
            assert err < TOL, (b, r, err)
            assert got[b * R + r] == int(np.argmax(lg[b * R + r]))
            if res["margin"] > MARGIN:
                assert got[b * R + r] == res["token"], (b, r, res["margin"])
            margins.append(res["margin"])
    # every row wrote its K/V at its own position, as sequential decoding does
    check_kv(list(dkv.k) + list(dkv.v), list(okv.k) + list(okv.v), dkv.page_table, B, cfg.ctx, R)
    return dec, rows, got, margins


def test_verify_pass_rows_match_sequential_oracle_tiny():
    cfg = synth.CONFIGS["tiny"].with_(B=2)
    _verify_vs_oracle(cfg, K=3, seed=21)


def test_verify_pass_nvfp4_two_layers_k7():
    cfg = synth.CONFIGS["tiny"].with_(fmt=synth.FMT_NVFP4, L=2, B=1)
    _verify_vs_oracle(cfg, K=7, seed=22)


def test_verify_with_greedy_drafts_accepts_all():
    """Drafts = the oracle's own greedy continuation: every draft stands (rows
    whose oracle margin is under the margin rule may legitimately differ)."""
    cfg = synth.CONFIGS["tiny"].with_(B=2)
    K = 3
    _, _, om, okv, _, _ = _setup(cfg, 23)
    t0 = synth.start_tokens(cfg, 23)[: cfg.B].tolist()
    drafts, clear = [], []
    for b in range(cfg.B):
        seq, ok = [t0[b]], True
        for r in range(K):
            res = oracle.decode_token(om, okv, b, seq[-1], cfg.ctx + r)
            ok = ok and res["margin"] > MARGIN
            seq.append(res["token"])
        drafts.append(seq[1:])
        clear.append(ok)
    dec, rows, got, _ = _verify_vs_oracle(cfg, K, 23, drafts=drafts)
    n_acc = torch.empty(cfg.B, dtype=torch.int32, device="cuda")
    nxt = torch.empty(cfg.B, dtype=torch.int32, device="cuda")
    bw.spec_accept(dec.tokens_in, dec.tokens_out, cfg.B, K + 1, n_acc, nxt)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        want = oracle.spec_accept(rows[b], got[b * (K + 1):(b + 1) * (K + 1)])
        assert (int(n_acc[b]), int(nxt[b])) == want
        if clear[b]:
            assert want[0] == K


def test_spec_accept_kernel_matches_oracle():
    """bw_spec_accept on planted token patterns, every n_rows, bit-exact;
    next token written in place into the next pass's first row; positions."""
    rng = np.random.default_rng(5)
    for R in range(1, bw.MAX_VERIFY_ROWS + 1):
        B = 37
        greedy = rng.integers(0, 50, size=(B, R)).astype(np.int32)
        rows = rng.integers(0, 50, size=(B, R)).astype(np.int32)
        for b in range(B):
            n = int(rng.integers(0, R))          # plant n matching drafts
            rows[b, 1:n + 1] = greedy[b, :n]
        ti = torch.from_numpy(rows.reshape(-1)).cuda()
        to = torch.from_numpy(greedy.reshape(-1)).cuda()
        n_acc = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        pos = torch.arange(B, dtype=torch.int32, device="cuda") * 100
        bw.spec_accept(ti, to, B, R, n_acc, next_out=ti, next_stride=R, pos=pos)
        torch.cuda.synchronize()
        ti_h = ti.cpu().numpy().reshape(B, R)
        for b in range(B):
            n, nxt = oracle.spec_accept(rows[b], greedy[b])
            assert int(n_acc[b]) == n
            assert int(pos[b]) == 100 * b + n + 1
            assert ti_h[b, 0] == nxt
            assert (ti_h[b, 1:] == rows[b, 1:]).all()


def test_spec_accept_rejects_bad_arguments():
    t = torch.zeros(8, dtype=torch.int32, device="cuda")
    with pytest.raises(bw.BWError):
        bw.spec_accept(t, t, 1, bw.MAX_VERIFY_ROWS + 1, t)
    with pytest.raises(bw.BWError):
        bw.spec_accept(t, t, 0, 1, t)
    with pytest.raises(bw.BWError):
        bw.spec_accept(t, t, 1, 2, t, next_out=t, next_stride=0)


@pytest.mark.slow
def test_verify_pass_27b_full_size_layers():
    """27B-class shapes (64/8 heads x 128, NVFP4), verify of K = 3 drafts, two layers."""
    cfg = synth.CONFIGS["27b"].with_(L=2)
    _verify_vs_oracle(cfg, K=3, seed=0, n_layers=2)
