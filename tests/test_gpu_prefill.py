"""GPU parity of chunked prefill (bw_prefill) against the CPU oracle.

The "bw24" deep-dive page, section 5, stage 3, pushes a prompt through in
chunks, one after another, each updating the KV cache, with logits returned
only for the last chunk.  Its oracle is plain token-by-token decoding of the
same prompt at the same positions: afterwards the cache holds every prompt
row's K/V at its position (every other slot untouched), and the result is the
greedy token -- and the logits -- after the last prompt token."""
import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import bw, runtime, synth
from gpu_util import MARGIN, TOL, check_kv, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_decode_b200 import build
    build.build()
    bw.lib()


def _setup(cfg, seed, n_layers=None):
    model = synth.make_model(cfg, "cuda", seed=seed, n_layers=n_layers)
    kv = synth.make_kv(cfg, "cuda", seed=seed, n_layers=n_layers)
    om, okv = oracle.Model(model), oracle.KV(kv)
    dm = runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS)
    dkv = runtime.DeviceKV(kv)
    return om, okv, dm, dkv


def _prefill_vs_oracle(cfg, n, chunk, seed, n_layers=None):
    om, okv, dm, dkv = _setup(cfg, seed, n_layers)
    prompt = synth.prompt_tokens(cfg, n, seed)
    pf = runtime.Prefiller(dm, dkv, chunk)
    logits = torch.empty(cfg.V, device="cuda")
    nxt = pf.run(prompt.to("cuda"), cfg.ctx, logits=logits)
    torch.cuda.synchronize()
    assert bw.read_error(pf.ws) == 0
    res = None
    for i, t in enumerate(prompt.tolist()):
        res = oracle.decode_token(om, okv, 0, t, cfg.ctx + i)
    lg = logits.cpu().numpy()
    assert rel_err(lg, res["logits"]) < TOL
    got = int(nxt.item())
    assert got == int(np.argmax(lg))
    if res["margin"] > MARGIN:
        assert got == res["token"], res["margin"]
    check_kv(list(dkv.k) + list(dkv.v), list(okv.k) + list(okv.v), dkv.page_table, 1, cfg.ctx, n)


@pytest.mark.parametrize("n,chunk", [(37, 3), (37, 8), (16, 8), (1, 4), (5, 1)])
def test_prefill_tiny_matches_sequential_decoding(n, chunk):
    # ragged last chunks, exact multiples, a one-token prompt, one row per chunk
    _prefill_vs_oracle(synth.CONFIGS["tiny"].with_(steps=64), n, chunk, seed=3)


def test_prefill_7b_two_layers_chunk4():
    # 7B shape (7 query heads per kv head: at most 4 rows per chunk), CUDA-core projections
    _prefill_vs_oracle(synth.CONFIGS["7b"], 13, 4, seed=5, n_layers=2)


def test_prefill_9b_nvfp4_two_layers_chunk8():
    # 8 rows per chunk: the NVFP4 projections run on the tensor cores
    _prefill_vs_oracle(synth.CONFIGS["9b"], 11, 8, seed=6, n_layers=2)


def test_prefill_rejects_bad_shapes_before_launching():
    cfg = synth.CONFIGS["7b"]
    om, okv, dm, dkv = _setup(cfg, 1, n_layers=1)
    tokens = synth.prompt_tokens(cfg, 8, 1).to("cuda")
    nxt = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    ws = bw.workspace(bw.prefill_workspace_bytes(dm.c, dkv.c, 8))
    before = [t.clone() for t in dkv.k]
    # 7 query heads per kv head x 5 rows exceeds the attention's 32 query rows
    with pytest.raises(bw.BWError) as e:
        bw.prefill(dm.c, dkv.c, tokens, 8, cfg.ctx, 5, nxt, ws)
    assert e.value.status == bw.ERR_UNSUPPORTED_SHAPE
    with pytest.raises(bw.BWError) as e:
        bw.prefill(dm.c, dkv.c, tokens, 8, cfg.ctx, 9, nxt, ws)
    assert e.value.status == bw.ERR_UNSUPPORTED_SHAPE
    # past the cache
    with pytest.raises(bw.BWError) as e:
        bw.prefill(dm.c, dkv.c, tokens, 8, cfg.max_pages * synth.PAGE_TOKENS - 4, 4, nxt, ws)
    assert e.value.status == bw.ERR_INVALID_ARG
    # a workspace sized for fewer rows
    small = bw.workspace(bw.prefill_workspace_bytes(dm.c, dkv.c, 2))
    with pytest.raises(bw.BWError) as e:
        bw.prefill(dm.c, dkv.c, tokens, 8, cfg.ctx, 4, nxt, small)
    assert e.value.status == bw.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(nxt.item()) == -7
    assert all(torch.equal(a, b) for a, b in zip(before, dkv.k))
