"""Pins of the CPU oracle to facts that do not come from the oracle itself:
library conversions (numpy fp16, torch float8), hand-computed golden blocks,
closed forms, invariants and fp64 brute force on tiny inputs."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from token_decode_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def _float(tok):
    return float("nan") if tok == "nan" else float(tok)


# ------------------------------------------------------------------ formats

def test_fp16_decode_all_codes_match_numpy():
    codes = np.arange(65536, dtype=np.uint16)
    ref = codes.view(np.float16).astype(np.float32)
    got = np.array([oracle.fp16_to_f32(int(c)) for c in codes], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_fp16_encode_round_to_nearest_even_matches_numpy():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10,
        (rng.standard_normal(5000) * 1e-5).astype(np.float32),       # fp16 subnormal range
        (rng.standard_normal(2000) * 7e4).astype(np.float32),        # overflow region
        # exact ties: halfway between fp16 neighbours
        (np.arange(1, 2000, dtype=np.float32) + 0.5) * np.float32(2.0 ** -10),
        np.array([65504, 65519.99, 65520, -65520, 2 ** -25, 2 ** -24 * 1.5, 2 ** -26, 0.0, -0.0,
                  np.inf, -np.inf], np.float32),
    ])
    got = np.array([oracle.f32_to_fp16(float(x)) for x in xs], np.uint16)
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    assert oracle.f32_to_fp16(float("nan")) & 0x7C00 == 0x7C00


def test_e4m3_golden_and_torch():
    for line in _golden_lines("e4m3_codes.txt"):
        code, val = line.split()
        got = oracle.e4m3_to_f32(int(code, 16))
        want = _float(val)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want)
    # every code against torch's float8_e4m3fn conversion
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_to_f32(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e2m1_table():
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        want = mags[c & 7] * (-1 if c & 8 else 1)
        assert oracle.e2m1_to_f32(c) == want


def _qmat(fmt, N, K, q, s=None, ts=1.0):
    return synth.QMat(fmt, N, K, torch.from_numpy(np.array(q, np.uint8)),
                      None if s is None else torch.from_numpy(np.array(s, np.uint8)), ts)


def test_q4_0_golden_blocks():
    for line in _golden_lines("q4_0_blocks.txt"):
        hexs, vals = line.split("|")
        blk = np.frombuffer(bytes.fromhex(hexs.strip()), np.uint8)
        want = np.array([_float(v) for v in vals.split()], np.float32)
        m = _qmat(synth.FMT_Q4_0, 1, 32, blk[None, :])
        got = oracle.dequant(m)[0]
        assert np.array_equal(got, want), (hexs, got, want)


def test_nvfp4_golden_blocks():
    for line in _golden_lines("nvfp4_blocks.txt"):
        lhs, vals = line.split("|")
        codes, sc, ts = lhs.split()
        q = np.frombuffer(bytes.fromhex(codes), np.uint8)
        s = np.frombuffer(bytes.fromhex(sc), np.uint8)
        want = np.array([_float(v) for v in vals.split()], np.float32)
        m = _qmat(synth.FMT_NVFP4, 1, 16, q[None, :], s[None, :], float(ts))
        got = oracle.dequant(m)[0]
        assert np.array_equal(got, want), (lhs, got, want)
        assert np.array_equal(np.signbit(got), np.signbit(want))


# ----------------------------------------------------------------- matvec

def _np_deq_q4_0(m):
    """Independent numpy decode used only by the brute-force pins."""
    b = m.q.numpy().reshape(m.N, m.K // 32, 18)
    d = b[..., :2].copy().view(np.float16).astype(np.float64)          # [N, nb, 1]
    qs = b[..., 2:]
    q = np.concatenate([qs & 15, qs >> 4], axis=-1).astype(np.float64)  # [N, nb, 32]
    return (d * (q - 8)).reshape(m.N, m.K)


_E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])


def _np_deq_nvfp4(m):
    q = m.q.numpy()
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(m.N, m.K)
    s = torch.from_numpy(m.s.numpy().copy()).view(torch.float8_e4m3fn).double().numpy()
    return _E2M1[codes] * np.repeat(s, 16, axis=1) * m.ts


def test_matvec_integer_exact_q4_0():
    """d = 1 and integer x: every product and partial sum is an exact integer
    in fp32, so the result must equal the int64 dot product exactly."""
    rng = np.random.default_rng(1)
    N, K = 7, 96
    q = rng.integers(0, 16, (N, K))
    blocks = np.zeros((N, K // 32, 18), np.uint8)
    blocks[..., 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    qb = q.reshape(N, K // 32, 32)
    blocks[..., 2:] = qb[..., :16] | (qb[..., 16:] << 4)
    x = rng.integers(-20, 21, K)
    m = _qmat(synth.FMT_Q4_0, N, K, blocks.reshape(N, -1))
    got = oracle.matvec(m, x.astype(np.float32))
    want = ((q - 8) * x).sum(axis=1)
    assert np.array_equal(got, want.astype(np.float32))


def test_matvec_integer_exact_nvfp4():
    """scale 2.0, ts 1 and integer x: products are multiples of 1, exact."""
    rng = np.random.default_rng(2)
    N, K = 5, 64
    codes = rng.integers(0, 16, (N, K))
    q = codes[:, 0::2] | (codes[:, 1::2] << 4)
    s = np.full((N, K // 16), 0x40, np.uint8)
    x = rng.integers(-9, 10, K)
    m = _qmat(synth.FMT_NVFP4, N, K, q, s, 1.0)
    got = oracle.matvec(m, x.astype(np.float32))
    want = (_E2M1[codes] * 2 * x).sum(axis=1)
    assert np.array_equal(got, want.astype(np.float32))


@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_matvec_one_hot_is_column_and_brute_force(fmt):
    N, K = 24, 128
    m = synth.quantize(synth.randn((N, K), 0.02, "cpu", 0, "mv"), fmt)
    deq = _np_deq_q4_0(m) if fmt == synth.FMT_Q4_0 else _np_deq_nvfp4(m)
    # dequantized rows equal the independent numpy decode (exact in fp64, then
    # one rounding to fp32: e2m1 * e4m3 is exact, so w is one rounded product)
    deq32 = deq.astype(np.float32)
    assert np.array_equal(oracle.dequant(m), deq32)
    for k in (0, 17, 31, 32, 127):
        e = np.zeros(K, np.float32)
        e[k] = 1
        assert np.array_equal(oracle.matvec(m, e), deq32[:, k])
    x = np.random.default_rng(3).standard_normal(K).astype(np.float32)
    got = oracle.matvec(m, x).astype(np.float64)
    want = deq @ x.astype(np.float64)
    assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want)) + 1e-12


# ---------------------------------------------------------- norm, rope, silu

def test_rmsnorm_closed_form_and_scale_invariance():
    H, c, eps = 64, 0.75, 1e-6
    g = np.linspace(0.5, 1.5, H).astype(np.float32)
    y = oracle.rmsnorm(np.full(H, c, np.float32), g, eps)
    want = g.astype(np.float64) * c / math.sqrt(c * c + eps)
    assert np.allclose(y, want, rtol=2e-7, atol=0)
    x = np.random.default_rng(4).standard_normal(H).astype(np.float32)
    for k in (-3, 5):
        a = oracle.rmsnorm(x, g, 0.0)
        b = oracle.rmsnorm(x * np.float32(2.0 ** k), g, 0.0)
        assert np.array_equal(a, b)


def test_rope_identity_pairing_norm_and_closed_form():
    hd, theta = 64, 1e6
    v = np.random.default_rng(5).standard_normal(hd).astype(np.float32)
    assert np.array_equal(oracle.rope(v, 0, theta), v)           # position 0: identity
    e0 = np.zeros(hd, np.float32)
    e0[3] = 1.0
    r = oracle.rope(e0, 777, theta)                              # pairs (i, i + hd/2)
    assert set(np.nonzero(r)[0]) <= {3, 3 + hd // 2}
    for p in (1, 100, 8191):
        r = oracle.rope(v, p, theta)
        n0 = v[: hd // 2] ** 2 + v[hd // 2:] ** 2
        n1 = r[: hd // 2] ** 2 + r[hd // 2:] ** 2
        assert np.allclose(n0, n1, rtol=1e-5)
    # hd = 2: the single pair rotates by exactly pos radians
    r = oracle.rope(np.array([1.0, 0.0], np.float32), 1, theta)
    assert abs(r[0] - math.cos(1.0)) < 1e-7 and abs(r[1] - math.sin(1.0)) < 1e-7
    # last pair: angle = pos * theta^(-(hd-2)/hd)
    i = hd // 2 - 1
    e = np.zeros(hd, np.float32)
    e[i] = 1
    ang = 4096 * theta ** (-2 * i / hd)
    r = oracle.rope(e, 4096, theta)
    assert abs(r[i] - math.cos(ang)) < 1e-6 and abs(r[i + hd // 2] - math.sin(ang)) < 1e-6


def test_silu_special_values():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(20.0) - 20.0) < 1e-5
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-7
    assert abs(oracle.silu(-30.0)) < 1e-10


# ---------------------------------------------------------------- attention

def _kv_case(nkv=2, hd=64, ctx=40, n_pages=None, seed=0, permute=True):
    P = 16
    npg = -(-ctx // P)
    n_pages = npg + 3 if n_pages is None else n_pages
    rng = np.random.default_rng(seed)
    logical_k = rng.standard_normal((ctx, nkv, hd)).astype(np.float16)
    logical_v = rng.standard_normal((ctx, nkv, hd)).astype(np.float16)
    table = rng.permutation(n_pages)[:npg] if permute else np.arange(npg)
    kpool = rng.standard_normal((n_pages, nkv, P, hd)).astype(np.float16)   # garbage elsewhere
    vpool = rng.standard_normal((n_pages, nkv, P, hd)).astype(np.float16)
    for j in range(ctx):
        kpool[table[j // P], :, j % P] = logical_k[j]
        vpool[table[j // P], :, j % P] = logical_v[j]

    class _KV:
        pass
    kv = _KV()
    kv.k = [kpool.view(np.uint16)]
    kv.v = [vpool.view(np.uint16)]
    kv.page_table = table.astype(np.int32)[None, :]
    kv.n_pages = n_pages
    kv.page_tokens = P
    return oracle.KV(kv), logical_k, logical_v


def test_attention_brute_force_fp64():
    kv, lk, lv = _kv_case()
    q = np.random.default_rng(9).standard_normal(64).astype(np.float32)
    for length in (1, 7, 16, 17, 40):
        got = oracle.attend_head(q, kv, 0, 0, 2, 1, length)
        k = lk[:length, 1].astype(np.float64)
        v = lv[:length, 1].astype(np.float64)
        s = k @ q.astype(np.float64) / math.sqrt(64)
        p = np.exp(s - s.max())
        want = (p / p.sum()) @ v
        assert np.max(np.abs(got - want)) < 2e-6 * max(1.0, np.max(np.abs(want)))


def test_attention_special_cases():
    kv, lk, lv = _kv_case(ctx=33)
    q = np.random.default_rng(10).standard_normal(64).astype(np.float32)
    # one position: the output is v_0 exactly
    assert np.array_equal(oracle.attend_head(q, kv, 0, 0, 2, 0, 1), lv[0, 0].astype(np.float32))
    # all keys equal: the output is the mean of V
    kv2, _, lv2 = _kv_case(ctx=33, seed=3)
    for a in kv2.k:
        a[:] = a[0, 0, 0]
    got = oracle.attend_head(q, kv2, 0, 0, 2, 0, 33)
    assert np.allclose(got, lv2[:33, 0].astype(np.float64).mean(0), atol=2e-6)
    # one key aligned with a large q: the output is that key's v
    kv3, lk3, lv3 = _kv_case(ctx=20, seed=4)
    big = (lk3[11, 0].astype(np.float32) * 40)
    got = oracle.attend_head(big, kv3, 0, 0, 2, 0, 20)
    assert np.allclose(got, lv3[11, 0].astype(np.float32), atol=1e-5)


def test_attention_paged_equals_contiguous():
    kv_p, lk, lv = _kv_case(seed=7, permute=True)
    kv_c, lk2, lv2 = _kv_case(seed=7, permute=False)
    assert np.array_equal(lk, lk2)
    q = np.random.default_rng(11).standard_normal(64).astype(np.float32)
    for length in (5, 40):
        a = oracle.attend_head(q, kv_p, 0, 0, 2, 1, length)
        b = oracle.attend_head(q, kv_c, 0, 0, 2, 1, length)
        assert np.array_equal(a, b)


# ------------------------------------------------------------ top-k, argmax

def test_topk_matches_full_sort_with_ties():
    rng = np.random.default_rng(12)
    for trial in range(50):
        r = rng.integers(-4, 5, 64).astype(np.float32) if trial % 2 else rng.standard_normal(64).astype(np.float32)
        idx, w = oracle.topk_softmax(r, 8)
        order = np.lexsort((np.arange(64), -r))[:8]          # value desc, index asc
        assert np.array_equal(idx, order)
        e = np.exp(r[order].astype(np.float64) - r[order].max())
        assert np.allclose(w, e / e.sum(), rtol=1e-6)
    idx, w = oracle.topk_softmax(np.zeros(16, np.float32), 16)
    assert np.array_equal(idx, np.arange(16)) and np.all(w == np.float32(1 / 16))


def test_argmax_planted_and_ties():
    v = np.random.default_rng(13).standard_normal(1000).astype(np.float32)
    v[613] = 9.0
    assert oracle.argmax(v)[0] == 613
    v[200] = 9.0                                    # tie: the lowest index wins
    i, margin = oracle.argmax(v)
    assert i == 200 and margin == 0.0
    v[200] = 8.5
    assert oracle.argmax(v) == (613, 0.5)


# ------------------------------------------------------- quantizer round trip

def test_quantizers_round_trip_within_format_bounds():
    x = synth.randn((16, 256), 0.02, "cpu", 0, "rt")
    m = synth.quantize_q4_0(x)
    deq = oracle.dequant(m)
    b = m.q.numpy().reshape(16, 8, 18)
    dabs = np.abs(b[..., :2].copy().view(np.float16).astype(np.float64))
    err = np.abs(deq.astype(np.float64) - x.numpy()).reshape(16, 8, 32)
    # rounding to the nearest level costs at most d/2; the clamp at q = 15 on the side
    # opposite to the largest element costs at most d; fp16 rounding of d adds 8 * 2^-11 d
    assert np.all(err <= dabs * (1.0 + 2.0 ** -7) + 1e-9)
    assert np.mean(err <= dabs * (0.5 + 2.0 ** -7) + 1e-9) > 0.95
    # the block's largest element is reproduced up to the fp16 rounding of d
    amax_err = np.take_along_axis(err, np.abs(x.numpy()).reshape(16, 8, 32).argmax(-1)[..., None], -1)
    assert np.all(amax_err <= dabs * 8 * 2.0 ** -11 + 1e-9)
    m4 = synth.quantize_nvfp4(x)
    deq4 = oracle.dequant(m4)
    # relative error of E2M1 rounding is at most 1/3 of the value (6 vs 4 spacing) per element,
    # and the block's largest element is reproduced within 1/6 + the E4M3 rounding of the scale
    assert np.max(np.abs(deq4 - x.numpy())) <= 0.25 * float(x.abs().max())
    assert np.linalg.norm(deq4 - x.numpy()) <= 0.2 * np.linalg.norm(x.numpy())


# ------------------------------------------------------- whole decode step

def _np_forward(model, kv_np, b, token, pos, write=True, rows_out=None):
    """fp64 numpy brute force of one decode token on a tiny model (contiguous
    per-position K/V gathered through the page table).  write=False reads the
    new position's K/V from kv_np as given instead of storing it (rounded to
    fp16) first; rows_out, when given, receives each layer's fp64 (k, v)."""
    cfg = model.cfg
    deq = (lambda m: _np_deq_q4_0(m)) if cfg.fmt == synth.FMT_Q4_0 else (lambda m: _np_deq_nvfp4(m))

    def norm(x, g):
        return x / np.sqrt(np.mean(x * x) + cfg.eps) * g.numpy().astype(np.float64)

    def rope(v, p):
        h = cfg.hd // 2
        i = np.arange(h)
        ang = p * cfg.theta ** (-2.0 * i / cfg.hd)
        c, s = np.cos(ang), np.sin(ang)
        a, bb = v[..., :h], v[..., h:]
        return np.concatenate([a * c - bb * s, bb * c + a * s], axis=-1)

    x = deq(model.embed)[token].copy()
    P = 16
    table = kv_np["table"][b]
    for l, ly in enumerate(model.layers):
        y = norm(x, ly.attn_norm)
        qkv = deq(ly.wqkv) @ y
        q = qkv[: cfg.nq * cfg.hd].reshape(cfg.nq, cfg.hd)
        k = qkv[cfg.nq * cfg.hd:(cfg.nq + cfg.nkv) * cfg.hd].reshape(cfg.nkv, cfg.hd)
        v = qkv[(cfg.nq + cfg.nkv) * cfg.hd:].reshape(cfg.nkv, cfg.hd)
        q, k = rope(q, pos), rope(k, pos)
        kp, vp = kv_np["k"][l], kv_np["v"][l]
        if rows_out is not None:
            rows_out[l] = (k.copy(), v.copy())
        if write:
            kp[table[pos // P], :, pos % P] = k.astype(np.float16)
            vp[table[pos // P], :, pos % P] = v.astype(np.float16)
        K = np.stack([kp[table[j // P], :, j % P] for j in range(pos + 1)]).astype(np.float64)
        Vv = np.stack([vp[table[j // P], :, j % P] for j in range(pos + 1)]).astype(np.float64)
        o = np.empty((cfg.nq, cfg.hd))
        for h in range(cfg.nq):
            g = h // (cfg.nq // cfg.nkv)
            s = K[:, g] @ q[h] / math.sqrt(cfg.hd)
            p = np.exp(s - s.max())
            o[h] = (p / p.sum()) @ Vv[:, g]
        x = x + deq(ly.wo) @ o.reshape(-1)
        y = norm(x, ly.ffn_norm)

        def ffn(wg, wu, wd):
            g_ = deq(wg) @ y
            return deq(wd) @ (g_ / (1 + np.exp(-g_)) * (deq(wu) @ y))
        if cfg.n_experts == 0:
            x = x + ffn(ly.wg, ly.wu, ly.wd)
        else:
            r = ly.router.numpy().astype(np.float64) @ y
            sel = np.lexsort((np.arange(cfg.n_experts), -r))[: cfg.topk]
            w = np.exp(r[sel] - r[sel].max())
            w /= w.sum()
            acc = sum(w[i] * ffn(ly.eg.mat(e), ly.eu.mat(e), ly.ed.mat(e)) for i, e in enumerate(sel))
            x = x + acc + ffn(ly.sg, ly.su, ly.sd)
    logits = deq(model.lm_head) @ norm(x, model.final_norm)
    return logits, x


def _tiny_moe():
    return synth.CONFIGS["tiny"].with_(name="tiny-moe", fmt=synth.FMT_NVFP4, F=0, n_experts=8,
                                       topk=2, F_exp=64, ctx=40, steps=4, B=2)


@pytest.mark.parametrize("which", ["tiny", "tiny_nvfp4", "tiny_moe"])
def test_decode_step_matches_fp64_brute_force(which):
    if which == "tiny":
        cfg = synth.CONFIGS["tiny"]
    elif which == "tiny_nvfp4":
        cfg = synth.CONFIGS["tiny"].with_(fmt=synth.FMT_NVFP4, L=2)
    else:
        cfg = _tiny_moe()
    model = synth.make_model(cfg, "cpu", seed=1)
    kv = synth.make_kv(cfg, "cpu", seed=1)
    om = oracle.Model(model)
    okv = oracle.KV(kv)
    kv_np = {"k": [t.numpy().view(np.float16).copy() for t in kv.k],
             "v": [t.numpy().view(np.float16).copy() for t in kv.v],
             "table": kv.page_table.numpy()}
    tok = int(synth.start_tokens(cfg, 1)[0])
    for step in range(3):
        pos = cfg.ctx + step
        res = oracle.decode_token(om, okv, 0, tok, pos, want_hidden=True)
        want_logits, want_x = _np_forward(model, kv_np, 0, tok, pos)
        err = np.max(np.abs(res["logits"] - want_logits)) / np.max(np.abs(want_logits))
        assert err < 2e-5, err
        errx = np.max(np.abs(res["hidden"][-1] - want_x)) / np.max(np.abs(want_x))
        assert errx < 2e-5, errx
        if res["margin"] > 1e-3:
            assert res["token"] == int(np.argmax(want_logits))
        tok = res["token"]


def test_decode_step_paging_batch_and_moe_dense_invariants():
    cfg = _tiny_moe()
    model = synth.make_model(cfg, "cpu", seed=2)
    om = oracle.Model(model)
    kv_perm = synth.make_kv(cfg, "cpu", seed=2, permute=True)
    # identical logical content under the identity page table
    kv_id = kv_perm.clone()
    kv_id.page_table = synth.page_table(cfg, "cpu", 2, permute=False)
    P = 16
    for l in range(cfg.L):
        for b in range(cfg.B):
            for j in range(cfg.max_pages):
                src = int(kv_perm.page_table[b, j])
                dst = int(kv_id.page_table[b, j])
                kv_id.k[l][dst] = kv_perm.k[l][src]
                kv_id.v[l][dst] = kv_perm.v[l][src]
    a, b_, c = oracle.KV(kv_perm), oracle.KV(kv_id), oracle.KV(kv_perm)
    toks = synth.start_tokens(cfg, 2)
    for seq in range(cfg.B):
        r1 = oracle.decode_token(om, a, seq, int(toks[seq]), cfg.ctx)
        r2 = oracle.decode_token(om, b_, seq, int(toks[seq]), cfg.ctx)
        r3 = oracle.decode_token(om, c, seq, int(toks[seq]), cfg.ctx, moe_dense=True)
        assert np.array_equal(r1["logits"], r2["logits"])          # paged == contiguous
        assert np.array_equal(r1["logits"], r3["logits"])          # sparse == dense experts
        assert np.array_equal(r1["moe_idx"], r3["moe_idx"])
    del P


def test_moe_all_experts_equal_weights_is_dense_mixture():
    """topk = E with a zero router: every expert gets weight 1/E, so the block
    output is the plain average of all expert FFNs plus the shared expert."""
    cfg = _tiny_moe().with_(topk=8, B=1, L=1)
    model = synth.make_model(cfg, "cpu", seed=3)
    model.layers[0].router = torch.zeros_like(model.layers[0].router)
    kv = synth.make_kv(cfg, "cpu", seed=3)
    kv_np = {"k": [t.numpy().view(np.float16).copy() for t in kv.k],
             "v": [t.numpy().view(np.float16).copy() for t in kv.v],
             "table": kv.page_table.numpy()}
    res = oracle.decode_token(oracle.Model(model), oracle.KV(kv), 0, 5, cfg.ctx, want_hidden=True)
    _, want_x = _np_forward(model, kv_np, 0, 5, cfg.ctx)
    assert np.max(np.abs(res["hidden"][-1] - want_x)) < 2e-5 * np.max(np.abs(want_x))
    assert sorted(res["moe_idx"][0].tolist()) == list(range(8))


# --------------------------------------------------------- speculative verify

def test_spec_accept_golden():
    """Hand-worked acceptance cases (tests/golden/spec_accept.txt)."""
    n_cases = 0
    for line in _golden_lines("spec_accept.txt"):
        rows, greedy, want = (part.split() for part in line.split("|"))
        got = oracle.spec_accept([int(t) for t in rows], [int(t) for t in greedy])
        assert got == (int(want[0]), int(want[1])), line
        n_cases += 1
    assert n_cases == 6


def test_spec_accept_reproduces_greedy_sequence():
    """The section-1 invariant by brute force: with a deterministic next-token
    function standing in for the model, the tokens a verify pass emits
    (accepted drafts, then the next token) are exactly the next tokens of
    plain sequential greedy decoding, for drafts that are right, partly right
    or wrong."""
    rng = np.random.default_rng(11)
    V = 7

    def greedy_next(prefix):
        h = 2166136261
        for t in prefix:
            h = ((h ^ int(t)) * 16777619) & 0xFFFFFFFF
        return h % V

    for _ in range(400):
        ctx = list(rng.integers(0, V, size=int(rng.integers(1, 5))))
        K = int(rng.integers(0, 7))
        truth = []
        seq = list(ctx)
        for _ in range(K + 1):
            seq.append(greedy_next(seq))
            truth.append(seq[-1])
        # drafts: the true continuation with random corruptions
        drafts = [t if rng.random() < 0.7 else int(rng.integers(0, V)) for t in truth[:K]]
        rows = [ctx[-1]] + drafts
        greedy = [greedy_next(ctx + drafts[:r]) for r in range(K + 1)]
        n, nxt = oracle.spec_accept(rows, greedy)
        emitted = drafts[:n] + [nxt]
        assert emitted == truth[: n + 1]
        # maximal: the next draft, if any, was wrong
        if n < K:
            assert drafts[n] != truth[n]


# ------------------------------------------------------- speculative drafting

@pytest.mark.parametrize("fmt", [synth.FMT_Q4_0, synth.FMT_NVFP4])
def test_draft_head_matches_fp64_brute_force(fmt):
    """The draft head, g = rmsnorm(h + E[tok]) * norm and z = W_draft g over the
    pruned vocabulary, against an fp64 evaluation with the test's own
    dequantizers."""
    cfg = synth.CONFIGS["tiny"].with_(fmt=fmt)
    model = synth.make_model(cfg, "cpu", seed=4)
    head = synth.make_draft_head(cfg, "cpu", seed=4)
    dh = oracle.DraftHead(head, model.embed, cfg.eps)
    deq = _np_deq_q4_0 if fmt == synth.FMT_Q4_0 else _np_deq_nvfp4
    E, W = deq(model.embed), deq(head.w)
    assert W.shape == (cfg.draft_vocab, cfg.H) and cfg.draft_vocab < cfg.V
    gam = head.norm.numpy().astype(np.float64)
    rng = np.random.default_rng(4)
    for tok in (0, 17, cfg.V - 1):
        h = rng.standard_normal(cfg.H).astype(np.float32) * 3
        d, g, z = oracle.draft_token(dh, h, tok)
        x = h.astype(np.float64) + E[tok]
        want_g = x / np.sqrt(np.mean(x * x) + cfg.eps) * gam
        want_z = W @ want_g
        assert np.max(np.abs(g - want_g)) < 2e-6 * np.max(np.abs(want_g))
        assert np.max(np.abs(z - want_z)) < 2e-5 * np.max(np.abs(want_z))
        assert 0 <= d < cfg.draft_vocab and z[d] == z.max() and d == int(np.argmax(z))
        top2 = np.sort(want_z)[-2:]
        if top2[1] - top2[0] > 1e-3:
            assert d == int(np.argmax(want_z))


def _mtp_setup(seed):
    cfg = synth.CONFIGS["tiny"].with_(steps=32)
    model = synth.make_model(cfg, "cpu", seed=seed)
    kv = synth.make_kv(cfg, "cpu", seed=seed)
    head = synth.make_draft_head(cfg, "cpu", seed=seed)
    om = oracle.Model(model)
    return cfg, model, kv, om, oracle.DraftHead(head, model.embed, cfg.eps)


@pytest.mark.parametrize("k", [1, 3, 5])
def test_mtp_output_is_the_greedy_output(k):
    """The section-1 gate on the oracle's own model: speculative decoding with
    the draft head emits exactly the tokens of plain greedy decoding."""
    cfg, model, kv, om, dh = _mtp_setup(5)
    tok, n = int(synth.start_tokens(cfg, 5)[0]), 12
    want = oracle.greedy_generate(om, oracle.KV(kv), 0, tok, cfg.ctx, n)
    got = oracle.mtp_generate(om, oracle.KV(kv), dh, 0, tok, cfg.ctx, n, k)
    assert got["tokens"] == want
    assert all(0 <= a <= k for a in got["accepted"])
    assert 1 + sum(a + 1 for a in got["accepted"]) >= n


def test_mtp_pass_counts_for_perfect_and_hopeless_drafts():
    """Drafts that are the true continuation are all accepted (K + 1 tokens per
    pass); drafts that are all wrong are all rejected (one token per pass); the
    output is the greedy output either way."""
    cfg, model, kv, om, dh = _mtp_setup(6)
    tok, n, k = int(synth.start_tokens(cfg, 6)[0]), 13, 3
    truth = oracle.greedy_generate(om, oracle.KV(kv), 0, tok, cfg.ctx, n + k + 1)
    first = cfg.ctx + 1          # position of the token the first verify pass starts from

    def perfect(t0, p, h, kk):
        i = p - first            # truth[i] is the token at position p
        assert truth[i] == t0
        return truth[i + 1: i + 1 + kk]

    def hopeless(t0, p, h, kk):
        i = p - first
        return [(t + 1) % cfg.V for t in truth[i + 1: i + 1 + kk]]

    got = oracle.mtp_generate(om, oracle.KV(kv), dh, 0, tok, cfg.ctx, n, k, drafter=perfect)
    assert got["tokens"] == truth[:n]
    assert got["accepted"] == [k] * got["passes"] and got["passes"] == math.ceil((n - 1) / (k + 1))
    got = oracle.mtp_generate(om, oracle.KV(kv), dh, 0, tok, cfg.ctx, n, k, drafter=hopeless)
    assert got["tokens"] == truth[:n]
    assert got["accepted"] == [0] * (n - 1)


# ------------------------------------------------------- FP8 (E4M3) KV cache

def test_e4m3_encoder_matches_torch_and_saturates():
    """The E4M3 encoder against torch's float8_e4m3fn conversion (round to
    nearest even) below the overflow midpoint 464; every code round-trips;
    magnitudes from 464 up saturate to 448 where torch gives NaN; NaN stays NaN."""
    codes = [c for c in range(256) if c & 0x7F != 0x7F]
    for c in codes:
        assert oracle.f32_to_e4m3(oracle.e4m3_to_f32(c)) == c, c
    vals = np.array([oracle.e4m3_to_f32(c) for c in range(0x7F)], np.float64)   # ascending magnitudes
    mids = (vals[:-1] + vals[1:]) / 2                                           # exact ties
    rng = np.random.default_rng(8)
    xs = np.concatenate([mids, -mids, rng.standard_normal(4000) * 30, rng.standard_normal(2000) * 0.01,
                         rng.uniform(-463.9, 463.9, 2000), [0.0, 2.0 ** -10, 3 * 2.0 ** -11, 447.9, 463.99]])
    xs = xs.astype(np.float32)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3(float(x)) for x in xs], np.uint8)
    assert np.array_equal(got, want)
    for x, c in ((464.0, 0x7E), (1e6, 0x7E), (float("inf"), 0x7E), (-500.0, 0xFE)):
        assert oracle.f32_to_e4m3(x) == c
    assert oracle.f32_to_e4m3(float("nan")) & 0x7F == 0x7F


def test_attention_over_e4m3_cache_matches_fp64_brute_force():
    """A query head over an FP8 cache with per-layer K and V scales, through a
    permuted page table, against fp64 softmax attention over torch's decoding
    of the same codes times the scales."""
    rng = np.random.default_rng(9)
    n_pages, nkv, P, hd, max_pages = 12, 2, 16, 64, 6
    kq = rng.integers(0, 256, size=(n_pages, nkv, P, hd), dtype=np.uint8)
    vq = rng.integers(0, 256, size=(n_pages, nkv, P, hd), dtype=np.uint8)
    kq[(kq & 0x7F) == 0x7F] = 0x30        # no NaN codes in a cache
    vq[(vq & 0x7F) == 0x7F] = 0x31
    table = rng.permutation(n_pages)[: 2 * max_pages].reshape(2, max_pages).astype(np.int32)

    class _KV:
        pass
    kv = _KV()
    kv.k = [torch.zeros((n_pages, nkv, P, hd), dtype=torch.int16)]
    kv.v = [torch.zeros((n_pages, nkv, P, hd), dtype=torch.int16)]
    kv.page_table = torch.from_numpy(table)
    kv.n_pages, kv.page_tokens = n_pages, P
    okv = oracle.KV(kv)
    dec = lambda a: torch.from_numpy(a.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    kf, vf = dec(kq), dec(vq)
    ks, vs = 0.0625, 0.03
    for b, kvh, length in ((0, 0, 1), (1, 1, 37), (1, 0, 90)):
        q = rng.standard_normal(hd).astype(np.float32)
        got = oracle.attend_head_e4m3(q, kq, vq, ks, vs, okv, b, nkv, kvh, length)
        K = np.stack([kf[table[b, j // P], kvh, j % P] for j in range(length)]) * ks
        V = np.stack([vf[table[b, j // P], kvh, j % P] for j in range(length)]) * vs
        s = K @ q.astype(np.float64) / math.sqrt(hd)
        p = np.exp(s - s.max())
        want = (p / p.sum()) @ V
        assert np.max(np.abs(got - want)) < 1e-5 * max(1.0, np.max(np.abs(want))), (b, kvh, length)


def test_decode_step_over_fp8_cache_matches_fp64_brute_force():
    """Whole decode steps over the FP8 cache: the row each step writes is the
    E4M3 rounding (torch float8) of k / scale and v / scale, and the logits
    and hidden state match the fp64 forward over the same stored values."""
    cfg = synth.CONFIGS["tiny"].with_(L=2)
    model = synth.make_model(cfg, "cpu", seed=7)
    kv = synth.make_kv_fp8(cfg, "cpu", seed=7)
    om, okv = oracle.Model(model), oracle.KV(kv)
    ks, vs = kv.k_scale.numpy().astype(np.float64), kv.v_scale.numpy().astype(np.float64)

    def dec8(a, s):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).to(torch.float64).numpy() * s

    def enc8(x, s):
        t = torch.from_numpy((x / s).astype(np.float32)).clamp(-448.0, 448.0)
        return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    table = kv.page_table.numpy()
    tok = int(synth.start_tokens(cfg, 7)[0])
    for step in range(3):
        pos = cfg.ctx + step
        res = oracle.decode_token(om, okv, 0, tok, pos, want_hidden=True)
        kv_np = {"k": [dec8(okv.k[l], ks[l]) for l in range(cfg.L)],
                 "v": [dec8(okv.v[l], vs[l]) for l in range(cfg.L)], "table": table}
        rows = {}
        want_logits, want_x = _np_forward(model, kv_np, 0, tok, pos, write=False, rows_out=rows)
        assert np.max(np.abs(res["logits"] - want_logits)) < 2e-5 * np.max(np.abs(want_logits))
        assert np.max(np.abs(res["hidden"][-1] - want_x)) < 2e-5 * np.max(np.abs(want_x))
        page, slot = table[0, pos // 16], pos % 16
        mism = 0
        for l in range(cfg.L):
            k, v = rows[l]
            for got, want in ((okv.k[l][page, :, slot], enc8(k, ks[l])), (okv.v[l][page, :, slot], enc8(v, vs[l]))):
                mism += int(np.sum(got != want))
                # a value within fp32 rounding of a tie may land on the neighbouring code
                assert np.all(np.abs(got.astype(np.int32) - want.astype(np.int32)) <= 1)
        assert mism <= 1
        tok = res["token"]
