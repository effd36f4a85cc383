"""ctypes wrapper of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by
the benchmark's CPU-baseline / reference leg -- never by the GPU library.  It
imports nothing from the GPU package; it takes any objects with the attribute
names of the seeded inputs (fmt, N, K, q, s, ts for a matrix; the layer and
model fields listed in oracle.h).

Every function here marshals arguments or sequences oracle calls (the
generation loops); the arithmetic is in oracle.c.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FMT_Q4_0 = 0
FMT_NVFP4 = 1


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C11, -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))):
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", _LIB, _SRC, "-lm"])
    return _LIB


class QMatC(C.Structure):
    _fields_ = [("fmt", C.c_int), ("N", C.c_int), ("K", C.c_int),
                ("q", C.c_void_p), ("s", C.c_void_p), ("ts", C.c_float)]


class LayerC(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("ffn_norm", C.c_void_p),
                ("wqkv", QMatC), ("wo", QMatC), ("wg", QMatC), ("wu", QMatC), ("wd", QMatC),
                ("router", C.c_void_p), ("eg", C.c_void_p), ("eu", C.c_void_p), ("ed", C.c_void_p),
                ("sg", QMatC), ("su", QMatC), ("sd", QMatC)]


class ModelC(C.Structure):
    _fields_ = [("L", C.c_int), ("H", C.c_int), ("nq", C.c_int), ("nkv", C.c_int), ("hd", C.c_int),
                ("F", C.c_int), ("V", C.c_int), ("n_experts", C.c_int), ("topk", C.c_int),
                ("F_exp", C.c_int), ("eps", C.c_float), ("theta", C.c_float),
                ("embed", QMatC), ("lm_head", QMatC), ("final_norm", C.c_void_p),
                ("layers", C.c_void_p)]


class KVC(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("n_pages", C.c_int),
                ("page_tokens", C.c_int), ("page_table", C.c_void_p), ("max_pages", C.c_int),
                ("kv_fmt", C.c_int), ("k_scale", C.c_void_p), ("v_scale", C.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        f = C.c_float
        p = C.c_void_p
        i = C.c_int
        sig = {
            "or_fp16_to_f32": (f, [C.c_uint16]),
            "or_f32_to_fp16": (C.c_uint16, [f]),
            "or_e4m3_to_f32": (f, [C.c_uint8]),
            "or_e2m1_to_f32": (f, [C.c_uint8]),
            "or_f32_to_e4m3": (C.c_uint8, [f]),
            "or_attend_head_e4m3": (None, [p, p, p, f, f, p, i, i, i, i, i, p]),
            "or_dequant_row": (None, [p, i, p]),
            "or_matvec": (None, [p, p, p]),
            "or_rmsnorm": (None, [p, p, i, f, p]),
            "or_rope": (None, [p, i, i, f]),
            "or_silu": (f, [f]),
            "or_attend_head": (None, [p, p, p, p, i, i, i, i, i, p]),
            "or_topk_softmax": (None, [p, i, i, p, p]),
            "or_argmax": (C.c_int32, [p, i, p]),
            "or_spec_accept": (C.c_int32, [p, p, i, p]),
            "or_draft_token": (C.c_int32, [p, p, p, f, p, C.c_int32, p, p]),
            "or_decode_token": (C.c_int32, [p, p, i, C.c_int32, i, i, p, p, p, p, p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _np(t, dtype=None):
    """torch tensor or array -> contiguous numpy array on the host."""
    if hasattr(t, "detach"):
        t = t.detach().cpu().numpy()
    a = np.ascontiguousarray(t)
    return a if dtype is None else a.view(dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


class QMat:
    """Host copy of one quantized matrix, kept alive for the C structs."""

    def __init__(self, m):
        self.fmt, self.N, self.K, self.ts = int(m.fmt), int(m.N), int(m.K), float(m.ts)
        self.q = _np(m.q, np.uint8)
        self.s = None if getattr(m, "s", None) is None else _np(m.s, np.uint8)
        self.c = QMatC(self.fmt, self.N, self.K, _ptr(self.q).value,
                       None if self.s is None else _ptr(self.s).value, self.ts)


def _empty_qmat() -> QMatC:
    return QMatC(0, 0, 0, None, None, 0.0)


# ------------------------------------------------------------ component API

def fp16_to_f32(h: int) -> float:
    return lib().or_fp16_to_f32(h)


def f32_to_fp16(x: float) -> int:
    return lib().or_f32_to_fp16(x)


def e4m3_to_f32(c: int) -> float:
    return lib().or_e4m3_to_f32(c)


def e2m1_to_f32(c: int) -> float:
    return lib().or_e2m1_to_f32(c)


def f32_to_e4m3(x: float) -> int:
    return int(lib().or_f32_to_e4m3(x))


def dequant(m, rows=None) -> np.ndarray:
    """Dequantized rows of m (all rows by default) as float32 [len(rows), K]."""
    qm = m if isinstance(m, QMat) else QMat(m)
    rows = range(qm.N) if rows is None else rows
    out = np.empty((len(rows), qm.K), np.float32)
    for r, n in enumerate(rows):
        lib().or_dequant_row(C.byref(qm.c), int(n), _ptr(out[r]))
    return out


def matvec(m, x) -> np.ndarray:
    qm = m if isinstance(m, QMat) else QMat(m)
    x = _np(x).astype(np.float32)
    y = np.empty(qm.N, np.float32)
    lib().or_matvec(C.byref(qm.c), _ptr(x), _ptr(y))
    return y


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    x = _np(x).astype(np.float32)
    g = _np(gamma).astype(np.float32)
    y = np.empty_like(x)
    lib().or_rmsnorm(_ptr(x), _ptr(g), x.size, eps, _ptr(y))
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    v = _np(v).astype(np.float32).copy()
    lib().or_rope(_ptr(v), v.size, pos, theta)
    return v


def silu(z: float) -> float:
    return lib().or_silu(z)


class KV:
    """Host copy of the paged KV cache (fp16 bits per layer, or E4M3 bytes with
    per-layer scales when the input carries k_scale / v_scale) + page table."""

    def __init__(self, kv, layers=None):
        L = len(kv.k) if layers is None else layers
        self.fp8 = getattr(kv, "k_scale", None) is not None
        elem = np.uint8 if self.fp8 else np.uint16
        self.k = [_np(kv.k[l], elem).copy() for l in range(L)]
        self.v = [_np(kv.v[l], elem).copy() for l in range(L)]
        self.page_table = _np(kv.page_table, np.int32).copy()
        self.n_pages = int(kv.n_pages)
        self.page_tokens = int(kv.page_tokens)
        self._kp = (C.c_void_p * L)(*[_ptr(a).value for a in self.k])
        self._vp = (C.c_void_p * L)(*[_ptr(a).value for a in self.v])
        self.k_scale = _np(kv.k_scale).astype(np.float32)[:L].copy() if self.fp8 else None
        self.v_scale = _np(kv.v_scale).astype(np.float32)[:L].copy() if self.fp8 else None
        self.c = KVC(C.cast(self._kp, C.c_void_p), C.cast(self._vp, C.c_void_p), self.n_pages,
                     self.page_tokens, _ptr(self.page_table).value, self.page_table.shape[1],
                     1 if self.fp8 else 0,
                     _ptr(self.k_scale).value if self.fp8 else None,
                     _ptr(self.v_scale).value if self.fp8 else None)


def attend_head(q, kv: KV, layer: int, b: int, nkv: int, kvh: int, length: int) -> np.ndarray:
    q = _np(q).astype(np.float32)
    out = np.empty_like(q)
    lib().or_attend_head(_ptr(q), _ptr(kv.k[layer]), _ptr(kv.v[layer]), C.byref(kv.c), b, nkv,
                         kvh, q.size, length, _ptr(out))
    return out


def attend_head_e4m3(q, kpool, vpool, k_scale: float, v_scale: float, kv: KV, b: int, nkv: int, kvh: int,
                     length: int) -> np.ndarray:
    """One query head over an E4M3 cache (byte pools [n_pages][nkv][16][hd] laid
    out like the fp16 ones, behind kv's page table)."""
    q = _np(q).astype(np.float32)
    kp = _np(kpool, np.uint8)
    vp = _np(vpool, np.uint8)
    out = np.empty_like(q)
    lib().or_attend_head_e4m3(_ptr(q), _ptr(kp), _ptr(vp), float(k_scale), float(v_scale), C.byref(kv.c), b, nkv,
                              kvh, q.size, length, _ptr(out))
    return out


def topk_softmax(r, k: int):
    r = _np(r).astype(np.float32)
    idx = np.empty(k, np.int32)
    w = np.empty(k, np.float32)
    lib().or_topk_softmax(_ptr(r), r.size, k, _ptr(idx), _ptr(w))
    return idx, w


def argmax(v):
    v = _np(v).astype(np.float32)
    margin = np.zeros(1, np.float32)
    i = lib().or_argmax(_ptr(v), v.size, _ptr(margin))
    return int(i), float(margin[0])


def spec_accept(rows, greedy):
    """(n accepted drafts, next token) of one verify pass; rows = [t0, d1..dK],
    greedy = the greedy token after each row."""
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    g = np.ascontiguousarray(np.asarray(greedy, dtype=np.int32))
    assert r.size == g.size and r.size >= 1
    nxt = np.zeros(1, np.int32)
    n = lib().or_spec_accept(_ptr(r), _ptr(g), r.size, _ptr(nxt))
    return int(n), int(nxt[0])


class DraftHead:
    """Host copy of a speculative draft head (norm gains [H], W_draft [V_draft][H])
    next to the main model's embedding, which it shares."""

    def __init__(self, head, embed, eps: float):
        self.norm = _np(head.norm).astype(np.float32)
        self.w = QMat(head.w)
        self.embed = embed if isinstance(embed, QMat) else QMat(embed)
        self.eps = float(eps)


def draft_token(dh: DraftHead, h, tok: int):
    """One draft: (token, g, z) with g = rmsnorm(h + deq(E)[tok]) * norm, the
    hidden the next draft starts from, and z the draft logits [V_draft]."""
    h = _np(h).astype(np.float32)
    g = np.empty(dh.embed.K, np.float32)
    z = np.empty(dh.w.N, np.float32)
    d = lib().or_draft_token(C.byref(dh.embed.c), C.byref(dh.w.c), _ptr(dh.norm), dh.eps, _ptr(h), int(tok),
                             _ptr(g), _ptr(z))
    return int(d), g, z


# --------------------------------------------------------------- the model

class Model:
    """Host copy of a seeded model (attribute layout of the input generator)."""

    def __init__(self, m, n_layers=None):
        cfg = m.cfg
        self.cfg = cfg
        L = len(m.layers) if n_layers is None else n_layers
        keep = []

        def qm(x):
            if x is None:
                return _empty_qmat()
            q = QMat(x)
            keep.append(q)
            return q.c

        def vec(t):
            a = _np(t).astype(np.float32)
            keep.append(a)
            return _ptr(a).value

        layers = (LayerC * L)()
        for l in range(L):
            ly = m.layers[l]
            c = layers[l]
            c.attn_norm = vec(ly.attn_norm)
            c.ffn_norm = vec(ly.ffn_norm)
            c.wqkv, c.wo = qm(ly.wqkv), qm(ly.wo)
            c.wg, c.wu, c.wd = qm(ly.wg), qm(ly.wu), qm(ly.wd)
            if ly.router is not None:
                c.router = vec(ly.router)
                for name in ("eg", "eu", "ed"):
                    st = getattr(ly, name)
                    arr = (QMatC * st.E)(*[qm(st.mat(e)) for e in range(st.E)])
                    keep.append(arr)
                    setattr(c, name, C.cast(arr, C.c_void_p).value)
                c.sg, c.su, c.sd = qm(ly.sg), qm(ly.su), qm(ly.sd)
        keep.append(layers)
        self.c = ModelC(L, cfg.H, cfg.nq, cfg.nkv, cfg.hd, cfg.F, cfg.V, cfg.n_experts, cfg.topk,
                        cfg.F_exp, cfg.eps, cfg.theta, qm(m.embed), qm(m.lm_head),
                        vec(m.final_norm), C.cast(layers, C.c_void_p).value)
        self._keep = keep

    def sliced(self, l0: int, l1: int) -> "ModelC":
        """A model struct over layers [l0, l1) of this one (same memory)."""
        c = ModelC.from_buffer_copy(self.c)
        c.L = l1 - l0
        c.layers = self.c.layers + l0 * C.sizeof(LayerC)
        return c


def decode_token(model: Model, kv: KV, b: int, token: int, pos: int, moe_dense: bool = False,
                 want_logits: bool = True, want_hidden: bool = False, layers=None):
    """One greedy token of sequence b at position pos.  Writes K/V of pos into kv.
    layers=(l0, l1) runs only those layers (a bounded sample of the step).
    Returns dict(token, margin, logits, hidden, moe_idx, moe_logits)."""
    cfg = model.cfg
    mc, kc = model.c, kv.c
    if layers is not None:
        mc = model.sliced(*layers)
        kc = KVC.from_buffer_copy(kv.c)
        kc.k = kv.c.k + layers[0] * C.sizeof(C.c_void_p)
        kc.v = kv.c.v + layers[0] * C.sizeof(C.c_void_p)
        if kv.fp8:
            kc.k_scale = kv.c.k_scale + layers[0] * 4
            kc.v_scale = kv.c.v_scale + layers[0] * 4
    L = mc.L
    logits = np.empty(cfg.V, np.float32) if want_logits else None
    hidden = np.empty((L + 1, cfg.H), np.float32) if want_hidden else None
    moe_idx = np.empty((L, cfg.topk), np.int32) if cfg.n_experts else None
    moe_logits = np.empty((L, cfg.n_experts), np.float32) if cfg.n_experts else None
    margin = np.zeros(1, np.float32)
    tok = lib().or_decode_token(C.byref(mc), C.byref(kc), b, int(token), int(pos),
                                int(moe_dense),
                                None if logits is None else _ptr(logits),
                                None if hidden is None else _ptr(hidden),
                                None if moe_idx is None else _ptr(moe_idx), _ptr(margin),
                                None if moe_logits is None else _ptr(moe_logits))
    return {"token": int(tok), "margin": float(margin[0]), "logits": logits, "hidden": hidden,
            "moe_idx": moe_idx, "moe_logits": moe_logits}


# ------------------------------------------------------ generation loops

def greedy_generate(model: Model, kv: KV, b: int, token: int, pos: int, n_tokens: int):
    """Plain greedy decoding: the n_tokens tokens after `token` at `pos`."""
    out = []
    for i in range(n_tokens):
        token = decode_token(model, kv, b, token, pos + i)["token"]
        out.append(token)
    return out


def mtp_generate(model: Model, kv: KV, dh: DraftHead, b: int, token: int, pos: int, n_tokens: int, k: int,
                 drafter=None):
    """Speculative decoding with K drafts per verify pass (the deep-dive page,
    section 5, stage 4, and section 1): one plain step gives the first token
    and the main model's last hidden state; then each pass drafts d1..dK with
    the draft head (or `drafter(t0, pos, h, k)` when given), runs the verify
    rows t0, d1..dK at positions p..p+K over the shared cache, accepts drafts
    while each equals the greedy token of the row before it, and emits the
    accepted drafts plus the greedy token after the last accepted row.  The
    next pass starts from that token and from the hidden state of that row.
    Returns dict(tokens, accepted per pass, passes)."""
    L = model.c.L
    res = decode_token(model, kv, b, token, pos, want_logits=False, want_hidden=True)
    out = [res["token"]]
    t0, p, h = res["token"], pos + 1, res["hidden"][L]
    accepted = []
    while len(out) < n_tokens:
        if drafter is None:
            drafts, g, t = [], h, t0
            for _ in range(k):
                t, g, _ = draft_token(dh, g, t)
                drafts.append(t)
        else:
            drafts = list(drafter(t0, p, h, k))
        rows = [t0] + drafts
        greedy, hid = [], []
        for r, tr in enumerate(rows):
            rr = decode_token(model, kv, b, tr, p + r, want_logits=False, want_hidden=True)
            greedy.append(rr["token"])
            hid.append(rr["hidden"][L])
        n, nxt = spec_accept(rows, greedy)
        accepted.append(n)
        out.extend(drafts[:n] + [nxt])
        t0, h, p = nxt, hid[n], p + n + 1
    return {"tokens": out[:n_tokens], "accepted": accepted, "passes": len(accepted)}
