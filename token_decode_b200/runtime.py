"""Device-side model and KV cache for the decode step: argument marshalling
for bw_decode_step.

Takes the seeded inputs (canonical weight bytes already on the GPU), converts
every matrix to the GPU layout with the library's repack kernels, builds the
RoPE tables with bw_rope_table, and fills the bw_model / bw_kv descriptors.
All arithmetic happens in libbw.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import bw
from .synth import FMT_Q4_0, FMT_NVFP4, PAGE_TOKENS


def _gpu_layout(m, up=None):
    """QMat (+ matching up-projection) -> (bw.QWeight, [tensors to keep alive])."""
    rows = m.N * (2 if up is not None else 1)
    qb, sb = bw.repack_bytes(rows, m.K)
    q = torch.empty((qb,), dtype=torch.uint8, device=m.q.device)
    s = torch.empty((sb,), dtype=torch.uint8, device=m.q.device)
    if m.fmt == FMT_Q4_0:
        bw.repack_q4_0(m.q, m.N, m.K, q, s, blocks_up=None if up is None else up.q)
    else:
        bw.repack_nvfp4(m.q, m.s, m.N, m.K, q, s, q_up=None if up is None else up.q,
                        s_up=None if up is None else up.s)
    qw = bw.QWeight(m.fmt, rows, m.K, bw._ptr(q), bw._ptr(s), m.ts,
                    up.ts if up is not None else m.ts)
    return qw, [q, s]


class DeviceModel:
    """GPU-layout weights + descriptors of one model (see include/bw.h)."""

    def __init__(self, model, max_pos: int):
        cfg = model.cfg
        self.cfg = cfg
        keep = []

        def qw(m, up=None):
            w, t = _gpu_layout(m, up)
            keep.extend(t)
            return w

        L = len(model.layers)
        self.layers = (bw.Layer * L)()
        for l, ly in enumerate(model.layers):
            c = self.layers[l]
            c.attn_norm = bw._ptr(ly.attn_norm)
            c.ffn_norm = bw._ptr(ly.ffn_norm)
            keep += [ly.attn_norm, ly.ffn_norm]
            c.wqkv = qw(ly.wqkv)
            c.wo = qw(ly.wo)
            if cfg.n_experts == 0:
                c.wgu = qw(ly.wg, ly.wu)
                c.wd = qw(ly.wd)
            else:
                self._moe_layer(c, ly, keep)
        self.cos = torch.empty((max_pos, cfg.hd // 2), dtype=torch.float32, device="cuda")
        self.sin = torch.empty_like(self.cos)
        bw.rope_table(cfg.theta, cfg.hd, max_pos, self.cos, self.sin)
        keep += [model.final_norm]
        self.c = bw.Model(L, cfg.H, cfg.nq, cfg.nkv, cfg.hd, cfg.F, cfg.V, cfg.n_experts, cfg.topk,
                          cfg.F_exp, cfg.eps, qw(model.embed), qw(model.lm_head),
                          bw._ptr(model.final_norm), bw._ptr(self.cos), bw._ptr(self.sin),
                          max_pos, C.cast(self.layers, C.c_void_p).value)
        self._keep = keep
        self.weight_bytes = sum(t.numel() * t.element_size() for t in keep)

    def _moe_layer(self, c, ly, keep):
        E, Fe, H = ly.eg.E, ly.eg.N, ly.eg.K
        gqb, gsb = bw.repack_bytes(2 * Fe, H)
        dqb, dsb = bw.repack_bytes(H, Fe)
        gq = torch.empty((E, gqb), dtype=torch.uint8, device="cuda")
        gs = torch.empty((E, gsb), dtype=torch.uint8, device="cuda")
        dq = torch.empty((E, dqb), dtype=torch.uint8, device="cuda")
        ds = torch.empty((E, dsb), dtype=torch.uint8, device="cuda")
        for e in range(E):
            g, u, d = ly.eg.mat(e), ly.eu.mat(e), ly.ed.mat(e)
            if g.fmt == FMT_Q4_0:
                bw.repack_q4_0(g.q, Fe, H, gq[e], gs[e], blocks_up=u.q)
                bw.repack_q4_0(d.q, H, Fe, dq[e], ds[e])
            else:
                bw.repack_nvfp4(g.q, g.s, Fe, H, gq[e], gs[e], q_up=u.q, s_up=u.s)
                bw.repack_nvfp4(d.q, d.s, H, Fe, dq[e], ds[e])
        gts = torch.stack([ly.eg.ts, ly.eu.ts], dim=1).contiguous().to("cuda")
        dts = ly.ed.ts.contiguous().to("cuda")
        c.router = bw._ptr(ly.router)
        c.egu_q, c.egu_s, c.ed_q, c.ed_s = bw._ptr(gq), bw._ptr(gs), bw._ptr(dq), bw._ptr(ds)
        c.egu_ts, c.ed_ts = bw._ptr(gts), bw._ptr(dts)
        keep += [ly.router, gq, gs, dq, ds, gts, dts]
        w, t = _gpu_layout(ly.sg, ly.su)
        c.sgu = w
        keep += t
        w, t = _gpu_layout(ly.sd)
        c.sd = w
        keep += t


class DeviceKV:
    """The paged KV pools (one per layer) + page table as a bw_kv: fp16 pools, or
    E4M3 byte pools with per-layer K/V scales when the cache carries k_scale."""

    def __init__(self, kv):
        self.k = kv.k
        self.v = kv.v
        self.page_table = kv.page_table.to(torch.int32).contiguous()
        L = len(kv.k)
        self._kp = (C.c_void_p * L)(*[bw._ptr(t) for t in kv.k])
        self._vp = (C.c_void_p * L)(*[bw._ptr(t) for t in kv.v])
        self.fp8 = getattr(kv, "k_scale", None) is not None
        if self.fp8:
            self._ks = (C.c_float * L)(*[float(x) for x in kv.k_scale.cpu().tolist()[:L]])
            self._vs = (C.c_float * L)(*[float(x) for x in kv.v_scale.cpu().tolist()[:L]])
        self.c = bw.KV(C.cast(self._kp, C.c_void_p).value, C.cast(self._vp, C.c_void_p).value,
                       int(kv.n_pages), int(self.page_table.shape[1]), bw._ptr(self.page_table),
                       bw.KV_E4M3 if self.fp8 else bw.KV_FP16,
                       C.cast(self._ks, C.c_void_p).value if self.fp8 else None,
                       C.cast(self._vs, C.c_void_p).value if self.fp8 else None)


class Decoder:
    """Owns a workspace and runs bw_decode_step for B sequences x n_rows."""

    def __init__(self, dm: DeviceModel, dkv: DeviceKV, B: int, n_rows: int = 1):
        self.dm, self.dkv, self.B, self.n_rows = dm, dkv, B, n_rows
        self.ws = bw.workspace(bw.decode_workspace_bytes(dm.c, dkv.c, B, n_rows))
        self.tokens_in = torch.zeros(B * n_rows, dtype=torch.int32, device="cuda")
        self.tokens_out = torch.zeros(B * n_rows, dtype=torch.int32, device="cuda")
        self.pos = torch.zeros(B, dtype=torch.int32, device="cuda")

    def step(self, logits=None, advance=False, stream=None, persistent=False):
        flags = (bw.STEP_ADVANCE if advance else 0) | (bw.STEP_PERSISTENT if persistent else 0)
        bw.decode_step(self.dm.c, self.dkv.c, self.tokens_in, self.pos, self.B, self.n_rows,
                       self.tokens_out, self.ws, logits=logits, flags=flags, stream=stream)


class DeviceDraftHead:
    """GPU-layout draft head (norm gains + W_draft) as a bw_draft_head."""

    def __init__(self, head):
        qw, keep = _gpu_layout(head.w)
        self.c = bw.DraftHead(bw._ptr(head.norm), qw)
        self._keep = keep + [head.norm]


class Prefiller:
    """Chunked prefill (bw_prefill) of the sequence in the cache's first page-table
    row: owns the workspace for `chunk` rows per step."""

    def __init__(self, dm: DeviceModel, dkv: DeviceKV, chunk: int):
        self.dm, self.dkv, self.chunk = dm, dkv, chunk
        self.ws = bw.workspace(bw.prefill_workspace_bytes(dm.c, dkv.c, chunk))
        self.next_token = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(self, tokens, pos0: int, logits=None, stream=None):
        """tokens: device int32 [n]; afterwards next_token holds the greedy token
        after the last prompt token."""
        bw.prefill(self.dm.c, self.dkv.c, tokens, int(tokens.numel()), int(pos0), self.chunk, self.next_token,
                   self.ws, logits=logits, stream=stream)
        return self.next_token


class SpecDecoder:
    """Speculative decoding of one sequence with K drafts per pass: a plain step
    gives the first token and the hidden state the draft head starts from; each
    pass then drafts (bw_mtp_draft), verifies the last token and the K drafts as
    K + 1 rows of one step (bw_decode_step) and accepts (bw_spec_accept), which
    also writes the next pass's first token and advances the position.  The
    plain and the verify steps share the model's KV cache."""

    def __init__(self, dm: DeviceModel, dkv: DeviceKV, ddh: DeviceDraftHead, K: int):
        self.dm, self.ddh, self.K = dm, ddh, K
        self.plain = Decoder(dm, dkv, 1)
        self.ver = Decoder(dm, dkv, 1, n_rows=K + 1)
        self.mws = bw.workspace(bw.mtp_workspace_bytes(dm.c, ddh.c))
        self.n_acc = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.first = True

    def start(self, token: int, pos: int, stream=None):
        """Plain step on `token` at `pos`: its greedy token is the first output."""
        self.plain.tokens_in.fill_(int(token))
        self.plain.pos.fill_(int(pos))
        self.plain.step(stream=stream)
        self.ver.tokens_in[:1].copy_(self.plain.tokens_out)
        self.ver.pos.fill_(int(pos) + 1)
        self.first = True

    def draft(self, stream=None):
        if self.first:
            hid = bw.decode_hidden(self.dm.c, self.plain.dkv.c, 1, 1, self.plain.ws)
            bw.mtp_draft(self.dm.c, self.ddh.c, hid, 1, self.ver.tokens_in, self.K, self.mws, stream=stream)
        else:
            hid = bw.decode_hidden(self.dm.c, self.ver.dkv.c, 1, self.K + 1, self.ver.ws)
            bw.mtp_draft(self.dm.c, self.ddh.c, hid, self.K + 1, self.ver.tokens_in, self.K, self.mws,
                         row=self.n_acc, stream=stream)

    def verify_accept(self, stream=None):
        self.ver.step(stream=stream)
        bw.spec_accept(self.ver.tokens_in, self.ver.tokens_out, 1, self.K + 1, self.n_acc,
                       next_out=self.ver.tokens_in, next_stride=self.K + 1, pos=self.ver.pos, stream=stream)
        self.first = False

    def step_pass(self, stream=None):
        """One pass; afterwards tokens_in[1..n_acc] (the accepted drafts) and
        tokens_in[0] (the greedy token after them) are its output."""
        self.draft(stream)
        self.verify_accept(stream)
