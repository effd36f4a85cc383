"""Per-kernel timing of the decode step: each libbw launch kind of one step
(QKV, attention, O, gate/up or MoE, down, LM head + argmax) replayed over
every layer of a model from a CUDA graph, timed with CUDA events on the
launching stream, reported as microseconds per launch and algorithmic GB/s
(the bytes of weights and KV that launch must touch, divided by its time).

"step" (batch 1, dense models) is the whole decode step run as one persistent
kernel (bw_decode_step with BW_STEP_PERSISTENT); "chain" is the whole step as
its usual chain of launches (for launch lists under ncu).

Also the small, self-contained target for `ncu` captures:

    python -m token_decode_b200.kernel_bench --config 7b --layers 2 --only gu --reps 2 --eager

launches only the named kernel kind, eagerly, `reps` times per layer.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import bw, runtime, synth


def _wbytes(w) -> int:
    """Algorithmic bytes of a packed matrix: 4-bit codes plus its block scales.
    Both formats come to 9/16 byte per weight (Q4_0: a 2-byte scale per 32
    weights; NVFP4: a 1-byte scale per 16)."""
    return w.N * w.K * 9 // 16


class KernelBench:
    """Holds the activations, workspace and launchers for one device model."""

    def __init__(self, dm: runtime.DeviceModel, dkv: runtime.DeviceKV, B: int, stream, pos: int):
        cfg = dm.cfg
        self.dm, self.dkv, self.cfg, self.B, self.st = dm, dkv, cfg, B, stream
        dev = "cuda"
        g = torch.Generator(device=dev)
        g.manual_seed(1234)
        self.x = torch.randn((B, cfg.H), device=dev, generator=g)
        self.gamma = torch.ones(cfg.H, device=dev)
        self.qkv = torch.randn((B, cfg.nqkv), device=dev, generator=g)
        self.att = torch.randn((B, cfg.nq * cfg.hd), device=dev, generator=g)
        F = cfg.F if cfg.n_experts == 0 else cfg.F_exp
        self.act = torch.randn((B, max(F, 1)), device=dev, generator=g) * 0.1
        self.logits = torch.empty((B, cfg.V), device=dev)
        self.am = torch.empty(B, dtype=torch.int32, device=dev)
        self.pos = torch.full((B,), pos, dtype=torch.int32, device=dev)
        self.avg_len = pos + 1
        n = bw.decode_workspace_bytes(dm.c, dkv.c, B, 1)
        self.ws = bw.workspace(n)

    # -- launchers ---------------------------------------------------------
    def _gemv(self, w, xin, y, flags, gamma=None, residual=None, argmax_out=None):
        if w.fmt == synth.FMT_Q4_0:
            bw.gemv_q4_0(w.q, w.s, w.N, w.K, xin, self.B, y, self.ws, gamma=gamma,
                         eps=self.cfg.eps, residual=residual, argmax_out=argmax_out,
                         flags=flags, stream=self.st)
        else:
            bw.gemv_nvfp4(w.q, w.s, w.ts, w.N, w.K, xin, self.B, y, self.ws, ts_up=w.ts_up,
                          gamma=gamma, eps=self.cfg.eps, residual=residual,
                          argmax_out=argmax_out, flags=flags, stream=self.st)

    def kinds(self):
        """name -> (launch(layer), algorithmic bytes(layer), per-layer?)"""
        cfg, dm, dkv = self.cfg, self.dm, self.dkv
        L = dm.c.L
        out = {}
        out["qkv"] = (lambda l: self._gemv(dm.layers[l].wqkv, self.x, self.qkv, bw.GEMV_RMSNORM,
                                           gamma=self.gamma),
                      lambda l: _wbytes(dm.layers[l].wqkv), L)
        kv_layer = 2 * cfg.nkv * cfg.hd * (1 if dkv.fp8 else 2) * self.B

        def attn(l):
            if dkv.fp8:
                bw.paged_attn_decode_fp8(self.qkv, dm.cos, dm.sin, dm.c.rope_max_pos, dkv.k[l], dkv.v[l],
                                         dkv._ks[l], dkv._vs[l], dkv.page_table, dkv.c.max_pages, dkv.c.n_pages,
                                         self.pos, self.B, 1, cfg.nq, cfg.nkv, cfg.hd, self.att, self.ws,
                                         stream=self.st)
            else:
                bw.paged_attn_decode(self.qkv, dm.cos, dm.sin, dm.c.rope_max_pos, dkv.k[l], dkv.v[l],
                                     dkv.page_table, dkv.c.max_pages, dkv.c.n_pages, self.pos, self.B, 1,
                                     cfg.nq, cfg.nkv, cfg.hd, self.att, self.ws, stream=self.st)
        out["attn"] = (attn, lambda l: kv_layer * (self.avg_len + 1), L)
        out["o"] = (lambda l: self._gemv(dm.layers[l].wo, self.att, self.x, bw.GEMV_RESIDUAL,
                                         residual=self.x),
                    lambda l: _wbytes(dm.layers[l].wo), L)
        if cfg.n_experts == 0:
            out["gu"] = (lambda l: self._gemv(dm.layers[l].wgu, self.x, self.act,
                                              bw.GEMV_RMSNORM | bw.GEMV_SILU_GATE, gamma=self.gamma),
                         lambda l: _wbytes(dm.layers[l].wgu), L)
            out["down"] = (lambda l: self._gemv(dm.layers[l].wd, self.act, self.x, bw.GEMV_RESIDUAL,
                                                residual=self.x),
                           lambda l: _wbytes(dm.layers[l].wd), L)
        else:
            mws = bw.workspace(bw.moe_workspace_bytes(dm.c, self.B))
            self._mws = mws
            exp_bytes = _wbytes(dm.layers[0].sgu) + _wbytes(dm.layers[0].sd)

            def moe(l):
                bw.moe_route_gemv(dm.c, dm.layers[l], self.x, self.B, mws, stream=self.st)
            # bytes: router + shared expert + the experts this launch selects, counted
            # by the caller from the router output (see moe_touched_bytes)
            out["moe"] = (moe, lambda l: 4 * cfg.n_experts * cfg.H + exp_bytes
                          + self.moe_expert_bytes, L)
        if self.with_step and self.B == 1 and cfg.n_experts == 0:
            # the whole batch-1 step: one persistent kernel (bw_decode_step); its
            # bytes are every matrix plus the KV read and written
            tin = torch.zeros(1, dtype=torch.int32, device="cuda")
            tout = torch.zeros(1, dtype=torch.int32, device="cuda")
            wsz = bw.decode_workspace_bytes(dm.c, dkv.c, 1, 1)
            self._sws = bw.workspace(wsz)
            step_b = sum(_wbytes(w) for ly in dm.layers for w in (ly.wqkv, ly.wo, ly.wgu, ly.wd)) + \
                _wbytes(dm.c.lm_head) + L * kv_layer * (self.avg_len + 1)

            def step(l):
                # no advance: every launch decodes the same position
                bw.decode_step(dm.c, dkv.c, tin, self.pos, 1, 1, tout, self._sws, flags=bw.STEP_PERSISTENT,
                               stream=self.st)
            out["step"] = (step, lambda l: step_b, 1)
        if self.with_chain:
            # the whole step as the usual chain of launches (bw_decode_step): the
            # target of launch-list captures; bytes as for "step"
            tin = torch.zeros(self.B, dtype=torch.int32, device="cuda")
            tout = torch.zeros(self.B, dtype=torch.int32, device="cuda")
            self._cws = bw.workspace(bw.decode_workspace_bytes(dm.c, dkv.c, self.B, 1))

            def chain(l):
                bw.decode_step(dm.c, dkv.c, tin, self.pos, self.B, 1, tout, self._cws, stream=self.st)
            out["chain"] = (chain, lambda l: 0, 1)
        lm = dm.c.lm_head
        out["lm_head"] = (lambda l: self._gemv(lm, self.x, self.logits, bw.GEMV_RMSNORM | bw.GEMV_ARGMAX,
                                               gamma=self.gamma, argmax_out=self.am),
                          lambda l: _wbytes(lm), 1)
        return out

    moe_expert_bytes = 0
    with_step = False   # also the persistent whole-step kernel (only when asked for by name)
    with_chain = False  # also the whole step as its chain of launches (only when asked for by name)

    def time(self, name, reps=10):
        """Graph of the kind over all its layers, replayed `reps` times."""
        fn, nbytes, n = self.kinds()[name]
        st = self.st
        with torch.cuda.stream(st):
            for l in range(n):
                fn(l)
            st.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=st):
                for l in range(n):
                    fn(l)
            for _ in range(3):
                gr.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for _ in range(reps):
                gr.replay()
            e1.record(st)
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * n)
        b = sum(nbytes(l) for l in range(n)) / n
        del gr
        return {"us_per_launch": round(us, 3), "bytes_per_launch": int(b),
                "GBps": round(b / us / 1e3, 1), "launches": n}


def moe_touched_bytes(dm, B, kb: KernelBench) -> int:
    """Bytes of the routed experts one MoE launch touches: route x once with
    the library's own router and count the distinct selected experts."""
    cfg = dm.cfg
    idx = torch.empty((B, cfg.topk), dtype=torch.int32, device="cuda")
    wts = torch.empty((B, cfg.topk), device="cuda")
    x = kb.x.clone()
    ws = bw.workspace(bw.moe_workspace_bytes(dm.c, B))
    bw.moe_route_gemv(dm.c, dm.layers[0], x, B, ws, topk_idx=idx, topk_w=wts, stream=kb.st)
    kb.st.synchronize()
    used = int(torch.unique(idx).numel())
    per = (2 * cfg.F_exp * cfg.H + cfg.H * cfg.F_exp) * 9 // 16
    return used * per


def run_all(dm, dkv, B, stream, pos, reps=10, only=None):
    kb = KernelBench(dm, dkv, B, stream, pos)
    kb.with_step = only == "step"
    kb.with_chain = only == "chain"
    if dm.cfg.n_experts:
        kb.moe_expert_bytes = moe_touched_bytes(dm, B, kb)
    res = {}
    for name in kb.kinds():
        if only and name != only:
            continue
        res[name] = kb.time(name, reps)
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--config", default="7b")
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--only", default=None)
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--eager", action="store_true",
                    help="launch without graphs (for profilers): reps x layers launches")
    a = ap.parse_args()
    from . import build
    build.build()
    bw.lib()
    cfg = synth.CONFIGS[a.config]
    if a.layers:
        cfg = cfg.with_(L=a.layers)
    if a.batch:
        cfg = cfg.with_(B=a.batch)
    model = synth.make_model(cfg, "cuda", seed=0, n_layers=cfg.L)
    kv = (synth.make_kv_fp8 if cfg.kv_fp8 else synth.make_kv)(cfg, "cuda", seed=0, n_layers=cfg.L)
    dm = runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS)
    dkv = runtime.DeviceKV(kv)
    del model
    st = torch.cuda.Stream()
    pos = cfg.ctx + cfg.steps // 2
    if a.eager:
        kb = KernelBench(dm, dkv, cfg.B, st, pos)
        kb.with_step = a.only == "step"
        kb.with_chain = a.only == "chain"
        if cfg.n_experts:
            kb.moe_expert_bytes = moe_touched_bytes(dm, cfg.B, kb)
        for name, (fn, _, n) in kb.kinds().items():
            if a.only and name != a.only:
                continue
            with torch.cuda.stream(st):
                for _ in range(a.reps):
                    for l in range(n):
                        fn(l)
        st.synchronize()
        err = bw.read_error(kb.ws)
        print(json.dumps({"eager": a.only or "all", "device_error_word": err}))
        raise SystemExit(0 if err == 0 else 1)
    res = run_all(dm, dkv, cfg.B, st, pos, a.reps, a.only)
    for k, v in res.items():
        print(json.dumps({"kernel": k, "config": cfg.name, "B": cfg.B, **v}))


if __name__ == "__main__":
    main()
