"""Host-side validation of a whole decode step (no GPU, nothing launched).

bw_decode_step with BW_STEP_VALIDATE_ONLY runs every check the step makes
before its first launch -- the descriptors, each launch's shape limits and
pointer alignment -- and returns.  Descriptors here hold fake, never
dereferenced device addresses: the workload configs must pass, and each
planted defect must be rejected with its status."""
import ctypes as C

import pytest

from token_decode_b200 import synth

OK, INVALID, UNSUPPORTED = 0, 1, 2


@pytest.fixture(scope="module")
def bw():
    from token_decode_b200 import build
    build.build()
    from token_decode_b200 import bw as bw_mod
    bw_mod.lib()
    return bw_mod


class _Step:
    """A bw_model / bw_kv pair of a config over fake 4 KiB-aligned addresses."""

    def __init__(self, bw, cfg, L=2):
        self.bw, self.cfg = bw, cfg
        self._next = 1 << 32

        def qw(N, K):
            return bw.QWeight(cfg.fmt, N, K, self.ptr(), self.ptr(), 1.0, 1.0)

        self.layers = (bw.Layer * L)()
        for c in self.layers:
            c.attn_norm, c.ffn_norm = self.ptr(), self.ptr()
            c.wqkv = qw(cfg.nqkv, cfg.H)
            c.wo = qw(cfg.H, cfg.nq * cfg.hd)
            if cfg.n_experts == 0:
                c.wgu = qw(2 * cfg.F, cfg.H)
                c.wd = qw(cfg.H, cfg.F)
            else:
                c.router = self.ptr()
                c.egu_q, c.egu_s, c.ed_q, c.ed_s = self.ptr(), self.ptr(), self.ptr(), self.ptr()
                c.egu_ts, c.ed_ts = self.ptr(), self.ptr()
                c.sgu = qw(2 * cfg.F_exp, cfg.H)
                c.sd = qw(cfg.H, cfg.F_exp)
        max_pos = cfg.max_pages * synth.PAGE_TOKENS
        self.m = bw.Model(L, cfg.H, cfg.nq, cfg.nkv, cfg.hd, cfg.F, cfg.V, cfg.n_experts, cfg.topk, cfg.F_exp,
                          cfg.eps, qw(cfg.V, cfg.H), qw(cfg.V, cfg.H), self.ptr(), self.ptr(), self.ptr(),
                          max_pos, C.cast(self.layers, C.c_void_p).value)
        self._kp = (C.c_void_p * L)(*[self.ptr() for _ in range(L)])
        self._vp = (C.c_void_p * L)(*[self.ptr() for _ in range(L)])
        self.kv = bw.KV(C.cast(self._kp, C.c_void_p).value, C.cast(self._vp, C.c_void_p).value,
                        cfg.n_pages, cfg.max_pages, self.ptr())

    def ptr(self):
        p = self._next
        self._next += 1 << 20
        return p

    def validate(self, B=None, n_rows=1, ws_bytes=None, ws=None):
        lib = self.bw.lib()
        B = self.cfg.B if B is None else B
        need = lib.bw_decode_workspace_bytes(C.byref(self.m), C.byref(self.kv), B, n_rows)
        return lib.bw_decode_step(C.byref(self.m), C.byref(self.kv), self.ptr(), self.ptr(), B, n_rows,
                                  self.ptr(), None, self.bw.STEP_VALIDATE_ONLY,
                                  self.ptr() if ws is None else ws, need if ws_bytes is None else ws_bytes, None)


_NV = synth.FMT_NVFP4


@pytest.mark.parametrize("name,over,n_rows", [
    ("tiny", {}, 1), ("tiny", dict(B=2), 4), ("tiny", dict(fmt=_NV, B=1), 8), ("tiny", dict(fmt=_NV, B=8), 1),
    ("tiny", dict(B=5), 1), ("tiny", dict(fmt=_NV, F=0, n_experts=16, topk=4, F_exp=64, B=4), 1),
    ("7b", {}, 1), ("9b", {}, 1), ("9b_b32", {}, 1), ("9b", {}, 8), ("27b", {}, 4), ("moe", {}, 1)])
def test_workload_descriptors_pass(bw, name, over, n_rows):
    """Every shape the GPU tests and the benchmark run passes the step's checks."""
    cfg = synth.CONFIGS[name].with_(**over)
    if n_rows > 1:
        cfg = cfg.with_(verify_k=n_rows - 1)
    assert _Step(bw, cfg).validate(n_rows=n_rows) == OK


def test_planted_defects_are_rejected_before_any_launch(bw):
    cfg7 = synth.CONFIGS["7b"]
    # shapes the kernels do not support
    assert _Step(bw, cfg7.with_(hd=96)).validate() == UNSUPPORTED             # head dim
    assert _Step(bw, cfg7.with_(nq=30)).validate() == UNSUPPORTED             # nq % nkv
    assert _Step(bw, cfg7).validate(n_rows=5) == UNSUPPORTED                  # 7 q heads x 5 rows > 32
    assert _Step(bw, synth.CONFIGS["27b"]).validate(n_rows=8) == UNSUPPORTED  # 8 q heads x 8 rows > 32
    assert _Step(bw, synth.CONFIGS["9b"]).validate(n_rows=9) == UNSUPPORTED   # more rows than a pass holds
    assert _Step(bw, cfg7.with_(V=152063)).validate() == UNSUPPORTED          # LM head rows % 8
    assert _Step(bw, cfg7.with_(ctx=200000)).validate() == UNSUPPORTED        # page-table width
    # misaligned or missing pointers, wrong matrix shapes
    s = _Step(bw, cfg7)
    s.layers[1].attn_norm += 4
    assert s.validate() == INVALID
    s = _Step(bw, cfg7)
    s.layers[0].wo.q += 8
    assert s.validate() == INVALID
    s = _Step(bw, cfg7)
    s.layers[1].wd.K -= 32
    assert s.validate() == INVALID
    s = _Step(bw, cfg7)
    s.m.final_norm += 4
    assert s.validate() == INVALID
    s = _Step(bw, cfg7)
    s._kp[1] = s._kp[1] + 2
    assert s.validate() == INVALID
    s = _Step(bw, cfg7)
    s.m.embed.fmt = 5
    s.m.lm_head.fmt = 5
    assert s.validate() == INVALID
    # workspace: too small, or off its 256-byte alignment
    s = _Step(bw, cfg7)
    need = bw.lib().bw_decode_workspace_bytes(C.byref(s.m), C.byref(s.kv), 1, 1)
    assert s.validate(ws_bytes=need - 256) == INVALID
    assert s.validate(ws=s.ptr() + 64) == INVALID
    # MoE: an expert table off its 16-byte alignment, too many experts, a shared
    # expert of another format
    cfgm = synth.CONFIGS["moe"]
    s = _Step(bw, cfgm)
    s.layers[1].ed_s += 8
    assert s.validate() == INVALID
    assert _Step(bw, cfgm.with_(n_experts=4096)).validate() == UNSUPPORTED
    s = _Step(bw, cfgm)
    s.layers[0].sgu.fmt = synth.FMT_Q4_0
    s.layers[0].sd.fmt = synth.FMT_Q4_0
    assert s.validate() == INVALID


def test_empty_inputs_are_rejected(bw):
    """Zero sequences, zero rows per sequence or zero layers of work are argument
    errors, reported before anything is queued."""
    s = _Step(bw, synth.CONFIGS["tiny"])
    assert s.validate(B=0) == INVALID
    assert s.validate(n_rows=0) == INVALID
    lib, p = bw.lib(), C.c_void_p
    fake = p(1 << 32)
    assert lib.bw_gemv_q4_0(fake, fake, 64, 64, fake, 0, None, 1e-6, None, fake, None, 0, fake, 1 << 20,
                            None) == INVALID
    assert lib.bw_gemv_nvfp4(fake, fake, 1.0, 1.0, 0, 64, fake, 1, None, 1e-6, None, fake, None, 0, fake,
                             1 << 20, None) == INVALID
    assert lib.bw_spec_accept(fake, fake, 0, 1, fake, None, 1, None, None) == INVALID


def test_embedding_pointers_are_checked(bw):
    lib, p = bw.lib(), C.c_void_p
    fake = p(1 << 32)
    # scales off the tiled layout's alignment; a workspace off its 256-byte alignment
    assert lib.bw_embed(0, fake, p((1 << 32) + 2), 1.0, 64, 64, fake, 1, fake, None, None) == INVALID
    assert lib.bw_embed(0, fake, fake, 1.0, 64, 64, fake, 1, fake, p((1 << 32) + 4), None) == INVALID
    s = _Step(bw, synth.CONFIGS["tiny"])
    s.m.embed.s += 2
    assert s.validate() == INVALID


def test_decode_hidden_points_at_the_step_residual_stream(bw):
    """bw_decode_hidden is host arithmetic: the residual stream is the first
    region after the workspace header, sized B*n_rows x H floats, and the same
    address for every call with the same shapes."""
    s = _Step(bw, synth.CONFIGS["9b_b32"])
    lib = bw.lib()
    ws = 1 << 40
    a = lib.bw_decode_hidden(C.byref(s.m), C.byref(s.kv), 32, 1, ws)
    assert a == ws + (1 << 18)
    assert lib.bw_decode_hidden(C.byref(s.m), C.byref(s.kv), 32, 1, ws) == a
    assert lib.bw_decode_hidden(C.byref(s.m), C.byref(s.kv), 0, 1, ws) is None
    assert lib.bw_decode_hidden(None, C.byref(s.kv), 32, 1, ws) is None
    need = lib.bw_decode_workspace_bytes(C.byref(s.m), C.byref(s.kv), 32, 1)
    assert (a - ws) + 32 * s.cfg.H * 4 <= need
