"""CPU-side checks of the C ABI: the library builds for sm_100a, loads, exports
every symbol include/bw.h declares, and rejects bad arguments on the host
before any launch (no kernel runs here)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from token_decode_b200 import build
    build.build()
    from token_decode_b200 import bw
    return bw.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "bw.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bw_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for must in ("bw_gemv_q4_0", "bw_gemv_nvfp4", "bw_rmsnorm_fused", "bw_paged_attn_decode",
                 "bw_moe_route_gemv", "bw_argmax", "bw_decode_step"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    from token_decode_b200 import bw
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) == set(bw.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", bw.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (bw_[a-z0-9_]+)$", out, flags=re.M))
    assert set(_declared()) <= exported


def test_library_is_built_for_sm_100a(lib):
    from token_decode_b200 import bw
    out = subprocess.run(["cuobjdump", "--list-elf", bw.LIB_PATH], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_status_strings_and_version(lib):
    from token_decode_b200 import bw
    assert lib.bw_abi_version() == 1
    assert bw.string(0) == "ok"
    assert "page" in bw.string(5)
    assert bw.string(99) == "unknown status"


def test_host_validation_rejects_bad_arguments(lib):
    p = C.c_void_p
    fake = p(4096)   # never dereferenced: validation fails first
    # null weights
    assert lib.bw_gemv_q4_0(None, fake, 64, 64, fake, 1, None, 1e-6, None, fake, None, 0, fake,
                            1 << 20, None) == 1
    # N not a multiple of 8
    assert lib.bw_gemv_q4_0(fake, fake, 60, 64, fake, 1, None, 1e-6, None, fake, None, 0, fake,
                            1 << 20, None) == 2
    # K not a multiple of 32
    assert lib.bw_gemv_nvfp4(fake, fake, 1.0, 1.0, 64, 48, fake, 1, None, 1e-6, None, fake, None,
                             0, fake, 1 << 20, None) == 2
    # RMSNORM without gamma
    assert lib.bw_gemv_q4_0(fake, fake, 64, 64, fake, 1, None, 1e-6, None, fake, None, 1, fake,
                            1 << 20, None) == 1
    # unaligned weights
    assert lib.bw_gemv_q4_0(p(4097), fake, 64, 64, fake, 1, None, 1e-6, None, fake, None, 0, fake,
                            1 << 20, None) == 1
    # RMSNORM with unaligned gains; a workspace off its 256-byte alignment
    assert lib.bw_gemv_q4_0(fake, fake, 64, 64, fake, 1, p(4100), 1e-6, None, fake, None, 1, fake,
                            1 << 20, None) == 1
    assert lib.bw_gemv_q4_0(fake, fake, 64, 64, fake, 1, None, 1e-6, None, fake, None, 0, p(4096 + 16),
                            1 << 20, None) == 1
    assert lib.bw_gemv_nvfp4(fake, fake, 1.0, 1.0, 64, 64, fake, 1, None, 1e-6, None, fake, None,
                             0, p(4096 + 128), 1 << 20, None) == 1
    assert lib.bw_workspace_init(p(4096 + 64), 1 << 20, None) == 1
    assert lib.bw_moe_route_gemv(fake, fake, fake, 32, None, None, p(4096 + 16), 1 << 30, None) == 1
    # attention: unsupported head dim, too many query rows per kv head
    args = [fake, fake, fake, 128, fake, fake, fake, 8, 8, fake, 1, 1, 8, 2, 96, fake, fake, 1 << 24, None]
    assert lib.bw_paged_attn_decode(*args) == 2
    args[11], args[12], args[13], args[14] = 4, 64, 2, 128    # G * n_rows = 128 > 32
    assert lib.bw_paged_attn_decode(*args) == 2
    args[16] = p(4096 + 32)                                   # unaligned workspace
    assert lib.bw_paged_attn_decode(*args) == 1
    # repack: rows not a multiple of 8
    assert lib.bw_repack_q4_0(fake, None, 12, 64, fake, fake, None) == 2
    assert lib.bw_rope_table(C.c_float(-1.0), 64, 16, fake, fake, None) == 1
    assert lib.bw_decode_step(None, None, None, None, 1, 1, None, None, 0, None, 0, None) == 1
    # verify acceptance: too many rows, no sequences, a zero stride for next_out
    assert lib.bw_spec_accept(fake, fake, 1, 9, fake, None, 1, None, None) == 1
    assert lib.bw_spec_accept(fake, fake, 0, 4, fake, None, 1, None, None) == 1
    assert lib.bw_spec_accept(fake, fake, 1, 4, fake, fake, 0, None, None) == 1
    # error drain: no destination, a misaligned destination or workspace
    assert lib.bw_drain_error(fake, None, None) == 1
    assert lib.bw_drain_error(fake, p(4098), None) == 1
    assert lib.bw_drain_error(p(4096 + 16), fake, None) == 1


def test_workspace_queries_are_host_only(lib):
    z = lib.bw_gemv_workspace_bytes(4608, 3584, 1, 0)
    assert z >= 1 << 18
    assert lib.bw_attn_workspace_bytes(1, 1, 28, 4, 128, 160) >= 1 << 18


def test_binding_refuses_host_and_strided_tensors():
    """The binding hands the library device addresses only: a host tensor (or
    a strided view) raises before any call instead of reaching a kernel."""
    import torch
    from token_decode_b200 import bw
    assert bw._ptr(None) is None and bw._ptr(4096) == 4096
    with pytest.raises(ValueError, match="device memory"):
        bw._ptr(torch.zeros(4))
    with pytest.raises(ValueError):
        bw.gemv_q4_0(torch.zeros(16, dtype=torch.uint8), 4096, 8, 32, 4096, 1, 4096, torch.zeros(1))


def test_noalloc_gemv_refuses_shapes_beyond_its_fixed_scratch(lib):
    """bw_gemv_q4_0_noalloc refuses, before touching any device, a shape whose
    split-K partial sums would not fit the fixed scratch array, and one with
    more row groups than its counters cover."""
    p = C.c_void_p
    fake = p(4096)   # never dereferenced: the shape check comes first
    # K = 131072 splits K into >= 37 slices: 37 x 4096 rows x 4 rows x 4 B > 768 KiB
    assert lib.bw_gemv_q4_0_noalloc(fake, fake, 4096, 131072, fake, 4, None, C.c_float(1e-6), None, fake,
                                    None, 0, None) == 2
    assert lib.bw_gemv_q4_0_noalloc(fake, fake, 262144, 512, fake, 1, None, C.c_float(1e-6), None, fake,
                                    None, 0, None) == 2
    assert lib.bw_gemv_q4_0_noalloc(fake, fake, 0, 512, fake, 1, None, C.c_float(1e-6), None, fake,
                                    None, 0, None) == 1
    assert lib.bw_read_error(fake, None, None) == 1


def test_prefill_host_checks_reject_before_any_launch():
    """bw_prefill refuses, on the host, a chunk the attention cannot hold (7
    query heads per kv head x 5 rows > 32), a chunk above the verify-row limit,
    a prompt running past the cache, and a workspace sized for fewer rows.
    Only calls that must fail before launching are made (descriptors point at
    host memory)."""
    import ctypes as C
    import numpy as np
    from token_decode_b200 import bw, synth
    L = bw.lib()
    keep = []

    def buf(n):
        a = np.zeros(n + 256, np.uint8)
        keep.append(a)
        return a.ctypes.data + (-a.ctypes.data % 256)

    cfg = synth.CONFIGS["7b"].with_(L=1)

    def qw(N, K):
        q, s = bw.repack_bytes(N, K)
        return bw.QWeight(cfg.fmt, N, K, buf(q), buf(s), 1.0, 1.0)

    layers = (bw.Layer * 1)()
    ly = layers[0]
    ly.attn_norm, ly.ffn_norm = buf(4 * cfg.H), buf(4 * cfg.H)
    ly.wqkv, ly.wo = qw(cfg.nqkv, cfg.H), qw(cfg.H, cfg.nq * cfg.hd)
    ly.wgu, ly.wd = qw(2 * cfg.F, cfg.H), qw(cfg.H, cfg.F)
    maxpos = cfg.max_pages * 16
    m = bw.Model(1, cfg.H, cfg.nq, cfg.nkv, cfg.hd, cfg.F, cfg.V, 0, 0, 0, cfg.eps, qw(cfg.V, cfg.H),
                 qw(cfg.V, cfg.H), buf(4 * cfg.H), buf(2 * maxpos * cfg.hd), buf(2 * maxpos * cfg.hd), maxpos,
                 C.cast(layers, C.c_void_p).value)
    pool = 16 * 2 * cfg.nkv * cfg.hd
    kp = (C.c_void_p * 1)(buf(pool))   # never read: every call below fails first
    vp = (C.c_void_p * 1)(buf(pool))
    kv = bw.KV(C.cast(kp, C.c_void_p).value, C.cast(vp, C.c_void_p).value, cfg.n_pages, cfg.max_pages,
               buf(4 * cfg.max_pages), 0, None, None)
    n8 = L.bw_prefill_workspace_bytes(C.byref(m), C.byref(kv), 8)
    assert n8 > L.bw_decode_workspace_bytes(C.byref(m), C.byref(kv), 1, 8)
    ws, tok, nxt = buf(n8), buf(4 * 64), buf(4)

    def run(n, pos0, chunk, ws_bytes=n8):
        return L.bw_prefill(C.byref(m), C.byref(kv), tok, n, pos0, chunk, nxt, None, ws, ws_bytes, None)

    assert run(8, cfg.ctx, 5) == bw.ERR_UNSUPPORTED_SHAPE     # 7 x 5 query rows
    assert run(8, cfg.ctx, 9) == bw.ERR_UNSUPPORTED_SHAPE     # above BW_MAX_VERIFY_ROWS
    assert run(8, maxpos - 4, 4) == bw.ERR_INVALID_ARG        # past the cache
    assert run(0, cfg.ctx, 4) == bw.ERR_INVALID_ARG
    assert run(8, cfg.ctx, 4, L.bw_prefill_workspace_bytes(C.byref(m), C.byref(kv), 4) - 1) == bw.ERR_INVALID_ARG
