"""ctypes binding of libbw (include/bw.h): same names, argument marshalling only.

Every computation runs in the library's CUDA kernels.  Loading fails loudly
when libbw.so is missing or no CUDA device is present; there is no fallback.
Tensors are passed as torch tensors (device memory) and converted to raw
pointers here; `stream` defaults to torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbw.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_BAD_PAGE_INDEX = range(6)
DEVERR_BAD_PAGE, DEVERR_TIMEOUT, DEVERR_BAD_TOKEN, DEVERR_BAD_POS = 1, 2, 4, 8
FMT_Q4_0, FMT_NVFP4 = 0, 1
KV_FP16, KV_E4M3 = 0, 1
GEMV_RMSNORM, GEMV_RESIDUAL, GEMV_SILU_GATE, GEMV_ARGMAX = 1, 2, 4, 8
STEP_ADVANCE = 1
STEP_VALIDATE_ONLY = 2
STEP_PERSISTENT = 4
MAX_VERIFY_ROWS = 8

# every symbol include/bw.h declares (checked by the CPU test-suite)
EXPORTS = (
    "bw_status_string", "bw_abi_version", "bw_workspace_init", "bw_read_error", "bw_drain_error",
    "bw_repack_bytes", "bw_repack_q4_0", "bw_repack_nvfp4", "bw_gemv_q4_0", "bw_gemv_nvfp4",
    "bw_gemv_workspace_bytes", "bw_gemv_q4_0_noalloc", "bw_rmsnorm_fused", "bw_embed", "bw_rope_table", "bw_argmax",
    "bw_paged_attn_decode", "bw_paged_attn_decode_fp8", "bw_attn_workspace_bytes", "bw_moe_route_gemv",
    "bw_moe_workspace_bytes", "bw_decode_step", "bw_decode_workspace_bytes", "bw_decode_hidden", "bw_spec_accept",
    "bw_decode_moe_route", "bw_mtp_draft", "bw_mtp_workspace_bytes", "bw_prefill", "bw_prefill_workspace_bytes",
)


class BWError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {string(status)} ({status})")


class QWeight(C.Structure):
    _fields_ = [("fmt", C.c_int), ("N", C.c_int), ("K", C.c_int), ("q", C.c_void_p),
                ("s", C.c_void_p), ("ts", C.c_float), ("ts_up", C.c_float)]


class Layer(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("ffn_norm", C.c_void_p),
                ("wqkv", QWeight), ("wo", QWeight), ("wgu", QWeight), ("wd", QWeight),
                ("router", C.c_void_p), ("egu_q", C.c_void_p), ("egu_s", C.c_void_p),
                ("ed_q", C.c_void_p), ("ed_s", C.c_void_p), ("egu_ts", C.c_void_p),
                ("ed_ts", C.c_void_p), ("sgu", QWeight), ("sd", QWeight)]


class Model(C.Structure):
    _fields_ = [("L", C.c_int), ("H", C.c_int), ("nq", C.c_int), ("nkv", C.c_int), ("hd", C.c_int),
                ("F", C.c_int), ("V", C.c_int), ("n_experts", C.c_int), ("topk", C.c_int),
                ("F_exp", C.c_int), ("eps", C.c_float), ("embed", QWeight), ("lm_head", QWeight),
                ("final_norm", C.c_void_p), ("rope_cos", C.c_void_p), ("rope_sin", C.c_void_p),
                ("rope_max_pos", C.c_int), ("layers", C.c_void_p)]


class DraftHead(C.Structure):
    _fields_ = [("norm", C.c_void_p), ("w", QWeight)]


class KV(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("n_pages", C.c_int), ("max_pages", C.c_int),
                ("page_table", C.c_void_p), ("kv_fmt", C.c_int), ("k_scale", C.c_void_p), ("v_scale", C.c_void_p)]


_lib = None


def lib() -> C.CDLL:
    """Load libbw.so (raises when it is missing or no CUDA device is present)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libbw.so not built ({LIB_PATH}); run `python -m token_decode_b200.build`")
        L = C.CDLL(LIB_PATH)
        p, i, f, u, z = C.c_void_p, C.c_int, C.c_float, C.c_uint, C.c_size_t
        sig = {
            "bw_status_string": (C.c_char_p, [i]),
            "bw_abi_version": (i, []),
            "bw_workspace_init": (i, [p, z, p]),
            "bw_read_error": (i, [p, p, p]),
            "bw_drain_error": (i, [p, p, p]),
            "bw_repack_bytes": (i, [i, i, p, p]),
            "bw_repack_q4_0": (i, [p, p, i, i, p, p, p]),
            "bw_repack_nvfp4": (i, [p, p, p, p, i, i, p, p, p]),
            "bw_gemv_q4_0": (i, [p, p, i, i, p, i, p, f, p, p, p, u, p, z, p]),
            "bw_gemv_nvfp4": (i, [p, p, f, f, i, i, p, i, p, f, p, p, p, u, p, z, p]),
            "bw_gemv_workspace_bytes": (z, [i, i, i, u]),
            "bw_gemv_q4_0_noalloc": (i, [p, p, i, i, p, i, p, f, p, p, p, u, p]),
            "bw_rmsnorm_fused": (i, [p, p, p, i, i, f, p, i, p]),
            "bw_embed": (i, [i, p, p, f, i, i, p, i, p, p, p]),
            "bw_rope_table": (i, [f, i, i, p, p, p]),
            "bw_argmax": (i, [p, i, i, p, p, p]),
            "bw_paged_attn_decode": (i, [p, p, p, i, p, p, p, i, i, p, i, i, i, i, i, p, p, z, p]),
            "bw_paged_attn_decode_fp8": (i, [p, p, p, i, p, p, f, f, p, i, i, p, i, i, i, i, i, p, p, z, p]),
            "bw_attn_workspace_bytes": (z, [i, i, i, i, i, i]),
            "bw_moe_route_gemv": (i, [p, p, p, i, p, p, p, z, p]),
            "bw_moe_workspace_bytes": (z, [p, i]),
            "bw_decode_step": (i, [p, p, p, p, i, i, p, p, u, p, z, p]),
            "bw_decode_workspace_bytes": (z, [p, p, i, i]),
            "bw_decode_hidden": (p, [p, p, i, i, p]),
            "bw_decode_moe_route": (i, [p, p, i, i, p, p, p]),
            "bw_mtp_draft": (i, [p, p, p, i, p, p, i, p, z, p]),
            "bw_mtp_workspace_bytes": (z, [p, p]),
            "bw_prefill": (i, [p, p, p, i, i, i, p, p, p, z, p]),
            "bw_prefill_workspace_bytes": (z, [p, p, i]),
            "bw_spec_accept": (i, [p, p, i, i, p, p, i, p, p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def string(status: int) -> str:
    return lib().bw_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise BWError(status, what)


def _ptr(t) -> int | None:
    """Device address of a tensor argument (None stays NULL, an int is taken
    as an address).  The library reads every pointer as dense device memory,
    so a host or strided tensor is refused here instead of reaching a kernel."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"libbw takes device memory; got a tensor on {t.device}")
    if not t.is_contiguous():
        raise ValueError("libbw takes dense (contiguous) tensors")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


# ------------------------------------------------------------------ wrappers

def workspace(nbytes: int, device="cuda", stream=None) -> torch.Tensor:
    """Allocate (through torch) and zero-fill a workspace of nbytes."""
    ws = torch.empty(max(nbytes, 1 << 18), dtype=torch.uint8, device=device)
    _check(lib().bw_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "bw_workspace_init")
    return ws


def read_error(ws: torch.Tensor, stream=None) -> int:
    out = C.c_uint32(0)
    _check(lib().bw_read_error(_ptr(ws), C.byref(out), _stream(stream)), "bw_read_error")
    return out.value


def drain_error(ws, dst: torch.Tensor, stream=None) -> None:
    """Enqueue: OR ws's device error word (ws None: the no-alloc scratch's)
    into dst[0] (a device int32/uint32 tensor) and clear it; no synchronization."""
    _check(lib().bw_drain_error(_ptr(ws), _ptr(dst), _stream(stream)), "bw_drain_error")


def repack_bytes(rows, K):
    """(code bytes, scale bytes) of a `rows` x K matrix in the tiled GPU layout."""
    qb, sb = C.c_size_t(0), C.c_size_t(0)
    _check(lib().bw_repack_bytes(rows, K, C.byref(qb), C.byref(sb)), "bw_repack_bytes")
    return qb.value, sb.value


def repack_q4_0(blocks, N, K, q_out, s_out, blocks_up=None, stream=None):
    _check(lib().bw_repack_q4_0(_ptr(blocks), _ptr(blocks_up), N, K, _ptr(q_out), _ptr(s_out),
                                _stream(stream)), "bw_repack_q4_0")


def repack_nvfp4(q, s, N, K, q_out, s_out, q_up=None, s_up=None, stream=None):
    _check(lib().bw_repack_nvfp4(_ptr(q), _ptr(s), _ptr(q_up), _ptr(s_up), N, K, _ptr(q_out),
                                 _ptr(s_out), _stream(stream)), "bw_repack_nvfp4")


def gemv_workspace_bytes(N, K, M, flags=0) -> int:
    return lib().bw_gemv_workspace_bytes(N, K, M, flags)


def gemv_q4_0(w_q, w_d, N, K, x, M, y, ws, gamma=None, eps=1e-6, residual=None, argmax_out=None,
              flags=0, stream=None):
    _check(lib().bw_gemv_q4_0(_ptr(w_q), _ptr(w_d), N, K, _ptr(x), M, _ptr(gamma), eps,
                              _ptr(residual), _ptr(y), _ptr(argmax_out), flags, _ptr(ws),
                              ws.numel(), _stream(stream)), "bw_gemv_q4_0")


def gemv_q4_0_noalloc(w_q, w_d, N, K, x, M, y, gamma=None, eps=1e-6, residual=None,
                      argmax_out=None, flags=0, stream=None):
    """bw_gemv_q4_0 with the library's fixed device scratch instead of a workspace,
    for callers that cannot allocate device memory."""
    _check(lib().bw_gemv_q4_0_noalloc(_ptr(w_q), _ptr(w_d), N, K, _ptr(x), M, _ptr(gamma), eps,
                                      _ptr(residual), _ptr(y), _ptr(argmax_out), flags,
                                      _stream(stream)), "bw_gemv_q4_0_noalloc")


def gemv_nvfp4(w_q, w_s, ts, N, K, x, M, y, ws, ts_up=None, gamma=None, eps=1e-6, residual=None,
               argmax_out=None, flags=0, stream=None):
    _check(lib().bw_gemv_nvfp4(_ptr(w_q), _ptr(w_s), ts, ts if ts_up is None else ts_up, N, K,
                               _ptr(x), M, _ptr(gamma), eps, _ptr(residual), _ptr(y),
                               _ptr(argmax_out), flags, _ptr(ws), ws.numel(), _stream(stream)),
           "bw_gemv_nvfp4")


def rmsnorm_fused(x, gamma, M, H, eps, y=None, add=None, y_fp16=False, stream=None):
    _check(lib().bw_rmsnorm_fused(_ptr(x), _ptr(add), _ptr(gamma), M, H, eps, _ptr(y), int(y_fp16),
                                  _stream(stream)), "bw_rmsnorm_fused")


def embed(fmt, e_q, e_s, ts, V, H, tokens, M, x, ws=None, stream=None):
    _check(lib().bw_embed(fmt, _ptr(e_q), _ptr(e_s), ts, V, H, _ptr(tokens), M, _ptr(x), _ptr(ws),
                          _stream(stream)), "bw_embed")


def rope_table(theta, hd, max_pos, cos_out, sin_out, stream=None):
    _check(lib().bw_rope_table(theta, hd, max_pos, _ptr(cos_out), _ptr(sin_out), _stream(stream)),
           "bw_rope_table")


def argmax(logits, M, V, idx_out, margin_out=None, stream=None):
    _check(lib().bw_argmax(_ptr(logits), M, V, _ptr(idx_out), _ptr(margin_out), _stream(stream)),
           "bw_argmax")


def attn_workspace_bytes(B, n_rows, nq, nkv, hd, max_pages) -> int:
    return lib().bw_attn_workspace_bytes(B, n_rows, nq, nkv, hd, max_pages)


def paged_attn_decode(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, page_table, max_pages,
                      n_pages, pos, B, n_rows, nq, nkv, hd, out, ws, stream=None):
    _check(lib().bw_paged_attn_decode(_ptr(qkv), _ptr(rope_cos), _ptr(rope_sin), rope_max_pos,
                                      _ptr(k_pool), _ptr(v_pool), _ptr(page_table), max_pages,
                                      n_pages, _ptr(pos), B, n_rows, nq, nkv, hd, _ptr(out),
                                      _ptr(ws), ws.numel(), _stream(stream)), "bw_paged_attn_decode")


def paged_attn_decode_fp8(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, k_scale, v_scale, page_table,
                          max_pages, n_pages, pos, B, n_rows, nq, nkv, hd, out, ws, stream=None):
    """bw_paged_attn_decode over an E4M3 cache (byte pools, per-layer scales)."""
    _check(lib().bw_paged_attn_decode_fp8(_ptr(qkv), _ptr(rope_cos), _ptr(rope_sin), rope_max_pos,
                                          _ptr(k_pool), _ptr(v_pool), float(k_scale), float(v_scale),
                                          _ptr(page_table), max_pages, n_pages, _ptr(pos), B, n_rows, nq, nkv,
                                          hd, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "bw_paged_attn_decode_fp8")


def moe_workspace_bytes(model: Model, R: int) -> int:
    return lib().bw_moe_workspace_bytes(C.byref(model), R)


def moe_route_gemv(model: Model, layer: Layer, x, R, ws, topk_idx=None, topk_w=None, stream=None):
    _check(lib().bw_moe_route_gemv(C.byref(model), C.byref(layer), _ptr(x), R, _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(ws), ws.numel(), _stream(stream)),
           "bw_moe_route_gemv")


def decode_workspace_bytes(model: Model, kv: KV, B: int, n_rows: int) -> int:
    return lib().bw_decode_workspace_bytes(C.byref(model), C.byref(kv), B, n_rows)


def decode_hidden(model: Model, kv: KV, B, n_rows, ws) -> torch.Tensor:
    """The step's residual stream inside ws as an fp32 [B*n_rows][H] view: each
    row's hidden state after the last layer, valid until the next step on ws."""
    addr = lib().bw_decode_hidden(C.byref(model), C.byref(kv), B, n_rows, _ptr(ws))
    if not addr:
        raise BWError(ERR_INVALID_ARG, "bw_decode_hidden")
    off = addr - ws.data_ptr()
    n = B * n_rows * model.H
    return ws[off: off + 4 * n].view(torch.float32).view(B * n_rows, model.H)


def decode_moe_route(model: Model, kv: KV, B, n_rows, ws):
    """(expert ids int32 [B*n_rows][topk], weights fp32 [B*n_rows][topk]): views
    into ws of the last MoE layer's expert choice in the latest step on ws."""
    ia, wa = C.c_void_p(0), C.c_void_p(0)
    _check(lib().bw_decode_moe_route(C.byref(model), C.byref(kv), B, n_rows, _ptr(ws), C.byref(ia),
                                     C.byref(wa)), "bw_decode_moe_route")
    n = B * n_rows * model.topk
    oi, ow = ia.value - ws.data_ptr(), wa.value - ws.data_ptr()
    return (ws[oi: oi + 4 * n].view(torch.int32).view(B * n_rows, model.topk),
            ws[ow: ow + 4 * n].view(torch.float32).view(B * n_rows, model.topk))


def decode_step(model: Model, kv: KV, tokens_in, pos, B, n_rows, tokens_out, ws, logits=None,
                flags=0, stream=None):
    _check(lib().bw_decode_step(C.byref(model), C.byref(kv), _ptr(tokens_in), _ptr(pos), B, n_rows,
                                _ptr(tokens_out), _ptr(logits), flags, _ptr(ws), ws.numel(),
                                _stream(stream)), "bw_decode_step")


def prefill_workspace_bytes(model: Model, kv: KV, chunk: int) -> int:
    return lib().bw_prefill_workspace_bytes(C.byref(model), C.byref(kv), chunk)


def prefill(model: Model, kv: KV, tokens, n, pos0, chunk, next_token, ws, logits=None, stream=None):
    """Chunked prefill of the sequence in kv's first page-table row (see bw.h)."""
    _check(lib().bw_prefill(C.byref(model), C.byref(kv), _ptr(tokens), n, pos0, chunk, _ptr(next_token),
                            _ptr(logits), _ptr(ws), ws.numel(), _stream(stream)), "bw_prefill")


def mtp_workspace_bytes(model: Model, dh: DraftHead) -> int:
    return lib().bw_mtp_workspace_bytes(C.byref(model), C.byref(dh))


def mtp_draft(model: Model, dh: DraftHead, hidden, n_rows, tokens, K, ws, row=None, stream=None):
    """K draft tokens into tokens[1..K] from tokens[0] and hidden row *row (see bw.h)."""
    _check(lib().bw_mtp_draft(C.byref(model), C.byref(dh), _ptr(hidden), n_rows, _ptr(row), _ptr(tokens), K,
                              _ptr(ws), ws.numel(), _stream(stream)), "bw_mtp_draft")


def spec_accept(tokens_in, tokens_out, B, n_rows, n_accept, next_out=None, next_stride=1, pos=None,
                stream=None):
    """Accepted draft count per sequence after a verify pass (see bw.h)."""
    _check(lib().bw_spec_accept(_ptr(tokens_in), _ptr(tokens_out), B, n_rows, _ptr(n_accept),
                                _ptr(next_out), next_stride, _ptr(pos), _stream(stream)),
           "bw_spec_accept")
