"""Seeded synthetic inputs for the decode step: configs, weights, KV context.

This module is the one thing the GPU path and the CPU oracle share.  It
builds the *inputs* only -- random-init weights packed in their canonical file
layouts, norm gains, router weights, the fp16 KV context, page tables and
start tokens.  It holds none of the decode arithmetic: no dequantization, no
matrix-vector product, no attention, no sampling.

Workload shapes follow the five decode workloads: a tiny single-layer model,
a 7B-class Q4_0 model, a 9B-class and a 27B-class NVFP4 model and a
35B-A3B-class NVFP4 mixture-of-experts model.  Weights are N(0, 0.02) before
quantization, the KV context is N(0, 1) rounded to fp16, page tables are seeded
random permutations of the physical pages.

Block formats (the workload definition; the pages only name "Q4"/"GGUF" and
"NVFP4"):
  Q4_0 : 32-weight blocks, 18 bytes = fp16 scale d + 16 bytes of nibbles;
         element j in the low nibble of byte j, element j+16 in the high
         nibble; w = d * (q - 8).
  NVFP4: 16-element blocks of E2M1 codes (element 2i in the low nibble of byte
         i), one E4M3 scale per block, one fp32 scale per tensor;
         w = e2m1 * e4m3 * ts.
The quantizers below are how the inputs are made (the encoding side); the
decoders live separately in the oracle and in the GPU kernels.
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Optional

import numpy as np
import torch

FMT_Q4_0 = 0
FMT_NVFP4 = 1
PAGE_TOKENS = 16


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    L: int
    H: int
    nq: int
    nkv: int
    hd: int
    F: int
    V: int
    fmt: int
    ctx: int            # synthetic context length already in the cache
    steps: int          # decode tokens per run
    B: int = 1          # sequences decoded together
    n_experts: int = 0  # 0: dense SwiGLU FFN
    topk: int = 0
    F_exp: int = 0      # expert (and shared expert) FFN width
    theta: float = 1.0e6
    eps: float = 1.0e-6
    verify_k: int = 0   # draft tokens checked by one speculative-verify pass
    draft_vocab: int = 32768   # output ids of the speculative draft head (the first ids)
    kv_fp8: bool = False       # the KV cache in E4M3 with per-layer scales (make_kv_fp8)
    prefill_prompt: int = 0    # prompt tokens of a timed chunked prefill (0: none)

    @property
    def nqkv(self) -> int:
        return (self.nq + 2 * self.nkv) * self.hd

    @property
    def max_pages(self) -> int:
        return -(-(self.ctx + self.steps + max(self.verify_k, 0) + 1) // PAGE_TOKENS)

    @property
    def n_pages(self) -> int:
        return self.B * self.max_pages

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Config("tiny-1L-h256-q4_0", L=1, H=256, nq=4, nkv=2, hd=64, F=704, V=1024,
                   fmt=FMT_Q4_0, ctx=128, steps=8, draft_vocab=256),
    "7b": Config("7b-dense-q4_0", L=28, H=3584, nq=28, nkv=4, hd=128, F=18944, V=152064,
                 fmt=FMT_Q4_0, ctx=2000, steps=512, prefill_prompt=2000),
    "9b": Config("9b-dense-nvfp4", L=36, H=4096, nq=32, nkv=8, hd=128, F=12288, V=151936,
                 fmt=FMT_NVFP4, ctx=4096, steps=256),
    "9b_b32": Config("9b-dense-nvfp4-b32", L=36, H=4096, nq=32, nkv=8, hd=128, F=12288,
                     V=151936, fmt=FMT_NVFP4, ctx=4096, steps=256, B=32),
    "27b": Config("27b-dense-nvfp4", L=64, H=5120, nq=64, nkv=8, hd=128, F=25600, V=151936,
                  fmt=FMT_NVFP4, ctx=8192, steps=128, verify_k=3),
    "9b_b32_fp8": Config("9b-dense-nvfp4-b32-fp8kv", L=36, H=4096, nq=32, nkv=8, hd=128, F=12288,
                         V=151936, fmt=FMT_NVFP4, ctx=4096, steps=256, B=32, kv_fp8=True),
    "moe": Config("35b-a3b-moe-nvfp4-b32", L=40, H=2048, nq=32, nkv=4, hd=128, F=0,
                  V=151936, fmt=FMT_NVFP4, ctx=2000, steps=128, B=32, n_experts=256,
                  topk=8, F_exp=512),
}


# --------------------------------------------------------------------- RNG

def _tensor_seed(seed: int, name: str) -> int:
    return (seed * 1_000_003 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF


def _gen(device, seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_tensor_seed(seed, name))
    return g


def randn(shape, std: float, device, seed: int, name: str) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(device, seed, name), device=device,
                       dtype=torch.float32) * std


# ------------------------------------------------------------- quantizers

@dataclasses.dataclass
class QMat:
    """A quantized matrix W[N][K] in its canonical (file) layout."""
    fmt: int
    N: int
    K: int
    q: torch.Tensor                    # uint8
    s: Optional[torch.Tensor] = None   # uint8 E4M3 scales (NVFP4)
    ts: float = 1.0                    # fp32 tensor scale (NVFP4)

    @property
    def nbytes(self) -> int:
        return self.q.numel() + (0 if self.s is None else self.s.numel())

    def to(self, device) -> "QMat":
        return QMat(self.fmt, self.N, self.K, self.q.to(device),
                    None if self.s is None else self.s.to(device), self.ts)


def quantize_q4_0(x: torch.Tensor) -> QMat:
    """Per 32-block: d = fp16(m / -8) with m the element of largest magnitude
    (first on ties); q = clamp(floor(x / d + 8.5), 0, 15); a zero block gets
    d = 0 and q = 8."""
    N, K = x.shape
    assert K % 32 == 0
    xb = x.reshape(N, K // 32, 32)
    i = xb.abs().argmax(dim=-1, keepdim=True)
    m = torch.gather(xb, -1, i)
    d = (m / -8.0).to(torch.float16)
    df = d.float()
    inv = torch.where(df != 0, 1.0 / df, torch.zeros_like(df))
    q = torch.clamp(torch.floor(xb * inv + 8.5), 0, 15).to(torch.uint8)
    qs = q[..., :16] | (q[..., 16:] << 4)
    blocks = torch.cat([d.view(torch.uint8), qs], dim=-1)      # [N, K/32, 18]
    return QMat(FMT_Q4_0, N, K, blocks.reshape(N, (K // 32) * 18).contiguous())


def e2m1_encode(y: torch.Tensor) -> torch.Tensor:
    """Round to the nearest E2M1 value, ties to the even mantissa, saturating at 6."""
    a = y.abs()
    code = ((a > 0.25).to(torch.uint8) + (a >= 0.75).to(torch.uint8) + (a > 1.25).to(torch.uint8)
            + (a >= 1.75).to(torch.uint8) + (a > 2.5).to(torch.uint8) + (a >= 3.5).to(torch.uint8)
            + (a > 5.0).to(torch.uint8))
    return code | ((y < 0).to(torch.uint8) << 3)


def quantize_nvfp4(x: torch.Tensor) -> QMat:
    """ts = amax / (6 * 448); per 16-block s = e4m3(amax_b / 6 / ts) (saturating at
    448); q = e2m1(x / (s * ts)); element 2i in the low nibble."""
    N, K = x.shape
    assert K % 16 == 0
    amax = float(x.abs().max())
    ts = float(np.float32(amax / (6.0 * 448.0))) if amax > 0 else 1.0
    xb = x.reshape(N, K // 16, 16)
    bamax = xb.abs().amax(dim=-1)
    s8 = (bamax / 6.0 / ts).clamp(max=448.0).to(torch.float8_e4m3fn)
    denom = (s8.float() * ts)[..., None]
    y = torch.where(denom > 0, xb / torch.where(denom > 0, denom, torch.ones_like(denom)),
                    torch.zeros_like(xb))
    code = e2m1_encode(y).reshape(N, K)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    return QMat(FMT_NVFP4, N, K, packed.contiguous(), s8.view(torch.uint8).reshape(N, K // 16).contiguous(), ts)


def quantize(x: torch.Tensor, fmt: int) -> QMat:
    return quantize_q4_0(x) if fmt == FMT_Q4_0 else quantize_nvfp4(x)


@dataclasses.dataclass
class QStack:
    """E matrices of one shape stored back to back (expert weights):
    q [E, ...], s [E, ...] (NVFP4), ts [E] fp32 (NVFP4; ones for Q4_0)."""
    fmt: int
    E: int
    N: int
    K: int
    q: torch.Tensor
    s: Optional[torch.Tensor]
    ts: torch.Tensor

    def mat(self, e: int) -> QMat:
        return QMat(self.fmt, self.N, self.K, self.q[e],
                    None if self.s is None else self.s[e], float(self.ts[e]))

    @property
    def nbytes_per_matrix(self) -> int:
        return (self.q.numel() + (0 if self.s is None else self.s.numel())) // self.E


def quantize_stack(x: torch.Tensor, fmt: int) -> QStack:
    """Quantize each of x[e] (shape [E, N, K]) as its own tensor."""
    mats = [quantize(x[e], fmt) for e in range(x.shape[0])]
    q = torch.stack([m.q for m in mats])
    s = None if fmt == FMT_Q4_0 else torch.stack([m.s for m in mats])
    ts = torch.tensor([m.ts for m in mats], dtype=torch.float32)
    return QStack(fmt, x.shape[0], x.shape[1], x.shape[2], q, s, ts)


# --------------------------------------------------------------- the model

@dataclasses.dataclass
class Layer:
    attn_norm: torch.Tensor
    ffn_norm: torch.Tensor
    wqkv: QMat
    wo: QMat
    wg: Optional[QMat] = None
    wu: Optional[QMat] = None
    wd: Optional[QMat] = None
    router: Optional[torch.Tensor] = None
    eg: Optional[QStack] = None
    eu: Optional[QStack] = None
    ed: Optional[QStack] = None
    sg: Optional[QMat] = None
    su: Optional[QMat] = None
    sd: Optional[QMat] = None


@dataclasses.dataclass
class Model:
    cfg: Config
    embed: QMat
    lm_head: QMat
    final_norm: torch.Tensor
    layers: list

    def weight_bytes_dense(self) -> int:
        """Bytes of every matrix a dense batch-1 step streams (not the embedding)."""
        n = self.lm_head.nbytes + self.final_norm.numel() * 4
        for ly in self.layers:
            n += ly.wqkv.nbytes + ly.wo.nbytes + (ly.attn_norm.numel() + ly.ffn_norm.numel()) * 4
            if ly.wg is not None:
                n += ly.wg.nbytes + ly.wu.nbytes + ly.wd.nbytes
        return n


def _qmat(shape, cfg: Config, device, seed, name, std=0.02) -> QMat:
    return quantize(randn(shape, std, device, seed, name), cfg.fmt)


def make_model(cfg: Config, device="cpu", seed: int = 0, n_layers: Optional[int] = None) -> Model:
    """Random-init weights of the config's shape, quantized to its format.
    n_layers (optional) builds only the first layers (used for partial checks)."""
    L = cfg.L if n_layers is None else n_layers
    layers = []
    for l in range(L):
        p = f"l{l}."
        ly = Layer(
            attn_norm=1.0 + randn((cfg.H,), 0.02, device, seed, p + "attn_norm"),
            ffn_norm=1.0 + randn((cfg.H,), 0.02, device, seed, p + "ffn_norm"),
            wqkv=_qmat((cfg.nqkv, cfg.H), cfg, device, seed, p + "wqkv"),
            wo=_qmat((cfg.H, cfg.nq * cfg.hd), cfg, device, seed, p + "wo"),
        )
        if cfg.n_experts == 0:
            ly.wg = _qmat((cfg.F, cfg.H), cfg, device, seed, p + "wg")
            ly.wu = _qmat((cfg.F, cfg.H), cfg, device, seed, p + "wu")
            ly.wd = _qmat((cfg.H, cfg.F), cfg, device, seed, p + "wd")
        else:
            E, Fe = cfg.n_experts, cfg.F_exp
            ly.router = randn((E, cfg.H), 1.0 / math.sqrt(cfg.H), device, seed, p + "router")
            ly.eg = quantize_stack(randn((E, Fe, cfg.H), 0.02, device, seed, p + "exp.g"), cfg.fmt)
            ly.eu = quantize_stack(randn((E, Fe, cfg.H), 0.02, device, seed, p + "exp.u"), cfg.fmt)
            ly.ed = quantize_stack(randn((E, cfg.H, Fe), 0.02, device, seed, p + "exp.d"), cfg.fmt)
            ly.sg = _qmat((Fe, cfg.H), cfg, device, seed, p + "sh.g")
            ly.su = _qmat((Fe, cfg.H), cfg, device, seed, p + "sh.u")
            ly.sd = _qmat((cfg.H, Fe), cfg, device, seed, p + "sh.d")
        layers.append(ly)
    return Model(
        cfg=cfg,
        embed=_qmat((cfg.V, cfg.H), cfg, device, seed, "embed"),
        lm_head=_qmat((cfg.V, cfg.H), cfg, device, seed, "lm_head"),
        final_norm=1.0 + randn((cfg.H,), 0.02, device, seed, "final_norm"),
        layers=layers,
    )


@dataclasses.dataclass
class DraftHead:
    """Weights of a speculative draft head: RMSNorm gains [H] and an output
    matrix over the first draft_vocab token ids, in the model's format (the
    draft head shares the model's embedding)."""
    norm: torch.Tensor
    w: QMat


def make_draft_head(cfg: Config, device="cpu", seed: int = 0) -> DraftHead:
    vd = min(cfg.draft_vocab, cfg.V)
    return DraftHead(norm=1.0 + randn((cfg.H,), 0.02, device, seed, "draft.norm"),
                     w=_qmat((vd, cfg.H), cfg, device, seed, "draft.w"))


# -------------------------------------------------------------- KV context

@dataclasses.dataclass
class KVCache:
    """Paged fp16 KV cache.  k[l], v[l]: uint16 (fp16 bits) [n_pages][nkv][16][hd];
    page_table: int32 [B][max_pages] (logical page -> physical page, shared by
    all layers)."""
    k: list
    v: list
    page_table: torch.Tensor
    n_pages: int
    page_tokens: int = PAGE_TOKENS
    # FP8 variant: k[l], v[l] hold E4M3 codes (uint8) and these hold one fp32
    # scale per layer (a code c stands for e4m3(c) * scale); None for fp16
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None

    def clone(self) -> "KVCache":
        return KVCache([t.clone() for t in self.k], [t.clone() for t in self.v],
                       self.page_table.clone(), self.n_pages, self.page_tokens,
                       None if self.k_scale is None else self.k_scale.clone(),
                       None if self.v_scale is None else self.v_scale.clone())

    def to(self, device) -> "KVCache":
        return KVCache([t.to(device) for t in self.k], [t.to(device) for t in self.v],
                       self.page_table.to(device), self.n_pages, self.page_tokens,
                       self.k_scale, self.v_scale)


def page_table(cfg: Config, device="cpu", seed: int = 0, permute: bool = True) -> torch.Tensor:
    n = cfg.n_pages
    if permute:
        perm = torch.randperm(n, generator=_gen("cpu", seed, "page_table"))
    else:
        perm = torch.arange(n)
    return perm.to(torch.int32).reshape(cfg.B, cfg.max_pages).to(device)


def make_kv(cfg: Config, device="cpu", seed: int = 0, permute: bool = True,
            n_layers: Optional[int] = None) -> KVCache:
    """Every slot of every page filled with N(0, 1) rounded to fp16 (positions
    0..ctx-1 are the synthetic context; later slots are overwritten by decode
    before they are read)."""
    L = cfg.L if n_layers is None else n_layers
    shape = (cfg.n_pages, cfg.nkv, PAGE_TOKENS, cfg.hd)
    ks, vs = [], []
    for l in range(L):
        ks.append(randn(shape, 1.0, device, seed, f"kv.k{l}").to(torch.float16).view(torch.int16))
        vs.append(randn(shape, 1.0, device, seed, f"kv.v{l}").to(torch.float16).view(torch.int16))
    return KVCache(ks, vs, page_table(cfg, device, seed, permute), cfg.n_pages)


def make_kv_fp8(cfg: Config, device="cpu", seed: int = 0, permute: bool = True,
                n_layers: Optional[int] = None) -> KVCache:
    """The FP8 (E4M3) variant of make_kv: the same N(0, 1) context stored as
    E4M3 codes of x / scale with per-layer scales 1/16 + l/256 (K) and
    1/20 + l/256 (V), rounded by torch's float8 conversion after clamping to
    the format's +-448."""
    L = cfg.L if n_layers is None else n_layers
    shape = (cfg.n_pages, cfg.nkv, PAGE_TOKENS, cfg.hd)
    k_scale = torch.tensor([1 / 16 + l / 256 for l in range(L)], dtype=torch.float32)
    v_scale = torch.tensor([1 / 20 + l / 256 for l in range(L)], dtype=torch.float32)
    ks, vs = [], []
    for l in range(L):
        for name, sc, out in (("k", k_scale[l], ks), ("v", v_scale[l], vs)):
            x = randn(shape, 1.0, device, seed, f"kv.{name}{l}") / sc.to(device)
            out.append(x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8))
    return KVCache(ks, vs, page_table(cfg, device, seed, permute), cfg.n_pages, PAGE_TOKENS, k_scale, v_scale)


def start_tokens(cfg: Config, seed: int = 0, n: Optional[int] = None) -> torch.Tensor:
    n = cfg.B if n is None else n
    return torch.randint(0, cfg.V, (n,), generator=_gen("cpu", seed, "tokens"), dtype=torch.int32)


def prompt_tokens(cfg: Config, n: int, seed: int = 0) -> torch.Tensor:
    """A synthetic prompt: n token ids uniform over the vocabulary."""
    return torch.randint(0, cfg.V, (n,), generator=_gen("cpu", seed, "prompt"), dtype=torch.int32)


def draft_tokens(cfg: Config, k: int, seed: int = 0) -> torch.Tensor:
    return torch.randint(0, cfg.V, (cfg.B, k), generator=_gen("cpu", seed, "drafts"), dtype=torch.int32)
