#!/usr/bin/env python3
"""Decode benchmark: greedy decode tok/s of the 7B-class Q4_0 model at batch 1
(28 layers, hidden 3584, 28/4 heads, FFN 18944, vocab 152064, ctx 2000 + 512
decode tokens), seeded synthetic random-init weights, on 1..N B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 7b] [--impl ours|reference]

One step = one greedy decode token for the batch: embedding, 28 layers
(fused RMSNorm+QKV GEMV, paged attention with RoPE + KV write, O GEMV +
residual, fused RMSNorm+gate/up GEMV with SiLU gate, down GEMV + residual),
final RMSNorm + LM-head GEMV + argmax.  The timed region replays CUDA graphs
of decode steps whose last kernel feeds the next step on the device.  Every
step streams ~4.1 GB of weights and KV (>> the 126 MB L2), so no L2 flush is
needed between steps.  Multi-GPU: independent replicas (weak scaling), one
process per GPU, time = max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s at batch 1 and 32; achieved HBM GB/s as % of 8 TB/s roofline"
NOMINAL_HBM_GBS = 8000.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons around the timed
    region (the body of the `with`); the summary keeps the samples whose
    timestamps fall inside it, or all of them when none does."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.out = ""
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        self.t0 = datetime.datetime.now()
        return self

    def __exit__(self, *a):
        self.t1 = datetime.datetime.now()
        time.sleep(0.1)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                ts = None
            active = {n for n, v in zip(self.REASONS, parts[4:8]) if v.lower() == "active"}
            rows.append((ts, sm, mx, active))
        inside = [r for r in rows if r[0] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 <= r[0] <= self.t1]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(set().union(*(r[3] for r in use))), "samples": len(use),
                "samples_in_timed_region": len(inside)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def job_throughput(ms_local, tokens_per_rank, world_size, device="cuda"):
    """Whole-job rate of N independent replicas: the slowest rank's time (max
    over ranks, on the device clock each rank measured) and every rank's
    tokens.  Returns (ms, tokens per second)."""
    ms = float(ms_local)
    if world_size > 1:
        import torch.distributed as dist
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, tokens_per_rank * world_size / (ms / 1000.0)


def workload_config(cfg, world_size):
    """The `config` object of the JSON line: the workload, identical for both arms."""
    return {"workload": cfg.name, "batch": cfg.B, "context": cfg.ctx,
            "decode_tokens_per_generation": cfg.steps, "layers": cfg.L, "hidden": cfg.H,
            "heads": f"{cfg.nq}/{cfg.nkv}x{cfg.hd}", "ffn": cfg.F, "vocab": cfg.V,
            "parallelism": f"replicas x{world_size}"}


def step_bytes(cfg, model, avg_ctx, moe_layer_bytes=0):
    """Algorithmic bytes of one decode step: every weight matrix streamed once
    (4.5-bit blocks + fp32 norm gains), the KV read over the context, the new
    K/V written (the embedding row is not counted).  A MoE layer adds
    moe_layer_bytes: its fp32 router, its shared expert and the experts the
    router selected (counted from the library's own routing of the batch)."""
    eb = 1 if cfg.kv_fp8 else 2          # bytes per cached element (E4M3 or fp16)
    kv_read = 2 * cfg.L * cfg.nkv * cfg.hd * eb * avg_ctx * cfg.B
    kv_write = 2 * cfg.L * cfg.nkv * cfg.hd * eb * cfg.B
    moe = cfg.L * moe_layer_bytes if cfg.n_experts else 0
    return model.weight_bytes_dense() + kv_read + kv_write + moe


# ncu summaries of the dominant kernels: DRAM traffic per launch, valid while the
# kernel sources a summary lists still hash to the value it records
_PROFILE_FILES = {("gu", "7b-dense-q4_0"): "gemv_gate_up_7b.md",
                  ("down", "7b-dense-q4_0"): "gemv_down_7b.md",
                  ("qkv", "7b-dense-q4_0"): "gemv_qkv_7b.md",
                  ("o", "7b-dense-q4_0"): "gemv_o_7b.md",
                  ("lm_head", "7b-dense-q4_0"): "gemv_lm_head_7b.md",
                  ("gu", "9b-dense-nvfp4"): "gemv_gate_up_9b.md",
                  ("gu", "27b-dense-nvfp4"): "gemv_gate_up_27b.md",
                  ("attn", "7b-dense-q4_0"): "attn_7b_b1.md",
                  ("attn", "27b-dense-nvfp4"): "attn_27b_b1.md",
                  ("attn", "9b-dense-nvfp4-b32"): "attn_9b_b32.md",
                  ("attn", "9b-dense-nvfp4-b32-fp8kv"): "attn_9b_b32_fp8.md",
                  ("gu", "9b-dense-nvfp4-b32"): "mma_gemm_gate_up_9b_b32.md"}
# (the MoE FFN is six launches: no single kernel's DRAM bytes stand for it)


def kernel_sources_sha(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "token_decode_b200",
                               "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic(kind, cfg_name):
    name = _PROFILE_FILES.get((kind, cfg_name))
    if name is None:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", name)
    if not os.path.exists(path):
        return None
    vals = {}
    for ln in open(path):
        if ln.startswith("- ") and ":" in ln:
            k, v = ln[2:].split(":", 1)
            vals[k.strip().strip("`")] = v.strip().strip("`")
    files = vals.get("kernel_sources", "").split()
    try:
        if not files or vals.get("kernel_sources_sha") != kernel_sources_sha(files):
            return None
        return int(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError, OSError):
        return None


def step_launches(cfg):
    """libbw kernel launches of one decode step: embedding; per layer QKV,
    attention, O and the FFN (dense gate/up + down, or the MoE block's
    RMSNorm, router, top-k, two grouped GEMVs and combine); LM head.  A
    projection is ceil(rows/4) CUDA-core GEMV launches, or (NVFP4 with more
    than 4 rows) an activation pack plus a tensor-core GEMM per 32 rows."""
    from token_decode_b200 import synth

    def proj(rows):
        if cfg.fmt == synth.FMT_NVFP4 and rows > 4:
            return 2 * ((rows + 31) // 32)
        return (rows + 3) // 4

    R = cfg.B
    per_layer = proj(R) + 1 + proj(R) + (6 if cfg.n_experts else 2 * proj(R))
    return 1 + cfg.L * per_layer + proj(R)


HEADLINE = "7b"                                   # the workload the metric is quoted on
SECONDARY = ("9b", "9b_b32", "9b_b32_fp8", "27b", "moe")   # the other decode workloads, one line


PERSISTENT = False   # --persistent: batch-1 dense steps as one persistent kernel (BW_STEP_PERSISTENT)


def uses_persistent_step(cfg) -> bool:
    """Whether the timed steps run as bw_decode_step's one-kernel persistent step."""
    return PERSISTENT and cfg.B == 1 and cfg.n_experts == 0


def measure(cfg, model, kv, dm, rank, world, local, steps, warmup, cpu_budget, stream, with_kernels=True):
    """Timed decode of one workload: device-timed graph replays, the end-to-end
    C-ABI loop with host tokens, the dominant kernel's roofline, and (rank 0,
    one GPU) the CPU oracle on a bounded sample."""
    from token_decode_b200 import bw, runtime, synth
    dkv = runtime.DeviceKV(kv)
    dec = runtime.Decoder(dm, dkv, cfg.B)
    toks = synth.start_tokens(cfg, rank)[: cfg.B]

    def reset():
        dec.tokens_in.copy_(toks)
        dec.pos.fill_(cfg.ctx)

    pers = uses_persistent_step(cfg)
    G = 16  # steps per captured graph
    graphs = {}

    def graph_for(n):
        if n not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                dec.step(advance=True, stream=stream, persistent=pers)   # warm the launch path outside capture
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(n):
                        dec.step(advance=True, stream=stream, persistent=pers)
            graphs[n] = g
        return graphs[n]

    def plan(nsteps, start):
        """Replays of (graph size) covering nsteps, restarting generations at cfg.steps."""
        out, done, p = [], 0, start
        while done < nsteps:
            left_gen = cfg.steps - p
            if left_gen <= 0:
                out.append("reset")
                p = 0
                continue
            n = min(G, nsteps - done, left_gen)
            out.append(n)
            done += n
            p += n
        return out, p

    def run(ops):
        with torch.cuda.stream(stream):
            for op in ops:
                if op == "reset":
                    reset()
                else:
                    graph_for(op).replay()

    torch.cuda.synchronize()
    warm_ops, p_after = plan(warmup, 0)
    timed_ops, _ = plan(steps, p_after)
    for op in warm_ops + timed_ops:
        if op != "reset":
            graph_for(op)
    # a graph's first replay also uploads it to the device: replay every graph
    # the timed region uses once, untimed
    run(timed_ops)
    # capture and upload ran extra steps: rebuild the exact start, then warm up
    with torch.cuda.stream(stream):
        reset()
    run(warm_ops)
    stream.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        run(timed_ops)
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    ms_local = e0.elapsed_time(e1)
    err = bw.read_error(dec.ws, stream)
    ms, value = job_throughput(ms_local, steps * cfg.B, world)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ms_step = ms / steps
    graphs.clear()

    # ---- end to end through the C ABI: host tokens in, host tokens out, every step
    pin_in = torch.empty(cfg.B, dtype=torch.int32).pin_memory()
    pin_out = torch.empty(cfg.B, dtype=torch.int32).pin_memory()
    pin_in.copy_(toks)
    n_e2e = min(steps, 32)
    with torch.cuda.stream(stream):
        reset()
    stream.synchronize()

    def e2e_step():
        with torch.cuda.stream(stream):
            dec.tokens_in.copy_(pin_in, non_blocking=True)
            dec.step(stream=stream, persistent=pers)
            dec.pos += 1
            pin_out.copy_(dec.tokens_out, non_blocking=True)
        stream.synchronize()
        pin_in.copy_(pin_out)

    for _ in range(3):
        e2e_step()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    f1.record(stream)
    f1.synchronize()
    _, e2e_value = job_throughput(f0.elapsed_time(f1), n_e2e * cfg.B, world)

    avg_ctx = cfg.ctx + (cfg.steps + 1) / 2
    peak, peak_kind = _peaks()
    kern, moe_bytes = {}, 0
    if with_kernels and (cfg.n_experts or not uses_persistent_step(cfg)):
        from token_decode_b200 import kernel_bench
        kern = kernel_bench.run_all(dm, dkv, cfg.B, stream, cfg.ctx + cfg.steps // 2, reps=5)
        moe_bytes = kern["moe"]["bytes_per_launch"] if cfg.n_experts else 0
    sb = step_bytes(cfg, model, avg_ctx, moe_bytes)
    step_gbs = sb / (ms_step / 1000.0) / 1e9
    if uses_persistent_step(cfg):
        # one kernel per step: its algorithmic bytes are the step's
        roof = {"bound": "hbm", "kernel": "step_persistent_kernel (the whole batch-1 step)",
                "achieved": round(step_gbs, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": round(step_gbs / peak, 4), "traffic": _ncu_traffic("step", cfg.name),
                "bytes_per_launch": int(sb), "avg_launch_us": round(ms_step * 1000.0, 2)}
        launches = 1
    else:
        dom = max(kern, key=lambda k: kern[k]["us_per_launch"] * kern[k]["launches"])
        roof = {"bound": "hbm", "kernel": KERNEL_NAMES.get(dom, dom), "achieved": kern[dom]["GBps"],
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(kern[dom]["GBps"] / peak, 4),
                "traffic": _ncu_traffic(dom, cfg.name), "bytes_per_launch": kern[dom]["bytes_per_launch"],
                "avg_launch_us": kern[dom]["us_per_launch"]}
        launches = step_launches(cfg)
    entry = {
        "workload": cfg.name, "value": round(value, 3), "unit": "tok/s", "batch": cfg.B,
        "ms_per_step": round(ms_step, 5), "steps": steps,
        "path": "persistent kernel (1 launch per step)" if uses_persistent_step(cfg)
                else "kernel chain (%d launches per step)" % step_launches(cfg),
        "dtype": ("q4_0 weights, fp32 accumulate" if cfg.fmt == synth.FMT_Q4_0 else
                  "nvfp4 weights, fp32 accumulate") + (", e4m3 KV (per-layer scales)" if cfg.kv_fp8 else ", fp16 KV"),
        "hbm_gbs_step": round(step_gbs, 1),
        "roofline_step_frac_of_8tbs": round(step_gbs / NOMINAL_HBM_GBS, 4),
        "roofline_step_frac_of_measured": round(step_gbs / peak, 4),
        "bytes_per_step": int(sb),
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": "tok/s", "steps": n_e2e,
                "h2d_bytes_per_step": 4 * cfg.B, "d2h_bytes_per_step": 4 * cfg.B,
                "path": "bw_decode_step via the C ABI, pinned host tokens in/out, sync each step"},
        "gpu_launches": launches * steps,
        "device_error_word": err,
        "clocks": clk.summary(),
    }
    if kern:
        entry["kernels"] = kern
    if cfg.verify_k:
        entry["verify_pass"] = verify_pass(cfg, dm, kv, stream, ms_step)
        entry["speculative"] = speculative(cfg, dm, kv, stream, ms_step)
    if cfg.prefill_prompt and cfg.B == 1:
        entry["prefill"] = prefill(cfg, dm, kv, stream)
    if rank == 0 and world == 1 and cpu_budget > 0:
        entry["cpu_baseline"] = cpu_baseline(cfg, model, kv, toks, budget_s=cpu_budget)
    del dec, dkv
    return entry


def verify_pass(cfg, dm, kv, stream, ms_plain):
    """Device time of one speculative-verify pass (the last token plus K drafts
    as K+1 rows of one step, bw_decode_step with n_rows = K+1) against a plain step."""
    from token_decode_b200 import bw, runtime, synth
    R = cfg.verify_k + 1
    dkv = runtime.DeviceKV(kv.clone())
    dec = runtime.Decoder(dm, dkv, 1, n_rows=R)
    t0 = synth.start_tokens(cfg, 0)[:1].tolist()
    rows = t0 + synth.draft_tokens(cfg, cfg.verify_k, 0)[0].tolist()
    dec.tokens_in.copy_(torch.tensor(rows, dtype=torch.int32))
    dec.pos.fill_(cfg.ctx)
    n = 8
    with torch.cuda.stream(stream):
        dec.step(stream=stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(n):
                dec.step(stream=stream)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / n
    err = bw.read_error(dec.ws, stream)
    del g
    return {"rows": R, "drafts": cfg.verify_k, "ms_per_pass": round(ms, 4),
            "vs_plain_step": round(ms / ms_plain, 3), "device_error_word": err,
            "path": "kernel chain, %d rows per projection" % R}


def prefill(cfg, dm, kv, stream):
    """Chunked prefill (bw_prefill) of a synthetic prompt of cfg.prefill_prompt
    tokens at positions 0.. into a copy of the cache: device time of one whole
    prefill after one untimed run (the time to the first token, less the host)."""
    from token_decode_b200 import bw, runtime, synth
    chunk = max(1, min(bw.MAX_VERIFY_ROWS, 32 // (cfg.nq // cfg.nkv)))
    pf = runtime.Prefiller(dm, runtime.DeviceKV(kv.clone()), chunk)
    tok = synth.prompt_tokens(cfg, cfg.prefill_prompt, 0).to("cuda")
    with torch.cuda.stream(stream):
        pf.run(tok, 0, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pf.run(tok, 0, stream=stream)
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    err = bw.read_error(pf.ws, stream)
    n = cfg.prefill_prompt
    return {"prompt_tokens": n, "chunk": chunk, "steps": -(-n // chunk), "ms": round(ms, 2),
            "tok_s": round(n / ms * 1000.0, 1), "device_error_word": err,
            "path": "bw_prefill: chunks of %d rows through bw_decode_step, logits for the last row only" % chunk}


def speculative(cfg, dm, kv, stream, ms_plain, passes=8):
    """Speculative decoding with the (synthetic, random-init) MTP draft head, K =
    cfg.verify_k drafts per pass: device time of CUDA-graph replays of whole
    passes (draft, verify, accept) and the tokens they emitted, counted on the
    device.  A random draft head rarely guesses the main model's greedy token,
    so the measured acceptance is low; the rate at full acceptance ((K + 1)
    tokens per pass at the same pass time) is reported beside it."""
    from token_decode_b200 import bw, runtime, synth
    K = cfg.verify_k
    head = synth.make_draft_head(cfg, "cuda", seed=0)
    ddh = runtime.DeviceDraftHead(head)
    sd = runtime.SpecDecoder(dm, runtime.DeviceKV(kv.clone()), ddh, K)
    tok = int(synth.start_tokens(cfg, 0)[0])
    total = torch.zeros(1, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(stream):
        sd.start(tok, cfg.ctx, stream=stream)
        sd.step_pass(stream=stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(passes):
                sd.step_pass(stream=stream)
                total.add_(sd.n_acc + 1)
        g.replay()
        total.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    n = int(total.item())
    err = bw.read_error(sd.ver.ws, stream) | bw.read_error(sd.mws, stream)
    del g
    ms_pass = ms / passes
    return {"drafts_per_pass": K, "draft_head": "synthetic random-init (N(0,0.02)), vocabulary %d" % head.w.N,
            "passes": passes, "tokens": n, "accepted_per_pass": round(n / passes - 1, 3),
            "ms_per_pass": round(ms_pass, 4), "effective_tok_s": round(n / (ms / 1000.0), 3),
            "tok_s_if_all_accepted": round((K + 1) / (ms_pass / 1000.0), 3),
            "plain_step_tok_s": round(1000.0 / ms_plain, 3), "device_error_word": err,
            "path": "bw_mtp_draft (2K launches) + bw_decode_step (K+1 rows) + bw_spec_accept, one graph"}


KERNEL_NAMES = {"gu": "gemv_kernel (fused RMSNorm + gate/up + SiLU gate)", "down": "gemv_kernel (down + residual)",
                "attn": "attn_g_kernel (paged GQA decode attention; attn_kernel above 8 query rows per kv head)", "qkv": "gemv_kernel (RMSNorm + QKV)",
                "o": "gemv_kernel (O + residual)", "lm_head": "gemv_kernel (LM head + argmax)",
                "moe": "MoE FFN (route + grouped expert GEMVs + combine)"}


def run_ours(args):
    from token_decode_b200 import build, bw, runtime, synth
    ws_, rank, local = dist_env()
    if ws_ > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    build.build()
    bw.lib()
    stream = torch.cuda.Stream()
    names = [args.config] + ([] if args.only else [n for n in SECONDARY if n != args.config])
    entries = {}
    cache = {}
    for i, name in enumerate(names):
        cfg = synth.CONFIGS[name]
        key = (cfg.L, cfg.H, cfg.nq, cfg.nkv, cfg.hd, cfg.F, cfg.V, cfg.fmt, cfg.n_experts)
        if key not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            model = synth.make_model(cfg, "cuda", seed=rank)
            cache[key] = (model, runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS))
        model, dm = cache[key]
        if dm.c.rope_max_pos < cfg.max_pages * synth.PAGE_TOKENS:
            dm = runtime.DeviceModel(model, cfg.max_pages * synth.PAGE_TOKENS)
            cache[key] = (model, dm)
        kv = (synth.make_kv_fp8 if cfg.kv_fp8 else synth.make_kv)(cfg, "cuda", seed=rank)
        head = i == 0
        steps = args.steps if head else max(4, min(args.steps, 16))
        entries[name] = measure(cfg, model, kv, dm, rank, ws_, local, steps, args.warmup,
                                0 if args.no_cpu_baseline else (args.cpu_budget if head else args.cpu_budget / 3),
                                stream)
        del kv
    h = entries[names[0]]
    hcfg = synth.CONFIGS[names[0]]
    line = {
        "metric": METRIC,
        "value": h["value"],
        "unit": "tok/s",
        "n_gpus": ws_,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": h["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": h["dtype"],
        "data": "synthetic (seeded random-init weights N(0,0.02) quantized; N(0,1) fp16 KV context)",
        "config": workload_config(hcfg, ws_),
        "l2": "inputs larger than L2: every step streams the whole model (%.2f GB for %s)" % (
            h["bytes_per_step"] / 1e9, hcfg.name),
        "timing": "CUDA graphs of 16 steps, on-device token/position advance; CUDA events on the launching stream",
    }
    for k in ("path", "hbm_gbs_step", "roofline_step_frac_of_8tbs", "roofline_step_frac_of_measured",
              "bytes_per_step", "roofline", "kernels", "e2e", "gpu_launches", "device_error_word", "clocks",
              "cpu_baseline", "verify_pass", "speculative", "prefill"):
        if k in h:
            line[k] = h[k]
    line["configs"] = {n: e for n, e in entries.items() if n != names[0]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_ > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def _oracle_setup(cfg, model, kv, n_layers=None):
    import oracle
    oracle.build()
    return oracle, oracle.Model(model, n_layers=n_layers), oracle.KV(kv, layers=n_layers)


def _oracle_token_seconds(oracle, om, okv, cfg, tok, n_layer_samples, t_budget, n_host_layers):
    """Seconds of one full oracle decode token, estimated from a bounded sample:
    the head alone (embedding + final norm + LM head) and single layers."""
    t = time.perf_counter()
    oracle.decode_token(om, okv, 0, tok, cfg.ctx, layers=(0, 0))
    t_head = time.perf_counter() - t
    per_layer = []
    for i in range(n_layer_samples):
        l = (i * 7) % n_host_layers
        t = time.perf_counter()
        oracle.decode_token(om, okv, 0, tok, cfg.ctx, layers=(l, l + 1))
        per_layer.append(max(0.0, time.perf_counter() - t - t_head))
        if sum(per_layer) > t_budget:
            break
    return t_head + cfg.L * statistics.mean(per_layer), t_head, per_layer


def cpu_baseline(cfg, model, kv, toks, budget_s=20.0, host_layers=4):
    """The oracle as it stands, one host thread, on a bounded sample of one
    sequence's decode token (its first host_layers layers are copied to the host)."""
    nl = min(cfg.L, host_layers)
    oracle, om, okv = _oracle_setup(cfg, model, kv, nl)
    tok_s, t_head, per_layer = _oracle_token_seconds(oracle, om, okv, cfg, int(toks[0]), 64, budget_s, nl)
    return {"value": round(1.0 / tok_s, 5), "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": f"embedding + LM head once ({t_head:.2f} s) and {len(per_layer)} single "
                      f"layers of one {cfg.name} sequence at ctx {cfg.ctx}, scaled to {cfg.L} layers "
                      f"(one token = {tok_s:.1f} s; the sequences of a batch run one after another), "
                      f"single-threaded fp32 C",
            "host_cores_total": os.cpu_count()}


def run_reference(args):
    """The CPU oracle as the reference arm: each step is one layer of the decode
    step (cycling through the layers) plus the timed embedding/LM-head share."""
    ws_, rank, local = dist_env()
    if rank != 0:
        return
    from token_decode_b200 import synth
    cfg = synth.CONFIGS[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    model = synth.make_model(cfg, dev, seed=0)
    kv = synth.make_kv(cfg, dev, seed=0)
    oracle, om, okv = _oracle_setup(cfg, model, kv)
    tok = int(synth.start_tokens(cfg, 0)[0])
    t = time.perf_counter()
    oracle.decode_token(om, okv, 0, tok, cfg.ctx, layers=(0, 0))
    t_head = time.perf_counter() - t
    for i in range(args.warmup):
        oracle.decode_token(om, okv, 0, tok, cfg.ctx, layers=(i % cfg.L, i % cfg.L + 1))
    per = []
    t_all = time.perf_counter()
    for i in range(args.steps):
        l = (i * 7) % cfg.L
        t = time.perf_counter()
        oracle.decode_token(om, okv, 0, tok, cfg.ctx, layers=(l, l + 1))
        per.append(max(0.0, time.perf_counter() - t - t_head))
    wall = time.perf_counter() - t_all
    tok_s = t_head + cfg.L * statistics.mean(per)
    value = cfg.B / tok_s
    line = {"metric": METRIC, "value": round(value, 5), "unit": "tok/s", "n_gpus": ws_,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * wall / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32 (CPU oracle)",
            "data": "synthetic (seeded random-init weights)", "impl": "reference",
            "config": workload_config(cfg, ws_),
            "cpu_baseline": {"value": round(value, 5), "unit": "tok/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step = one of the {cfg.L} layers of one decode token "
                                       f"(+ embedding/LM head timed once, {t_head:.2f} s), scaled "
                                       f"to a full token"},
            "e2e": {"value": round(value, 5), "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--config", default="7b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--only", action="store_true", help="measure only --config (no other workloads)")
    ap.add_argument("--persistent", action="store_true",
                    help="batch-1 dense steps as one persistent kernel (BW_STEP_PERSISTENT)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    global PERSISTENT
    PERSISTENT = args.persistent
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
