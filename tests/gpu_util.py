"""Shared helpers of the GPU parity tests (imported by tests only)."""
import numpy as np
import torch


def rel_err(got, want) -> float:
    """Normwise relative error max|g - w| / max|w| (elementwise relative error is
    undefined near zero)."""
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    den = np.max(np.abs(w))
    return float(np.max(np.abs(g - w)) / (den if den > 0 else 1.0))


def bits(a):
    return np.ascontiguousarray(np.asarray(a, np.float32)).view(np.uint32)


def cuda_ok() -> bool:
    return torch.cuda.is_available()


# the tolerance the workload states for fp32-accumulated hidden states and logits
TOL = 2e-3
# argmax tokens must agree whenever the oracle's top-2 margin exceeds this
MARGIN = 1e-2


def check_kv(gpu_pools, ora_pools, page_table, B, first_pos, n_new, page_tokens=16):
    """The KV cache after a step: every slot the step did not write is
    bit-identical to the oracle's; the rows it wrote (positions first_pos ..
    first_pos + n_new - 1 of each sequence) agree within the tolerance (fp16
    roundings of values whose fp32 sums differ only by summation order, or by
    the tensor-core path's fp16 activations)."""
    pt = np.asarray(page_table.cpu() if hasattr(page_table, "cpu") else page_table)
    for gpu_pool, ora_pool in zip(gpu_pools, ora_pools):
        # pools are [page][kv head][slot][dim]: bring (page, slot) to the front
        g = gpu_pool.cpu().numpy().view(np.uint16).transpose(0, 2, 1, 3)
        o = np.asarray(ora_pool).view(np.uint16).transpose(0, 2, 1, 3)
        written = np.zeros((g.shape[0], g.shape[1]), dtype=bool)   # [page][slot]
        for b in range(B):
            for p in range(first_pos, first_pos + n_new):
                written[pt[b, p // page_tokens], p % page_tokens] = True
        untouched = ~written
        assert np.array_equal(g[untouched], o[untouched])
        gw = g[written].view(np.float16).astype(np.float64)
        ow = o[written].view(np.float16).astype(np.float64)
        assert rel_err(gw, ow) < TOL


def parallel_rows(fn, items):
    """fn(item) for every item, on host threads (the oracle's C calls release the
    interpreter lock; rows of different sequences touch disjoint KV pages)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    items = list(items)
    if len(items) <= 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(max_workers=min(len(items), os.cpu_count() or 1)) as ex:
        return list(ex.map(fn, items))
