"""Full-size parity helper: the CPU oracle over row blocks in host threads.

Per-row groups are independent, so running the oracle's definition on each
block of rows gives exactly the whole matrix's result; nothing of the
method's arithmetic lives here.  The C oracle releases the GIL inside each
call, so the blocks run on all host cores.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle


def host_threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(64, n))


def _bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def compare_rows(w: np.ndarray, got: dict, qbits: int, p: float, export: bool = True,
                 block_rows: int | None = None) -> dict:
    """Compare the GPU outputs in ``got`` (host arrays keyed "dq", "packed",
    "codes", "scale_f16", "scale_f32", "clip"; any subset) with the oracle on
    every row of ``w``.  Returns {output: mismatch count} (all zero when the
    outputs agree bit for bit) and the first mismatching row per output."""
    rows, cols = w.shape
    if block_rows is None:
        block_rows = max(1, min(rows, (1 << 22) // max(cols, 1)))
    starts = list(range(0, rows, block_rows))

    def one(r0):
        r1 = min(rows, r0 + block_rows)
        ref = oracle.quantize(np.ascontiguousarray(w[r0:r1]), qbits, p, export=export)
        res = {}
        if ref.status != oracle.OR_OK:
            res["status"] = (1, r0)
            return res
        for key, g in got.items():
            want = getattr(ref, key)
            g_blk = g[r0:r1]
            bad = np.nonzero(_bits(np.ascontiguousarray(g_blk)) != _bits(want))[0]
            res[key] = (int(bad.size), r0 + int(bad[0]) if bad.size else None)
        return res

    counts = {k: 0 for k in got}
    first = {k: None for k in got}
    with ThreadPoolExecutor(max_workers=host_threads()) as ex:
        for res in ex.map(one, starts):
            if "status" in res:
                counts["status"] = counts.get("status", 0) + 1
                continue
            for k, (n, r) in res.items():
                counts[k] += n
                if n and (first[k] is None or r < first[k]):
                    first[k] = r
    return {"mismatches": counts, "first_row": first}


def quantize_many(items, qbits: int, p: float, export: bool) -> list:
    """The oracle on several whole tensors in parallel host threads."""
    def one(w):
        return oracle.quantize(np.ascontiguousarray(w), qbits, p, export=export)
    with ThreadPoolExecutor(max_workers=host_threads()) as ex:
        return list(ex.map(one, items))
