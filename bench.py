"""Benchmark: weight GB/s through the fused int6/int8 fake-quant + export pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one "step"): the bandwidth-stress weight set -- fp32 matrices
16384x16384, 65536x4096 and 262144x512 plus their bf16 copies (Student-t,
3 degrees of freedom, std 0.02, drawn on the GPU from a seeded generator).
For each of the six matrices a step makes two libgq calls:
  (i)  int6 per row at p = 0.9999: percentile clip select + scale + round +
       clamp + dequant + 4-in-3 pack in ONE kernel (outputs w_hat, packed
       codes, binary16 scales);
  (ii) int8 per row absmax (outputs w_hat, int8 codes, binary16 scales).
Every matrix is larger than L2, so no flush is needed between steps.

value = input weight bytes of all calls / device time of the K timed steps
(CUDA events, barrier + synchronize on both sides, max over ranks); the JSON
line also carries the roofline of the fused kernel, the CPU oracle baseline
(rank 0, N = 1), an end-to-end figure with host buffers, the SM clocks seen
during the timed region, and separate measurements of the other operations
of the path (STE backward, dequant on load, per-tensor select, batched
exports of the model-shaped weight sets, passthrough).

Multi-GPU (torchrun): every rank quantizes its own weight set (independent
replicas, weak scaling); there is no collective on the data path, only a
barrier and a max-reduction of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "weight GB/s through fused fake-quant+export and % of B200 HBM peak"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0          # B200 HBM3e data-sheet figure, reported beside the measured peak
FALLBACK_BF16_TFLOPS = 1590.0
WORKLOAD = ("bandwidth stress: fp32 16384x16384, 65536x4096, 262144x512 and bf16 copies "
            "(Student-t nu=3, std 0.02); per matrix int6 per-row p=0.9999 clip-select+"
            "fake-quant+pack (w_hat, packed, fp16 scales) and int8 per-row absmax "
            "(w_hat, int8 codes, fp16 scales)")


# ------------------------------------------------------------ distributed --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (the slowest rank sets the job's time)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_throughput(units_per_rank: float, elapsed_s_per_rank: float, world: int, device=None):
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    total = sum_over_ranks(units_per_rank, world, device)
    t = max_over_ranks(elapsed_s_per_rank, world, device)
    return total / t, t


# ------------------------------------------------------------------ peaks --

def bf16_peak():
    """Dense bf16 tensor peak (TFLOP/s): the measured cuBLAS burst figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FUSED_KERNEL_SOURCES = ("gq_device.cuh", "gq_kernels.cuh", "gq_rowquant_tma.cuh")


def kernel_source_hash():
    """Hash of the sources the fused per-row kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int6_int8_weight_b200", "csrc")
    for name in FUSED_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_PATH = os.path.join(ROOT, "profiles", "rowquant_traffic.json")


def traffic_per_launch(kernel_hash, calls):
    """Average ncu DRAM bytes (read + write) of one full-size launch of the
    step, scaled from the per-row traffic of a smaller capture of the same
    launches (traffic grows with the rows a launch processes), if it was taken
    on the current kernel sources; else (None, None)."""
    try:
        with open(TRAFFIC_PATH) as f:
            d = json.load(f)
    except Exception:
        return None, None
    if d.get("kernel_source_hash") != kernel_hash:
        return None, None
    per = d.get("per_call", {})
    tot = 0.0
    for _, _, _, name in calls:
        if name not in per:
            return None, None
        rows = int(name.split()[1].split("x")[0])
        tot += per[name]["dram_bytes_per_row"] * rows
    return tot / len(calls), d


def record_traffic(csv_path, shrink):
    """Turn the ncu CSV of one shrunken step (dram__bytes_read.sum,
    dram__bytes_write.sum, gpu__time_duration.sum of the 12 fused launches,
    in call order) into profiles/rowquant_traffic.json."""
    import csv
    rows = [r for r in csv.reader(open(csv_path)) if len(r) > 10]
    H = rows[0]
    iid, mi, vi, ki = H.index("ID"), H.index("Metric Name"), H.index("Metric Value"), H.index("Kernel Name")
    per_id, names = {}, {}
    for r in rows[1:]:
        if "rowquant" not in r[ki]:
            continue
        per_id.setdefault(int(r[iid]), {})[r[mi]] = float(r[vi].replace(",", ""))
    ids = sorted(per_id)
    calls = []
    for dt in ("f32", "bf16"):
        for (R, Cc) in synth.BANDWIDTH_SHAPES:
            for q in (6, 8):
                calls.append((f"{dt} {R}x{Cc} int{q}", R // shrink, Cc, 4 if dt == "f32" else 2, q))
    assert len(ids) == len(calls), (len(ids), len(calls))
    per_call = {}
    for i, (name, r_small, cols, esz, q) in zip(ids, calls):
        m = per_id[i]
        dram = m["dram__bytes_read.sum"] + m["dram__bytes_write.sum"]
        prb = 3 * ((cols + 3) // 4) if q == 6 else cols
        alg = r_small * (cols * 2 * esz + prb + 2)
        per_call[name] = {"rows_captured": r_small, "dram_read_bytes": int(m["dram__bytes_read.sum"]),
                          "dram_write_bytes": int(m["dram__bytes_write.sum"]),
                          "algorithmic_bytes": int(alg), "traffic_over_algorithmic": round(dram / alg, 4),
                          "dram_bytes_per_row": dram / r_small, "ns": m.get("gpu__time_duration.sum")}
    out = {"kernel": "gq::rowquant_tma_kernel<false> (no column scales)",
           "kernel_source_hash": kernel_source_hash(), "shrink": shrink, "per_call": per_call,
           "note": (f"ncu dram__bytes_read.sum + dram__bytes_write.sum (1 pass) of each of the 12 fused "
                    f"launches of one step with every matrix's rows divided by {shrink}; bench.py scales "
                    "each launch's bytes per row to the full row count"),
           "command": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                       f"--clock-control none -k regex:rowquant -s 36 -c 12 --csv --log-file "
                       f"{csv_path} python bench.py --shrink {shrink} --steps 1 "
                       "--warmup 3 --skip-cpu --skip-rows --no-e2e")}
    with open(TRAFFIC_PATH, "w") as f:
        json.dump(out, f, indent=1)
    return out


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="gq_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 8:
                        rows.append(parts)
            os.unlink(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s >= 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def physical_gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


REJECT = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


# ----------------------------------------------------------- GPU workload --

class Workload:
    """The six matrices, their preallocated outputs and one descriptor per call."""

    def __init__(self, gq, device, seed, only=None, shrink=1):
        """``only``: restrict to the calls whose name contains this text
        (e.g. "f32 16384x16384 int6"), for profiling a single launch.
        ``shrink``: divide every matrix's row count by this factor (a smaller
        case of the same launches for counter captures; never a bench line)."""
        self.gq = gq
        self.mats = []
        self.shrink = shrink
        want = []
        for dt in ("f32", "bf16"):
            for i, (r, c) in enumerate(synth.BANDWIDTH_SHAPES):
                # calls are named by the full-size shape, also when shrunken
                names = [f"{dt} {r}x{c} int{q}" for q in (6, 8)]
                if only is None or any(only in nm for nm in names):
                    want.append((dt, i, r // shrink, c))
        mats32 = {}
        for dt, i, r, c in want:
            if i not in mats32:
                mats32[i] = synth.draw_bandwidth_matrix(r, c, i, device=device, seed=seed)
        for dt, i, r, c in want:
            self.mats.append(mats32[i] if dt == "f32" else mats32[i].to(torch.bfloat16))
        if not any(dt == "f32" for dt, *_ in want):
            mats32.clear()
        self.calls = []     # (desc array, input bytes, algorithmic bytes, name)
        self.outs = []
        for W in self.mats:
            rows, cols = W.shape
            esz = W.element_size()
            for qbits, p in ((6, 0.9999), (8, 1.0)):
                name = f"{'f32' if esz == 4 else 'bf16'} {rows * shrink}x{cols} int{qbits}"
                if only is not None and only not in name:
                    continue
                dq = torch.empty_like(W)
                prb = gq.gq_packed_row_bytes(cols, qbits)
                packed = torch.empty((rows, prb), dtype=torch.uint8, device=device)
                h = torch.empty(rows, dtype=torch.float16, device=device)
                d = gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=qbits,
                                gran=gq.GQ_PER_ROW, reserved=0, rows=rows, cols=cols, ld=cols,
                                p=p, dq=dq.data_ptr(), codes=0, packed=packed.data_ptr(),
                                scale_f16=h.data_ptr(), scale_f32=0, clip=0)
                arr = gq._arr([d])
                in_bytes = rows * cols * esz
                alg = rows * cols * (2 * esz) + rows * prb + 2 * rows
                self.calls.append((arr, in_bytes, alg, name))
                self.outs.append((dq, packed, h))
        self.in_bytes = sum(c[1] for c in self.calls)
        self.alg_bytes = sum(c[2] for c in self.calls)

    def step(self, stream_handle, events=None):
        L = self.gq.LIB
        for i, (arr, _, _, _) in enumerate(self.calls):
            if events is not None:
                events[2 * i].record()
            st = L.gq_export_pack(arr, 1, None, 0, None, stream_handle)
            if events is not None:
                events[2 * i + 1].record()
            if st != 0:
                raise RuntimeError(f"gq_export_pack failed: {st}")


def time_region(fn, steps, world, device):
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for k in range(steps):
        fn(k)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end) / 1e3


def flush_l2(buf):
    buf.add_(1)     # writes 2x L2 worth of bytes


def measure_rows(gq, device, peak):
    """Each remaining operation of the path, timed alone with CUDA events
    (5 warm-ups, median of 50 reps; L2 flushed between reps when the working
    set fits L2).  The model-shaped batches (the single 512x1536 matrix, the
    9-layer export, the 11-layer training step, the 12-layer mixed-bit export)
    also carry the single-threaded CPU oracle's time on the same inputs."""
    out = {}
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)   # 256 MiB

    def timed(fn, reps=50, flush_between=False):
        for _ in range(5):
            fn()
        ts = []
        for _ in range(reps):
            if flush_between:
                flush_l2(flush)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            e.synchronize()
            ts.append(s.elapsed_time(e) / 1e3)
        return statistics.median(ts)

    def record(name, seconds, alg_bytes, in_bytes, launches, note="", flops=None):
        gbs = alg_bytes / seconds / 1e9
        out[name] = {"ms": round(seconds * 1e3, 4), "weight_gbs": round(in_bytes / seconds / 1e9, 1),
                     "alg_gbs": round(gbs, 1), "hbm_frac": round(gbs / peak, 3),
                     "launches": launches, **({"note": note} if note else {})}
        if flops is not None:
            tf = flops / seconds / 1e12
            out[name]["tflops"] = round(tf, 1)
            out[name]["tensor_frac"] = round(tf / tf_peak, 3)

    # STE backward on the 16384^2 shape: copy (fp32) and accumulate (bf16)
    n = 16384 * 16384
    g32 = torch.randn(n, device=device)
    w32 = torch.empty_like(g32)
    record("ste_bwd copy f32 16384^2", timed(lambda: gq.gq_ste_bwd(g32.data_ptr(), w32.data_ptr(), 0, n, 0)),
           8 * n, 4 * n, 1)
    gb = g32.to(torch.bfloat16)
    wb = torch.zeros_like(gb)
    record("ste_bwd accumulate bf16 16384^2",
           timed(lambda: gq.gq_ste_bwd(gb.data_ptr(), wb.data_ptr(), 1, n, 1)), 6 * n, 2 * n, 1)
    del g32, w32, gb, wb

    # dequant on load of int6 codes to fp32, 16384^2
    W = synth.draw_bandwidth_matrix(16384, 16384, 0, device=device)
    (o,) = gq.export_pack([gq.Request(W, 6, 0.9999, want_dq=False)], check_status=False)
    outd = torch.empty_like(W)
    record("dequant int6 -> f32 16384^2",
           timed(lambda: gq.gq_dequant(o.packed.data_ptr(), o.scale_f16.data_ptr(), 6, 0, 16384, 16384,
                                       outd.data_ptr(), 0)),
           n * 4.75 + 2 * 16384, n * 0.75, 1)
    # training fake-quant forward bf16 (w_hat only)
    Wb = W.to(torch.bfloat16)
    dqb = torch.empty_like(Wb)
    d = gq.GQTensor(w=Wb.data_ptr(), dtype=1, qbits=6, gran=0, reserved=0, rows=16384, cols=16384,
                    ld=16384, p=1.0, dq=dqb.data_ptr(), codes=0, packed=0, scale_f16=0, scale_f32=0, clip=0)
    arr = gq._arr([d])
    record("fakequant train bf16 16384^2 int6 absmax",
           timed(lambda: gq.LIB.gq_fakequant_fwd(arr, 1, 0, None, 0, None, None)), 4 * n, 2 * n, 1)
    # snapshot averaging fused with the training fake-quant (bf16 weights,
    # binary32 running mean and EMA updated in place; no w_hat written)
    avg = torch.zeros(16384, 16384, device=device)
    d0 = gq.GQTensor(w=Wb.data_ptr(), dtype=1, qbits=6, gran=0, reserved=0, rows=16384, cols=16384,
                     ld=16384, p=1.0, dq=0, codes=0, packed=0, scale_f16=0, scale_f32=0, clip=0)
    arr0 = gq._arr([d0])
    for kind, name, count in ((gq.GQ_AVG_MEAN, "mean", 5), (gq.GQ_AVG_EMA, "EMA 0.997", 0)):
        aa = gq._avg_arr([gq.GQAvg(avg=avg.data_ptr(), kind=kind, decay=0.997, count=count)])
        record(f"fakequant + snapshot {name} bf16 16384^2 int6 (average only)",
               timed(lambda: gq.LIB.gq_fakequant_average(arr0, aa, 1, 0, None, 0, None, None)),
               10 * n, 2 * n, 1, note="reads w (2 B) and the binary32 average (4 B), writes the average (4 B)")
    # AWQ: int6 per-row export of the column-scaled bf16 weight (w_hat,
    # packed codes, fp16 scales), column scales from synthetic statistics
    t_awq = torch.from_numpy(synth.awq_col_scales(np.random.default_rng(3), 16384)).to(device)
    pk = torch.empty(16384, gq.gq_packed_row_bytes(16384, 6), dtype=torch.uint8, device=device)
    h16 = torch.empty(16384, dtype=torch.float16, device=device)
    da = gq.GQTensor(w=Wb.data_ptr(), dtype=1, qbits=6, gran=0, reserved=0, rows=16384, cols=16384,
                     ld=16384, p=0.9999, dq=dqb.data_ptr(), codes=0, packed=pk.data_ptr(),
                     scale_f16=h16.data_ptr(), scale_f32=0, clip=0, col_scale=t_awq.data_ptr())
    arra = gq._arr([da])
    record("AWQ column-scaled export bf16 16384^2 int6 p=0.9999",
           timed(lambda: gq.LIB.gq_export_pack(arra, 1, None, 0, None, None)),
           4.75 * n + 2 * 16384 + 4 * 16384, 2 * n, 1,
           note="reads w (2 B), writes w_hat (2 B) + packed (0.75 B); pipelined row kernel, each staged row rescaled in place")
    del W, o, outd, Wb, dqb, avg, pk, h16, t_awq

    # the consuming GEMM with the int6 dequant in its weight load (tcgen05),
    # against cuBLAS on the pre-dequantized bf16 weight; decode-like (small M,
    # weight-read bound) and prefill-like (tensor bound) shapes
    tf_peak, _ = bf16_peak()
    for M, N, K in ((16, 16384, 16384), (128, 16384, 16384), (4096, 8192, 8192)):
        Wg = synth.draw_bandwidth_matrix(N, K, 0, device=device)
        (q,) = gq.export_pack([gq.Request(Wg, 6, 0.9999, want_dq=False)], check_status=False)
        del Wg
        X = (torch.randn(M, K, device=device) * 0.5).to(torch.bfloat16)
        Y = torch.empty(M, N, device=device)
        wbytes = q.packed.numel() + 2 * N
        alg = wbytes + 2 * M * K + 4 * M * N
        fl = 2 * M * N * K
        record(f"gemm dequant-on-load int6 M{M} N{N} K{K}",
               timed(lambda: gq.gemm_dequant(X, q.packed, q.scale_f16, 6, y=Y), flush_between=True),
               alg, wbytes, 1, note="packed int6 + fp16 scales + bf16 X read, fp32 Y written", flops=fl)
        Wh = gq.dequant(q.packed, q.scale_f16, 6, N, K, out_dtype=torch.bfloat16)
        record(f"cuBLAS bf16 on pre-dequantized weight M{M} N{N} K{K}",
               timed(lambda: torch.matmul(X, Wh.t()), flush_between=True),
               2 * N * K + 2 * M * K + 2 * M * N, 2 * N * K, None,
               note="torch.matmul, bf16 W_hat read, bf16 Y; not counting the dequant pass", flops=fl)
        del q, X, Y, Wh
    # the same GEMM with the fake-quant in the weight load (training forward),
    # decode-sized batch over bf16 weights with training-mode row scales, and
    # the 11-layer d528 model's two input widths
    for M, N, K in ((16, 16384, 16384), (64, 1584, 528), (64, 528, 1584)):
        Wb = synth.draw_bandwidth_matrix(N, K, 0, device=device).to(torch.bfloat16)
        (cl,) = gq.row_clip_select([gq.Request(Wb, 6, 1.0)])
        X = (torch.randn(M, K, device=device) * 0.5).to(torch.bfloat16)
        Y = torch.empty(M, N, device=device)
        wbytes = 2 * N * K + 4 * N
        record(f"gemm fake-quant-on-load int6 from bf16 M{M} N{N} K{K}",
               timed(lambda: gq.gemm_fakequant(X, Wb, cl.clip, 6, y=Y), flush_between=True),
               wbytes + 2 * M * K + 4 * M * N, wbytes, 1,
               note="bf16 weights + fp32 clips + bf16 X read, fp32 Y written", flops=2 * M * N * K)
        del Wb, cl, X, Y

    # model-shaped batched workloads (L2-resident: flushed between reps)
    def oracle_time(items, export):
        """Single-threaded CPU oracle on the same tensors: (seconds, bytes)."""
        import oracle
        t0 = time.perf_counter()
        nb = 0
        for w, qbits, p, per_tensor in items:
            if qbits == 16:
                oracle.passthrough_f16(w)
            else:
                r = oracle.quantize(w, qbits, p, per_tensor=per_tensor, export=export)
                assert r.status == 0
            nb += w.size * w.itemsize
        return time.perf_counter() - t0, nb

    def batch(specs_arrays, export=True, per_tensor_override=None, name="", note="", ste=False):
        descs, keep, host_items = [], [], []
        alg = inb = 0
        for spec, w in specs_arrays:
            W = torch.from_numpy(w).to(device) if isinstance(w, np.ndarray) else w
            if W.dtype == torch.int16:
                W = W.view(torch.bfloat16)
            if W.dim() == 1:
                W = W.view(1, -1)
            rows, cols = W.shape
            esz = W.element_size()
            keep.append(W)
            w_host = w if isinstance(w, np.ndarray) else W.cpu().numpy()
            if w_host.dtype == np.int16:
                w_host = w_host.view(np.uint16)
            w_host = w_host.reshape(rows, cols)
            if spec.qbits == 16:
                out16 = torch.empty((rows, cols), dtype=torch.float16, device=device)
                keep.append(out16)
                descs.append(gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=16, gran=0,
                                         reserved=0, rows=rows, cols=cols, ld=cols, p=1.0, dq=0, codes=0,
                                         packed=out16.data_ptr(), scale_f16=0, scale_f32=0, clip=0))
                alg += rows * cols * (esz + 2)
                inb += rows * cols * esz
                host_items.append((w_host, 16, 1.0, False))
                continue
            per_tensor = spec.per_tensor if per_tensor_override is None else per_tensor_override
            prb = gq.gq_packed_row_bytes(cols, spec.qbits)
            dq = torch.empty_like(W)
            packed = torch.empty((rows, prb), dtype=torch.uint8, device=device) if export else None
            h = torch.empty(rows, dtype=torch.float16, device=device) if export else None
            keep += [dq, packed, h]
            descs.append(gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=spec.qbits,
                                     gran=1 if per_tensor else 0, reserved=0, rows=rows, cols=cols, ld=cols,
                                     p=spec.p, dq=dq.data_ptr(), codes=0,
                                     packed=packed.data_ptr() if export else 0,
                                     scale_f16=h.data_ptr() if export else 0, scale_f32=0, clip=0))
            alg += rows * cols * 2 * esz + (rows * prb + 2 * rows if export else 0)
            inb += rows * cols * esz
            host_items.append((w_host, spec.qbits, spec.p, per_tensor))
        arr = gq._arr(descs)
        nbytes = gq.gq_workspace_size(descs)
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        keep.append(ws)
        if export:
            fn = lambda: gq.LIB.gq_export_pack(arr, len(descs), ws.data_ptr(), ws.numel(), None, None)  # noqa: E731
        else:
            fn = lambda: gq.LIB.gq_fakequant_fwd(arr, len(descs), 0, ws.data_ptr(), ws.numel(), None, None)  # noqa: E731
        launches = None
        if ste:
            # the STE backward of the same step: one flat gradient buffer for
            # all weights (bf16 N(0, 1e-3^2)), copied to the weight gradient
            numel = sum(int(np.prod(d.rows * d.cols)) for d in descs)
            g_flat = (torch.randn(numel, device=device) * 1e-3).to(torch.bfloat16)
            gw_flat = torch.empty_like(g_flat)
            keep += [g_flat, gw_flat]
            fwd = fn

            def fn():
                fwd()
                gq.gq_ste_bwd(g_flat.data_ptr(), gw_flat.data_ptr(), 1, numel, 0)
            alg += 4 * numel
        t = timed(fn, flush_between=True)
        record(name, t, alg, inb, launches, note)
        cs, cb = oracle_time(host_items, export)
        if ste:
            import oracle
            g_host = g_flat.cpu().view(torch.int16).numpy().view(np.uint16)
            t0 = time.perf_counter()
            oracle.ste_bwd(g_host)
            cs += time.perf_counter() - t0
        out[name]["cpu_oracle"] = {"gbs": round(cb / cs / 1e9, 4), "seconds": round(cs, 3), "cores": 1,
                                   "kind": "oracle", "sample": "the whole batch, single-threaded C oracle"}

    # the single 512x1536 fp32 matrix: int6 absmax export (w_hat, codes,
    # packed, binary16 scales) + STE copy of a same-shape gradient
    w0, g0 = synth.draw_single_matrix()
    W0, G0 = torch.from_numpy(w0).to(device), torch.from_numpy(g0).to(device)
    dq0, cd0 = torch.empty_like(W0), torch.empty(W0.shape, dtype=torch.int8, device=device)
    pk0 = torch.empty(512, gq.gq_packed_row_bytes(1536, 6), dtype=torch.uint8, device=device)
    h0, gw0 = torch.empty(512, dtype=torch.float16, device=device), torch.empty_like(G0)
    arr0c = gq._arr([gq.GQTensor(w=W0.data_ptr(), dtype=0, qbits=6, gran=0, reserved=0, rows=512, cols=1536,
                                 ld=1536, p=1.0, dq=dq0.data_ptr(), codes=cd0.data_ptr(), packed=pk0.data_ptr(),
                                 scale_f16=h0.data_ptr(), scale_f32=0, clip=0)])

    def c0():
        gq.LIB.gq_export_pack(arr0c, 1, None, 0, None, None)
        gq.gq_ste_bwd(G0.data_ptr(), gw0.data_ptr(), 0, 512 * 1536, 0)
    n0 = 512 * 1536
    record("single 512x1536 export int6 absmax + STE", timed(c0, flush_between=True),
           n0 * (4 + 4 + 1 + 0.75) + 2 * 512 + 8 * n0, 4 * n0 + 4 * n0, 2,
           note="cold L2; w_hat, codes, packed, fp16 scales + STE copy")
    import oracle
    t0 = time.perf_counter()
    oracle.quantize(w0, 6, 1.0, export=True)
    oracle.ste_bwd(g0)
    cs0 = time.perf_counter() - t0
    out["single 512x1536 export int6 absmax + STE"]["cpu_oracle"] = {
        "gbs": round(8 * n0 / cs0 / 1e9, 4), "seconds": round(cs0, 3), "cores": 1, "kind": "oracle",
        "sample": "the whole matrix and gradient, single-threaded C oracle"}
    del W0, G0, dq0, cd0, pk0, h0, gw0

    ws9 = synth.draw_gpt9()
    batch([(s, ws9[s.name]) for s in synth.gpt9_specs()], name="gpt9 export batched (55 matrices + 27 fp16)",
          note="cold L2; one gq_export_pack call")
    ws12 = synth.draw_gpt12()
    specs12 = synth.gpt12_mixed_specs()
    batch([(s, ws12[s.name]) for s in specs12], name="gpt12 mixed export per-row batched",
          note="cold L2; int8 emb/head/bigram + int6 p=.999")
    blocks = [s for s in specs12 if s.qbits == 6]
    batch([(s, ws12[s.name]) for s in blocks], per_tensor_override=True,
          name="gpt12 int6 per-tensor p=.999 batched", note="cold L2; 3 select passes + quantize pass")
    wsu = synth.draw_unified11()
    batch([(s, wsu[s.name].view(np.int16)) for s in synth.unified11_train().specs], export=False,
          name="unified11 bf16 train step: fake-quant batched + STE", ste=True,
          note="cold L2; one iteration: w_hat (fp32 scales) of the 44 weights + STE copy of their gradients")
    # GPTQ-lite export of the 11-layer d528 model: 44 bf16 weights, each
    # against the binary64 Hessian of 2048 synthetic input rows of its own
    gptq_rows(gq, device, out, record)
    torch.cuda.synchronize()
    return out


FP64_FMA_PER_SM_CLK = 64       # B200: 64 binary64 FMA per SM per clock (CUDA cores)


def fp64_peak_tflops(sm_mhz=None):
    """Binary64 FMA peak derived from the SM count and clock: 148 SMs x 64 FMA
    x 2 flops x clock (the measured SM clock when given, else 1965 MHz)."""
    mhz = sm_mhz or 1965.0
    return 148 * FP64_FMA_PER_SM_CLK * 2 * mhz * 1e6 / 1e12


def gptq_rows(gq, device, out, record):
    specs = synth.unified11_train().specs
    wsu = synth.draw_unified11()
    rng = np.random.default_rng(21)
    items = []
    for s in specs:
        W = torch.from_numpy(wsu[s.name].view(np.int16).copy()).to(device).view(torch.bfloat16)
        x = synth.gptq_calibration(rng, 2048, s.shape[1])
        items.append((s, W, x, torch.from_numpy(x).to(device)))
    Hs = [gq.gptq_hessian(X) for (_, _, _, X) in items]
    reqs = [gq.Request(W, 6, 1.0, want_dq=False) for (_, W, _, _) in items]
    # binary64 flops: the recurrence (rows * cols^2) and the Cholesky (cols^3 / 3)
    fl = sum(s.shape[0] * s.shape[1] ** 2 + s.shape[1] ** 3 / 3.0 for (s, _, _, _) in items)
    fl_h = sum(2 * 2048 * s.shape[1] ** 2 / 2 for (s, _, _, _) in items)

    def run_all():
        gq.gptq_quantize_batch(reqs, Hs, check_status=False)

    def hess_all():
        for (_, _, _, X), H in zip(items, Hs):
            gq.gptq_hessian(X, H)

    for name, fn, flops, note in (
            ("gptq unified11 export (44 weights, int6 per row)", run_all, fl,
             "one gq_gptq_quantize_batch call: binary64 recurrence + Cholesky, Hessians given; "
             "packed int6 + fp16 scales"),
            ("gptq unified11 Hessians (2048 input rows each)", hess_all, fl_h, "H = 2 X^T X in binary64")):
        t = statistics.median(_time_reps(fn, 5))
        tf = flops / t / 1e12
        out[name] = {"ms": round(t * 1e3, 3), "fp64_tflops": round(tf, 2),
                     "alu_frac": round(tf / fp64_peak_tflops(), 3), "bound": "alu (binary64 FMA)",
                     "peak_tflops": round(fp64_peak_tflops(), 1), "peak_source": "derived: 148 SM x 64 FMA x 2 x 1965 MHz",
                     "note": note}
    # CPU oracle on the first layer's four weights
    from oracle import gptq as OG
    t0 = time.perf_counter()
    for (s, W, x, _) in items[:4]:
        OG.gptq(wsu[s.name], OG.hessian(x), 6, 1.0)
    cs = time.perf_counter() - t0
    fl4 = sum(s.shape[0] * s.shape[1] ** 2 + s.shape[1] ** 3 / 3.0 for (s, _, _, _) in items[:4])
    out["gptq unified11 export (44 weights, int6 per row)"]["cpu_oracle"] = {
        "seconds": round(cs, 3), "fp64_gflops": round(fl4 / cs / 1e9, 3), "cores": 1, "kind": "oracle",
        "sample": "the first layer's four weights (numpy binary64, LAPACK inverse and Cholesky)"}


def _time_reps(fn, reps):
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) / 1e3)
    return ts


def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    from int6_int8_weight_b200 import gq
    peak, peak_kind = hbm_peak()

    only = args.only.replace("_", " ") if args.only else None
    wl = Workload(gq, device, seed=4 + rank, only=only, shrink=args.shrink)
    handle = torch.cuda.current_stream(device).cuda_stream
    ncalls = len(wl.calls)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * ncalls)] for _ in range(args.steps)]

    for _ in range(args.warmup):
        wl.step(handle)

    clocks = None
    for attempt in range(2):
        sampler = ClockSampler(physical_gpu_index(local))
        sampler.start()
        elapsed = time_region(lambda k: wl.step(handle, events[k]), args.steps, world, device)
        clocks = sampler.stop()
        if not clocks or not (set(clocks["reasons"]) & REJECT):
            break
    value_bps, t_max = job_throughput(wl.in_bytes * args.steps, elapsed, world, device)

    # per-launch durations of the fused kernel inside the timed region
    launch_s = 0.0
    per_call = [0.0] * ncalls
    for k in range(args.steps):
        for i in range(ncalls):
            dt = events[k][2 * i].elapsed_time(events[k][2 * i + 1]) / 1e3
            per_call[i] += dt
            launch_s += dt
    achieved = wl.alg_bytes * args.steps / launch_s / 1e9
    traffic_launch, tinfo = traffic_per_launch(kernel_source_hash(), wl.calls)
    traffic = None
    if traffic_launch is not None and not args.only and args.shrink == 1:
        traffic = int(traffic_launch)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4), "spec_gbs": SPEC_HBM_GBS,
                "traffic": traffic, "algorithmic_bytes_per_launch": int(wl.alg_bytes / ncalls),
                "kernel": "rowquant_tma_kernel (fused clip-select + quantize + dequant + pack), all "
                          f"{ncalls} launches of a step",
                "algorithmic_bytes_per_step": wl.alg_bytes,
                "per_launch": {wl.calls[i][3]: {"ms": round(per_call[i] / args.steps * 1e3, 4),
                                                "alg_gbs": round(wl.calls[i][2] * args.steps / per_call[i] / 1e9, 1)}
                               for i in range(ncalls)}}
    if tinfo:
        roofline["traffic_note"] = tinfo.get("note")

    # end to end through the public API with pinned host buffers
    e2e = None if args.no_e2e else measure_e2e(gq, wl, device, world, handle, max(2, min(args.steps, 5)))

    cpu = None
    rows_extra = None
    if world == 1 and rank == 0:
        if not args.skip_cpu:
            cpu = cpu_baseline_sample(wl, args.cpu_fraction)
        if not args.skip_rows:
            rows_extra = measure_rows(gq, device, peak)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value_bps / 1e9, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_max / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "shapes": [list(s) for s in synth.BANDWIDTH_SHAPES],
                       "dtypes": ["f32", "bf16"], "calls_per_step": ncalls,
                       "input_bytes_per_step": wl.in_bytes, "l2": "inputs larger than L2 (256 MiB-1 GiB each)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "hbm_frac_step": round(wl.alg_bytes * args.steps / t_max / 1e9 / peak, 4),
            "hbm_frac_step_of_spec": round(wl.alg_bytes * args.steps / t_max / 1e9 / SPEC_HBM_GBS, 4),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": ncalls * args.steps, "rows": rows_extra,
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        torch.distributed.destroy_process_group()


def measure_e2e(gq, wl, device, world, handle, steps):
    """Same metric with the inputs copied in from pinned host memory and the
    exported artifact (packed codes + binary16 scales) copied back, each step.

    Three streams overlap the work matrix by matrix: the host-to-device copy
    of matrix i+1 and the device-to-host copy of matrix i-1's artifact run
    while matrix i is quantized.  Events keep every buffer's reuse in order:
    a matrix is not overwritten before the previous step's calls on it have
    finished, and its outputs are not rewritten before they have been copied
    back."""
    host_in = [W.cpu().pin_memory() for W in wl.mats]
    host_out = [(p.cpu().pin_memory(), h.cpu().pin_memory()) for (_, p, h) in wl.outs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(p.numel() + h.numel() * 2 for p, h in host_out)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_cmp = torch.cuda.current_stream(device)
    nm = len(wl.mats)
    calls_of = [[] for _ in range(nm)]
    for ci in range(len(wl.calls)):
        calls_of[ci // 2].append(ci)          # two calls (int6, int8) per matrix, in order
    ev = lambda: torch.cuda.Event()  # noqa: E731
    done_cmp = [None] * nm                    # last compute on matrix i (its input is free)
    done_out = [None] * nm                    # last copy-back of matrix i's outputs

    def one(_k):
        L = gq.LIB
        for i in range(nm):
            with torch.cuda.stream(s_in):
                if done_cmp[i] is not None:
                    s_in.wait_event(done_cmp[i])
                wl.mats[i].copy_(host_in[i], non_blocking=True)
                e_in = ev()
                e_in.record(s_in)
            s_cmp.wait_event(e_in)
            if done_out[i] is not None:
                s_cmp.wait_event(done_out[i])
            for ci in calls_of[i]:
                st = L.gq_export_pack(wl.calls[ci][0], 1, None, 0, None, handle)
                if st != 0:
                    raise RuntimeError(f"gq_export_pack failed: {st}")
            done_cmp[i] = ev()
            done_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_cmp[i])
                for ci in calls_of[i]:
                    (po, ho), (_, p, h) = host_out[ci], wl.outs[ci]
                    po.copy_(p, non_blocking=True)
                    ho.copy_(h, non_blocking=True)
                done_out[i] = ev()
                done_out[i].record(s_out)

    def joined(k):
        one(k)
        # the step ends when its last copy-back has landed
        for e in done_out:
            s_cmp.wait_event(e)

    joined(0)
    elapsed = time_region(joined, steps, world, device)
    v, _ = job_throughput(wl.in_bytes * steps, elapsed, world, device)
    del host_in, host_out
    return {"value": round(v / 1e9, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": ("pinned host weights -> device, libgq export calls, packed codes + fp16 scales -> "
                     "host; copies in, quantization and copies out overlap on three streams, matrix by "
                     "matrix")}


# ----------------------------------------------------------- CPU oracle --

def oracle_sample(mats_host, fraction):
    """Run the oracle on the first rows of each matrix (both calls of the step).
    Returns (input bytes processed, seconds)."""
    import oracle
    total_bytes, t0 = 0, time.perf_counter()
    for w in mats_host:
        for qbits, p in ((6, 0.9999), (8, 1.0)):
            r = oracle.quantize(w, qbits, p, export=True)
            assert r.status == 0
            total_bytes += w.shape[0] * w.shape[1] * w.itemsize
    return total_bytes, time.perf_counter() - t0


def sample_rows_host(mats, fraction):
    out = []
    for W in mats:
        n = max(1, int(W.shape[0] * fraction))
        t = W[:n].contiguous().cpu()
        if t.dtype == torch.bfloat16:
            out.append(t.view(torch.int16).numpy().view(np.uint16))
        else:
            out.append(t.numpy())
    return out


def cpu_baseline_sample(wl, fraction):
    mats = sample_rows_host(wl.mats, fraction)
    nbytes, secs = oracle_sample(mats, fraction)
    return {"value": round(nbytes / secs / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "seconds": round(secs, 2),
            "sample": f"first {fraction:.4g} of the rows of each of the six matrices, both calls "
                      f"(int6 p=0.9999 export and int8 absmax), single-threaded C oracle"}


def run_reference(args, world, rank, local):
    """The oracle as the reference arm: same metric and config, each step a
    bounded sample of the workload (the first rows of every matrix), sized so
    that warm-up plus all steps take about a minute of host time."""
    if rank != 0:
        return
    import oracle  # noqa: F401  (built on first use)
    device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    budget_s = 60.0
    # calibrate: one row of each matrix
    mats = [synth.draw_bandwidth_matrix(min(r, 64), c, i, device=device, seed=4)
            for i, (r, c) in enumerate(synth.BANDWIDTH_SHAPES)]
    mats += [W.to(torch.bfloat16) for W in list(mats)]
    host_full = sample_rows_host(mats, 1.0)
    probe = [h[:1] for h in host_full]
    b, s = oracle_sample(probe, 1.0)
    per_row_set = max(s, 1e-4)                    # seconds for one row of every matrix
    rows_per_step = int(budget_s / (args.steps + args.warmup) / per_row_set)
    rows_per_step = max(1, min(64, rows_per_step))
    host = [h[:rows_per_step] for h in host_full]
    for _ in range(args.warmup):
        oracle_sample([h[:1] for h in host], 1.0)
    tot_b, tot_s = 0, 0.0
    for _ in range(args.steps):
        b, s = oracle_sample(host, 1.0)
        tot_b += b
        tot_s += s
    v = tot_b / tot_s / 1e9
    sample = (f"first {rows_per_step} rows of each of the six matrices per step, both calls "
              "(int6 p=0.9999 export, int8 absmax), single-threaded C oracle")
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_s / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "shapes": [list(s) for s in synth.BANDWIDTH_SHAPES],
                       "dtypes": ["f32", "bf16"], "l2": "host run", "parallelism": "single CPU thread"},
            "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gemm(args):
    """The consuming GEMM alone on one shape (``--gemm M,N,K,QBITS`` for the
    dequant from packed codes, ``--gemm M,N,K,QBITS,bf16|f32`` for the
    fake-quant from weights with training-mode scales): synthetic weight,
    random bf16 X, ``warmup`` then ``steps`` back-to-back calls timed with
    CUDA events.  An entry point for profiling; one JSON line of its own."""
    import torch
    from int6_int8_weight_b200 import gq
    parts = args.gemm.split(",")
    M, N, K, qbits = (int(v) for v in parts[:4])
    wmode = parts[4] if len(parts) > 4 else None
    device = torch.device("cuda")
    W = synth.draw_bandwidth_matrix(N, K, 0, device=device)
    X = (torch.randn(M, K, device=device) * 0.5).to(torch.bfloat16)
    Y = torch.empty(M, N, device=device)
    if wmode is None:
        (q,) = gq.export_pack([gq.Request(W, qbits, 0.9999, want_dq=False)], check_status=False)
        del W
        fn = lambda: gq.gemm_dequant(X, q.packed, q.scale_f16, qbits, y=Y)  # noqa: E731
        wbytes = q.packed.numel() + 2 * N
        name = f"M{M} N{N} K{K} int{qbits}"
    else:
        Wm = W.to(torch.bfloat16) if wmode == "bf16" else W
        (c,) = gq.row_clip_select([gq.Request(Wm, qbits, 1.0)])
        fn = lambda: gq.gemm_fakequant(X, Wm, c.clip, qbits, y=Y)  # noqa: E731
        wbytes = Wm.numel() * Wm.element_size() + 4 * N
        name = f"M{M} N{N} K{K} fake-quant int{qbits} from {wmode}"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / max(args.steps, 1)
    print(json.dumps({"gemm": name, "us_per_call": round(us, 2),
                      "tflops": round(2 * M * N * K / us / 1e6, 1),
                      "alg_gbs": round((wbytes + 2 * M * K + 4 * M * N) / us / 1e3, 1)}), flush=True)


def run_batch(args):
    """One model-shaped batched call alone (``--batch NAME``), for profiling
    a single launch: ``gpt9`` (export of the 9-layer model), ``gpt12`` (mixed
    per-row export of the 12-layer model), ``gpt12pt`` (per-tensor export of
    its 72 block matrices) or ``unified11`` (bf16 training fake-quant of the
    11-layer d528 model's 44 weights).  ``warmup`` then ``steps`` calls
    through the C ABI, timed with CUDA events; one JSON line of its own."""
    import torch
    from int6_int8_weight_b200 import gq
    device = torch.device("cuda")
    if args.batch == "gpt9":
        ws = synth.draw_gpt9()
        items, export = [(s, ws[s.name], False) for s in synth.gpt9_specs()], True
    elif args.batch == "gpt12":
        ws = synth.draw_gpt12()
        items, export = [(s, ws[s.name], s.per_tensor) for s in synth.gpt12_mixed_specs()], True
    elif args.batch == "gpt12pt":
        ws = synth.draw_gpt12()
        items, export = [(s, ws[s.name], True) for s in synth.gpt12_mixed_specs() if s.qbits == 6], True
    elif args.batch == "unified11":
        ws = synth.draw_unified11()
        items, export = [(s, ws[s.name].view(np.int16), False) for s in synth.unified11_train().specs], False
    else:
        raise SystemExit(f"unknown batch {args.batch!r}")
    descs, keep = [], []
    for spec, w, per_tensor in items:
        W = torch.from_numpy(np.ascontiguousarray(w)).to(device)
        if W.dtype == torch.int16:
            W = W.view(torch.bfloat16)
        if W.dim() == 1:
            W = W.view(1, -1)
        rows, cols = W.shape
        keep.append(W)
        if spec.qbits == 16:
            o = torch.empty((rows, cols), dtype=torch.float16, device=device)
            keep.append(o)
            descs.append(gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=16, gran=0, reserved=0,
                                     rows=rows, cols=cols, ld=cols, p=1.0, dq=0, codes=0, packed=o.data_ptr(),
                                     scale_f16=0, scale_f32=0, clip=0))
            continue
        dq = torch.empty_like(W)
        prb = gq.gq_packed_row_bytes(cols, spec.qbits)
        pk = torch.empty((rows, prb), dtype=torch.uint8, device=device) if export else None
        h = torch.empty(rows, dtype=torch.float16, device=device) if export else None
        keep += [dq, pk, h]
        descs.append(gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=spec.qbits,
                                 gran=1 if per_tensor else 0, reserved=0, rows=rows, cols=cols, ld=cols,
                                 p=spec.p, dq=dq.data_ptr(), codes=0, packed=pk.data_ptr() if export else 0,
                                 scale_f16=h.data_ptr() if export else 0, scale_f32=0, clip=0))
    arr = gq._arr(descs)
    nb = gq.gq_workspace_size(descs)
    wsb = torch.empty(max(nb, 256), dtype=torch.uint8, device=device)
    if export:
        fn = lambda: gq.LIB.gq_export_pack(arr, len(descs), wsb.data_ptr(), wsb.numel(), None, None)  # noqa: E731
    else:
        fn = lambda: gq.LIB.gq_fakequant_fwd(arr, len(descs), 0, wsb.data_ptr(), wsb.numel(), None, None)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"batch": args.batch, "tensors": len(descs),
                      "us_per_call": round(a.elapsed_time(b) * 1e3 / max(args.steps, 1), 2)}), flush=True)


def run_awq(args):
    """The AWQ column-scaled int6 export alone (``--awq ROWS,COLS``): a bf16
    synthetic weight, column scales from synthetic activation statistics,
    p = 0.9999; ``warmup`` then ``steps`` calls timed with CUDA events.  An
    entry point for profiling that kernel; it prints one JSON line of its own."""
    import torch
    from int6_int8_weight_b200 import gq
    rows, cols = (int(v) for v in args.awq.split(","))
    device = torch.device("cuda")
    Wb = synth.draw_bandwidth_matrix(rows, cols, 0, device=device).to(torch.bfloat16)
    t = torch.from_numpy(synth.awq_col_scales(np.random.default_rng(3), cols)).to(device)
    dq = torch.empty_like(Wb)
    pk = torch.empty(rows, gq.gq_packed_row_bytes(cols, 6), dtype=torch.uint8, device=device)
    h16 = torch.empty(rows, dtype=torch.float16, device=device)
    d = gq.GQTensor(w=Wb.data_ptr(), dtype=1, qbits=6, gran=0, reserved=0, rows=rows, cols=cols, ld=cols,
                    p=0.9999, dq=dq.data_ptr(), codes=0, packed=pk.data_ptr(), scale_f16=h16.data_ptr(),
                    scale_f32=0, clip=0, col_scale=t.data_ptr())
    arr = gq._arr([d])
    for _ in range(args.warmup):
        gq.LIB.gq_export_pack(arr, 1, None, 0, None, None)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        gq.LIB.gq_export_pack(arr, 1, None, 0, None, None)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / max(args.steps, 1)
    alg = rows * cols * 4.75 + 2 * rows + 4 * cols
    print(json.dumps({"awq": f"bf16 {rows}x{cols} int6 p=0.9999", "ms_per_call": round(ms, 4),
                      "alg_gbs": round(alg / ms / 1e6, 1)}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-fraction", type=float, default=1.0 / 16)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-rows", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default=None,
                    help="restrict the step to calls whose name contains this text, "
                         "underscores for spaces, e.g. f32_16384x16384_int6")
    ap.add_argument("--gemm", default=None,
                    help="profile the dequant-on-load GEMM alone on M,N,K,QBITS (one JSON line of its own)")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide every bandwidth matrix's rows by this factor (smaller case for ncu "
                         "counter captures; its line is not a bench value)")
    ap.add_argument("--record-traffic", default=None, metavar="CSV",
                    help="write profiles/rowquant_traffic.json from the ncu CSV of a --shrink run")
    ap.add_argument("--awq", default=None,
                    help="profile the AWQ column-scaled bf16 int6 export alone on ROWS,COLS (one JSON line of its own)")
    ap.add_argument("--batch", default=None, choices=["gpt9", "gpt12", "gpt12pt", "unified11"],
                    help="profile one model-shaped batched call alone (one JSON line of its own)")
    args = ap.parse_args(argv)
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.shrink), indent=1))
        return
    if args.gemm:
        run_gemm(args)
        return
    if args.awq:
        run_awq(args)
        return
    if args.batch:
        run_batch(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank, local)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
