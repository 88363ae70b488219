"""GPU parity: libgq (through its C ABI) against the CPU oracle, bit for bit.

Every comparison is exact: int8 codes, packed bytes and binary16 scales
byte-for-byte, and binary32 / bf16 outputs bit-for-bit (tolerance 0 ulp: each
output is one correctly rounded IEEE operation on both sides).

Workloads: the single 512x1536 matrix, the 9-layer GPT export, the 11-layer
bf16 training fake-quant + STE over 100 iterations, the 12-layer mixed-bit
export, every row of the 16384^2 / 65536x4096 / 262144x512 bandwidth
matrices (fp32 and bf16, int6 and int8), and edge cases
(empty, ragged, strided, misaligned, ties, zeros, every selection path,
non-finite input, binary16 overflow).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import oracle_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int6_int8_weight_b200 import gq as mod
    return mod


# ---------------------------------------------------------------- helpers --

def to_dev(a: np.ndarray) -> torch.Tensor:
    """fp32 arrays -> float32; uint16 arrays (bf16 bits) -> bfloat16."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def to_host(t: torch.Tensor) -> np.ndarray:
    """Exact host copy: float32 as float32, bf16/fp16 as uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bits(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.float32:
        return a.view(np.uint32)
    return a


def assert_same(got: np.ndarray, want: np.ndarray, what: str):
    g, w = bits(got), bits(want)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    bad = np.nonzero(g != w)
    if bad[0].size:
        idx = tuple(b[0] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} mismatches, first at {idx}: "
                             f"got {g[idx]!r} want {w[idx]!r}")


def check_quantized(o, ref, what, export=True, per_tensor=False, want_codes=True):
    assert o.status == 0, (what, o.status)
    assert ref.status == oracle.OR_OK
    if o.dq is not None:
        assert_same(to_host(o.dq), ref.dq, what + " dq")
    if want_codes and o.codes is not None:
        assert_same(to_host(o.codes), ref.codes, what + " codes")
    if o.packed is not None:
        assert_same(to_host(o.packed), ref.packed, what + " packed")
    if o.scale_f16 is not None:
        assert_same(to_host(o.scale_f16), ref.scale_f16, what + " scale_f16")
    if o.scale_f32 is not None:
        assert_same(to_host(o.scale_f32), ref.scale_f32, what + " scale_f32")
    if o.clip is not None:
        assert_same(to_host(o.clip), ref.clip, what + " clip")


def full_request(gq, W, qbits, p, per_tensor=False):
    return gq.Request(W, qbits, p, per_tensor, want_dq=True, want_codes=True,
                      want_packed=True, want_scale_f16=True, want_scale_f32=True, want_clip=True)


def run_export_and_check(gq, w_np, qbits, p, per_tensor=False, what=""):
    W = to_dev(w_np)
    (o,) = gq.export_pack([full_request(gq, W, qbits, p, per_tensor)])
    ref = oracle.quantize(w_np, qbits, p, per_tensor=per_tensor, export=True)
    check_quantized(o, ref, what or f"export q{qbits} p{p} pt{per_tensor}")
    return o, ref


def run_train_and_check(gq, w_np, qbits, p, per_tensor=False, what=""):
    W = to_dev(w_np)
    r = gq.Request(W, qbits, p, per_tensor, want_dq=True, want_codes=True,
                   want_scale_f32=True, want_clip=True)
    (o,) = gq.fakequant([r], mode=gq.GQ_SCALE_F32)
    ref = oracle.quantize(w_np, qbits, p, per_tensor=per_tensor, export=False)
    check_quantized(o, ref, what or f"train q{qbits} p{p} pt{per_tensor}")
    return o, ref


# ------------------------------------------------------ the five workloads --

def test_single_matrix_export_train_ste(gq):
    w, g = synth.draw_single_matrix()
    o, ref = run_export_and_check(gq, w, 6, 1.0, what="512x1536 export")
    back = gq.dequant(o.packed, o.scale_f16, 6, *w.shape)
    assert_same(to_host(back), ref.dq, "dequant round trip")
    run_train_and_check(gq, w, 6, 1.0, what="512x1536 train")
    G = to_dev(g)
    assert_same(to_host(gq.ste_bwd(G)), oracle.ste_bwd(g), "ste copy")
    acc = to_dev(w.copy())
    gq.ste_bwd(G, acc)
    assert_same(to_host(acc), oracle.ste_bwd(g, w, accumulate=True), "ste accumulate")


def test_gpt9_batched_export(gq):
    ws = synth.draw_gpt9()
    specs = synth.gpt9_specs()
    reqs, refs = [], []
    for s in specs:
        w = ws[s.name]
        if s.qbits == 16:
            reqs.append(gq.Request(to_dev(w.reshape(1, -1)), 16, want_dq=False))
            refs.append(("fp16", oracle.passthrough_f16(w.reshape(1, -1))))
        else:
            reqs.append(gq.Request(to_dev(w), s.qbits, s.p, want_dq=True, want_codes=True,
                                   want_clip=True))
            refs.append(("q", oracle.quantize(w, s.qbits, s.p, export=True)))
    outs = gq.export_pack(reqs)       # one batched call
    assert len(outs) == 55 + 27
    for s, o, (kind, ref) in zip(specs, outs, refs):
        if kind == "fp16":
            assert_same(to_host(o.packed), ref, s.name)
        else:
            check_quantized(o, ref, s.name)


def test_unified11_bf16_training_steps(gq):
    """The 11-layer d528 bf16 training workload as specified: 100 iterations
    of the batched training-mode fake-quant (int6 absmax, binary32 scales)
    plus the STE backward of a fresh gradient, the weights drifting between
    iterations; every output of iterations 0, 1, 50 and 99 is compared with
    the oracle bit for bit."""
    ws = synth.draw_unified11()
    specs = synth.unified11_train().specs
    W = {s.name: to_dev(ws[s.name]) for s in specs}
    check_iters = {0, 1, 50, 99}
    oracle.default()
    for it in range(100):
        reqs = [gq.Request(W[s.name], 6, 1.0, want_dq=True, want_scale_f32=True) for s in specs]
        outs = gq.fakequant(reqs, mode=gq.GQ_SCALE_F32)
        grads, perts = {}, {}
        for s in specs:
            g, pert = synth.training_step_noise(tuple(s.shape), it, device=DEV)
            grads[s.name] = g.to(torch.bfloat16)
            perts[s.name] = pert
        gw = {s.name: gq.ste_bwd(grads[s.name]) for s in specs}
        if it in check_iters:
            w_np = [to_host(W[s.name]) for s in specs]
            refs = oracle_rows.quantize_many(w_np, 6, 1.0, export=False)
            for s, o, ref in zip(specs, outs, refs):
                assert o.status == 0 and ref.status == oracle.OR_OK
                assert_same(to_host(o.dq), ref.dq, f"iter {it} {s.name} dq")
                assert_same(to_host(o.scale_f32), ref.scale_f32, f"iter {it} {s.name} scale")
                g_np = to_host(grads[s.name])
                assert_same(to_host(gw[s.name]), oracle.ste_bwd(g_np), f"iter {it} {s.name} ste")
        # weights drift between steps (input generation, not the method)
        for s in specs:
            W[s.name] = (W[s.name].float() + perts[s.name]).to(torch.bfloat16)


def test_gpt12_mixed_export(gq):
    ws = synth.draw_gpt12()
    specs = synth.gpt12_mixed_specs()
    for per_tensor in (False, True):
        reqs, refs = [], []
        for s in specs:
            if per_tensor and s.qbits != 6:
                continue
            w = ws[s.name]
            reqs.append(gq.Request(to_dev(w), s.qbits, s.p, per_tensor, want_dq=True,
                                   want_codes=True, want_clip=True, want_scale_f32=True))
            refs.append((s.name, oracle.quantize(w, s.qbits, s.p, per_tensor=per_tensor, export=True)))
        outs = gq.export_pack(reqs)
        for o, (name, ref) in zip(outs, refs):
            check_quantized(o, ref, f"{name} per_tensor={per_tensor}")


@pytest.mark.parametrize("shape_idx", [0, 1, 2])
def test_bandwidth_matrices_full_parity(gq, shape_idx):
    """The bandwidth-stress workload at full size, every row of every call of
    the step compared with the oracle bit for bit: fp32 and bf16, int6 at
    p = 0.9999 (w_hat, packed, binary16 scales) and int8 absmax (w_hat, code
    bytes, binary16 scales), one call per matrix as the benchmark makes it."""
    rows, cols = synth.BANDWIDTH_SHAPES[shape_idx]
    W = synth.draw_bandwidth_matrix(rows, cols, shape_idx, device=DEV)
    oracle.default()      # built before the worker threads share it
    for dtype in (torch.float32, torch.bfloat16):
        Wd = W if dtype == torch.float32 else W.to(torch.bfloat16)
        w_host = to_host(Wd)
        for qbits, p in ((6, 0.9999), (8, 1.0)):
            (o,) = gq.export_pack([gq.Request(Wd, qbits, p, want_dq=True, want_codes=False)])
            assert o.status == 0
            got = {"dq": to_host(o.dq), "packed": to_host(o.packed), "scale_f16": to_host(o.scale_f16)}
            del o
            res = oracle_rows.compare_rows(w_host, got, qbits, p, export=True)
            assert all(v == 0 for v in res["mismatches"].values()), \
                (f"{rows}x{cols} {dtype} int{qbits}", res)
        del Wd, w_host
    # property at full size: every packed row decodes to the dq row
    (o,) = gq.export_pack([gq.Request(W, 6, 0.9999, want_dq=True)])
    back = gq.dequant(o.packed, o.scale_f16, 6, rows, cols)
    assert torch.equal(back.view(torch.int32), o.dq.view(torch.int32))


# -------------------------------------------------------------- edge cases --

EDGE_SHAPES = [(1, 1), (1, 7), (3, 5), (2, 17), (5, 33), (4, 131), (3, 1000), (2, 2049),
               (3, 4099), (2, 16384 + 3), (1, 70001), (37, 128), (300, 64)]


@pytest.mark.parametrize("rows,cols", EDGE_SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_shapes_all_paths(gq, rows, cols, dtype):
    rng = np.random.default_rng(rows * 1000 + cols)
    w = synth.random_matrix(rng, rows, cols, "mix")
    if dtype == "bf16":
        w = synth.to_bf16_bits(w).reshape(rows, cols)
    # p values covering m = 1, 2, 3..4, 5..8 and radix (m > 8) where cols allow
    ps = [1.0, 0.9999, 0.999, 0.99, 0.9, 0.5, 1e-6]
    for p in ps:
        for qbits in (6, 8):
            run_export_and_check(gq, w, qbits, p, what=f"{rows}x{cols} {dtype} q{qbits} p{p}")
    run_train_and_check(gq, w, 6, 0.97, what=f"{rows}x{cols} {dtype} train")
    run_export_and_check(gq, w, 6, 0.999, per_tensor=True, what=f"{rows}x{cols} per-tensor")
    run_train_and_check(gq, w, 8, 0.5, per_tensor=True, what=f"{rows}x{cols} per-tensor train")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1536, 512), (333, 1000), (700, 97)])
def test_per_tensor_large_flat(gq, dtype, rows, cols):
    """Per-tensor groups spanning many select items: the vector loads of the
    histogram passes (several unrolled trips per thread, then the remainder
    and a scalar tail) must count every element once."""
    rng = np.random.default_rng(rows + cols)
    w = synth.random_matrix(rng, rows, cols, "t3")
    if dtype == "bf16":
        w = synth.to_bf16_bits(w).reshape(rows, cols)
    for p in (0.999, 0.9, 0.5):
        run_export_and_check(gq, w, 6, p, per_tensor=True, what=f"{rows}x{cols} {dtype} per-tensor p{p}")


def _p_for_rank(n, m):
    """A p whose clip is the m-th largest of n keys, checked with the oracle's rule."""
    p = (n - m + 1) / n
    assert oracle.k_from_p(n, p) == n - m + 1
    return p


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", ["zeros", "constant", "three_values", "ties_at_rank", "t3"])
def test_per_tensor_select_ties_and_tails(gq, dtype, case):
    """Per-tensor groups with heavy ties (all-zero, all-equal, three values,
    ties at the selected rank) and sizes that end inside a 16-byte vector,
    at ranks from 1 to a few thousand: every select pass must count each
    element once and the tie-breaking must not matter."""
    rng = np.random.default_rng(len(case) * 17 + (dtype == "bf16"))
    chunk = 16384 if dtype == "f32" else 32768
    shapes = [(3, chunk // 3 + 33),            # just over 16 / 32 K elements, odd tail
              (chunk // 64 + 1, 64 + 3),       # ragged row length
              (5 * chunk // 512 + 1, 512)]     # several select blocks
    for rows, cols in shapes:
        n = rows * cols
        if case == "zeros":
            w = np.zeros((rows, cols), np.float32)
        elif case == "constant":
            w = np.full((rows, cols), -0.0125, np.float32)
        elif case == "three_values":
            w = rng.choice(np.array([0.0, 0.25, -0.5], np.float32), size=(rows, cols))
        elif case == "ties_at_rank":
            w = (rng.integers(-3, 4, size=(rows, cols)) * 0.125).astype(np.float32)
        else:
            w = synth.random_matrix(rng, rows, cols, "t3")
        if dtype == "bf16":
            w = synth.to_bf16_bits(w).reshape(rows, cols)
        limit = chunk // 4 + 1
        ranks = sorted({1, 2, min(n, 200), min(n, limit), min(n, limit + 1)})
        for m in ranks:
            run_export_and_check(gq, w, 6, _p_for_rank(n, m), per_tensor=True,
                                 what=f"{case} {dtype} {rows}x{cols} m={m}")


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 8, 9, 64, 1000])
@pytest.mark.parametrize("cols", [1536, 4096])
def test_every_selection_rank(gq, m, cols):
    """p chosen so that the clip is exactly the m-th largest |w| of each row."""
    rng = np.random.default_rng(m * 7 + cols)
    w = synth.random_matrix(rng, 12, cols, "t3")
    k = cols - m + 1
    p = (k - 0.5) / cols        # ceil(p * cols) == k
    assert oracle.k_from_p(cols, p) == k
    run_export_and_check(gq, w, 6, p, what=f"m={m} cols={cols}")


def test_ties_and_zero_rows(gq):
    rng = np.random.default_rng(3)
    w = synth.random_matrix(rng, 40, 300, "ties")
    w[3] = 0.0
    w[7, :150] = 0.0
    w[9] = -0.0
    w[11] = 0.125
    for p in (1.0, 0.9, 0.5, 0.01):
        run_export_and_check(gq, w, 6, p, what=f"ties p{p}")
        run_train_and_check(gq, w, 8, p, what=f"ties train p{p}")


def test_tiny_values_binary16_subnormal_scales(gq):
    rng = np.random.default_rng(4)
    w = synth.random_matrix(rng, 64, 96, "tiny")
    w[0] *= 1e-3                  # scale underflows binary16 -> zero codes
    w[1] = w[1] * 1e-30           # binary32 subnormal values
    run_export_and_check(gq, w, 6, 1.0, what="tiny export")
    run_export_and_check(gq, w, 8, 0.9, what="tiny export int8")
    run_train_and_check(gq, w, 6, 1.0, what="tiny train")


def test_near_tie_quotients(gq):
    """Rows whose quotients sit on and next to every half-integer boundary."""
    rng = np.random.default_rng(5)
    rows = []
    for _ in range(16):
        c = np.float32(rng.uniform(0.01, 0.1))
        s = np.float32(c / np.float32(31))
        vals = [c]
        for h2 in range(-61, 62, 2):
            base = np.float32(np.float32(h2 / 2) * s)
            x = base
            for d in (-2, -1, 0, 1, 2):
                y = base
                for _ in range(abs(d)):
                    y = np.nextafter(y, np.float32(np.inf if d > 0 else -np.inf))
                if abs(y) <= c:
                    vals.append(y)
        vals = np.array(vals[:300], np.float32)
        rows.append(np.pad(vals, (0, 300 - vals.size)))
    w = np.stack(rows).astype(np.float32)
    run_train_and_check(gq, w, 6, 1.0, what="near ties train")
    run_export_and_check(gq, w, 6, 1.0, what="near ties export")


def test_strided_and_misaligned_inputs(gq):
    rng = np.random.default_rng(6)
    full = synth.random_matrix(rng, 50, 600, "t3")
    Wf = to_dev(full)
    for cols in (512, 511, 333):
        view = Wf[:, :cols]                     # ld = 600 > cols
        (o,) = gq.export_pack([full_request(gq, view, 6, 0.99)])
        ref = oracle.quantize(full, 6, 0.99, export=True, cols=cols)
        check_quantized(o, ref, f"strided cols={cols}")
    # base pointer offset by one element: no 16-byte alignment anywhere
    flat = to_dev(synth.random_matrix(rng, 1, 40 * 257 + 1, "normal").ravel())
    view = flat[1:].view(40, 257)
    (o,) = gq.export_pack([full_request(gq, view, 6, 0.98)])
    ref = oracle.quantize(to_host(view), 6, 0.98, export=True)
    check_quantized(o, ref, "misaligned base")
    bflat = to_dev(synth.random_matrix(rng, 1, 40 * 257 + 3, "normal").ravel()).to(torch.bfloat16)
    bview = bflat[3:].view(40, 257)
    (o,) = gq.export_pack([full_request(gq, bview, 8, 0.98)])
    ref = oracle.quantize(to_host(bview), 8, 0.98, export=True)
    check_quantized(o, ref, "misaligned bf16 base")


def test_empty_tensors_are_noops(gq):
    for shape in ((0, 16), (16, 0), (0, 0)):
        W = torch.zeros(shape, device=DEV)
        (o,) = gq.export_pack([gq.Request(W, 6, 0.9, want_dq=True)])
        assert o.status == 0
        (o,) = gq.export_pack([gq.Request(W, 6, 0.9, per_tensor=True)])
        assert o.status == 0
    assert gq.dequant(torch.zeros(0, dtype=torch.uint8, device=DEV),
                      torch.zeros(0, dtype=torch.float16, device=DEV), 6, 0, 8).numel() == 0
    gq.ste_bwd(torch.zeros(0, device=DEV))


def test_nonfinite_and_range_status(gq):
    w = np.full((6, 64), 0.01, np.float32)
    w[1, 5] = np.inf
    w[2, 9] = np.nan
    w[3, 0] = -np.inf
    (o,) = gq.export_pack([gq.Request(to_dev(w), 6, 1.0)])
    assert o.status & gq.GQ_STATUS_NONFINITE
    for p in (0.95, 0.5):                       # top-m and radix paths
        (o,) = gq.export_pack([gq.Request(to_dev(w), 6, p)])
        assert o.status & gq.GQ_STATUS_NONFINITE
        (o,) = gq.export_pack([gq.Request(to_dev(w), 6, p, per_tensor=True)])
        assert o.status & gq.GQ_STATUS_NONFINITE
    big = np.full((2, 8), 1.0, np.float32)
    big[1, 3] = 3.0e6                           # 3e6 / 31 > 65504
    (o,) = gq.export_pack([gq.Request(to_dev(big), 6, 1.0)])
    assert o.status & gq.GQ_STATUS_RANGE
    (o,) = gq.fakequant([gq.Request(to_dev(big), 6, 1.0)], mode=gq.GQ_SCALE_F32)
    assert o.status == 0
    ok = np.full((2, 8), 1.0, np.float32)
    (o,) = gq.export_pack([gq.Request(to_dev(ok), 6, 1.0)])
    assert o.status == 0                        # cleared by the call


def test_dequant_all_layouts(gq):
    rng = np.random.default_rng(8)
    for rows, cols in ((7, 13), (64, 512), (3, 4099)):
        w = synth.random_matrix(rng, rows, cols, "mix")
        for qbits in (6, 8):
            for per_tensor in (False, True):
                ref = oracle.quantize(w, qbits, 0.99, per_tensor=per_tensor, export=True)
                P = torch.from_numpy(ref.packed).to(DEV)
                H = torch.from_numpy(ref.scale_f16.view(np.int16)).to(DEV).view(torch.float16)
                out = gq.dequant(P, H, qbits, rows, cols, per_tensor)
                assert_same(to_host(out), ref.dq, f"dequant {rows}x{cols} q{qbits}")
                outb = gq.dequant(P, H, qbits, rows, cols, per_tensor, out_dtype=torch.bfloat16)
                want = oracle.dequant(ref.packed, ref.scale_f16, qbits, rows, cols, per_tensor, out_bf16=True)
                assert_same(to_host(outb), want, "dequant bf16")


def test_ste_tails_and_offsets(gq):
    rng = np.random.default_rng(9)
    for n in (1, 3, 8, 1001, 4096 + 5):
        for dt in ("f32", "bf16"):
            g = synth.random_matrix(rng, 1, n + 1, "normal").ravel()
            a = synth.random_matrix(rng, 1, n + 1, "normal").ravel()
            if dt == "bf16":
                g, a = synth.to_bf16_bits(g), synth.to_bf16_bits(a)
            G, A = to_dev(g), to_dev(a)
            for off in (0, 1):
                got = gq.ste_bwd(G[off:off + n].contiguous() if off == 0 else G[off:off + n])
                assert_same(to_host(got), oracle.ste_bwd(g[off:off + n]), f"ste copy {n} {dt}")
                acc = A[off:off + n].clone() if off == 0 else A.clone()[off:off + n]
                gq.ste_bwd(G[off:off + n], acc)
                assert_same(to_host(acc), oracle.ste_bwd(g[off:off + n], a[off:off + n], accumulate=True),
                            f"ste acc {n} {dt} off{off}")


def test_autograd_function(gq):
    rng = np.random.default_rng(10)
    w = synth.random_matrix(rng, 32, 96, "t3")
    W = to_dev(w).requires_grad_(True)
    out = gq.FakeQuantSTE.apply(W, 6, 1.0, False)
    ref = oracle.quantize(w, 6, 1.0, export=False)
    assert_same(to_host(out), ref.dq, "autograd forward")
    gout = torch.randn_like(out)
    out.backward(gout)
    assert torch.equal(W.grad.view(torch.int32), gout.view(torch.int32))


def test_export_state_dict_plan(gq):
    ws = synth.draw_gpt9()
    named = {k: to_dev(v) for k, v in ws.items()}
    named["step"] = torch.arange(70000, device=DEV)
    res = gq.export_state_dict(named)
    assert res["step"][0] == "raw"
    assert res["tok_emb.weight"][0] == "int8"
    assert res["blocks.0.attn_scale"][0] == "fp16"
    assert res["blocks.0.mlp.fc.weight"][0] == "int6"
    o = res["tok_emb.weight"][1]
    ref = oracle.quantize(ws["tok_emb.weight"], 8, 0.9999, export=True)
    assert_same(to_host(o.packed), ref.packed, "plan int8")
    o = res["blocks.2.attn.c_k.weight"][1]
    ref = oracle.quantize(ws["blocks.2.attn.c_k.weight"], 6, 0.9999, export=True)
    assert_same(to_host(o.packed), ref.packed, "plan int6")
    o = res["blocks.4.mlp_scale"][1]
    assert_same(to_host(o.packed).ravel(), oracle.passthrough_f16(ws["blocks.4.mlp_scale"]), "plan fp16")


def test_workspace_error_on_device(gq):
    W = torch.ones((4, 8), device=DEV)
    d = gq.GQTensor(w=W.data_ptr(), dtype=0, qbits=6, gran=1, reserved=0, rows=4, cols=8, ld=8,
                    p=1.0, dq=0, codes=0, packed=W.data_ptr(), scale_f16=W.data_ptr(),
                    scale_f32=0, clip=0)
    with pytest.raises(gq.GQError) as e:
        gq.gq_export_pack([d], ws=0, ws_bytes=0)
    assert e.value.status == 4


def test_pipelined_mixed_team_sizes_one_launch(gq):
    """One batch whose rows need every team size (1..16 warps) and both
    dtypes: the pipelined kernel switches team shape from tile to tile."""
    rng = np.random.default_rng(11)
    shapes = [(70, 512), (33, 1536), (21, 4096), (5, 16384), (300, 128), (40, 528), (17, 1584)]
    reqs, refs = [], []
    for j, (r, c) in enumerate(shapes):
        for dt in ("f32", "bf16"):
            w = synth.random_matrix(rng, r, c, ("t3", "mix", "normal")[j % 3])
            if dt == "bf16":
                w = synth.to_bf16_bits(w).reshape(r, c)
            p = (1.0, 0.9999, 0.99, 0.5)[(j + len(reqs)) % 4]
            qb = 6 if (j + len(reqs)) % 3 else 8
            reqs.append(full_request(gq, to_dev(w), qb, p))
            refs.append((f"{r}x{c} {dt} q{qb} p{p}", oracle.quantize(w, qb, p, export=True)))
    outs = gq.export_pack(reqs)
    for o, (name, ref) in zip(outs, refs):
        check_quantized(o, ref, "mixed " + name)


def test_pipelined_strided_bf16_and_two_stage_rows(gq):
    rng = np.random.default_rng(12)
    full = synth.to_bf16_bits(synth.random_matrix(rng, 24, 1040, "t3")).reshape(24, 1040)
    Wf = to_dev(full)
    (o,) = gq.export_pack([full_request(gq, Wf[:, :1024], 6, 0.999)])   # ld 1040, rows bulk-copied one by one
    ref = oracle.quantize(full, 6, 0.999, export=True, cols=1024)
    check_quantized(o, ref, "strided bf16")
    # 80 KB rows: two 80 KB stages instead of three 64 KB ones
    w = synth.random_matrix(rng, 9, 20000, "mix")
    run_export_and_check(gq, w, 6, 0.9999, what="two-stage 20000 cols")
    run_train_and_check(gq, w, 8, 0.3, what="two-stage 20000 cols radix")
    run_export_and_check(gq, w, 6, 0.999, per_tensor=True, what="two-stage per-tensor")


def test_pipelined_repeatability_stress(gq):
    """Many back-to-back launches over many tiles per block (both tile-teams
    busy, every stage reused many times): outputs must be identical launch
    after launch and match the oracle on sampled rows; status stays 0."""
    rng = np.random.default_rng(13)
    for (rows, cols, dt) in ((65536, 512, torch.bfloat16), (16384, 2048, torch.float32),
                             (2048, 16384, torch.float32)):
        W = synth.draw_bandwidth_matrix(rows, cols, 7, device=DEV).to(dt)
        first = None
        for it in range(12):
            (o,) = gq.export_pack([gq.Request(W, 6, 0.9999, want_dq=True)])
            assert o.status == 0
            if first is None:
                first = o
                idx = np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, 24)]))
                ti = torch.from_numpy(idx).to(DEV)
                ref = oracle.quantize(to_host(W.index_select(0, ti)), 6, 0.9999, export=True)
                assert_same(to_host(o.packed.index_select(0, ti)), ref.packed, f"{rows}x{cols} packed")
                assert_same(to_host(o.dq.index_select(0, ti)), ref.dq, f"{rows}x{cols} dq")
            else:
                assert torch.equal(o.packed, first.packed), (rows, cols, it)
                assert torch.equal(o.dq.view(torch.int16 if dt == torch.bfloat16 else torch.int32),
                                   first.dq.view(torch.int16 if dt == torch.bfloat16 else torch.int32)), (rows, cols, it)
                assert torch.equal(o.scale_f16.view(torch.int16), first.scale_f16.view(torch.int16))
