"""Pins of the CPU oracle against facts that do not come from the oracle itself.

* hand-worked examples (tests/golden/*.txt, each with its derivation),
* brute force with exact rational arithmetic on tiny inputs (tests/exact.py),
* library routines for the special cases that reduce to them
  (torch.kthvalue, torch CPU division + round-half-even, numpy float16,
  torch bfloat16),
* invariants (|q| <= qmax, clip maps to +-qmax, error bound, pack round trip
  over every code quadruple, STE identity, dequant == export w_hat),
* snapshot averaging: the first snapshot is copied, and the mean of two
  snapshots, a mean step with weight 1/4 and an EMA step with decay 1/2
  equal the exact rational results on dyadic inputs; decay 0 / 1 keep the
  snapshot / the average; a long EMA of a constant follows 1 - d^k,
* AWQ column scaling: every element equals the exact rational product rounded
  once to binary32 (and to bf16 for bf16 weights); t = 1 and a uniform power
  of two leave the codes unchanged.

The ``orc`` fixture is parametrised so that ``test_oracle_mutants.py`` can run
the same checks against oracle copies with a planted mistake.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import plan
import synth
from tests import exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


# ------------------------------------------------------------ golden files --

def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            d[key] = vals
    return d


WORKED = ["worked_int6_absmax.txt", "worked_int6_percentile.txt",
          "worked_int8_absmax.txt", "worked_int6_f16_subnormal_scale.txt",
          "worked_int6_clamp.txt"]


def check_worked_example(orc, name):
    g = _read_golden(name)
    scale = float(g["w_scaled_by"][0])
    w = (np.array([float(v) for v in g["w"]]) / scale).astype(np.float32)[None]
    qbits = int(g["qbits"][0])
    r = orc.quantize(w, qbits, float(g["p"][0]), export=bool(int(g["export"][0])))
    assert r.status == oracle.OR_OK
    assert r.clip[0] == np.float32(float(g["clip_scaled"][0]) / scale)
    assert int(r.scale_f16[0]) == int(g["scale_f16"][0], 16)
    assert r.codes[0].tolist() == [int(v) for v in g["codes"]]
    want_dq = (np.array([float(v) for v in g["dq_scaled"]]) / scale).astype(np.float32)
    assert np.array_equal(r.dq[0], want_dq)
    if "dq_signbit" in g:
        assert np.signbit(r.dq[0]).astype(int).tolist() == [int(v) for v in g["dq_signbit"]]
    if "packed" in g:
        assert r.packed[0].tolist() == [int(v, 16) for v in g["packed"]]


@pytest.mark.parametrize("name", WORKED)
def test_worked_examples(orc, name):
    check_worked_example(orc, name)


def check_k_from_p(orc):
    g = []
    with open(os.path.join(GOLDEN, "k_from_p.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                n, p, k = line.split()
                g.append((int(n), float(p), int(k)))
    for n, p, k in g:
        assert orc.k_from_p(n, p) == k, (n, p)


def test_k_from_p_golden(orc):
    check_k_from_p(orc)


def test_k_from_p_matches_exact_ceiling(orc):
    """Away from integers, ceil of the double product equals the exact ceiling."""
    rng = np.random.default_rng(11)
    for _ in range(2000):
        n = int(rng.integers(1, 1 << 22))
        p = float(rng.uniform(1e-6, 1.0))
        exact_prod = Fraction(p) * n
        if abs(exact_prod - round(exact_prod)) < Fraction(1, 1 << 20):
            continue
        want = min(n, max(1, math.ceil(exact_prod)))
        assert orc.k_from_p(n, p) == want


# ------------------------------------------------ brute force, exact maths --

def check_brute_force(orc, trials=300, seed=5):
    rng = np.random.default_rng(seed)
    for trial in range(trials):
        rows = int(rng.integers(1, 5))
        cols = int(rng.integers(1, 9))
        kind = ["normal", "t3", "mix", "ties", "tiny"][trial % 5]
        w = synth.random_matrix(rng, rows, cols, kind)
        if trial % 7 == 3:
            w[0, : cols // 2] = 0.0           # partly zero rows
        if trial % 11 == 5:
            w[:] = 0.0                         # all-zero group
        qbits = 6 if trial % 3 else 8
        p = 1.0 if trial % 5 == 0 else float(rng.uniform(0.05, 1.0))
        export = bool(trial % 2)
        per_tensor = trial % 6 == 1
        r = orc.quantize(w, qbits, p, per_tensor=per_tensor, export=export)
        assert r.status == oracle.OR_OK
        groups = [w.ravel()] if per_tensor else list(w)
        for gi, gw in enumerate(groups):
            k = min(len(gw), max(1, math.ceil(p * len(gw))))
            ref = exact.quantize_group_exact([float(x) for x in gw], qbits, k, export)
            assert Fraction(float(r.clip[gi])) == ref["clip"], (trial, gi)
            assert Fraction(float(r.scale_f32[gi])) == ref["s"], (trial, gi)
            if export:
                assert Fraction(float(orc.f16_bits_to_f32(r.scale_f16[gi:gi + 1])[0])) == ref["h"]
            got_q = (r.codes.ravel() if per_tensor else r.codes[gi]).tolist()
            assert got_q == ref["q"], (trial, gi)
            got_dq = r.dq.ravel() if per_tensor else r.dq[gi]
            assert [Fraction(float(x)) for x in got_dq] == ref["dq"], (trial, gi)
            # q == 0 gives +0.0
            for q, x in zip(got_q, got_dq):
                if q == 0:
                    assert not np.signbit(x)


def test_brute_force_exact(orc):
    check_brute_force(orc)


def test_brute_force_bf16_exact(orc):
    """bf16 input: widened exactly, computed in fp32, w_hat rounded to bf16."""
    rng = np.random.default_rng(6)
    for trial in range(120):
        cols = int(rng.integers(1, 9))
        wf = synth.random_matrix(rng, 1, cols, ["normal", "mix", "ties"][trial % 3])
        wb = synth.to_bf16_bits(wf).reshape(1, cols)
        vals = synth.bf16_bits_to_f32(wb).ravel()
        p = float(rng.uniform(0.1, 1.0))
        export = bool(trial % 2)
        r = orc.quantize(wb, 6, p, export=export)
        k = min(cols, max(1, math.ceil(p * cols)))
        ref = exact.quantize_group_exact([float(x) for x in vals], 6, k, export)
        assert r.codes[0].tolist() == ref["q"]
        got = synth.bf16_bits_to_f32(r.dq[0])
        want = [exact.rnbf16(x) for x in ref["dq"]]
        assert [Fraction(float(x)) for x in got] == want


def check_near_ties(orc, n_scales=12, seed=16):
    """Quotients on, and one or two ulps either side of, every half-integer
    boundary: the codes must follow the correctly rounded binary32 division
    (exact rational reference), not an approximation of it."""
    rng = np.random.default_rng(seed)
    for si in range(n_scales):
        qbits, qmax = ((6, 31), (8, 127))[si % 2]
        export = bool((si // 2) % 2)
        c = np.float32(rng.uniform(0.01, 0.1))
        s32 = Fraction(exact.rn32(Fraction(float(c)) / qmax))
        s = exact.rn16(s32) if export else s32
        vals = [float(c)]
        for h2 in range(-2 * qmax + 3, 2 * qmax - 2, 2):       # odd multiples of 1/2
            base = np.float32(float(exact.rn32(Fraction(h2, 2) * s)))
            for d in (-2, -1, 0, 1, 2):
                x = base
                for _ in range(abs(d)):
                    x = np.nextafter(x, np.float32(np.inf if d > 0 else -np.inf))
                if abs(float(x)) <= float(c):
                    vals.append(float(x))
        w = np.array(vals, np.float32)[None]
        r = orc.quantize(w, qbits, 1.0, export=export)
        assert Fraction(float(r.scale_f32[0])) == s
        for x, q in zip(vals, r.codes[0].tolist()):
            t = exact.rn32(Fraction(x) / s)
            assert q == exact.nearest_int_even(t, -qmax, qmax), (si, x)


def test_near_tie_quotients_exact(orc):
    check_near_ties(orc)


def test_percentile_rank_brute_force(orc):
    rng = np.random.default_rng(7)
    for _ in range(500):
        n = int(rng.integers(1, 12))
        v = (rng.integers(-6, 7, n) * 0.5).astype(np.float32)   # many ties
        k = int(rng.integers(1, n + 1))
        want = exact.kth_smallest_by_counting([abs(float(x)) for x in v], k)
        assert orc.kth_smallest_abs(v, k) == float(want)


# ------------------------------------------------- library special cases --

def check_kthvalue(orc):
    rng = np.random.default_rng(8)
    for kind in ("t3", "mix", "ties"):
        w = synth.random_matrix(rng, 37, 203, kind)
        for p in (1.0, 0.9999, 0.999, 0.9, 0.5, 0.01):
            r = orc.quantize(w, 6, p, export=False)
            k = orc.k_from_p(203, p)
            want = torch.kthvalue(torch.from_numpy(np.abs(w)), k, dim=1).values.numpy()
            assert np.array_equal(r.clip, want), (kind, p)
            rt = orc.quantize(w, 8, p, per_tensor=True, export=False)
            kt = orc.k_from_p(w.size, p)
            want_t = torch.kthvalue(torch.from_numpy(np.abs(w).ravel()), kt).values.item()
            assert rt.clip[0] == np.float32(want_t)


def test_clip_equals_torch_kthvalue(orc):
    check_kthvalue(orc)


def test_absmax_special_case(orc):
    rng = np.random.default_rng(9)
    w = synth.random_matrix(rng, 64, 777, "t3")
    r = orc.quantize(w, 6, 1.0)
    assert np.array_equal(r.clip, np.abs(w).max(axis=1))


def check_torch_round(orc):
    """q = clamp(round_half_even(clip(w) / s)) and w_hat = q * s, computed with
    torch CPU binary32 ops, for both scale modes and both bit widths."""
    rng = np.random.default_rng(10)
    for kind in ("normal", "t3", "mix"):
        w = synth.random_matrix(rng, 48, 512, kind)
        for qbits, qmax in ((6, 31), (8, 127)):
            for export in (False, True):
                for p in (1.0, 0.99):
                    r = orc.quantize(w, qbits, p, export=export)
                    W = torch.from_numpy(w)
                    c = torch.from_numpy(r.clip)[:, None]
                    s = torch.from_numpy(r.scale_f32)[:, None]
                    wc = torch.maximum(torch.minimum(W, c), -c)
                    q = torch.round(wc / s).clamp(-qmax, qmax)
                    assert np.array_equal(r.codes, q.to(torch.int8).numpy()), (kind, qbits, export)
                    dq = (q + 0.0) * s    # + 0.0 turns -0.0 codes into +0.0
                    assert np.array_equal(r.dq.view(np.uint32), dq.numpy().view(np.uint32))
                    if not export:
                        want_s = (torch.from_numpy(r.clip) / float(qmax)).numpy()
                        assert np.array_equal(r.scale_f32, want_s)


def test_quantize_equals_torch_cpu(orc):
    check_torch_round(orc)


def _f32_patterns(rng):
    """Binary32 bit patterns: every exponent with random and boundary fractions."""
    exps = np.arange(0, 256, dtype=np.uint32)
    fr = np.concatenate([
        rng.integers(0, 1 << 23, 2048, dtype=np.uint32),
        np.array([0, 1, 0xFFF, 0x1000, 0x1001, 0x1FFF, 0x2000, 0x3000, 0x7FFFFF,
                  0x7FE000, 0x7FF000, 0x7FEFFF], np.uint32),
    ])
    # fractions whose dropped bits sit exactly at, just below and above a tie,
    # for every shift a binary16 subnormal result can take
    for sh in range(13, 25):
        half = np.uint32(1 << (sh - 1)) if sh < 24 else np.uint32(0)
        base = rng.integers(0, 1 << 23, 64, dtype=np.uint32) & ~np.uint32((1 << min(sh, 23)) - 1)
        fr = np.concatenate([fr, base | half, base | (half - 1 if half else 0), base | (half + 1)])
    fr &= np.uint32(0x7FFFFF)
    pats = (exps[:, None] << np.uint32(23)) | fr[None, :]
    pats = pats.ravel()
    return np.concatenate([pats, pats | np.uint32(0x80000000)])


def check_f16(orc):
    rng = np.random.default_rng(12)
    pats = _f32_patterns(rng)
    x = pats.view(np.float32)
    x = x[~np.isnan(x)]
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = orc.f32_to_f16_bits(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(hex(pats[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]
    # and a dense random sweep
    y = rng.integers(0, 1 << 32, 1 << 21, dtype=np.uint64).astype(np.uint32).view(np.float32)
    y = y[~np.isnan(y)]
    with np.errstate(over="ignore"):
        want_y = y.astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.f32_to_f16_bits(y), want_y)


def test_f16_conversion_equals_numpy(orc):
    check_f16(orc)


def test_f16_decode_all_patterns(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_bits_to_f32(h)
    want = h.view(np.float16).astype(np.float32)
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.all(np.isnan(got[~fin]))


def check_bf16(orc):
    rng = np.random.default_rng(13)
    pats = np.concatenate([_f32_patterns(rng),
                           rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32)])
    x = pats.view(np.float32)
    x = x[~np.isnan(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16_bits(x), want)


def test_bf16_conversion_equals_torch(orc):
    check_bf16(orc)


def test_every_bf16_input_quantizes_like_torch(orc):
    """Exhaustive over the 65536 bf16 patterns (finite ones), several scales."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = synth.bf16_bits_to_f32(b)
    x = x[np.isfinite(x)]
    for qmax in (31, 127):
        for s in (2.0 ** -5, float(np.float32(1.0) / np.float32(31)), 0.0123, 3.0e-8, 1.0e30):
            s = float(np.float32(s))
            c = float(np.float32(qmax * s * 1.01))
            q = orc.quantize_values(x, c, s, qmax)
            X = torch.from_numpy(x)
            wc = torch.clamp(X, -c, c)
            tq = torch.round(wc / s).clamp(-qmax, qmax).to(torch.int8).numpy()
            assert np.array_equal(q, tq), (qmax, s)


# --------------------------------------------------------------- invariants --

def check_invariants(orc):
    ws = synth.draw_gpt9()
    for name in ("blocks.0.attn.c_q.weight", "blocks.3.mlp.proj.weight", "tok_emb.weight"):
        w = ws[name]
        for qbits, qmax in ((6, 31), (8, 127)):
            for export in (False, True):
                for p in (1.0, 0.9999, 0.99):
                    r = orc.quantize(w, qbits, p, export=export)
                    assert np.abs(r.codes.astype(int)).max() <= qmax
                    c = r.clip[:, None]
                    s = r.scale_f32[:, None]
                    normal_scale = (s[:, 0] >= 2.0 ** -14) if export else (s[:, 0] >= 2.0 ** -126)
                    at_clip = (np.abs(w) == c) & normal_scale[:, None]
                    assert np.all(np.abs(r.codes[at_clip].astype(int)) == qmax)
                    wc = np.clip(w, -c, c).astype(np.float64)
                    err = np.abs(wc - r.dq.astype(np.float64))
                    bound = s.astype(np.float64) * (0.5 + 2 * qmax * 2.0 ** -23)
                    assert np.all(err <= bound)
                    if export:
                        back = orc.dequant(r.packed, r.scale_f16, qbits, *w.shape)
                        assert np.array_equal(back.view(np.uint32), r.dq.view(np.uint32))


def test_invariants(orc):
    check_invariants(orc)


def check_pack_roundtrip_exhaustive(orc):
    """Every quadruple of codes in [-31, 31]: pack then unpack is the identity,
    and each 3-byte group equals the little-endian 24-bit sum of 6-bit fields.
    Swept in 63 chunks (first code fixed) to keep memory small."""
    v = np.arange(-31, 32, dtype=np.int32)
    b, c, d = np.meshgrid(v, v, v, indexing="ij")
    rest = np.stack([b.ravel(), c.ravel(), d.ravel()], axis=1)          # 63^3 x 3
    quad = np.empty((rest.shape[0], 4), np.int32)
    quad[:, 1:] = rest
    for a in range(-31, 32):
        quad[:, 0] = a
        q = quad.astype(np.int8).ravel()
        packed = orc.pack6_row(q)
        assert np.array_equal(orc.unpack6_row(packed, q.size), q)
        u = quad & 0x3F
        val = u[:, 0] | (u[:, 1] << 6) | (u[:, 2] << 12) | (u[:, 3] << 18)
        g = packed.reshape(-1, 3).astype(np.int32)
        assert np.array_equal(g[:, 0] | (g[:, 1] << 8) | (g[:, 2] << 16), val)


def test_pack_roundtrip_exhaustive(orc):
    check_pack_roundtrip_exhaustive(orc)


def test_pack_ragged_tail_zero_padded(orc):
    for cols in range(1, 10):
        q = np.full(cols, -31, np.int8)
        b = orc.pack6_row(q)
        assert b.size == 3 * ((cols + 3) // 4)
        back = orc.unpack6_row(b, 4 * ((cols + 3) // 4))
        assert np.all(back[:cols] == -31) and np.all(back[cols:] == 0)


def test_ste_identity_and_accumulate(orc):
    w, g = synth.draw_single_matrix()
    out = orc.ste_bwd(g)
    assert np.array_equal(out.view(np.uint32), g.view(np.uint32))
    acc = orc.ste_bwd(g, w, accumulate=True)
    assert np.array_equal(acc, (torch.from_numpy(w) + torch.from_numpy(g)).numpy())
    gb = synth.to_bf16_bits(g)
    wb = synth.to_bf16_bits(w)
    assert np.array_equal(orc.ste_bwd(gb), gb)
    accb = orc.ste_bwd(gb, wb, accumulate=True)
    tb = (torch.from_numpy(synth.bf16_bits_to_f32(wb)) + torch.from_numpy(synth.bf16_bits_to_f32(gb)))
    want = tb.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(accb, want)


def test_passthrough_equals_numpy_f16(orc):
    x = synth.draw_gpt9()["blocks.0.attn_scale"]
    assert np.array_equal(orc.passthrough_f16(x), x.astype(np.float16).view(np.uint16))


def test_zero_group_and_errors(orc):
    w = np.zeros((3, 5), np.float32)
    w[1] = [1e-3, -2e-3, 0, 0, 5e-4]
    r = orc.quantize(w, 6, 1.0)
    assert r.status == oracle.OR_OK
    assert np.all(r.codes[0] == 0) and not np.any(np.signbit(r.dq[0]))
    assert r.scale_f16[0] == 0 and r.scale_f16[2] == 0
    # tiny group whose binary16 scale underflows to 0 -> all codes 0
    t = np.array([[1e-9, -2e-9]], np.float32)
    r = orc.quantize(t, 6, 1.0)
    assert r.scale_f16[0] == 0 and np.all(r.codes == 0)
    # binary16 overflow of the scale is a range error; training mode is fine
    big = np.array([[3e6, -1.0]], np.float32)
    assert orc.quantize(big, 6, 1.0, export=True).status == oracle.OR_ERR_RANGE
    assert orc.quantize(big, 6, 1.0, export=False).status == oracle.OR_OK
    # non-finite input is reported
    bad = np.array([[1.0, np.inf]], np.float32)
    assert orc.quantize(bad, 6, 1.0).status == oracle.OR_ERR_NONFINITE
    bad = np.array([[np.nan, 1.0]], np.float32)
    assert orc.quantize(bad, 8, 0.5).status == oracle.OR_ERR_NONFINITE
    # bad arguments
    assert orc.quantize(w, 7, 1.0).status == oracle.OR_ERR_ARG
    assert orc.quantize(w, 6, 0.0).status == oracle.OR_ERR_ARG
    assert orc.quantize(w, 6, 1.5).status == oracle.OR_ERR_ARG


def test_per_tensor_single_row_equals_per_row(orc):
    rng = np.random.default_rng(14)
    w = synth.random_matrix(rng, 1, 1000, "mix")
    a = orc.quantize(w, 6, 0.97)
    b = orc.quantize(w, 6, 0.97, per_tensor=True)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.packed, b.packed)
    assert a.scale_f16[0] == b.scale_f16[0]


def test_strided_rows_use_first_cols(orc):
    rng = np.random.default_rng(15)
    full = synth.random_matrix(rng, 6, 40, "t3")
    a = orc.quantize(full, 6, 0.9, cols=33)
    b = orc.quantize(np.ascontiguousarray(full[:, :33]), 6, 0.9)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.dq, b.dq)


# ------------------------------------------------------------ export plan --

def test_export_plan_rules():
    P = plan.DEFAULT_INT8_PATTERNS
    assert plan.classify("tok_emb.weight", (1024, 512), True, P) == ("int8", (1024, 512))
    assert plan.classify("lm_head.weight", (1792, 512), True, P) == ("int8", (1792, 512))
    assert plan.classify("blocks.0.mlp.fc.weight", (1536, 512), True, P) == ("int6", (1536, 512))
    assert plan.classify("blocks.0.attn_scale", (512,), True, P) == ("fp16", None)
    # small wins over a name match; exactly 65536 elements is not small
    assert plan.classify("tok_emb.weight", (100, 512), True, P) == ("fp16", None)
    assert plan.classify("x", (256, 256), True, P) == ("int6", (256, 256))
    assert plan.classify("x", (255, 256), True, P) == ("fp16", None)
    assert plan.classify("step", (70000,), False, P) == ("raw", None)
    assert plan.classify("conv", (256, 32, 3, 3), True, P) == ("int6", (256, 288))
    assert plan.classify("conv", (64, 32, 3, 3), True, P) == ("fp16", None)
    assert plan.patterns_from_env("a.weight, b ,") == ("a.weight", "b")
    assert plan.patterns_from_env(None) == P


# ------------------------------------------------------ snapshot averaging --

def _dyadic(rng, n, lo=-2 ** 10, hi=2 ** 10, shift=8):
    """Values k / 2^shift with small integers k: sums, halves and quarters of
    them are exact in binary32."""
    return (rng.integers(lo, hi, size=n).astype(np.float64) / 2 ** shift).astype(np.float32)


def check_average(orc, seed=31):
    rng = np.random.default_rng(seed)
    M, E = oracle.AVG_MEAN, oracle.AVG_EMA
    # the first snapshot replaces whatever the average held (a stale average
    # of a far larger magnitude would leave a trace if it were blended in)
    x = rng.standard_normal(257).astype(np.float32)
    stale = (rng.standard_normal(257) * 1e30).astype(np.float32)
    a = orc.average_update(stale, x, M, count=0)
    assert np.array_equal(a.view(np.uint32), x.view(np.uint32))
    xb = synth.to_bf16_bits(x)
    a = orc.average_update(stale, xb, M, count=0)
    assert np.array_equal(a.view(np.uint32), (xb.astype(np.uint32) << 16))
    # mean of two snapshots, and a mean step with t = 1/4, are exact here
    x0, x1 = _dyadic(rng, 500), _dyadic(rng, 500)
    a = orc.average_update(np.zeros(500, np.float32), x0, M, count=0)
    a = orc.average_update(a, x1, M, count=1)
    want = [float((Fraction(float(u)) + Fraction(float(v))) / 2) for u, v in zip(x0, x1)]
    assert np.array_equal(a, np.array(want, np.float32))
    a3 = _dyadic(rng, 500)
    a = orc.average_update(a3, x1, M, count=3)
    want = [float(Fraction(float(u)) + (Fraction(float(v)) - Fraction(float(u))) / 4)
            for u, v in zip(a3, x1)]
    assert np.array_equal(a, np.array(want, np.float32))
    # EMA with decay 1/2 is the exact midpoint; decay 0 keeps the snapshot,
    # decay 1 the average (non-zero values: the +-0 sums are not at issue)
    a = orc.average_update(x0, x1, E, decay=0.5)
    want = [float((Fraction(float(u)) + Fraction(float(v))) / 2) for u, v in zip(x0, x1)]
    assert np.array_equal(a, np.array(want, np.float32))
    nz0 = np.where(x0 == 0, np.float32(0.5), x0)
    nz1 = np.where(x1 == 0, np.float32(0.25), x1)
    assert np.array_equal(orc.average_update(nz0, nz1, E, decay=0.0), nz1)
    assert np.array_equal(orc.average_update(nz0, nz1, E, decay=1.0), nz0)
    # the pages' decay over 300 steps of a constant snapshot: 1 - 0.997^k
    # (float32 rounding over 300 steps stays far inside 1e-4)
    a = np.zeros(4, np.float32)
    one = np.ones(4, np.float32)
    for _ in range(300):
        a = orc.average_update(a, one, E, decay=0.997)
    assert np.all(np.abs(a - (1.0 - 0.997 ** 300)) < 1e-4)
    # arguments outside the definition are refused
    for bad in (dict(kind=2), dict(kind=E, decay=1.5), dict(kind=M, count=-1)):
        with pytest.raises(ValueError):
            orc.average_update(x0, x1, bad.pop("kind"), **bad)


def test_average_pins(orc):
    check_average(orc)


def test_fakequant_average_composes(orc):
    """The fused reference is the fake-quant output fed to the average."""
    rng = np.random.default_rng(3)
    w = synth.random_matrix(rng, 7, 40, "t3")
    avg = rng.standard_normal((7, 40)).astype(np.float32)
    ref, a = orc.fakequant_average(w, avg, 6, 0.99, oracle.AVG_MEAN, count=2)
    assert np.array_equal(a, orc.average_update(avg, ref.dq, oracle.AVG_MEAN, count=2))
    assert np.array_equal(ref.dq, orc.quantize(w, 6, 0.99, export=False).dq)


def check_col_scale(orc, seed=41):
    """AWQ column scaling (reading R12): each element is the exact product
    w[r, c] * t[c] rounded once to binary32 (then, for bf16 weights, to the
    nearest even bf16), computed here with rational arithmetic; t = 1 leaves
    the weight and its quantization unchanged; a uniform power of two scales
    the codes' clip and scale exactly."""
    rng = np.random.default_rng(seed)
    rows, cols, ld = 5, 37, 41                       # rows != cols, strided rows
    w = np.zeros((rows, ld), np.float32)
    w[:, :cols] = (rng.standard_normal((rows, cols)) * 0.03).astype(np.float32)
    w[:, cols:] = 1e30                               # past the used columns: never read
    t = (rng.random(cols) * 3.0 + 0.05).astype(np.float32)
    got = orc.col_scale(w, t, cols)
    for r in range(rows):
        for c in range(cols):
            want = exact.rn32(Fraction(float(w[r, c])) * Fraction(float(t[c])))
            assert Fraction(float(got[r, c])) == want, (r, c)
    wb = synth.to_bf16_bits(w[:, :cols]).reshape(rows, cols)
    gotb = orc.col_scale(wb, t)
    for r in range(rows):
        for c in range(cols):
            x = Fraction(float((np.uint32(wb[r, c]) << np.uint32(16)).view(np.float32)))
            want = exact.rnbf16(exact.rn32(x * Fraction(float(t[c]))))
            have = Fraction(float((np.uint32(gotb[r, c]) << np.uint32(16)).view(np.float32)))
            assert have == want, (r, c)
    # t = 1: the same weight, the same export
    ones = np.ones(cols, np.float32)
    assert np.array_equal(orc.col_scale(w, ones, cols).view(np.uint32), w[:, :cols].view(np.uint32))
    a = orc.quantize(w[:, :cols].copy(), 6, 0.95, col_scale=ones)
    b = orc.quantize(w[:, :cols].copy(), 6, 0.95)
    assert np.array_equal(a.packed, b.packed) and np.array_equal(a.scale_f16, b.scale_f16)
    # a uniform power of two: the same codes, clip and scale times 4 (training mode)
    four = np.full(cols, 4.0, np.float32)
    a = orc.quantize(w[:, :cols].copy(), 8, 0.9, export=False, col_scale=four)
    b = orc.quantize(w[:, :cols].copy(), 8, 0.9, export=False)
    assert np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.clip, b.clip * 4) and np.array_equal(a.scale_f32, b.scale_f32 * 4)


def test_col_scale_pins(orc):
    check_col_scale(orc)
