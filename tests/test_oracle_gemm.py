"""Pins of the consuming-GEMM reference (oracle/gemm.py), on the CPU: a
hand-worked 2 x 3 x 16 product, exact rational sums on small cases, and the
stated error of the binary64 product against exactly rounded sums."""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import oracle
import synth
from oracle import gemm as GM

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, *v = line.split()
                out.setdefault(k, []).append(v)
    return out


def test_worked_2x3x16():
    g = _read("gemm_dequant_2x3x16.txt")
    codes = np.array([[int(v) for v in r] for r in g["codes"]], np.int8)
    packed = np.stack([oracle.pack6_row(r) for r in codes])
    scale = np.array([int(v, 16) for v in g["scale_f16"][0]], np.uint16)
    w = GM.w_hat_bf16(packed, scale, 6, 3, 16)
    x = oracle.f32_to_bf16_bits(np.array([[float(v) for v in r] for r in g["x"]], np.float32)).reshape(2, 16)
    want = np.array([[float(v) for v in r] for r in g["y"]])
    y, _ = GM.contraction(x, w)
    assert np.array_equal(y, want)
    ye, _ = GM.contraction_exact(x, w, [(m, n) for m in range(2) for n in range(3)])
    assert np.array_equal(ye.reshape(2, 3), want)


def test_exact_sums_against_fractions():
    rng = np.random.default_rng(31)
    K = 40
    x = synth.to_bf16_bits((rng.standard_normal((3, K)) * 0.5).astype(np.float32)).reshape(3, K)
    wq = oracle.quantize(synth.random_matrix(rng, 4, K, "t3"), 6, 1.0, export=True)
    w = GM.w_hat_bf16(wq.packed, wq.scale_f16, 6, 4, K)
    pairs = [(m, n) for m in range(3) for n in range(4)]
    ye, ae = GM.contraction_exact(x, w, pairs)
    xd, wd = GM.widen_bf16(x), GM.widen_bf16(w)
    for i, (m, n) in enumerate(pairs):
        exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xd[m], wd[n]))
        assert ye[i] == float(exact)                      # rounded once to binary64
        assert ae[i] == float(sum(abs(Fraction(float(a)) * Fraction(float(b))) for a, b in zip(xd[m], wd[n])))


def test_binary64_product_within_its_stated_error():
    rng = np.random.default_rng(32)
    M, N, K = 6, 9, 2048
    x = synth.to_bf16_bits((rng.standard_normal((M, K)) * 0.5).astype(np.float32)).reshape(M, K)
    wq = oracle.quantize(synth.random_matrix(rng, N, K, "t3"), 8, 0.9999, export=True)
    w = GM.w_hat_bf16(wq.packed, wq.scale_f16, 8, N, K)
    y, a = GM.contraction(x, w)
    pairs = [(m, n) for m in range(M) for n in range(N)]
    ye, ae = GM.contraction_exact(x, w, pairs)
    for i, (m, n) in enumerate(pairs):
        assert abs(y[m, n] - ye[i]) <= K * 2.0 ** -53 * ae[i]
        assert abs(a[m, n] - ae[i]) <= K * 2.0 ** -53 * ae[i]
    # W_hat is the bf16 w_hat of the export itself
    wb = oracle.quantize(oracle.f32_to_bf16_bits(synth.random_matrix(rng, 5, 64, "t3")).reshape(5, 64), 6, 1.0,
                         export=True)
    assert np.array_equal(GM.w_hat_bf16(wb.packed, wb.scale_f16, 6, 5, 64), wb.dq)
