"""Pins of the GPTQ-lite oracle (oracle/gptq.py), on the CPU.

The oracle restates the published GPTQ algorithm (Cholesky factor of the
inverse Hessian, lazy batches).  It is pinned against things that do not
share its formulation:
  * a hand-worked case (tests/golden/gptq_error_feedback.txt) where the error
    feedback turns a 0 into a 1;
  * a diagonal Hessian decouples the columns, so GPTQ must equal plain
    round-to-nearest, checked against exact rational rounding;
  * the textbook optimal-brain-quantizer recursion: after each column,
    update the remaining weights with the inverse of the REMAINING Hessian,
    recomputed from scratch (no Cholesky factor, no lazy batches);
  * the batch size must not change the result;
  * the layer-wise proxy loss tr((W - Q) H (W - Q)^T) must beat plain
    rounding on correlated inputs;
  * planted mistakes in the oracle's source are each caught by one of these.
"""
from __future__ import annotations

import os
import sys
import types
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import gptq as G
from tests import exact

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


def _calibration(rng, n, cols, corr=0.9):
    """Correlated synthetic layer inputs (AR(1) across features)."""
    z = rng.standard_normal((n, cols))
    x = np.empty_like(z)
    x[:, 0] = z[:, 0]
    for j in range(1, cols):
        x[:, j] = corr * x[:, j - 1] + np.sqrt(1 - corr * corr) * z[:, j]
    return x.astype(np.float32)


def _weights(rng, rows, cols):
    return (rng.standard_t(3, (rows, cols)) * 0.02 / np.sqrt(3)).astype(np.float32)


def _scales(w, qbits, p):
    base = oracle.quantize(w, qbits, p, export=True)
    return base.clip.astype(np.float64), oracle.f16_bits_to_f32(base.scale_f16).astype(np.float64)


# ------------------------------------------------------------------ pins --

def check_golden(mod):
    g = _read("gptq_error_feedback.txt")
    scale = float(g["w_scaled_by"][0][0])
    w = (np.array([[float(v) for v in r] for r in g["row"]]) / scale).astype(np.float32)
    H = np.array([float(v) for v in g["H"][0]]).reshape(3, 3)
    r = mod.gptq(w, H, int(g["qbits"][0][0]), float(g["p"][0][0]), percdamp=float(g["percdamp"][0][0]))
    assert r.status == 0
    assert r.scale_f16.tolist() == [int(v, 16) for v in g["scale_f16"][0]]
    assert r.codes.tolist() == [[int(v) for v in row] for row in g["codes"]]


def check_diagonal_hessian_is_rtn(mod):
    rng = np.random.default_rng(11)
    for rows, cols, qbits, p in ((7, 19, 6, 1.0), (5, 40, 8, 0.9), (9, 33, 6, 0.95)):
        w = _weights(rng, rows, cols)
        H = np.diag(rng.uniform(0.5, 2.0, cols))
        r = mod.gptq(w, H, qbits, p)
        c, s = _scales(w, qbits, p)
        qmax = 31 if qbits == 6 else 127
        for i in range(rows):
            for j in range(cols):
                if s[i] == 0:
                    want = 0
                else:
                    wc = min(max(Fraction(float(w[i, j])), -Fraction(c[i])), Fraction(c[i]))
                    want = exact.nearest_int_even(wc / Fraction(s[i]), -qmax, qmax)
                assert r.codes[i, j] == want, (rows, cols, i, j)


def obs_reference(w, H, qbits, p, percdamp=G.PERCDAMP):
    """Column by column: quantize column q of the remaining set F, then move
    the remaining weights by -(w_q - quant(w_q)) / [H_F^-1]_qq * (H_F^-1)_q,:,
    with H_F^-1 the inverse of the Hessian restricted to F, recomputed from
    scratch at every step (the optimal-brain-quantizer update the GPTQ paper
    starts from)."""
    rows, cols = w.shape
    qmax = 31 if qbits == 6 else 127
    c, s = _scales(w, qbits, p)
    W = w.astype(np.float64).copy()
    Hd = np.array(H, dtype=np.float64, copy=True)
    for j in range(cols):                      # dead inputs
        if Hd[j, j] == 0.0:
            Hd[j, j] = 1.0
            W[:, j] = 0.0
    lam = percdamp * np.trace(Hd) / cols       # damping
    Hd = Hd + lam * np.eye(cols)
    Q = np.zeros((rows, cols), np.int64)
    for j in range(cols):
        F = list(range(j, cols))
        Hinv_F = np.linalg.inv(Hd[np.ix_(F, F)])
        for i in range(rows):
            v = min(max(W[i, j], -c[i]), c[i])
            q = 0 if s[i] == 0 else int(min(max(np.rint(v / s[i]), -qmax), qmax))
            Q[i, j] = q
            W[i, F] -= (W[i, j] - q * s[i]) / Hinv_F[0, 0] * Hinv_F[0, :]
    return Q


def check_matches_obs_recursion(mod):
    rng = np.random.default_rng(12)
    for rows, cols, qbits, p, block in ((6, 20, 6, 1.0, 128), (4, 31, 6, 0.9, 7), (5, 24, 8, 1.0, 5)):
        w = _weights(rng, rows, cols)
        x = _calibration(rng, 64, cols)
        H = G.hessian(x)
        got = mod.gptq(w, H, qbits, p, block=block)
        want = obs_reference(w, H, qbits, p)
        assert np.array_equal(got.codes.astype(np.int64), want), (rows, cols, block)


def check_block_size_invariance(mod):
    rng = np.random.default_rng(13)
    w = _weights(rng, 12, 70)
    H = G.hessian(_calibration(rng, 200, 70))
    ref = mod.gptq(w, H, 6, 0.99, block=128)
    for b in (1, 3, 16, 64):
        assert np.array_equal(mod.gptq(w, H, 6, 0.99, block=b).codes, ref.codes), b


def check_beats_rtn_and_invariants(mod):
    rng = np.random.default_rng(14)
    rows, cols = 64, 96
    w = _weights(rng, rows, cols)
    H = G.hessian(_calibration(rng, 512, cols))
    r = mod.gptq(w, H, 6, 0.999)
    base = oracle.quantize(w, 6, 0.999, export=True)
    s = oracle.f16_bits_to_f32(base.scale_f16).astype(np.float64)
    assert np.abs(r.codes.astype(int)).max() <= 31
    assert np.array_equal(r.scale_f16, base.scale_f16)              # G1: scales of the export
    assert np.array_equal(r.dq, (r.codes * s[:, None]).astype(np.float32))
    d_g = w.astype(np.float64) - r.codes * s[:, None]
    d_r = w.astype(np.float64) - base.codes * s[:, None]
    loss_g = np.einsum("ij,jk,ik->", d_g, H, d_g)
    loss_r = np.einsum("ij,jk,ik->", d_r, H, d_r)
    assert loss_g < 0.8 * loss_r, (loss_g, loss_r)
    # packed rows decode to the codes
    for i in range(0, rows, 13):
        assert np.array_equal(oracle.unpack6_row(r.packed[i], cols), r.codes[i])


def check_dead_input(mod):
    rng = np.random.default_rng(15)
    x = _calibration(rng, 100, 12)
    x[:, 5] = 0.0                                   # an input that is never active
    w = _weights(rng, 4, 12)
    r = mod.gptq(w, G.hessian(x), 6, 1.0)
    assert (r.codes[:, 5] == 0).all()


PINS = [check_golden, check_diagonal_hessian_is_rtn, check_matches_obs_recursion,
        check_block_size_invariance, check_beats_rtn_and_invariants, check_dead_input]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_gptq_oracle_pin(pin):
    pin(G)


def test_bf16_weights_give_bf16_w_hat():
    rng = np.random.default_rng(16)
    w32 = _weights(rng, 8, 24)
    wb = oracle.f32_to_bf16_bits(w32).reshape(8, 24)
    H = G.hessian(_calibration(rng, 50, 24))
    r = G.gptq(wb, H, 6, 1.0)
    base = oracle.quantize(wb, 6, 1.0, export=True)
    assert np.array_equal(r.scale_f16, base.scale_f16)
    s = oracle.f16_bits_to_f32(r.scale_f16)
    assert np.array_equal(r.dq, oracle.f32_to_bf16_bits((r.codes * s[:, None]).astype(np.float32)).reshape(8, 24))


# --------------------------------------------------------------- mutants --

MUTANTS = {
    "drop_feedback": ("W1[:, j:] -= np.outer(err, U[i1 + j, i1 + j:i2])", "pass"),
    "feedback_sign": ("W1[:, j:] -= np.outer(err, U[i1 + j, i1 + j:i2])",
                      "W1[:, j:] += np.outer(err, U[i1 + j, i1 + j:i2])"),
    "drop_lazy_update": ("W[:, i2:] -= E1 @ U[i1:i2, i2:]", "pass"),
    "lower_factor": ("U = np.linalg.cholesky(Hinv).T", "U = np.linalg.cholesky(Hinv)"),
    "factor_of_H": ("Hinv = np.linalg.inv(H)", "Hinv = H"),
    "error_not_scaled": ("err = (col - q * s) / U[i1 + j, i1 + j]", "err = (col - q * s)"),
    "no_damping": ("H[np.diag_indices(cols)] += percdamp * np.mean(np.diag(H))", "pass"),
    "error_from_quotient": ("err = (col - q * s) / U[i1 + j, i1 + j]",
                            "err = (col / np.where(s == 0, 1, s) - q) / U[i1 + j, i1 + j]"),
}


def _mutant(old, new):
    src = open(G.__file__).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new).replace("from . import default as _c_oracle",
                                        "from oracle import default as _c_oracle")
    name = f"gptq_mutant_{abs(hash((old, new)))}"
    mod = types.ModuleType(name)
    sys.modules[name] = mod          # dataclasses look their module up there
    exec(compile(src, name + ".py", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_gptq_mutant_is_caught(name):
    mod = _mutant(*MUTANTS[name])
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, np.linalg.LinAlgError, ValueError):
            return
    pytest.fail(f"planted mistake {name!r} passed every GPTQ pin")
