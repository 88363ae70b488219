"""GPTQ-lite oracle: column-by-column quantization with error feedback.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library and never imports it.  Parity unpinned against the
pages' authors' own code (the pages hold none); pinned against the published
algorithm by ``tests/test_oracle_gptq.py``.

Source: "Record: Unified Attention + FA3 + Legal TTT" (PR #1202), section
"Quantization": "GPTQ-lite", bits 6, scope weights.  The page names the method
and gives nothing else.  The reading taken here is the published GPTQ
algorithm (Frantar, Ashkboos, Hoefler, Alistarh, "GPTQ: Accurate Post-Training
Quantization for Generative Pre-trained Transformers", 2022, Algorithm 1),
"lite" meaning the plain algorithm on this library's existing per-row grid:
no reordering of columns, no group-wise scales, no search over scales.

Readings (each the plainest one; the numbering is used in the tests):
  G1  Grid.  One binary16 scale per row, exactly as the export computes it
      from the ORIGINAL row (percentile clip c = k-th smallest |w|, s =
      binary16(c / qmax)); GPTQ changes the codes, never the scales.  A column
      value v is quantized the way the export quantizes a weight: clip to
      [-c, c], divide by s, round half to even, clamp to [-qmax, qmax]
      (s = 0 gives 0).  Every step of GPTQ, this quotient included, is
      carried out in binary64.
  G2  Hessian.  H = 2 X^T X for calibration inputs X [n, cols] (the layer's
      inputs, one row per token), in binary64.  (The scale of H does not
      matter: the algorithm is invariant to H -> a H, damping included.)
  G3  Dead inputs.  A zero diagonal entry H[j, j] is set to 1 and column j
      of the working weights to 0.
  G4  Damping.  lambda = percdamp * mean(diag H) is added to the diagonal,
      percdamp = 0.01.
  G5  U = the upper-triangular Cholesky factor of H^-1 (H^-1 = U^T U).
  G6  Lazy batches of B = 128 columns.
Outputs are those of the export: int8 codes, binary16 scales, the packed
int6 / int8 rows, and w_hat = q * s (binary32; bf16 weights get bf16 w_hat).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import default as _c_oracle

PERCDAMP = 0.01
BLOCK = 128


@dataclass
class GPTQResult:
    status: int
    codes: np.ndarray        # int8 [rows, cols]
    scale_f16: np.ndarray    # uint16 [rows]
    dq: np.ndarray           # float32 (or bf16 bits as uint16) [rows, cols]
    packed: np.ndarray       # uint8 [rows, packed row bytes]
    quotient: np.ndarray     # float64 [rows, cols]: the value each code rounds (after the clip, before rounding)


def _widen(w: np.ndarray) -> np.ndarray:
    """fp32 weights, or bf16 bit patterns (uint16), widened exactly to binary64."""
    if w.dtype == np.uint16:
        return (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return w.astype(np.float64)


def hessian(x: np.ndarray) -> np.ndarray:
    """G2: H = 2 X^T X in binary64 for X [n, cols] (fp32, or bf16 bits)."""
    xd = _widen(np.ascontiguousarray(x))
    return 2.0 * (xd.T @ xd)


def _quantize_column(v: np.ndarray, c: np.ndarray, s: np.ndarray, qmax: int):
    """G1: the export's quantizer on one column of values, in binary64.
    Returns (codes as float64, the quotient that was rounded)."""
    vc = np.minimum(np.maximum(v, -c), c)
    t = np.zeros_like(vc)
    nz = s != 0.0
    t[nz] = vc[nz] / s[nz]
    r = np.rint(t)                       # round half to even
    q = np.minimum(np.maximum(r, -qmax), qmax)
    q[~nz] = 0.0
    return q, t


def gptq(w: np.ndarray, H: np.ndarray, qbits: int = 6, p: float = 1.0,
         percdamp: float = PERCDAMP, block: int = BLOCK) -> GPTQResult:
    """GPTQ of a weight w [rows, cols] (rows = output features) against the
    Hessian H [cols, cols] of its inputs, in the order of Algorithm 1."""
    assert w.ndim == 2 and H.shape == (w.shape[1], w.shape[1])
    rows, cols = w.shape
    qmax = 31 if qbits == 6 else 127
    C = _c_oracle()
    # G1: clip and binary16 scale of every original row, as the export takes them
    base = C.quantize(np.ascontiguousarray(w), qbits, p, export=True)
    if base.status != 0:
        empty = np.zeros((0,))
        return GPTQResult(base.status, base.codes, base.scale_f16, base.dq, base.packed, empty)
    c = base.clip.astype(np.float64)
    s = C.f16_bits_to_f32(base.scale_f16).astype(np.float64)

    W = _widen(w).copy()
    H = np.array(H, dtype=np.float64, copy=True)
    # G3: dead inputs
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    W[:, dead] = 0.0
    # G4: damping
    H[np.diag_indices(cols)] += percdamp * np.mean(np.diag(H))
    # G5: U, the upper Cholesky factor of H^-1
    Hinv = np.linalg.inv(H)
    U = np.linalg.cholesky(Hinv).T
    # G6: columns in lazy batches of `block`
    Q = np.zeros((rows, cols))
    T = np.zeros((rows, cols))
    for i1 in range(0, cols, block):
        i2 = min(i1 + block, cols)
        W1 = W[:, i1:i2].copy()
        E1 = np.zeros((rows, i2 - i1))
        for j in range(i2 - i1):
            col = W1[:, j]
            q, t = _quantize_column(col, c, s, qmax)
            err = (col - q * s) / U[i1 + j, i1 + j]
            # feed the error forward into the rest of this batch
            W1[:, j:] -= np.outer(err, U[i1 + j, i1 + j:i2])
            E1[:, j] = err
            Q[:, i1 + j] = q
            T[:, i1 + j] = t
        # and, once per batch, into every later column
        W[:, i2:] -= E1 @ U[i1:i2, i2:]

    codes = Q.astype(np.int8)
    dq32 = (Q * s[:, None]).astype(np.float32)          # exact: q * s has at most 19 bits
    dq32[codes == 0] = 0.0                              # +0.0 for q = 0 (never -0.0)
    dq = C.f32_to_bf16_bits(dq32).reshape(rows, cols) if w.dtype == np.uint16 else dq32
    prb = C.packed_row_bytes(cols, qbits)
    if qbits == 6:
        packed = np.stack([C.pack6_row(codes[r]) for r in range(rows)]) if rows else \
            np.zeros((0, prb), np.uint8)
    else:
        packed = codes.view(np.uint8).copy()
    return GPTQResult(0, codes, base.scale_f16.copy(), dq, packed, T)
