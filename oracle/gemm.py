"""Reference of the dequant-on-load GEMM: Y = X W_hat^T.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library and never imports it.

What it computes (the reading of the consuming GEMM, from "SubSixteen v2",
section Other -- straight-through fake quantization in the forward pass, so
the layer's matmul consumes the fake-quant weight -- and the int6 / int8
storage of "... Int6AWQ MixedBits", Mixed-bit quantization details):
    W_hat[n, k] = bf16(RN(q[n, k] * s[n]))   (the C oracle's dequant, bf16 out)
    Y[m, n]     = sum_k X[m, k] * W_hat[n, k] (X bf16)
as a real number.  Every product of two bf16 values is exact in binary64, so
the only error of a reference is in the sum:
  contraction()       binary64 matrix product (a library primitive); its
                      error is at most K * 2^-53 * sum_k |X W_hat| (a sum of
                      K terms in binary64), pinned against exact sums;
  contraction_exact() the exact sum rounded once to binary64 (math.fsum),
                      for chosen (m, n) entries.
Both also return sum_k |X[m, k] W_hat[n, k]|, the scale of the error bound
of a binary32 accumulation.
"""
from __future__ import annotations

import math

import numpy as np

from . import default as _c_oracle


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> binary64, exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def w_hat_bf16(packed: np.ndarray, scale_f16: np.ndarray, qbits: int, n: int, k: int) -> np.ndarray:
    """W_hat as bf16 bits [n, k] from packed rows and binary16 row scales."""
    return _c_oracle().dequant(packed, scale_f16, qbits, n, k, out_bf16=True)


def contraction(x_bf16: np.ndarray, w_bf16: np.ndarray):
    """(Y, sum |x w|) for all entries: X [M, K] and W_hat [N, K] as bf16 bits."""
    xd, wd = widen_bf16(x_bf16), widen_bf16(w_bf16)
    return xd @ wd.T, np.abs(xd) @ np.abs(wd).T


def contraction_exact(x_bf16: np.ndarray, w_bf16: np.ndarray, pairs):
    """(Y, sum |x w|) for the entries (m, n) in ``pairs``, each sum exact and
    rounded once to binary64."""
    xd, wd = widen_bf16(x_bf16), widen_bf16(w_bf16)
    y = np.empty(len(pairs))
    a = np.empty(len(pairs))
    for i, (m, n) in enumerate(pairs):
        prod = xd[m] * wd[n]                  # exact: 8-bit x 8-bit significands
        y[i] = math.fsum(prod.tolist())
        a[i] = math.fsum(np.abs(prod).tolist())
    return y, a
