"""GPU parity of AWQ column scaling (gq_tensor.col_scale) against the oracle.

With column scales t the quantized group is w'[r, c] = RN_dtype(w[r, c] * t[c])
and every output (clip, scales, codes, packed bytes, w_hat) is that of w'.
Both sides round the same operations the same way, so the outputs must match
bit for bit.  Covered: fp32 and bf16 weights; int6 and int8; absmax, the
register top-M select and the radix select; the warp-team (<= 2048 columns)
and block-team row kernels; ragged column counts; strided rows; scale vectors
that are 16-byte aligned (vector loads) or only 4-byte aligned; export and
training-mode fake quant.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_gpu_parity import assert_same, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int6_int8_weight_b200 import gq as mod
    return mod


def _scales_dev(t, misalign):
    if not misalign:
        return torch.from_numpy(t).cuda()
    buf = torch.zeros(t.size + 1, dtype=torch.float32, device="cuda")
    buf[1:].copy_(torch.from_numpy(t))
    return buf[1:]                                  # 4-byte aligned only


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(300, 512), (64, 4096), (9, 16384), (37, 1000), (5, 130)])
def test_awq_export_matches_oracle(gq, dtype, rows, cols):
    rng = np.random.default_rng(rows * 3 + cols + (dtype == "bf16"))
    w = synth.random_matrix(rng, rows, cols, "t3")
    if dtype == "bf16":
        w = synth.to_bf16_bits(w).reshape(rows, cols)
    t = synth.awq_col_scales(rng, cols)
    W = to_dev(w)
    for misalign in (False, True):
        T = _scales_dev(t, misalign)
        for qbits, p in ((6, 0.9999), (6, 0.99), (8, 1.0)):
            (o,) = gq.export_pack([gq.Request(W, qbits, p, want_packed=True, want_scale_f16=True,
                                              want_scale_f32=True, want_clip=True, col_scale=T)])
            torch.cuda.synchronize()
            ref = oracle.quantize(w, qbits, p, export=True, col_scale=t)
            what = f"{dtype} {rows}x{cols} q{qbits} p{p} misaligned {misalign}"
            assert ref.status == oracle.OR_OK
            assert_same(to_host(o.packed), ref.packed, f"{what}: packed")
            assert_same(to_host(o.scale_f16).view(np.uint16), ref.scale_f16, f"{what}: scale_f16")
            assert_same(to_host(o.clip), ref.clip, f"{what}: clip")
            assert_same(to_host(o.dq), ref.dq, f"{what}: w_hat")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_awq_fakequant_strided_rows(gq, dtype):
    rng = np.random.default_rng(7 + (dtype == "bf16"))
    rows, cols, ld = 48, 1500, 1536
    full = synth.random_matrix(rng, rows, ld, "mix")
    if dtype == "bf16":
        full = synth.to_bf16_bits(full).reshape(rows, ld)
    t = synth.awq_col_scales(rng, cols)
    W = to_dev(full)
    (o,) = gq.fakequant([gq.Request(W, 6, 0.999, want_scale_f32=True, want_codes=True, cols=cols,
                                    col_scale=torch.from_numpy(t).cuda())])
    torch.cuda.synchronize()
    ref = oracle.quantize(full, 6, 0.999, export=False, cols=cols, col_scale=t)
    assert_same(to_host(o.dq), ref.dq, f"{dtype} strided: w_hat")
    assert_same(to_host(o.codes), ref.codes, f"{dtype} strided: codes")
    assert_same(to_host(o.scale_f32), ref.scale_f32, f"{dtype} strided: scale")


def test_awq_unit_scales_equal_plain_export(gq):
    """t = 1 is the plain export, on the fused row kernel's input."""
    rng = np.random.default_rng(9)
    w = synth.random_matrix(rng, 256, 2048, "t3")
    W = to_dev(w)
    ones = torch.ones(2048, device="cuda")
    (a,) = gq.export_pack([gq.Request(W, 6, 0.9999, want_packed=True, want_scale_f16=True, col_scale=ones)])
    (b,) = gq.export_pack([gq.Request(W, 6, 0.9999, want_packed=True, want_scale_f16=True)])
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed) and torch.equal(a.dq, b.dq)
    assert torch.equal(a.scale_f16.view(torch.int16), b.scale_f16.view(torch.int16))
