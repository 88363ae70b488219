"""GPU parity of gq_fakequant_average against the CPU oracle, bit for bit.

The fused pass fake-quantizes each tensor and updates a binary32 running
average of its quantize-dequantize snapshots: the mean of n snapshots
(n = 0 copies the snapshot) or an exponential moving average.  Both sides
take the snapshot as the model holds it (bf16 w_hat widened exactly) and do
each step as one correctly rounded binary32 operation, so the averages, the
optional w_hat and the scales must match exactly (0 ulp).

Paths covered: the pipelined kernel's branch-free loops (average only, and
average + w_hat), its generic loop (a 4-byte aligned average, rows with a
zero scale), the fallback kernel (a misaligned weight base), per-tensor
groups and binary16-scale mode.
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


def _weights(rng, rows, cols, dtype, kind="t3"):
    w = synth.random_matrix(rng, rows, cols, kind)
    return synth.to_bf16_bits(w).reshape(rows, cols) if dtype == "bf16" else w


def _run(gq, w_np, avg_np, qbits, p, kind, count=0, decay=0.997, per_tensor=False, want_dq=False,
         mode=0, w_dev=None, avg_dev=None):
    W = to_dev(w_np) if w_dev is None else w_dev
    A = torch.from_numpy(avg_np.copy()).cuda() if avg_dev is None else avg_dev
    r = gq.Request(W, qbits, p, per_tensor, want_dq=want_dq, want_scale_f32=True)
    (o,) = gq.fakequant_average([r], [A], kind=kind, count=count, decay=decay, mode=mode)
    torch.cuda.synchronize()
    ref, want = oracle.fakequant_average(w_np, avg_np, qbits, p, kind, count=count, decay=decay,
                                         per_tensor=per_tensor, export=mode == 1)
    return o, A, ref, want


def _check(o, A, ref, want, what, want_dq=False):
    assert o.status == 0, (what, o.status)
    assert ref.status == oracle.OR_OK
    assert_same(to_host(A).reshape(want.shape), want, f"{what}: average")
    assert_same(to_host(o.scale_f32), ref.scale_f32, f"{what}: scale")
    if want_dq:
        assert_same(to_host(o.dq), ref.dq, f"{what}: w_hat")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(300, 512), (64, 4096), (9, 16384), (37, 1000)])
def test_average_matches_oracle(gq, dtype, rows, cols):
    rng = np.random.default_rng(rows + cols + (dtype == "bf16"))
    w = _weights(rng, rows, cols, dtype)
    stale = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    # weights 1, 1/2, 1/3 and 1/7 (the last two inexact in binary32)
    for kind, count, decay in ((gq.GQ_AVG_MEAN, 0, 0.0), (gq.GQ_AVG_MEAN, 1, 0.0),
                               (gq.GQ_AVG_MEAN, 2, 0.0), (gq.GQ_AVG_MEAN, 6, 0.0),
                               (gq.GQ_AVG_EMA, 0, 0.997), (gq.GQ_AVG_EMA, 0, 0.5)):
        for want_dq in (False, True):
            for qbits, p in ((6, 0.9999), (8, 1.0)):
                o, A, ref, want = _run(gq, w, stale, qbits, p, kind, count, decay, want_dq=want_dq)
                _check(o, A, ref, want, f"{dtype} {rows}x{cols} k{kind} n{count} d{decay} "
                                        f"dq{want_dq} q{qbits}", want_dq)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_average_generic_and_fallback_paths(gq, dtype):
    rng = np.random.default_rng(11 + (dtype == "bf16"))
    rows, cols = 96, 768
    w = _weights(rng, rows, cols, dtype)
    w[5] = 0                                       # a zero-scale row (generic loop)
    stale = rng.standard_normal((rows, cols)).astype(np.float32)
    # an average that is only 4-byte aligned: the generic loop of the fused kernel
    flat = torch.empty(rows * cols + 1, dtype=torch.float32, device="cuda")
    A = flat[1:].view(rows, cols)
    A.copy_(torch.from_numpy(stale))
    o, A, ref, want = _run(gq, w, stale, 6, 0.999, gq.GQ_AVG_MEAN, 3, avg_dev=A, want_dq=True)
    _check(o, A, ref, want, f"{dtype} 4-byte aligned average", True)
    # a weight base that is not 16-byte aligned: the fallback kernel
    Wt = to_dev(np.concatenate([np.zeros(8, w.dtype), w.ravel()]))
    Wv = Wt[1:1 + rows * cols].view(rows, cols)
    w_np = to_host(Wv)
    o, A, ref, want = _run(gq, w_np, stale, 8, 0.99, gq.GQ_AVG_EMA, 0, 0.997, w_dev=Wv, want_dq=True)
    _check(o, A, ref, want, f"{dtype} misaligned weight (fallback kernel)", True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_average_per_tensor_and_f16_mode(gq, dtype):
    rng = np.random.default_rng(23 + (dtype == "bf16"))
    w = _weights(rng, 256, 512, dtype, "mix")
    stale = rng.standard_normal((256, 512)).astype(np.float32)
    o, A, ref, want = _run(gq, w, stale, 6, 0.999, gq.GQ_AVG_MEAN, 2, per_tensor=True, want_dq=True)
    _check(o, A, ref, want, f"{dtype} per-tensor", True)
    o, A, ref, want = _run(gq, w, stale, 6, 0.9999, gq.GQ_AVG_EMA, 0, 0.997, mode=1, want_dq=True)
    _check(o, A, ref, want, f"{dtype} binary16 scales", True)


def test_average_sequence_of_snapshots(gq):
    """A short training run: the weights drift, the mean and the EMA follow
    the fake-quant snapshots, and every step stays bit-exact."""
    rng = np.random.default_rng(5)
    w = synth.random_matrix(rng, 128, 1536, "normal")
    mean = np.zeros_like(w)
    ema = np.zeros_like(w)
    Am = torch.zeros(128, 1536, device="cuda")
    Ae = torch.zeros(128, 1536, device="cuda")
    W = to_dev(w)
    for step in range(6):
        r = gq.Request(W, 6, 0.9999, want_dq=False)
        gq.fakequant_average([r], [Am], kind=gq.GQ_AVG_MEAN, count=step)
        r = gq.Request(W, 6, 0.9999, want_dq=False)
        gq.fakequant_average([r], [Ae], kind=gq.GQ_AVG_EMA, decay=0.997)
        ref = oracle.quantize(w, 6, 0.9999, export=False)
        mean = oracle.average_update(mean, ref.dq, oracle.AVG_MEAN, count=step)
        ema = oracle.average_update(ema, ref.dq, oracle.AVG_EMA, decay=0.997)
        torch.cuda.synchronize()
        assert_same(to_host(Am), mean, f"mean after {step + 1} snapshots")
        assert_same(to_host(Ae), ema, f"EMA after {step + 1} snapshots")
        w = (w + (rng.standard_normal(w.shape) * 2e-3).astype(np.float32)).astype(np.float32)
        W.copy_(torch.from_numpy(w))


def test_average_argument_errors(gq):
    W = torch.ones(4, 8, device="cuda")
    A = torch.zeros(4, 8, device="cuda")
    d = gq.GQTensor(w=W.data_ptr(), dtype=0, qbits=6, gran=0, reserved=0, rows=4, cols=8, ld=8, p=1.0,
                    dq=0, codes=0, packed=0, scale_f16=0, scale_f32=0, clip=0)
    ok = gq.GQAvg(avg=A.data_ptr(), kind=0, decay=0.0, count=0)
    gq.gq_fakequant_average([d], [ok], 0)
    for bad, code in ((dict(kind=2), 1), (dict(kind=1, decay=1.5), 1), (dict(count=-1), 1),
                      (dict(count=1 << 24), 1), (dict(avg=0), 1), (dict(avg=A.data_ptr() + 2), 3)):
        a = gq.GQAvg(avg=A.data_ptr(), kind=0, decay=0.0, count=0)
        for k, v in bad.items():
            setattr(a, k, v)
        with pytest.raises(gq.GQError) as e:
            gq.gq_fakequant_average([d], [a], 0)
        assert e.value.status == code, bad
    codes = torch.empty(4, 8, dtype=torch.int8, device="cuda")
    d.codes = codes.data_ptr()
    with pytest.raises(gq.GQError):
        gq.gq_fakequant_average([d], [ok], 0)
