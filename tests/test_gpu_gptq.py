"""GPU parity of GPTQ-lite (gq_gptq_hessian, gq_gptq_quantize) against the
CPU oracle (oracle/gptq.py), called through the C ABI.

Both sides work in binary64 but not in the same order (the library factors
the reversed Hessian and runs a left-looking recurrence; the oracle inverts H
and feeds errors forward in lazy batches), so a code can legitimately differ
only where its quotient sits on a rounding boundary to within the binary64
noise of the two orders.  The tolerance written here: every binary16 scale
equal; every code equal, except that a row may differ from its first
mismatch on if the oracle's quotient there is within 1e-6 of a half-integer,
and at most 1 % of the rows may do so (none does on these inputs).  The
packed bytes and w_hat must be exactly those of the library's own codes.
The Hessian itself is compared to relative 1e-12.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import gptq as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int6_int8_weight_b200 import gq as mod
    return mod


def _host(t):
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_against_oracle(gq, w, x, qbits, p, percdamp=0.01, what=""):
    W, X = _dev(w), _dev(x)
    H = gq.gptq_hessian(X)
    H_ref = G.hessian(x)
    H_got = H.cpu().numpy()
    scale = np.abs(H_ref).max() + 1e-300
    assert np.abs(H_got - H_ref).max() <= 1e-12 * scale, what + " hessian"
    o = gq.gptq_quantize(gq.Request(W, qbits, p, want_dq=True, want_codes=True, want_clip=True), H, percdamp)
    torch.cuda.synchronize()
    assert o.status == 0, (what, o.status)
    ref = G.gptq(w, H_ref, qbits, p, percdamp=percdamp)
    assert ref.status == 0
    assert np.array_equal(_host(o.scale_f16), ref.scale_f16), what + " scales"
    codes = _host(o.codes)
    bad_rows = np.nonzero((codes != ref.codes).any(axis=1))[0]
    for r in bad_rows:
        j = int(np.nonzero(codes[r] != ref.codes[r])[0][0])
        t = ref.quotient[r, j]
        assert abs(abs(t - np.floor(t)) - 0.5) < 1e-6, (what, "code mismatch off a tie", r, j, t,
                                                        int(codes[r, j]), int(ref.codes[r, j]))
    assert len(bad_rows) <= max(1, w.shape[0] // 100), (what, len(bad_rows))
    # outputs of the library's own codes
    s = oracle.f16_bits_to_f32(_host(o.scale_f16))
    dq32 = (codes * s[:, None]).astype(np.float32)
    dq32[codes == 0] = 0.0
    want_dq = oracle.f32_to_bf16_bits(dq32).reshape(codes.shape) if w.dtype == np.uint16 else dq32
    got_dq = _host(o.dq)
    assert np.array_equal(got_dq.view(np.uint32) if got_dq.dtype == np.float32 else got_dq,
                          want_dq.view(np.uint32) if want_dq.dtype == np.float32 else want_dq), what + " dq"
    packed = _host(o.packed)
    if qbits == 6:
        for r in range(codes.shape[0]):
            assert np.array_equal(packed[r], oracle.pack6_row(codes[r])), (what, r)
    else:
        assert np.array_equal(packed.view(np.int8), codes), what
    base = oracle.quantize(w, qbits, p, export=True)
    assert np.array_equal(_host(o.clip).view(np.uint32), base.clip.view(np.uint32)), what + " clip"
    return o, ref


CASES = [
    # rows, cols, dtype, qbits, p, n calibration rows
    (96, 200, "f32", 6, 1.0, 512),
    (33, 64, "f32", 8, 1.0, 256),
    (130, 517, "bf16", 6, 0.999, 700),     # ragged: rows % 4, cols % 64
    (256, 528, "bf16", 6, 1.0, 1024),      # the 11-layer model's width
    (40, 1584, "f32", 6, 0.9999, 2048),    # its MLP-down input width
    (17, 130, "f32", 8, 0.9, 100),
]


@pytest.mark.parametrize("rows,cols,dtype,qbits,p,n", CASES)
def test_gptq_matches_oracle(gq, rows, cols, dtype, qbits, p, n):
    rng = np.random.default_rng(rows * 7 + cols)
    w = synth.random_matrix(rng, rows, cols, "t3")
    if dtype == "bf16":
        w = synth.to_bf16_bits(w).reshape(rows, cols)
    x = synth.gptq_calibration(rng, n, cols)
    check_against_oracle(gq, w, x, qbits, p, what=f"{rows}x{cols} {dtype} int{qbits} p{p}")


def test_gptq_dead_input_and_no_damping(gq):
    rng = np.random.default_rng(5)
    w = synth.random_matrix(rng, 24, 96, "t3")
    x = synth.gptq_calibration(rng, 300, 96, dead=(0, 17, 95))
    o, _ = check_against_oracle(gq, w, x, 6, 1.0, what="dead inputs")
    assert (_host(o.codes)[:, [0, 17, 95]] == 0).all()
    x2 = synth.gptq_calibration(rng, 400, 96)
    check_against_oracle(gq, w, x2, 6, 1.0, percdamp=0.0, what="no damping")


def test_gptq_diagonal_hessian_is_plain_export(gq):
    """A Hessian without coupling leaves nothing to feed forward: the codes are
    those of gq_export_pack (the same binary16 scales, round half to even)."""
    rng = np.random.default_rng(6)
    w = synth.random_matrix(rng, 64, 256, "mix")
    W = _dev(w)
    H = torch.diag(torch.from_numpy(rng.uniform(0.5, 2.0, 256))).cuda()
    o = gq.gptq_quantize(gq.Request(W, 6, 0.999, want_dq=True, want_codes=True), H)
    (e,) = gq.export_pack([gq.Request(W, 6, 0.999, want_dq=True, want_codes=True, want_packed=True,
                                      want_scale_f16=True)])
    torch.cuda.synchronize()
    assert torch.equal(o.codes, e.codes) and torch.equal(o.packed, e.packed)
    assert torch.equal(o.scale_f16.view(torch.int16), e.scale_f16.view(torch.int16))


def test_gptq_unified11_model(gq):
    """All 44 weights of the 11-layer d528 model (bf16), each against the
    Hessian of its own synthetic inputs."""
    ws = synth.draw_unified11()
    specs = synth.unified11_train().specs
    rng = np.random.default_rng(21)
    oracle.default()
    for i, s in enumerate(specs):
        if i % 4 and i > 8:            # every layer's first weight, and all of the first two layers
            continue
        x = synth.gptq_calibration(rng, 512, s.shape[1])
        check_against_oracle(gq, ws[s.name], x, 6, 1.0, what=s.name)


def test_gptq_argument_errors(gq):
    W = torch.zeros(8, 16, device="cuda")
    H = torch.eye(16, dtype=torch.float64, device="cuda")
    with pytest.raises(ValueError):
        gq.gptq_quantize(gq.Request(W, 6, 1.0, per_tensor=True), H)
    with pytest.raises(ValueError):
        gq.gptq_quantize(gq.Request(W, 6, 1.0), H[:8, :8].contiguous())
    d = gq.GQTensor(w=W.data_ptr(), dtype=0, qbits=6, gran=0, reserved=0, rows=8, cols=16, ld=16, p=1.0,
                    dq=0, codes=0, packed=W.data_ptr(), scale_f16=W.data_ptr(), scale_f32=0, clip=0)
    import ctypes as C
    assert gq.LIB.gq_gptq_quantize(C.byref(d), H.data_ptr(), 0.01, None, 0, None, None) == 4   # no workspace
    assert gq.LIB.gq_gptq_quantize(C.byref(d), H.data_ptr(), -1.0, None, 0, None, None) == 1   # bad percdamp
    d.cols = 6000
    d.ld = 6000
    assert gq.LIB.gq_gptq_quantize(C.byref(d), H.data_ptr(), 0.01, None, 0, None, None) == 2   # too wide


def test_gptq_batch_equals_single_calls(gq):
    """gq_gptq_quantize_batch over weights of different shapes, dtypes and
    bit widths gives, bitwise, the outputs of one gq_gptq_quantize per
    weight (whose parity with the oracle the tests above check)."""
    rng = np.random.default_rng(44)
    shapes = [(96, 200, "f32", 6, 1.0), (130, 517, "bf16", 6, 0.999), (40, 1584, "f32", 6, 0.9999),
              (33, 64, "f32", 8, 1.0), (256, 528, "bf16", 6, 1.0)]
    reqs, Hs = [], []
    for rows, cols, dt, qbits, p in shapes:
        w = synth.random_matrix(rng, rows, cols, "t3")
        if dt == "bf16":
            w = synth.to_bf16_bits(w).reshape(rows, cols)
        reqs.append(gq.Request(_dev(w), qbits, p, want_dq=True, want_codes=True, want_clip=True))
        Hs.append(gq.gptq_hessian(_dev(synth.gptq_calibration(rng, 300, cols))))
    outs = gq.gptq_quantize_batch(reqs, Hs)
    for r, H, o in zip(reqs, Hs, outs):
        one = gq.gptq_quantize(gq.Request(r.w, r.qbits, r.p, want_dq=True, want_codes=True, want_clip=True), H)
        torch.cuda.synchronize()
        assert o.status == 0 and one.status == 0
        assert torch.equal(o.codes, one.codes) and torch.equal(o.packed, one.packed)
        assert torch.equal(o.scale_f16.view(torch.int16), one.scale_f16.view(torch.int16))
        assert torch.equal(o.dq.view(torch.int16) if o.dq.dtype == torch.bfloat16 else o.dq.view(torch.int32),
                           one.dq.view(torch.int16) if one.dq.dtype == torch.bfloat16 else one.dq.view(torch.int32))
        assert torch.equal(o.clip.view(torch.int32), one.clip.view(torch.int32))


def test_gptq_batch_unified11_model(gq):
    """All 44 weights of the 11-layer d528 model in one batched call: each
    equal to its single call, and the first layer's four against the oracle."""
    ws = synth.draw_unified11()
    specs = synth.unified11_train().specs
    rng = np.random.default_rng(22)
    xs = [synth.gptq_calibration(rng, 512, s.shape[1]) for s in specs]
    reqs = [gq.Request(_dev(ws[s.name]), 6, 1.0, want_dq=True, want_codes=True) for s in specs]
    Hs = [gq.gptq_hessian(_dev(x)) for x in xs]
    outs = gq.gptq_quantize_batch(reqs, Hs)
    for i, (s, r, H, o) in enumerate(zip(specs, reqs, Hs, outs)):
        assert o.status == 0, s.name
        if i % 7 == 0:
            one = gq.gptq_quantize(gq.Request(r.w, 6, 1.0, want_dq=True, want_codes=True), H)
            torch.cuda.synchronize()
            assert torch.equal(o.codes, one.codes) and torch.equal(o.packed, one.packed), s.name
    for i in range(4):
        ref = G.gptq(ws[specs[i].name], G.hessian(xs[i]), 6, 1.0)
        codes = _host(outs[i].codes)
        bad = np.nonzero((codes != ref.codes).any(axis=1))[0]
        for r in bad:
            j = int(np.nonzero(codes[r] != ref.codes[r])[0][0])
            t = ref.quotient[r, j]
            assert abs(abs(t - np.floor(t)) - 0.5) < 1e-6, (specs[i].name, r, j, t)
        assert len(bad) <= max(1, codes.shape[0] // 100)


def test_gptq_batch_argument_errors(gq):
    import ctypes as C
    W = torch.zeros(8, 16, device="cuda")
    H = torch.eye(16, dtype=torch.float64, device="cuda")
    d = gq.GQTensor(w=W.data_ptr(), dtype=0, qbits=6, gran=0, reserved=0, rows=8, cols=16, ld=16, p=1.0,
                    dq=0, codes=0, packed=W.data_ptr(), scale_f16=W.data_ptr(), scale_f32=0, clip=0)
    arr = gq._arr([d, d])
    hp = (C.c_void_p * 2)(H.data_ptr(), H.data_ptr())
    L = gq.LIB
    assert L.gq_gptq_batch_workspace_size(arr, 2) == 2 * L.gq_gptq_workspace_size(8, 16)
    assert L.gq_gptq_quantize_batch(arr, 2, hp, 0.01, None, 0, None, None) == 4        # no workspace
    assert L.gq_gptq_quantize_batch(arr, 2, None, 0.01, None, 0, None, None) == 1      # no Hessians
    assert L.gq_gptq_quantize_batch(arr, 2, hp, -1.0, None, 0, None, None) == 1        # bad percdamp
    assert L.gq_gptq_quantize_batch(arr, 0, hp, 0.01, None, 0, None, None) == 0        # nothing to do
