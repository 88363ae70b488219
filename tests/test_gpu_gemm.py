"""GPU parity of the consuming GEMMs against the oracle: gq_gemm_dequant (the
weight rebuilt from packed codes) and gq_gemm_fakequant (fake-quantized from
fp32 / bf16 weights and row clips in the weight load).

Y = X @ W_hat^T where W_hat[n, k] = bf16(RN(q[n, k] * s[n])) comes from the
packed codes and binary16 scales.  The reference is oracle/gemm.py: W_hat
from the C oracle's dequant and the contraction in binary64 (whole matrices)
or exactly rounded (sampled entries of the full-size shapes).  Inputs are
seeded: small weights exported by the oracle, or, at full size, arbitrary
packed code bytes and binary16 scales from the input generator.

Tolerance.  Every product of two bf16 values is exact in binary32; the tensor
cores add them in binary32 in their own order: K/16 MMA steps (each at most
2^-23 relative, allowing truncation), two accumulators joined by one
addition for small token tiles, and, when a tile's K range is split over
blocks, at most a few partial sums added into Y.  So
    |Y - exact| <= (K/8 + 16) * 2^-24 * sum_k |X * W_hat|,
checked element by element (the binary64 reference's own error, at most
K * 2^-53 of the same sum, is added to the bound).

Every call also passes a status word, which must stay 0 (no expired wait),
and the columns of Y past N (a row pitch wider than N) must stay untouched.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import gemm as GM

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int6_int8_weight_b200 import gq as mod
    return mod


def _bound(K, abs_sum):
    return ((K / 8 + 16) * 2.0 ** -24 + K * 2.0 ** -53) * abs_sum


def _run(gq, x, packed, scale, qbits, N, K):
    M = x.shape[0]
    X = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
    P = torch.from_numpy(packed).cuda()
    S = torch.from_numpy(scale.view(np.int16).copy()).cuda().view(torch.float16)
    ldy = N + 3                          # a pitch wider than N: the padding must stay untouched
    Ypad = torch.full((M, ldy), 7.0, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = gq.LIB.gq_gemm_dequant(X.data_ptr(), M, K, K, P.data_ptr(), S.data_ptr(), qbits, N,
                                Ypad.data_ptr(), ldy, st.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 0 and int(st[0]) == 0, (rc, int(st[0]))
    assert bool((Ypad[:, N:] == 7.0).all())
    return Ypad[:, :N]


def _x(rng, M, K):
    return synth.to_bf16_bits((rng.standard_normal((M, K)) * 0.5).astype(np.float32)).reshape(M, K)


def _case(gq, M, N, K, qbits, seed, p=0.9999):
    rng = np.random.default_rng(seed)
    ref = oracle.quantize(synth.random_matrix(rng, N, K, "t3"), qbits, p, export=True)
    assert ref.status == oracle.OR_OK
    x = _x(rng, M, K)
    Y = _run(gq, x, ref.packed, ref.scale_f16, qbits, N, K)
    y_ref, a = GM.contraction(x, GM.w_hat_bf16(ref.packed, ref.scale_f16, qbits, N, K))
    got = Y.cpu().numpy().astype(np.float64)
    bad = np.argwhere(np.abs(got - y_ref) > _bound(K, a))
    assert bad.size == 0, (f"M{M} N{N} K{K} q{qbits}: {len(bad)} outside the bound, first {tuple(bad[0])}: "
                           f"got {got[tuple(bad[0])]!r} want {y_ref[tuple(bad[0])]!r}")


@pytest.mark.parametrize("qbits", [6, 8])
@pytest.mark.parametrize("M,N,K", [
    (128, 128, 64),       # one tile, one K stage
    (128, 256, 512),      # two weight tiles, eight K stages
    (1, 128, 64),         # a single token (a 16-token tile, TMA zero-fills the rest)
    (77, 300, 1024),      # ragged M and N
    (5, 130, 576),        # N % 4 == 2
    (64, 512, 8192),      # long K: a tile's K range split over blocks
    (300, 384, 2048),     # two 256-token tiles
    (33, 256, 1024),      # a 64-token tile, 31 of them padding
    (257, 128, 512),      # one token past a single 256-token tile
    (96, 1584, 528),      # the 11-layer model: K = 528 (int6 rows of 396 bytes: 4-byte copies)
    (40, 528, 1584),      # its MLP-down input: K = 1584 (int6 rows of 1188 bytes)
    (16, 256, 16),        # a single 16-wide K step (the rest of the stage zero-filled)
])
def test_gemm_dequant_matches_oracle(gq, M, N, K, qbits):
    _case(gq, M, N, K, qbits, seed=M * 7 + N + K + qbits)


@pytest.mark.parametrize("qbits", [6, 8])
def test_gemm_dequant_whole_tile_mode(gq, qbits):
    """Enough tiles for every block to take whole tiles (plain stores)."""
    _case(gq, 1024, 16384, 256, qbits, seed=77 + qbits)


@pytest.mark.parametrize("M,N,K", [(16, 16384, 16384), (128, 16384, 16384), (4096, 8192, 8192)])
def test_gemm_dequant_benchmark_shapes_sampled(gq, M, N, K):
    """The shapes the benchmark times, at full size, in the launch
    configuration it times: 1024 sampled entries (and the four corners)
    against exactly rounded sums."""
    qbits = 6
    rng = np.random.default_rng(M + N + K)
    prb = 3 * ((K + 3) // 4)
    packed = synth.random_packed_codes(rng, N, prb)
    scale = synth.random_f16_scales(rng, N)
    x = _x(rng, M, K)
    Y = _run(gq, x, packed, scale, qbits, N, K)
    ms = np.concatenate([[0, M - 1, 0, M - 1], rng.integers(0, M, 1024)])
    ns = np.concatenate([[0, 0, N - 1, N - 1], rng.integers(0, N, 1024)])
    rows = np.unique(ns)
    w = GM.w_hat_bf16(packed[rows], scale[rows], qbits, len(rows), K)
    where = {int(n): i for i, n in enumerate(rows)}
    ye, a = GM.contraction_exact(x, w, [(int(m), where[int(n)]) for m, n in zip(ms, ns)])
    got = Y.cpu().numpy().astype(np.float64)[ms, ns]
    bad = np.nonzero(np.abs(got - ye) > _bound(K, a))[0]
    assert bad.size == 0, (M, N, K, len(bad), int(ms[bad[0]]), int(ns[bad[0]]), got[bad[0]], ye[bad[0]])


def test_gemm_dequant_errors(gq):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros(8, 48, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(8, dtype=torch.float16, device="cuda")
    Y = torch.empty(4, 8, device="cuda")
    L = gq.LIB
    args = [X.data_ptr(), 4, 64, 64, packed.data_ptr(), scale.data_ptr(), 6, 8, Y.data_ptr(), 8, None, None]
    assert L.gq_gemm_dequant(*args) == 0
    bad = list(args); bad[6] = 7                          # qbits
    assert L.gq_gemm_dequant(*bad) == 1
    bad = list(args); bad[2] = 50; bad[3] = 56            # int6 rows of 39 bytes: neither TMA nor 4-byte copies
    assert L.gq_gemm_dequant(*bad) == 2
    bad = list(args); bad[0] = X.data_ptr() + 2           # misaligned activations
    assert L.gq_gemm_dequant(*bad) == 3
    bad = list(args); bad[2] = 48; bad[3] = 52            # activation pitch not a multiple of 8
    assert L.gq_gemm_dequant(*bad) == 3
    bad = list(args); bad[9] = 6                          # ldy < N
    assert L.gq_gemm_dequant(*bad) == 1
    empty = list(args); empty[1] = 0                      # M = 0: nothing to do
    assert L.gq_gemm_dequant(*empty) == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("qbits", [6, 8])
def test_gemm_dequant_fresh_inputs(gq, qbits):
    """Shapes whose rings wrap, each run on three fresh allocations."""
    for M, N, K in ((128, 256, 512), (256, 256, 512), (300, 384, 2048), (16, 512, 4096)):
        for rep in range(3):
            _case(gq, M, N, K, qbits, seed=1000 * rep + M + N + K + qbits)


@pytest.mark.parametrize("wdt", ["f32", "bf16"])
@pytest.mark.parametrize("M,N,K,qbits,mode,p", [
    (16, 1584, 528, 6, 0, 1.0),       # the 11-layer model's unified projection, training scales
    (64, 528, 1584, 6, 0, 1.0),       # its MLP down projection
    (100, 256, 1000, 8, 1, 0.999),    # binary16 scales, percentile clip, ragged K
    (300, 384, 2048, 6, 1, 0.9999),   # two 256-token tiles
    (1, 128, 40, 6, 0, 1.0),          # K shorter than a stage
    (1024, 16384, 128, 6, 0, 1.0),    # whole tiles
])
def test_gemm_fakequant_matches_oracle(gq, wdt, M, N, K, qbits, mode, p):
    """W_hat is the fake-quant output of gq_fakequant_fwd for the same weight
    (rounded to bf16 for fp32 weights); the clips come from the library's own
    select and must equal the oracle's."""
    rng = np.random.default_rng(M + N + K + qbits)
    w = synth.random_matrix(rng, N, K, "t3")
    if wdt == "bf16":
        w = synth.to_bf16_bits(w).reshape(N, K)
        W = torch.from_numpy(w.view(np.int16).copy()).cuda().view(torch.bfloat16)
    else:
        W = torch.from_numpy(w).cuda()
    (c,) = gq.row_clip_select([gq.Request(W, qbits, p)])
    x = _x(rng, M, K)
    X = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
    ldy = N + 1
    Ypad = torch.full((M, ldy), 7.0, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = gq.LIB.gq_gemm_fakequant(X.data_ptr(), M, K, K, W.data_ptr(), 1 if wdt == "bf16" else 0, K,
                                  c.clip.data_ptr(), qbits, mode, N, Ypad.data_ptr(), ldy, st.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 0 and int(st[0]) == 0, (rc, int(st[0]))
    assert bool((Ypad[:, N:] == 7.0).all())
    ref = oracle.quantize(w, qbits, p, export=mode == 1)
    assert ref.status == oracle.OR_OK
    assert np.array_equal(c.clip.cpu().numpy().view(np.uint32), ref.clip.view(np.uint32))
    w_hat = ref.dq if wdt == "bf16" else oracle.f32_to_bf16_bits(ref.dq).reshape(N, K)
    y_ref, a = GM.contraction(x, w_hat)
    got = Ypad[:, :N].cpu().numpy().astype(np.float64)
    bad = np.argwhere(np.abs(got - y_ref) > _bound(K, a))
    assert bad.size == 0, (f"{wdt} M{M} N{N} K{K}: {len(bad)} outside the bound, first {tuple(bad[0])}: "
                           f"got {got[tuple(bad[0])]!r} want {y_ref[tuple(bad[0])]!r}")


def test_gemm_fakequant_errors(gq):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(8, 64, device="cuda")
    clip = torch.ones(8, device="cuda")
    Y = torch.empty(4, 8, device="cuda")
    L = gq.LIB
    args = [X.data_ptr(), 4, 64, 64, W.data_ptr(), 0, 64, clip.data_ptr(), 6, 0, 8, Y.data_ptr(), 8, None, None]
    assert L.gq_gemm_fakequant(*args) == 0
    bad = list(args); bad[5] = 3                          # weight dtype
    assert L.gq_gemm_fakequant(*bad) == 1
    bad = list(args); bad[9] = 2                          # scale mode
    assert L.gq_gemm_fakequant(*bad) == 1
    bad = list(args); bad[6] = 62                         # weight pitch: not a multiple of 16 bytes
    assert L.gq_gemm_fakequant(*bad) in (1, 3)
    bad = list(args); bad[7] = None                       # no clips
    assert L.gq_gemm_fakequant(*bad) == 1
    torch.cuda.synchronize()


# Decode-sized batches (M <= 16) take the register-level kernel
# (gq_gemm_decode.cuh): units of 256 weight rows x 512 of K, K permuted alike
# in X and W_hat inside each 64-wide stage, partial sums added into Y.
@pytest.mark.parametrize("qbits", [6, 8])
@pytest.mark.parametrize("M,N,K", [
    (1, 8, 64),           # one 8-row column group, one stage
    (2, 1000, 512),       # ragged row block, one K unit
    (7, 257, 1024),       # one row past a row block
    (9, 4104, 2048),      # N % 256 = 8
    (15, 300, 528),       # K past the first unit by 16 (a short last stage)
    (16, 1584, 528),      # the 11-layer model's unified projection
    (16, 528, 1584),      # its MLP-down projection
    (3, 100, 16),         # a single 16-wide slice of a stage
    (16, 2048, 5120),     # ten K units per row block
])
def test_gemm_decode_matches_oracle(gq, M, N, K, qbits):
    _case(gq, M, N, K, qbits, seed=M * 11 + N + K + qbits)


@pytest.mark.parametrize("M", [16, 5])
def test_gemm_decode_unit_runs_sampled(gq, M):
    """Many units per block, whose runs cross row blocks (flushes in the
    middle of a run): sampled entries against exactly rounded sums."""
    N, K, qbits = 8192, 16384, 6
    rng = np.random.default_rng(M + 5)
    prb = 3 * ((K + 3) // 4)
    packed = synth.random_packed_codes(rng, N, prb)
    scale = synth.random_f16_scales(rng, N)
    x = _x(rng, M, K)
    Y = _run(gq, x, packed, scale, qbits, N, K)
    ms = np.concatenate([[0, M - 1, 0, M - 1], rng.integers(0, M, 2048)])
    ns = np.concatenate([[0, 0, N - 1, N - 1], rng.integers(0, N, 2048)])
    rows = np.unique(ns)
    w = GM.w_hat_bf16(packed[rows], scale[rows], qbits, len(rows), K)
    where = {int(n): i for i, n in enumerate(rows)}
    ye, a = GM.contraction_exact(x, w, [(int(m), where[int(n)]) for m, n in zip(ms, ns)])
    got = Y.cpu().numpy().astype(np.float64)[ms, ns]
    bad = np.nonzero(np.abs(got - ye) > _bound(K, a))[0]
    assert bad.size == 0, (M, len(bad), int(ms[bad[0]]), int(ns[bad[0]]), got[bad[0]], ye[bad[0]])


def test_gemm_decode_activation_pitch(gq):
    """X rows wider than K (ldx = K + 24): only the first K columns count."""
    M, N, K, qbits = 12, 640, 1024, 6
    rng = np.random.default_rng(9)
    ref = oracle.quantize(synth.random_matrix(rng, N, K, "t3"), qbits, 1.0, export=True)
    xw = _x(rng, M, K + 24)
    X = torch.from_numpy(xw.view(np.int16).copy()).cuda().view(torch.bfloat16)
    P = torch.from_numpy(ref.packed).cuda()
    S = torch.from_numpy(ref.scale_f16.view(np.int16).copy()).cuda().view(torch.float16)
    Y = torch.empty(M, N, device="cuda")
    assert gq.LIB.gq_gemm_dequant(X.data_ptr(), M, K, K + 24, P.data_ptr(), S.data_ptr(), qbits, N,
                                  Y.data_ptr(), N, None, None) == 0
    torch.cuda.synchronize()
    y_ref, a = GM.contraction(np.ascontiguousarray(xw[:, :K]), GM.w_hat_bf16(ref.packed, ref.scale_f16, qbits, N, K))
    got = Y.cpu().numpy().astype(np.float64)
    assert (np.abs(got - y_ref) <= _bound(K, a)).all()
