"""GPU parity of the dequant-on-load GEMM (gq_gemm_dequant) against the oracle.

Y = X @ W_hat^T where W_hat[n, k] = bf16(RN(q[n, k] * s[n])) comes from the
packed codes and binary16 scales of an export.  The inputs are made on the
CPU: the oracle exports a random weight (codes, scales) and dequantizes it to
bf16 (W_hat); X is random bf16.  The reference is the exact product sum in
float64 of those bf16 values.

Tolerance.  Every product of two bf16 values is exact in binary32; the tensor
cores add them in binary32 in their own order: 16 products per instruction
(relative error at most 2^-23 for that partial sum) and K/16 accumulations in
all (each at most 2^-23 relative, allowing truncation), spread over two
accumulators that one final binary32 addition joins.  So
    |Y - exact| <= (K/16 * 2^-23 + 2 * 2^-23) * sum_k |X * W_hat|
                 = (K/8 + 4) * 2^-24 * sum_k |X * W_hat|,
the bound of the header, which the test checks element by element.

Every call also passes a status word, which must stay 0 (no expired wait),
and one test repeats shapes on freshly allocated inputs: a race between the
code loads and the refill of their ring slot showed only there (cold caches
on the first call).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int6_int8_weight_b200 import gq as mod
    return mod


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(gq, M, N, K, qbits, seed, p=0.9999):
    rng = np.random.default_rng(seed)
    w = synth.random_matrix(rng, N, K, "t3")
    ref = oracle.quantize(w, qbits, p, export=True)
    assert ref.status == oracle.OR_OK
    w_hat = oracle.dequant(ref.packed, ref.scale_f16, qbits, N, K, out_bf16=True)   # bf16 bits [N, K]
    x = synth.to_bf16_bits((rng.standard_normal((M, K)) * 0.5).astype(np.float32)).reshape(M, K)
    X = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
    packed = torch.from_numpy(ref.packed).cuda()
    scale = torch.from_numpy(ref.scale_f16.view(np.int16).copy()).cuda().view(torch.float16)
    # Y rows padded to a multiple of 4 floats (16-byte aligned rows); the
    # padding must stay untouched
    ldy = (N + 3) // 4 * 4
    Ypad = torch.full((M, ldy), 7.0, device="cuda")
    Y = Ypad[:, :N]
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = gq.LIB.gq_gemm_dequant(X.data_ptr(), M, K, K, packed.data_ptr(), scale.data_ptr(), qbits, N,
                                Y.data_ptr(), ldy, st.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == 0 and int(st[0]) == 0, (rc, int(st[0]))
    assert bool((Ypad[:, N:] == 7.0).all())
    xf, wf = _bf16_to_f64(x), _bf16_to_f64(w_hat)
    exact = xf @ wf.T
    bound = (K / 8 + 4) * 2.0 ** -24 * (np.abs(xf) @ np.abs(wf).T)
    got = Y.cpu().numpy().astype(np.float64)
    err = np.abs(got - exact)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (f"M{M} N{N} K{K} q{qbits}: {len(bad)} outside the bound, first {tuple(bad[0])}: "
                           f"got {got[tuple(bad[0])]!r} exact {exact[tuple(bad[0])]!r} bound {bound[tuple(bad[0])]!r}")
    return err, bound


@pytest.mark.parametrize("qbits", [6, 8])
@pytest.mark.parametrize("M,N,K", [
    (128, 128, 64),       # one tile, one K step (M <= 128: swapped operands, 128 tokens)
    (128, 256, 512),      # two N tiles, eight K steps (a full ring and more)
    (1, 128, 64),         # a single activation row (a 16-token tile, TMA zero-fills the rest)
    (77, 300, 1024),      # ragged M and N (partial tiles, N % 4 == 0)
    (5, 130, 576),        # N % 4 == 2: the scalar tail columns
    (64, 512, 8192),      # small M, long K: split K with vector atomics
    (300, 384, 2048),     # several M tiles
    (33, 256, 1024),      # swapped operands with a 64-token tile, 31 of them padding
    (129, 128, 512),      # one token past the swapped range: the 128 x 128 form, ragged
])
def test_gemm_dequant_matches_exact_sum(gq, M, N, K, qbits):
    _case(gq, M, N, K, qbits, seed=M * 7 + N + K + qbits)


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
    bad = list(args); bad[2] = 48; bad[3] = 48            # K not a multiple of 64
    assert L.gq_gemm_dequant(*bad) == 2
    bad = list(args); bad[0] = X.data_ptr() + 2           # misaligned activations
    assert L.gq_gemm_dequant(*bad) == 3
    bad = list(args); bad[9] = 6                          # ldy < N
    assert L.gq_gemm_dequant(*bad) == 1
    empty = list(args); empty[1] = 0                      # M = 0: nothing to do
    assert L.gq_gemm_dequant(*empty) == 0


@pytest.mark.parametrize("qbits", [6, 8])
def test_gemm_dequant_fresh_inputs(gq, qbits):
    """Shapes whose code ring wraps, each run on three fresh allocations."""
    for M, N, K in ((128, 256, 512), (256, 256, 512), (300, 384, 2048), (16, 512, 4096)):
        for rep in range(3):
            _case(gq, M, N, K, qbits, seed=1000 * rep + M + N + K + qbits)
