"""The timeout path of the pipelined row kernel's bounded waits, on the GPU.

The kernel waits on mbarriers for its own bulk copies into shared memory;
every wait gives up after a time limit, the tile-team that gave up leaves its
loop together, the launch records GQ_STATUS_TIMEOUT and ends.  A test hook
(gq_test_arm_wait_expiry, test-only) makes that happen without a fault: one
tile's copy announces 16 bytes more than it transfers, so the tile's barrier
never completes although every issued copy does, and the waits of that
launch give up after a few milliseconds.  Nothing is left in flight when the
kernel returns.  The test checks the status word, that the call ends
promptly, and that the next ordinary call is bit-exact against the oracle.
"""
from __future__ import annotations

import time

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


def _export_desc(gq, W, qbits, p):
    rows, cols = W.shape
    dq = torch.empty_like(W)
    packed = torch.empty((rows, gq.gq_packed_row_bytes(cols, qbits)), dtype=torch.uint8, device=W.device)
    h = torch.empty(rows, dtype=torch.float16, device=W.device)
    d = gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=qbits, gran=0, reserved=0,
                    rows=rows, cols=cols, ld=cols, p=p, dq=dq.data_ptr(), codes=0,
                    packed=packed.data_ptr(), scale_f16=h.data_ptr(), scale_f32=0, clip=0)
    return d, (dq, packed, h)


@pytest.mark.parametrize("dtype,cols,tile", [("f32", 1024, 5), ("bf16", 4096, 0), ("f32", 16384, 150)])
def test_wait_expiry_sets_timeout_and_library_recovers(gq, dtype, cols, tile):
    rng = np.random.default_rng(cols + tile)
    rows = 2048 if cols <= 4096 else 512
    w = synth.random_matrix(rng, rows, cols, "t3")
    if dtype == "bf16":
        w = synth.to_bf16_bits(w).reshape(rows, cols)
        W = torch.from_numpy(w.view(np.int16).copy()).cuda().view(torch.bfloat16)
    else:
        W = torch.from_numpy(w).cuda()
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")

    # armed call: the wait on the poisoned tile runs out after 5 ms
    d, _ = _export_desc(gq, W, 6, 0.9999)
    assert gq.LIB.gq_test_arm_wait_expiry(tile, 5_000_000) == 0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gq.gq_export_pack([d], d_status=status.data_ptr())
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status[0]) & gq.GQ_STATUS_TIMEOUT, status.tolist()
    assert elapsed < 2.0, elapsed          # a few 5 ms waits, not the 4 s default

    # the hook was consumed: the next call is an ordinary one, bit-exact
    d, (dq, packed, h) = _export_desc(gq, W, 6, 0.9999)
    gq.gq_export_pack([d], d_status=status.data_ptr())
    torch.cuda.synchronize()
    assert int(status[0]) == 0, status.tolist()
    ref = oracle.quantize(w, 6, 0.9999, export=True)
    got_dq = dq.cpu()
    got_dq = (got_dq.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16"
              else got_dq.numpy().view(np.uint32))
    want_dq = ref.dq if dtype == "bf16" else ref.dq.view(np.uint32)
    assert np.array_equal(got_dq, want_dq)
    assert np.array_equal(packed.cpu().numpy(), ref.packed)
    assert np.array_equal(h.cpu().view(torch.int16).numpy().view(np.uint16), ref.scale_f16)
