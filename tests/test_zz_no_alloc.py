"""gq_export_pack_noalloc: export for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: runtimes that own a fixed
device-memory budget and give out only the tensors, code that must not trigger
cudaMalloc's implicit synchronization, plain C hosts without an allocator.
For them gq_export_pack_noalloc takes its per-tensor scratch from a fixed
array inside libgq.  This test calls it through the C ABI and checks that its
outputs equal those of gq_export_pack (bit for bit, the tolerance of every
parity test here) on two calls in a row with different inputs, so that what
the first call leaves in the shared array cannot leak into the second; the
outputs are also checked against the CPU oracle.

The file is named so that pytest collects it last; it must also pass alone in
a fresh process (the first call on the device sets the array up).
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


def _batch(gq, mats):
    """Descriptors with freshly allocated outputs: per-tensor and per-row,
    int6 and int8, fp32 and bf16 (per-tensor groups are the ones that use the
    scratch)."""
    descs, outs = [], []
    for i, W in enumerate(mats):
        rows, cols = W.shape
        per_tensor = i % 2 == 0
        qbits = 6 if i % 3 else 8
        p = (0.999, 0.9, 1.0, 0.5)[i % 4]
        dq = torch.empty_like(W)
        packed = torch.empty((rows, gq.gq_packed_row_bytes(cols, qbits)), dtype=torch.uint8, device=W.device)
        groups = 1 if per_tensor else rows
        h = torch.empty(groups, dtype=torch.float16, device=W.device)
        clip = torch.empty(groups, dtype=torch.float32, device=W.device)
        codes = torch.empty((rows, cols), dtype=torch.int8, device=W.device)
        descs.append(gq.GQTensor(w=W.data_ptr(), dtype=gq._dtype_code(W), qbits=qbits,
                                 gran=1 if per_tensor else 0, reserved=0, rows=rows, cols=cols,
                                 ld=cols, p=p, dq=dq.data_ptr(), codes=codes.data_ptr(),
                                 packed=packed.data_ptr(), scale_f16=h.data_ptr(), scale_f32=0,
                                 clip=clip.data_ptr()))
        outs.append((dq, codes, packed, h, clip))
    return descs, outs


def _mats(seed):
    rng = np.random.default_rng(seed)
    shapes = [(256, 512), (96, 1536), (512, 512), (33, 4101), (300, 128), (7, 77)]
    mats = []
    for j, (r, c) in enumerate(shapes):
        W = torch.from_numpy(synth.random_matrix(rng, r, c, ("t3", "mix", "normal")[j % 3])).cuda()
        mats.append(W if j % 2 else W.to(torch.bfloat16))
    return mats


def _same(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def test_noalloc_matches_export_on_two_calls(gq):
    status = torch.zeros(16, dtype=torch.int32, device="cuda")
    for call, seed in enumerate((101, 202)):
        mats = _mats(seed)
        want_descs, want = _batch(gq, mats)
        nbytes = gq.gq_workspace_size(want_descs)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        gq.gq_export_pack(want_descs, ws=ws.data_ptr(), ws_bytes=nbytes)
        got_descs, got = _batch(gq, mats)
        gq.gq_export_pack_noalloc(got_descs, d_status=status.data_ptr())
        torch.cuda.synchronize()
        assert status[: len(mats)].eq(0).all(), (call, status.tolist())
        for i, (g, w) in enumerate(zip(got, want)):
            for name, x, y in zip(("dq", "codes", "packed", "scale_f16", "clip"), g, w):
                assert _same(x, y), (call, i, name)
        for i, (W, d, g) in enumerate(zip(mats, got_descs, got)):
            w_host = W.cpu()
            w_np = (w_host.view(torch.int16).numpy().view(np.uint16) if W.dtype == torch.bfloat16
                    else w_host.numpy())
            ref = oracle.quantize(w_np, d.qbits, d.p, per_tensor=d.gran == 1, export=True)
            assert ref.status == 0
            dq_np = g[0].cpu()
            dq_np = (dq_np.view(torch.int16).numpy().view(np.uint16) if W.dtype == torch.bfloat16
                     else dq_np.numpy().view(np.uint32))
            want_dq = ref.dq.view(np.uint32) if ref.dq.dtype == np.float32 else ref.dq
            assert np.array_equal(dq_np, want_dq), (call, i, "dq vs oracle")
            assert np.array_equal(g[1].cpu().numpy(), ref.codes), (call, i, "codes vs oracle")
            assert np.array_equal(g[2].cpu().numpy(), ref.packed), (call, i, "packed vs oracle")
            assert np.array_equal(g[3].cpu().view(torch.int16).numpy().view(np.uint16), ref.scale_f16), \
                (call, i, "scale_f16 vs oracle")


def test_noalloc_rejects_batches_beyond_its_scratch(gq):
    W = torch.ones((4, 8), device="cuda")
    out = torch.empty(64, dtype=torch.uint8, device="cuda")
    d = gq.GQTensor(w=W.data_ptr(), dtype=0, qbits=6, gran=1, reserved=0, rows=4, cols=8, ld=8,
                    p=1.0, dq=0, codes=0, packed=out.data_ptr(), scale_f16=out.data_ptr(),
                    scale_f32=0, clip=0)
    with pytest.raises(gq.GQError) as e:
        gq.gq_export_pack_noalloc([d] * 65)
    assert e.value.status == 4          # GQ_ERR_WORKSPACE, nothing launched
    gq.gq_export_pack_noalloc([d] * 64)  # the stated maximum is accepted
    torch.cuda.synchronize()
