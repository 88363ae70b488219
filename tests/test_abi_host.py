"""Host-side checks of libgq (no GPU needed, no kernel launched).

* the library builds for sm_100a and exports every entry point that
  include/gq.h declares;
* the host-only entry points (k from p, packed row bytes, the export plan)
  agree with the oracle;
* argument errors come back before anything is launched.
"""
from __future__ import annotations

import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from oracle import plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gq():
    from int6_int8_weight_b200 import build
    build.build()
    from int6_int8_weight_b200 import gq as mod
    return mod


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "gq.h")).read()
    return sorted(set(re.findall(r"GQ_API\s+[\w\s\*]+?\b(gq_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("gq_row_clip_select", "gq_fakequant_fwd", "gq_ste_bwd", "gq_export_pack",
              "gq_dequant"):
        assert s in syms


def test_library_exports_every_declared_symbol(gq):
    out = subprocess.run(["nm", "-D", "--defined-only", gq.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert hasattr(gq.LIB, s)
    assert set(gq.EXPORTED) <= set(declared_symbols())


def test_header_compiles_as_c():
    src = '#include "gq.h"\nint main(void){gq_tensor t; (void)t; return (int)sizeof(gq_tensor);}\n'
    out = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-fsyntax-only",
                          "-I", os.path.join(ROOT, "include"), "-x", "c", "-"],
                         input=src, text=True, capture_output=True)
    assert out.returncode == 0, out.stderr


def test_struct_layout_matches_binding(gq):
    assert C.sizeof(gq.GQTensor) == 112      # static_assert(sizeof(gq_tensor) == 112) in gq_api.cu
    assert gq.GQTensor.p.offset == 48 and gq.GQTensor.clip.offset == 96
    assert gq.GQTensor.col_scale.offset == 104


def test_k_from_p_matches_oracle(gq):
    rng = np.random.default_rng(21)
    for _ in range(3000):
        n = int(rng.integers(1, 1 << 30))
        p = float(rng.uniform(0, 1)) if rng.random() < 0.9 else float(rng.choice([1.0, 0.5, 0.9999, 0.999]))
        if p == 0.0:
            continue
        assert gq.gq_k_from_p(n, p) == oracle.k_from_p(n, p)
    assert gq.gq_k_from_p(0, 0.5) == -1
    assert gq.gq_k_from_p(10, 0.0) == -1
    assert gq.gq_k_from_p(10, 1.5) == -1


def test_packed_row_bytes(gq):
    for cols in range(0, 40):
        for qb in (6, 8, 16):
            assert gq.gq_packed_row_bytes(cols, qb) == oracle.packed_row_bytes(cols, qb)
    assert gq.gq_packed_row_bytes(10, 7) == -1


def test_plan_matches_oracle(gq):
    cases = [
        ("tok_emb.weight", (1024, 512), True), ("lm_head.weight", (1792, 512), True),
        ("blocks.0.mlp.fc.weight", (1536, 512), True), ("blocks.0.attn_scale", (512,), True),
        ("tok_emb.weight", (100, 512), True), ("x", (256, 256), True), ("x", (255, 256), True),
        ("step", (70000,), False), ("conv", (256, 32, 3, 3), True), ("scalar", (), True),
        ("bigram.embed.weight", (2048, 128), True),
    ]
    for pats_env in (None, "bigram,lm_head.weight", " mlp.fc , tok_emb.weight"):
        pats = plan.patterns_from_env(pats_env)
        for name, shape, is_float in cases:
            want, _ = plan.classify(name, shape, is_float, pats)
            assert gq.plan_kind(name, shape, is_float, pats_env) == want, (name, pats_env)


def test_status_strings(gq):
    for s in range(9):
        assert gq.gq_status_string(s)


def _desc(gq, **kw):
    base = dict(w=0x10000, dtype=0, qbits=6, gran=0, reserved=0, rows=4, cols=8, ld=8, p=1.0,
                dq=0x20000, codes=0, packed=0x30000, scale_f16=0x40000, scale_f32=0, clip=0)
    base.update(kw)
    return gq.GQTensor(**base)


@pytest.mark.parametrize("bad,code", [
    (dict(w=0), 1), (dict(dtype=3), 1), (dict(qbits=7), 1), (dict(gran=2), 1),
    (dict(reserved=1), 1), (dict(p=0.0), 1), (dict(p=1.5), 1), (dict(p=float("nan")), 1),
    (dict(ld=4), 1), (dict(rows=-1), 1), (dict(packed=0), 1), (dict(scale_f16=0), 1),
    (dict(w=0x10001), 3), (dict(dq=0x20002), 3), (dict(scale_f16=0x40001), 3),
    (dict(rows=1 << 61, cols=1 << 10, ld=1 << 10), 1),
])
def test_export_argument_errors(gq, bad, code):
    st = gq.LIB.gq_export_pack(gq._arr([_desc(gq, **bad)]), 1, None, 0, None, None)
    assert st == code


def test_other_argument_errors(gq):
    L = gq.LIB
    # fake-quant needs dq and refuses packed output
    assert L.gq_fakequant_fwd(gq._arr([_desc(gq)]), 1, 0, None, 0, None, None) == 1
    assert L.gq_fakequant_fwd(gq._arr([_desc(gq, packed=0, dq=0)]), 1, 0, None, 0, None, None) == 1
    # scale_f16 only in the binary16 mode
    assert L.gq_fakequant_fwd(gq._arr([_desc(gq, packed=0)]), 1, 0, None, 0, None, None) == 1
    assert L.gq_fakequant_fwd(gq._arr([_desc(gq, packed=0)]), 1, 5, None, 0, None, None) == 1
    # clip select needs clip and nothing else
    assert L.gq_row_clip_select(gq._arr([_desc(gq, dq=0, packed=0, scale_f16=0)]), 1, None, 0,
                                None, None) == 1
    # per-tensor needs workspace
    d = _desc(gq, gran=1)
    assert gq.gq_workspace_size([d]) > 0
    assert L.gq_export_pack(gq._arr([d]), 1, None, 0, None, None) == 4
    assert L.gq_export_pack(gq._arr([d]), 1, C.c_void_p(0x100000), 16, None, None) == 4
    # negative n / null array
    assert L.gq_export_pack(None, 1, None, 0, None, None) == 1
    assert L.gq_export_pack(gq._arr([d]), -1, None, 0, None, None) == 1
    # passthrough descriptors take no quantized outputs
    assert L.gq_export_pack(gq._arr([_desc(gq, qbits=16)]), 1, None, 0, None, None) == 1
    # STE and dequant argument checks
    assert L.gq_ste_bwd(None, None, 0, 8, 0, None) == 1
    assert L.gq_ste_bwd(C.c_void_p(0x1000), C.c_void_p(0x2000), 2, 8, 0, None) == 1
    assert L.gq_ste_bwd(C.c_void_p(0x1001), C.c_void_p(0x2000), 0, 8, 0, None) == 3
    assert L.gq_ste_bwd(C.c_void_p(0x1000), C.c_void_p(0x2000), 0, 8, 2, None) == 1
    assert L.gq_ste_bwd(None, None, 0, 0, 0, None) == 0            # empty is a no-op
    assert L.gq_dequant(C.c_void_p(0x1000), C.c_void_p(0x2000), 7, 0, 4, 4, C.c_void_p(0x3000), 0,
                        None) == 1
    assert L.gq_dequant(None, None, 6, 0, 4, 4, None, 0, None) == 1
    assert L.gq_dequant(None, None, 6, 0, 0, 4, None, 0, None) == 0  # empty is a no-op
    # empty batch is a no-op
    assert L.gq_export_pack(gq._arr([]), 0, None, 0, None, None) == 0
    # AWQ column scales: per-row quantizing groups only, 4-byte aligned
    assert L.gq_export_pack(gq._arr([_desc(gq, col_scale=0x50002)]), 1, None, 0, None, None) == 3
    assert L.gq_export_pack(gq._arr([_desc(gq, gran=1, col_scale=0x50000)]), 1, None, 0, None, None) == 2
    assert L.gq_export_pack(gq._arr([_desc(gq, qbits=16, dq=0, scale_f16=0, col_scale=0x50000)]), 1, None, 0,
                            None, None) == 2


def test_last_cuda_error_starts_clear(gq):
    assert gq.LIB.gq_last_cuda_error() == 0
    assert gq.LIB.gq_last_cuda_error_string().decode() == "no error"


def test_gemm_argument_errors_before_launch(gq):
    """gq_gemm_dequant refuses bad arguments on the host, before any CUDA call
    (fake device addresses are never dereferenced)."""
    L = gq.LIB
    X, P, S, Y = 0x100000, 0x200000, 0x300000, 0x400000
    ok = [X, 4, 64, 64, P, S, 6, 8, Y, 8, None, None]
    bad_cases = [
        (dict(i=6, v=7), 1),            # qbits
        (dict(i=1, v=-1), 1),           # M < 0
        (dict(i=3, v=32), 1),           # ldx < K
        (dict(i=9, v=4), 1),            # ldy < N
        (dict(i=2, v=50, j=3, w=56), 2),  # int6 rows of 39 bytes: neither TMA nor 4-byte copies
        (dict(i=0, v=X + 2), 3),        # activations not 16-byte aligned
        (dict(i=3, v=68), 3),           # activation pitch not a multiple of 8
        (dict(i=4, v=P + 8), 3),        # packed codes (48-byte rows) not 16-byte aligned
        (dict(i=8, v=Y + 2), 3),        # Y not 4-byte aligned
        (dict(i=0, v=0), 1),            # null activations
    ]
    for case, code in bad_cases:
        args = list(ok)
        args[case["i"]] = case["v"]
        if "j" in case:
            args[case["j"]] = case["w"]
        assert L.gq_gemm_dequant(*args) == code, (case, code)
    empty = list(ok)
    empty[1] = 0                        # M = 0: nothing to do, nothing launched
    assert L.gq_gemm_dequant(*empty) == 0


def test_wait_expiry_hook_rejects_bad_arguments(gq):
    # host-only: a rejected request arms nothing and launches nothing
    assert gq.LIB.gq_test_arm_wait_expiry(-1, 5_000_000) == 1
    assert gq.LIB.gq_test_arm_wait_expiry(0, 999_999) == 1
    assert gq.LIB.gq_test_arm_wait_expiry(0, 4_000_000_001) == 1


def test_gemm_fakequant_argument_errors_before_launch(gq):
    """gq_gemm_fakequant likewise (fake device addresses never dereferenced)."""
    L = gq.LIB
    X, W, C, Y = 0x100000, 0x200000, 0x300000, 0x400000
    ok = [X, 4, 64, 64, W, 0, 64, C, 6, 0, 8, Y, 8, None, None]
    for i, v, code in ((5, 2, 1), (9, 5, 1), (8, 4, 1), (6, 32, 1), (10, -1, 1), (4, W + 4, 3), (6, 66, 3),
                       (7, C + 2, 3), (7, 0, 1), (0, X + 8, 3)):
        args = list(ok)
        args[i] = v
        assert L.gq_gemm_fakequant(*args) == code, (i, v, code)
    empty = list(ok)
    empty[1] = 0
    assert L.gq_gemm_fakequant(*empty) == 0
