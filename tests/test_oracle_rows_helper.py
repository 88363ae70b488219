"""The full-size parity helper (oracle over row blocks in threads) is not
vacuous: it reports zero mismatches for the oracle's own whole-matrix result
and finds a single flipped bit or byte in any output."""
from __future__ import annotations

import numpy as np

import oracle
import synth
from tests import oracle_rows


def test_row_blocks_equal_whole_matrix_and_catch_flips():
    rng = np.random.default_rng(7)
    w = synth.random_matrix(rng, 300, 96, "t3")
    for qbits, p in ((6, 0.9), (8, 1.0)):
        ref = oracle.quantize(w, qbits, p, export=True)
        got = {"dq": ref.dq.copy(), "packed": ref.packed.copy(), "scale_f16": ref.scale_f16.copy(),
               "codes": ref.codes.copy()}
        res = oracle_rows.compare_rows(w, got, qbits, p, block_rows=7)
        assert all(v == 0 for v in res["mismatches"].values()), res
        for key, (r, c) in (("dq", (123, 5)), ("packed", (299, 0)), ("codes", (0, 95))):
            bad = {k: v.copy() for k, v in got.items()}
            a = bad[key].view(np.uint32) if bad[key].dtype == np.float32 else bad[key].view(np.uint8)
            a[r, c] ^= 1
            res = oracle_rows.compare_rows(w, bad, qbits, p, block_rows=64)
            assert res["mismatches"][key] == 1 and res["first_row"][key] == r, (key, res)
        bad = dict(got, scale_f16=got["scale_f16"].copy())
        bad["scale_f16"][42] ^= 1
        res = oracle_rows.compare_rows(w, bad, qbits, p)
        assert res["mismatches"]["scale_f16"] == 1 and res["first_row"]["scale_f16"] == 42


def test_quantize_many_matches_one_by_one():
    rng = np.random.default_rng(8)
    ws = [synth.random_matrix(rng, r, c, "normal") for r, c in ((5, 8), (17, 33), (64, 128))]
    many = oracle_rows.quantize_many(ws, 6, 1.0, export=False)
    for w, m in zip(ws, many):
        one = oracle.quantize(w, 6, 1.0, export=False)
        assert np.array_equal(m.dq.view(np.uint32), one.dq.view(np.uint32))
        assert np.array_equal(m.codes, one.codes)
