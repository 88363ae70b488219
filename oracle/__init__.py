"""CPU oracle for per-row / per-tensor int6/int8 weight quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``int6_int8_weight_b200``) and never imports it.

The arithmetic lives in ``gq_oracle.c`` (plain single-threaded C, one IEEE op
per step; the readings it takes are listed in that file's header).  This module
only marshals numpy arrays into it.  ``plan.py`` holds the export plan (which
tensor is stored as fp16, int8 or int6).

Method sources: the parameter-golf pages "SubSixteen v2: Int6 QAT + MLP 3x +
SWA + Sliding Window" (PR #69: STE fake quantization, quant_range [-31, 31]),
"Swiglu gating_ QAT_..." (PR #2159, Key Explored Modifications 1, 13-16:
STE QAT, int8 export, per-row / per-tensor scales, percentile clipping, small
tensor fp16 passthrough), "Record: Unified Attention + FA3 + Legal TTT"
(PR #1202: int8 embeddings) and "... Int6AWQ MixedBits" (PR #1495: mixed-bit
promotion by name).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np

from . import build as _build

OR_OK, OR_ERR_ARG, OR_ERR_RANGE, OR_ERR_NONFINITE, OR_ERR_NOMEM = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
AVG_MEAN, AVG_EMA = 0, 1


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    """float32 arrays are fp32; uint16 arrays carry bf16 bit patterns."""
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {a.dtype}")


@dataclass
class QuantResult:
    status: int
    clip: np.ndarray      # float32 [groups]
    scale_f32: np.ndarray  # float32 [groups], the scale used to quantize
    scale_f16: np.ndarray | None  # uint16 [groups] (export mode)
    codes: np.ndarray     # int8 [rows, cols]
    dq: np.ndarray        # same dtype as the input, [rows, cols]
    packed: np.ndarray    # uint8 [rows, packed_row_bytes]


class Oracle:
    """numpy front end of one loaded copy of the C oracle."""

    def __init__(self, path: str):
        L = C.CDLL(path)
        vp, i64, i32, f32, f64 = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_double
        L.or_quantize.argtypes = [vp, i32, i64, i64, i64, i32, i32, f64, i32,
                                  vp, vp, vp, vp, vp, vp]
        L.or_quantize.restype = i32
        L.or_dequant.argtypes = [vp, vp, i32, i32, i64, i64, vp, i32]
        L.or_dequant.restype = i32
        L.or_ste_bwd.argtypes = [vp, vp, i32, i64, i32]
        L.or_ste_bwd.restype = i32
        L.or_col_scale.argtypes = [vp, i32, i64, i64, i64, vp, vp]
        L.or_col_scale.restype = i32
        L.or_passthrough_f16.argtypes = [vp, i32, i64, vp]
        L.or_passthrough_f16.restype = i32
        L.or_average_update.argtypes = [vp, vp, i32, i64, i32, i64, f32]
        L.or_average_update.restype = i32
        L.or_k_from_p.argtypes = [i64, f64]
        L.or_k_from_p.restype = i64
        L.or_packed_row_bytes.argtypes = [i64, i32]
        L.or_packed_row_bytes.restype = i64
        L.or_kth_smallest_abs.argtypes = [vp, i64, i64, vp]
        L.or_kth_smallest_abs.restype = f32
        L.or_f32_to_f16_array.argtypes = [vp, i64, vp]
        L.or_f16_to_f32_array.argtypes = [vp, i64, vp]
        L.or_f32_to_bf16_array.argtypes = [vp, i64, vp]
        L.or_quantize_array.argtypes = [vp, i64, f32, f32, i32, vp]
        L.or_pack6_row.argtypes = [vp, i64, vp]
        L.or_unpack6_row.argtypes = [vp, i64, vp]
        self.L = L
        self.path = path

    def k_from_p(self, n: int, p: float) -> int:
        return int(self.L.or_k_from_p(n, p))

    def packed_row_bytes(self, cols: int, qbits: int) -> int:
        return int(self.L.or_packed_row_bytes(cols, qbits))

    def col_scale(self, w: np.ndarray, t: np.ndarray, cols: int | None = None) -> np.ndarray:
        """AWQ column scaling (reading R12 in gq_oracle.c): the dense
        [rows, cols] weight RN_dtype(w[r, c] * t[c]) in w's dtype."""
        assert w.ndim == 2
        w = np.ascontiguousarray(w)
        rows, ld = w.shape
        cols = ld if cols is None else cols
        t = np.ascontiguousarray(t, dtype=np.float32).ravel()
        assert t.size >= cols
        out = np.zeros((rows, cols), w.dtype)
        st = self.L.or_col_scale(_ptr(w), _dtype_code(w), rows, cols, ld, _ptr(t), _ptr(out))
        if st != OR_OK:
            raise ValueError(f"oracle col_scale status {st}")
        return out

    def quantize(self, w: np.ndarray, qbits: int, p: float = 1.0,
                 per_tensor: bool = False, export: bool = True,
                 cols: int | None = None, col_scale: np.ndarray | None = None) -> QuantResult:
        """Fake-quant forward / export of a 2-D weight ``w`` ([rows, ld]).

        ``cols`` (default: all of ``ld``) selects the used columns of each row.
        ``col_scale`` (AWQ, per-row only): quantize RN_dtype(w * t[column])
        instead of w.
        """
        assert w.ndim == 2
        if col_scale is not None:
            assert not per_tensor, "column scaling is defined for per-row groups"
            w = self.col_scale(w, col_scale, cols)
            cols = None
        w = np.ascontiguousarray(w)
        rows, ld = w.shape
        cols = ld if cols is None else cols
        dt = _dtype_code(w)
        groups = 1 if per_tensor else rows
        clip = np.zeros(groups, np.float32)
        s32 = np.zeros(groups, np.float32)
        s16 = np.zeros(groups, np.uint16) if export else None
        codes = np.zeros((rows, cols), np.int8)
        dq = np.zeros((rows, cols), w.dtype)
        packed = np.zeros((rows, max(self.packed_row_bytes(cols, qbits), 0)), np.uint8)
        st = self.L.or_quantize(_ptr(w), dt, rows, cols, ld, qbits, int(per_tensor),
                                float(p), int(export), _ptr(clip), _ptr(s32), _ptr(s16),
                                _ptr(codes), _ptr(dq), _ptr(packed))
        return QuantResult(int(st), clip, s32, s16, codes, dq, packed)

    def dequant(self, packed: np.ndarray, scale_f16: np.ndarray, qbits: int,
                rows: int, cols: int, per_tensor: bool = False,
                out_bf16: bool = False) -> np.ndarray:
        """Dequant on load from packed codes and binary16 scales."""
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        scale_f16 = np.ascontiguousarray(scale_f16, dtype=np.uint16)
        out = np.zeros((rows, cols), np.uint16 if out_bf16 else np.float32)
        st = self.L.or_dequant(_ptr(packed), _ptr(scale_f16), qbits, int(per_tensor),
                               rows, cols, _ptr(out), BF16 if out_bf16 else F32)
        if st != OR_OK:
            raise ValueError(f"oracle dequant status {st}")
        return out

    def ste_bwd(self, g_out: np.ndarray, g_w: np.ndarray | None = None,
                accumulate: bool = False) -> np.ndarray:
        """Straight-through backward: g_w = g_out, or g_w + g_out."""
        g_out = np.ascontiguousarray(g_out)
        dt = _dtype_code(g_out)
        res = np.zeros_like(g_out) if g_w is None else np.array(g_w, copy=True)
        st = self.L.or_ste_bwd(_ptr(g_out), _ptr(res), dt, g_out.size, int(accumulate))
        if st != OR_OK:
            raise ValueError(f"oracle ste status {st}")
        return res

    def average_update(self, avg: np.ndarray, x: np.ndarray, kind: int, count: int = 0,
                       decay: float = 0.997) -> np.ndarray:
        """Snapshot averaging (readings R10 / R11 in gq_oracle.c): the new
        binary32 average after snapshot ``x`` (float32, or bf16 bits as
        uint16); ``kind`` AVG_MEAN with ``count`` snapshots already in
        ``avg``, or AVG_EMA with ``decay``."""
        x = np.ascontiguousarray(x)
        res = np.array(avg, dtype=np.float32, copy=True).reshape(x.shape)
        st = self.L.or_average_update(_ptr(res), _ptr(x), _dtype_code(x), x.size, int(kind),
                                      int(count), float(decay))
        if st != OR_OK:
            raise ValueError(f"oracle average status {st}")
        return res

    def fakequant_average(self, w: np.ndarray, avg: np.ndarray, qbits: int, p: float, kind: int,
                          count: int = 0, decay: float = 0.997, per_tensor: bool = False,
                          export: bool = False):
        """Fake-quant of ``w`` followed by the average update with its output
        as the snapshot; returns (QuantResult, new average)."""
        ref = self.quantize(w, qbits, p, per_tensor=per_tensor, export=export)
        return ref, self.average_update(avg, ref.dq, kind, count, decay)

    def passthrough_f16(self, x: np.ndarray) -> np.ndarray:
        """Small-tensor passthrough: binary16 bit patterns (uint16) of ``x``."""
        x = np.ascontiguousarray(x)
        out = np.zeros(x.shape, np.uint16)
        st = self.L.or_passthrough_f16(_ptr(x), _dtype_code(x), x.size, _ptr(out))
        if st != OR_OK:
            raise ValueError(f"oracle passthrough status {st}")
        return out

    def kth_smallest_abs(self, v: np.ndarray, k: int) -> float:
        v = np.ascontiguousarray(v, dtype=np.float32).ravel()
        scratch = np.empty_like(v)
        return float(self.L.or_kth_smallest_abs(_ptr(v), v.size, k, _ptr(scratch)))

    def f32_to_f16_bits(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float32).ravel()
        out = np.empty(x.size, np.uint16)
        self.L.or_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
        return out

    def f16_bits_to_f32(self, h: np.ndarray) -> np.ndarray:
        h = np.ascontiguousarray(h, dtype=np.uint16).ravel()
        out = np.empty(h.size, np.float32)
        self.L.or_f16_to_f32_array(_ptr(h), h.size, _ptr(out))
        return out

    def f32_to_bf16_bits(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float32).ravel()
        out = np.empty(x.size, np.uint16)
        self.L.or_f32_to_bf16_array(_ptr(x), x.size, _ptr(out))
        return out

    def quantize_values(self, w: np.ndarray, c: float, s: float, qmax: int) -> np.ndarray:
        """Codes of ``w`` for a given clip and scale (the quantize step alone)."""
        w = np.ascontiguousarray(w, dtype=np.float32).ravel()
        q = np.empty(w.size, np.int8)
        self.L.or_quantize_array(_ptr(w), w.size, c, s, qmax, _ptr(q))
        return q

    def pack6_row(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.int8).ravel()
        out = np.empty(3 * ((q.size + 3) // 4), np.uint8)
        self.L.or_pack6_row(_ptr(q), q.size, _ptr(out))
        return out

    def unpack6_row(self, b: np.ndarray, cols: int) -> np.ndarray:
        b = np.ascontiguousarray(b, dtype=np.uint8).ravel()
        out = np.empty(cols, np.int8)
        self.L.or_unpack6_row(_ptr(b), cols, _ptr(out))
        return out


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``gq_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def __getattr__(name):
    # module-level access to the default oracle's methods: oracle.quantize(...)
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)
