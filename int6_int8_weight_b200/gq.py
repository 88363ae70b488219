"""Thin Python binding of libgq (include/gq.h) over ctypes.

Argument marshalling only: every step of the quantization runs in the CUDA
kernels of libgq.so.  PyTorch provides device memory and streams.  There is no
CPU fallback: if the library is missing, importing this module raises.

Low level: ``GQTensor`` mirrors ``gq_tensor`` and the ``gq_*`` functions take
the same arguments as the C entry points (pointers as ints, the stream as a
``torch.cuda.Stream`` or None for the current stream).

High level: ``fakequant`` / ``export_pack`` / ``row_clip_select`` take torch
tensors, allocate the requested outputs and return them; ``FakeQuantSTE`` is
the autograd function of the straight-through estimator; ``dequant`` and
``ste_bwd`` wrap the remaining calls; ``plan_kind`` / ``export_state_dict``
apply the mixed-bit export plan.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgq.so")

GQ_OK = 0
GQ_F32, GQ_BF16 = 0, 1
GQ_PER_ROW, GQ_PER_TENSOR = 0, 1
GQ_SCALE_F32, GQ_SCALE_F16 = 0, 1
GQ_STATUS_NONFINITE, GQ_STATUS_RANGE, GQ_STATUS_TIMEOUT = 1, 2, 4
GQ_AVG_MEAN, GQ_AVG_EMA = 0, 1
GQ_KIND_RAW, GQ_KIND_FP16, GQ_KIND_INT8, GQ_KIND_INT6 = 0, 1, 2, 3
KIND_NAMES = {GQ_KIND_RAW: "raw", GQ_KIND_FP16: "fp16", GQ_KIND_INT8: "int8", GQ_KIND_INT6: "int6"}

STATUS_NAMES = {0: "GQ_OK", 1: "GQ_ERR_INVALID_ARG", 2: "GQ_ERR_UNSUPPORTED",
                3: "GQ_ERR_MISALIGNED", 4: "GQ_ERR_WORKSPACE", 5: "GQ_ERR_RANGE",
                6: "GQ_ERR_NONFINITE", 7: "GQ_ERR_CUDA", 8: "GQ_ERR_TIMEOUT"}

EXPORTED = ("gq_row_clip_select", "gq_fakequant_fwd", "gq_fakequant_average", "gq_ste_bwd", "gq_export_pack",
            "gq_export_pack_noalloc", "gq_dequant", "gq_gemm_dequant", "gq_workspace_size", "gq_packed_row_bytes", "gq_k_from_p",
            "gq_plan_kind", "gq_status_string", "gq_last_cuda_error", "gq_last_cuda_error_string",
            "gq_test_arm_wait_expiry", "gq_gptq_quantize", "gq_gptq_hessian", "gq_gptq_workspace_size",
            "gq_gemm_fakequant", "gq_gptq_quantize_batch", "gq_gptq_batch_workspace_size")


class GQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}" + (f" ({detail})" if detail else ""))
        self.status = status


class GQTensor(C.Structure):
    _fields_ = [
        ("w", C.c_void_p), ("dtype", C.c_int32), ("qbits", C.c_int32),
        ("gran", C.c_int32), ("reserved", C.c_int32),
        ("rows", C.c_int64), ("cols", C.c_int64), ("ld", C.c_int64),
        ("p", C.c_double),
        ("dq", C.c_void_p), ("codes", C.c_void_p), ("packed", C.c_void_p),
        ("scale_f16", C.c_void_p), ("scale_f32", C.c_void_p), ("clip", C.c_void_p),
        ("col_scale", C.c_void_p),
    ]


class GQAvg(C.Structure):
    _fields_ = [("avg", C.c_void_p), ("kind", C.c_int32), ("decay", C.c_float), ("count", C.c_int64)]


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libgq.so not found at {LIB_PATH}; build it with "
            "`python -m int6_int8_weight_b200.build` (no CPU fallback exists)")
    L = C.CDLL(LIB_PATH)
    vp, i32, i64, sz, f64 = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_double
    T = C.POINTER(GQTensor)
    L.gq_row_clip_select.argtypes = [T, i32, vp, sz, vp, vp]
    L.gq_fakequant_fwd.argtypes = [T, i32, i32, vp, sz, vp, vp]
    L.gq_fakequant_average.argtypes = [T, C.POINTER(GQAvg), i32, i32, vp, sz, vp, vp]
    L.gq_export_pack.argtypes = [T, i32, vp, sz, vp, vp]
    L.gq_export_pack_noalloc.argtypes = [T, i32, vp, vp]
    L.gq_ste_bwd.argtypes = [vp, vp, i32, i64, i32, vp]
    L.gq_dequant.argtypes = [vp, vp, i32, i32, i64, i64, vp, i32, vp]
    L.gq_gemm_dequant.argtypes = [vp, i64, i64, i64, vp, vp, i32, i64, vp, i64, vp, vp]
    L.gq_gemm_fakequant.argtypes = [vp, i64, i64, i64, vp, i32, i64, vp, i32, i32, i64, vp, i64, vp, vp]
    for f in ("gq_row_clip_select", "gq_fakequant_fwd", "gq_fakequant_average", "gq_export_pack",
              "gq_export_pack_noalloc",
              "gq_ste_bwd", "gq_dequant", "gq_gemm_dequant", "gq_gemm_fakequant"):
        getattr(L, f).restype = i32
    L.gq_gptq_quantize.argtypes = [T, vp, f64, vp, sz, vp, vp]
    L.gq_gptq_quantize.restype = i32
    L.gq_gptq_quantize_batch.argtypes = [T, i32, C.POINTER(vp), f64, vp, sz, vp, vp]
    L.gq_gptq_quantize_batch.restype = i32
    L.gq_gptq_batch_workspace_size.argtypes = [T, i32]
    L.gq_gptq_batch_workspace_size.restype = sz
    L.gq_gptq_hessian.argtypes = [vp, i32, i64, i64, i64, vp, i32, vp]
    L.gq_gptq_hessian.restype = i32
    L.gq_gptq_workspace_size.argtypes = [i64, i64]
    L.gq_gptq_workspace_size.restype = sz
    L.gq_test_arm_wait_expiry.argtypes = [i64, C.c_uint64]
    L.gq_test_arm_wait_expiry.restype = i32
    L.gq_workspace_size.argtypes = [T, i32]
    L.gq_workspace_size.restype = sz
    L.gq_packed_row_bytes.argtypes = [i64, i32]
    L.gq_packed_row_bytes.restype = i64
    L.gq_k_from_p.argtypes = [i64, f64]
    L.gq_k_from_p.restype = i64
    L.gq_plan_kind.argtypes = [C.c_char_p, C.POINTER(C.c_int64), i32, i32, C.c_char_p, i64]
    L.gq_plan_kind.restype = i32
    L.gq_status_string.argtypes = [i32]
    L.gq_status_string.restype = C.c_char_p
    L.gq_last_cuda_error.argtypes = []
    L.gq_last_cuda_error.restype = i32
    L.gq_last_cuda_error_string.argtypes = []
    L.gq_last_cuda_error_string.restype = C.c_char_p
    return L


LIB = _load()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != GQ_OK:
        detail = LIB.gq_last_cuda_error_string().decode() if status == 7 else ""
        raise GQError(status, where, detail)


def _arr(descs):
    arr = (GQTensor * max(1, len(descs)))()
    for i, d in enumerate(descs):
        arr[i] = d
    return arr


# ---------------------------------------------------------- low level ABI --

def gq_row_clip_select(descs, ws=0, ws_bytes=0, d_status=0, stream=None):
    _check(LIB.gq_row_clip_select(_arr(descs), len(descs), ws or None, ws_bytes,
                                  d_status or None, _stream(stream)), "gq_row_clip_select")


def gq_fakequant_fwd(descs, mode, ws=0, ws_bytes=0, d_status=0, stream=None):
    _check(LIB.gq_fakequant_fwd(_arr(descs), len(descs), mode, ws or None, ws_bytes,
                                d_status or None, _stream(stream)), "gq_fakequant_fwd")


def _avg_arr(avgs):
    arr = (GQAvg * max(1, len(avgs)))()
    for i, a in enumerate(avgs):
        arr[i] = a
    return arr


def gq_fakequant_average(descs, avgs, mode, ws=0, ws_bytes=0, d_status=0, stream=None):
    _check(LIB.gq_fakequant_average(_arr(descs), _avg_arr(avgs), len(descs), mode, ws or None, ws_bytes,
                                    d_status or None, _stream(stream)), "gq_fakequant_average")


def gq_export_pack(descs, ws=0, ws_bytes=0, d_status=0, stream=None):
    _check(LIB.gq_export_pack(_arr(descs), len(descs), ws or None, ws_bytes,
                              d_status or None, _stream(stream)), "gq_export_pack")


def gq_export_pack_noalloc(descs, d_status=0, stream=None):
    """gq_export_pack with the library's fixed scratch instead of a workspace."""
    _check(LIB.gq_export_pack_noalloc(_arr(descs), len(descs), d_status or None, _stream(stream)),
           "gq_export_pack_noalloc")


def gq_ste_bwd(g_out_ptr, g_w_ptr, dtype, numel, accumulate, stream=None):
    _check(LIB.gq_ste_bwd(g_out_ptr or None, g_w_ptr or None, dtype, numel, int(accumulate),
                          _stream(stream)), "gq_ste_bwd")


def gq_dequant(packed_ptr, scale_ptr, qbits, gran, rows, cols, out_ptr, out_dtype, stream=None):
    _check(LIB.gq_dequant(packed_ptr or None, scale_ptr or None, qbits, gran, rows, cols,
                          out_ptr or None, out_dtype, _stream(stream)), "gq_dequant")


def gq_gemm_dequant(x_ptr, M, K, ldx, packed_ptr, scale_ptr, qbits, N, y_ptr, ldy, d_status=0, stream=None):
    _check(LIB.gq_gemm_dequant(x_ptr, M, K, ldx, packed_ptr, scale_ptr, qbits, N, y_ptr, ldy,
                               d_status or None, _stream(stream)), "gq_gemm_dequant")


def gq_workspace_size(descs) -> int:
    return int(LIB.gq_workspace_size(_arr(descs), len(descs)))


def gq_packed_row_bytes(cols: int, qbits: int) -> int:
    return int(LIB.gq_packed_row_bytes(cols, qbits))


def gq_k_from_p(n: int, p: float) -> int:
    return int(LIB.gq_k_from_p(n, p))


def gq_plan_kind(name: str, shape, is_float: bool, patterns: str | None = None,
                 small_numel: int = 65536) -> int:
    arr = (C.c_int64 * max(1, len(shape)))(*shape)
    return int(LIB.gq_plan_kind(name.encode(), arr, len(shape), int(is_float),
                                None if patterns is None else patterns.encode(), small_numel))


def gq_status_string(status: int) -> str:
    return LIB.gq_status_string(status).decode()


# --------------------------------------------------------- torch helpers --

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GQ_F32
    if t.dtype == torch.bfloat16:
        return GQ_BF16
    raise TypeError(f"libgq takes float32 or bfloat16 weights, got {t.dtype}")


def _ptr(t: torch.Tensor | None) -> int:
    return 0 if t is None else t.data_ptr()


@dataclass
class Quantized:
    """Outputs of one quantized tensor (None where not requested)."""
    dq: torch.Tensor | None = None
    codes: torch.Tensor | None = None
    packed: torch.Tensor | None = None
    scale_f16: torch.Tensor | None = None
    scale_f32: torch.Tensor | None = None
    clip: torch.Tensor | None = None
    status: int = 0


@dataclass
class Request:
    """One tensor to quantize: the weight view [rows, ld] and what to produce."""
    w: torch.Tensor
    qbits: int = 6
    p: float = 1.0
    per_tensor: bool = False
    want_dq: bool = True
    want_codes: bool = False
    want_packed: bool = False
    want_scale_f16: bool = False
    want_scale_f32: bool = False
    want_clip: bool = False
    cols: int | None = None
    col_scale: torch.Tensor | None = None   # AWQ: fp32 [cols] column scales (per-row groups)


def _as_2d(w: torch.Tensor):
    if w.dim() != 2:
        raise ValueError("weights are passed as 2-D [rows, cols] views")
    if w.stride(1) != 1:
        raise ValueError("rows must be contiguous (stride(1) == 1)")
    return w.shape[0], w.shape[1], w.stride(0)


def _prepare(reqs, export: bool):
    descs, outs = [], []
    for r in reqs:
        rows, cols, ld = _as_2d(r.w)
        if r.cols is not None:
            cols = r.cols
        dev = r.w.device
        groups = 1 if r.per_tensor else rows
        o = Quantized()
        if r.qbits == 16:
            o.packed = torch.empty((rows, cols), dtype=torch.float16, device=dev)
        else:
            if r.want_dq:
                o.dq = torch.empty((rows, cols), dtype=r.w.dtype, device=dev)
            if r.want_codes:
                o.codes = torch.empty((rows, cols), dtype=torch.int8, device=dev)
            if r.want_packed:
                o.packed = torch.empty((rows, gq_packed_row_bytes(cols, r.qbits)),
                                       dtype=torch.uint8, device=dev)
            if r.want_scale_f16:
                o.scale_f16 = torch.empty(groups, dtype=torch.float16, device=dev)
            if r.want_scale_f32:
                o.scale_f32 = torch.empty(groups, dtype=torch.float32, device=dev)
            if r.want_clip:
                o.clip = torch.empty(groups, dtype=torch.float32, device=dev)
        d = GQTensor(w=_ptr(r.w), dtype=_dtype_code(r.w), qbits=r.qbits,
                     gran=GQ_PER_TENSOR if r.per_tensor else GQ_PER_ROW, reserved=0,
                     rows=rows, cols=cols, ld=ld, p=float(r.p), dq=_ptr(o.dq),
                     codes=_ptr(o.codes), packed=_ptr(o.packed), scale_f16=_ptr(o.scale_f16),
                     scale_f32=_ptr(o.scale_f32), clip=_ptr(o.clip))
        if r.col_scale is not None:
            cs = r.col_scale
            if cs.dtype != torch.float32 or cs.dim() != 1 or cs.stride(0) != 1 or cs.numel() < cols \
                    or cs.device != dev:
                raise ValueError("col_scale must be a contiguous fp32 [cols] tensor on the weight's device")
            d.col_scale = cs.data_ptr()
        descs.append(d)
        outs.append(o)
    return descs, outs


class _Scratch:
    """Per-device workspace and status buffers kept between calls (torch memory)."""

    def __init__(self):
        self.ws: dict = {}

    def workspace(self, device, nbytes):
        key = (device, "ws")
        buf = self.ws.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
            self.ws[key] = buf
        return buf

    def status(self, device, n):
        key = (device, "st")
        buf = self.ws.get(key)
        if buf is None or buf.numel() < n:
            buf = torch.empty(max(n, 256), dtype=torch.int32, device=device)
            self.ws[key] = buf
        return buf


_SCRATCH = _Scratch()


def _run(fn_name, reqs, export, mode=None, stream=None, check_status=True, avgs=None):
    if not reqs:
        return []
    descs, outs = _prepare(reqs, export)
    dev = reqs[0].w.device
    nbytes = gq_workspace_size(descs)
    ws = _SCRATCH.workspace(dev, nbytes) if nbytes else None
    st = _SCRATCH.status(dev, len(descs))
    args = dict(ws=_ptr(ws), ws_bytes=0 if ws is None else ws.numel(), d_status=st.data_ptr(),
                stream=stream)
    if fn_name == "fakequant":
        gq_fakequant_fwd(descs, mode, **args)
    elif fn_name == "average":
        gq_fakequant_average(descs, avgs, mode, **args)
    elif fn_name == "export":
        gq_export_pack(descs, **args)
    else:
        gq_row_clip_select(descs, **args)
    if check_status:
        stv = st[: len(descs)].cpu().tolist()
        for o, s in zip(outs, stv):
            o.status = int(s)
    return outs


def fakequant(reqs, mode=GQ_SCALE_F32, stream=None, check_status=True):
    """Batched STE fake-quant forward (one launch for the batch)."""
    return _run("fakequant", reqs, False, mode, stream, check_status)


def fakequant_average(reqs, averages, kind=GQ_AVG_MEAN, count=0, decay=0.997, mode=GQ_SCALE_F32,
                      stream=None, check_status=True):
    """Fake-quant of each request fused with the update of its running
    average of quantize-dequantize snapshots (``averages``: float32 tensors
    of the weights' shape, updated in place).  ``kind`` GQ_AVG_MEAN with
    ``count`` snapshots already averaged, or GQ_AVG_EMA with ``decay``.
    w_hat is returned only for requests with ``want_dq``."""
    avgs = []
    for r, a in zip(reqs, averages, strict=True):
        if a.dtype != torch.float32 or not a.is_contiguous() or a.shape != r.w.shape:
            raise ValueError("averages are contiguous float32 tensors of the weight's shape")
        avgs.append(GQAvg(avg=a.data_ptr(), kind=kind, decay=float(decay), count=int(count)))
    return _run("average", reqs, False, mode, stream, check_status, avgs)


def export_pack(reqs, stream=None, check_status=True):
    """Batched export (binary16 scales, packed codes; qbits 16 = passthrough)."""
    for r in reqs:
        if r.qbits != 16:
            r.want_packed = True
            r.want_scale_f16 = True
    return _run("export", reqs, True, None, stream, check_status)


def row_clip_select(reqs, stream=None, check_status=True):
    for r in reqs:
        r.want_dq = False
        r.want_clip = True
    return _run("select", reqs, False, None, stream, check_status)


def dequant(packed: torch.Tensor, scale_f16: torch.Tensor, qbits: int, rows: int, cols: int,
            per_tensor: bool = False, out_dtype=torch.float32, stream=None) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=out_dtype, device=packed.device)
    gq_dequant(packed.data_ptr(), scale_f16.data_ptr(), qbits,
               GQ_PER_TENSOR if per_tensor else GQ_PER_ROW, rows, cols, out.data_ptr(),
               _dtype_code(out), stream)
    return out


def gemm_dequant(x: torch.Tensor, packed: torch.Tensor, scale_f16: torch.Tensor, qbits: int,
                 y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X @ W_hat^T with W_hat = bf16(q * s) rebuilt from the export's
    packed codes and binary16 row scales inside the GEMM (tcgen05).  ``x``
    is bf16 [M, K] (rows contiguous), ``packed`` uint8 [N, packed row bytes]
    and ``scale_f16`` fp16 [N]; Y is fp32 [M, N]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with contiguous rows")
    M, K = x.shape
    N = packed.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    gq_gemm_dequant(x.data_ptr(), M, K, x.stride(0), packed.data_ptr(), scale_f16.data_ptr(), qbits, N,
                    y.data_ptr(), y.stride(0), 0, stream)
    return y


def gptq_hessian(x: torch.Tensor, H: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H = 2 X^T X (new fp64 tensor) or H += 2 X^T X (in place) for calibration
    inputs ``x`` fp32 / bf16 [n, cols] with contiguous rows (GPTQ-lite)."""
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D [n, cols] tensor with contiguous rows")
    n, cols = x.shape
    accumulate = H is not None
    if H is None:
        H = torch.empty((cols, cols), dtype=torch.float64, device=x.device)
    elif H.dtype != torch.float64 or H.shape != (cols, cols) or not H.is_contiguous():
        raise ValueError("H must be a contiguous fp64 [cols, cols] tensor")
    _check(LIB.gq_gptq_hessian(x.data_ptr(), _dtype_code(x), n, cols, x.stride(0), H.data_ptr(),
                               int(accumulate), _stream(stream)), "gq_gptq_hessian")
    return H


def gptq_quantize(req: Request, H: torch.Tensor, percdamp: float = 0.01, stream=None,
                  check_status: bool = True) -> Quantized:
    """GPTQ-lite export of ``req.w`` (per row, qbits 6 / 8) against the fp64
    Hessian ``H`` of its inputs; packed codes and binary16 scales are always
    produced, the other outputs as requested."""
    if req.per_tensor or req.qbits not in (6, 8) or req.col_scale is not None:
        raise ValueError("GPTQ-lite takes per-row int6 / int8 requests without column scales")
    r = Request(**{**req.__dict__, "want_packed": True, "want_scale_f16": True, "want_scale_f32": False})
    (d,), (o,) = _prepare([r], True)
    if H.dtype != torch.float64 or not H.is_contiguous() or H.shape != (d.cols, d.cols):
        raise ValueError("H must be a contiguous fp64 [cols, cols] tensor")
    dev = req.w.device
    nbytes = LIB.gq_gptq_workspace_size(d.rows, d.cols)
    ws = _SCRATCH.workspace(dev, nbytes)
    st = _SCRATCH.status(dev, 1)
    _check(LIB.gq_gptq_quantize(C.byref(d), H.data_ptr(), float(percdamp), ws.data_ptr(), ws.numel(),
                                st.data_ptr(), _stream(stream)), "gq_gptq_quantize")
    if check_status:
        o.status = int(st[0].item())
    return o


def gptq_quantize_batch(reqs, Hs, percdamp: float = 0.01, stream=None,
                        check_status: bool = True) -> list:
    """GPTQ-lite of several weights in one call (gq_gptq_quantize_batch): the
    outputs of gptq_quantize for each (request, Hessian) pair, bitwise."""
    if len(reqs) != len(Hs):
        raise ValueError("one Hessian per request")
    rs = []
    for req in reqs:
        if req.per_tensor or req.qbits not in (6, 8) or req.col_scale is not None:
            raise ValueError("GPTQ-lite takes per-row int6 / int8 requests without column scales")
        rs.append(Request(**{**req.__dict__, "want_packed": True, "want_scale_f16": True, "want_scale_f32": False}))
    descs, outs = _prepare(rs, True)
    for d, H in zip(descs, Hs):
        if H.dtype != torch.float64 or not H.is_contiguous() or H.shape != (d.cols, d.cols):
            raise ValueError("each H must be a contiguous fp64 [cols, cols] tensor")
    if not descs:
        return outs
    dev = reqs[0].w.device
    arr = _arr(descs)
    nbytes = LIB.gq_gptq_batch_workspace_size(arr, len(descs))
    ws = _SCRATCH.workspace(dev, nbytes)
    st = _SCRATCH.status(dev, len(descs))
    hp = (C.c_void_p * len(descs))(*[H.data_ptr() for H in Hs])
    _check(LIB.gq_gptq_quantize_batch(arr, len(descs), hp, float(percdamp), ws.data_ptr(), ws.numel(),
                                      st.data_ptr(), _stream(stream)), "gq_gptq_quantize_batch")
    if check_status:
        sv = st[:len(descs)].cpu().tolist()
        for o, v in zip(outs, sv):
            o.status = int(v)
    return outs


def gemm_fakequant(x: torch.Tensor, w: torch.Tensor, clip: torch.Tensor, qbits: int = 6,
                   mode: int = GQ_SCALE_F32, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = X @ W_hat^T with W_hat the fake-quant weight of ``w`` (fp32 / bf16
    [N, K], rows contiguous) under the row clips ``clip`` (fp32 [N]), built in
    the GEMM's weight load (tcgen05); binary32 (GQ_SCALE_F32) or binary16
    (GQ_SCALE_F16) row scales as in gq_fakequant_fwd.  ``x`` is bf16 [M, K]."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with contiguous rows")
    if w.dim() != 2 or w.stride(1) != 1 or clip.dtype != torch.float32 or not clip.is_contiguous():
        raise ValueError("w must be [N, K] with contiguous rows and clip a contiguous fp32 [N] tensor")
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(LIB.gq_gemm_fakequant(x.data_ptr(), M, K, x.stride(0), w.data_ptr(), _dtype_code(w), w.stride(0),
                                 clip.data_ptr(), qbits, mode, N, y.data_ptr(), y.stride(0), None,
                                 _stream(stream)), "gq_gemm_fakequant")
    return y


def ste_bwd(g_out: torch.Tensor, g_w: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """g_w = g_out (new tensor) or g_w += g_out (in place) through libgq."""
    if not g_out.is_contiguous():
        raise ValueError("g_out must be contiguous")
    accumulate = g_w is not None
    if g_w is None:
        g_w = torch.empty_like(g_out)
    elif not g_w.is_contiguous() or g_w.shape != g_out.shape or g_w.dtype != g_out.dtype:
        raise ValueError("g_w must match g_out and be contiguous")
    gq_ste_bwd(g_out.data_ptr(), g_w.data_ptr(), _dtype_code(g_out), g_out.numel(),
               accumulate, stream)
    return g_w


class FakeQuantSTE(torch.autograd.Function):
    """w_hat = fakequant(w) forward; identity (straight-through) backward."""

    @staticmethod
    def forward(ctx, w, qbits=6, p=1.0, per_tensor=False):
        (o,) = fakequant([Request(w.detach(), qbits, p, per_tensor)], check_status=False)
        return o.dq

    @staticmethod
    def backward(ctx, g):
        return ste_bwd(g.contiguous()), None, None, None


def plan_kind(name, shape, is_float, patterns=None, small_numel=65536) -> str:
    return KIND_NAMES[gq_plan_kind(name, tuple(shape), is_float, patterns, small_numel)]


def patterns_from_env() -> str | None:
    return os.environ.get("QUANT_INT8_NAME_PATTERNS")


def export_state_dict(named, p_int6=0.9999, p_int8=0.9999, patterns=None, stream=None):
    """Export a dict name -> tensor with the mixed-bit plan, in ONE batched call.

    Returns name -> (kind, Quantized or tensor).  Non-floating tensors are
    returned as they are.
    """
    patterns = patterns if patterns is not None else patterns_from_env()
    reqs, names, kinds, result = [], [], [], {}
    for name, t in named.items():
        kind = plan_kind(name, tuple(t.shape), t.is_floating_point(), patterns)
        if kind == "raw":
            result[name] = (kind, t)
            continue
        if kind == "fp16":
            w2 = t.reshape(1, -1)
            reqs.append(Request(w2, 16, want_dq=False))
        else:
            w2 = t.reshape(t.shape[0], -1) if t.dim() != 2 else t
            reqs.append(Request(w2, 8 if kind == "int8" else 6,
                                p_int8 if kind == "int8" else p_int6, want_dq=False))
        names.append(name)
        kinds.append(kind)
    outs = export_pack(reqs, stream=stream)
    for name, kind, o in zip(names, kinds, outs):
        result[name] = (kind, o)
    return result
