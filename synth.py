"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and arranges them into named tensors.  It
holds none of the quantization arithmetic, and neither the oracle nor the CUDA
library is imported here.  Every tensor is synthetic: the pages' models are
trained on FineWeb-style text that is not available, so weights of the same
shapes and of the stated distributions stand in for them.

Recipes (all draws in float64, scaled in float64, rounded once to fp32; bf16
copies are the round-to-nearest-even of the fp32 values):

* ``normal(std)``: ``std * z`` with ``z`` standard normal.
* ``student_t3(std)``: Student-t with 3 degrees of freedom rescaled to the
  given standard deviation, ``t = z0 / sqrt((z1^2 + z2^2 + z3^2) / 3)``
  (the textbook construction), times ``std / sqrt(3)``.
* ``outlier_mix``: ``z`` standard normal, ``u`` uniform [0, 1);
  ``0.2 z`` where ``u < 0.01`` else ``0.02 z``.
* ``awq_col_scales(cols)``: per-input-column activation statistics
  ``a = |z0| * exp(1.5 z1)`` (a few channels far louder than the rest), and
  the column scales a quantizer takes from them in the AWQ style,
  ``t = a^0.5 / sqrt(max(a^0.5) * min(a^0.5))`` in float64, rounded to fp32.
  The pages give no rule from statistics to scales; this only draws an input
  of the right kind.

Host workloads use ``numpy.random.default_rng(seed)`` with tensors drawn in the
manifest order below; the bandwidth workload is drawn on the GPU from a seeded
``torch.Generator`` (it is 2.5 GiB of fp32, too slow to draw on the host).
"""
from __future__ import annotations

import functools
import math
from dataclasses import dataclass, field

import numpy as np


@dataclass
class Spec:
    """One named weight of a workload and how it is to be quantized."""
    name: str
    shape: tuple
    qbits: int = 6          # 6, 8, or 16 (fp16 passthrough)
    p: float = 1.0
    per_tensor: bool = False


@dataclass
class Workload:
    name: str
    seed: int
    specs: list = field(default_factory=list)
    dtype: str = "f32"      # "f32" or "bf16"


# ----------------------------------------------------------------- helpers --

def _normal(rng, n, std):
    return (rng.standard_normal(n) * std).astype(np.float32)


def _student_t3(rng, n, std, chunk=1 << 20):
    out = np.empty(n, np.float32)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        z = rng.standard_normal((4, m))
        t = z[0] / np.sqrt((z[1] ** 2 + z[2] ** 2 + z[3] ** 2) / 3.0)
        out[i:i + m] = t * (std / math.sqrt(3.0))
    return out


def _outlier_mix(rng, n):
    z = rng.standard_normal(n)
    u = rng.random(n)
    return np.where(u < 0.01, 0.2 * z, 0.02 * z).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 -> bf16 (nearest even) via torch; returns uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------- the workloads --

def single_matrix() -> Workload:
    """One fp32 512x1536 matrix, N(0, 0.02^2), int6 per row at p = 1 (absmax)."""
    return Workload("single fp32 512x1536 int6 absmax", 0,
                    [Spec("w", (512, 1536), 6, 1.0)])


def gpt9_specs(layers=9, d=512, kv=256, mlp=1536, vocab=1024, p6=0.9999, p8=0.9999):
    """Full parameter set of a 9-layer GPT (d 512, 8 query / 4 KV heads of 64,
    MLP 1536, vocab 1024, tied embeddings) as in the SubSixteen v2 page."""
    specs = [Spec("tok_emb.weight", (vocab, d), 8, p8)]
    for i in range(layers):
        b = f"blocks.{i}."
        specs += [
            Spec(b + "attn.c_q.weight", (d, d), 6, p6),
            Spec(b + "attn.c_k.weight", (kv, d), 6, p6),
            Spec(b + "attn.c_v.weight", (kv, d), 6, p6),
            Spec(b + "attn.proj.weight", (d, d), 6, p6),
            Spec(b + "attn.q_gain", (d,), 16),
            Spec(b + "attn_scale", (d,), 16),
            Spec(b + "mlp_scale", (d,), 16),
            Spec(b + "mlp.fc.weight", (mlp, d), 6, p6),
            Spec(b + "mlp.proj.weight", (d, mlp), 6, p6),
        ]
    return specs


def gpt9_export() -> Workload:
    return Workload("9-layer GPT d512 export (int6 p=.9999, int8 tok_emb, fp16 vectors)",
                    1, gpt9_specs())


def unified11_train() -> Workload:
    """11 layers, d 528, 4 heads, 3x MLP, unified QKV projection; bf16 weights,
    int6 per-row absmax fake-quant for training."""
    specs = []
    for i in range(11):
        b = f"blocks.{i}."
        specs += [
            Spec(b + "attn.unified.weight", (1584, 528), 6, 1.0),
            Spec(b + "attn.proj.weight", (528, 528), 6, 1.0),
            Spec(b + "mlp.fc.weight", (1584, 528), 6, 1.0),
            Spec(b + "mlp.proj.weight", (528, 1584), 6, 1.0),
        ]
    return Workload("11-layer unified-attention d528 bf16 QAT", 2, specs, "bf16")


def gpt12_mixed_specs():
    specs = [
        Spec("tok_emb.weight", (1792, 512), 8, 0.9999),
        Spec("lm_head.weight", (1792, 512), 8, 0.9999),
        Spec("bigram.embed.weight", (2048, 128), 8, 0.9999),
    ]
    for i in range(12):
        b = f"blocks.{i}."
        for nm, shp in (("attn.c_q.weight", (512, 512)), ("attn.c_k.weight", (256, 512)),
                        ("attn.c_v.weight", (256, 512)), ("attn.proj.weight", (512, 512)),
                        ("mlp.fc.weight", (1536, 512)), ("mlp.proj.weight", (512, 1536))):
            specs.append(Spec(b + nm, shp, 6, 0.999))
    return specs


def gpt12_mixed() -> Workload:
    """12 layers, d 512, GQA 8/4, MLP 1536, vocab 1792: embeddings and head
    int8, block matrices int6 at p = .999, plus a BigramHash 2048x128 table."""
    return Workload("12-layer GPT vocab1792 mixed-bit export", 3, gpt12_mixed_specs())


BANDWIDTH_SHAPES = ((16384, 16384), (65536, 4096), (262144, 512))


# ------------------------------------------------------------------ draws --

def draw_single_matrix():
    """(W, G): W ~ N(0, 0.02^2) and a N(0, 1) gradient, both fp32 512x1536."""
    rng = np.random.default_rng(0)
    w = _normal(rng, 512 * 1536, 0.02).reshape(512, 1536)
    g = _normal(rng, 512 * 1536, 1.0).reshape(512, 1536)
    return w, g


@functools.lru_cache(maxsize=1)
def draw_gpt9():
    """Dict name -> fp32 array, Student-t(3) scaled to std 0.02, seed 1.
    Cached: callers must not modify the arrays."""
    rng = np.random.default_rng(1)
    out = {}
    for s in gpt9_specs():
        n = int(np.prod(s.shape))
        out[s.name] = _student_t3(rng, n, 0.02).reshape(s.shape)
    return out


def draw_unified11():
    """Dict name -> bf16 bit patterns (uint16), N(0, 0.02^2) rounded, seed 2."""
    rng = np.random.default_rng(2)
    out = {}
    for s in unified11_train().specs:
        n = int(np.prod(s.shape))
        out[s.name] = to_bf16_bits(_normal(rng, n, 0.02)).reshape(s.shape)
    return out


def draw_gpt12():
    """Dict name -> fp32 array, 1 % N(0, 0.2^2) outliers in N(0, 0.02^2), seed 3."""
    rng = np.random.default_rng(3)
    out = {}
    for s in gpt12_mixed_specs():
        n = int(np.prod(s.shape))
        out[s.name] = _outlier_mix(rng, n).reshape(s.shape)
    return out


def training_step_noise(shape, iteration, device="cpu", seed=2):
    """(grad, perturbation) for one training iteration of the 11-layer model:
    grad ~ N(0, 1e-3^2) and perturbation ~ N(0, 1e-4^2), fp32, drawn from a
    torch generator seeded (seed, iteration)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + iteration)
    grad = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * 1e-3
    pert = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * 1e-4
    return grad, pert


def draw_bandwidth_matrix(rows, cols, index, device="cuda", seed=4, chunk_rows=None):
    """Student-t(3) fp32 [rows, cols] scaled to std 0.02, drawn on ``device``
    from a torch generator seeded (seed, index), in row chunks."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + index)
    out = torch.empty((rows, cols), dtype=torch.float32, device=device)
    chunk_rows = chunk_rows or max(1, (1 << 26) // cols)
    scale = 0.02 / math.sqrt(3.0)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        z = torch.randn((4, r1 - r0, cols), generator=g, device=device, dtype=torch.float32)
        chi = (z[1] * z[1] + z[2] * z[2] + z[3] * z[3]) / 3.0
        out[r0:r1] = z[0] / torch.sqrt(chi) * scale
    return out


def random_matrix(rng, rows, cols, kind="normal"):
    """Small fp32 test matrices of assorted distributions (tests only)."""
    n = rows * cols
    if kind == "normal":
        x = _normal(rng, n, 0.02)
    elif kind == "t3":
        x = _student_t3(rng, n, 0.02)
    elif kind == "mix":
        x = _outlier_mix(rng, n)
    elif kind == "ties":
        x = (rng.integers(-8, 9, n) * 0.125).astype(np.float32)
    elif kind == "tiny":
        # magnitudes near 2^-20, where binary16 scales fall in the subnormal range
        x = (rng.standard_normal(n) * 2.0 ** -20).astype(np.float32)
    elif kind == "zeros":
        x = np.zeros(n, np.float32)
    else:
        raise ValueError(kind)
    return x.reshape(rows, cols)


def awq_col_scales(rng, cols):
    """fp32 [cols] column scales drawn from synthetic activation statistics
    (recipe in the module docstring)."""
    a = np.abs(rng.standard_normal(cols)) * np.exp(1.5 * rng.standard_normal(cols)) + 1e-3
    r = np.sqrt(a)
    return (r / math.sqrt(r.max() * r.min())).astype(np.float32)


def gptq_calibration(rng, n, cols, rho=0.8, dead=()):
    """Synthetic layer inputs for GPTQ-lite calibration: fp32 [n, cols], one
    row per token.  Neighbouring features are correlated (AR(1) with
    coefficient ``rho`` across the feature index) and every feature has its
    own log-normal magnitude (a few large-activation channels), as the inputs
    of a transformer layer have.  Columns listed in ``dead`` are zero (inputs
    that are never active)."""
    z = rng.standard_normal((n, cols))
    x = np.empty_like(z)
    x[:, 0] = z[:, 0]
    k = math.sqrt(1.0 - rho * rho)
    for j in range(1, cols):
        x[:, j] = rho * x[:, j - 1] + k * z[:, j]
    x *= np.exp(0.5 * rng.standard_normal(cols))[None, :]
    for j in dead:
        x[:, j] = 0.0
    return x.astype(np.float32)


def unified11_gptq_inputs():
    """Per layer of the 11-layer d528 model, the input dimension of each of its
    four weights (unified projection, out-projection, MLP up, MLP down), in the
    order of unified11_train().specs."""
    return [s.shape[1] for s in unified11_train().specs]


def random_packed_codes(rng, rows, row_bytes):
    """Arbitrary packed code bytes [rows, row_bytes] (uint8): inputs for the
    consuming GEMM, which accepts any 6- or 8-bit field."""
    return rng.integers(0, 256, (rows, row_bytes), dtype=np.uint8)


def random_f16_scales(rng, rows, lo=2.0 ** -12, hi=2.0 ** -5):
    """Positive binary16 row scales as uint16 bit patterns, log-uniform in
    [lo, hi] (normal binary16 numbers)."""
    v = np.exp(rng.uniform(math.log(lo), math.log(hi), rows)).astype(np.float16)
    return v.view(np.uint16)
