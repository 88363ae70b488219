"""Export plan oracle: how each named tensor of a state dict is stored.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources: "Swiglu gating_ QAT_..." (parameter-golf PR #2159), Key Explored
Modifications 16 (small tensors pass through as FP16); "... Int6AWQ
MixedBits" (PR #1495), "Mixed-bit quantization details": int6 is the default
export, tensors named by ``QUANT_INT8_NAME_PATTERNS`` are promoted to int8, and
the default list is ``tok_emb.weight`` and ``lm_head.weight``.

Readings (the pages give neither a threshold nor a match rule):
  * "small" means fewer than 65536 elements;
  * a pattern matches when it is a substring of the tensor name; the
    environment variable holds a comma-separated list;
  * precedence: non-floating -> raw, small -> fp16, pattern -> int8,
    everything else -> int6 per row; a tensor that is not 2-D is viewed as
    [shape[0], numel / shape[0]].
"""
from __future__ import annotations

DEFAULT_INT8_PATTERNS = ("tok_emb.weight", "lm_head.weight")
SMALL_NUMEL = 65536


def patterns_from_env(value: str | None) -> tuple[str, ...]:
    if value is None:
        return DEFAULT_INT8_PATTERNS
    return tuple(s.strip() for s in value.split(",") if s.strip())


def classify(name: str, shape: tuple[int, ...], is_float: bool,
             patterns: tuple[str, ...] = DEFAULT_INT8_PATTERNS,
             small_numel: int = SMALL_NUMEL) -> tuple[str, tuple[int, int] | None]:
    """Return (kind, 2-D view) with kind in {"raw", "fp16", "int8", "int6"}."""
    numel = 1
    for d in shape:
        numel *= d
    if not is_float:
        return "raw", None
    if numel < small_numel:
        return "fp16", None
    for pat in patterns:
        if pat in name:
            return "int8", _view2d(shape, numel)
    return "int6", _view2d(shape, numel)


def _view2d(shape: tuple[int, ...], numel: int) -> tuple[int, int]:
    if len(shape) == 2:
        return (shape[0], shape[1])
    if len(shape) == 0 or shape[0] == 0:
        return (1, numel)
    return (shape[0], numel // shape[0])
