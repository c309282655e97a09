"""Comparison helpers and tolerances shared by the GPU parity tests.

Tolerances (bf16 storage with fp32 accumulation, against the fp64 oracle):
logits relative L2 <= 1e-2, max absolute <= 5e-2, loss absolute <= 1e-2,
top-1 agreement >= 99.5%; all-fp32 mode: relative L2 <= 1e-4.
Top-1 is reported two ways: literally (same argmax index) and tie-aware
(the oracle logit of the GPU's argmax is within the max-abs tolerance of the
oracle's maximum), because random-init logits hold many near-ties that
bf16 rounding can legitimately reorder.
"""
import numpy as np

BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 5e-2
BF16_LOSS_ABS = 1e-2
BF16_TOP1 = 0.995
FP32_REL_L2 = 1e-4


def rel_l2(a, ref) -> float:
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm((a - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_abs(a, ref) -> float:
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(ref, np.float64)).max())


def top1(gpu_logits, ref_logits, tie_tol=BF16_MAX_ABS):
    """(literal agreement, tie-aware agreement) over all rows."""
    g = np.asarray(gpu_logits).reshape(-1, gpu_logits.shape[-1])
    r = np.asarray(ref_logits).reshape(-1, ref_logits.shape[-1])
    ga = g.argmax(-1)
    ra = r.argmax(-1)
    literal = float((ga == ra).mean())
    rmax = r.max(-1)
    picked = np.take_along_axis(r, ga[:, None], -1)[:, 0]
    tie_aware = float((rmax - picked <= tie_tol).mean())
    return literal, tie_aware
