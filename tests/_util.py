"""Shared helpers for the GPU parity tests (tolerances, float32 views)."""
import numpy as np
import torch

# LM-head tolerance: fp32 accumulation versus the oracle's fp64.  Per element
# |gpu - ref| <= 1e-3 * max(|ref|, rms(ref row)), so near-zero logits are not
# held to a relative bound they cannot have.
LOGIT_RTOL = 1e-3


def assert_logits_close(gpu: np.ndarray, ref: np.ndarray, rtol: float = LOGIT_RTOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    scale = np.maximum(np.abs(ref), rms)
    err = np.abs(gpu - ref)
    bad = err > rtol * scale
    assert not bad.any(), (
        f"{bad.sum()} of {bad.size} logits off; worst rel {np.max(err / np.maximum(scale, 1e-300)):.3e}")
    return float(np.max(err / np.maximum(scale, 1e-300)))


def f32(x: float) -> float:
    """The value a float argument has after the C ABI narrows it to fp32."""
    return float(np.float32(x))


def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to("cuda")
