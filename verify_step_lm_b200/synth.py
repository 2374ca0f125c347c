"""Seeded synthetic inputs for the verify step.

This module is shared by the tests, the benchmark and the scripts that drive
the CPU oracle.  It holds none of the verify step's arithmetic (no softmax, no
top-p, no acceptance test, no dequantised matmul): it only draws random
numbers and lays them out in the shapes the verify step consumes.

* Uniforms come from SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): the 64-bit output for key
  ``seed XOR counter`` is shifted right by 40 and scaled by 2**-24, so every
  uniform is a multiple of 2**-24 in [0, 1) and is exact in fp32 and fp64.
* Gaussian tensors come from a seeded ``torch.Generator`` (CPU or CUDA).
* The group-64 int4 copy of the LM head is the draft head's storage format
  (the pages' "draft-only 4-bit LM head", hazakura.dev MTPLX notes, Layer 0):
  a one-time model-conversion step, not part of the verify step.  The format
  is fixed as symmetric int4, one bf16 scale per 64 consecutive weights of a
  row, ``s = bf16_rne(amax / 7)``, ``q = clamp(rint(w / s), -7, 7)`` (ties to
  even), stored as the nibble ``q + 8``; weight ``2j`` of a row sits in the
  low nibble of byte ``j``.  ``s == 0`` gives ``q == 0``.
"""
from __future__ import annotations

import numpy as np
import torch

SPLITMIX_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
GROUP = 64          # int4 quantisation group (weights per scale)


# --------------------------------------------------------------------------
# uniforms
# --------------------------------------------------------------------------
def splitmix64(keys) -> np.ndarray:
    """First SplitMix64 output for a generator seeded with each key (uint64)."""
    z = np.asarray(keys, dtype=np.uint64) + SPLITMIX_GAMMA
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def uniforms(seed: int, counters) -> np.ndarray:
    """fp32 uniforms on the 2**-24 grid in [0, 1), one per counter."""
    keys = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) ^ np.asarray(counters, dtype=np.uint64)
    bits = splitmix64(keys) >> np.uint64(40)
    return (bits.astype(np.float64) * 2.0 ** -24).astype(np.float32)


def slots_per_sequence(K: int) -> int:
    """Uniform slots per (trial, sequence): K accept, K+1 sample, K draft."""
    return 3 * K + 1


def step_uniforms(seed: int, trial: int, B: int, K: int) -> dict:
    """Uniforms for one verify step of B sequences with K drafts each.

    Counter of slot ``s`` of sequence ``b`` in trial ``t`` is
    ``(t * B + b) * (3K + 1) + s``; slots ``[0, K)`` are the acceptance
    uniforms, ``[K, 2K+1)`` the sampling uniforms (one per position, the
    residual/bonus draw uses the one at the first rejected position, or at K),
    ``[2K+1, 3K+1)`` the uniforms used to draw the draft tokens themselves.
    """
    S = slots_per_sequence(K)
    base = (np.uint64(trial) * np.uint64(B) + np.arange(B, dtype=np.uint64)) * np.uint64(S)
    ctr = base[:, None] + np.arange(S, dtype=np.uint64)[None, :]
    u = uniforms(seed, ctr)
    return {
        "u_accept": np.ascontiguousarray(u[:, :K]),
        "u_sample": np.ascontiguousarray(u[:, K:2 * K + 1]),
        "u_draft": np.ascontiguousarray(u[:, 2 * K + 1:]),
    }


# --------------------------------------------------------------------------
# gaussian tensors
# --------------------------------------------------------------------------
def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian(shape, std: float, seed: int, device="cpu", dtype=torch.bfloat16,
             chunk_rows: int = 8192) -> torch.Tensor:
    """N(0, std^2) values drawn in fp32 and rounded to ``dtype``.

    Large tensors are drawn in row chunks (each chunk from its own seed
    derived from ``seed``) so that host memory stays bounded; the result only
    depends on (shape, std, seed, chunk_rows, device type).
    """
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    out = torch.empty(shape, dtype=dtype, device=device)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        g = _gen(int(splitmix64(np.uint64(seed) ^ np.uint64(r0))) & 0x7FFFFFFFFFFFFFFF, device)
        x = torch.randn((r1 - r0,) + shape[1:], generator=g, dtype=torch.float32, device=device)
        out[r0:r1] = (x * std).to(dtype)
    return out


def make_head(V: int, h: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """Target LM head W[V, h] bf16 ~ N(0, std^2) (nn.Linear out x in layout)."""
    return gaussian((V, h), std, seed, device)


def make_hidden(B: int, K: int, h: int, sigma: float, seed: int, device="cpu"):
    """Hidden states for B sequences.

    Ht [B*(K+1), h] bf16 ~ N(0,1); Hd [B*K, h] = bf16(Ht[b,i] + N(0, sigma^2))
    for the first K positions of every sequence (the draft rows are noisy
    copies of the target rows, which sets the acceptance rate).
    """
    Ht = gaussian((B * (K + 1), h), 1.0, seed, device)
    noise = gaussian((B * K, h), 1.0, seed ^ 0x5EED, device, dtype=torch.float32)
    base = Ht.view(B, K + 1, h)[:, :K, :].reshape(B * K, h).float()
    Hd = (base + sigma * noise).to(torch.bfloat16)
    return Ht.contiguous(), Hd.contiguous()


def make_logits(rows: int, V: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """fp32 logits rows ~ N(0, std^2) (the statistics of a random-weight head)."""
    return gaussian((rows, V), std, seed, device, dtype=torch.float32)


def make_verify_logits(B: int, K: int, V: int, std: float, tau: float, seed: int,
                       device="cpu", grid: float | None = None):
    """Target logits [B, K+1, V] and draft logits [B, K, V] (fp32).

    Draft row i of a sequence is target row i plus N(0, tau^2).  With
    ``grid`` set, every logit is rounded to a multiple of ``grid`` so that
    exact ties are common (exercises the lower-index tie rule).
    """
    t = make_logits(B * (K + 1), V, std, seed, device).view(B, K + 1, V)
    n = make_logits(B * K, V, tau, seed ^ 0xD4AF7, device).view(B, K, V)
    d = t[:, :K, :] + n
    if grid:
        t = torch.round(t / grid) * grid
        d = torch.round(d / grid) * grid
    return t.contiguous(), d.contiguous()


# --------------------------------------------------------------------------
# int4 group-64 storage of the draft head (model conversion, see module doc)
# --------------------------------------------------------------------------
def quantize_int4_g64(W: torch.Tensor, chunk_rows: int = 16384):
    """Return (Wq uint8 [N, Kd/2], S bf16 [N, Kd/64]) for bf16 W [N, Kd]."""
    assert W.dtype == torch.bfloat16 and W.dim() == 2
    N, Kd = W.shape
    assert Kd % GROUP == 0, "row length must be a multiple of 64"
    Wq = torch.empty((N, Kd // 2), dtype=torch.uint8, device=W.device)
    S = torch.empty((N, Kd // GROUP), dtype=torch.bfloat16, device=W.device)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        w = W[r0:r1].float().view(r1 - r0, Kd // GROUP, GROUP)
        amax = w.abs().amax(dim=2)
        s = (amax / 7.0).to(torch.bfloat16)
        sf = s.float().unsqueeze(2)
        q = torch.where(sf > 0, torch.round(w / torch.where(sf > 0, sf, torch.ones_like(sf))),
                        torch.zeros_like(w))
        q = q.clamp_(-7, 7).to(torch.int32) + 8
        q = q.view(r1 - r0, Kd)
        packed = (q[:, 0::2] | (q[:, 1::2] << 4)).to(torch.uint8)
        Wq[r0:r1] = packed
        S[r0:r1] = s
    return Wq.contiguous(), S.contiguous()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bits of a CPU bf16 tensor as a numpy array (no copy)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
