"""CPU oracle for the speculative-decoding verify step (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``verify_step_lm_b200`` never does, and this package imports nothing from it.

The arithmetic lives in ``mtpv_oracle.c`` (plain C, fp64, no BLAS); this file
only compiles it with gcc and marshals numpy arrays.  Each wrapper names the
passage of the pages it follows:

* ``lm_head_bf16`` / ``lm_head_int4g64`` -- the K+1 target rows through the
  bf16 LM head and the K draft rows through the draft-only 4-bit head
  (hazakura.dev MTPLX notes, "4-layer architecture", Layer 0).
* ``warp`` -- temperature softmax then top-p (devtrends.cc MTPLX overview:
  temperature=0.6 / top_p=0.95 sampling is reproduced exactly).
* ``verify`` / ``verify_dist`` -- Leviathan-Chen acceptance, residual
  correction and bonus token (devtrends.cc overview; hazakura.dev notes,
  Layer 2 cycle).
* ``sample_rows`` -- one draw from each row's warped distribution (the draft
  phase's own sampling step, hazakura.dev notes, Layer 2 "Draft").
* ``silu_mul`` / ``gate_up_int4g64`` -- the gated MLP of a decoder layer:
  silu(x . G^T) * (x . U^T) with an int4 g64 gate||up head (the matmuls of
  the small-M regime beyond the LM head, hazakura.dev notes, Layer 0;
  gist.science BaseRT explainer, fused op chains).  Plain numpy in fp64.

Every function here is pinned by tests in ``tests/test_oracle_*.py`` against
closed forms, brute force on tiny inputs and independent library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mtpv_oracle.c")
_LIB = os.path.join(_HERE, "libmtpv_oracle.so")

FLAG_RATIO = 1
FLAG_DRAW = 2
FLAG_TOPP = 4
WINDOW = 1e-5

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.mtpvo_lm_head_bf16.argtypes = [P, I, I, I, P, P, I, I]
        lib.mtpvo_lm_head_int4g64.argtypes = [P, I, I, I, P, P, P, I, I]
        lib.mtpvo_quantize_int4g64.argtypes = [P, I, I, P, P]
        lib.mtpvo_warp.argtypes = [P, I, D, D, P, P]
        lib.mtpvo_warp.restype = I
        lib.mtpvo_draw.argtypes = [P, I, D, P]
        lib.mtpvo_draw.restype = I
        lib.mtpvo_verify.argtypes = [P, P, P, P, P, I, I, I, D, D, P, P, P, P, P]
        lib.mtpvo_verify_dist.argtypes = [P, P, P, I, I, D, D, P, P, P]
        lib.mtpvo_verify_dist.restype = I
        lib.mtpvo_sample_rows.argtypes = [P, I, I, D, D, P, P, P, P]
        for f in (lib.mtpvo_lm_head_bf16, lib.mtpvo_lm_head_int4g64, lib.mtpvo_quantize_int4g64,
                  lib.mtpvo_verify, lib.mtpvo_sample_rows):
            f.restype = None
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _split(n: int, parts: int):
    parts = max(1, min(parts, n))
    edges = [n * i // parts for i in range(parts + 1)]
    return list(zip(edges[:-1], edges[1:]))


# ---------------------------------------------------------------------------
# LM heads
# ---------------------------------------------------------------------------
def lm_head_bf16(x_bits: np.ndarray, W_bits: np.ndarray, threads: int = 1,
                 rows: tuple[int, int] | None = None) -> np.ndarray:
    """fp64 logits y[M, N] = x . W^T for bf16 bit patterns x [M,Kd], W [N,Kd].

    ``rows=(n0, n1)`` computes only vocabulary rows n0..n1-1 (the rest of the
    output stays 0), for spot checks of large heads.
    """
    lib = _load()
    x = _c(x_bits, np.uint16)
    W = _c(W_bits, np.uint16)
    M, Kd = x.shape
    N = W.shape[0]
    assert W.shape[1] == Kd
    y = np.zeros((M, N), dtype=np.float64)
    n0, n1 = rows if rows else (0, N)
    jobs = [(n0 + a, n0 + b) for a, b in _split(n1 - n0, threads)]
    with ThreadPoolExecutor(len(jobs)) as ex:
        list(ex.map(lambda r: lib.mtpvo_lm_head_bf16(_p(x), M, Kd, N, _p(W), _p(y), r[0], r[1]), jobs))
    return y


def lm_head_int4g64(x_bits: np.ndarray, Wq: np.ndarray, S_bits: np.ndarray, threads: int = 1,
                    rows: tuple[int, int] | None = None) -> np.ndarray:
    """fp64 draft logits through the int4 group-64 head (see mtpv_oracle.c)."""
    lib = _load()
    x = _c(x_bits, np.uint16)
    q = _c(Wq, np.uint8)
    S = _c(S_bits, np.uint16)
    M, Kd = x.shape
    N = q.shape[0]
    assert Kd % 64 == 0 and q.shape[1] * 2 == Kd and S.shape == (N, Kd // 64)
    y = np.zeros((M, N), dtype=np.float64)
    n0, n1 = rows if rows else (0, N)
    jobs = [(n0 + a, n0 + b) for a, b in _split(n1 - n0, threads)]
    with ThreadPoolExecutor(len(jobs)) as ex:
        list(ex.map(lambda r: lib.mtpvo_lm_head_int4g64(_p(x), M, Kd, N, _p(q), _p(S), _p(y),
                                                        r[0], r[1]), jobs))
    return y


def quantize_int4g64(W_bits: np.ndarray):
    """(Wq uint8 [N, Kd/2], S bf16 bits [N, Kd/64]) of bf16 bit patterns W."""
    lib = _load()
    W = _c(W_bits, np.uint16)
    N, Kd = W.shape
    assert Kd % 64 == 0
    Wq = np.zeros((N, Kd // 2), dtype=np.uint8)
    S = np.zeros((N, Kd // 64), dtype=np.uint16)
    lib.mtpvo_quantize_int4g64(_p(W), N, Kd, _p(Wq), _p(S))
    return Wq, S


# ---------------------------------------------------------------------------
# sampler
# ---------------------------------------------------------------------------
_INFO_KEYS = ("m", "Z", "kept_sum", "kept", "cut_token", "next_token", "gap_lo", "gap_hi",
              "p_cut", "p_next")


def warp(logits: np.ndarray, T: float, top_p: float):
    """(p', info) for one row of logits (fp64)."""
    lib = _load()
    l = _c(logits, np.float64)
    V = l.shape[0]
    p = np.zeros(V, dtype=np.float64)
    info = np.zeros(10, dtype=np.float64)
    st = lib.mtpvo_warp(_p(l), V, float(T), float(top_p), _p(p), _p(info))
    d = dict(zip(_INFO_KEYS, info.tolist()))
    d["status"] = st
    return p, d


def draw(w: np.ndarray, u: float):
    """(x, margin relative to w_x) of the inverse-CDF draw from weights w."""
    lib = _load()
    w = _c(w, np.float64)
    m = np.zeros(1, dtype=np.float64)
    x = lib.mtpvo_draw(_p(w), w.shape[0], float(u), _p(m))
    return x, float(m[0])


def verify(target_logits, draft_logits, drafts, u_accept, u_sample, T: float, top_p: float,
           threads: int = 1) -> dict:
    """Sampling mode for B sequences.

    target_logits [B, K+1, V], draft_logits [B, K, V] (any float type, widened
    to fp64), drafts [B, K] int, u_accept [B, K], u_sample [B, K+1] fp32.
    Returns tokens [B, K+1] (-1 padded), accepted [B], status [B],
    flags [B] (FLAG_*), margins [B, 3] (ratio, draw relative, top-p relative).
    """
    lib = _load()
    tl = _c(target_logits, np.float64)
    dl = _c(draft_logits, np.float64)
    d = _c(drafts, np.int32)
    ua = _c(u_accept, np.float32)
    us = _c(u_sample, np.float32)
    B, K1, V = tl.shape
    K = K1 - 1
    assert dl.shape == (B, K, V) and d.shape == (B, K) and ua.shape == (B, K) and us.shape == (B, K1)
    out = {
        "tokens": np.zeros((B, K1), dtype=np.int32),
        "accepted": np.zeros(B, dtype=np.int32),
        "status": np.zeros(B, dtype=np.int32),
        "flags": np.zeros(B, dtype=np.int32),
        "margins": np.zeros((B, 3), dtype=np.float64),
    }

    def run(r):
        b0, b1 = r
        nb = b1 - b0
        lib.mtpvo_verify(_p(tl[b0:b1]), _p(dl[b0:b1]), _p(d[b0:b1]), _p(ua[b0:b1]), _p(us[b0:b1]),
                         nb, K, V, float(T), float(top_p),
                         _p(out["tokens"][b0:b1]), _p(out["accepted"][b0:b1]),
                         _p(out["status"][b0:b1]), _p(out["flags"][b0:b1]),
                         _p(out["margins"][b0:b1]))

    jobs = _split(B, threads)
    with ThreadPoolExecutor(len(jobs)) as ex:
        list(ex.map(run, jobs))
    return out


def verify_dist(target_logits, draft_logits, drafts, T: float, top_p: float):
    """Distribution mode for one sequence: (acc [K], res [K, V], bonus [V], status)."""
    lib = _load()
    tl = _c(target_logits, np.float64)
    dl = _c(draft_logits, np.float64)
    d = _c(drafts, np.int32)
    K1, V = tl.shape
    K = K1 - 1
    acc = np.zeros(K, dtype=np.float64)
    res = np.zeros((K, V), dtype=np.float64)
    bonus = np.zeros(V, dtype=np.float64)
    st = lib.mtpvo_verify_dist(_p(tl), _p(dl), _p(d), K, V, float(T), float(top_p),
                               _p(acc), _p(res), _p(bonus))
    return acc, res, bonus, st


def sample_rows(logits, T: float, top_p: float, u, threads: int = 1):
    """(tokens [R], margins [R], status [R]): one draw from each row's p'."""
    lib = _load()
    l = _c(logits, np.float64)
    R, V = l.shape
    uu = _c(u, np.float32).reshape(R)
    out = np.zeros(R, dtype=np.int32)
    mr = np.zeros(R, dtype=np.float64)
    st = np.zeros(R, dtype=np.int32)

    def run(r):
        a, b = r
        lib.mtpvo_sample_rows(_p(l[a:b]), b - a, V, float(T), float(top_p), _p(uu[a:b]),
                              _p(out[a:b]), _p(mr[a:b]), _p(st[a:b]))

    jobs = _split(R, threads)
    with ThreadPoolExecutor(len(jobs)) as ex:
        list(ex.map(run, jobs))
    return out, mr, st


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """silu(g) * u elementwise in fp64, silu(g) = g / (1 + exp(-g))."""
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def gate_up_int4g64(x_bits: np.ndarray, Wq: np.ndarray, S_bits: np.ndarray, F: int,
                    cols=None, threads: int = 1) -> np.ndarray:
    """h[M, F] (or the columns ``cols`` of it) = silu(x . G^T) * (x . U^T) for
    the int4 g64 head [2F, Kd] whose rows 0..F-1 are G and F..2F-1 are U."""
    cols = np.arange(F) if cols is None else np.asarray(cols)
    g = lm_head_int4g64(x_bits, Wq[cols], S_bits[cols], threads=threads)
    u = lm_head_int4g64(x_bits, Wq[F + cols], S_bits[F + cols], threads=threads)
    return silu_mul(g, u)
