"""verify_step_lm_b200: the speculative-decoding verify step on NVIDIA B200.

A thin ctypes binding over ``libmtpv.so`` (C ABI in ``include/mtpv.h``).  The
functions here only marshal arguments: every step of the verify path runs in
the library's sm_100a kernels.  PyTorch provides device memory and the CUDA
stream (the current stream of the tensors' device).  There is no CPU fallback:
if the library is missing or fails to load, every call raises.

Public functions mirror the C names without the ``mtpv_`` prefix:
``lm_head_smallm``, ``verify``, ``sample``, ``verify_step``,
``verify_step_host`` and the ``*_workspace_bytes`` queries.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmtpv.so")

OK = 0
W_BF16 = 0
W_INT4_G64 = 1
ROW_OK, ROW_BAD_DRAFT, ROW_NONFINITE, ROW_TIMEOUT = 0, 1, 2, 3

_lib = None


class MtpvError(RuntimeError):
    """A libmtpv call returned a non-zero status."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libmtpv.so from this package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmtpv.so not built ({LIB_PATH}); run python -m verify_step_lm_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "mtpv_version": ([], I),
        "mtpv_set_wait_polls": ([I], None),
        "mtpv_status_string": ([I], ctypes.c_char_p),
        "mtpv_lm_head_workspace_bytes": ([I, I, I, I], Z),
        "mtpv_lm_head_smallm": ([P, I, I, I, P, P, I, P, P, Z, P], I),
        "mtpv_lm_head_pair_workspace_bytes": ([I, I, I, I], Z),
        "mtpv_lm_head_pair": ([P, I, P, P, P, I, P, P, P, I, I, P, Z, P], I),
        "mtpv_int4_proj_workspace_bytes": ([I, I, I], Z),
        "mtpv_int4_proj": ([P, I, I, I, P, P, P, P, Z, P], I),
        "mtpv_int4_gate_up_workspace_bytes": ([I, I, I], Z),
        "mtpv_int4_gate_up": ([P, I, I, I, P, P, P, P, Z, P], I),
        "mtpv_verify_workspace_bytes": ([I, I, I], Z),
        "mtpv_verify": ([P, P, P, P, P, I, I, I, F, F, P, P, P, P, Z, P], I),
        "mtpv_sample_workspace_bytes": ([I, I], Z),
        "mtpv_sample": ([P, I, I, F, F, P, P, P, P, Z, P], I),
        "mtpv_draft_loop_workspace_bytes": ([I, I, I, I], Z),
        "mtpv_draft_loop": ([P, P, P, P, I, I, I, I, F, F, P, P, P, Z, P], I),
        "mtpv_verify_step_workspace_bytes": ([I, I, I, I], Z),
        "mtpv_verify_step": ([P, P, P, P, P, P, P, P, I, I, I, I, F, F, P, P, P, P, P, P, Z, P], I),
        "mtpv_verify_step_host_workspace_bytes": ([I, I, I, I], Z),
        "mtpv_verify_step_host": ([P, P, P, P, P, P, P, P, I, I, I, I, F, F, P, P, P, P, Z, P], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _ptr(t):
    # a plain int (or None for NULL): ctypes converts it for a c_void_p argument
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, st: int):
    if st != OK:
        raise MtpvError(fn, st, load().mtpv_status_string(st).decode())


def version() -> int:
    return load().mtpv_version()


def set_wait_polls(polls: int) -> None:
    """Bound of the sampler's device-side waits (polls; < 0: the default)."""
    load().mtpv_set_wait_polls(int(polls))


def status_string(st: int) -> str:
    return load().mtpv_status_string(st).decode()


# ---------------------------------------------------------------------------
# workspace queries
# ---------------------------------------------------------------------------
def lm_head_workspace_bytes(M: int, Kd: int, N: int, fmt: int) -> int:
    return load().mtpv_lm_head_workspace_bytes(M, Kd, N, fmt)


def verify_workspace_bytes(B: int, K: int, V: int) -> int:
    return load().mtpv_verify_workspace_bytes(B, K, V)


def sample_workspace_bytes(R: int, V: int) -> int:
    return load().mtpv_sample_workspace_bytes(R, V)


def verify_step_workspace_bytes(B: int, K: int, V: int, h: int) -> int:
    return load().mtpv_verify_step_workspace_bytes(B, K, V, h)


def verify_step_host_workspace_bytes(B: int, K: int, V: int, h: int) -> int:
    return load().mtpv_verify_step_host_workspace_bytes(B, K, V, h)


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled device byte buffer of at least ``nbytes`` (256-byte
    aligned); the projections' workspaces must start zeroed."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------------------
# compute calls (all asynchronous on the current stream unless noted)
# ---------------------------------------------------------------------------
def lm_head_smallm(x, w, scales, fmt: int, y, ws=None, stream=None):
    """y[M, N] (fp32) = x[M, Kd] (bf16) . Wd^T for a bf16 or int4-g64 head."""
    M, Kd = x.shape
    N = w.shape[0]
    if ws is None:
        need = lm_head_workspace_bytes(M, Kd, N, fmt)
        ws = workspace(need, x.device) if need else None
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check("mtpv_lm_head_smallm", load().mtpv_lm_head_smallm(
        _ptr(x), M, Kd, N, _ptr(w), _ptr(scales), fmt, _ptr(y), _ptr(ws), wsb, _stream(stream)))
    return y


def lm_head_pair(xt, w, yt, xd, wq, scales, yd, ws=None, stream=None):
    """Both heads of a verify step: yt = xt . W^T (bf16), yd = xd . deq(wq, scales)^T (int4 g64)."""
    Mt, Kd = xt.shape
    Md = xd.shape[0]
    N = w.shape[0]
    if ws is None:
        ws = workspace(load().mtpv_lm_head_pair_workspace_bytes(Mt, Md, Kd, N), xt.device)
    wsb = ws.numel() * ws.element_size()
    _check("mtpv_lm_head_pair", load().mtpv_lm_head_pair(
        _ptr(xt), Mt, _ptr(w), _ptr(yt), _ptr(xd), Md, _ptr(wq), _ptr(scales), _ptr(yd), Kd, N,
        _ptr(ws), wsb, _stream(stream)))
    return yt, yd


def int4_proj(x, wq, scales, y, ws=None, stream=None):
    """y[M, N] (fp32) = x[M, Kd] (bf16) . deq(wq, scales)^T, split-K for decoder projections."""
    M, Kd = x.shape
    N = wq.shape[0]
    if ws is None:
        ws = workspace(load().mtpv_int4_proj_workspace_bytes(M, Kd, N), x.device)
    _check("mtpv_int4_proj", load().mtpv_int4_proj(
        _ptr(x), M, Kd, N, _ptr(wq), _ptr(scales), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def int4_gate_up(x, wq, scales, h, ws=None, stream=None):
    """h[M, F] = silu(x . G^T) * (x . U^T) with G, U the two halves of the [2F, Kd] int4 head."""
    M, Kd = x.shape
    F = wq.shape[0] // 2
    if ws is None:
        ws = workspace(load().mtpv_int4_gate_up_workspace_bytes(M, Kd, F), x.device)
    _check("mtpv_int4_gate_up", load().mtpv_int4_gate_up(
        _ptr(x), M, Kd, F, _ptr(wq), _ptr(scales), _ptr(h), _ptr(ws), ws.numel(), _stream(stream)))
    return h


def verify(target_logits, draft_logits, draft_tokens, u_accept, u_sample, temperature: float,
           top_p: float, out_tokens, out_accepted, row_status=None, ws=None, stream=None):
    """Leviathan-Chen verification of B sequences (see mtpv_verify)."""
    B, K1, V = target_logits.shape
    K = K1 - 1
    if ws is None:
        ws = workspace(verify_workspace_bytes(B, K, V), target_logits.device)
    _check("mtpv_verify", load().mtpv_verify(
        _ptr(target_logits), _ptr(draft_logits), _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample),
        B, K, V, float(temperature), float(top_p), _ptr(out_tokens), _ptr(out_accepted),
        _ptr(row_status), _ptr(ws), ws.numel(), _stream(stream)))
    return out_tokens, out_accepted


def sample(logits, temperature: float, top_p: float, u, out, row_status=None, ws=None, stream=None):
    """One draw from the warped distribution of every row of ``logits`` [R, V]."""
    R, V = logits.shape
    if ws is None:
        ws = workspace(sample_workspace_bytes(R, V), logits.device)
    _check("mtpv_sample", load().mtpv_sample(
        _ptr(logits), R, V, float(temperature), float(top_p), _ptr(u), _ptr(out), _ptr(row_status),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out


def draft_loop(w_draft, s_draft, h_draft, u_draft, B: int, K: int, temperature: float, top_p: float,
               out_drafts, draft_logits=None, ws=None, stream=None):
    """The draft phase: K positions, each an int4-head projection and one draw from q'."""
    V = w_draft.shape[0]
    h = h_draft.shape[-1]
    if ws is None:
        ws = workspace(load().mtpv_draft_loop_workspace_bytes(B, K, V, h), w_draft.device)
    _check("mtpv_draft_loop", load().mtpv_draft_loop(
        _ptr(w_draft), _ptr(s_draft), _ptr(h_draft), _ptr(u_draft), B, K, V, h, float(temperature),
        float(top_p), _ptr(out_drafts), _ptr(draft_logits), _ptr(ws), ws.numel(), _stream(stream)))
    return out_drafts


def verify_step(w_target, w_draft, s_draft, h_target, h_draft, draft_tokens, u_accept, u_sample,
                B: int, K: int, temperature: float, top_p: float, out_tokens, out_accepted,
                row_status=None, target_logits=None, draft_logits=None, ws=None, stream=None):
    """Both LM heads and the verification in one call (see mtpv_verify_step)."""
    V, h = w_target.shape
    if ws is None:
        ws = workspace(verify_step_workspace_bytes(B, K, V, h), w_target.device)
    _check("mtpv_verify_step", load().mtpv_verify_step(
        _ptr(w_target), _ptr(w_draft), _ptr(s_draft), _ptr(h_target), _ptr(h_draft),
        _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample), B, K, V, h, float(temperature),
        float(top_p), _ptr(out_tokens), _ptr(out_accepted), _ptr(row_status), _ptr(target_logits),
        _ptr(draft_logits), _ptr(ws), ws.numel(), _stream(stream)))
    return out_tokens, out_accepted


def verify_step_host(w_target, w_draft, s_draft, h_target, h_draft, draft_tokens, u_accept,
                     u_sample, B: int, K: int, temperature: float, top_p: float, out_tokens,
                     out_accepted, row_status=None, ws=None, stream=None):
    """verify_step with per-step inputs/outputs in host (ideally pinned) memory.

    Synchronous: returns after the outputs are in the host buffers.
    """
    V, h = w_target.shape
    if ws is None:
        ws = workspace(verify_step_host_workspace_bytes(B, K, V, h), w_target.device)
    _check("mtpv_verify_step_host", load().mtpv_verify_step_host(
        _ptr(w_target), _ptr(w_draft), _ptr(s_draft), _ptr(h_target), _ptr(h_draft),
        _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample), B, K, V, h, float(temperature),
        float(top_p), _ptr(out_tokens), _ptr(out_accepted), _ptr(row_status), _ptr(ws), ws.numel(),
        _stream(stream)))
    return out_tokens, out_accepted
