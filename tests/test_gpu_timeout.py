"""The sampler's bounded device-side waits report a timeout instead of hanging.

mtpv_set_wait_polls(0) makes every first wait on a bulk copy give up at once
(the kernel then waits again, with the default bound, for the copy it issued),
so the timeout path runs deterministically without any fault: every sequence
is reported MTPV_ROW_TIMEOUT with out_accepted = -1 and tokens -1, the
sampled rows likewise, and the next call with the default bound is back to
oracle parity on the same inputs.  The vocabulary is a multiple of 4 so that
every slice takes the bulk-copy path.
"""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import cuda, f32

pytestmark = pytest.mark.gpu

T, TOP_P = 0.6, 0.95


def _case(B, K, V, seed):
    tl, dl = synth.make_verify_logits(B, K, V, 1.43, 0.43, seed)
    u = synth.step_uniforms(seed, 0, B, K)
    d, _, _ = oracle.sample_rows(dl.reshape(B * K, V).double().numpy(), f32(T), f32(TOP_P),
                                 u["u_draft"].reshape(-1), threads=8)
    return tl, dl, d.reshape(B, K), u


def _verify(tl, dl, d, u):
    B, K1, V = tl.shape
    out_t = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    out_a = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    rs = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    mtpv.verify(cuda(tl), cuda(dl), cuda(torch.as_tensor(d, dtype=torch.int32)),
                cuda(torch.as_tensor(u["u_accept"])), cuda(torch.as_tensor(u["u_sample"])), T, TOP_P,
                out_t, out_a, rs)
    torch.cuda.synchronize()
    return out_t.cpu().numpy(), out_a.cpu().numpy(), rs.cpu().numpy()


@pytest.fixture
def give_up_at_once():
    mtpv.set_wait_polls(0)
    try:
        yield
    finally:
        mtpv.set_wait_polls(-1)


def test_verify_reports_timeout_then_recovers(give_up_at_once):
    B, K, V = 3, 3, 151936
    tl, dl, d, u = _case(B, K, V, seed=4242)
    tok, acc, rs = _verify(tl, dl, d, u)
    assert (rs == mtpv.ROW_TIMEOUT).all(), rs
    assert (acc == -1).all() and (tok == -1).all()
    mtpv.set_wait_polls(-1)
    tok, acc, rs = _verify(tl, dl, d, u)
    ref = oracle.verify(tl.double().numpy(), dl.double().numpy(), d, u["u_accept"], u["u_sample"],
                        f32(T), f32(TOP_P), threads=8)
    assert (rs == 0).all()
    ok = ref["flags"] == 0
    assert np.array_equal(acc[ok], ref["accepted"][ok])
    assert np.array_equal(tok[ok], ref["tokens"][ok])


def test_sample_reports_timeout(give_up_at_once):
    R, V = 4, 151936
    logits = synth.make_verify_logits(1, R - 1, V, 1.43, 0.43, 77)[0].reshape(R, V)
    uu = torch.full((R,), 0.5, dtype=torch.float32, device="cuda")
    tok = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    rs = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    mtpv.sample(cuda(logits), T, TOP_P, uu, tok, rs)
    torch.cuda.synchronize()
    assert (rs.cpu().numpy() == mtpv.ROW_TIMEOUT).all()
    assert (tok.cpu().numpy() == -1).all()
