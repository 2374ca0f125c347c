"""mtpv_verify_noalloc, the verify call for callers that cannot allocate.

Callers inside an allocation-free decode loop, plug-ins whose host framework
owns all device memory, or hooks running during stream capture cannot give
the library a workspace; mtpv_verify_noalloc uses scratch compiled into the
library instead.  This test calls it through the C ABI and checks that two
calls in a row give exactly what mtpv_verify (caller workspace) gives on the
same inputs (temperature and top-p cuts, greedy, top_p = 1, vocabularies
that are and are not multiples of 4), that it agrees with the oracle outside
flagged boundary cases, and that a request larger than the fixed scratch is
refused on the host.  It lives in its own file, collected last, and needs no state from
other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import build as mtpv_build
from verify_step_lm_b200 import synth

pytestmark = pytest.mark.gpu

UNSUPPORTED = 2


def noalloc_fn():
    mtpv_build.build()
    lib = mtpv.load()
    f = lib.mtpv_verify_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [P, P, P, P, P, I, I, I, F, F, P, P, P, P]
    f.restype = I
    return f


def inputs(B, K, V, seed):
    tl, dl = synth.make_verify_logits(B, K, V, 1.43, 0.43, seed)
    rng = np.random.default_rng(seed)
    d = dl.argmax(dim=2).int().numpy()
    mask = rng.random(d.shape) < 0.25
    d[mask] = rng.integers(0, V, size=int(mask.sum()))
    u = synth.step_uniforms(seed, 0, B, K)
    g = lambda t: torch.as_tensor(t).contiguous().cuda()
    return g(tl), g(dl), g(d.astype(np.int32)), g(u["u_accept"]), g(u["u_sample"])


def outputs(B, K):
    return (torch.full((B, K + 1), -5, dtype=torch.int32, device="cuda"),
            torch.full((B,), -5, dtype=torch.int32, device="cuda"),
            torch.full((B,), -5, dtype=torch.int32, device="cuda"))


def p(t):
    return ctypes.c_void_p(t.data_ptr())


# (B, K, V, T, top_p, seed): the benchmark's vocabulary, a smaller one with a
# top-p cut, greedy and top_p = 1 on a vocabulary that is not a multiple of 4
# (slices that are not 16-byte aligned take the plain-load paths)
CASES = [(4, 3, 151936, 0.6, 0.95, 11), (9, 2, 4096, 1.0, 0.8, 12), (5, 3, 4097, 0.0, 0.95, 13),
         (6, 1, 4097, 0.7, 1.0, 14)]


@pytest.mark.parametrize("first,second", [(0, 1), (2, 3)])
def test_noalloc_matches_workspace_verify_on_two_calls_in_a_row(first, second):
    f = noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    got, want = [], []
    for B, K, V, T, top_p, seed in (CASES[first], CASES[second]):   # two calls back to back
        tl, dl, d, ua, us = inputs(B, K, V, seed)
        ot, oa, rs = outputs(B, K)
        st = f(p(tl), p(dl), p(d), p(ua), p(us), B, K, V, T, top_p, p(ot), p(oa), p(rs), stream)
        assert st == 0, mtpv.status_string(st)
        got.append((ot, oa, rs))
        wt, wa, wr = outputs(B, K)
        mtpv.verify(tl, dl, d, ua, us, T, top_p, wt, wa, wr)
        want.append((wt, wa, wr))
    torch.cuda.synchronize()
    for (ot, oa, rs), (wt, wa, wr) in zip(got, want):
        # integer outputs of the same computation on the same inputs: exact
        assert torch.equal(ot, wt) and torch.equal(oa, wa) and torch.equal(rs, wr)
        assert (oa >= 0).all()


def test_noalloc_against_the_oracle():
    import oracle
    f = noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, K, V, T, top_p, seed = 16, 3, 4097, 0.6, 0.95, 15
    tl, dl, d, ua, us = inputs(B, K, V, seed)
    ot, oa, rs = outputs(B, K)
    st = f(p(tl), p(dl), p(d), p(ua), p(us), B, K, V, T, top_p, p(ot), p(oa), p(rs), stream)
    assert st == 0, mtpv.status_string(st)
    torch.cuda.synchronize()
    f32 = lambda x: float(np.float32(x))
    ref = oracle.verify(tl.cpu().double().numpy(), dl.cpu().double().numpy(), d.cpu().numpy(),
                        ua.cpu().numpy(), us.cpu().numpy(), f32(T), f32(top_p))
    same = (ot.cpu().numpy() == ref["tokens"]).all(axis=1) & (oa.cpu().numpy() == ref["accepted"])
    assert (same | (ref["flags"] != 0)).all()
    assert np.array_equal(rs.cpu().numpy(), ref["status"])


def test_noalloc_refuses_requests_beyond_its_scratch():
    f = noalloc_fn()
    a = ctypes.c_void_p(1 << 20)   # never dereferenced: refused before any launch
    # K = 3: 230 sequences fit in 64 KiB, 231 do not
    assert f(a, a, a, a, a, 231, 3, 1000, 0.6, 0.95, a, a, None, None) == UNSUPPORTED
    assert f(None, a, a, a, a, 1, 3, 1000, 0.6, 0.95, a, a, None, None) == 1
