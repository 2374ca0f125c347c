"""Pins for the oracle's Leviathan-Chen verify step.

The central pin is the pages' claim that speculative sampling leaves the
output distribution unchanged (hazakura.dev MTPLX notes, results table:
"max_diff = 0.0"; devtrends.cc overview: temperature=0.6 / top_p=0.95 give the
same responses as without MTP).  On vocabularies of at most 8 tokens the test
enumerates every draft outcome and every accept/reject branch, runs verify
steps until K+1 tokens are out, and compares the probability of every emitted
sequence with the product of the target's warped conditionals.  A mismatched
draft distribution must break the identity (the pages warn that a draft head
that does not match the weights breaks the mathematics: devtrends.cc
overview, project limits).
"""
import itertools
import json
import os
from collections import defaultdict

import numpy as np
import pytest

import oracle
from verify_step_lm_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.json")))
T_PAGES = GOLDEN["temperature"]["value"]
TOPP_PAGES = GOLDEN["top_p"]["value"]
MAX_DIFF_PAGES = GOLDEN["distribution_max_diff"]["value"]
# The pages report 0.0 at display precision; fp64 sums of <= 8^4 terms carry
# rounding of a few 1e-16, so the bar is 1e-12.
TOL = max(MAX_DIFF_PAGES, 1e-12)


# --------------------------------------------------------------------------
# prefix-dependent pseudo-random logits (a stand-in "model")
# --------------------------------------------------------------------------
def _prefix_key(prefix, salt):
    h = np.uint64(salt)
    for t in prefix:
        h = synth.splitmix64(h ^ np.uint64((t + 1) * 0x100000001B3))
    return int(h)


def _gauss(key, V):
    u1 = synth.uniforms(key, np.arange(V) * 2).astype(np.float64) + 2.0 ** -25
    u2 = synth.uniforms(key, np.arange(V) * 2 + 1).astype(np.float64)
    return np.sqrt(-2 * np.log(u1)) * np.cos(2 * np.pi * u2)


class Model:
    def __init__(self, V, std, tau, seed, grid=None, draft_mismatch=False):
        self.V, self.std, self.tau, self.seed, self.grid = V, std, tau, seed, grid
        self.draft_mismatch = draft_mismatch

    def target(self, prefix):
        l = self.std * _gauss(_prefix_key(prefix, self.seed), self.V)
        return np.round(l / self.grid) * self.grid if self.grid else l

    def draft(self, prefix):
        l = self.target(prefix) + self.tau * _gauss(_prefix_key(prefix, self.seed + 7), self.V)
        return np.round(l / self.grid) * self.grid if self.grid else l

    def draft_sampling(self, prefix):
        """Logits the drafts are actually drawn from."""
        if self.draft_mismatch:
            return self.draft(prefix) + 1.5 * _gauss(_prefix_key(prefix, self.seed + 99), self.V)
        return self.draft(prefix)


def one_step(model, prefix, K, T, top_p):
    """Distribution of the tokens emitted by one verify step at ``prefix``."""
    V = model.V
    out = defaultdict(float)
    qcache = {}

    def q_sample(pre):
        if pre not in qcache:
            qcache[pre] = oracle.warp(model.draft_sampling(pre), T, top_p)[0]
        return qcache[pre]

    for drafts in itertools.product(range(V), repeat=K):
        pd = 1.0
        for i in range(K):
            pd *= q_sample(prefix + drafts[:i])[drafts[i]]
            if pd == 0.0:
                break
        if pd == 0.0:
            continue
        tl = np.stack([model.target(prefix + drafts[:i]) for i in range(K + 1)])
        dl = np.stack([model.draft(prefix + drafts[:i]) for i in range(K)])
        acc, res, bonus, st = oracle.verify_dist(tl, dl, np.array(drafts), T, top_p)
        assert st == 0
        pa = pd
        for n in range(K):
            prej = pa * (1.0 - acc[n])
            if prej > 0:
                for x in range(V):
                    if res[n, x] > 0:
                        out[drafts[:n] + (x,)] += prej * res[n, x]
            pa *= acc[n]
        for x in range(V):
            if bonus[x] > 0:
                out[tuple(drafts) + (x,)] += pa * bonus[x]
    return out


def emitted_distribution(model, K, T, top_p, need):
    result = defaultdict(float)
    frontier = {(): 1.0}
    while frontier:
        nxt = defaultdict(float)
        for emitted, pm in frontier.items():
            for e, pe in one_step(model, emitted, K, T, top_p).items():
                full = emitted + e
                if len(full) >= need:
                    result[full[:need]] += pm * pe
                else:
                    nxt[full] += pm * pe
        frontier = nxt
    return result


def autoregressive_distribution(model, T, top_p, need):
    out = {}
    for seq in itertools.product(range(model.V), repeat=need):
        p = 1.0
        for j in range(need):
            p *= oracle.warp(model.target(seq[:j]), T, top_p)[0][seq[j]]
            if p == 0.0:
                break
        if p > 0:
            out[seq] = p
    return out


def max_diff(a, b):
    keys = set(a) | set(b)
    return max(abs(a.get(k, 0.0) - b.get(k, 0.0)) for k in keys)


CASES = [
    # (V, K, T, top_p, std, tau, grid)
    (4, 3, T_PAGES, TOPP_PAGES, 1.5, 0.5, None),
    (4, 3, T_PAGES, 1.0, 1.0, 1.0, None),
    (6, 2, T_PAGES, TOPP_PAGES, 1.2, 0.8, None),
    (8, 2, 1.0, 0.8, 1.0, 0.6, None),
    (5, 2, 0.9, 0.7, 1.0, 0.5, 0.5),      # exact ties in logits
    (4, 1, T_PAGES, TOPP_PAGES, 2.0, 2.0, None),
    (5, 3, 0.0, TOPP_PAGES, 1.0, 0.7, None),  # greedy
]


@pytest.mark.parametrize("V,K,T,top_p,std,tau,grid", CASES)
def test_emitted_distribution_equals_autoregressive(V, K, T, top_p, std, tau, grid):
    model = Model(V, std, tau, seed=1234 + V * 10 + K, grid=grid)
    spec = emitted_distribution(model, K, T, top_p, need=K + 1)
    ar = autoregressive_distribution(model, T, top_p, need=K + 1)
    assert abs(sum(spec.values()) - 1.0) < 1e-12
    assert max_diff(spec, ar) <= TOL


def test_mismatched_draft_distribution_breaks_identity():
    # Drafts drawn from a distribution other than the q' used in the ratio:
    # the identity must fail visibly (negative control for the test above).
    model = Model(4, 1.5, 0.5, seed=77, draft_mismatch=True)
    spec = emitted_distribution(model, 2, T_PAGES, TOPP_PAGES, need=3)
    ar = autoregressive_distribution(model, T_PAGES, TOPP_PAGES, need=3)
    assert max_diff(spec, ar) > 1e-3


def test_single_position_closed_form():
    # V=3, K=1, T=1, top_p=1: p = softmax(lt), q = softmax(ld).
    lt = np.log(np.array([[0.5, 0.3, 0.2], [0.1, 0.6, 0.3]]))
    ld = np.log(np.array([[0.2, 0.6, 0.2]]))
    acc, res, bonus, st = oracle.verify_dist(lt, ld, np.array([1]), 1.0, 1.0)
    assert abs(acc[0] - 0.5) < 1e-15               # min(1, 0.3/0.6)
    np.testing.assert_allclose(res[0], [1.0, 0.0, 0.0], atol=1e-15)  # max(0,p-q) = (0.3,0,0)
    np.testing.assert_allclose(bonus, [0.1, 0.6, 0.3], atol=1e-15)
    acc, res, bonus, st = oracle.verify_dist(lt, ld, np.array([0]), 1.0, 1.0)
    assert acc[0] == 1.0                           # p/q = 2.5 -> accept surely


def _random_batch(B, K, V, seed, T=T_PAGES, top_p=TOPP_PAGES, tau=0.5, grid=None):
    tl, dl = synth.make_verify_logits(B, K, V, 1.43, tau, seed, grid=grid)
    tl, dl = tl.double().numpy(), dl.double().numpy()
    u = synth.step_uniforms(seed, 0, B, K)
    d, _, _ = oracle.sample_rows(dl.reshape(B * K, V), T, top_p, u["u_draft"].reshape(-1))
    return tl, dl, d.reshape(B, K), u


def test_greedy_reduces_to_argmax_agreement():
    B, K, V = 64, 3, 257
    tl, dl, _, u = _random_batch(B, K, V, seed=5, T=0.0)
    # drafts: the draft argmax, sometimes replaced by a random token
    rng = np.random.default_rng(0)
    d = dl.argmax(axis=2).astype(np.int32)
    mask = rng.random((B, K)) < 0.3
    d[mask] = rng.integers(0, V, size=mask.sum())
    r = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], 0.0, TOPP_PAGES)
    for b in range(B):
        at = tl[b].argmax(axis=1)
        n = next((i for i in range(K) if d[b, i] != at[i]), K)
        assert r["accepted"][b] == n
        assert list(r["tokens"][b, :n]) == list(d[b, :n])
        assert r["tokens"][b, n] == at[n]
        assert (r["tokens"][b, n + 1:] == -1).all()
    # uniforms do not matter at T == 0
    r2 = oracle.verify(tl, dl, d, np.zeros_like(u["u_accept"]), 1 - 2.0 ** -24 +
                       np.zeros_like(u["u_sample"]), 0.0, TOPP_PAGES)
    assert np.array_equal(r["tokens"], r2["tokens"])


def test_small_temperature_matches_greedy():
    B, K, V = 32, 3, 500
    tl, dl, _, u = _random_batch(B, K, V, seed=6)
    d = dl.argmax(axis=2).astype(np.int32)
    r0 = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], 0.0, TOPP_PAGES)
    r1 = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], 1e-4, TOPP_PAGES)
    assert np.array_equal(r0["tokens"], r1["tokens"])


def test_bonus_and_output_invariants():
    B, K, V = 200, 3, 300
    tl, dl, d, u = _random_batch(B, K, V, seed=7)
    r = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], T_PAGES, TOPP_PAGES, threads=4)
    assert (r["status"] == 0).all()
    seen_bonus = seen_reject = 0
    for b in range(B):
        n = r["accepted"][b]
        toks = r["tokens"][b]
        assert 0 <= n <= K
        assert (toks[: n + 1] >= 0).all() and (toks[n + 1:] == -1).all()
        assert list(toks[:n]) == list(d[b, :n])
        x = toks[n]
        p, _ = oracle.warp(tl[b, n], T_PAGES, TOPP_PAGES)
        assert p[x] > 0                        # emitted token lies in the top-p support
        if n == K:
            seen_bonus += 1                    # bonus present exactly when all K accepted
        else:
            seen_reject += 1
            q, _ = oracle.warp(dl[b, n], T_PAGES, TOPP_PAGES)
            assert p[x] > q[x]                 # residual token: p' exceeds q'
    assert seen_bonus > 0 and seen_reject > 0


def test_sampling_mode_agrees_with_distribution_mode():
    """Histogram of the first emitted token over many uniform draws matches the
    distribution mode's marginal (chi-square), tying the two modes together."""
    K, V = 2, 6
    rng = np.random.default_rng(3)
    tl = rng.standard_normal((1, K + 1, V))
    dl = tl[:, :K] + 0.7 * rng.standard_normal((1, K, V))
    T, top_p = T_PAGES, TOPP_PAGES
    q0, _ = oracle.warp(dl[0, 0], T, top_p)
    p0, _ = oracle.warp(tl[0, 0], T, top_p)
    N = 20000
    d0, _, _ = oracle.sample_rows(np.repeat(dl[0, :1], N, 0), T, top_p,
                                  synth.uniforms(11, np.arange(N)))
    drafts = np.stack([d0, np.zeros(N, dtype=np.int32)], axis=1)
    ua = synth.uniforms(12, np.arange(N * K)).reshape(N, K)
    us = synth.uniforms(13, np.arange(N * (K + 1))).reshape(N, K + 1)
    r = oracle.verify(np.repeat(tl, N, 0), np.repeat(dl, N, 0), drafts, ua, us, T, top_p, threads=4)
    first = r["tokens"][:, 0]
    counts = np.bincount(first, minlength=V)
    expected = p0 * N
    m = expected > 0
    chi2 = (((counts - expected) ** 2)[m] / expected[m]).sum()
    assert counts[~m].sum() == 0
    assert chi2 < 25.0   # 5 dof: P(chi2 > 25) ~ 1.4e-4


def test_data_errors_reported_per_sequence():
    B, K, V = 3, 2, 50
    tl, dl, d, u = _random_batch(B, K, V, seed=8)
    d = d.copy()
    d[0, 1] = V            # out of range
    tl = tl.copy()
    tl[2, 0, 5] = np.nan   # non-finite
    r = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], T_PAGES, TOPP_PAGES)
    assert list(r["status"]) == [1, 0, 2]
    assert r["accepted"][0] == -1 and (r["tokens"][0] == -1).all()
    assert r["accepted"][2] == -1 and (r["tokens"][2] == -1).all()
    assert r["accepted"][1] >= 0


def test_identical_rows_accept_everything():
    B, K, V = 8, 3, 100
    tl, _, _, u = _random_batch(B, K, V, seed=9)
    dl = tl[:, :K].copy()
    d, _, _ = oracle.sample_rows(dl.reshape(-1, V), T_PAGES, TOPP_PAGES, u["u_draft"].reshape(-1))
    r = oracle.verify(tl, dl, d.reshape(B, K), u["u_accept"], u["u_sample"], T_PAGES, TOPP_PAGES)
    assert (r["accepted"] == K).all()


def test_flags_are_rare_on_the_tiny_workload():
    B, K, V = 1000, 3, 4096
    tl, dl, d, u = _random_batch(B, K, V, seed=10)
    r = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], T_PAGES, TOPP_PAGES, threads=8)
    assert (r["flags"] != 0).mean() < 0.01
