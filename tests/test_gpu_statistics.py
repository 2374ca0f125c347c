"""Statistics of the tokens the GPU emits, checked without the oracle's code.

Speculative sampling is exact: the tokens it emits are distributed as plain
sampling from the warped target distribution (hazakura.dev MTPLX notes,
results table: identical distributions, max_diff = 0.0; devtrends.cc MTPLX
overview, "no second model" section: temperature 0.6 / top_p 0.95 sampling is
unchanged).  With one fixed set of logits (the small verify step: hidden 512,
vocabulary 4096, K = 3, produced by the library's own heads) and fresh
uniforms in every trial, the k-th emitted token, over the trials that accepted
at least k drafts, must follow p'_k, the warped target row k.  Each trial
draws its drafts with mtpv_sample from q' and then runs mtpv_verify.

p' is computed here with numpy from its definition (softmax at temperature T,
ranks by (logit desc, index asc), keep a rank while the mass before it is
below top_p, renormalise); Pearson's chi-square is taken over the support,
tail bins merged until every expected count is at least 5, and a token
outside the support must never appear.  10^6 trials.

Negative control: when mtpv_verify is told a draft distribution other than
the one the drafts were drawn from, the emitted tokens no longer follow p'
(devtrends.cc overview, limitations: draft and target weights that do not
match break the exactness), and the same test must reject them.
"""
import numpy as np
import pytest
import torch
from scipy.stats import chi2

import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import f32

pytestmark = pytest.mark.gpu

K, V, H = 3, 4096, 512
T, TOP_P = 0.6, 0.95
TRIALS = 1_000_000
CONTROL_TRIALS = 204_800
BATCH = 8192        # sequences per call: B (2K + 1) = 57344 rows


def warped(l: np.ndarray) -> np.ndarray:
    """p' of one row of logits (fp64), straight from the definition."""
    l = l.astype(np.float64)
    Tq, Pq = f32(T), f32(TOP_P)     # the values the C ABI sees
    e = np.exp((l - l.max()) / Tq)
    p = e / e.sum()
    order = np.lexsort((np.arange(len(l)), -l))
    before = np.concatenate([[0.0], np.cumsum(p[order])[:-1]])
    kept = before < Pq
    kept[0] = True
    w = np.zeros_like(p)
    w[order[kept]] = p[order[kept]]
    return w / w.sum()


def chi_square(counts: np.ndarray, probs: np.ndarray):
    """(p-value, statistic, dof) of counts against probs; bins with expected
    count < 5 merged, smallest first.  Counts outside the support fail."""
    n = counts.sum()
    support = probs > 0
    assert counts[~support].sum() == 0, "a token outside the warped support was emitted"
    E = n * probs[support]
    O = counts[support].astype(np.float64)
    order = np.argsort(-E, kind="stable")
    E, O = E[order], O[order]
    ge, go = [], []
    ae = ao = 0.0
    for e, o in zip(E[::-1], O[::-1]):   # from the smallest expectation up
        ae += e
        ao += o
        if ae >= 5.0:
            ge.append(ae)
            go.append(ao)
            ae = ao = 0.0
    if ae > 0.0:
        ge[-1] += ae
        go[-1] += ao
    ge, go = np.array(ge), np.array(go)
    x2 = float(np.sum((go - ge) ** 2 / ge))
    dof = len(ge) - 1
    return float(chi2.sf(x2, dof)), x2, dof


@pytest.fixture(scope="module")
def logits():
    """Target rows [K+1, V] and draft rows [K, V] of the small verify step,
    through the library's bf16 and int4 heads."""
    W = synth.make_head(V, H, 0.05, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    Ht, Hd = synth.make_hidden(1, K, H, 0.3, seed=7, device="cuda")
    tl = torch.empty((K + 1, V), dtype=torch.float32, device="cuda")
    dl = torch.empty((K, V), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(Ht, W, None, mtpv.W_BF16, tl)
    mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, dl)
    torch.cuda.synchronize()
    return tl, dl


def emitted_counts(tl, dl_drafts, dl_verify, trials, seed):
    """counts[k, v]: how often token v was emitted k-th, over `trials` trials."""
    counts = torch.zeros((K + 1, V), dtype=torch.int64, device="cuda")
    done, t = 0, 0
    while done < trials:
        B = min(BATCH, trials - done)
        u = synth.step_uniforms(seed, t, B, K)
        tlb = tl.unsqueeze(0).expand(B, K + 1, V).contiguous()
        dsrc = dl_drafts.unsqueeze(0).expand(B, K, V).contiguous()
        d = torch.empty((B * K,), dtype=torch.int32, device="cuda")
        mtpv.sample(dsrc.view(B * K, V), T, TOP_P, torch.as_tensor(u["u_draft"].reshape(-1)).cuda(), d)
        dver = dsrc if dl_verify is dl_drafts else dl_verify.unsqueeze(0).expand(B, K, V).contiguous()
        ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
        oa = torch.empty((B,), dtype=torch.int32, device="cuda")
        rs = torch.empty((B,), dtype=torch.int32, device="cuda")
        mtpv.verify(tlb, dver, d.view(B, K), torch.as_tensor(u["u_accept"]).cuda(),
                    torch.as_tensor(u["u_sample"]).cuda(), T, TOP_P, ot, oa, rs)
        assert int((rs != 0).sum()) == 0 and int((oa < 0).sum()) == 0
        for k in range(K + 1):
            sel = oa >= k
            counts[k] += torch.bincount(ot[sel, k].long(), minlength=V)
        done += B
        t += 1
        del tlb, dsrc, dver
    return counts.cpu().numpy()


def test_emitted_tokens_follow_the_warped_target(logits):
    tl, dl = logits
    counts = emitted_counts(tl, dl, dl, TRIALS, seed=2024)
    assert counts[0].sum() == TRIALS
    tl64 = tl.double().cpu().numpy()
    for k in range(K + 1):
        pv, x2, dof = chi_square(counts[k], warped(tl64[k]))
        print(f"\nposition {k}: {counts[k].sum()} tokens, chi2 {x2:.1f} on {dof} dof, p = {pv:.3g}")
        assert pv > 1e-4, (k, x2, dof)
    # every position is reached often enough to mean something
    assert counts[K].sum() > TRIALS // 10


def test_mismatched_draft_distribution_is_rejected(logits):
    tl, dl = logits
    wrong = (dl * 0.85).contiguous()   # a flatter q' than the drafts came from
    counts = emitted_counts(tl, dl, wrong, CONTROL_TRIALS, seed=4048)
    pv, x2, dof = chi_square(counts[0], warped(tl.double().cpu().numpy()[0]))
    print(f"\ncontrol: chi2 {x2:.1f} on {dof} dof, p = {pv:.3g}")
    assert x2 > dof + 20.0 * np.sqrt(2.0 * dof)
