"""Parity of the whole verify step at the Qwen-class shape (hidden 5120,
vocabulary 151936, K = 3, T = 0.6, top_p = 0.95).

1. Ten thousand seeded steps (seeds 0..9999, the workload's own step count)
   in sampler-parity mode: each step's hidden states and uniforms come from
   its seed; the step runs through mtpv_verify_step (16 sequences per call,
   B (K + 1) = 64 rows); its own fp32 logits are copied to the host and the
   fp64 oracle runs the warp, the acceptance tests and the draw on them.
   Accept counts and token ids must be identical on every trial the oracle
   does not flag as a boundary case, and the flagged trials must stay under
   0.01 % of all trials (the bound the verify step's exactness claim is held
   to).  The drafts are drawn by the library's own mtpv_sample from q'.
2. 64 steps of one sequence each, through the launch configuration the
   benchmark times (both heads in one persistent launch, then the two
   sampler kernels): the logits on sampled vocabulary rows (every 97th row
   plus the ragged tail) against the oracle's fp64 projection within 1e-3
   relative, and tokens / accept counts against the oracle run on the step's
   own logits.

The pages: exact Leviathan-Chen sampling with residual correction that keeps
temperature 0.6 / top_p 0.95 sampling unchanged (devtrends.cc MTPLX overview,
"no second model" section), with identical distributions, max_diff = 0.0
(hazakura.dev MTPLX notes, results table).
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close, f32

pytestmark = pytest.mark.gpu

K, V, H = 3, 151936, 5120
T, TOP_P = 0.6, 0.95
SIGMA, WSTD = 0.3, 0.02
STEPS = int(os.environ.get("MTPV_PARITY_STEPS", "10000"))
BATCH = 16          # sequences per mtpv_verify_step call: B (K + 1) = 64 rows
FLAG_LIMIT = 1e-4   # flagged trials / trials


def host_threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return os.cpu_count() or 1


@pytest.fixture(scope="module")
def heads():
    W = synth.make_head(V, H, WSTD, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    return W, Wq, S


def step_inputs(seeds, k=K, sigma=SIGMA):
    """Hidden states and uniforms of the steps `seeds`, one sequence each,
    laid out as one batch (sequence b = seeds[b])."""
    hts, hds, us = [], [], []
    for s in seeds:
        Ht, Hd = synth.make_hidden(1, k, H, sigma, seed=int(s), device="cuda")
        hts.append(Ht)
        hds.append(Hd)
        us.append(synth.step_uniforms(int(s), 0, 1, k))
    u = {key: np.concatenate([x[key] for x in us]) for key in us[0]}
    return torch.cat(hts), torch.cat(hds), u


def library_drafts(Hd, Wq, S, u_draft, t=T):
    """The draft phase's own sampling: q' from the int4 head, one draw per row."""
    dl0 = torch.empty((Hd.shape[0], V), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, dl0)
    d = torch.empty((Hd.shape[0],), dtype=torch.int32, device="cuda")
    mtpv.sample(dl0, t, TOP_P, torch.as_tensor(u_draft.reshape(-1)).cuda(), d)
    return d


def run_step(W, Wq, S, Ht, Hd, d, u, B, k=K, t=T):
    tl = torch.empty((B, k + 1, V), dtype=torch.float32, device="cuda")
    dl = torch.empty((B, k, V), dtype=torch.float32, device="cuda")
    ot = torch.full((B, k + 1), -9, dtype=torch.int32, device="cuda")
    oa = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    rs = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    mtpv.verify_step(W, Wq, S, Ht, Hd, d.view(B, k), torch.as_tensor(u["u_accept"]).cuda(),
                     torch.as_tensor(u["u_sample"]).cuda(), B, k, t, TOP_P, ot, oa, rs, tl, dl)
    return tl, dl, ot, oa, rs


def oracle_check(tl, dl, d, u, ot, oa, rs, t=T):
    """Sampler-parity check of one batch on the host; returns (trials,
    flagged, accepted counts) or raises on an unflagged mismatch."""
    k = d.shape[1]
    ref = oracle.verify(tl, dl, d, u["u_accept"], u["u_sample"], f32(t), f32(TOP_P), threads=1)
    mism = (ot != ref["tokens"]).any(axis=1) | (oa != ref["accepted"])
    bad = mism & (ref["flags"] == 0)
    if bad.any():
        i = int(np.nonzero(bad)[0][0])
        raise AssertionError(f"unflagged mismatch: gpu {ot[i]} / {oa[i]}, oracle {ref['tokens'][i]} / "
                             f"{ref['accepted'][i]}")
    if not np.array_equal(rs, ref["status"]):
        raise AssertionError(f"row status differs: gpu {rs}, oracle {ref['status']}")
    return len(oa), int((ref["flags"] != 0).sum()), np.bincount(oa, minlength=k + 1)


def test_ten_thousand_steps_sampler_parity(heads):
    W, Wq, S = heads
    workers = host_threads()
    trials = flagged = 0
    acc_hist = np.zeros(K + 1, dtype=np.int64)
    pending = []

    def drain(keep):
        nonlocal trials, flagged, acc_hist
        while len(pending) > keep:
            n, f, h = pending.pop(0).result()
            trials += n
            flagged += f
            acc_hist += h

    with ThreadPoolExecutor(workers) as pool:
        for s0 in range(0, STEPS, BATCH):
            seeds = np.arange(s0, min(STEPS, s0 + BATCH))
            B = len(seeds)
            Ht, Hd, u = step_inputs(seeds)
            d = library_drafts(Hd, Wq, S, u["u_draft"])
            tl, dl, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, B)
            host = [x.cpu().numpy() for x in (tl, dl, d.view(B, K), ot, oa, rs)]
            pending.append(pool.submit(oracle_check, host[0], host[1], host[2], u, *host[3:]))
            drain(2 * workers)
        drain(0)
    rate = flagged / trials
    bound = (-math.log(0.05) if flagged == 0 else flagged + 2.0 * math.sqrt(flagged) + 2.0) / trials
    print(f"\n{trials} steps: {flagged} flagged (rate {rate:.2e}, ~95% upper bound {bound:.2e}); "
          f"accepted-count histogram {acc_hist.tolist()}")
    assert trials == STEPS
    assert rate < FLAG_LIMIT, (flagged, trials)
    # the random-init heads with draft noise 0.3 accept often but not always
    assert acc_hist[K] > 0 and acc_hist[0] > 0


def test_bench_launch_configuration_64_steps(heads):
    W, Wq, S = heads
    rows = np.unique(np.concatenate([np.arange(0, V, 97), np.arange(V - 64, V)]))
    ridx = torch.as_tensor(rows).cuda()
    Wb_rows = synth.bf16_bits(W[ridx].cpu())
    Wq_rows = Wq[ridx].cpu().numpy()
    S_rows = synth.bf16_bits(S[ridx].cpu())
    flagged = 0
    for seed in range(64):
        Ht, Hd, u = step_inputs([20000 + seed])
        d = library_drafts(Hd, Wq, S, u["u_draft"])
        tl, dl, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, 1)
        torch.cuda.synchronize()
        ref_t = oracle.lm_head_bf16(synth.bf16_bits(Ht.cpu()), Wb_rows, threads=8)
        ref_d = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq_rows, S_rows, threads=8)
        assert_logits_close(tl.view(K + 1, V)[:, ridx].cpu().numpy(), ref_t)
        assert_logits_close(dl.view(K, V)[:, ridx].cpu().numpy(), ref_d)
        n, f, _ = oracle_check(tl.cpu().numpy(), dl.cpu().numpy(), d.view(1, K).cpu().numpy(), u,
                               ot.cpu().numpy(), oa.cpu().numpy(), rs.cpu().numpy())
        flagged += f
    assert flagged <= 1


@pytest.mark.parametrize("sigma", [0.1, 0.3, 1.0])
@pytest.mark.parametrize("t", [0.6, 0.0])
@pytest.mark.parametrize("k", [1, 2, 3])
def test_depth_sweep_cell(heads, k, t, sigma):
    """One cell of the draft-depth sweep (the pages' depth 1/2/3 tuning,
    devtrends.cc MTPLX overview, feature list: tune --retune): 32 steps at
    draft depth k, temperature t (0 = greedy) and draft noise sigma, in
    sampler-parity mode; prints the cell's flagged trials and acceptance."""
    W, Wq, S = heads
    trials = flagged = 0
    acc = np.zeros(k + 1, dtype=np.int64)
    for s0 in (0, 16):
        seeds = np.arange(30000 + s0, 30000 + s0 + 16)
        Ht, Hd, u = step_inputs(seeds, k, sigma)
        d = library_drafts(Hd, Wq, S, u["u_draft"], t)
        tl, dl, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, 16, k, t)
        n, f, h = oracle_check(tl.cpu().numpy(), dl.cpu().numpy(), d.view(16, k).cpu().numpy(), u,
                               ot.cpu().numpy(), oa.cpu().numpy(), rs.cpu().numpy(), t)
        trials += n
        flagged += f
        acc += h
    rate = float((acc * np.arange(k + 1)).sum()) / (trials * k)
    print(f"\nK={k} T={t} sigma={sigma}: {trials} steps, {flagged} flagged, acceptance {rate:.3f}")
    assert flagged <= 1


def test_large_vocab_batched_step():
    """Eight sequences at vocabulary 248320 (hidden 5120, K = 3): 32 target
    rows through the bf16 head and 24 draft rows through the int4 head, both
    on the tensor-memory kernels (one pass over the weights), then the
    sampler.  Logits on a strided sample of vocabulary rows against the
    oracle's fp64 projection; tokens and accept counts against the oracle
    run on the step's own logits."""
    B, k, V8 = 8, 3, 248320
    W = synth.make_head(V8, H, WSTD, seed=4242, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    Ht, Hd = synth.make_hidden(B, k, H, SIGMA, seed=77, device="cuda")
    u = synth.step_uniforms(77, 0, B, k)
    dl0 = torch.empty((B * k, V8), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, dl0)
    d = torch.empty((B * k,), dtype=torch.int32, device="cuda")
    mtpv.sample(dl0, T, TOP_P, torch.as_tensor(u["u_draft"].reshape(-1)).cuda(), d)
    tl = torch.empty((B, k + 1, V8), dtype=torch.float32, device="cuda")
    dl = torch.empty((B, k, V8), dtype=torch.float32, device="cuda")
    ot = torch.full((B, k + 1), -9, dtype=torch.int32, device="cuda")
    oa = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    rs = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    mtpv.verify_step(W, Wq, S, Ht, Hd, d.view(B, k), torch.as_tensor(u["u_accept"]).cuda(),
                     torch.as_tensor(u["u_sample"]).cuda(), B, k, T, TOP_P, ot, oa, rs, tl, dl)
    torch.cuda.synchronize()
    assert torch.equal(dl.view(B * k, V8), dl0)  # the step's draft logits are the draft phase's
    rows = np.unique(np.concatenate([np.arange(0, V8, 89), np.arange(V8 - 200, V8)]))
    ridx = torch.as_tensor(rows).cuda()
    ref_t = oracle.lm_head_bf16(synth.bf16_bits(Ht.cpu()), synth.bf16_bits(W[ridx].cpu()), threads=8)
    ref_d = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq[ridx].cpu().numpy(),
                                   synth.bf16_bits(S[ridx].cpu()), threads=8)
    assert_logits_close(tl.view(B * (k + 1), V8)[:, ridx].cpu().numpy(), ref_t)
    assert_logits_close(dl.view(B * k, V8)[:, ridx].cpu().numpy(), ref_d)
    n, f, h = oracle_check(tl.cpu().numpy(), dl.cpu().numpy(), d.view(B, k).cpu().numpy(), u,
                           ot.cpu().numpy(), oa.cpu().numpy(), rs.cpu().numpy())
    assert n == B and f <= 1
