"""GPU parity of mtpv_verify and mtpv_sample against the fp64 oracle.

Both sides read the same fp32 logits (drawn by the seeded generator), the
same drafts (drawn by the oracle from q') and the same uniforms.  Accepted
counts and token ids must be identical on every trial the oracle does not
flag as a boundary case (uniform within 1e-5 of the acceptance ratio; draw
target within 1e-5 of the chosen bin's width from a bin edge; a top-p cut
within 1e-5 of the cut token's mass whose shift changes the outcome), and
flagged trials must stay under 0.01 % of all trials.
"""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import cuda, f32

pytestmark = pytest.mark.gpu

T_PAGES, TOPP_PAGES = 0.6, 0.95
FLAG_LIMIT = 1e-4


class Tally:
    trials = 0
    flagged = 0


def gpu_verify(tl, dl, d, ua, us, T, top_p, row_status=True):
    B, K1, V = tl.shape
    K = K1 - 1
    out_t = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    out_a = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    rs = torch.full((B,), -7, dtype=torch.int32, device="cuda") if row_status else None
    mtpv.verify(cuda(tl), cuda(dl), cuda(torch.as_tensor(d, dtype=torch.int32)),
                cuda(torch.as_tensor(ua)), cuda(torch.as_tensor(us)), T, top_p, out_t, out_a, rs)
    torch.cuda.synchronize()
    return out_t.cpu().numpy(), out_a.cpu().numpy(), None if rs is None else rs.cpu().numpy()


def make_case(B, K, V, seed, T=T_PAGES, top_p=TOPP_PAGES, std=1.43, tau=0.43, grid=None):
    tl, dl = synth.make_verify_logits(B, K, V, std, tau, seed, grid=grid)
    u = synth.step_uniforms(seed, 0, B, K)
    d, _, st = oracle.sample_rows(dl.reshape(B * K, V).double().numpy(), f32(T), f32(top_p),
                                  u["u_draft"].reshape(-1), threads=8)
    return tl, dl, d.reshape(B, K), u


def check_parity(tl, dl, d, u, T, top_p, tally=True):
    tok, acc, rs = gpu_verify(tl, dl, d, u["u_accept"], u["u_sample"], T, top_p)
    ref = oracle.verify(tl.double().numpy(), dl.double().numpy(), d, u["u_accept"], u["u_sample"],
                        f32(T), f32(top_p), threads=8)
    mism = (tok != ref["tokens"]).any(axis=1) | (acc != ref["accepted"])
    unflagged = mism & (ref["flags"] == 0)
    assert not unflagged.any(), (
        f"{unflagged.sum()} unflagged mismatches, first at {np.nonzero(unflagged)[0][:5]}: "
        f"gpu {tok[unflagged][:3]} oracle {ref['tokens'][unflagged][:3]}")
    assert np.array_equal(rs, ref["status"])
    if tally:
        Tally.trials += len(acc)
        Tally.flagged += int((ref["flags"] != 0).sum())
    return tok, acc, ref


def test_tiny_config_1000_trials_batched():
    # hidden 512 / vocab 4096 verify, 1000 seeded trials as 1000 sequences
    tok, acc, ref = check_parity(*make_case(1000, 3, 4096, seed=1), T_PAGES, TOPP_PAGES)
    assert 0.2 < (acc == 3).mean() < 0.95   # acceptance is neither trivial nor zero


def test_tiny_config_single_sequence_launches():
    for seed in range(40):
        check_parity(*make_case(1, 3, 4096, seed=100 + seed), T_PAGES, TOPP_PAGES)


def test_qwen_class_vocab_sampler():
    # vocab 151936, K = 3: the benchmark's sampler shape, 64 sequences per launch
    for seed in range(3):
        check_parity(*make_case(64, 3, 151936, seed=200 + seed), T_PAGES, TOPP_PAGES)
    check_parity(*make_case(1, 3, 151936, seed=299), T_PAGES, TOPP_PAGES)


def test_large_vocab_batched():
    check_parity(*make_case(8, 3, 248320, seed=300), T_PAGES, TOPP_PAGES)


@pytest.mark.parametrize("K", [1, 2, 3, 8, 16])
def test_draft_depths(K):
    check_parity(*make_case(32, K, 5000, seed=400 + K), T_PAGES, TOPP_PAGES)


@pytest.mark.parametrize("T,top_p", [(1.0, 1.0), (0.6, 1.0), (1.3, 0.5), (0.2, 0.9), (1e-3, 0.95),
                                     (0.6, 0.999)])
def test_temperature_and_top_p_grid(T, top_p):
    check_parity(*make_case(64, 3, 3000, seed=500, T=T, top_p=top_p), T, top_p)


def test_greedy():
    tl, dl, _, u = make_case(128, 3, 7000, seed=600, T=0.0)
    d = dl.argmax(dim=2).int().numpy()
    rng = np.random.default_rng(0)
    mask = rng.random(d.shape) < 0.3
    d[mask] = rng.integers(0, 7000, size=mask.sum())
    tok, acc, ref = check_parity(tl, dl, d, u, 0.0, TOPP_PAGES)
    assert (ref["flags"] == 0).all()


def test_ties_on_a_coarse_logit_grid():
    # logits on a 0.25 grid: many exact ties at the top-p cut and in the argmax
    for seed in range(4):
        check_parity(*make_case(64, 3, 4096, seed=700 + seed, grid=0.25), T_PAGES, TOPP_PAGES)
        check_parity(*make_case(64, 3, 4096, seed=710 + seed, T=0.0, grid=0.25), 0.0, TOPP_PAGES)


def crossing_bin_size(row, T, top_p):
    """Tokens in the level-1 bin where the descending mass reaches top_p Z
    (2048 bins linear in (m - l) over the row's range, fp32 as the kernel
    bins them; masses exact here)."""
    L = np.asarray(row, dtype=np.float32)
    m, mn = L.max(), L.min()
    inv_w = np.float32(2048) / np.float32(m - mn)
    b = np.minimum(2047, np.floor((m - L) * inv_w)).astype(np.int64)
    e = np.exp((L.astype(np.float64) - float(m)) / T)
    mass = np.bincount(b, weights=e, minlength=2048)
    c = np.cumsum(mass)
    return int(np.bincount(b, minlength=2048)[min(2047, int(np.searchsorted(c, top_p * c[-1])))])


def test_crossing_bins_sorted_by_the_bitonic_network():
    # logits on a 0.5 grid over 30000 tokens: the crossing logit value is
    # shared by hundreds to thousands of tokens, more than one thread each
    # (512) and within the candidate buffer (4096), so CTA 0 sorts them with
    # its bitonic network before the exact cut
    B, K, V = 8, 3, 30000
    tl, dl, d, u = make_case(B, K, V, seed=930, grid=0.5)
    rows = list(tl.reshape(-1, V).numpy()) + list(dl.reshape(-1, V).numpy())
    sizes = [crossing_bin_size(r, T_PAGES, TOPP_PAGES) for r in rows]
    assert any(512 < n <= 4096 for n in sizes), sizes
    check_parity(tl, dl, d, u, T_PAGES, TOPP_PAGES)


def test_degenerate_rows_take_the_radix_path():
    # all-equal rows and a two-level row: the crossing bin holds far more
    # tokens than the candidate buffer, so the cut comes from the radix select
    B, K, V = 4, 2, 60000
    tl = torch.zeros((B, K + 1, V), dtype=torch.float32)
    dl = torch.zeros((B, K, V), dtype=torch.float32)
    tl[1] = 1.5
    tl[2, :, : V // 2] = 2.0
    dl[3, :, ::3] = 0.5
    u = synth.step_uniforms(9, 0, B, K)
    d, _, _ = oracle.sample_rows(dl.reshape(B * K, V).double().numpy(), f32(T_PAGES), f32(TOPP_PAGES),
                                 u["u_draft"].reshape(-1))
    for top_p in (TOPP_PAGES, 0.5, 0.123):
        check_parity(tl, dl, d.reshape(B, K), u, T_PAGES, top_p, tally=False)


@pytest.mark.parametrize("V", [1, 2, 7, 15, 33])
def test_tiny_vocabularies(V):
    # fewer tokens than CTAs in a cluster: empty slices must be harmless
    check_parity(*make_case(16, 2, V, seed=800 + V), T_PAGES, TOPP_PAGES)
    check_parity(*make_case(16, 2, V, seed=850 + V, T=0.0), 0.0, TOPP_PAGES)


def test_identical_target_and_draft_rows_accept_all():
    B, K, V = 32, 3, 2048
    tl, _, _, u = make_case(B, K, V, seed=900)
    dl = tl[:, :K].clone()
    d, _, _ = oracle.sample_rows(dl.reshape(B * K, V).double().numpy(), f32(T_PAGES), f32(TOPP_PAGES),
                                 u["u_draft"].reshape(-1))
    tok, acc, _ = check_parity(tl, dl, d.reshape(B, K), u, T_PAGES, TOPP_PAGES)
    assert (acc == K).all()


def test_data_errors_are_reported_not_faulted():
    B, K, V = 6, 3, 1000
    tl, dl, d, u = make_case(B, K, V, seed=901)
    d = d.copy()
    d[0, 2] = V
    d[1, 0] = -1
    tl = tl.clone()
    dl = dl.clone()
    tl[2, 1, 17] = float("nan")
    dl[3, 0, 999] = float("inf")
    tl[4, 3, 0] = float("-inf")
    tok, acc, rs = gpu_verify(tl, dl, d, u["u_accept"], u["u_sample"], T_PAGES, TOPP_PAGES)
    assert list(rs) == [1, 1, 2, 2, 2, 0]
    assert (acc[:5] == -1).all() and (tok[:5] == -1).all()
    check_parity(tl, dl, d, u, T_PAGES, TOPP_PAGES, tally=False)


def test_uniform_extremes():
    B, K, V = 64, 3, 4096
    tl, dl, d, u = make_case(B, K, V, seed=902)
    u["u_accept"][:] = 0.0
    u["u_sample"][:32] = 0.0
    u["u_sample"][32:] = np.float32(1 - 2 ** -24)
    check_parity(tl, dl, d, u, T_PAGES, TOPP_PAGES, tally=False)


def test_workspace_reuse_across_calls():
    # the call clears its own counters: back-to-back calls on one workspace
    B, K, V = 16, 3, 4096
    tl, dl, d, u = make_case(B, K, V, seed=903)
    ws = mtpv.workspace(mtpv.verify_workspace_bytes(B, K, V))
    ws.fill_(0xAB)
    outs = []
    for _ in range(3):
        ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
        oa = torch.empty((B,), dtype=torch.int32, device="cuda")
        mtpv.verify(cuda(tl), cuda(dl), cuda(torch.as_tensor(d)), cuda(torch.as_tensor(u["u_accept"])),
                    cuda(torch.as_tensor(u["u_sample"])), T_PAGES, TOPP_PAGES, ot, oa, ws=ws)
        outs.append(ot.cpu())
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    ref = oracle.verify(tl.double().numpy(), dl.double().numpy(), d, u["u_accept"], u["u_sample"],
                        f32(T_PAGES), f32(TOPP_PAGES))
    ok = (ref["flags"] != 0) | (outs[0].numpy() == ref["tokens"]).all(axis=1)
    assert ok.all()


@pytest.mark.parametrize("T,top_p", [(T_PAGES, TOPP_PAGES), (1.0, 1.0), (0.0, TOPP_PAGES)])
def test_sample_rows_parity(T, top_p):
    R, V = 256, 30000
    l = synth.make_logits(R, V, 1.43, seed=77)
    u = synth.uniforms(78, np.arange(R))
    out = torch.empty((R,), dtype=torch.int32, device="cuda")
    rs = torch.empty((R,), dtype=torch.int32, device="cuda")
    mtpv.sample(cuda(l), T, top_p, cuda(torch.as_tensor(u)), out, rs)
    torch.cuda.synchronize()
    ref, margin, st = oracle.sample_rows(l.double().numpy(), f32(T), f32(top_p), u, threads=8)
    flagged = margin < oracle.WINDOW if T > 0 else np.zeros(R, bool)
    got = out.cpu().numpy()
    assert ((got == ref) | flagged).all()
    assert (rs.cpu().numpy() == 0).all()


def test_flag_rate_under_limit():
    """Runs last in this module: the boundary-case rate over every trial above."""
    assert Tally.trials >= 1000
    assert Tally.flagged / Tally.trials < FLAG_LIMIT, (Tally.flagged, Tally.trials)
