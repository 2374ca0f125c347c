"""mtpv_draft_loop: the draft phase (K positions, each an int4-head
projection followed by one draw from q').

The draft logits are compared with the fp64 oracle (<= 1e-3 relative, row
rms floor); the draft tokens with the oracle's own draw on the GPU's fp32
draft logits, identical except where the oracle flags the draw as within
1e-5 of a bin edge (relative to the chosen bin).
"""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close, f32

pytestmark = pytest.mark.gpu

T, TOP_P = 0.6, 0.95


def run_case(B, K, V, h, wstd, seed, with_logits=True):
    W = synth.make_head(V, h, wstd, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    _, Hd = synth.make_hidden(B, K, h, 0.3, seed=seed, device="cuda")
    u = synth.step_uniforms(seed, 0, B, K)
    ud = torch.as_tensor(u["u_draft"]).reshape(B, K).contiguous().cuda()
    d = torch.full((B, K), -9, dtype=torch.int32, device="cuda")
    dl = torch.full((B, K, V), float("nan"), device="cuda") if with_logits else None
    mtpv.draft_loop(Wq, S, Hd, ud, B, K, T, TOP_P, d, dl)
    torch.cuda.synchronize()
    return Wq, S, Hd, u, d, dl


@pytest.mark.parametrize("B,K", [(1, 3), (1, 1), (3, 2), (4, 5)])
def test_tiny_draft_loop_against_oracle(B, K):
    V, h = 4096, 512
    Wq, S, Hd, u, d, dl = run_case(B, K, V, h, 0.05, seed=40 + B * 10 + K)
    ref_l = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()),
                                   threads=8)
    got_l = dl.reshape(B * K, V).cpu().numpy()
    assert_logits_close(got_l, ref_l)
    tok, margin, st = oracle.sample_rows(got_l.astype(np.float64), f32(T), f32(TOP_P),
                                         u["u_draft"].reshape(-1), threads=8)
    got = d.reshape(-1).cpu().numpy()
    assert ((got == tok) | (margin < oracle.WINDOW)).all()
    assert (st == 0).all() and (got >= 0).all()


def test_draft_logits_optional():
    B, K, V, h = 2, 3, 4096, 512
    *_, d1, _ = run_case(B, K, V, h, 0.05, seed=9)
    *_, d2, _ = run_case(B, K, V, h, 0.05, seed=9, with_logits=False)
    assert torch.equal(d1, d2)


def test_qwen_class_draft_loop():
    B, K, V, h = 1, 3, 151936, 5120
    Wq, S, Hd, u, d, dl = run_case(B, K, V, h, 0.02, seed=3)
    got_l = dl.reshape(B * K, V).cpu().numpy()
    rows = np.arange(0, V, 53)
    ref_l = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq[rows].cpu().numpy(),
                                   synth.bf16_bits(S[rows].cpu()), threads=8)
    assert_logits_close(got_l[:, rows], ref_l)
    tok, margin, st = oracle.sample_rows(got_l.astype(np.float64), f32(T), f32(TOP_P),
                                         u["u_draft"].reshape(-1), threads=8)
    got = d.reshape(-1).cpu().numpy()
    assert ((got == tok) | (margin < oracle.WINDOW)).all()
