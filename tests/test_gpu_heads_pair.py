"""mtpv_lm_head_pair: both heads of a verify step in one call.

The fused kernel runs each head's arithmetic exactly as mtpv_lm_head_smallm
does, so its logits must equal the single-head calls bit for bit, on the
shapes the fused kernel takes and on the ones that fall back to two
launches; one shape is also checked against the fp64 oracle.  The verify
step's own logits (mtpv_verify_step) must equal them as well.
"""
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close

pytestmark = pytest.mark.gpu


def heads(N, Kd, seed, wstd=0.02):
    W = synth.make_head(N, Kd, wstd, seed=seed, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    return W, Wq, S


def hidden(M, Kd, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((M, Kd), generator=g, device="cuda").to(torch.bfloat16)


# (Mt, Md, Kd, N): fused shapes, then shapes that take two launches
SHAPES = [(4, 3, 5120, 151936), (2, 1, 5120, 151936), (3, 2, 512, 4096), (1, 1, 512, 1000),
          (4, 4, 1024, 4099), (8, 6, 512, 4096), (4, 8, 5120, 20000), (8, 8, 5120, 20011),
          (4, 3, 640, 4096), (12, 3, 512, 4096), (9, 9, 1024, 3000)]


@pytest.mark.parametrize("Mt,Md,Kd,N", SHAPES)
def test_pair_equals_single_head_calls(Mt, Md, Kd, N):
    W, Wq, S = heads(N, Kd, 100 + Kd)
    xt, xd = hidden(Mt, Kd, 1), hidden(Md, Kd, 2)
    yt = torch.full((Mt, N), float("nan"), device="cuda")
    yd = torch.full((Md, N), float("nan"), device="cuda")
    mtpv.lm_head_pair(xt, W, yt, xd, Wq, S, yd)
    rt = torch.empty_like(yt)
    rd = torch.empty_like(yd)
    mtpv.lm_head_smallm(xt, W, None, mtpv.W_BF16, rt)
    mtpv.lm_head_smallm(xd, Wq, S, mtpv.W_INT4_G64, rd)
    torch.cuda.synchronize()
    assert torch.equal(yt, rt)
    assert torch.equal(yd, rd)


def test_pair_against_oracle_on_sampled_rows():
    Mt, Md, Kd, N = 4, 3, 5120, 151936
    W, Wq, S = heads(N, Kd, 7)
    xt, xd = hidden(Mt, Kd, 3), hidden(Md, Kd, 4)
    yt = torch.empty((Mt, N), device="cuda")
    yd = torch.empty((Md, N), device="cuda")
    mtpv.lm_head_pair(xt, W, yt, xd, Wq, S, yd)
    torch.cuda.synchronize()
    rows = torch.arange(0, N, 37)  # spans every CTA's share of the vocabulary, ragged tail included
    ref_t = oracle.lm_head_bf16(synth.bf16_bits(xt.cpu()), synth.bf16_bits(W[rows].cpu()), threads=8)
    ref_d = oracle.lm_head_int4g64(synth.bf16_bits(xd.cpu()), Wq[rows].cpu().numpy(),
                                   synth.bf16_bits(S[rows].cpu()), threads=8)
    assert_logits_close(yt[:, rows].cpu().numpy(), ref_t)
    assert_logits_close(yd[:, rows].cpu().numpy(), ref_d)


def test_pair_exact_on_small_integers():
    """Power-of-two scales, small-integer activations: every sum is exact in
    fp32, so the fused kernel equals the fp64 oracle bit for bit."""
    Mt, Md, Kd, N = 4, 3, 1024, 2000
    g = torch.Generator().manual_seed(5)
    W = (torch.randint(-7, 8, (N, Kd), generator=g).float() * 0.25).to(torch.bfloat16).cuda()
    Wq = torch.randint(0, 256, (N, Kd // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    S = torch.pow(2.0, torch.randint(-2, 3, (N, Kd // 64), generator=g).float()).to(torch.bfloat16)
    xt = torch.randint(-3, 4, (Mt, Kd), generator=g).float().to(torch.bfloat16).cuda()
    xd = torch.randint(-3, 4, (Md, Kd), generator=g).float().to(torch.bfloat16).cuda()
    yt = torch.empty((Mt, N), device="cuda")
    yd = torch.empty((Md, N), device="cuda")
    mtpv.lm_head_pair(xt, W, yt, xd, Wq.cuda(), S.cuda(), yd)
    torch.cuda.synchronize()
    ref_t = oracle.lm_head_bf16(synth.bf16_bits(xt.cpu()), synth.bf16_bits(W.cpu()), threads=8)
    ref_d = oracle.lm_head_int4g64(synth.bf16_bits(xd.cpu()), Wq.numpy(), synth.bf16_bits(S), threads=8)
    assert (yt.cpu().double().numpy() == ref_t).all()
    assert (yd.cpu().double().numpy() == ref_d).all()


@pytest.mark.parametrize("B,K", [(1, 3), (1, 1), (2, 3)])
def test_verify_step_logits_equal_single_head_calls(B, K):
    V, h = 151936, 5120
    W, Wq, S = heads(V, h, 11)
    Ht, Hd = synth.make_hidden(B, K, h, 0.3, seed=6, device="cuda")
    u = synth.step_uniforms(6, 0, B, K)
    d = torch.zeros((B, K), dtype=torch.int32, device="cuda")
    tl = torch.empty((B, K + 1, V), device="cuda")
    dl = torch.empty((B, K, V), device="cuda")
    ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    oa = torch.empty((B,), dtype=torch.int32, device="cuda")
    mtpv.verify_step(W, Wq, S, Ht, Hd, d, torch.as_tensor(u["u_accept"]).cuda(),
                     torch.as_tensor(u["u_sample"]).cuda(), B, K, 0.6, 0.95, ot, oa, None, tl, dl)
    rt = torch.empty((B * (K + 1), V), device="cuda")
    rd = torch.empty((B * K, V), device="cuda")
    mtpv.lm_head_smallm(Ht, W, None, mtpv.W_BF16, rt)
    mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, rd)
    torch.cuda.synchronize()
    assert torch.equal(tl.view(B * (K + 1), V), rt)
    assert torch.equal(dl.view(B * K, V), rd)
