"""Decoder-layer projections with int4 g64 weights (mtpv_int4_proj,
mtpv_int4_gate_up) at the small-M shapes of a 27B-class layer, against the
fp64 oracle: <= 1e-3 relative per element (row-rms floor) on sampled
columns; bit-exact on small-integer inputs; deterministic across calls."""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close

pytestmark = pytest.mark.gpu

# (name, Kd, N): attention qkv and o, MLP down; gate||up is tested separately
SHAPES = [("qkv", 5120, 7168), ("o", 5120, 5120), ("down", 17408, 5120)]

_heads = {}


def head(N, Kd, seed):
    key = (N, Kd, seed)
    if key not in _heads:
        W = synth.make_head(N, Kd, 0.02, seed=seed, device="cuda")
        _heads[key] = synth.quantize_int4_g64(W)
    return _heads[key]


def hidden(M, Kd, seed):
    return synth.gaussian((M, Kd), 1.0, seed, "cuda")


@pytest.mark.parametrize("name,Kd,N", SHAPES)
@pytest.mark.parametrize("M", [1, 3, 4, 8])
def test_projection_against_oracle(name, Kd, N, M):
    Wq, S = head(N, Kd, 21)
    x = hidden(M, Kd, 100 + M)
    y = torch.full((M, N), float("nan"), device="cuda")
    mtpv.int4_proj(x, Wq, S, y)
    torch.cuda.synchronize()
    cols = np.arange(0, N, 7)
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x.cpu()), Wq[cols].cpu().numpy(),
                                 synth.bf16_bits(S[cols].cpu()), threads=8)
    assert_logits_close(y[:, cols].cpu().numpy(), ref)
    assert not torch.isnan(y).any()


@pytest.mark.parametrize("M", [1, 2, 5, 6, 8])
def test_gate_up_silu_against_oracle(M):
    F, Kd = 17408, 5120
    Wq, S = head(2 * F, Kd, 22)
    x = hidden(M, Kd, 200 + M)
    h = torch.full((M, F), float("nan"), device="cuda")
    mtpv.int4_gate_up(x, Wq, S, h)
    torch.cuda.synchronize()
    cols = np.arange(3, F, 11)
    ref = oracle.gate_up_int4g64(synth.bf16_bits(x.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()),
                                 F, cols=cols, threads=8)
    assert_logits_close(h[:, cols].cpu().numpy(), ref)
    assert not torch.isnan(h).any()


def test_projection_exact_on_small_integers_and_deterministic():
    M, Kd, N = 4, 17408, 1000
    g = torch.Generator().manual_seed(9)
    Wq = torch.randint(0, 256, (N, Kd // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    S = torch.pow(2.0, torch.randint(-2, 3, (N, Kd // 64), generator=g).float()).to(torch.bfloat16)
    x = torch.randint(-3, 4, (M, Kd), generator=g).float().to(torch.bfloat16)
    y1 = torch.empty((M, N), device="cuda")
    y2 = torch.empty((M, N), device="cuda")
    mtpv.int4_proj(x.cuda(), Wq.cuda(), S.cuda(), y1)
    mtpv.int4_proj(x.cuda(), Wq.cuda(), S.cuda(), y2)
    torch.cuda.synchronize()
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x), Wq.numpy(), synth.bf16_bits(S), threads=8)
    assert (y1.cpu().double().numpy() == ref).all()
    assert torch.equal(y1, y2)


def test_many_rows_take_several_passes():
    # 20 rows at Kd = 17408: one pass of the wide kernel; every row checked on sampled columns
    M, Kd, N = 20, 17408, 5120
    Wq, S = head(N, Kd, 21)
    x = hidden(M, Kd, 300)
    y = torch.empty((M, N), device="cuda")
    mtpv.int4_proj(x, Wq, S, y)
    torch.cuda.synchronize()
    cols = np.arange(1, N, 13)
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x.cpu()), Wq[cols].cpu().numpy(),
                                 synth.bf16_bits(S[cols].cpu()), threads=8)
    assert_logits_close(y[:, cols].cpu().numpy(), ref)


# Ragged shapes: a single group, a stage with one valid group (Kd = 576),
# scale rows that straddle 16-byte chunks (Kd / 64 not a multiple of 8),
# N not a multiple of the 128-row tile, fewer stages than SMs.
RAGGED = [(1, 64, 1), (3, 576, 200), (8, 11008, 1000), (5, 192, 129), (2, 1088, 7168), (7, 5120, 130)]


@pytest.mark.parametrize("M,Kd,N", RAGGED)
def test_ragged_projection_against_oracle(M, Kd, N):
    Wq, S = head(N, Kd, 31)
    x = hidden(M, Kd, 400 + M)
    y = torch.full((M, N), float("nan"), device="cuda")
    ws = mtpv.workspace(mtpv.load().mtpv_int4_proj_workspace_bytes(M, Kd, N))
    mtpv.int4_proj(x, Wq, S, y, ws=ws)
    torch.cuda.synchronize()
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()), threads=8)
    assert_logits_close(y.cpu().numpy(), ref)
    # the error word is clear and every ticket counter is back at zero
    assert int(ws[:4].view(torch.int32).item()) == 0
    tiles = (N + 127) // 128
    assert not ws[256:256 + 4 * tiles].any()


@pytest.mark.parametrize("M,Kd,F", [(1, 64, 1), (4, 576, 1001), (8, 192, 37), (3, 11008, 300)])
def test_ragged_gate_up_against_oracle(M, Kd, F):
    Wq, S = head(2 * F, Kd, 32)
    x = hidden(M, Kd, 500 + M)
    h = torch.full((M, F), float("nan"), device="cuda")
    ws = mtpv.workspace(mtpv.load().mtpv_int4_gate_up_workspace_bytes(M, Kd, F))
    mtpv.int4_gate_up(x, Wq, S, h, ws=ws)
    torch.cuda.synchronize()
    ref = oracle.gate_up_int4g64(synth.bf16_bits(x.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()), F,
                                 threads=8)
    assert_logits_close(h.cpu().numpy(), ref)
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert not ws[256:256 + 4 * ((F + 63) // 64)].any()


def test_one_workspace_serves_successive_shapes():
    # the counters a call leaves at zero are what the next call needs
    shapes = [(3, 5120, 7168), (1, 17408, 5120), (8, 576, 200), (3, 5120, 7168)]
    need = max(mtpv.load().mtpv_int4_proj_workspace_bytes(M, Kd, N) for M, Kd, N in shapes)
    shared = mtpv.workspace(need)
    for M, Kd, N in shapes:
        Wq, S = head(N, Kd, 33)
        x = hidden(M, Kd, 600 + M)
        a = torch.empty((M, N), device="cuda")
        b = torch.empty((M, N), device="cuda")
        mtpv.int4_proj(x, Wq, S, a, ws=shared)
        mtpv.int4_proj(x, Wq, S, b)
        torch.cuda.synchronize()
        assert torch.equal(a, b)
    assert int(shared[:4].view(torch.int32).item()) == 0


# Passes of 9..32 rows run on the wide kernel (2..4 n-tiles of 8 rows);
# 33 and 40 rows take a wide pass and a narrow one.
@pytest.mark.parametrize("M,Kd,N", [(9, 5120, 7168), (12, 576, 200), (16, 192, 129), (24, 5120, 1000),
                                    (32, 11008, 1000), (33, 1088, 300), (40, 5120, 130)])
def test_wide_passes_against_oracle(M, Kd, N):
    Wq, S = head(N, Kd, 41)
    x = hidden(M, Kd, 700 + M)
    y = torch.full((M, N), float("nan"), device="cuda")
    ws = mtpv.workspace(mtpv.load().mtpv_int4_proj_workspace_bytes(M, Kd, N))
    mtpv.int4_proj(x, Wq, S, y, ws=ws)
    torch.cuda.synchronize()
    cols = np.arange(0, N, 5) if N > 2000 else np.arange(N)
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x.cpu()), Wq[cols].cpu().numpy(), synth.bf16_bits(S[cols].cpu()),
                                 threads=8)
    assert_logits_close(y[:, cols].cpu().numpy(), ref)
    assert not torch.isnan(y).any()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert not ws[256:512].any()  # ticket counters (one per SM) back at zero


@pytest.mark.parametrize("M,Kd,F", [(12, 5120, 1001), (20, 576, 37)])
def test_wide_gate_up_against_oracle(M, Kd, F):
    Wq, S = head(2 * F, Kd, 42)
    x = hidden(M, Kd, 800 + M)
    h = torch.full((M, F), float("nan"), device="cuda")
    mtpv.int4_gate_up(x, Wq, S, h)
    torch.cuda.synchronize()
    ref = oracle.gate_up_int4g64(synth.bf16_bits(x.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()), F,
                                 threads=8)
    assert_logits_close(h.cpu().numpy(), ref)


def test_wide_pass_exact_on_small_integers_and_deterministic():
    M, Kd, N = 24, 4096, 700
    g = torch.Generator().manual_seed(19)
    Wq = torch.randint(0, 256, (N, Kd // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    S = torch.pow(2.0, torch.randint(-2, 3, (N, Kd // 64), generator=g).float()).to(torch.bfloat16)
    x = torch.randint(-3, 4, (M, Kd), generator=g).float().to(torch.bfloat16)
    y1 = torch.empty((M, N), device="cuda")
    y2 = torch.empty((M, N), device="cuda")
    mtpv.int4_proj(x.cuda(), Wq.cuda(), S.cuda(), y1)
    mtpv.int4_proj(x.cuda(), Wq.cuda(), S.cuda(), y2)
    torch.cuda.synchronize()
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x), Wq.numpy(), synth.bf16_bits(S), threads=8)
    assert (y1.cpu().double().numpy() == ref).all()
    assert torch.equal(y1, y2)
