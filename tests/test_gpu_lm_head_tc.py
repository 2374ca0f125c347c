"""The bf16 LM head for 9..64 activation rows on the tensor-memory path
(tcgen05.mma with the accumulator in tensor memory, TMA-fed shared-memory
stages), which reads every weight once whatever the row count.

Checked against the fp64 oracle within 1e-3 relative on ragged shapes (N
not a multiple of the 128-row tile, a single k slice, rows not a multiple
of 16), bit for bit on small integers (every partial sum exact), bit for bit
between two calls, and with its error word (the first word of the
workspace: a bounded device wait gave up) left at zero.  The passage: the
verify pass's small-row-count matmul through the LM head (hazakura.dev
MTPLX notes, "4-layer architecture", Layer 0), here batched over sequences.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close

pytestmark = pytest.mark.gpu


def run(x, W):
    M, Kd = x.shape
    N = W.shape[0]
    need = mtpv.lm_head_workspace_bytes(M, Kd, N, mtpv.W_BF16)
    assert need >= 4
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(x.cuda(), W.cuda(), None, mtpv.W_BF16, y, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a bounded wait of the kernel gave up"
    return y


@pytest.mark.parametrize("M,Kd,N", [(9, 512, 4097), (16, 64, 129), (17, 5120, 1000), (24, 512, 128),
                                    (32, 5120, 3001), (40, 1024, 127), (64, 512, 5000), (33, 192, 1)])
def test_against_oracle(M, Kd, N):
    W = synth.make_head(N, Kd, 0.02, seed=N + 3 * Kd)
    x = synth.gaussian((M, Kd), 1.0, seed=M + Kd)
    y = run(x, W).cpu().numpy()
    assert np.isfinite(y).all()
    assert_logits_close(y, oracle.lm_head_bf16(synth.bf16_bits(x), synth.bf16_bits(W), threads=8))


@pytest.mark.parametrize("M,N", [(32, 2000), (9, 257), (64, 130)])
def test_bit_exact_on_small_integers(M, N):
    rng = np.random.default_rng(M)
    Kd = 1024
    x = torch.tensor(rng.integers(-4, 5, size=(M, Kd)), dtype=torch.float32).to(torch.bfloat16)
    W = torch.tensor(rng.integers(-8, 9, size=(N, Kd)), dtype=torch.float32).to(torch.bfloat16)
    y = run(x, W).cpu().numpy()
    assert np.array_equal(y.astype(np.float64), oracle.lm_head_bf16(synth.bf16_bits(x), synth.bf16_bits(W)))


def test_repeatable_and_equal_to_row_subsets():
    # the same rows alone (a smaller M) give the same values: every output
    # element is its own dot product
    N, Kd = 20000, 5120
    W = synth.make_head(N, Kd, 0.02, seed=9, device="cuda")
    x = synth.gaussian((32, Kd), 1.0, seed=10, device="cuda")
    a = run(x, W)
    b = run(x, W)
    assert torch.equal(a, b)
    c = run(x[:17].contiguous(), W)
    assert torch.equal(a[:17], c)


def test_workspace_is_required():
    M, Kd, N = 20, 512, 300
    lib = mtpv.load()
    x = torch.zeros((M, Kd), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((N, Kd), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.mtpv_lm_head_smallm(p(x), M, Kd, N, p(W), None, mtpv.W_BF16, p(y), None, 0, None)
    assert st == 3  # MTPV_ERR_WORKSPACE


# ---------------------------------------------------------------------------
# int4 group-64 head (dequantised into tensor memory, fp16 MMA)
# ---------------------------------------------------------------------------
def run_int4(x, Wq, S):
    M, Kd = x.shape
    N = Wq.shape[0]
    need = mtpv.lm_head_workspace_bytes(M, Kd, N, mtpv.W_INT4_G64)
    assert need >= 4
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(x.cuda(), Wq.cuda(), S.cuda(), mtpv.W_INT4_G64, y, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a bounded wait of the kernel gave up"
    return y


@pytest.mark.parametrize("M,Kd,N", [(9, 512, 4097), (24, 5120, 3001), (32, 1024, 129), (64, 512, 300),
                                    (17, 2048, 1), (48, 8192, 200)])
def test_int4_against_oracle(M, Kd, N):
    W = synth.make_head(N, Kd, 0.02, seed=7 * N + Kd)
    Wq, S = synth.quantize_int4_g64(W)
    x = synth.gaussian((M, Kd), 1.0, seed=3 * M + Kd)
    y = run_int4(x, Wq, S).cpu().numpy()
    assert np.isfinite(y).all()
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x), Wq.numpy(), synth.bf16_bits(S), threads=8)
    assert_logits_close(y, ref)


@pytest.mark.parametrize("M,N", [(24, 1500), (9, 300), (64, 129)])
def test_int4_bit_exact_on_small_integers(M, N):
    # power-of-two scales, small-integer activations: the products and every
    # partial sum are exact in fp32 (within 20 bits of each other)
    rng = np.random.default_rng(100 + M)
    Kd = 1024
    Wq = torch.tensor(rng.integers(0, 256, size=(N, Kd // 2)), dtype=torch.uint8)
    S = torch.tensor(2.0 ** rng.integers(-2, 3, size=(N, Kd // 64)), dtype=torch.float32).to(torch.bfloat16)
    x = torch.tensor(rng.integers(-3, 4, size=(M, Kd)), dtype=torch.float32).to(torch.bfloat16)
    y = run_int4(x, Wq, S).cpu().numpy()
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x), Wq.numpy(), synth.bf16_bits(S))
    assert np.array_equal(y.astype(np.float64), ref)


def test_int4_repeatable_and_wide_scale_range():
    # rows whose group scales span 2^12 (and one all-zero row): the per-row
    # power of two keeps every dequantised weight exact in fp16
    N, Kd, M = 3000, 5120, 24
    W = synth.make_head(N, Kd, 0.02, seed=21)
    W[5] *= 4096.0
    W[6] *= 1.0 / 4096.0
    W[7] = 0.0
    W[8, :64] *= 2048.0
    Wq, S = synth.quantize_int4_g64(W.to(torch.bfloat16))
    x = synth.gaussian((M, Kd), 1.0, seed=22)
    a = run_int4(x, Wq, S)
    b = run_int4(x, Wq, S)
    assert torch.equal(a, b)
    ref = oracle.lm_head_int4g64(synth.bf16_bits(x), Wq.numpy(), synth.bf16_bits(S), threads=8)
    assert_logits_close(a.cpu().numpy(), ref)
