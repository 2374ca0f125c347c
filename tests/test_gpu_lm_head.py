"""GPU parity of mtpv_lm_head_smallm against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close, cuda

pytestmark = pytest.mark.gpu


def run_gpu(x, w, scales, fmt):
    M = x.shape[0]
    N = w.shape[0]
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    mtpv.lm_head_smallm(cuda(x), cuda(w), None if scales is None else cuda(scales), fmt, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def bits(t):
    return synth.bf16_bits(t)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_bf16_tiny_config_all_M(M):
    # the tiny verify config: hidden 512, vocab 4096, W ~ N(0, 0.05^2)
    W = synth.make_head(4096, 512, 0.05, seed=12345)
    x = synth.gaussian((M, 512), 1.0, seed=M)
    y = run_gpu(x, W, None, mtpv.W_BF16)
    assert_logits_close(y, oracle.lm_head_bf16(bits(x), bits(W), threads=8))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_int4_tiny_config_all_M(M):
    W = synth.make_head(4096, 512, 0.05, seed=12345)
    Wq, S = synth.quantize_int4_g64(W)
    x = synth.gaussian((M, 512), 1.0, seed=100 + M)
    y = run_gpu(x, Wq, S, mtpv.W_INT4_G64)
    assert_logits_close(y, oracle.lm_head_int4g64(bits(x), Wq.numpy(), bits(S), threads=8))


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,Kd,N", [(3, 64, 1), (4, 192, 999), (2, 1024, 4097), (16, 512, 300),
                                    (32, 256, 77), (12, 5120, 513), (6, 17408, 130), (8, 17408, 64),
                                    (3, 58112, 40)])
def test_ragged_shapes(fmt, M, Kd, N):
    # N not a multiple of the rows per warp, Kd not a multiple of the lane
    # stride, M above 8 (row groups), long Kd limited by shared memory
    W = synth.make_head(N, Kd, 0.02, seed=N + Kd)
    x = synth.gaussian((M, Kd), 1.0, seed=M * 7 + Kd)
    if fmt == 0:
        ref = oracle.lm_head_bf16(bits(x), bits(W), threads=8)
        y = run_gpu(x, W, None, fmt)
    else:
        Wq, S = synth.quantize_int4_g64(W)
        ref = oracle.lm_head_int4g64(bits(x), Wq.numpy(), bits(S), threads=8)
        y = run_gpu(x, Wq, S, fmt)
    assert np.isfinite(y).all()
    assert_logits_close(y, ref)


def test_bf16_bit_exact_on_small_integers():
    # integer activations and weights: every fp32 partial sum is exact, so the
    # GPU must equal the oracle bit for bit whatever its summation order
    rng = np.random.default_rng(0)
    M, Kd, N = 4, 1024, 2000
    x = torch.tensor(rng.integers(-4, 5, size=(M, Kd)), dtype=torch.float32).to(torch.bfloat16)
    W = torch.tensor(rng.integers(-8, 9, size=(N, Kd)), dtype=torch.float32).to(torch.bfloat16)
    y = run_gpu(x, W, None, mtpv.W_BF16)
    assert np.array_equal(y.astype(np.float64), oracle.lm_head_bf16(bits(x), bits(W)))


def test_int4_bit_exact_on_small_integers():
    rng = np.random.default_rng(1)
    M, Kd, N = 3, 1024, 1500
    Wq = torch.tensor(rng.integers(0, 256, size=(N, Kd // 2)), dtype=torch.uint8)
    S = torch.tensor(2.0 ** rng.integers(-2, 3, size=(N, Kd // 64)), dtype=torch.float32).to(torch.bfloat16)
    x = torch.tensor(rng.integers(-3, 4, size=(M, Kd)), dtype=torch.float32).to(torch.bfloat16)
    y = run_gpu(x, Wq, S, mtpv.W_INT4_G64)
    assert np.array_equal(y.astype(np.float64), oracle.lm_head_int4g64(bits(x), Wq.numpy(), bits(S)))


def test_one_hot_activation_returns_a_weight_column():
    W = synth.make_head(3000, 512, 0.05, seed=3)
    x = torch.zeros((2, 512), dtype=torch.bfloat16)
    x[0, 5] = 1.0
    x[1, 511] = 1.0
    y = run_gpu(x, W, None, mtpv.W_BF16)
    assert np.array_equal(y[0], W.float().numpy()[:, 5])
    assert np.array_equal(y[1], W.float().numpy()[:, 511])


@pytest.mark.parametrize("M,fmt", [(4, 0), (3, 1), (32, 0), (24, 1)])
def test_qwen_class_head_sampled_rows(M, fmt):
    """Full-size head (vocab 151936, hidden 5120) in the launch shape of the
    benchmark; the oracle checks a strided sample of vocabulary rows."""
    V, h = 151936, 5120
    W = synth.make_head(V, h, 0.02, seed=12345, device="cuda")
    x = synth.gaussian((M, h), 1.0, seed=7 + M, device="cuda")
    y = torch.empty((M, V), dtype=torch.float32, device="cuda")
    if fmt == 0:
        mtpv.lm_head_smallm(x, W, None, fmt, y)
    else:
        Wq, S = synth.quantize_int4_g64(W)
        mtpv.lm_head_smallm(x, Wq, S, fmt, y)
    torch.cuda.synchronize()
    yc = y.cpu().numpy()
    # every 41st vocabulary row (rows of every warp's tiles across the grid),
    # plus two contiguous windows and the ragged tail
    rows = np.unique(np.concatenate([np.arange(0, V, 41), np.arange(77777, 77841), np.arange(V - 64, V)]))
    ridx = torch.as_tensor(rows).cuda()
    xb = bits(x.cpu())
    if fmt == 0:
        ref = oracle.lm_head_bf16(xb, bits(W[ridx].cpu()), threads=8)
    else:
        ref = oracle.lm_head_int4g64(xb, Wq[ridx].cpu().numpy(), bits(S[ridx].cpu()), threads=8)
    assert_logits_close(yc[:, rows], ref)
    assert np.isfinite(yc).all()
