"""Pins for the oracle's LM-head projections and the int4 group-64 format.

The oracle's fp64 loops are checked against integer arithmetic (exact),
against numpy's float64 matmul on an independently unpacked head, and the
storage format against an independent byte-level restatement.
"""
import numpy as np
import pytest
import torch

import oracle
from verify_step_lm_b200 import synth


def _bits(t):
    return synth.bf16_bits(t)


def _bf16_from_float(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_bf16_head_exact_on_small_integers():
    # Small integers are exact in bf16, and every partial sum is an integer far
    # below 2**53, so the fp64 result must equal int64 matmul bit for bit.
    rng = np.random.default_rng(1)
    M, Kd, N = 5, 192, 77
    xi = rng.integers(-8, 9, size=(M, Kd))
    wi = rng.integers(-16, 17, size=(N, Kd))
    y = oracle.lm_head_bf16(_bits(_bf16_from_float(xi)), _bits(_bf16_from_float(wi)))
    ref = (xi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float64)
    assert np.array_equal(y, ref)


def test_bf16_head_matches_numpy_float64():
    rng = np.random.default_rng(2)
    M, Kd, N = 4, 512, 300
    x = _bf16_from_float(rng.standard_normal((M, Kd)))
    W = _bf16_from_float(0.05 * rng.standard_normal((N, Kd)))
    y = oracle.lm_head_bf16(_bits(x), _bits(W), threads=3)
    ref = x.double().numpy() @ W.double().numpy().T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_bf16_head_one_hot_selects_a_column():
    rng = np.random.default_rng(3)
    Kd, N = 128, 50
    W = _bf16_from_float(rng.standard_normal((N, Kd)))
    x = np.zeros((2, Kd), dtype=np.float32)
    x[0, 17] = 1.0
    x[1, 100] = -2.0
    y = oracle.lm_head_bf16(_bits(_bf16_from_float(x)), _bits(W))
    assert np.array_equal(y[0], W.double().numpy()[:, 17])
    assert np.array_equal(y[1], -2.0 * W.double().numpy()[:, 100])


def test_bf16_head_row_subset():
    rng = np.random.default_rng(4)
    x = _bf16_from_float(rng.standard_normal((3, 64)))
    W = _bf16_from_float(rng.standard_normal((40, 64)))
    full = oracle.lm_head_bf16(_bits(x), _bits(W))
    part = oracle.lm_head_bf16(_bits(x), _bits(W), rows=(10, 25))
    assert np.array_equal(part[:, 10:25], full[:, 10:25])
    assert not part[:, :10].any() and not part[:, 25:].any()


def _unpack_int4(Wq, S):
    """Independent dequantisation: low nibble is the even weight."""
    lo = (Wq & 0x0F).astype(np.int64) - 8
    hi = (Wq >> 4).astype(np.int64) - 8
    q = np.empty((Wq.shape[0], Wq.shape[1] * 2), dtype=np.int64)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    s = torch.tensor(S.view(np.int16)).view(torch.bfloat16).double().numpy()
    return q, np.repeat(s, 64, axis=1)


def test_int4_head_exact_on_small_integers():
    # Scales that are powers of two and integer activations: exact in fp64.
    rng = np.random.default_rng(5)
    M, Kd, N = 3, 256, 33
    Wq = rng.integers(0, 256, size=(N, Kd // 2), dtype=np.uint8)
    s = 2.0 ** rng.integers(-3, 4, size=(N, Kd // 64))
    S = _bits(_bf16_from_float(s))
    xi = rng.integers(-5, 6, size=(M, Kd))
    y = oracle.lm_head_int4g64(_bits(_bf16_from_float(xi)), Wq, S)
    q, sc = _unpack_int4(Wq, S)
    ref = xi.astype(np.float64) @ (q * sc).T
    assert np.array_equal(y, ref)


def test_int4_head_matches_numpy_float64():
    rng = np.random.default_rng(6)
    M, Kd, N = 8, 512, 129
    W = _bf16_from_float(0.02 * rng.standard_normal((N, Kd)))
    Wq, S = synth.quantize_int4_g64(W)
    x = _bf16_from_float(rng.standard_normal((M, Kd)))
    y = oracle.lm_head_int4g64(_bits(x), Wq.numpy(), _bits(S), threads=2)
    q, sc = _unpack_int4(Wq.numpy(), _bits(S))
    ref = x.double().numpy() @ (q * sc).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_quantizer_generator_matches_oracle_bytes():
    rng = np.random.default_rng(7)
    W = _bf16_from_float(0.02 * rng.standard_normal((257, 320)))
    Wq_t, S_t = synth.quantize_int4_g64(W)
    Wq_o, S_o = oracle.quantize_int4g64(_bits(W))
    assert np.array_equal(Wq_t.numpy(), Wq_o)
    assert np.array_equal(_bits(S_t), S_o)


def test_quantizer_edge_cases():
    # zero group -> scale 0 and nibble 8; amax 7 -> scale 1, q = rint(w) with
    # ties to even (2.5 -> 2, 3.5 -> 4, -0.5 -> -0); clamping at +-7.
    row = np.zeros((3, 64), dtype=np.float32)
    row[1, :8] = [7.0, 2.5, 3.5, -0.5, 1.5, -7.0, 0.25, -2.5]
    row[2, :2] = [1e-3, -1e-3]
    W = _bf16_from_float(row)
    Wq_o, S_o = oracle.quantize_int4g64(_bits(W))
    Wq_t, S_t = synth.quantize_int4_g64(W)
    assert np.array_equal(Wq_t.numpy(), Wq_o) and np.array_equal(_bits(S_t), S_o)
    q, sc = _unpack_int4(Wq_o, S_o)
    assert sc[0, 0] == 0.0 and (q[0] == 0).all()
    assert sc[1, 0] == 1.0
    assert list(q[1, :8]) == [7, 2, 4, 0, 2, -7, 0, -2]
    assert (q[2, :2] == [7, -7]).all()


def test_quantizer_round_trip_error_is_at_most_half_a_step():
    rng = np.random.default_rng(8)
    W = _bf16_from_float(0.02 * rng.standard_normal((64, 256)))
    Wq, S = oracle.quantize_int4g64(_bits(W))
    q, sc = _unpack_int4(Wq, S)
    w = W.double().numpy()
    err = np.abs(q * sc - w)
    # s = bf16(amax/7) may round below amax/7, so the top weight can clamp: the
    # bound is half a step plus the clamp overshoot amax - 7s.
    amax = np.repeat(np.abs(w).reshape(64, 4, 64).max(axis=2), 64, axis=1)
    bound = 0.5 * sc + np.maximum(0.0, amax - 7 * sc) + 1e-12
    assert (err <= bound).all()
