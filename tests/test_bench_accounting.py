"""The algorithmic bytes behind bench.py's roofline figures, recomputed here
from the tensor shapes (bf16 head [V, h], int4 g64 head: nibbles [V, h/2]
and bf16 scales [V, h/64], bf16 hidden rows, fp32 logits written by the
heads and read once by the sampler).  The literals are the figures the
profiles and the design notes quote."""
import bench


def expected(B, K, V, h):
    Mt, Md = B * (K + 1), B * K
    w = V * h * 2
    wq = V * (h // 2)
    s = V * (h // 64) * 2
    xt, xd = Mt * h * 2, Md * h * 2
    yt, yd = Mt * V * 4, Md * V * 4
    return {"bf16_launch": w + xt + yt, "int4_launch": wq + s + xd + yd,
            "total": w + wq + s + xt + xd + 2 * (yt + yd)}


def test_single_sequence_step_bytes():
    c = bench.CONFIGS["qwen27b"]
    got = bench.step_bytes(c)
    exp = expected(c["B"], c["K"], c["V"], c["h"])
    for k, v in exp.items():
        assert got[k] == v, k
    # both heads in one launch (the roofline's dominant kernel), and the step
    assert got["bf16_launch"] + got["int4_launch"] == 1_973_416_448
    assert got["total"] == 1_977_670_656


def test_eight_sequence_step_bytes():
    c = bench.CONFIGS["b8_v248k"]
    assert (c["B"], c["K"], c["V"], c["h"]) == (8, 3, 248320, 5120)
    got = bench.step_bytes(c)
    exp = expected(8, 3, 248320, 5120)
    for k, v in exp.items():
        assert got[k] == v, k
    assert got["bf16_launch"] == 2_574_909_440
    assert got["int4_launch"] == 699_514_880
    assert got["total"] == 3_330_048_000
