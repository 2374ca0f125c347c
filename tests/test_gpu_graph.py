"""The verify step captured in CUDA graphs and replayed.

The pages cache the compiled verify graph and replay it every step
(hazakura.dev MTPLX notes, "4-layer architecture", Layer 0: GraphBank).  The
library's analogue is a stream capture of mtpv_verify_step (a memset of the
heads' work counter, the two-head kernel and the two sampler kernels, the
sampler kernels as programmatic dependents) or of mtpv_verify.  A replayed
graph must give exactly what the uncaptured call gives on the same inputs:
tokens, accept counts, row status and both logit buffers, bit for bit; and
on the trials the oracle does not flag, the oracle's tokens when it runs on
those logits.  The graphs are replayed in rotation, so every replay follows
one that wrote other values into the same buffers.
"""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import f32

pytestmark = pytest.mark.gpu

T, TOP_P = 0.6, 0.95
ORDER = [0, 1, 2, 3, 2, 0, 3, 1, 1, 0]


def pool(B, K, V, h, wstd, n, seed0):
    W = synth.make_head(V, h, wstd, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    steps = []
    dl0 = torch.empty((B * K, V), dtype=torch.float32, device="cuda")
    for j in range(n):
        Ht, Hd = synth.make_hidden(B, K, h, 0.3, seed=seed0 + j, device="cuda")
        u = synth.step_uniforms(seed0 + j, 0, B, K)
        mtpv.lm_head_smallm(Hd, Wq, S, mtpv.W_INT4_G64, dl0)
        d = torch.empty((B * K,), dtype=torch.int32, device="cuda")
        mtpv.sample(dl0, T, TOP_P, torch.as_tensor(u["u_draft"].reshape(-1)).cuda(), d)
        steps.append(dict(Ht=Ht, Hd=Hd, d=d.view(B, K), ua=torch.as_tensor(u["u_accept"]).cuda(),
                          us=torch.as_tensor(u["u_sample"]).cuda(), u=u))
    torch.cuda.synchronize()
    return W, Wq, S, steps


class Outs:
    def __init__(self, B, K, V):
        self.tl = torch.empty((B, K + 1, V), dtype=torch.float32, device="cuda")
        self.dl = torch.empty((B, K, V), dtype=torch.float32, device="cuda")
        self.ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
        self.oa = torch.empty((B,), dtype=torch.int32, device="cuda")
        self.rs = torch.empty((B,), dtype=torch.int32, device="cuda")

    def snapshot(self):
        return [x.clone() for x in (self.tl, self.dl, self.ot, self.oa, self.rs)]


def check_graph_replay_of_step(B, K, V, h, wstd, seed0):
    W, Wq, S, steps = pool(B, K, V, h, wstd, 4, seed0)
    o = Outs(B, K, V)
    ws = mtpv.workspace(mtpv.verify_step_workspace_bytes(B, K, V, h))

    def step(j):
        s = steps[j]
        mtpv.verify_step(W, Wq, S, s["Ht"], s["Hd"], s["d"], s["ua"], s["us"], B, K, T, TOP_P,
                         o.ot, o.oa, o.rs, o.tl, o.dl, ws)

    eager = []
    for j in range(len(steps)):   # uncaptured calls (also the launch set-up before capture)
        step(j)
        torch.cuda.synchronize()
        eager.append(o.snapshot())
    graphs = []
    for j in range(len(steps)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(j)
        graphs.append(g)
    torch.cuda.synchronize()
    for j in ORDER:
        graphs[j].replay()
        torch.cuda.synchronize()
        for got, want in zip(o.snapshot(), eager[j]):
            assert torch.equal(got, want), f"replay of step {j} differs from the uncaptured call"
    # the uncaptured results against the oracle on their own logits
    for j, (tl, dl, ot, oa, rs) in enumerate(eager):
        s = steps[j]
        ref = oracle.verify(tl.cpu().numpy(), dl.cpu().numpy(), s["d"].cpu().numpy(), s["u"]["u_accept"],
                            s["u"]["u_sample"], f32(T), f32(TOP_P), threads=8)
        same = (ot.cpu().numpy() == ref["tokens"]).all(axis=1) & (oa.cpu().numpy() == ref["accepted"])
        assert (same | (ref["flags"] != 0)).all()
        assert np.array_equal(rs.cpu().numpy(), ref["status"])
    del graphs


def test_graph_replay_qwen_class_step():
    check_graph_replay_of_step(1, 3, 151936, 5120, 0.02, 500)


def test_graph_replay_small_step_two_sequences():
    check_graph_replay_of_step(2, 3, 4096, 512, 0.05, 600)


def test_graph_replay_of_verify_alone():
    B, K, V = 8, 3, 151936
    cases = []
    for j in range(4):
        tl, dl = synth.make_verify_logits(B, K, V, 1.43, 0.43, seed=700 + j, device="cuda")
        u = synth.step_uniforms(700 + j, 0, B, K)
        d = torch.empty((B * K,), dtype=torch.int32, device="cuda")
        mtpv.sample(dl.view(B * K, V), T, TOP_P, torch.as_tensor(u["u_draft"].reshape(-1)).cuda(), d)
        cases.append((tl, dl, d.view(B, K), torch.as_tensor(u["u_accept"]).cuda(),
                      torch.as_tensor(u["u_sample"]).cuda()))
    ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    oa = torch.empty((B,), dtype=torch.int32, device="cuda")
    rs = torch.empty((B,), dtype=torch.int32, device="cuda")
    ws = mtpv.workspace(mtpv.verify_workspace_bytes(B, K, V))
    eager = []
    for c in cases:
        mtpv.verify(*c, T, TOP_P, ot, oa, rs, ws=ws)
        torch.cuda.synchronize()
        eager.append((ot.clone(), oa.clone(), rs.clone()))
    graphs = []
    for c in cases:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            mtpv.verify(*c, T, TOP_P, ot, oa, rs, ws=ws)
        graphs.append(g)
    for j in ORDER:
        graphs[j].replay()
        torch.cuda.synchronize()
        assert torch.equal(ot, eager[j][0]) and torch.equal(oa, eager[j][1]) and torch.equal(rs, eager[j][2])
    del graphs
