"""The whole verify step through mtpv_verify_step / mtpv_verify_step_host.

The LM-head part is compared with the fp64 oracle (<= 1e-3 relative); the
sampler part is the same kernel as mtpv_verify, so the step must equal
mtpv_verify run on the step's own logits.  Token agreement with the oracle
run end to end on its own fp64 logits is reported (fp32 versus fp64
accumulation moves rare draws; it is not a parity gate).
"""
import numpy as np
import pytest
import torch

import oracle
import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import synth
from _util import assert_logits_close, cuda, f32

pytestmark = pytest.mark.gpu

T, TOP_P = 0.6, 0.95


def make_inputs(B, K, V, h, seed, wstd, sigma=0.3, device="cpu"):
    W = synth.make_head(V, h, wstd, seed=12345, device=device)
    Wq, S = synth.quantize_int4_g64(W)
    Ht, Hd = synth.make_hidden(B, K, h, sigma, seed=seed, device=device)
    u = synth.step_uniforms(seed, 0, B, K)
    return W, Wq, S, Ht, Hd, u


def draft_tokens_from_oracle(Hd, Wq, S, B, K, u):
    dl = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq.cpu().numpy(), synth.bf16_bits(S.cpu()),
                                threads=8)
    d, _, _ = oracle.sample_rows(dl, f32(T), f32(TOP_P), u["u_draft"].reshape(-1), threads=8)
    return d.reshape(B, K), dl


def run_step(W, Wq, S, Ht, Hd, d, u, B, K):
    V, h = W.shape
    tl = torch.empty((B, K + 1, V), dtype=torch.float32, device="cuda")
    dl = torch.empty((B, K, V), dtype=torch.float32, device="cuda")
    ot = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    oa = torch.empty((B,), dtype=torch.int32, device="cuda")
    rs = torch.empty((B,), dtype=torch.int32, device="cuda")
    mtpv.verify_step(cuda(W), cuda(Wq), cuda(S), cuda(Ht), cuda(Hd), cuda(torch.as_tensor(d)),
                     cuda(torch.as_tensor(u["u_accept"])), cuda(torch.as_tensor(u["u_sample"])),
                     B, K, T, TOP_P, ot, oa, rs, tl, dl)
    torch.cuda.synchronize()
    return tl, dl, ot, oa, rs


@pytest.mark.parametrize("B", [1, 4])
def test_tiny_step_against_oracle_and_components(B):
    K, V, h = 3, 4096, 512
    agree = total = 0
    for seed in range(10):
        W, Wq, S, Ht, Hd, u = make_inputs(B, K, V, h, seed, 0.05)
        d, dl_ref = draft_tokens_from_oracle(Hd, Wq, S, B, K, u)
        tl, dl, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, B, K)
        tl_ref = oracle.lm_head_bf16(synth.bf16_bits(Ht), synth.bf16_bits(W), threads=8)
        assert_logits_close(tl.reshape(B * (K + 1), V).cpu().numpy(), tl_ref)
        assert_logits_close(dl.reshape(B * K, V).cpu().numpy(), dl_ref)
        # the step's sampler equals mtpv_verify on the step's own logits
        ot2 = torch.empty_like(ot)
        oa2 = torch.empty_like(oa)
        mtpv.verify(tl, dl, cuda(torch.as_tensor(d)), cuda(torch.as_tensor(u["u_accept"])),
                    cuda(torch.as_tensor(u["u_sample"])), T, TOP_P, ot2, oa2)
        torch.cuda.synchronize()
        assert torch.equal(ot, ot2) and torch.equal(oa, oa2)
        assert (rs.cpu() == 0).all()
        # end to end against the oracle on its own fp64 logits (reported)
        ref = oracle.verify(tl_ref.reshape(B, K + 1, V), dl_ref.reshape(B, K, V), d, u["u_accept"],
                            u["u_sample"], f32(T), f32(TOP_P))
        agree += int((ot.cpu().numpy() == ref["tokens"]).all(axis=1).sum())
        total += B
    print(f"end-to-end token agreement with the fp64 oracle: {agree}/{total}")
    assert agree >= 0.8 * total


# Outputs of mtpv_verify_step_host: all page-locked (the sampler writes them
# in host memory itself), all pageable (written to the workspace and copied
# back), one of each kind (copied back), no row_status.  B (K + 1) = 64 fills
# the by-value block of per-position inputs.
@pytest.mark.parametrize("B,K,outputs", [(2, 3, "pinned"), (2, 3, "pageable"), (2, 3, "mixed"),
                                         (2, 3, "no_status"), (16, 3, "pinned"), (8, 7, "pageable")])
def test_host_io_step_equals_device_step(B, K, outputs):
    V, h = 4096, 512
    W, Wq, S, Ht, Hd, u = make_inputs(B, K, V, h, 5, 0.05)
    d, _ = draft_tokens_from_oracle(Hd, Wq, S, B, K, u)
    _, _, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, B, K)
    pin = lambda t: torch.as_tensor(t).contiguous().pin_memory()
    mk = lambda shape, pinned: (torch.full(shape, -9, dtype=torch.int32).pin_memory() if pinned
                                else torch.full(shape, -9, dtype=torch.int32))
    ot_h = mk((B, K + 1), outputs in ("pinned", "mixed", "no_status"))
    oa_h = mk((B,), outputs in ("pinned", "no_status"))
    rs_h = None if outputs == "no_status" else mk((B,), outputs == "pinned")
    # drafts and uniforms may sit in pageable memory: the host reads them
    d_h = torch.from_numpy(np.ascontiguousarray(d, np.int32))
    ua_h = torch.as_tensor(u["u_accept"]).contiguous()
    mtpv.verify_step_host(cuda(W), cuda(Wq), cuda(S), pin(Ht), pin(Hd), d_h, ua_h, pin(u["u_sample"]), B, K,
                          T, TOP_P, ot_h, oa_h, rs_h)
    assert torch.equal(ot_h, ot.cpu()) and torch.equal(oa_h, oa.cpu())
    if rs_h is not None:
        assert torch.equal(rs_h, rs.cpu())


def test_qwen_class_step_full_size():
    """hidden 5120, vocab 151936, K = 3: the benchmark's step; logits against
    the oracle (all draft rows; every 53rd vocabulary row and the ragged tail
    of the target rows), tokens against the oracle run on the step's own logits."""
    B, K, V, h = 1, 3, 151936, 5120
    W, Wq, S, Ht, Hd, u = make_inputs(B, K, V, h, 11, 0.02, device="cuda")
    # drafts: the oracle's draft distribution needs the draft logits; compute
    # them on the host for the three draft rows
    dl_ref = oracle.lm_head_int4g64(synth.bf16_bits(Hd.cpu()), Wq.cpu().numpy(),
                                    synth.bf16_bits(S.cpu()), threads=8)
    d, _, _ = oracle.sample_rows(dl_ref, f32(T), f32(TOP_P), u["u_draft"].reshape(-1), threads=4)
    d = d.reshape(B, K)
    tl, dl, ot, oa, rs = run_step(W, Wq, S, Ht, Hd, d, u, B, K)
    assert_logits_close(dl.reshape(B * K, V).cpu().numpy(), dl_ref)
    rows = torch.as_tensor(np.unique(np.concatenate([np.arange(0, V, 53), np.arange(V - 40, V)]))).cuda()
    tl_ref = oracle.lm_head_bf16(synth.bf16_bits(Ht.cpu()), synth.bf16_bits(W[rows].cpu()), threads=8)
    assert_logits_close(tl.reshape(B * (K + 1), V)[:, rows].cpu().numpy(), tl_ref)
    n = int(oa.item())
    assert 0 <= n <= K and int(rs.item()) == 0
    toks = ot.cpu().numpy()[0]
    assert list(toks[:n]) == list(d[0, :n]) and toks[n] >= 0 and (toks[n + 1:] == -1).all()
    # the step's tokens against the oracle run on the step's own logits
    ref = oracle.verify(tl.cpu().numpy(), dl.cpu().numpy(), d, u["u_accept"], u["u_sample"], f32(T),
                        f32(TOP_P))
    assert ref["flags"][0] != 0 or (np.array_equal(toks, ref["tokens"][0]) and n == ref["accepted"][0])
    assert ref["status"][0] == 0
