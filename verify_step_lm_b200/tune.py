"""Draft-depth auto-tune: how many draft tokens K per cycle, or none.

The pages' automatic depth tuning (devtrends.cc MTPLX overview and the
devtrends.ru page, main-features list, first item: the model is run at
depths 1, 2 and 3 on the user's own hardware, the fastest depth is kept, and
drafting is switched off when plain autoregressive decoding is faster)
picks the depth that maximises tokens per second.  One speculative cycle with
depth K costs a draft phase (K draft positions), one forward pass of the
target model's body over K + 1 tokens and one verify step, and emits n + 1
tokens, n the number of accepted drafts; autoregressive decoding pays one
body pass and one LM-head step per token.  So

    throughput(K) = (E[n_K] + 1) / (t_draft(K) + t_body + t_verify(K)),
    throughput(0) = 1 / (t_body + t_ar),

and the tuner returns the K with the largest throughput (0: do not draft).
The body (the transformer layers) is outside this library; decode is a
weight stream, so a pass over a few tokens costs about what a pass over one
costs, t_body = the body's weight bytes / HBM bandwidth (by default a
27B-parameter model at 4 bits, 13.5 GB, over the measured copy bandwidth).

``measure`` times the library's own calls on the GPU (draft loop, verify
step, and one autoregressive step: the bf16 head for one row plus one draw)
over seeded synthetic steps, and counts accepted drafts from the verify
step's outputs.  ``python -m verify_step_lm_b200.tune`` prints the table as
one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics


def expected_tokens_constant(alpha: float, K: int) -> float:
    """E[n] + 1 when every draft is accepted with probability alpha, the
    drafts stopping at the first rejection: sum_{i=0..K} alpha^i."""
    if alpha == 1.0:
        return float(K + 1)
    return (1.0 - alpha ** (K + 1)) / (1.0 - alpha)


def throughput(tokens_per_cycle: float, cycle_ms: float) -> float:
    """Tokens per second of one configuration."""
    return 1e3 * tokens_per_cycle / cycle_ms


def choose_depth(table: dict) -> int:
    """The depth with the largest throughput.

    ``table[K] = {"tokens_per_cycle": ..., "cycle_ms": ...}`` for every
    measured depth, with ``table[0]`` the autoregressive baseline
    (one token per ``cycle_ms``).  Ties go to the smaller depth.
    """
    best, best_tps = None, -1.0
    for K in sorted(table):
        tps = throughput(table[K]["tokens_per_cycle"], table[K]["cycle_ms"])
        if tps > best_tps:
            best, best_tps = K, tps
    return best


def decide(res: dict, body_ms: float) -> dict:
    """The tuning table with the model body's time added to every cycle, and
    the chosen depth."""
    table = {K: {"tokens_per_cycle": r["tokens_per_cycle"], "cycle_ms": r["cycle_ms"] + body_ms}
             for K, r in res["depths"].items()}
    table[0] = {"tokens_per_cycle": 1.0, "cycle_ms": res["ar"]["cycle_ms"] + body_ms}
    return {"body_ms": body_ms, "choice": choose_depth(table),
            "tokens_per_s": {K: throughput(v["tokens_per_cycle"], v["cycle_ms"]) for K, v in table.items()}}


def measure(W, Wq, S, depths, T: float, top_p: float, sigma: float, steps: int = 32,
            warmup: int = 3, B: int = 1, seed0: int = 5000) -> dict:
    """GPU measurement of the tuning table for the given heads.

    W (bf16 [V, h]) is the target head, (Wq, S) its int4 g64 copy used by the
    draft head; hidden states, drafts and uniforms are seeded synthetic
    stand-ins (draft rows = target rows + N(0, sigma^2), which sets the
    acceptance rate).  Returns {"depths": {K: row}, "ar": row, "choice": K}.
    """
    import torch

    import verify_step_lm_b200 as mtpv
    from verify_step_lm_b200 import synth

    dev = W.device
    V, h = W.shape
    stream = torch.cuda.current_stream(dev)

    def timed(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n):
            evs[i][0].record(stream)
            fn(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    rows = {}
    for K in depths:
        pool = []
        for i in range(steps):
            Ht, Hd = synth.make_hidden(B, K, h, sigma, seed=seed0 + 97 * K + i, device=dev)
            u = synth.step_uniforms(seed0 + K, i, B, K)
            pool.append((Ht, Hd, {k: torch.as_tensor(v).contiguous().to(dev) for k, v in u.items()}))
        d = torch.empty((B, K), dtype=torch.int32, device=dev)
        tl = torch.empty((B, K + 1, V), dtype=torch.float32, device=dev)
        dl = torch.empty((B, K, V), dtype=torch.float32, device=dev)
        ot = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
        oa = torch.empty((B,), dtype=torch.int32, device=dev)
        dws = mtpv.workspace(mtpv.load().mtpv_draft_loop_workspace_bytes(B, K, V, h), dev)
        vws = mtpv.workspace(mtpv.verify_step_workspace_bytes(B, K, V, h), dev)
        accepted = []

        def draft(i):
            Ht, Hd, u = pool[i % steps]
            mtpv.draft_loop(Wq, S, Hd, u["u_draft"], B, K, T, top_p, d, None, ws=dws)

        def verify(i):
            Ht, Hd, u = pool[i % steps]
            mtpv.verify_step(W, Wq, S, Ht, Hd, d, u["u_accept"], u["u_sample"], B, K, T, top_p,
                             ot, oa, None, tl, dl, ws=vws)

        for i in range(warmup):
            draft(i)
            verify(i)
        t_draft = timed(draft, steps)
        t_verify = timed(verify, steps)
        for i in range(steps):  # acceptance, with each step's own drafts
            draft(i)
            verify(i)
            accepted.append(oa.clone())
        torch.cuda.synchronize()
        n = torch.stack(accepted).float()
        mean_n = float(n.mean())
        rows[K] = {"tokens_per_cycle": mean_n + 1.0, "cycle_ms": t_draft + t_verify,
                   "draft_ms": t_draft, "verify_ms": t_verify, "mean_accepted": mean_n,
                   "acceptance_rate": mean_n / K}
        rows[K]["tokens_per_s"] = throughput(rows[K]["tokens_per_cycle"], rows[K]["cycle_ms"])

    # autoregressive baseline: the bf16 head for one row, then one draw
    x = synth.make_hidden(1, 1, h, sigma, seed=seed0 - 1, device=dev)[0][:1]
    y = torch.empty((1, V), dtype=torch.float32, device=dev)
    uu = torch.full((1,), 0.5, dtype=torch.float32, device=dev)
    tok = torch.empty((1,), dtype=torch.int32, device=dev)
    sws = mtpv.workspace(mtpv.sample_workspace_bytes(1, V), dev)

    def ar(i):
        mtpv.lm_head_smallm(x, W, None, mtpv.W_BF16, y)
        mtpv.sample(y, T, top_p, uu, tok, ws=sws)

    for i in range(warmup):
        ar(i)
    t_ar = timed(ar, steps)
    table = dict(rows)
    table[0] = {"tokens_per_cycle": 1.0, "cycle_ms": t_ar}
    ar_row = {"tokens_per_cycle": 1.0, "cycle_ms": t_ar, "tokens_per_s": throughput(1.0, t_ar)}
    return {"depths": rows, "ar": ar_row, "choice": choose_depth(table)}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--vocab", type=int, default=151936)
    ap.add_argument("--hidden", type=int, default=5120)
    ap.add_argument("--wstd", type=float, default=0.02)
    ap.add_argument("--depths", default="1,2,3,4")
    ap.add_argument("--temperature", type=float, default=0.6)
    ap.add_argument("--top-p", type=float, default=0.95)
    ap.add_argument("--sigma", type=float, default=0.3)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--body-gb", type=float, default=13.5,
                    help="weight bytes of the target model's body, GB (27B parameters at 4 bits)")
    ap.add_argument("--hbm-gbs", type=float, default=None,
                    help="HBM bandwidth for the body's time (default: the measured copy peak)")
    args = ap.parse_args()
    hbm = args.hbm_gbs
    if hbm is None:
        try:
            root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
            with open(os.path.join(root, "MEASURED_PEAKS.json")) as f:
                hbm = float(json.load(f)["hbm_gbs"])
        except Exception:
            hbm = 6650.0

    from verify_step_lm_b200 import synth

    W = synth.make_head(args.vocab, args.hidden, args.wstd, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    res = measure(W, Wq, S, [int(k) for k in args.depths.split(",")], args.temperature, args.top_p,
                  args.sigma, steps=args.steps)
    res["with_body"] = decide(res, 1e3 * args.body_gb / hbm)
    res["config"] = {"vocab": args.vocab, "hidden": args.hidden, "temperature": args.temperature,
                     "top_p": args.top_p, "sigma": args.sigma, "steps": args.steps,
                     "body_gb": args.body_gb, "hbm_gbs": hbm, "data": "synthetic"}
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
