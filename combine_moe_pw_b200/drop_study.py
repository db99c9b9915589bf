"""Drop-rate study: sender and receiver drops across capacity factors and
sequence lengths, computed by the library's own kernels on the GPU.

"Marin 开始公开训练 535B 参数 MoE 模型", section 四: fewer independent sequences
per batch (longer context) balance the experts worse, the earlier expert-parallel
code dropped about 7% at 4K context and about 40% at 65K, pooled-wave about 3% at
4K, and higher capacity factors are one listed remedy.  Those figures come from a
trained router; this study runs the same rules on the synthetic router logits
(N(0,1) + a per-(sequence, expert) bias N(0, sigma_b^2)) so the trends can be
read off: drops against the factor, against the sequence length, and the split
between sender and receiver drops.

Drops do not depend on the latent width, so the study uses an 8-wide latent; the
routing, sender assignment, pack and receiver bucketing are the full kernels.

    python -m combine_moe_pw_b200.drop_study [--tokens 262144] \
        [--seq-lens 4096,8192,16384,65536] [--cf 100,110,125,150,200] [--sigma-b 0.5]

Each row also carries the sequence-level balance term of the batch
(moe_pw_seq_balance with alpha = 1: the mean over sequences of
sum_e f_e P_e, exactly 1 when every sequence spreads its assignments evenly),
the quantity the pages' third remedy, sequence-level balancing, would train
down.

Prints one JSON object per (seq_len, cf) and a summary table.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import moe_pw as mp
from . import synth


def sequence_balance(b: "mp.Buffers", seq_len: int) -> float:
    """Mean over the batch's sequences of sum_e f_e P_e (the balance term
    with alpha = 1) for the routing in b.idx."""
    cfg = b.cfg
    n_seq = cfg.T // seq_len
    dev = b.logits.device
    f = torch.empty((n_seq, cfg.E), dtype=torch.float32, device=dev)
    P = torch.empty_like(f)
    loss = torch.empty((n_seq,), dtype=torch.float32, device=dev)
    ws = torch.empty((max(mp.moe_pw_seq_balance_plan(cfg, seq_len), 256),), dtype=torch.uint8,
                     device=dev)
    mp.moe_pw_seq_balance(cfg, seq_len, 1.0, b.logits, b.idx, f, P, loss, ws)
    return float(loss.double().mean().item())


def study(tokens: int, seq_lens, cfs, sigma_b: float = 0.5, recv_cfs=None, seed: int = 0,
          device="cuda"):
    """Yield one dict per (seq_len, cf_send, cf_recv)."""
    base = synth.WORKLOADS["rack"].with_(T=tokens, D=8, sigma_b=sigma_b, seed=seed)
    recv_cfs = recv_cfs or [None]
    for L in seq_lens:
        w = base.with_(seq_len=L)
        logits = torch.from_numpy(synth.logits(w)).to(device)
        balance = None
        for cf in cfs:
            for rcf in recv_cfs:
                rc = round(cf * 115 / 110) if rcf is None else rcf
                ww = w.with_(cf_send_pct=cf, cf_recv_pct=rc)
                b = mp.Buffers(mp.Config.from_workload(ww), device=device)
                b.logits.copy_(logits)
                b.x.zero_()
                b.route()
                b.dispatch()
                st = b.stats()
                if balance is None:  # depends on the routing only, not on the factors
                    balance = sequence_balance(b, L)
                TK = ww.T * ww.k
                yield {"tokens": ww.T, "seq_len": L, "sequences": ww.T // L, "sigma_b": sigma_b,
                       "cf_send": cf / 100, "cf_recv": rc / 100,
                       "C_s": b.sizes.C_s, "C_r": b.sizes.C_r,
                       "sender_dropped": st.sender_dropped, "receiver_dropped": st.receiver_dropped,
                       "kept": st.kept, "assignments": TK,
                       "drop_sender": st.sender_dropped / TK, "drop_receiver": st.receiver_dropped / TK,
                       "drop_total": (st.sender_dropped + st.receiver_dropped) / TK,
                       "sequence_balance": balance}
                del b


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=262144)
    ap.add_argument("--seq-lens", default="4096,8192,16384,65536")
    ap.add_argument("--cf", default="100,110,125,150,200",
                    help="sender factors in percent; the receiver factor keeps the pages' ratio "
                         "1.15/1.10 unless --recv-cf is given")
    ap.add_argument("--recv-cf", default="")
    ap.add_argument("--sigma-b", type=float, default=0.5)
    a = ap.parse_args()
    rows = list(study(a.tokens, [int(v) for v in a.seq_lens.split(",")],
                      [int(v) for v in a.cf.split(",")], a.sigma_b,
                      [int(v) for v in a.recv_cf.split(",")] if a.recv_cf else None))
    for r in rows:
        print(json.dumps(r))
    print(f"{'seq_len':>8} {'cf_s':>5} {'cf_r':>5} {'sender':>8} {'receiver':>9} {'total':>7} "
          f"{'balance':>8}")
    for r in rows:
        print(f"{r['seq_len']:8d} {r['cf_send']:5.2f} {r['cf_recv']:5.2f} {100*r['drop_sender']:7.2f}% "
              f"{100*r['drop_receiver']:8.2f}% {100*r['drop_total']:6.2f}% "
              f"{r['sequence_balance']:8.4f}")


if __name__ == "__main__":
    main()
