"""Reports how much of the proxy's Stage-2 selection the exact selection shares
on the seeded synthetic layers: |TopK(|s~|) ∩ TopK(|s|)| / k per token, s~ the
Stage-1 proxy state and s the exact intermediate state (oracle-s of Prox §3.1).
The paper quotes this overlap for trained weights; the synthetic layers have
none of their structure, so the figure is reported, not pinned.

TEST INFRASTRUCTURE: calls only the oracle and the seeded generators.

    python -m oracle.mask_overlap [config ...] [--tokens N] [--s1 P] [--s2 P]
"""

from __future__ import annotations

import argparse

import numpy as np

import synth
from oracle import prox_oracle as orc


def overlap(name: str, tokens: int, s1: float, s2: int):
    cfg = synth.get_config(name)
    lay = synth.make_layer(cfg, n_tokens=tokens)
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)
    tau = orc.calibrate_tau(lay.x_cal, s1)
    k = cfg.k(s2)
    out = []
    for x in lay.x_eval[:tokens]:
        _, g_t, u_t, _ = orc.proxy_intermediate(x, tau, qg, sg, qu, su)
        proxy = orc.topk_channels(orc.proxy_scores(g_t, u_t), k)
        exact = orc.oracle_s_mask(x, lay.w_gate, lay.w_up, k)
        out.append(np.intersect1d(proxy, exact).size / k)
    return k, np.asarray(out)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("configs", nargs="*", default=["tiny", "llama3_8b"])
    ap.add_argument("--tokens", type=int, default=8)
    ap.add_argument("--s1", type=float, default=50.0)
    ap.add_argument("--s2", type=int, default=70)
    args = ap.parse_args()
    for name in args.configs:
        k, ov = overlap(name, args.tokens, args.s1 / 100.0, args.s2)
        print(f"{name}: s1 {args.s1:g}%, s2 {args.s2}% (k {k}), {ov.size} tokens: "
              f"overlap mean {ov.mean():.4f} min {ov.min():.4f} max {ov.max():.4f}")


if __name__ == "__main__":
    main()
