"""Top-1 agreement of FlashHead with the dense head on the synthetic heads (oracle only).

The write-up reports the share of tokens where the two-stage head's greedy
token equals the dense head's argmax (section 1.2.2: 97 % on Llama-3.2).
This script measures the same quantity for the seeded synthetic heads with
the fp64 oracle -- a property of the method on these inputs, not of any
kernel -- separately for planted hidden states (6 mu_j + noise) and pure
noise states. It is reported, not gated.

    python -m oracle.report_quality [--states 64] [--configs 0,1,2]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def agreement(cfg_id: int, n_states: int):
    import numpy as np
    import oracle
    import synth
    cfg, head, hid, _ = synth.make_config(cfg_id)
    n = min(n_states, hid.H.shape[0])
    H = hid.H[:n]
    tok, _, _ = oracle.decode(head, H, cfg.p)
    _, am = oracle.dense_head(head.E, H)
    planted = hid.planted[:n] >= 0
    match = tok == am
    return {
        "config": cfg_id, "name": cfg.name, "p": cfg.p, "c": cfg.c, "states": int(n),
        "planted_states": int(planted.sum()),
        "top1_agreement_planted": round(float(match[planted].mean()), 4) if planted.any() else None,
        "top1_agreement_pure": round(float(match[~planted].mean()), 4) if (~planted).any() else None,
        "top1_agreement_all": round(float(match.mean()), 4),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--states", type=int, default=64)
    ap.add_argument("--configs", default="0,1,2")
    args = ap.parse_args()
    for c in args.configs.split(","):
        t0 = time.perf_counter()
        rec = agreement(int(c), args.states)
        rec["seconds"] = round(time.perf_counter() - t0, 1)
        print(json.dumps(rec), flush=True)


if __name__ == "__main__":
    main()
