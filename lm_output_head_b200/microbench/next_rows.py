"""Timing of the entry points beyond the single-token path, one JSON line each.

- fh_adaptive_probes (write-up section 1.2.2): probes per row from a row of
  centroid scores, Llama-3.2-1B-shaped head (c = 8016), B = 1 and 64; the
  scores were just written by fh_centroid_scores (L2-warm, as in a decode).
- fh_speculative_verify (write-up section 4.2): FlashHead drafts checked
  against the dense logits (v = 128256) at B = 1 and 8; logits just written by
  fh_dense_head (L2-warm); bytes = logits + candidate ids read.
- The compact uint16 C2T (write-up section 2.2.1) against int32 on the tiny
  head (v = 4096), single-token decode back to back: same kernel, half the
  C2T bytes.

CUDA events on the launching stream, median over the repeats (each repeat
one call, after 3 warm-up calls).

    python -m lm_output_head_b200.microbench.next_rows [--repeats N]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--repeats", type=int, default=50)
    args = ap.parse_args()
    import numpy as np
    import torch
    import synth
    import lm_output_head_b200 as fh

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.repeats):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    dev = "cuda"
    cfg, head, hid, _ = synth.make_config(1, n_states=64)
    dh = fh.FlashHead(fh.bf16_from_bits(head.E, dev), torch.from_numpy(head.C2T).to(dev),
                      C=fh.bf16_from_bits(head.C, dev), max_batch=64, max_probes=cfg.p)
    shape = f"v{cfg.v} d{cfg.d} c{cfg.c} b{cfg.b}"
    for B in (1, 64):
        H = fh.bf16_from_bits(hid.H[:B], dev)
        S = dh.centroid_scores(H)
        us = timed(lambda: dh.adaptive_probes(S, 0.9, 64, 2048))
        ps = dh.adaptive_probes(S, 0.9, 64, 2048).cpu().numpy()
        print(json.dumps({"entry": "fh_adaptive_probes", "shape": shape, "B": B, "tau": 0.9, "p_range": [64, 2048],
                          "us": round(us, 2), "rows_per_s": round(B / us * 1e6, 1),
                          "p_chosen_median": float(np.median(ps)), "scores_bytes": B * cfg.c * 4,
                          "device_status": dh.device_status()}), flush=True)
    for B in (1, 8):
        H = fh.bf16_from_bits(hid.H[:B], dev)
        ids = torch.empty((B, cfg.p), dtype=torch.int32, device=dev)
        dh.decode(H, cfg.p, out_cluster_ids=ids)
        toks, logits_c = dh.candidate_logits(H, ids)
        draft = toks.gather(1, logits_c.argmax(1, keepdim=True)).squeeze(1).contiguous()
        _, z = dh.dense_head(H, want_logits=True)
        rng = np.random.default_rng(3)
        ua = torch.from_numpy(rng.random(B, dtype=np.float32)).to(dev)
        ur = torch.from_numpy(rng.random(B, dtype=np.float32)).to(dev)
        n = toks.shape[1]
        us = timed(lambda: fh.speculative_verify(dh, z, toks, draft, 1.0, ua, ur))
        by = B * cfg.v * 4 + B * n * 4
        print(json.dumps({"entry": "fh_speculative_verify", "shape": shape, "B": B, "candidates": n,
                          "us": round(us, 2), "rows_per_s": round(B / us * 1e6, 1), "bytes": by,
                          "GBps": round(by / us / 1e3, 1), "device_status": dh.device_status()}), flush=True)
    dh.close()

    cfg0, head0, hid0, _ = synth.make_config(0, n_states=64)
    E0 = fh.bf16_from_bits(head0.E, dev)
    C0 = fh.bf16_from_bits(head0.C, dev)
    H0 = fh.bf16_from_bits(hid0.H, dev)
    res = {}
    for name, T in (("int32", torch.from_numpy(head0.C2T).to(dev)),
                    ("uint16", torch.from_numpy(head0.C2T.astype(np.uint16).view(np.int16)).to(dev))):
        h = fh.FlashHead(E0, T, C=C0, max_batch=1, max_probes=cfg0.p)
        out = torch.empty(1, dtype=torch.int32, device=dev)

        def loop():
            for i in range(200):
                h.decode(H0[i % 64:i % 64 + 1], cfg0.p, out_tokens=out)
        res[name] = round(timed(loop) / 200, 3)
        res[name + "_status"] = h.device_status()
        h.close()
    print(json.dumps({"entry": "fh_decode B=1, C2T int32 vs uint16",
                      "shape": f"v{cfg0.v} d{cfg0.d} c{cfg0.c} b{cfg0.b} p{cfg0.p} (L2-resident head)",
                      "us_per_token": res, "c2t_bytes": {"int32": cfg0.v * 4, "uint16": cfg0.v * 2}}), flush=True)


if __name__ == "__main__":
    main()
