"""Timing of the batched path on the Gemma-3-shaped head (v 262144, d 1152,
c 16384 balanced clusters of 16, p 1024, INT4 centroids, bf16 tokens, B 256
planted hidden states): the tcgen05 centroid GEMM, the tcgen05 dense head
(fused argmax), and the whole batched decode (GEMM keys, per-row top-p,
de-duplicated candidate logits, argmax). CUDA events on the launching
stream, median of the timed repeats; prints one JSON line.

    python -m lm_output_head_b200.microbench.batched_head [--repeats N]
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
    ap.add_argument("--repeats", type=int, default=20)
    ap.add_argument("--batch", type=int, default=256)
    args = ap.parse_args()
    import torch
    import synth
    import lm_output_head_b200 as fh
    cfg, head, hid, _ = synth.make_config(4, n_states=args.batch)
    dev = "cuda"
    E = fh.bf16_from_bits(head.E, dev)
    C2T = torch.from_numpy(head.C2T).to(dev)
    Cq = torch.from_numpy(head.C_q).to(dev)
    Cs = fh.bf16_from_bits(head.C_scales, dev)
    dh = fh.FlashHead(E, C2T, C_q=Cq, C_scales=Cs, max_batch=args.batch, max_probes=cfg.p)
    H = fh.bf16_from_bits(hid.H[:args.batch], dev)
    B = args.batch

    def timeit(fn):
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

    scores = torch.empty((B, cfg.c), dtype=torch.float32, device=dev)
    am = torch.empty(B, dtype=torch.int32, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)
    t_c = timeit(lambda: dh.centroid_scores(H, out=scores))
    t_d = timeit(lambda: dh.dense_head(H, out_argmax=am))
    t_x = timeit(lambda: dh.decode(H, cfg.p, out_tokens=tok))
    union = dh.query(1)
    status = dh.device_status()
    fl_c = 2.0 * B * cfg.c * cfg.d
    fl_d = 2.0 * B * cfg.v * cfg.d
    print(json.dumps({
        "workload": f"Gemma-3-shaped head v{cfg.v} d{cfg.d} c{cfg.c} b{cfg.b} p{cfg.p} INT4 centroids, B={B}",
        "centroid_gemm_us": round(t_c, 2), "centroid_gemm_tflops": round(fl_c / t_c / 1e6, 1),
        "dense_gemm_us": round(t_d, 2), "dense_gemm_tflops": round(fl_d / t_d / 1e6, 1),
        "decode_us": round(t_x, 2), "decode_tokens_per_s": round(B / t_x * 1e6, 1),
        "union_clusters": union, "union_of_possible": round(union / min(cfg.c, B * cfg.p), 4),
        "device_status": status}), flush=True)
    dh.close()


if __name__ == "__main__":
    main()
