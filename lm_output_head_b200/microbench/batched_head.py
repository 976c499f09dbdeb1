"""Timing of the batched path (B > 1), and of the fused kernel at B = 1 for
the INT4-centroid head.

For each requested head shape and batch: the whole batched decode (centroid
keys -- tcgen05 GEMM at B >= 64, CUDA cores below --, per-row top-p,
de-duplicated candidate logits, argmax or inverse-CDF draw), its algorithmic
bytes (centroid bytes once + every distinct chosen cluster's token rows and
C2T row once + hidden rows + uniforms + outputs) and achieved GB/s; at
B >= 64 also the tcgen05 centroid GEMM and the tcgen05 dense head (fused
argmax) with their TFLOP/s. CUDA events on the launching stream, median of the
timed repeats, each on a cold L2 (a buffer twice the L2 written and read back
before it, outside the events); one JSON line per case.

    python -m lm_output_head_b200.microbench.batched_head [--repeats N] [--cases 4:256,3:32,2:16,2:4,2:1]
    python -m lm_output_head_b200.microbench.batched_head --residency 4:256 [--repeats N]
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


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def run_case(cfg_id, B, repeats):
    import numpy as np
    import torch
    import synth
    import lm_output_head_b200 as fh
    cfg, head, hid, uni = synth.make_config(cfg_id, n_states=max(B, 64))
    dev = "cuda"
    E = fh.bf16_from_bits(head.E, dev)
    C2T = torch.from_numpy(head.C2T).to(dev)
    if head.C_q is not None:
        dh = fh.FlashHead(E, C2T, C_q=torch.from_numpy(head.C_q).to(dev),
                          C_scales=fh.bf16_from_bits(head.C_scales, dev), max_batch=B, max_probes=cfg.p)
        cbytes = head.C_q.nbytes + head.C_scales.nbytes
    else:
        dh = fh.FlashHead(E, C2T, C=fh.bf16_from_bits(head.C, dev), max_batch=B, max_probes=cfg.p)
        cbytes = head.C.nbytes
    H = fh.bf16_from_bits(hid.H[:B], dev)
    gumbel = cfg.mode == "gumbel"
    kw = {}
    ubytes = 0
    if gumbel:
        rng = np.random.default_rng(5)
        kw = dict(mode="gumbel", T=cfg.temperature,
                  u_clusters=torch.from_numpy(rng.random((B, cfg.c), dtype=np.float32)).to(dev),
                  u_token=torch.from_numpy(rng.random(B, dtype=np.float32)).to(dev))
        ubytes = B * cfg.c * 4 + B * 4

    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)

    def timeit(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(repeats):
            # cold L2: a buffer twice the L2 written and read back before the call, outside the events
            flush.fill_(1)
            flush.view(torch.int64).sum()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    tok = torch.empty(B, dtype=torch.int32, device=dev)
    t_x = timeit(lambda: dh.decode(H, cfg.p, out_tokens=tok, **kw))
    union = dh.query(1)
    abytes = cbytes + union * (cfg.b * cfg.d * 2 + cfg.b * 4) + B * cfg.d * 2 + ubytes + B * 4
    peak, kind = measured_hbm_peak()
    rec = {"workload": f"config {cfg_id}: v{cfg.v} d{cfg.d} c{cfg.c} b{cfg.b} p{cfg.p} "
                       f"{'INT4' if head.C_q is not None else 'bf16'} centroids, B={B}, {cfg.mode}",
           "decode_us": round(t_x, 2), "decode_tokens_per_s": round(B / t_x * 1e6, 1),
           "union_clusters": union, "union_of_possible": round(union / min(cfg.c, B * cfg.p), 4),
           "algorithmic_bytes": int(abytes), "achieved_GBps": round(abytes / t_x / 1e3, 1),
           "frac_of_hbm_peak": round(abytes / t_x / 1e3 / peak, 4), "peak_kind": kind,
           "protocol": "cold L2: 2 x L2 written and read back before every timed call, outside the events; "
                       "median of the timed calls"}
    if B >= 64:
        scores = torch.empty((B, cfg.c), dtype=torch.float32, device=dev)
        am = torch.empty(B, dtype=torch.int32, device=dev)
        t_c = timeit(lambda: dh.centroid_scores(H, out=scores))
        t_d = timeit(lambda: dh.dense_head(H, out_argmax=am))
        rec.update({"centroid_gemm_us": round(t_c, 2),
                    "centroid_gemm_tflops": round(2.0 * B * cfg.c * cfg.d / t_c / 1e6, 1),
                    "dense_gemm_us": round(t_d, 2),
                    "dense_gemm_tflops": round(2.0 * B * cfg.v * cfg.d / t_d / 1e6, 1)})
    rec["device_status"] = dh.device_status()
    dh.close()
    print(json.dumps(rec), flush=True)


def run_b1(cfg_id, steps, int8=False):
    """One hidden state per step through the fused kernel, steps issued back to
    back and rotated over enough head copies that every step reads its
    centroid and token rows from HBM (the protocol of bench.py). With int8,
    the head's centroids are quantised to INT8 group-32 codes."""
    import ctypes
    import torch
    import synth
    import lm_output_head_b200 as fh
    cfg, head, hid, _ = synth.make_config(cfg_id)
    dev = torch.device("cuda", 0)
    if int8:
        head.C_q, head.C_scales = synth.quantize_int8_g32(head.C)
    int4 = head.C_q is not None and not int8
    cbytes = head.C_q.nbytes + head.C_scales.nbytes if head.C_q is not None else head.C.nbytes
    abytes = cbytes + cfg.p * cfg.b * cfg.d * 2 + cfg.p * cfg.b * 4 + cfg.d * 2 + 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_copies = max(3, -(-4 * l2 // abytes) + 1)
    E0 = fh.bf16_from_bits(head.E, dev)
    T0 = torch.from_numpy(head.C2T).to(dev)
    heads = []
    for i in range(n_copies):
        E, T = (E0, T0) if i == 0 else (E0.clone(), T0.clone())
        if head.C_q is not None:
            heads.append(fh.FlashHead(E, T, C_q=torch.from_numpy(head.C_q).to(dev),
                                      C_scales=fh.bf16_from_bits(head.C_scales, dev), max_batch=1,
                                      max_probes=cfg.p))
        else:
            heads.append(fh.FlashHead(E, T, C=fh.bf16_from_bits(head.C, dev), max_batch=1, max_probes=cfg.p))
    Hd = fh.bf16_from_bits(hid.H, dev)
    out = torch.empty(1, dtype=torch.int32, device=dev)
    lib = heads[0]._lib
    sptr = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    optr = ctypes.c_void_p(out.data_ptr())
    hptrs = [ctypes.c_void_p(Hd[i].data_ptr()) for i in range(Hd.shape[0])]
    handles = [h._h for h in heads]

    def step(i):
        st = lib.fh_decode(handles[i % n_copies], hptrs[i % len(hptrs)], 1, cfg.p, 0, 1.0, None, None, optr,
                           None, None, sptr)
        if st != 0:
            raise RuntimeError(f"fh_decode returned {st}")
    for i in range(20):
        step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(20 + i)
    e1.record()
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / steps
    peak, kind = measured_hbm_peak()
    status = max(h.device_status() for h in heads)
    for h in heads:
        h.close()
    print(json.dumps({
        "workload": f"config {cfg_id}: v{cfg.v} d{cfg.d} c{cfg.c} b{cfg.b} p{cfg.p} "
                    f"{'INT8' if int8 else 'INT4' if int4 else 'bf16'} centroids, B=1 greedy, fused kernel",
        "us_per_token": round(us, 3), "tokens_per_s": round(1e6 / us, 1), "algorithmic_bytes": int(abytes),
        "achieved_GBps": round(abytes / us / 1e3, 1), "frac_of_hbm_peak": round(abytes / us / 1e3 / peak, 4),
        "peak_kind": kind, "head_copies": n_copies, "device_status": status}), flush=True)


def run_residency(cfg_id, B, repeats):
    """Hot-cluster residency on a batch whose planted clusters recur (write-up
    section 2.2.1). Three protocols, each call after a cold-L2 flush and a fixed
    device-side wait: (a) the decode alone; (b) the recurring clusters' token
    rows requested into L2 by fh_prefetch_clusters before the wait, so they have
    landed when the events start (an ideal resident cache: the most any
    residency scheme can save); (c) the same request issued inside the events
    just before the decode (no cache kept across steps)."""
    import numpy as np
    import torch
    import synth
    import lm_output_head_b200 as fh
    cfg, head, hid, _ = synth.make_config(cfg_id, n_states=max(B, 64))
    dev = "cuda"
    E = fh.bf16_from_bits(head.E, dev)
    C2T = torch.from_numpy(head.C2T).to(dev)
    if head.C_q is not None:
        dh = fh.FlashHead(E, C2T, C_q=torch.from_numpy(head.C_q).to(dev),
                          C_scales=fh.bf16_from_bits(head.C_scales, dev), max_batch=B, max_probes=cfg.p)
    else:
        dh = fh.FlashHead(E, C2T, C=fh.bf16_from_bits(head.C, dev), max_batch=B, max_probes=cfg.p)
    H = fh.bf16_from_bits(hid.H[:B], dev)
    planted = hid.planted[:B]
    hot_np = np.unique(planted[planted >= 0]).astype(np.int32)
    hot = torch.from_numpy(hot_np).to(dev)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)

    def once(pre, inside):
        # everything is queued before the GPU reaches it (no host sync inside), so no protocol
        # times a launch from the host; a fixed device-side wait after the flush lets a
        # request issued before the events land first
        flush.fill_(1)
        flush.view(torch.int64).sum()
        if pre:
            dh.prefetch_clusters(hot)
        torch.cuda._sleep(40000)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        if inside:
            dh.prefetch_clusters(hot)
        dh.decode(H, cfg.p, out_tokens=tok)
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e3

    for _ in range(3):
        once(False, False)
    res = {"cold": [], "hot_resident": [], "hot_requested_in_step": []}
    for _ in range(repeats):  # interleaved, so drift affects all three alike
        res["cold"].append(once(False, False))
        res["hot_resident"].append(once(True, False))
        res["hot_requested_in_step"].append(once(False, True))
    union = dh.query(1)
    med = {k: round(statistics.median(v), 2) for k, v in res.items()}
    hot_bytes = len(hot_np) * (cfg.b * cfg.d * 2 + cfg.b * 4)
    rec = {"workload": f"config {cfg_id}: v{cfg.v} d{cfg.d} c{cfg.c} b{cfg.b} p{cfg.p}, B={B}, "
                       f"{len(hot_np)} recurring planted clusters",
           "decode_us_median": med, "hot_clusters": len(hot_np), "hot_token_row_bytes": int(hot_bytes),
           "union_clusters": union,
           "union_token_row_bytes": int(union * (cfg.b * cfg.d * 2 + cfg.b * 4)),
           "saving_if_resident_us": round(med["cold"] - med["hot_resident"], 2),
           "saving_if_resident_frac": round((med["cold"] - med["hot_resident"]) / med["cold"], 4),
           "protocol": f"{repeats} interleaved repeats of each protocol, 2 x L2 written and read back before "
                       "every call, then a ~20 us device-side wait, all queued ahead of the GPU; medians", "device_status": dh.device_status()}
    dh.close()
    print(json.dumps(rec), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--repeats", type=int, default=20)
    ap.add_argument("--cases", default="4:256,3:32,2:16,2:4,2:1",
                    help="comma-separated config:batch pairs (batch 1: the fused kernel, back to back; "
                         "config 'NQ8' = config N with INT8 centroids, batch 1 only)")
    ap.add_argument("--b1-steps", type=int, default=1000)
    ap.add_argument("--residency", default=None, metavar="CONFIG:BATCH",
                    help="instead of the cases: the hot-cluster residency experiment on this config and batch")
    args = ap.parse_args()
    if args.residency:
        cs, bs = args.residency.split(":")
        run_residency(int(cs), int(bs), args.repeats)
        return
    for case in args.cases.split(","):
        cs, bs = case.split(":")
        int8 = cs.endswith("Q8")
        cfg_id, B = int(cs[:-2] if int8 else cs), int(bs)
        if B == 1:
            run_b1(cfg_id, args.b1_steps, int8=int8)
        else:
            run_case(cfg_id, B, args.repeats)


if __name__ == "__main__":
    main()
