"""Timing of the balanced clustering builder (write-up section 2.1) on one GPU.

Token rows: the seeded planted-cluster embedding matrix of a head shape (as
used by the benchmark). For the chosen shape it times, with CUDA events on
the launching stream:

- row normalisation (bytes: v*d*2 read + v*d*2 written);
- k-means++ seeding (c draws; each reads the v*d*2 normalised rows once),
  timed on a smaller balanced shape with the same d (``--seed-v``,
  ``--seed-c``; the full shape's 8016 draws over 525 MB would take minutes):
  bytes against HBM;
- the v x c similarity product on the tcgen05 GEMM (2*v*c*d flops; also
  reported as TFLOP/s against the measured bf16 GEMM peak, burst and
  sustained);
- one balanced assignment (proposal rounds, time);
- one centre update (reads every row once);
- a whole build of a few iterations from c distinct random tokens as the
  initial centres (the seeding is timed on its own above): time per
  iteration.

One JSON line per quantity.

    python -m lm_output_head_b200.microbench.cluster_build [--config 1] [--steps 3]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0.0)) or None, \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--repeats", type=int, default=3)
    ap.add_argument("--seed-v", type=int, default=32768)
    ap.add_argument("--seed-c", type=int, default=2048)
    args = ap.parse_args()

    import numpy as np
    import torch
    import synth
    import lm_output_head_b200 as fh
    from lm_output_head_b200.cluster import ClusterBuilder

    cfg, head, _, _ = synth.make_config(args.config, n_states=1)
    v, d, c = head.v, head.d, head.c
    hbm, tflops, tflops_sus, kind = peaks()
    E = fh.bf16_from_bits(head.E, "cuda")
    cb = ClusterBuilder(v, d, c)
    shape = f"v{v} d{d} c{c} b{v // c}"

    def timed(fn, repeats):
        best = None
        out = None
        for _ in range(repeats):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record()
            out = fn()
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        return best, out

    def emit(**kw):
        kw["shape"] = shape
        kw["peak_kind"] = kind
        print(json.dumps(kw), flush=True)

    ms, En = timed(lambda: cb.normalize(E), args.repeats)
    by = 2 * v * d * 2
    emit(step="normalize", ms=round(ms, 4), bytes=by, GBps=round(by / ms / 1e6, 1),
         frac_of_hbm=round(by / ms / 1e6 / hbm, 4))

    # seeding on a smaller balanced shape with the same d: its own builder and token rows
    sv, sc = args.seed_v, args.seed_c
    rng = np.random.default_rng(1)
    Es = torch.from_numpy(rng.standard_normal((sv, d), dtype=np.float32)).to(torch.bfloat16).cuda()
    cbs = ClusterBuilder(sv, d, sc)
    Ens = cbs.normalize(Es)
    us = torch.from_numpy(rng.uniform(size=sc).astype(np.float32)).cuda()
    ms, _ = timed(lambda: cbs.seed(Ens, us), 1)
    by = (sc - 1) * sv * d * 2
    emit(step="seed", seed_shape=f"v{sv} d{d} c{sc}", ms=round(ms, 3), draws=sc, bytes=by,
         GBps=round(by / ms / 1e6, 1), frac_of_hbm=round(by / ms / 1e6 / hbm, 4),
         us_per_draw=round(ms * 1e3 / sc, 2), status=cbs.device_status(),
         note="normalised rows of one draw: %.0f MB (L2 holds 126 MB)" % (sv * d * 2 / 1e6))
    cbs.close()
    del Es, Ens

    ids = torch.from_numpy(np.sort(rng.choice(v, size=c, replace=False)).astype(np.int32)).cuda()
    C = cb.gather(En, ids)
    ms, S = timed(lambda: cb.similarities(En, C), args.repeats)
    fl = 2.0 * v * c * d
    emit(step="similarities", ms=round(ms, 4), flops=fl, TFLOPs=round(fl / ms / 1e9, 1),
         frac_of_bf16=round(fl / ms / 1e9 / tflops, 4),
         frac_of_bf16_sustained=round(fl / ms / 1e9 / tflops_sus, 4) if tflops_sus else None,
         out_bytes=4 * v * c)

    t0 = time.perf_counter()
    ms, res = timed(lambda: cb.assign(S), 1)
    _, m, rounds = res
    emit(step="assign", ms=round(ms, 3), rounds=rounds, wall_s=round(time.perf_counter() - t0, 3),
         s_bytes_per_full_pass=4 * v * c, status=cb.device_status())

    ms, _ = timed(lambda: cb.update(En, m, C), args.repeats)
    by = v * d * 2 + c * d * 2
    emit(step="update", ms=round(ms, 4), bytes=by, GBps=round(by / ms / 1e6, 1))

    t0 = time.perf_counter()
    ms, (Cout, m2, it) = timed(lambda: cb.build(E, init_ids=ids, max_iter=args.steps), 1)
    emit(step="build", init="c distinct random tokens", ms=round(ms, 1), iterations=it, max_iter=args.steps,
         ms_per_iteration=round(ms / max(1, it), 1), wall_s=round(time.perf_counter() - t0, 2),
         status=cb.device_status())
    cb.close()


if __name__ == "__main__":
    main()
