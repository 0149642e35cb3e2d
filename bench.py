#!/usr/bin/env python
"""LCA decode benchmark: tokens/s and cache-read GB/s against the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W]       # the default suite
    python bench.py --workload NAME ...                         # one workload
    python bench.py --impl reference ...                        # the CPU oracle, timed on host cores

The default run times the fused LCA decode step on 8 sequences of 131072
cached tokens (the headline line, with plain MLA decode (g = 1) over the same
inputs as an in-run comparison, the unfused condense-then-attend path, and
the end-to-end decode loop), then, at N = 1, the other workloads under
"configs": decode from kept representatives on the same 8 x 131072 shape
(the page's 90% KV-cache reading), 32 x 32768 and 1 x 1048576 decode and
the 131072-token blockwise prefill, each with its own timing, roofline and
clocks (and CPU baseline where the oracle has that mode).

One decode step = one whole fused LCA decode step (summary query,
importance, group softmax pooling, anchor pick, split-L attention over
[representatives || window], log-sum-exp combine, W_UV up-projection) for
every sequence of the batch, through the C ABI.  Inputs are synthetic and
seeded (see mla_latent_space_lca_b200/inputs.py) and resident in HBM.
Multi-GPU (torchrun): each rank decodes its own batch (weak scaling, no
data-path collective); timing is the max over ranks.  Rank 0 prints one JSON
line.  The measurement code lives in benchmarks/ (decode, prefill, the other
decode modes and the reference arm)."""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from benchmarks.common import VARIANTS  # noqa: E402
from mla_latent_space_lca_b200.inputs import WORKLOADS  # noqa: E402

HEADLINE = "decode_b8_l128k"
SUITE = ("decode_b32_l32k", "decode_b1_l1m", "prefill_b1_l128k")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="default 2000 (decode), 10 (prefill)")
    ap.add_argument("--warmup", type=int, default=None, help="default 20 (decode), 3 (prefill)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None,
                    help=f"one workload only (default: the suite, headline {HEADLINE})")
    ap.add_argument("--no-suite", action="store_true", help="default run: the headline workload only")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="end-to-end steps (default: as many as the timed steps, so that both figures are "
                         "taken in the same power state)")
    ap.add_argument("--e2e-full-copy", type=int, default=2,
                    help="decode: also time N steps that copy the whole cache in from the host")
    ap.add_argument("--no-e2e-graph", action="store_true",
                    help="decode: skip the end-to-end loop replayed from CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stored", action="store_true",
                    help="decode: stored-representative mode (groups condensed once and kept)")
    ap.add_argument("--unfused-compare", type=int, default=100,
                    help="decode: also time N steps of the unfused path (condense, then attend stored reps)")
    ap.add_argument("--varlen", action="store_true",
                    help="decode: a ragged batch, lengths drawn uniformly from [L/8, 15L/8] (mean L)")
    ap.add_argument("--split-l", action="store_true",
                    help="decode: every sequence's cache split along L over the ranks (strong scaling)")
    ap.add_argument("--split-blocks", action="store_true",
                    help="prefill: one prompt's query blocks split over the ranks by work (strong scaling)")
    ap.add_argument("--variant", choices=list(VARIANTS), default="lca",
                    help="the method, or one of the page's two ablations: decode runs lca_condense "
                         "+ lca_decode_attn (the fused kernel has only the method), prefill passes it on")
    ap.add_argument("--mla-compare", type=int, default=None,
                    help="decode: also time N plain MLA decode steps (g = 1, every row attended) on the "
                         "same inputs (default: the headline's step count on the headline workload, else "
                         "0); prefill: N full "
                         "causal MLA prefills (w = L)")
    return ap.parse_args(argv)


def defaults(args, workload):
    prefill = WORKLOADS[workload]["kind"] == "prefill"
    steps = args.steps if args.steps is not None else (10 if prefill else 2000)
    warmup = args.warmup if args.warmup is not None else (3 if prefill else 20)
    return steps, warmup


def suite_entry(line):
    """The keys a nested workload keeps (its own timing, roofline, CPU
    baseline and clocks)."""
    keep = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "ms_per_step_at_max_clock", "config",
            "cache_gbps", "cache_frac_of_hbm", "read_gbps", "kv_rows_read_fraction", "step_tflops", "roofline",
            "kernels_ms_per_step", "gpu_launches", "clocks", "cpu_baseline", "e2e")
    return {k: line[k] for k in keep if k in line}


def run_ours(args, rank, world, local_rank):
    from benchmarks.decode import run_decode
    from benchmarks.modes import run_split, run_stored, run_varlen
    from benchmarks.prefill import run_prefill

    torch.cuda.set_device(local_rank)
    single = args.workload is not None
    workload = args.workload or HEADLINE
    steps, warmup = defaults(args, workload)
    if args.e2e_steps is None:
        args.e2e_steps = steps
    kind = WORKLOADS[workload]["kind"]
    if args.stored or args.varlen or args.split_l:
        args.workload, args.steps, args.warmup = workload, steps, warmup
        fn = run_stored if args.stored else run_split if args.split_l else run_varlen
        return fn(args, rank, world, local_rank)
    with_cpu = not args.no_cpu_baseline
    if kind == "prefill":
        return run_prefill(args, workload, rank, world, local_rank, steps, warmup, split=args.split_blocks,
                           mla_compare=args.mla_compare or 0, with_cpu=with_cpu)
    # the in-run MLA comparison runs as many steps as the headline, right
    # after it, with its own clock record (the step is power-capped when long)
    mla = args.mla_compare if args.mla_compare is not None else (0 if single else steps)
    line = run_decode(args, workload, rank, world, local_rank, steps, warmup, mla_compare=mla,
                      unfused_compare=args.unfused_compare, e2e_graph=not args.no_e2e_graph,
                      e2e_full_copy=args.e2e_full_copy, cpu_seconds=args.cpu_seconds, with_cpu=with_cpu)
    if single or args.no_suite or args.variant != "lca" or world > 1:
        return line
    # the other workloads, each measured on its own (N = 1 only)
    nested = {}
    # decode from kept representatives on the headline's shape: the page's
    # 90% KV-cache reading (each step reads 7% of the rows)
    st_args = argparse.Namespace(**vars(args))
    st_args.workload, st_args.steps, st_args.warmup = HEADLINE, min(steps, 500), max(3, min(warmup, 20))
    st_args.e2e_steps = st_args.steps
    sub = run_stored(st_args, rank, world, local_rank)
    if sub is not None:
        nested[HEADLINE + "_stored"] = suite_entry(sub)
    for wl in SUITE:
        s, w = defaults(args, wl)
        if WORKLOADS[wl]["kind"] == "prefill":
            sub = run_prefill(args, wl, rank, world, local_rank, min(s, 10), min(w, 3), e2e=False,
                              with_cpu=with_cpu)
        else:
            sub = run_decode(args, wl, rank, world, local_rank, min(s, 500), max(3, min(w, 20)), e2e=False,
                             cpu_seconds=args.cpu_seconds / 2, with_cpu=with_cpu)
        if sub is not None:
            nested[wl] = suite_entry(sub)
    if line is not None:
        line["configs"] = nested
    return line


def main(argv=None):
    args = parse(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.variant != "lca" and (args.stored or args.varlen or args.split_l):
        raise SystemExit("--variant applies to the plain decode and prefill workloads only")
    if args.impl == "reference":
        from benchmarks.reference import run_reference
        workload = args.workload or HEADLINE
        args.steps, args.warmup = defaults(args, workload)
        line = run_reference(args, workload, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
