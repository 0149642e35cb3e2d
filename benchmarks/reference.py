"""The reference arm: there is no installable reference implementation (the
page ships no code), so the reference is the CPU oracle, as it stands,
timed on the host cores on the same workload, metric and unit as the
GPU arm, each step a bounded sample of that workload.  Rank 0 alone runs."""
from __future__ import annotations

import statistics

from mla_latent_space_lca_b200.inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs

from .common import (METRIC, PREFILL_METRIC, ROW_BYTES, VARIANTS, cpu_baseline, decode_config, prefill_config,
                     prefill_cpu_baseline)

REF_BUDGET_S = 150.0   # whole reference-arm run (all K + W steps), seconds


def run_reference(args, workload, rank, world):
    if rank != 0:
        return None
    wl = WORKLOADS[workload]
    v = VARIANTS[args.variant]
    per_step = REF_BUDGET_S / max(1, args.steps + args.warmup)
    if wl["kind"] == "prefill":
        import oracle
        inp = make_prefill_inputs(wl["B"], wl["L"], seed=0)
        # blocks per step so that all K + W steps fit REF_BUDGET_S
        n0 = oracle.num_threads()
        _, _, _, t0 = prefill_cpu_baseline(inp, n0, steps=1, variant=v)
        n = max(1, min(2 * n0, int(n0 * per_step / max(t0[0], 1e-6))))
        tok_s, cores, sample, times = prefill_cpu_baseline(inp, n, steps=args.steps, warmup=args.warmup,
                                                           variant=v)
        metric = PREFILL_METRIC
        config = prefill_config(workload, wl["B"], wl["L"], world, args.variant, False, (0, wl["L"]))
    else:
        inp = make_decode_inputs(wl["B"], wl["L"], seed=0)
        # size each step's sample so that all K + W steps fit REF_BUDGET_S:
        # time one single-sequence call first
        _, _, _, t1 = cpu_baseline(inp, 0, steps=1, warmup=0, seqs=1, variant=v)
        seqs = max(1, min(wl["B"], int(per_step / max(t1[0], 1e-6))))
        tok_s, cores, sample, times = cpu_baseline(inp, 0, steps=args.steps, warmup=args.warmup, seqs=seqs,
                                                   variant=v)
        metric = METRIC
        config = decode_config(workload, wl["B"], wl["L"], world, args.variant,
                               wl["B"] * wl["L"] * ROW_BYTES < (256 << 20))
    ms = 1e3 * statistics.mean(times)
    return {
        "impl": "reference", "metric": metric, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config,
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
