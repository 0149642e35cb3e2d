"""Blockwise LCA prefill (lca_prefill_block) of B prompts of L tokens.

Replicas by default (each rank its own prompts); with split=True every rank
holds the same prompt and computes its work-balanced range of query blocks
(strong scaling, no data-path collective).  The roofline is the attention
kernel's algorithmic flops against the sustained bf16 tensor peak."""
from __future__ import annotations

import gc
import time

import torch

from mla_latent_space_lca_b200.inputs import WORKLOADS, make_prefill_inputs

from .common import (PREFILL_METRIC, VARIANTS, ClockSampler, barrier, device_ok, kernel_profile, max_over_ranks,
                     measured_tensor_peak, ncu_traffic, prefill_config, prefill_cpu_baseline, prefill_flops,
                     replica_seed, time_steps)


def run_prefill(args, workload, rank, world, local_rank, steps, warmup, *, split=False, mla_compare=0,
                e2e=True, with_cpu=True):
    """Time `steps` whole prefills of `workload`; returns rank 0's line."""
    import mla_latent_space_lca_b200 as lca
    from mla_latent_space_lca_b200.split_blocks import prefill_block_ranges

    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[workload]
    B, L = wl["B"], wl["L"]
    inp = make_prefill_inputs(B, L, seed=0 if split else replica_seed(rank))
    qs, ql = prefill_block_ranges(L, world)[rank] if split else (0, L)
    cache, q, w_uv = inp.cache.to(dev), inp.q.to(dev), inp.w_uv.to(dev)
    ws = lca.workspace(4, B, L, ql, device=dev)
    out = torch.empty(B, ql, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    variant = VARIANTS[args.variant]

    def step():
        lca.lca_prefill_block(cache, q, w_uv, qs, ql, scale=inp.scale, out=out, ws=ws, stream=stream,
                              variant=variant)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    n0 = lca.launch_count()
    if sampler:
        sampler.mark()
    ms_local = time_steps(step, steps, stream)
    if sampler:
        sampler.mark()
    launches = (lca.launch_count() - n0) / steps
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(ms_local, world, dev)
    if sampler:
        sampler.stop()
    n_prof = min(steps, 3)
    prof = kernel_profile(lca, step, n_prof)

    e2e_ms = None
    h2d = d2h = 0
    if e2e:
        # end to end: the cache rows the range reads (0 .. qs+ql-1) and its
        # queries from pinned host memory, its output rows back to host
        pin = [inp.cache[:, :qs + ql].pin_memory(), inp.q[:, qs:qs + ql].pin_memory()]
        h_out = torch.empty(B, ql, 16, 128, dtype=torch.float32).pin_memory()
        dcache = torch.empty_like(inp.cache, device=dev)
        dq = torch.empty_like(inp.q, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in pin)
        d2h = h_out.numel() * 4

        def e2e_step():
            dcache[:, :qs + ql].copy_(pin[0], non_blocking=True)
            dq[:, qs:qs + ql].copy_(pin[1], non_blocking=True)
            lca.lca_prefill_block(dcache, dq, w_uv, qs, ql, scale=inp.scale, out=out, ws=ws, variant=variant)
            h_out.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(time_steps(e2e_step, max(1, min(args.e2e_steps, 3)), stream), world, dev)
        del dcache, dq, pin, h_out

    # in-run comparison: full causal MLA prefill over the same inputs (the same
    # path with a window covering the whole sequence, so nothing is condensed)
    mla_ms = None
    if mla_compare and not split:
        ws_mla = lca.workspace(4, B, L, L, w=L, device=dev)

        def mla_step():
            lca.lca_prefill_block(cache, q, w_uv, 0, L, w=L, scale=inp.scale, out=out, ws=ws_mla,
                                  stream=stream)

        mla_step()
        torch.cuda.synchronize()
        mla_ms = max_over_ranks(time_steps(mla_step, mla_compare, stream), world, dev)
        del ws_mla
    device_ok(lca)

    line = None
    if rank == 0:
        tokens = B * L * (1 if split else world)
        fl = prefill_flops(L, inp.w, qs // 16, (qs + ql) // 16)   # rank 0's blocks
        step_flops = B * sum(fl.values()) * (1 if split else world)
        if split:   # the whole job's flops: every rank's range
            step_flops = B * sum(prefill_flops(L, inp.w).values())
        peak, peak_kind = measured_tensor_peak()
        attn = prof.get("attn_prefill")
        attn_ms = attn[1] / attn[0] if attn else None
        attn_flops_launch = B * fl["attention"] / (attn[0] / n_prof) if attn else None
        achieved = attn_flops_launch / (attn_ms / 1e3) / 1e12 if attn_ms else None
        traffic = ncu_traffic(workload, "attn_prefill") if not split and not variant else None
        line = {
            "metric": PREFILL_METRIC, "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong" if split else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": prefill_config(workload, B, L, world, args.variant, split, (qs, qs + ql)),
            "step_tflops": step_flops / (ms / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "attn_prefill", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "TFLOP/s",
                         "frac": achieved / peak if achieved else None,
                         "traffic": traffic, "algorithmic_flops_per_launch": attn_flops_launch,
                         "launch_ms": attn_ms},
            "kernels_ms_per_step": {k: v[1] / n_prof for k, v in prof.items()},
            "gpu_launches": launches,
            "clocks": sampler.summary() if sampler else None,
        }
        if e2e_ms is not None:
            line["e2e"] = {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        if mla_ms is not None:
            mla_fl = prefill_flops(L, L)
            line["mla_prefill"] = {"ms_per_step": mla_ms, "tokens_per_s": tokens / (mla_ms / 1e3),
                                   "speedup_of_lca": mla_ms / ms,
                                   "step_tflops": B * sum(mla_fl.values()) / (mla_ms / 1e3) / 1e12}
        if world == 1 and with_cpu:
            import oracle
            tok_s, cores, sample, _ = prefill_cpu_baseline(inp, 2 * oracle.num_threads(), variant=variant)
            line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                    "kind": "oracle", "sample": sample}
    del cache, q, w_uv, ws, out, inp
    gc.collect()
    torch.cuda.empty_cache()
    return line
