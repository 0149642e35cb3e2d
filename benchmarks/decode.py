"""The fused LCA decode step (lca_decode), or an ablation through
lca_condense + lca_decode_attn, timed on one workload.

One step = one whole decode step (summary query, importance, group softmax
pooling, anchor pick, split-L attention over [representatives || window],
log-sum-exp combine, W_UV up-projection) for every sequence of the batch,
through the C ABI.  Inputs are seeded and synthetic
(mla_latent_space_lca_b200/inputs.py) and resident in HBM."""
from __future__ import annotations

import gc
import time

import torch

from mla_latent_space_lca_b200.inputs import WORKLOADS, make_decode_inputs

from .common import (METRIC, ROW_BYTES, VARIANTS, ClockSampler, barrier, cpu_baseline, decode_config, device_ok,
                     flush_buffer, kernel_profile, max_over_ranks, measured_hbm_peak, ncu_traffic, replica_seed,
                     time_steps)


def run_decode(args, workload, rank, world, local_rank, steps, warmup, *, mla_compare=0, unfused_compare=0,
               e2e=True, e2e_graph=True, e2e_full_copy=0, cpu_seconds=10.0, with_cpu=True):
    """Time `steps` decode steps of `workload`; returns rank 0's line (a
    dict; None on other ranks)."""
    import mla_latent_space_lca_b200 as lca

    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[workload]
    assert wl["kind"] == "decode"
    B, L = wl["B"], wl["L"]
    inp = make_decode_inputs(B, L, seed=replica_seed(rank))
    cache, q_recent, q, w_uv = (inp.cache.to(dev), inp.q_recent.to(dev), inp.q.to(dev), inp.w_uv.to(dev))
    ws = lca.workspace(3, B, L, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    variant = VARIANTS[args.variant]
    rep_v = (torch.empty(B, max(1, lca.num_groups(L)), 576, dtype=torch.bfloat16, device=dev)
             if variant else None)

    def decode(q_rec, q_now, st=stream, dst=None):   # st None: the current stream (a graph capture's)
        o = out if dst is None else dst
        if variant:
            # an ablation: condense with it, then attend the representatives
            lca.lca_condense(cache, q_rec, scale=inp.scale, rep=rep_v, ws=ws, stream=st, variant=variant)
            lca.lca_decode_attn(cache, rep_v, q_now, w_uv, scale=inp.scale, out=o, ws=ws, stream=st)
        else:
            lca.lca_decode(cache, q_rec, q_now, w_uv, scale=inp.scale, out=o, ws=ws, stream=st)

    def step():
        decode(q_recent, q)

    # a cache smaller than twice the 126 MB L2 would be served from L2 on
    # back-to-back steps: flush L2 before every step and time steps one by one
    flush = flush_buffer(B * L * ROW_BYTES, dev)
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
    ms_local = time_steps(step, steps, stream, flush)
    if sampler:
        sampler.mark()
    launches = (lca.launch_count() - n0) / steps
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(ms_local, world, dev)
    if sampler:
        sampler.stop()

    # in-run comparison: the unfused path (condense to stored representatives,
    # then attention over them), which writes and re-reads the representatives
    unfused_ms = condense_ms = None
    if unfused_compare and lca.num_groups(L) > 0 and not variant:
        rep_u = torch.empty(B, lca.num_groups(L), 576, dtype=torch.bfloat16, device=dev)

        def unfused_step():
            lca.lca_condense(cache, q_recent, scale=inp.scale, rep=rep_u, ws=ws, stream=stream)
            lca.lca_decode_attn(cache, rep_u, q, w_uv, scale=inp.scale, out=out, ws=ws, stream=stream)

        for _ in range(3):
            unfused_step()
        torch.cuda.synchronize()
        unfused_ms = max_over_ranks(time_steps(unfused_step, unfused_compare, stream, flush), world, dev)
        uprof = kernel_profile(lca, unfused_step, min(unfused_compare, 200), flush)
        ucond = uprof.get("condense")
        condense_ms = ucond[1] / ucond[0] if ucond else None
        del rep_u

    # in-run comparison: plain MLA decode (g = 1) over the whole cache, the
    # same inputs, timed the same way
    mla = None
    if mla_compare and not variant:
        def mla_step():
            lca.mla_decode_attn(cache, q, w_uv, inp.scale, out=out, ws=ws, stream=stream)

        for _ in range(3):
            mla_step()
        torch.cuda.synchronize()
        msampler = ClockSampler(local_rank) if rank == 0 else None
        time.sleep(0.25 if msampler else 0)
        if msampler:
            msampler.mark()
        mla_ms_local = time_steps(mla_step, mla_compare, stream, flush)
        if msampler:
            msampler.mark()
            msampler.stop()
        mla_ms = max_over_ranks(mla_ms_local, world, dev)
        mprof = kernel_profile(lca, mla_step, min(mla_compare, 200), flush)
        mattn = mprof.get("attn_decode")
        mla = {"ms_per_step": mla_ms, "attn_ms": mattn[1] / mattn[0] if mattn else None,
               "clocks": msampler.summary() if msampler else None, "steps": mla_compare}

    # per-kernel durations (CUDA events around each launch, on its stream)
    prof = kernel_profile(lca, step, min(steps, 200), flush)

    e2e_ms = graph_ms = full_ms = None
    h2d = d2h = 0
    if e2e:
        # end to end through the public API, as a decode loop runs: the cache
        # is state resident on the device (the prefill wrote it), and so are
        # the recent queries, kept as a ring (only their mean is used); every
        # step brings the new token's row (into row L-1 of each sequence) and
        # its query from pinned host memory, puts the query into the ring's
        # oldest slot, decodes, and delivers the result to host memory.
        # Steps are timed one by one, with the L2 flush between them when the
        # cache would otherwise stay in L2.
        # No copy engine: lca_append_token reads the new rows and queries in
        # place from pinned host memory (and leaves a device copy of the
        # query for the decode), and the decode's tail writes out straight
        # into pinned host memory.
        h_rows = inp.cache[:, L - 1].contiguous().pin_memory()
        h_q = inp.q.pin_memory()
        dq = torch.empty_like(h_q, device=dev)
        ring = inp.q_recent.to(dev)
        h_out = torch.empty(B, 16, 128, dtype=torch.float32).pin_memory()
        h2d = (h_rows.numel() + h_q.numel()) * 2
        d2h = h_out.numel() * 4
        slot = [0]

        def e2e_step():
            lca.lca_append_token(cache, L - 1, h_rows, q=h_q, ring=ring, slot=slot[0], q_out=dq)
            slot[0] = (slot[0] + 1) % ring.shape[1]
            decode(ring, dq, dst=h_out)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        n_e2e = max(1, args.e2e_steps)
        xev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        for a_, b_ in xev:
            if flush is not None:
                flush.zero_()
            a_.record(stream)
            e2e_step()
            b_.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in xev) / n_e2e, world, dev)
        decode(ring, dq)   # the last step again, on the device path
        torch.cuda.synchronize()
        assert torch.equal(h_out, out.cpu())

        # the same loop with each step captured once in a CUDA graph (one
        # graph per ring slot: the slot a step writes is part of the step)
        # and replayed: the copies and launches of a step go to the GPU in
        # one call
        if e2e_graph:
            def graph_step(sl):
                lca.lca_append_token(cache, L - 1, h_rows, q=h_q, ring=ring, slot=sl, q_out=dq)
                decode(ring, dq, st=None, dst=h_out)

            graphs = []
            for sl in range(ring.shape[1]):
                gph = torch.cuda.CUDAGraph()
                # thread-local capture: other host threads (a process group's
                # watchdog) may keep making CUDA calls meanwhile
                with torch.cuda.graph(gph, capture_error_mode="thread_local"):
                    graph_step(sl)
                graphs.append(gph)
            for i in range(3):
                graphs[i % len(graphs)].replay()
            torch.cuda.synchronize()
            barrier(world)
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(n_e2e)]
            for i, (a_, b_) in enumerate(gev):
                if flush is not None:
                    flush.zero_()
                a_.record(stream)
                graphs[i % len(graphs)].replay()
                b_.record(stream)
            torch.cuda.synchronize()
            graph_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in gev) / n_e2e, world, dev)
            decode(ring, dq)   # the last step again, on the device path
            torch.cuda.synchronize()
            assert torch.equal(h_out, out.cpu())
            del graphs

        # for reference: the same step with the whole cache and all recent
        # queries copied in from the host
        if e2e_full_copy and not variant:
            pin_cache = inp.cache.pin_memory()
            pin = [t.pin_memory() for t in (inp.q_recent, inp.q)]
            dbuf = [torch.empty_like(t, device=dev) for t in pin]
            dcache = torch.empty_like(pin_cache, device=dev)
            x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            x0.record(stream)
            for _ in range(e2e_full_copy):
                dcache.copy_(pin_cache, non_blocking=True)
                for d, h in zip(dbuf, pin):
                    d.copy_(h, non_blocking=True)
                lca.lca_decode(dcache, dbuf[0], dbuf[1], w_uv, scale=inp.scale, out=out, ws=ws)
                h_out.copy_(out, non_blocking=True)
            x1.record(stream)
            torch.cuda.synchronize()
            full_ms = max_over_ranks(x0.elapsed_time(x1) / e2e_full_copy, world, dev)
            del dcache, pin_cache
    device_ok(lca)

    line = None
    if rank == 0:
        tokens = B * world
        value = tokens / (ms / 1e3)
        gbs = B * L * ROW_BYTES * world / (ms / 1e3) / 1e9
        peak, peak_kind = measured_hbm_peak()
        if variant:
            # the ablation's step is dominated by the condensation: 16 m
            # history rows read and m representatives written per sequence
            attn = prof.get("condense")
            algo_bytes = B * 17 * lca.num_groups(L) * ROW_BYTES
            traffic = None
            rl_kernel = f"condense ({args.variant})"
        else:
            attn = prof.get("attn_decode")
            algo_bytes = B * L * ROW_BYTES
            traffic = ncu_traffic(workload)
            rl_kernel = "attn_decode (fused LCA)"
        attn_ms = attn[1] / attn[0] if attn else None
        achieved = algo_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
        clocks = sampler.summary() if sampler else None
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": decode_config(workload, B, L, world, args.variant, flush is not None),
            "cache_gbps": gbs, "cache_frac_of_hbm": gbs / world / peak,
            "cache_frac_of_nominal_8tbs": gbs / world / 8000.0,
            "roofline": {"bound": "hbm", "kernel": rl_kernel,
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak if achieved else None, "traffic": traffic,
                         "algorithmic_bytes_per_launch": algo_bytes,
                         "launch_ms": attn_ms},
            "kernels_ms_per_step": {k: v[1] / v[0] for k, v in prof.items()},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
            # the step's time scaled to the maximum SM clock: how much of a
            # gap to another run is the clock (the step is partly SM-bound)
            line["ms_per_step_at_max_clock"] = ms * clocks["sm_mhz"] / clocks["sm_max_mhz"]
        if e2e_ms is not None:
            line["e2e"] = {
                "value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": ("lca_decode" if not variant else "lca_condense + lca_decode_attn") +
                        " in a decode loop: cache and recent-query ring resident on the device; "
                        "per step lca_append_token reads the new token's rows and query in place from pinned "
                        "host memory into the cache and the ring, and the decode writes out straight into "
                        "pinned host memory (no copy-engine transfers)"}
        if graph_ms is not None:
            line["e2e_graph"] = {
                "value": tokens / (graph_ms / 1e3), "unit": "tokens/s", "ms_per_step": graph_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "the e2e loop with each step (append from host memory, decode into host memory) "
                        "captured once as a CUDA graph through the same public calls and replayed"}
        if full_ms is not None:
            line["e2e_full_cache_copy"] = {
                "value": tokens / (full_ms / 1e3), "unit": "tokens/s", "ms_per_step": full_ms,
                "h2d_bytes_per_step": B * L * ROW_BYTES + (inp.q_recent.numel() + inp.q.numel()) * 2,
                "d2h_bytes_per_step": d2h,
                "note": "the whole cache copied in from the host every step (bounded by the host link)"}
        if mla is not None:
            line["mla_path"] = {
                "ms_per_step": mla["ms_per_step"], "tokens_per_s": tokens / (mla["ms_per_step"] / 1e3),
                "lca_speedup": mla["ms_per_step"] / ms,
                "steps": mla["steps"], "clocks": mla["clocks"],
                "attn_ms": mla["attn_ms"],
                "attn_frac_of_hbm": (algo_bytes / (mla["attn_ms"] / 1e3) / 1e9 / peak) if mla["attn_ms"] else None,
                "note": "mla_decode_attn (g = 1): every cached row attended, same inputs and timing; "
                        "reads the same bytes as the fused LCA step, with 16x the attention rows"}
        if unfused_ms is not None:
            m = lca.num_groups(L)
            line["unfused_path"] = {
                "ms_per_step": unfused_ms, "tokens_per_s": tokens / (unfused_ms / 1e3),
                "fused_speedup": unfused_ms / ms,
                "algorithmic_bytes_per_step": B * (L + 2 * m) * ROW_BYTES,
                "note": "lca_condense (reads the cache, writes m representatives) then lca_decode_attn "
                        "(re-reads them and the window)"}
            if condense_ms:
                # condense_kernel alone: the 16 m history rows read, the m representatives written
                cbytes = B * 17 * m * ROW_BYTES
                line["unfused_path"]["condense_kernel"] = {
                    "launch_ms": condense_ms, "algorithmic_bytes_per_launch": cbytes,
                    "achieved_gbs": cbytes / (condense_ms / 1e3) / 1e9,
                    "frac_of_measured_hbm": cbytes / (condense_ms / 1e3) / 1e9 / peak}
        if world == 1 and with_cpu:
            tok_s, cores, sample, _ = cpu_baseline(inp, cpu_seconds, variant=variant)
            line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                    "kind": "oracle", "sample": sample}
    del cache, q_recent, q, w_uv, ws, out, rep_v, flush, inp
    gc.collect()
    torch.cuda.empty_cache()
    return line
