"""Decode modes beyond the fused step: stored representatives (the page's
90% KV-cache reading), a ragged batch, and every sequence split along its
cache over the ranks.  Each returns rank 0's JSON line as a dict."""
from __future__ import annotations

import time

import torch

from mla_latent_space_lca_b200.inputs import WORKLOADS, make_decode_inputs

from .common import (METRIC, ROW_BYTES, ClockSampler, L2Flush, cpu_baseline, flush_buffer, max_over_ranks,
                     measured_hbm_peak, ncu_traffic, replica_seed)


def stored_cpu_baseline(inp, budget_s: float):
    """The oracle's step over kept representatives (attention over [bf16
    representatives || window], then W_UV) on one sequence, timed for about
    budget_s on the host cores; the representatives come from the oracle's
    own condensation, built before the timed loop."""
    import numpy as np

    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits

    c = bf16_bits(inp.cache[:1])
    qr, qb, w = bf16_bits(inp.q_recent[:1]), bf16_bits(inp.q[:1]), bf16_bits(inp.w_uv)
    r = oracle.lca_condense(c, qr, inp.g, inp.w, inp.scale)
    rep = bf16_bits(torch.from_numpy(np.concatenate([r["rep_c"], r["rep_k"]], axis=2)).to(torch.bfloat16))
    n, total, t_start = 0, 0.0, time.time()
    while n == 0 or time.time() - t_start < budget_s:
        t0 = time.perf_counter()
        oracle.lca_attend_reps(c, rep, qb, w, inp.g, inp.w, inp.scale)
        total += time.perf_counter() - t0
        n += 1
    return {"value": n / total, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"1 of {inp.B} sequences (L={inp.L}) per oracle call, {n} calls, {total:.1f} s of CPU "
                      "time: attention over the kept representatives and the window, then W_UV"}


def run_stored(args, rank, world, local_rank):
    """Stored-representative decode: the representative cache is built once
    (untimed); a step is lca_decode_stored, plus every 16th step the append of
    one group per sequence (the rate at which groups leave the window).  The
    rows a step reads ((m + w') x 1152 B per sequence) fit in L2 at these
    sizes, so L2 is flushed before every step and steps are timed one by one."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca

    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    B, L = wl["B"], wl["L"]
    inp = make_decode_inputs(B, L, seed=replica_seed(rank))
    cache, q_recent, q, w_uv = (inp.cache.to(dev), inp.q_recent.to(dev), inp.q.to(dev),
                                inp.w_uv.to(dev))
    m = lca.num_groups(L)
    rep = torch.empty(B, max(m, 1), 576, dtype=torch.bfloat16, device=dev)
    ws = lca.workspace(3, B, L, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    lca.lca_condense_append(cache, q_recent, rep, 0, scale=inp.scale, ws=ws, stream=stream)
    flush = L2Flush(dev)

    def step(i):
        if i % 16 == 15 and m > 0:   # one group per sequence leaves the window every 16 steps
            lca.lca_condense_append(cache, q_recent, rep, m - 1, scale=inp.scale, ws=ws, stream=stream)
        lca.lca_decode_stored(cache, rep, q, w_uv, scale=inp.scale, out=out, ws=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    n0 = lca.launch_count()
    if sampler:
        sampler.mark()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    launches = (lca.launch_count() - n0) / args.steps
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, world, dev)
    barrier()
    if sampler:
        sampler.stop()

    # per-kernel times (events around each launch), L2 flushed before each step
    lca.profile_enable(True)
    prof_steps = min(args.steps, 160)
    for i in range(prof_steps):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)

    # end to end, as a decode loop runs: cache, kept representatives and the
    # recent-query ring resident on the device; per step lca_append_token
    # reads the new token's row (into row L-1) and its query (into the ring's
    # oldest slot, and a device copy for the decode) in place from pinned
    # host memory, every 16th step the append of the group that left the
    # window, the decode writing out straight into pinned host memory; steps
    # timed one by one with the L2 flush between them
    pin_row = inp.cache[:, L - 1].contiguous().pin_memory()
    pin_q = inp.q.pin_memory()
    ring = q_recent.clone()
    dq = torch.empty_like(pin_q, device=dev)
    h_out = torch.empty(B, 16, 128, dtype=torch.float32).pin_memory()
    h2d = pin_row.numel() * 2 + pin_q.numel() * 2
    n_step = [0]

    def e2e_step():
        i = n_step[0]
        n_step[0] += 1
        lca.lca_append_token(cache, L - 1, pin_row, q=pin_q, ring=ring, slot=i % ring.shape[1], q_out=dq,
                             stream=stream)
        if i % 16 == 15 and m > 0:
            lca.lca_condense_append(cache, ring, rep, m - 1, scale=inp.scale, ws=ws, stream=stream)
        lca.lca_decode_stored(cache, rep, dq, w_uv, scale=inp.scale, out=h_out, ws=ws, stream=stream)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(1, args.e2e_steps)
    xev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
    for a_, b_ in xev:
        flush.zero_()
        a_.record(stream)
        e2e_step()
        b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in xev) / n_e2e, world, dev)
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    if rank != 0:
        return None
    rows = m + (L - 16 * m)                     # kept representatives + window rows
    read_bytes = B * rows * ROW_BYTES
    peak, peak_kind = measured_hbm_peak()
    attn = prof.get("attn_decode")
    attn_ms = attn[1] / attn[0] if attn else None
    achieved = read_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
    line = {
        "metric": METRIC, "value": B * world / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": "stored representatives", "B_per_gpu": B, "L": L,
                   "g": 16, "w": 1024, "kept_rows_per_seq": rows, "parallelism": f"replicas x{world}",
                   "l2": L2Flush.NOTE},
        "read_gbps": read_bytes * world / (ms / 1e3) / 1e9,
        "kv_rows_read_fraction": rows / L,
        "roofline": {"bound": "hbm", "kernel": "attn_decode (stored representatives)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None,
                     "traffic": ncu_traffic(args.workload + "_stored"),
                     "algorithmic_bytes_per_launch": read_bytes, "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / prof_steps for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": B * world / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h_out.numel() * 4,
                "note": "decode loop: cache, kept representatives and recent-query ring resident on the "
                        "device; per step lca_append_token reads the new token's row and query in place from "
                        "pinned host memory (every 16th step also the append of one group), and the decode "
                        "writes out straight into pinned host memory"},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = stored_cpu_baseline(inp, args.cpu_seconds / 2)
    return line


def run_varlen(args, rank, world, local_rank):
    """Decode of a ragged batch (lca_decode_varlen): B sequences whose
    lengths are drawn, seeded, uniformly from [L/8, 15L/8] (mean L), held in
    one [B, 15L/8, 576] buffer.  Algorithmic bytes: the rows each sequence
    holds, read once."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca

    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    assert wl["kind"] == "decode"
    B, L = wl["B"], wl["L"]
    L_max = L // 8 * 15
    gen = torch.Generator().manual_seed(1000 + replica_seed(rank))
    lens = torch.randint(L // 8, L_max + 1, (B,), generator=gen, dtype=torch.int32)
    inp = make_decode_inputs(B, L_max, seed=replica_seed(rank))
    cache, q_recent, q, w_uv = (inp.cache.to(dev), inp.q_recent.to(dev), inp.q.to(dev), inp.w_uv.to(dev))
    lens_d = lens.to(dev)
    rows = int(lens.sum())
    ws = lca.workspace(3, B, L_max, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        lca.lca_decode_varlen(cache, lens_d, q_recent, q, w_uv, scale=inp.scale, out=out, ws=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    n0 = lca.launch_count()
    if sampler:
        sampler.mark()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    launches = (lca.launch_count() - n0) / args.steps
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    if sampler:
        sampler.stop()
    lca.profile_enable(True)
    for _ in range(min(args.steps, 200)):
        step()
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)

    # end to end, as a decode loop runs: cache and recent-query ring resident;
    # per step each sequence's new row (at its own last position) and its
    # query in from pinned host memory, out back
    idx = torch.arange(B, device=dev)
    last_row = (lens_d - 1).long()
    pin_rows = inp.cache[torch.arange(B), (lens - 1).long()].contiguous().pin_memory()
    pin_q = inp.q.pin_memory()
    ring = q_recent.clone()
    drows = torch.empty_like(pin_rows, device=dev)
    dq = torch.empty_like(pin_q, device=dev)
    h_out = torch.empty(B, 16, 128, dtype=torch.float32).pin_memory()
    h2d = pin_rows.numel() * 2 + pin_q.numel() * 2
    n_step = [0]

    def e2e_step():
        drows.copy_(pin_rows, non_blocking=True)
        cache[idx, last_row] = drows
        dq.copy_(pin_q, non_blocking=True)
        ring[:, n_step[0] % ring.shape[1]].copy_(dq)
        n_step[0] += 1
        lca.lca_decode_varlen(cache, lens_d, ring, dq, w_uv, scale=inp.scale, out=out, ws=ws)
        h_out.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    n_e2e = max(1, args.e2e_steps)
    for _ in range(n_e2e):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / n_e2e, world, dev)
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    if rank != 0:
        return None
    peak, peak_kind = measured_hbm_peak()
    attn = prof.get("attn_decode")
    attn_ms = attn[1] / attn[0] if attn else None
    algo_bytes = rows * ROW_BYTES
    achieved = algo_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
    line = {
        "metric": METRIC, "value": B * world / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "mode": "ragged batch", "B_per_gpu": B,
                   "lengths": f"uniform in [{L // 8}, {L_max}] (seeded), total {rows} rows",
                   "g": 16, "w": 1024, "parallelism": f"replicas x{world}",
                   "l2": "cache rows far larger than the 126 MB L2; no flush"},
        "cache_gbps": algo_bytes * world / (ms / 1e3) / 1e9,
        "cache_frac_of_nominal_8tbs": algo_bytes / (ms / 1e3) / 1e9 / 8000.0,
        "roofline": {"bound": "hbm", "kernel": "attn_decode (fused LCA, ragged)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None, "traffic": None,
                     "algorithmic_bytes_per_launch": algo_bytes, "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / v[0] for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": B * world / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h_out.numel() * 4,
                "note": "decode loop: cache and recent-query ring resident; per step each sequence's new row "
                        "and query in from pinned host memory, out back"},
    }
    return line


def run_split(args, rank, world, local_rank):
    """Decode with every sequence's cache split along L over the ranks: rank r
    holds rows shard_bounds(L, world)[r] of the same B sequences; a step is
    its shard record, an all-gather of the records and the merge + W_UV.
    The whole job decodes B tokens per step whatever the rank count."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca
    from mla_latent_space_lca_b200.split_l import shard_bounds, split_l_decode

    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    assert wl["kind"] == "decode"
    B, L = wl["B"], wl["L"]
    inp = make_decode_inputs(B, L, seed=0)          # the same sequences on every rank
    row0, row1 = shard_bounds(L, world)[rank]
    h_shard = inp.cache[:, row0:row1].contiguous()
    cache = h_shard.to(dev)
    q_recent, q, w_uv = inp.q_recent.to(dev), inp.q.to(dev), inp.w_uv.to(dev)
    ws = lca.workspace(3, B, L, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(c=cache, qr=q_recent, qq=q):
        split_l_decode(c, qr, qq, w_uv, L, row0, scale=inp.scale, out=out, ws=ws)

    def barrier():
        if world > 1:
            dist.barrier()

    shard_bytes = B * (row1 - row0) * ROW_BYTES
    flush = flush_buffer(shard_bytes, dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.25 if sampler else 0)
    n0 = lca.launch_count()
    if sampler:
        sampler.mark()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a_, b_ in ev:
        if flush is not None:
            flush.zero_()
        a_.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    total_ms = sum(a_.elapsed_time(b_) for a_, b_ in ev)
    if sampler:
        sampler.mark()
    launches = (lca.launch_count() - n0) / args.steps
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(total_ms / args.steps, world, dev)
    if sampler:
        sampler.stop()

    prof_steps = min(args.steps, 200)
    lca.profile_enable(True)
    for _ in range(prof_steps):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)

    # the fused single-device decode of the same sequences, for comparison (one rank)
    fused_ms = None
    if world == 1:
        def fused():
            lca.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, out=out, ws=ws)
        for _ in range(3):
            fused()
        torch.cuda.synchronize()
        fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(min(args.steps, 200))]
        for a_, b_ in fev:
            if flush is not None:
                flush.zero_()
            a_.record(stream)
            fused()
            b_.record(stream)
        torch.cuda.synchronize()
        fused_ms = sum(a_.elapsed_time(b_) for a_, b_ in fev) / len(fev)

    # end to end, as a decode loop runs: each rank's shard and its
    # recent-query ring stay resident; per step the rank holding row L-1
    # takes the new token's row, every rank the query (into the ring's oldest
    # slot), from pinned host memory; out back
    last = row1 == L
    pin_row = inp.cache[:, L - 1].contiguous().pin_memory() if last else None
    pin_q = inp.q.pin_memory()
    ring = q_recent.clone()
    dq = torch.empty_like(pin_q, device=dev)
    h_out = torch.empty(B, 16, 128, dtype=torch.float32).pin_memory()
    h2d = (pin_row.numel() * 2 if last else 0) + pin_q.numel() * 2
    n_step = [0]

    def e2e_step():
        if last:
            cache[:, L - 1 - row0].copy_(pin_row, non_blocking=True)
        dq.copy_(pin_q, non_blocking=True)
        ring[:, n_step[0] % ring.shape[1]].copy_(dq)
        n_step[0] += 1
        step(cache, ring, dq)
        h_out.copy_(out, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize()
    barrier()
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
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    if rank != 0:
        return None
    peak, peak_kind = measured_hbm_peak()
    attn = prof.get("attn_decode")
    attn_ms = attn[1] / attn[0] if attn else None
    achieved = shard_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
    line = {
        "metric": METRIC, "value": B / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "L": L, "g": 16, "w": 1024, "heads": 16,
                   "d_c": 512, "d_r": 64, "parallelism": f"split-L x{world}",
                   "rank0_rows": [row0, row1],
                   "l2": ("shard larger than the 126 MB L2; no flush" if flush is None else
                          L2Flush.NOTE)},
        "cache_gbps": B * L * ROW_BYTES / (ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": "attn_decode (fused LCA, rank 0's shard)",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None,
                     "traffic": ncu_traffic(args.workload) if world == 1 else None,
                     "algorithmic_bytes_per_launch": shard_bytes, "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / v[0] for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": B / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h_out.numel() * 4},
    }
    if fused_ms is not None:
        line["fused_decode_ms_per_step"] = fused_ms
    if world == 1 and not args.no_cpu_baseline:
        tok_s, cores, sample, _ = cpu_baseline(inp, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    return line
