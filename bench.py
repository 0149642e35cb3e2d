#!/usr/bin/env python
"""LCA decode benchmark: tokens/s and cache-read GB/s against the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores
    python bench.py --workload prefill_b1_l128k --steps 10 --warmup 3   # blockwise prefill

One step = one whole fused LCA decode step (summary query, importance,
group softmax pooling, anchor pick, split-L attention over
[representatives || window], log-sum-exp combine, W_UV up-projection) for
every sequence of the batch, through the C ABI.  Inputs are synthetic and
seeded (see mla_latent_space_lca_b200/inputs.py) and resident in HBM; the
default workload's cache (1.2 GB) is ~10x the L2, so no flush is needed
between steps.  Multi-GPU (torchrun): each rank decodes its own batch (weak
scaling, no data-path collective); timing is the max over ranks.  Rank 0
prints one JSON line.

The prefill workload times one blockwise prefill of the whole sequence
(lca_prefill_block over [0, L)) per step; its roofline is the attention
kernel's algorithmic flops against the sustained bf16 tensor peak.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from mla_latent_space_lca_b200.inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs  # noqa: E402

ROW_BYTES = 576 * 2
METRIC = "LCA decode tokens/s and cache-read GB/s (fraction of B200 HBM roofline)"
PREFILL_METRIC = "LCA blockwise prefill tokens/s (fraction of B200 bf16 tensor roofline)"
PROFILE_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
# lca_params.variant: the method and the two ablations of the page's ablation table
VARIANTS = {"lca": 0, "pool_position": 1, "sparse": 2}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="default 2000 (decode), 10 (prefill)")
    ap.add_argument("--warmup", type=int, default=None, help="default 20 (decode), 3 (prefill)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_b32_l32k")
    ap.add_argument("--e2e-steps", type=int, default=20)
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
    ap.add_argument("--mla-compare", type=int, default=0,
                    help="decode: also time N plain MLA decode steps (g = 1, every row attended) on the "
                         "same inputs; prefill: N full causal MLA prefills (w = L)")
    return ap.parse_args()


def measured_tensor_peak():
    """Sustained bf16 GEMM peak (a kernel timed inside a long step)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except (OSError, KeyError, ValueError):
        return 1400.0, "fallback (sustained)"


def prefill_flops(L: int, w: int, k0: int = 0, k1: int | None = None, g: int = 16):
    """Algorithmic flops of a blockwise prefill over [0, L): block k has
    m_k = max(0, floor((16k - w)/16)) representatives; its query t attends
    m_k + (t - 16 m_k + 1) keys, each 16 heads x (576 + 512) x 2 flops; the
    condensation scores (folded summary query, 576 x 2) and pools (512 x 2)
    every history row of the block; W_UV is 16 x 512 x 128 x 2 per query.
    Blocks k0 .. k1-1 (default: all)."""
    cw = -(-w // 16)
    att = cond = 0
    k1 = L // 16 if k1 is None else k1
    for k in range(k0, k1):
        m = max(0, k - cw)
        keys = 16 * m + sum(16 * k + tt - 16 * m + 1 for tt in range(16))
        att += keys * 16 * (576 + 512) * 2
        cond += 16 * m * (576 + 512) * 2
    wuv = 16 * (k1 - k0) * 16 * 512 * 128 * 2
    return {"attention": att, "condense": cond, "wuv": wuv}


def prefill_cpu_baseline(inp, n_blocks: int, steps: int = 1, warmup: int = 0, variant: int = 0):
    """The oracle on `n_blocks` evenly spaced blocks of the prefill (their
    average cost matches the whole range's); tokens/s extrapolated."""
    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits

    nb = inp.L // 16
    blocks = sorted(set(int(round(x)) for x in
                        [i * (nb - 1) / max(1, n_blocks - 1) for i in range(n_blocks)]))
    c, q, w = bf16_bits(inp.cache), bf16_bits(inp.q), bf16_bits(inp.w_uv)
    for _ in range(warmup):
        oracle.lca_prefill(c, q, w, 0, inp.L, 16, inp.w, inp.scale, blocks=blocks, want_olat=False,
                           variant=variant)
    times = []
    for _ in range(max(1, steps)):
        t0 = time.perf_counter()
        oracle.lca_prefill(c, q, w, 0, inp.L, 16, inp.w, inp.scale, blocks=blocks, want_olat=False,
                           variant=variant)
        times.append(time.perf_counter() - t0)
    tok_s = 16 * len(blocks) * inp.B / statistics.mean(times)
    sample = (f"{len(blocks)} evenly spaced blocks of {nb} (16 queries each) per oracle call, "
              f"{len(times)} calls; tokens/s extrapolated to the whole prefill")
    return tok_s, oracle.num_threads(), sample, times


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.marks = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t0, t1 = (self.marks + [0, 0])[:2] if len(self.marks) >= 2 else (0, 1e30)
        inside = [r for t, r in self.rows if t0 <= t <= t1]
        note = None
        if not inside:
            # timed region shorter than the sampling period: nearest sample
            inside = [min(self.rows, key=lambda tr: abs(tr[0] - t0))[1]]
            note = "timed region shorter than one 100 ms sample; nearest sample"
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in inside if len(r) > 8 and num(r[1]) is not None]
        mx = [num(r[2]) for r in inside if len(r) > 8 and num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for k, nm in enumerate(names):
                if len(r) > 5 + k and r[5 + k].lower().startswith("active"):
                    reasons.add(nm)
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
               "samples": len(inside)}
        if note:
            out["note"] = note
        return out


def source_hash():
    h = hashlib.sha256()
    for f in ("attn_decode.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "mla_latent_space_lca_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    try:
        with open(PROFILE_FILE) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("source_hash") != source_hash():
            return None
        return e["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


REF_BUDGET_S = 150.0   # whole reference-arm run (all K + W steps), seconds


def cpu_baseline(inp, budget_s: float, steps: int = 0, warmup: int = 0, seqs: int = 0, variant: int = 0):
    """The oracle as it stands, on host cores, over a bounded sample of the
    workload (whole sequences; `seqs` per call, else ~2 s worth).  An
    ablation runs the oracle's condensation with it, rounds the
    representatives to bf16 as the GPU stores them, and attends them.
    Returns (tokens/s, cores, sample text, per-step seconds)."""
    import numpy as np

    import oracle
    from mla_latent_space_lca_b200.inputs import bf16_bits

    def decode(c, qr, q, w):
        if not variant:
            return oracle.lca_decode(c, qr, q, w, inp.g, inp.w, inp.scale)
        r = oracle.lca_condense(c, qr, inp.g, inp.w, inp.scale, variant=variant)
        rep = bf16_bits(torch.from_numpy(np.concatenate([r["rep_c"], r["rep_k"]], axis=2)).to(torch.bfloat16))
        return oracle.lca_attend_reps(c, rep, q, w, inp.g, inp.w, inp.scale)

    B = inp.cache.shape[0]
    # sample size: sequences whose oracle decode takes ~1-3 s
    per_seq_guess = inp.L * 16 * 576 * 2 / 3e9
    S = seqs if seqs > 0 else max(1, min(B, int(2.0 / max(per_seq_guess, 1e-6))))
    S = min(S, B)
    sl = list(range(S))
    c = bf16_bits(inp.cache[:S])
    qr = bf16_bits(inp.q_recent[:S])
    q = bf16_bits(inp.q[:S])
    w = bf16_bits(inp.w_uv)
    for _ in range(warmup):
        decode(c, qr, q, w)
    times = []
    t_start = time.time()
    n = 0
    while True:
        t0 = time.perf_counter()
        decode(c, qr, q, w)
        times.append(time.perf_counter() - t0)
        n += 1
        if (steps and n >= steps) or (not steps and time.time() - t_start >= budget_s):
            break
    tok_s = S * n / sum(times)
    sample = (f"{S} of {B} sequences (L={inp.L}) per oracle call, {n} calls, "
              f"{sum(times):.1f} s of CPU time")
    del sl
    return tok_s, oracle.num_threads(), sample, times


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time (all ranks call this at the same point)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Each rank decodes its own batch (weak scaling): seed = rank."""
    return rank


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    if wl["kind"] == "prefill":
        import oracle
        inp = make_prefill_inputs(wl["B"], wl["L"], seed=0)
        # blocks per step so that all K + W steps fit REF_BUDGET_S
        n0 = oracle.num_threads()
        v = VARIANTS[args.variant]
        _, _, _, t0 = prefill_cpu_baseline(inp, n0, steps=1, variant=v)
        per_step = REF_BUDGET_S / max(1, args.steps + args.warmup)
        n = max(1, min(2 * n0, int(n0 * per_step / max(t0[0], 1e-6))))
        tok_s, cores, sample, times = prefill_cpu_baseline(inp, n, steps=args.steps, warmup=args.warmup,
                                                           variant=v)
        ms = 1e3 * statistics.mean(times)
        line = {
            "impl": "reference", "metric": PREFILL_METRIC, "value": tok_s, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "B": wl["B"], "L": wl["L"], "g": 16, "w": 1024,
                       "variant": args.variant},
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    inp = make_decode_inputs(wl["B"], wl["L"], seed=0)
    # size each step's sample so that all K + W steps fit REF_BUDGET_S: time
    # one single-sequence call first
    v = VARIANTS[args.variant]
    _, _, _, t1 = cpu_baseline(inp, 0, steps=1, warmup=0, seqs=1, variant=v)
    per_step = REF_BUDGET_S / max(1, args.steps + args.warmup)
    seqs = max(1, min(wl["B"], int(per_step / max(t1[0], 1e-6))))
    tok_s, cores, sample, times = cpu_baseline(inp, 0, steps=args.steps, warmup=args.warmup, seqs=seqs,
                                               variant=v)
    ms = 1e3 * statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": wl["B"], "L": wl["L"], "g": 16, "w": 1024,
                   "variant": args.variant},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    assert wl["kind"] == "decode"
    B, L = wl["B"], wl["L"]
    inp = make_decode_inputs(B, L, seed=replica_seed(rank))
    cache, q_recent, q, w_uv = (inp.cache.to(dev), inp.q_recent.to(dev), inp.q.to(dev),
                                inp.w_uv.to(dev))
    ws = lca.workspace(3, B, L, device=dev)
    out = torch.empty(B, 16, 128, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    variant = VARIANTS[args.variant]
    rep_v = (torch.empty(B, max(1, lca.num_groups(L)), 576, dtype=torch.bfloat16, device=dev)
             if variant else None)

    def decode(q_rec, q_now, st=stream):   # st None: the current stream (a graph capture's)
        if variant:
            # an ablation: condense with it, then attend the representatives
            lca.lca_condense(cache, q_rec, scale=inp.scale, rep=rep_v, ws=ws, stream=st, variant=variant)
            lca.lca_decode_attn(cache, rep_v, q_now, w_uv, scale=inp.scale, out=out, ws=ws, stream=st)
        else:
            lca.lca_decode(cache, q_rec, q_now, w_uv, scale=inp.scale, out=out, ws=ws, stream=st)

    def step():
        decode(q_recent, q)

    def barrier():
        if world > 1:
            dist.barrier()

    # a cache smaller than twice the 126 MB L2 would be served from L2 on
    # back-to-back steps: flush L2 before every step and time steps one by one
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if B * L * ROW_BYTES < (256 << 20) else None
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
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        total_ms = e0.elapsed_time(e1)
    else:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a_, b_ in ev:
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

    # in-run comparison: the unfused path (condense to stored representatives,
    # then attention over them), which writes and re-reads the representatives
    unfused_ms = condense_ms = None
    if args.unfused_compare and lca.num_groups(L) > 0 and not variant:
        rep_u = torch.empty(B, lca.num_groups(L), 576, dtype=torch.bfloat16, device=dev)

        def unfused_step():
            lca.lca_condense(cache, q_recent, scale=inp.scale, rep=rep_u, ws=ws, stream=stream)
            lca.lca_decode_attn(cache, rep_u, q, w_uv, scale=inp.scale, out=out, ws=ws, stream=stream)

        for _ in range(3):
            unfused_step()
        torch.cuda.synchronize()
        # timed like the main loop: back to back, or one by one after an L2
        # flush when the cache would otherwise stay in L2
        uev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.unfused_compare if flush is not None else 1)]
        if flush is None:
            uev[0][0].record(stream)
            for _ in range(args.unfused_compare):
                unfused_step()
            uev[0][1].record(stream)
        else:
            for a_, b_ in uev:
                flush.zero_()
                a_.record(stream)
                unfused_step()
                b_.record(stream)
        torch.cuda.synchronize()
        unfused_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in uev) / args.unfused_compare, world, dev)
        lca.profile_enable(True)
        for _ in range(min(args.unfused_compare, 200)):
            if flush is not None:
                flush.zero_()
            unfused_step()
        torch.cuda.synchronize()
        uprof = lca.profile_collect()
        lca.profile_enable(False)
        ucond = uprof.get("condense")
        condense_ms = ucond[1] / ucond[0] if ucond else None
        del rep_u

    # in-run comparison: plain MLA decode (g = 1) over the whole cache, the
    # same inputs, timed the same way
    mla = None
    if args.mla_compare and not variant:
        def mla_step():
            lca.mla_decode_attn(cache, q, w_uv, inp.scale, out=out, ws=ws, stream=stream)

        for _ in range(3):
            mla_step()
        torch.cuda.synchronize()
        mev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.mla_compare)]
        for a_, b_ in mev:
            if flush is not None:
                flush.zero_()
            a_.record(stream)
            mla_step()
            b_.record(stream)
        torch.cuda.synchronize()
        mla_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in mev) / args.mla_compare, world, dev)
        lca.profile_enable(True)
        for _ in range(min(args.mla_compare, 200)):
            if flush is not None:
                flush.zero_()
            mla_step()
        torch.cuda.synchronize()
        mprof = lca.profile_collect()
        lca.profile_enable(False)
        mattn = mprof.get("attn_decode")
        mla = {"ms_per_step": mla_ms, "attn_ms": mattn[1] / mattn[0] if mattn else None}

    # per-kernel durations (CUDA events around each launch, on its stream)
    prof_steps = min(args.steps, 200)
    lca.profile_enable(True)
    for _ in range(prof_steps):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)

    # end to end through the public API, as a decode loop runs: the cache is
    # state resident on the device (the prefill wrote it), and so are the
    # recent queries, kept as a ring (only their mean is used); every step
    # brings the new token's row (into row L-1 of each sequence) and its
    # query from pinned host memory, puts the query into the ring's oldest
    # slot, decodes, and reads the result back.  Steps are timed one by one,
    # with the L2 flush between them when the cache would otherwise stay in L2.
    pin_row = inp.cache[:, L - 1].contiguous().pin_memory()
    pin_q = inp.q.pin_memory()
    ring = inp.q_recent.to(dev)
    h_out = torch.empty(B, 16, 128, dtype=torch.float32).pin_memory()
    dq = torch.empty_like(pin_q, device=dev)
    h2d = pin_row.numel() * 2 + pin_q.numel() * 2
    d2h = h_out.numel() * 4
    slot = [0]

    def e2e_step():
        cache[:, L - 1].copy_(pin_row, non_blocking=True)
        dq.copy_(pin_q, non_blocking=True)
        ring[:, slot[0]].copy_(dq)
        slot[0] = (slot[0] + 1) % ring.shape[1]
        decode(ring, dq)
        h_out.copy_(out, non_blocking=True)

    for _ in range(3):
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
    assert torch.equal(h_out, out.cpu())

    # the same loop with each step captured once in a CUDA graph (one graph
    # per ring slot: the slot a step writes is part of the step) and replayed:
    # the copies and launches of a step go to the GPU in one call
    graph_ms = None
    if not args.no_e2e_graph:
        def graph_step(sl):
            cache[:, L - 1].copy_(pin_row, non_blocking=True)
            dq.copy_(pin_q, non_blocking=True)
            ring[:, sl].copy_(dq)
            decode(ring, dq, st=None)
            h_out.copy_(out, non_blocking=True)

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
        barrier()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        for i, (a_, b_) in enumerate(gev):
            if flush is not None:
                flush.zero_()
            a_.record(stream)
            graphs[i % len(graphs)].replay()
            b_.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in gev) / n_e2e, world, dev)
        assert torch.equal(h_out, out.cpu())
        del graphs

    # for reference: the same step with the whole cache and all recent
    # queries copied in from the host
    full_ms = None
    if args.e2e_full_copy and not variant:
        pin_cache = inp.cache.pin_memory()
        pin = [t.pin_memory() for t in (inp.q_recent, inp.q)]
        dbuf = [torch.empty_like(t, device=dev) for t in pin]
        dcache = torch.empty_like(pin_cache, device=dev)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(args.e2e_full_copy):
            dcache.copy_(pin_cache, non_blocking=True)
            for d, h in zip(dbuf, pin):
                d.copy_(h, non_blocking=True)
            lca.lca_decode(dcache, dbuf[0], dbuf[1], w_uv, scale=inp.scale, out=out, ws=ws)
            h_out.copy_(out, non_blocking=True)
        x1.record(stream)
        torch.cuda.synchronize()
        full_ms = max_over_ranks(x0.elapsed_time(x1) / args.e2e_full_copy, world, dev)
        del dcache, pin_cache
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")

    if rank != 0:
        return
    tokens = B * world
    value = tokens / (ms / 1e3)
    gbs = B * L * ROW_BYTES * world / (ms / 1e3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    if variant:
        # the ablation's step is dominated by the condensation: 16 m history
        # rows read and m representatives written per sequence
        attn = prof.get("condense")
        algo_bytes = B * 17 * lca.num_groups(L) * ROW_BYTES
        traffic = None
        rl_kernel = f"condense ({args.variant})"
    else:
        attn = prof.get("attn_decode")
        algo_bytes = B * L * ROW_BYTES
        traffic = ncu_traffic(args.workload)
        rl_kernel = "attn_decode (fused LCA)"
    attn_ms = attn[1] / attn[0] if attn else None
    achieved = algo_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "B_per_gpu": B, "L": L, "g": 16, "w": 1024,
                   "heads": 16, "d_c": 512, "d_r": 64, "parallelism": f"replicas x{world}",
                   "variant": args.variant,
                   "l2": ("inputs (B*L*1152 B) larger than the 126 MB L2; no flush" if flush is None else
                          "flushed (256 MB write) before every step; steps timed one by one")},
        "cache_gbps": gbs, "cache_frac_of_hbm": gbs / world / peak,
        "cache_frac_of_nominal_8tbs": gbs / world / 8000.0,
        "roofline": {"bound": "hbm", "kernel": rl_kernel,
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None, "traffic": traffic,
                     "algorithmic_bytes_per_launch": algo_bytes,
                     "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / v[0] for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": ("lca_decode" if not variant else "lca_condense + lca_decode_attn") +
                        " in a decode loop: cache and recent-query ring resident on the device; "
                        "per step the new token's row and query in from pinned host memory, out back"},
    }
    if graph_ms is not None:
        line["e2e_graph"] = {
            "value": tokens / (graph_ms / 1e3), "unit": "tokens/s", "ms_per_step": graph_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "the e2e loop with each step (copies in, decode, copy out) captured once as a CUDA "
                    "graph through the same public calls and replayed"}
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
    if world == 1 and not args.no_cpu_baseline:
        tok_s, cores, sample, _ = cpu_baseline(inp, args.cpu_seconds, variant=variant)
        line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)


def run_ours_stored(args, rank, world, local_rank):
    """Stored-representative decode: the representative cache is built once
    (untimed); a step is lca_decode_stored, plus every 16th step the append of
    one group per sequence (the rate at which groups leave the window).  The
    rows a step reads ((m + w') x 1152 B per sequence) fit in L2 at these
    sizes, so L2 is flushed before every step and steps are timed one by one."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca

    torch.cuda.set_device(local_rank)
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

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
    # recent-query ring resident on the device; per step the new token's row
    # (into row L-1) and its query from pinned memory, the query into the
    # ring's oldest slot, every 16th step the append of the group that left
    # the window, the decode, out back; steps timed one by one with the L2
    # flush between them
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
        cache[:, L - 1].copy_(pin_row, non_blocking=True)
        dq.copy_(pin_q, non_blocking=True)
        ring[:, i % ring.shape[1]].copy_(dq)
        if i % 16 == 15 and m > 0:
            lca.lca_condense_append(cache, ring, rep, m - 1, scale=inp.scale, ws=ws, stream=stream)
        lca.lca_decode_stored(cache, rep, dq, w_uv, scale=inp.scale, out=out, ws=ws, stream=stream)
        h_out.copy_(out, non_blocking=True)

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
        return
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
                   "l2": "flushed (256 MB write) before every step; steps timed one by one"},
        "read_gbps": read_bytes * world / (ms / 1e3) / 1e9,
        "kv_rows_read_fraction": rows / L,
        "roofline": {"bound": "hbm", "kernel": "attn_decode (stored representatives)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None, "traffic": None,
                     "algorithmic_bytes_per_launch": read_bytes, "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / prof_steps for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": B * world / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h_out.numel() * 4,
                "note": "decode loop: cache, kept representatives and recent-query ring resident on the "
                        "device; per step the new token's row and query in from pinned host memory (every "
                        "16th step also the append of one group), out back"},
    }
    print(json.dumps(line), flush=True)


def run_ours_varlen(args, rank, world, local_rank):
    """Decode of a ragged batch (lca_decode_varlen): B sequences whose
    lengths are drawn, seeded, uniformly from [L/8, 15L/8] (mean L), held in
    one [B, 15L/8, 576] buffer.  Algorithmic bytes: the rows each sequence
    holds, read once."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca

    torch.cuda.set_device(local_rank)
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
        return
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
    print(json.dumps(line), flush=True)


def run_ours_split(args, rank, world, local_rank):
    """Decode with every sequence's cache split along L over the ranks: rank r
    holds rows shard_bounds(L, world)[r] of the same B sequences; a step is
    its shard record, an all-gather of the records and the merge + W_UV.
    The whole job decodes B tokens per step whatever the rank count."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca
    from mla_latent_space_lca_b200.split_l import shard_bounds, split_l_decode

    torch.cuda.set_device(local_rank)
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if shard_bytes < (256 << 20) else None
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
        return
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
                          "flushed (256 MB write) before every step")},
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
    print(json.dumps(line), flush=True)


def run_ours_prefill(args, rank, world, local_rank):
    """Blockwise prefill of B prompts of L tokens.  Replicas by default (each
    rank its own prompts); with --split-blocks every rank holds the same
    prompt and computes its work-balanced range of query blocks (strong
    scaling, no data-path collective)."""
    import torch.distributed as dist

    import mla_latent_space_lca_b200 as lca
    from mla_latent_space_lca_b200.split_blocks import prefill_block_ranges

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    B, L = wl["B"], wl["L"]
    split = args.split_blocks
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
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark()
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
    for _ in range(min(args.steps, 3)):
        step()
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)

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
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    n_e2e = max(1, min(args.e2e_steps, 3))
    for _ in range(n_e2e):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1) / n_e2e, world, dev)
    # in-run comparison: full causal MLA prefill over the same inputs (the same
    # path with a window covering the whole sequence, so nothing is condensed)
    mla_ms = None
    if args.mla_compare and not split:
        ws_mla = lca.workspace(4, B, L, L, w=L, device=dev)

        def mla_step():
            lca.lca_prefill_block(cache, q, w_uv, 0, L, w=L, scale=inp.scale, out=out, ws=ws_mla,
                                  stream=stream)

        mla_step()
        torch.cuda.synchronize()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(args.mla_compare):
            mla_step()
        m1.record(stream)
        torch.cuda.synchronize()
        mla_ms = max_over_ranks(m0.elapsed_time(m1) / args.mla_compare, world, dev)
        del ws_mla
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    if rank != 0:
        return
    tokens = B * L * (1 if split else world)
    fl = prefill_flops(L, inp.w, qs // 16, (qs + ql) // 16)   # rank 0's blocks
    step_flops = B * sum(fl.values()) * (1 if split else world)
    if split:   # the whole job's flops: every rank's range
        step_flops = B * sum(prefill_flops(L, inp.w).values())
    peak, peak_kind = measured_tensor_peak()
    attn = prof.get("attn_prefill")
    attn_ms = attn[1] / attn[0] if attn else None
    attn_flops_launch = B * fl["attention"] / (attn[0] / min(args.steps, 3)) if attn else None
    achieved = attn_flops_launch / (attn_ms / 1e3) / 1e12 if attn_ms else None
    line = {
        "metric": PREFILL_METRIC, "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "variant": args.variant, "B_per_gpu": B, "L": L, "q_len": L,
                   "g": 16, "w": 1024,
                   "heads": 16, "d_c": 512, "d_r": 64,
                   "parallelism": f"split-blocks x{world}" if split else f"replicas x{world}",
                   "rank0_queries": [qs, qs + ql],
                   "l2": "queries (B*L*16*1152 B) and representatives far larger than the 126 MB L2; no flush"},
        "step_tflops": step_flops / (ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "attn_prefill", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": achieved / peak if achieved else None,
                     "traffic": None, "algorithmic_flops_per_launch": attn_flops_launch,
                     "launch_ms": attn_ms},
        "kernels_ms_per_step": {k: v[1] / min(args.steps, 3) for k, v in prof.items()},
        "gpu_launches": launches,
        "clocks": sampler.summary() if sampler else None,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
    }
    if mla_ms is not None:
        mla_fl = prefill_flops(L, L)
        line["mla_prefill"] = {"ms_per_step": mla_ms, "tokens_per_s": tokens / (mla_ms / 1e3),
                               "speedup_of_lca": mla_ms / ms,
                               "step_tflops": B * sum(mla_fl.values()) / (mla_ms / 1e3) / 1e12}
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        tok_s, cores, sample, _ = prefill_cpu_baseline(inp, 2 * oracle.num_threads(), variant=variant)
        line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    prefill = WORKLOADS[args.workload]["kind"] == "prefill"
    if args.steps is None:
        args.steps = 10 if prefill else 2000
    if args.warmup is None:
        args.warmup = 3 if prefill else 20
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.variant != "lca" and (args.stored or args.varlen or args.split_l):
        raise SystemExit("--variant applies to the plain decode and prefill workloads only")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if prefill:
            fn = run_ours_prefill
        else:
            fn = (run_ours_stored if args.stored else run_ours_split if args.split_l else
                  run_ours_varlen if args.varlen else run_ours)
        fn(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
