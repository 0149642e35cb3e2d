"""Shared pieces of the benchmark: peaks, clock sampling, DRAM traffic from
the committed ncu summaries, the oracle's CPU baselines, timing helpers and
the workload config dict (one function, so both arms print the same one)."""
from __future__ import annotations

import hashlib
import json
import os
import statistics
import subprocess
import threading
import time

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mla_latent_space_lca_b200", "csrc")
ROW_BYTES = 576 * 2
METRIC = "LCA decode tokens/s and cache-read GB/s (fraction of B200 HBM roofline)"
PREFILL_METRIC = "LCA blockwise prefill tokens/s (fraction of B200 bf16 tensor roofline)"
PROFILE_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
# lca_params.variant: the method and the two ablations of the page's ablation table
VARIANTS = {"lca": 0, "pool_position": 1, "sparse": 2}
# kernel sources whose hash keys a committed DRAM-traffic figure
KERNEL_SOURCES = {
    "attn_decode": ("attn_decode.cuh", "common.cuh"),
    "attn_prefill": ("prefill.cuh", "common.cuh"),
}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def measured_tensor_peak():
    """Sustained bf16 GEMM peak (a kernel timed inside a long step)."""
    p = _peaks()
    if "bf16_tflops_sustained" in p:
        return float(p["bf16_tflops_sustained"]), "measured (sustained)"
    return 1400.0, "fallback (sustained)"


def measured_hbm_peak():
    p = _peaks()
    if "hbm_gbs" in p:
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


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


def source_hash(kernel: str = "attn_decode") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str = "attn_decode"):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary (profiles/ncu_traffic.json), if it was taken on the current
    kernel source; None otherwise."""
    try:
        with open(PROFILE_FILE) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("kernel", "attn_decode") != kernel or e.get("source_hash") != source_hash(kernel):
            return None
        return e["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


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


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class L2Flush:
    """Evicts every input from the 126 MB L2 between timed steps: writes a
    256 MB buffer, then reads another 256 MB buffer, so that the L2 is left
    holding clean lines of that second buffer.  (After the write alone the
    L2 is full of dirty lines, and the next step would pay for writing the
    flush buffer back to HBM as its own reads evict them.)"""

    BYTES = 256 << 20

    def __init__(self, dev):
        self.w = torch.empty(self.BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(self.BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def zero_(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)

    NOTE = ("flushed before every step (256 MB written, then another 256 MB read, so the L2 holds "
            "none of the inputs and no dirty lines); steps timed one by one")


def time_steps(step, n: int, stream, flush=None) -> float:
    """Milliseconds per step over n steps with CUDA events on `stream`:
    back to back, or (flush given) one by one after an L2 flush."""
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / n


def kernel_profile(lca, step, n: int, flush=None) -> dict:
    """Per-kernel {name: (launches, total ms)} over n steps (CUDA events the
    library records around each of its launches, on the call's stream)."""
    lca.profile_enable(True)
    for _ in range(n):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = lca.profile_collect()
    lca.profile_enable(False)
    return prof


def flush_buffer(nbytes_inputs: int, dev):
    """An L2 flush (L2Flush) between steps when the inputs would otherwise
    stay in the 126 MB L2; None when they are larger."""
    return L2Flush(dev) if nbytes_inputs < (256 << 20) else None


def decode_config(workload: str, B: int, L: int, world: int, variant: str = "lca", flushed: bool = False):
    """The `config` dict of a decode line (both arms)."""
    return {"workload": workload, "B_per_gpu": B, "L": L, "g": 16, "w": 1024,
            "heads": 16, "d_c": 512, "d_r": 64, "parallelism": f"replicas x{world}",
            "variant": variant,
            "l2": (L2Flush.NOTE if flushed else "inputs (B*L*1152 B) larger than the 126 MB L2; no flush")}


def prefill_config(workload: str, B: int, L: int, world: int, variant: str = "lca", split: bool = False,
                   q_range=None):
    """The `config` dict of a prefill line (both arms)."""
    c = {"workload": workload, "variant": variant, "B_per_gpu": B, "L": L, "q_len": L,
         "g": 16, "w": 1024, "heads": 16, "d_c": 512, "d_r": 64,
         "parallelism": f"split-blocks x{world}" if split else f"replicas x{world}",
         "l2": "queries (B*L*16*1152 B) far larger than the 126 MB L2; no flush"}
    if q_range is not None:
        c["rank0_queries"] = list(q_range)
    return c


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
    return tok_s, oracle.num_threads(), sample, times


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


def device_ok(lca):
    rc, detail = lca.device_status(clear=True)
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
