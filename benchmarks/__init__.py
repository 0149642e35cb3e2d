"""Measurement of the hot path, split by workload kind; bench.py at the
repository root is the entry point.

  common    peaks, clock sampling, per-kernel DRAM traffic from the committed
            ncu summaries, the oracle's CPU baselines, timing helpers
  decode    the fused decode step (and its in-run comparisons and
            end-to-end loops)
  prefill   the blockwise prefill
  modes     stored-representative, ragged-batch and split-L decode
  reference the reference arm: the CPU oracle on the same workload
"""
