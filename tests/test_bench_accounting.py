"""The benchmark's algorithmic work counts, on the CPU.

The roofline fractions divide these counts by measured kernel times, so they
are pinned here:
- against closed forms;
- against the work split of the multi-device prefill, a second
  implementation;
- against the magnitudes worked out for the 128K prefill from the method's
  definition: rep attention ~1.84e13 flops, window ~4.7e12, condensation
  ~1.15e12, W_UV ~2.7e11.
"""
import types

import pytest

from mla_latent_space_lca_b200.inputs import WORKLOADS
from mla_latent_space_lca_b200.split_blocks import block_flops


@pytest.fixture(scope="module")
def bench():
    from benchmarks import common
    ns = types.SimpleNamespace(**{k: getattr(common, k) for k in dir(common) if not k.startswith("_")})
    ns.WORKLOADS = WORKLOADS
    return ns


PER_KEY = 16 * (576 + 512) * 2        # 16 heads, q.k over 576 and p.v over 512


def test_prefill_without_history_is_causal_attention(bench):
    """w >= L: nothing is condensed, and query t attends t + 1 rows."""
    L = 256
    f = bench.prefill_flops(L, w=L)
    assert f["condense"] == 0
    assert f["attention"] == L * (L + 1) // 2 * PER_KEY
    assert f["wuv"] == L * 16 * 512 * 128 * 2


def test_prefill_single_block_after_the_window(bench):
    """Block k = cw + 3 (w = 32, so cw = 2): m = 3 groups condensed, 48
    history rows scored and pooled; each of the block's 16 queries attends 3
    representatives plus the window from row 48 to itself."""
    w, k = 32, 5
    f = bench.prefill_flops(16 * (k + 1), w=w, k0=k, k1=k + 1)
    m = 3
    keys = sum(m + (16 * k + tt - 16 * m + 1) for tt in range(16))
    assert f["attention"] == keys * PER_KEY
    assert f["condense"] == 16 * m * (576 + 512) * 2


@pytest.mark.parametrize("L,w", [(131072, 1024), (4096, 1000), (1600, 0)])
def test_prefill_counts_match_the_device_split(bench, L, w):
    f = bench.prefill_flops(L, w)
    assert sum(f.values()) == sum(block_flops(k, w=w) for k in range(L // 16))


def test_prefill_128k_magnitudes(bench):
    f = bench.prefill_flops(131072, 1024)
    assert f["attention"] == pytest.approx(1.84e13 + 4.7e12, rel=0.02)
    assert f["condense"] == pytest.approx(1.15e12, rel=0.02)
    assert f["wuv"] == pytest.approx(2.7e11, rel=0.02)


def test_decode_workloads(bench):
    """The decode workloads: B x L cached rows of 1152 B, about 1.208 GB for
    the three long ones."""
    for name in ("decode_b32_l32k", "decode_b8_l128k", "decode_b1_l1m"):
        wl = bench.WORKLOADS[name]
        assert wl["kind"] == "decode"
        assert wl["B"] * wl["L"] * bench.ROW_BYTES == 1207959552
    assert bench.ROW_BYTES == 1152
    assert set(bench.VARIANTS) == {"lca", "pool_position", "sparse"}


@pytest.mark.parametrize("variant", [0, 1, 2])
def test_cpu_baseline_runs_each_variant(bench, variant):
    """The oracle baselines the benchmark times (its reference arm too) run
    for the method and both ablations, on a tiny decode and prefill."""
    from mla_latent_space_lca_b200.inputs import make_decode_inputs, make_prefill_inputs
    inp = make_decode_inputs(2, 1100, seed=3)
    tok_s, cores, sample, times = bench.cpu_baseline(inp, 0, steps=1, seqs=2, variant=variant)
    assert tok_s > 0 and cores >= 1 and len(times) == 1 and "2 of 2 sequences" in sample
    pre = make_prefill_inputs(1, 1024, w=128, seed=4)
    tok_s, _, sample, times = bench.prefill_cpu_baseline(pre, 4, steps=1, variant=variant)
    assert tok_s > 0 and len(times) == 1


def test_both_arms_print_the_same_config():
    """The reference arm's config dict is built by the same function as the
    GPU arm's, for every workload of the default suite."""
    import bench as entry
    from benchmarks import common
    for wl in (entry.HEADLINE,) + entry.SUITE:
        spec = WORKLOADS[wl]
        if spec["kind"] == "decode":
            flushed = spec["B"] * spec["L"] * common.ROW_BYTES < (256 << 20)
            a = common.decode_config(wl, spec["B"], spec["L"], 1, "lca", flushed)
            assert a["workload"] == wl and a["B_per_gpu"] == spec["B"] and a["L"] == spec["L"]
            assert not flushed
        else:
            a = common.prefill_config(wl, spec["B"], spec["L"], 1, "lca", False, (0, spec["L"]))
            assert a["rank0_queries"] == [0, spec["L"]]


def test_default_run_arguments():
    import bench as entry
    a = entry.parse([])
    assert a.workload is None and entry.defaults(a, entry.HEADLINE) == (2000, 20)
    assert entry.defaults(a, "prefill_b1_l128k") == (10, 3)
    a = entry.parse(["--steps", "7", "--warmup", "4"])
    assert entry.defaults(a, entry.HEADLINE) == (7, 4)
