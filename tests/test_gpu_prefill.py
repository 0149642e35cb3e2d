"""GPU parity of the blockwise LCA prefill (lca_prefill_block, through the C
ABI) against the fp64 CPU oracle on the same seeded inputs.

Same bar as the decode tests: outputs (out and o_lat) within max-abs 2e-2,
mean-abs 2e-3 and relative L2 1e-2 of fp64; anchors bit-exact except where
the oracle's own fp64 scores put the GPU's pick within 1e-4 * max|s| of the
group maximum.  The oracle evaluates a subset of blocks where the full range
would take it too long (blocks are independent given the cache); the subsets
always include the first and last blocks, the blocks around the window edge,
the 128-block condense tiles and the 256-block chunks of the GPU path.
Where a near-tie anchor went the other way on the GPU, the outputs are
compared with the oracle re-run on the GPU's anchors (forced-anchor mode).
Output buffers carry guard regions that must stay untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_prefill_inputs

from parity import Canaries, FORCED_RERUNS, compare, prefill_anchor_check

pytestmark = pytest.mark.gpu
G = 16


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def run_gpu(inp, q_start, q_len, w, variant=oracle.LCA, canaries=True):
    cache, q, w_uv = inp.cache.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    B = inp.B
    m_last = oracle.num_groups(q_start + q_len - G, G, w)
    cn = Canaries() if canaries else None
    alloc = cn.empty if cn else (lambda shape, dt: torch.empty(shape, dtype=dt, device="cuda"))
    anchor = alloc((B, q_len // G, max(m_last, 1)), torch.int32)
    anchor.fill_(-1)
    o_lat = alloc((B, q_len, 16, 512), torch.float32)
    out = alloc((B, q_len, 16, 128), torch.float32)
    api.lca_prefill_block(cache, q, w_uv, q_start, q_len, w=w, out=out, o_lat=o_lat, anchor=anchor,
                          variant=variant)
    torch.cuda.synchronize()
    if cn:
        cn.check("lca_prefill_block")
    return out, o_lat, anchor


def check_prefill(inp, q_start, q_len, w, blocks=None, gpu=None, variant=oracle.LCA, max_flip_frac=0.01):
    """Compare the GPU prefill of [q_start, q_start+q_len) with the oracle on
    `blocks` (absolute block indices; None = all).  At most max_flip_frac of
    the groups may be near-tie anchor flips (None: no bound, for inputs with
    planted ties).  Returns the number of flips."""
    out, o_lat, anchor = gpu if gpu is not None else run_gpu(inp, q_start, q_len, w, variant)
    k0 = q_start // G
    if blocks is None:
        blocks = list(range(k0, k0 + q_len // G))
    blocks = sorted(set(int(k) for k in blocks))
    cache_b, q_b = bf16_bits(inp.cache), bf16_bits(inp.q)
    ol_ref, out_ref, anc_ref = oracle.lca_prefill(cache_b, q_b, bf16_bits(inp.w_uv), q_start, q_len, G, w,
                                                  inp.scale, blocks=blocks, want_anchor=True, variant=variant)
    anc = anchor.cpu().numpy()
    n_bad, n_all = prefill_anchor_check(cache_b, q_b, w, inp.scale, k0, blocks, anc, anc_ref)
    if max_flip_frac is not None:
        assert n_bad <= max(1, int(n_all * max_flip_frac)), f"{n_bad} near-tie anchor flips of {n_all}"
    if n_bad:
        # two valid results: compare with the oracle run on the GPU's anchors
        forced = np.where(anc < 0, 0, anc)
        ol_ref, out_ref, _ = oracle.lca_prefill(cache_b, q_b, bf16_bits(inp.w_uv), q_start, q_len, G, w,
                                                inp.scale, blocks=blocks, variant=variant, anchor_in=forced)
        FORCED_RERUNS["calls"] += 1
        FORCED_RERUNS["flips"] += n_bad
    rows = np.concatenate([np.arange((k - k0) * G, (k - k0 + 1) * G) for k in blocks])
    rows_t = torch.as_tensor(rows, device="cuda")
    compare(out.index_select(1, rows_t).cpu().numpy(), out_ref[:, rows], "prefill out")
    compare(o_lat.index_select(1, rows_t).cpu().numpy(), ol_ref[:, rows], "prefill o_lat")
    return n_bad


@pytest.mark.parametrize("B,L,w,q_start,q_len,peak", [
    (1, 1024, 128, 0, 1024, 1.0),          # one rep tile, several window tiles
    (2, 1024 + 7, 100, 0, 1024, 1.0),      # w not a multiple of 16, cache longer than the range
    (1, 512, 1024, 0, 512, 1.0),           # every block inside the window: causal MLA
    (1, 640, 0, 0, 640, 1.0),              # w = 0: window is the block itself
    (2, 2000, 200, 16 * 40, 16 * 37, 30.0),  # mid-sequence range, peaked queries
    (1, 64, 16, 48, 16, 1.0),              # a single block
])
def test_prefill_small(B, L, w, q_start, q_len, peak):
    inp = make_prefill_inputs(B, L, w=w, seed=300 + L + w, peak=peak)
    check_prefill(inp, q_start, q_len, w)


@pytest.mark.parametrize("B", [1, 2])
def test_prefill_tiles_and_chunks(B):
    """More than one condense block tile (128 blocks), several representative
    tiles per block and two 256-block chunks per sequence; sampled blocks."""
    L, w = 16 * 300, 256
    inp = make_prefill_inputs(B, L, w=w, seed=41 + B)
    blocks = [0, 1, 15, 16, 17, 30, 127, 128, 129, 200, 255, 256, 257, 298, 299]
    check_prefill(inp, 0, L, w, blocks=blocks)


def test_prefill_peaked_anchors():
    """Queries x30 make pooling and anchors far from uniform."""
    B, L, w = 2, 16 * 160, 512
    inp = make_prefill_inputs(B, L, w=w, seed=43, peak=30.0)
    check_prefill(inp, 0, L, w, blocks=[31, 32, 33, 64, 100, 127, 128, 158, 159])


@pytest.mark.parametrize("variant", [oracle.POOL_POSITION, oracle.SPARSE])
def test_prefill_ablations(variant):
    """The two ablations of the page's ablation table: the RoPE key pooled
    with the latent's weights, or the anchor token's whole row.  Peaked
    queries make the weights far from uniform; the blocks span two condense
    block tiles, several representative tiles and the window edge."""
    B, L, w = 2, 16 * 300, 256
    inp = make_prefill_inputs(B, L, w=w, seed=44, peak=30.0)
    check_prefill(inp, 0, L, w, blocks=[0, 15, 16, 17, 60, 127, 128, 129, 255, 256, 299], variant=variant)


@pytest.mark.parametrize("variant", [oracle.POOL_POSITION, oracle.SPARSE])
def test_prefill_ablations_ragged_window_mid_range(variant):
    """The ablations with a window that is not a multiple of 16, a range
    that starts mid-sequence and a cache longer than the range."""
    B, L, w = 1, 16 * 90 + 5, 100
    inp = make_prefill_inputs(B, L, w=w, seed=45, peak=30.0)
    check_prefill(inp, 16 * 20, 16 * 70, w, variant=variant)


def test_prefill_range_split_consistency():
    """Two calls over adjacent ranges give the rows of one call over both."""
    B, L, w = 1, 16 * 96, 256
    inp = make_prefill_inputs(B, L, w=w, seed=47)
    full, _, _ = run_gpu(inp, 0, L, w, canaries=False)
    a, _, _ = run_gpu(inp, 0, 16 * 40, w, canaries=False)
    b, _, _ = run_gpu(inp, 16 * 40, L - 16 * 40, w, canaries=False)
    torch.testing.assert_close(torch.cat([a, b], dim=1), full, rtol=0, atol=0)


def test_prefill_split_over_ranks_by_work():
    """The work-balanced ranges a split over three devices would take (with
    chunk edges inside them) give, concatenated, the rows of one call."""
    from mla_latent_space_lca_b200.split_blocks import prefill_block_ranges
    B, L, w = 2, 16 * 700, 512
    inp = make_prefill_inputs(B, L, w=w, seed=48)
    full, _, _ = run_gpu(inp, 0, L, w, canaries=False)
    parts = [run_gpu(inp, qs, ql, w, canaries=False)[0] for qs, ql in prefill_block_ranges(L, 3, w=w)]
    torch.testing.assert_close(torch.cat(parts, dim=1), full, rtol=0, atol=0)


def test_prefill_full_size_sampled():
    """The 128K-token prefill (B = 1, L = 131072, w = 1024) in one call, the
    launch configuration the benchmark times; the oracle checks sampled
    blocks: the first, the window edge, chunk edges and the last ones."""
    B, L, w = 1, 131072, 1024
    inp = make_prefill_inputs(B, L, w=w, seed=0)
    gpu = run_gpu(inp, 0, L, w)
    nb = L // G
    blocks = [0, 63, 64, 65, 255, 256, 4095, 4096, nb - 2, nb - 1]
    check_prefill(inp, 0, L, w, blocks=blocks, gpu=gpu)
