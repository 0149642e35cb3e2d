"""GPU parity of the decode split along the cache.

Each shard's record from lca_decode_shard holds o normalised over the shard's
rows and lse2, the base-2 log-sum-exp of the shard's logits. It is checked
against the oracle's shard, and lca_combine_shards's merge of all records
against the unsplit decode. Shards run one after another on one device; the
exchange between devices is a plain all-gather of the records, covered on
CPU by the gloo tests.

Tolerances: o and out take the suite's bar (max-abs 2e-2, mean-abs 2e-3,
relative L2 1e-2). lse2 = M + log2(den): the kernel's denominator sums
attention weights whose relative error is at most the bf16 rounding of 2^-9,
so |d lse2| <= 2^-9 / ln 2 ~ 2.8e-3; the test bounds it at 3e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs
from mla_latent_space_lca_b200.split_l import shard_bounds

from parity import FORCED_RERUNS, check_anchors, compare, lca_decode_reference

pytestmark = pytest.mark.gpu

LSE2_TOL = 3e-3
LOG2E = 1.0 / math.log(2.0)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def run_shards(cache, q_recent, q, L, cuts, with_anchor=True):
    """cuts [0, c1, ..., L] -> (records [n, B*16*513], anchors per shard)."""
    B = cache.shape[0]
    recs = torch.empty(len(cuts) - 1, api.shard_record_floats(B), device="cuda")
    anchors = []
    for s, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
        m_s = max(0, (min(r1, api.num_groups(L) * 16) - r0) // 16)
        anc = torch.full((B, max(m_s, 1)), -1, dtype=torch.int32, device="cuda") if with_anchor else None
        api.lca_decode_shard(cache[:, r0:r1].contiguous(), q_recent, q, L, r0, part=recs[s], anchor=anc)
        anchors.append(None if anc is None else (anc[:, :m_s], r0))
    return recs, anchors


def unpack(recs, B):
    n = recs.shape[0]
    r = recs.double().cpu().numpy()
    return r[:, : B * 16 * 512].reshape(n, B, 16, 512), r[:, B * 16 * 512:].reshape(n, B, 16)


@pytest.mark.parametrize("peak", [1.0, 30.0])
def test_shard_records_and_merge_match_oracle(peak):
    B, L = 2, 4096 + 21                       # m = 193 groups
    inp = make_decode_inputs(B, L, seed=61, peak=peak)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    c, qr, qb, wb = bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q), bf16_bits(inp.w_uv)
    m = api.num_groups(L)
    ol_ref, out_ref, a_ref = oracle.lca_decode(c, qr, qb, wb, 16, 1024, inp.scale)
    score = oracle.lca_condense(c, qr, 16, 1024, inp.scale)["score"]
    balanced = [0] + [b for _, b in shard_bounds(L, 3)]
    # one group alone, a ragged middle run, and the window alone
    ragged = [0, 16, 64 * 16 + 48, m * 16, L]
    for cuts in (balanced, ragged):
        recs, anchors = run_shards(cache, q_recent, q, L, cuts)
        o, lse2 = unpack(recs, B)
        gpu_anchor = np.concatenate([a.cpu().numpy() + r0 for a, r0 in anchors], axis=1)
        nt, n = check_anchors(gpu_anchor, a_ref, score)
        assert nt <= max(2, n // 1000)
        # near-tie flips: every reference is taken with the GPU's anchors
        forced = gpu_anchor if nt else None
        ol_r, out_r = ol_ref, out_ref
        if nt:
            ol_r, out_r, _ = oracle.lca_decode(c, qr, qb, wb, 16, 1024, inp.scale, anchor_in=forced)
            FORCED_RERUNS["calls"] += 1
            FORCED_RERUNS["flips"] += nt
        for s, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
            o_ref, lse_ref, _ = oracle.lca_decode_shard(c, qr, qb, 16, 1024, inp.scale, r0, r1, anchor_in=forced)
            compare(o[s], o_ref, f"shard [{r0},{r1}) o")
            d = np.abs(lse2[s] - lse_ref * LOG2E).max()
            assert d <= LSE2_TOL, f"shard [{r0},{r1}) lse2 off by {d:.3e}"
        ol = torch.empty(B, 16, 512, device="cuda")
        out = api.lca_combine_shards(recs, w_uv, B, o_lat=ol)
        torch.cuda.synchronize()
        compare(ol.cpu().numpy(), ol_r, "merged o_lat")
        compare(out.cpu().numpy(), out_r, "merged out")


def test_one_shard_merge_is_bit_exact_with_decode():
    """A single shard [0, L) runs the fused decode's kernels with the same
    split; merging one record multiplies by exactly 1, so out is identical."""
    B, L = 3, 9000
    inp = make_decode_inputs(B, L, seed=62)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    recs, _ = run_shards(cache, q_recent, q, L, [0, L], with_anchor=False)
    got = api.lca_combine_shards(recs, w_uv, B)
    ref = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


def test_merge_is_order_free():
    B, L = 2, 6000
    inp = make_decode_inputs(B, L, seed=63)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    cuts = [0] + [b for _, b in shard_bounds(L, 4)]
    recs, _ = run_shards(cache, q_recent, q, L, cuts, with_anchor=False)
    a = api.lca_combine_shards(recs, w_uv, B)
    b = api.lca_combine_shards(recs.flip(0).contiguous(), w_uv, B)
    torch.cuda.synchronize()
    torch.testing.assert_close(a, b, rtol=1e-5, atol=1e-6)


def test_million_token_sequence_in_eight_shards():
    """The million-token decode split into the eight shards a split over
    eight devices would hold, against the oracle and the fused decode."""
    B, L = 1, 1 << 20
    inp = make_decode_inputs(B, L, seed=0)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    cuts = [0] + [b for _, b in shard_bounds(L, 8)]
    recs, anchors = run_shards(cache, q_recent, q, L, cuts)
    ol, ol_fused = (torch.empty(B, 16, 512, device="cuda") for _ in range(2))
    out = api.lca_combine_shards(recs, w_uv, B, o_lat=ol)
    fused_anchor = torch.empty(B, api.num_groups(L), dtype=torch.int32, device="cuda")
    fused = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, o_lat=ol_fused, anchor=fused_anchor)
    torch.cuda.synchronize()
    c, qr, qb, wb = bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q), bf16_bits(inp.w_uv)
    gpu_anchor = np.concatenate([a.cpu().numpy() + r0 for a, r0 in anchors], axis=1)
    _, out_ref, _, nt = lca_decode_reference(c, qr, qb, wb, gpu_anchor, inp.scale)
    assert nt <= max(3, gpu_anchor.size // 1000)
    compare(out.cpu().numpy(), out_ref, "8-shard out")
    # against the fused decode: other split points give other reference
    # maxima, so the bf16-rounded attention weights differ at the 2^-9 level
    # (o_lat to that level); out adds each path's own bf16 rounding of o_lat
    a, b = ol.double().cpu().numpy(), ol_fused.double().cpu().numpy()
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 2e-3
    compare(out.cpu().numpy(), fused.cpu().numpy(), "8-shard out vs fused")
    # the fused kernel and the shards condense every group the same way
    assert np.array_equal(gpu_anchor, fused_anchor.cpu().numpy())
