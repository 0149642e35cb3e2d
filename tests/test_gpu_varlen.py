"""GPU parity of the ragged-batch decode (lca_decode_varlen): every sequence
of the batch has its own length and is decoded as lca_decode decodes it
alone.

The cache buffer holds the longest length. Rows past each sequence's own
length are filled with NaN, so a single one of them reaching the result
would show. Checks:

- against the oracle, sequence by sequence, on its own rows: out, o_lat and
  anchors, with the suite's bar;
- equal lengths reproduce lca_decode bit for bit;
- g = 1 is MLA decode of each sequence's rows;
- a batch with more sequences than SMs and lengths from 1 to 3000 matches
  the single-sequence GPU calls;
- the stored-representative mode (lca_decode_stored_varlen), with NaN in the
  representative cache past each sequence's groups.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs

from parity import Canaries, compare, lca_decode_reference

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def ragged(inp, lens):
    """The batch's cache on the device, rows past each length set to NaN."""
    cache = inp.cache.clone()
    for b, n in enumerate(lens):
        cache[b, n:].view(torch.int16).fill_(NAN_BF16)
    return cache.cuda()


def run(inp, lens, g=16, w=1024):
    B, L = inp.B, inp.L
    cache = ragged(inp, lens)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    m = api.num_groups(L, 16, w) if g != 1 else 0
    cn = Canaries()
    anchor = cn.empty((B, max(m, 1)), torch.int32)
    anchor.fill_(-1)
    o_lat = cn.empty((B, 16, 512), torch.float32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode_varlen(cache, lens_d, inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda(), g=g, w=w,
                          scale=inp.scale, out=out, o_lat=o_lat, anchor=anchor if g != 1 else None)
    torch.cuda.synchronize()
    cn.check("lca_decode_varlen")
    return out.cpu().numpy(), o_lat.cpu().numpy(), anchor.cpu().numpy()[:, :m]


@pytest.mark.parametrize("w", [1024, 64])
def test_ragged_batch_matches_oracle_per_sequence(w):
    L = 9000
    lens = [1, 1000, 1024, 1040, 5013, 9000, 63, 64 * 50 + 17]
    inp = make_decode_inputs(len(lens), L, seed=101, peak=10.0)
    out, o_lat, anchor = run(inp, lens, w=w)
    for b, n in enumerate(lens):
        c = bf16_bits(inp.cache[b:b + 1, :n])
        qr, qb, wb = bf16_bits(inp.q_recent[b:b + 1]), bf16_bits(inp.q[b:b + 1]), bf16_bits(inp.w_uv)
        mb = oracle.num_groups(n, 16, w)
        ol_ref, out_ref, _, _ = lca_decode_reference(c, qr, qb, wb, anchor[b:b + 1, :mb], inp.scale, w=w)
        compare(o_lat[b:b + 1], ol_ref, f"o_lat seq {b} (len {n})")
        compare(out[b:b + 1], out_ref, f"out seq {b} (len {n})")


def test_equal_lengths_reproduce_lca_decode():
    B, L = 4, 9000
    inp = make_decode_inputs(B, L, seed=102)
    out, o_lat, anchor = run(inp, [L] * B)
    m = api.num_groups(L)
    ref_anchor = torch.empty(B, m, dtype=torch.int32, device="cuda")
    ref_olat = torch.empty(B, 16, 512, device="cuda")
    ref = api.lca_decode(inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda(), scale=inp.scale,
                         o_lat=ref_olat, anchor=ref_anchor)
    torch.cuda.synchronize()
    assert np.array_equal(out, ref.cpu().numpy())
    assert np.array_equal(o_lat, ref_olat.cpu().numpy())
    assert np.array_equal(anchor, ref_anchor.cpu().numpy())


def test_ragged_mla():
    L = 5000
    lens = [1, 77, 4096, 5000, 2500]
    inp = make_decode_inputs(len(lens), L, seed=103)
    out, o_lat, _ = run(inp, lens, g=1)
    for b, n in enumerate(lens):
        c = bf16_bits(inp.cache[b:b + 1, :n])
        ol_ref, out_ref = oracle.mla_decode(c, bf16_bits(inp.q[b:b + 1]), bf16_bits(inp.w_uv), inp.scale)
        compare(out[b:b + 1], out_ref, f"mla out seq {b} (len {n})")
        compare(o_lat[b:b + 1], ol_ref, f"mla o_lat seq {b} (len {n})")


def test_many_sequences_match_single_calls():
    B, L = 300, 3000
    rng = np.random.default_rng(104)
    lens = [int(x) for x in rng.integers(1, L + 1, size=B)]
    lens[:4] = [1, L, 1024, 1040]
    inp = make_decode_inputs(B, L, seed=104)
    out, o_lat, _ = run(inp, lens)
    w_uv = inp.w_uv.cuda()
    for b, n in enumerate(lens):
        ol1 = torch.empty(1, 16, 512, device="cuda")
        one = api.lca_decode(inp.cache[b:b + 1, :n].cuda(), inp.q_recent[b:b + 1].cuda(), inp.q[b:b + 1].cuda(),
                             w_uv, scale=inp.scale, o_lat=ol1)
        torch.cuda.synchronize()
        a, r = o_lat[b].astype(np.float64), ol1[0].double().cpu().numpy()
        # other split points give other reference maxima: each side rounds
        # its attention weights to bf16 (2^-9 relative) independently
        assert np.linalg.norm(a - r) / np.linalg.norm(r) <= 2.0 ** -8, (b, n)
        compare(out[b:b + 1], one.cpu().numpy(), f"seq {b} (len {n}) vs its own call")


def test_ragged_stored_decode():
    """Stored representatives for a ragged batch: each sequence's groups are
    appended by a call on its own views (as a decode loop does when its
    length crosses a group boundary); rows of the representative cache past
    each sequence's groups hold NaN."""
    L = 6000
    lens = [1, 900, 1040, 3017, 6000, 2222]
    B = len(lens)
    inp = make_decode_inputs(B, L, seed=105, peak=10.0)
    cache = ragged(inp, lens)
    q_recent, q, w_uv = inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    cap = api.num_groups(L) + 7
    rep = torch.empty(B, cap, 576, dtype=torch.bfloat16, device="cuda")
    rep.view(torch.int16).fill_(NAN_BF16)
    for b, n in enumerate(lens):
        if api.num_groups(n) > 0:
            api.lca_condense_append(cache[b:b + 1, :n], q_recent[b:b + 1], rep[b:b + 1], 0, scale=inp.scale)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o_lat = torch.empty(B, 16, 512, device="cuda")
    out = api.lca_decode_stored_varlen(cache, rep, lens_d, q, w_uv, scale=inp.scale, o_lat=o_lat)
    torch.cuda.synchronize()
    for b, n in enumerate(lens):
        mb = api.num_groups(n)
        c = bf16_bits(inp.cache[b:b + 1, :n])
        rep_bits = rep[b:b + 1, :mb].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        ol_ref, out_ref = oracle.lca_attend_reps(c, rep_bits, bf16_bits(inp.q[b:b + 1]), bf16_bits(inp.w_uv), 16,
                                                 1024, inp.scale)
        compare(o_lat[b:b + 1].cpu().numpy(), ol_ref, f"stored o_lat seq {b} (len {n})")
        compare(out[b:b + 1].cpu().numpy(), out_ref, f"stored out seq {b} (len {n})")
        one = api.lca_decode_stored(cache[b:b + 1, :n], rep[b:b + 1], q[b:b + 1], w_uv, scale=inp.scale)
        torch.cuda.synchronize()
        compare(out[b:b + 1].cpu().numpy(), one.cpu().numpy(), f"stored seq {b} vs its own call")


@pytest.mark.parametrize("g", [16, 1])
def test_fewer_tiles_than_ctas(g):
    """A ragged batch whose whole tile list is shorter than the grid: CTAs
    that own no tile write no partial slot, and the merge must skip them."""
    L = 1200
    lens = [5, 700, 1100, 64, 1200]
    inp = make_decode_inputs(len(lens), L, seed=106, peak=10.0)
    out, o_lat, _ = run(inp, lens, g=g)
    for b, n in enumerate(lens):
        c = bf16_bits(inp.cache[b:b + 1, :n])
        qb, wb = bf16_bits(inp.q[b:b + 1]), bf16_bits(inp.w_uv)
        if g == 1:
            ol_ref, out_ref = oracle.mla_decode(c, qb, wb, inp.scale)
        else:
            ol_ref, out_ref, _ = oracle.lca_decode(c, bf16_bits(inp.q_recent[b:b + 1]), qb, wb, 16, 1024, inp.scale)
        compare(o_lat[b:b + 1], ol_ref, f"o_lat seq {b} (len {n})")
        compare(out[b:b + 1], out_ref, f"out seq {b} (len {n})")
