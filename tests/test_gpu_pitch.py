"""A cache held as rows 0 .. L-1 of each sequence of a preallocated
[B, L_max, 576] buffer (lca_params.cache_pitch = L_max, derived by the
binding from the view buf[:, :L]).

Every entry point must give bit-identical results to the packed cache. The
kernels see the same rows through their tensor maps, so nothing may differ.
Rows L .. L_max-1 are filled with NaN, so a single read past a sequence's
end would turn the outputs into NaN. The packed runs are themselves checked
against the oracle in test_gpu_decode, test_gpu_stored, test_gpu_prefill and
test_gpu_split_l."""
import pytest
import torch

from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import make_decode_inputs, make_prefill_inputs
from mla_latent_space_lca_b200.split_l import shard_bounds

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def in_buffer(cache, extra):
    """The cache as the first L rows of each sequence of a NaN-filled buffer."""
    B, L, D = cache.shape
    buf = torch.empty(B, L + extra, D, dtype=torch.bfloat16, device="cuda")
    buf.view(torch.int16).fill_(NAN_BF16)
    buf[:, :L] = cache
    view = buf[:, :L]
    assert not view.is_contiguous()
    return view


def dev(inp):
    return inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()


def test_fused_decode_and_mla():
    inp = make_decode_inputs(3, 5000, seed=81, peak=10.0)
    cache, q_recent, q, w_uv = dev(inp)
    view = in_buffer(cache, 777)
    m = api.num_groups(5000)
    res = []
    for c in (cache, view):
        anchor = torch.full((3, m), -1, dtype=torch.int32, device="cuda")
        o_lat = torch.empty(3, 16, 512, device="cuda")
        out = api.lca_decode(c, q_recent, q, w_uv, scale=inp.scale, o_lat=o_lat, anchor=anchor)
        mla = api.mla_decode_attn(c, q, w_uv, inp.scale)
        res.append((out, o_lat, anchor, mla))
    torch.cuda.synchronize()
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_condense_attend_and_stored():
    inp = make_decode_inputs(2, 3000 + 9, seed=82)
    cache, q_recent, q, w_uv = dev(inp)
    view = in_buffer(cache, 130)
    m = api.num_groups(3009)
    res = []
    for c in (cache, view):
        anchor = torch.full((2, m), -1, dtype=torch.int32, device="cuda")
        rep = api.lca_condense(c, q_recent, scale=inp.scale, anchor=anchor)
        two = api.lca_decode_attn(c, rep, q, w_uv, scale=inp.scale)
        kept = torch.zeros(2, m + 40, 576, dtype=torch.bfloat16, device="cuda")
        api.lca_condense_append(c, q_recent, kept, 0, scale=inp.scale)
        stored = api.lca_decode_stored(c, kept, q, w_uv, scale=inp.scale)
        res.append((rep, anchor, two, kept, stored))
    torch.cuda.synchronize()
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_growing_cache_in_one_buffer():
    """A decode loop over one preallocated buffer: at each length L the
    result equals the packed decode of the first L rows."""
    L0, steps, L_max = 1024 + 16 * 20 + 3, 40, 1024 + 16 * 40
    inp = make_decode_inputs(4, L0 + steps, seed=83)
    full, q_recent, q, w_uv = dev(inp)
    buf = torch.empty(4, L_max, 576, dtype=torch.bfloat16, device="cuda")
    buf.view(torch.int16).fill_(NAN_BF16)
    ws = api.workspace(3, 4, L_max)
    for L in range(L0, L0 + steps):
        buf[:, L - 1 if L > L0 else 0: L] = full[:, L - 1 if L > L0 else 0: L]   # append the new row(s)
        got = api.lca_decode(buf[:, :L], q_recent, q, w_uv, scale=inp.scale, ws=ws).clone()
        ref = api.lca_decode(full[:, :L].contiguous(), q_recent, q, w_uv, scale=inp.scale)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), L


def test_shards_as_views_of_one_cache():
    """Split-L shards passed as views of one cache (no copies) match shards
    copied out to packed buffers."""
    inp = make_decode_inputs(2, 4096 + 21, seed=84)
    cache, q_recent, q, w_uv = dev(inp)
    L = cache.shape[1]
    view = in_buffer(cache, 100)
    cuts = [0] + [b for _, b in shard_bounds(L, 3)]
    recs = []
    for src, copy in ((cache, True), (view, False)):
        r = torch.empty(3, api.shard_record_floats(2), device="cuda")
        for s, (r0, r1) in enumerate(zip(cuts[:-1], cuts[1:])):
            piece = src[:, r0:r1].contiguous() if copy else src[:, r0:r1]
            api.lca_decode_shard(piece, q_recent, q, L, r0, scale=inp.scale, part=r[s])
        recs.append(r)
    torch.cuda.synchronize()
    assert torch.equal(recs[0], recs[1])


def test_prefill():
    inp = make_prefill_inputs(2, 2048, seed=85)
    cache, q, w_uv = inp.cache.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    view = in_buffer(cache, 64)
    outs = [api.lca_prefill_block(c, q, w_uv, 0, 2048, w=256, scale=inp.scale) for c in (cache, view)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
