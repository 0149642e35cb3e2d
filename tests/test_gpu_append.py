"""lca_append_token (a decode loop's per-step bookkeeping in one launch)
against torch's own indexed assignment, bit for bit: the new rows land in
row `pos` of a pitched cache view, the queries in one slot of the ring,
nothing else changes, and a decode call right after sees them."""
import pytest
import torch

from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import make_decode_inputs

pytestmark = pytest.mark.gpu


def rand_bf16(*shape, gen):
    return torch.randn(*shape, generator=gen).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,L_max,L,g,slot", [(3, 200, 150, 16, 5), (8, 64, 64, 16, 15), (1, 10, 1, 4, 0)])
def test_append_matches_indexed_assignment(B, L_max, L, g, slot):
    gen = torch.Generator().manual_seed(B * 1000 + L)
    buf = rand_bf16(B, L_max, 576, gen=gen)
    ring = rand_bf16(B, g, 16, 576, gen=gen)
    rows = rand_bf16(B, 576, gen=gen)
    q = rand_bf16(B, 16, 576, gen=gen)
    want_buf, want_ring = buf.clone(), ring.clone()
    want_buf[:, L - 1] = rows
    want_ring[:, slot] = q
    api.lca_append_token(buf[:, :L], L - 1, rows, q=q, ring=ring, slot=slot)
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), want_buf.view(torch.int16))
    assert torch.equal(ring.view(torch.int16), want_ring.view(torch.int16))
    # rows only
    rows2 = rand_bf16(B, 576, gen=gen)
    want_buf[:, 0] = rows2
    api.lca_append_token(buf[:, :L], 0, rows2)
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), want_buf.view(torch.int16))


def test_decode_after_append_sees_the_new_token():
    B, L = 4, 5000
    inp = make_decode_inputs(B, L, seed=91)
    base = inp.cache.cuda()
    ring0 = inp.q_recent.cuda()
    gen = torch.Generator().manual_seed(92)
    rows = rand_bf16(B, 576, gen=gen)
    q = (torch.randn(B, 16, 576, generator=gen) / 24).to(torch.bfloat16).cuda()
    w_uv = inp.w_uv.cuda()
    # by hand
    c1, r1 = base.clone(), ring0.clone()
    c1[:, L - 1] = rows
    r1[:, 3] = q
    ref = api.lca_decode(c1, r1, q, w_uv, scale=inp.scale)
    # through the helper, issued right before the decode on the same stream
    c2, r2 = base.clone(), ring0.clone()
    api.lca_append_token(c2, L - 1, rows, q=q, ring=r2, slot=3)
    got = api.lca_decode(c2, r2, q, w_uv, scale=inp.scale)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


def test_append_reads_pinned_host_memory_in_place():
    """rows and q straight from pinned host memory (no copy), with the second
    copy of q for the decode: the same bytes as indexed assignment."""
    B, L_max, L, g, slot = 5, 300, 257, 16, 9
    gen = torch.Generator().manual_seed(7)
    buf = rand_bf16(B, L_max, 576, gen=gen)
    ring = rand_bf16(B, g, 16, 576, gen=gen)
    h_rows = torch.randn(B, 576, generator=gen).to(torch.bfloat16).pin_memory()
    h_q = torch.randn(B, 16, 576, generator=gen).to(torch.bfloat16).pin_memory()
    q_out = torch.zeros(B, 16, 576, dtype=torch.bfloat16, device="cuda")
    want_buf, want_ring = buf.clone(), ring.clone()
    want_buf[:, L - 1] = h_rows.cuda()
    want_ring[:, slot] = h_q.cuda()
    api.lca_append_token(buf[:, :L], L - 1, h_rows, q=h_q, ring=ring, slot=slot, q_out=q_out)
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), want_buf.view(torch.int16))
    assert torch.equal(ring.view(torch.int16), want_ring.view(torch.int16))
    assert torch.equal(q_out.cpu().view(torch.int16), h_q.view(torch.int16))


def test_decode_writes_out_into_pinned_host_memory():
    """out in pinned host memory, written in place by the tail: bit-identical
    to out on the device, for the fused step and for plain MLA."""
    B, L = 3, 4000
    inp = make_decode_inputs(B, L, seed=93)
    cache, qr, q, w_uv = (t.cuda() for t in (inp.cache, inp.q_recent, inp.q, inp.w_uv))
    ref = api.lca_decode(cache, qr, q, w_uv, scale=inp.scale)
    h_out = torch.full((B, 16, 128), float("nan")).pin_memory()
    api.lca_decode(cache, qr, q, w_uv, scale=inp.scale, out=h_out)
    torch.cuda.synchronize()
    assert torch.equal(h_out, ref.cpu())
    ref_m = api.mla_decode_attn(cache, q, w_uv, inp.scale)
    h_out.fill_(float("nan"))
    api.mla_decode_attn(cache, q, w_uv, inp.scale, out=h_out)
    torch.cuda.synchronize()
    assert torch.equal(h_out, ref_m.cpu())


def test_pageable_host_memory_is_refused_before_launch():
    """A pageable host buffer is refused by the binding, and by the C entry
    point's own pointer check (nothing is launched)."""
    import ctypes

    from mla_latent_space_lca_b200 import _lib
    B, L = 2, 64
    cache = torch.zeros(B, L, 576, dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros(B, 576, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        api.lca_append_token(cache, L - 1, pageable)
    n0 = api.launch_count()
    rc = _lib.lib().lca_append_token(ctypes.c_void_p(pageable.data_ptr()), ctypes.c_void_p(cache.data_ptr()), B, L,
                                     L - 1, None, None, 0, 0, None, None)
    assert rc == _lib.LCA_ERR_INVALID_ARG
    assert api.launch_count() == n0
    torch.cuda.synchronize()
    assert torch.count_nonzero(cache) == 0
