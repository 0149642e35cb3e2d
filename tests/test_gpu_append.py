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
