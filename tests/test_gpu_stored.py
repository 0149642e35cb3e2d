"""GPU parity of stored-representative decode (lca_condense_append +
lca_decode_stored, through the C ABI) against the fp64 oracle.

Each group is condensed once, at the decode step where it leaves the window
(cache length w + 16 (j + 1)), with that step's summary query, and kept in a
representative cache; every step then attends [kept representatives ||
window].  Same bar as the other parity tests (tests/parity.py), near-tie
anchor flips included: the outputs are then compared with the oracle re-run
on the GPU's anchors.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200._lib import LCA_ERR_INVALID_ARG, LcaError
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs, make_prefill_inputs

from parity import FORCED_RERUNS, NEAR_TIE, Canaries, compare

pytestmark = pytest.mark.gpu
G = 16


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


class Stream:
    """A decode stream over one fixed set of positions: cache rows and the
    query of every position are known up front; step(L) appends the groups
    that left the window and attends at cache length L."""

    def __init__(self, inp, w, rep_cap):
        self.inp, self.w = inp, w
        self.cache = inp.cache.cuda()
        self.q = inp.q.cuda()
        self.w_uv = inp.w_uv.cuda()
        B = inp.B
        self.rep = torch.full((B, rep_cap, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.anchor = torch.full((B, rep_cap), -1, dtype=torch.int32, device="cuda")
        self.m = 0

    def view(self, L):
        return self.cache[:, :L].contiguous()

    def catch_up(self, L):
        """Append groups one by one at the step each leaves the window."""
        target = api.num_groups(L, G, self.w)
        while self.m < target:
            Lj = self.w + G * (self.m + 1)
            self.append(Lj)

    def append(self, L):
        q_recent = self.q[:, L - G:L].contiguous()
        self.m = api.lca_condense_append(self.view(L), q_recent, self.rep, self.m, w=self.w,
                                         scale=self.inp.scale, anchor=self.anchor)

    def step(self, L):
        if api.num_groups(L, G, self.w) > self.m:
            self.append(L)
        cn = Canaries()
        o_lat = cn.empty((self.inp.B, 16, 512), torch.float32)
        out = cn.empty((self.inp.B, 16, 128), torch.float32)
        api.lca_decode_stored(self.view(L), self.rep, self.q[:, L - 1].contiguous(), self.w_uv,
                              w=self.w, scale=self.inp.scale, out=out, o_lat=o_lat)
        torch.cuda.synchronize()
        cn.check(f"lca_decode_stored L={L}")
        return out, o_lat


def check_step(st, L, out, o_lat):
    inp = st.inp
    c = bf16_bits(inp.cache[:, :L])
    qa = bf16_bits(inp.q[:, :L])
    ol_ref, out_ref, anc_ref = oracle.lca_decode_stored(c, qa, bf16_bits(inp.w_uv), G, st.w, inp.scale)
    torch.cuda.synchronize()
    m = anc_ref.shape[1]
    got = st.anchor[:, :m].cpu().numpy()
    flips = np.argwhere(got != anc_ref)
    for b, j in flips:
        Lj = st.w + G * (j + 1)
        sc = oracle.lca_condense(np.ascontiguousarray(c[:, :Lj]), np.ascontiguousarray(qa[:, Lj - G:Lj]),
                                 G, st.w, inp.scale)["score"][b, j]
        gi = int(got[b, j]) - j * G
        assert 0 <= gi < G, f"anchor outside group ({b}, {j})"
        gap = sc[int(anc_ref[b, j]) - j * G] - sc[gi]
        assert gap <= NEAR_TIE * np.abs(sc).max(), f"anchor mismatch ({b}, {j}) gap {gap}"
    if len(flips):
        ol_ref, out_ref, _ = oracle.lca_decode_stored(c, qa, bf16_bits(inp.w_uv), G, st.w, inp.scale,
                                                      anchor_in=got)
        FORCED_RERUNS["calls"] += 1
        FORCED_RERUNS["flips"] += len(flips)
    compare(out.cpu().numpy(), out_ref, f"stored out L={L}")
    compare(o_lat.cpu().numpy(), ol_ref, f"stored o_lat L={L}")


@pytest.mark.parametrize("w,peak", [(64, 1.0), (100, 30.0)])
def test_stored_stream(w, peak):
    B, L1 = 2, 400
    inp = make_prefill_inputs(B, L1, w=w, seed=500 + w, peak=peak)
    st = Stream(inp, w, rep_cap=32)
    L0 = 200
    st.catch_up(L0 - 1)
    for L in range(L0, L1 + 1):
        out, o_lat = st.step(L)
        if L % 37 == 0 or (L - w) % G == 0 or L == L1:
            check_step(st, L, out, o_lat)


def test_append_from_zero_is_condense_and_stored_is_decode_attn():
    """One append of every group at the current step writes exactly what
    lca_condense writes, and attending them at stride rep_cap gives exactly
    lca_decode_attn's result."""
    B, L = 3, 1024 + 16 * 45 + 7
    inp = make_decode_inputs(B, L, seed=61)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    m = api.num_groups(L)
    rep = api.lca_condense(cache, q_recent, scale=inp.scale)
    cap = m + 13
    rep_s = torch.full((B, cap, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert api.lca_condense_append(cache, q_recent, rep_s, 0, scale=inp.scale) == m
    torch.cuda.synchronize()
    assert torch.equal(rep_s[:, :m].view(torch.int16), rep.view(torch.int16))
    assert torch.isnan(rep_s[:, m:].float()).all()          # capacity rows untouched
    a = api.lca_decode_attn(cache, rep, q, w_uv, scale=inp.scale)
    b = api.lca_decode_stored(cache, rep_s, q, w_uv, scale=inp.scale)   # NaN rows >= m are never read
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_stored_rejects_small_capacity():
    inp = make_decode_inputs(1, 2048, seed=62)
    cache, q_recent = inp.cache.cuda(), inp.q_recent.cuda()
    m = api.num_groups(2048)
    rep = torch.empty(1, m - 1, 576, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(LcaError) as e:
        api.lca_condense_append(cache, q_recent, rep, 0, scale=inp.scale)
    assert e.value.status == LCA_ERR_INVALID_ARG


def test_stored_full_size_128k():
    """L = 131072, w = 1024: the 8128 groups appended one at a time at their
    exit steps, then one stored decode step checked against the oracle."""
    B, L, w = 1, 131072, 1024
    inp = make_prefill_inputs(B, L, w=w, seed=7)
    st = Stream(inp, w, rep_cap=api.num_groups(L, G, w))
    st.catch_up(L)
    out, o_lat = st.step(L)
    check_step(st, L, out, o_lat)
