"""Decode steps inside a CUDA graph.

Every library call is a set of asynchronous launches on the caller's stream,
with no allocation and no synchronisation. The launches carry the
programmatic-dependent-launch attribute. A step captured once into a graph
therefore replays with the eager result, and replays after the inputs are
rewritten in place follow the new inputs.

The first call on a device does one-time host setup (device attributes,
kernel attributes, the tensor-map encoder), so each test makes an eager call
before capturing.
"""
import pytest
import torch

from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import make_decode_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def _inputs(seed, B=4, L=9000):
    inp = make_decode_inputs(B, L, seed=seed)
    return inp, [t.cuda() for t in (inp.cache, inp.q_recent, inp.q, inp.w_uv)]


@pytest.mark.parametrize("path", ["fused", "stored", "mla"])
def test_step_replays_in_a_cuda_graph(path):
    inp, (cache, q_recent, q, w_uv) = _inputs(91)
    inp2, (cache2, q_recent2, q2, _) = _inputs(92)
    B, L = inp.B, inp.L
    m = api.num_groups(L)
    ws = api.workspace(3, B, L)
    out = torch.empty(B, 16, 128, device="cuda")
    rep = torch.zeros(B, m, 576, dtype=torch.bfloat16, device="cuda")

    def step():
        if path == "fused":
            api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, out=out, ws=ws)
        elif path == "stored":
            api.lca_condense_append(cache, q_recent, rep, 0, scale=inp.scale, ws=ws)
            api.lca_decode_stored(cache, rep, q, w_uv, scale=inp.scale, out=out, ws=ws)
        else:
            api.mla_decode_attn(cache, q, w_uv, inp.scale, out=out, ws=ws)

    step()                                       # eager, before any capture
    torch.cuda.synchronize()
    ref1 = out.clone()
    cache.copy_(cache2), q_recent.copy_(q_recent2), q.copy_(q2)
    step()
    torch.cuda.synchronize()
    ref2 = out.clone()
    cache.copy_(inp.cache), q_recent.copy_(inp.q_recent), q.copy_(inp.q)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref1)
    # rewrite the inputs in place: the replay follows them
    cache.copy_(cache2), q_recent.copy_(q_recent2), q.copy_(q2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref2)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref2)
    del g
