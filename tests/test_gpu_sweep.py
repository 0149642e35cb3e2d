"""GPU parity over a seeded sweep of shapes, and concurrent use.

The sweep draws batch sizes, window sizes w (0, 17, 64, 1024), group counts
and ragged tails around the group, tile and window boundaries, and query
scales (flat to peaked). For each shape three paths are checked against the
fp64 oracle:

- the fused decode (lca_decode): out, o_lat and anchors;
- plain MLA decode (mla_decode_attn);
- condense, then attention over the stored representatives
  (lca_condense -> lca_decode_attn). The oracle attends the GPU's own bf16
  representative rows, so the two steps are checked separately.

Same bar as test_gpu_decode.

Concurrency: decodes of different batches on two CUDA streams, and from two
host threads, each with its own workspace, give bit-identical results to the
same calls run alone. The kernels use no atomics, and the split-L partition
depends only on the shapes.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs

from parity import Canaries, compare, lca_decode_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.device_status(clear=True)
    yield
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {rc} detail {detail:#x}"


def sweep_cases(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for k in range(n):
        w = int(rng.choice([0, 17, 64, 1024]))
        B = int(rng.integers(1, 5))
        if rng.random() < 0.85:
            L = max(1, w + 16 * int(rng.integers(0, 200)) + int(rng.integers(0, 16)))
        else:                       # shorter than the window: nothing condensed
            L = int(rng.integers(1, max(2, w + 1)))
        peak = float(rng.choice([1.0, 10.0, 30.0]))
        cases.append((B, L, w, peak, 1000 + k))
    # edges the draw may miss: nothing condensed, an empty window (w = 0 and
    # L a multiple of g), a single group and nothing else
    cases += [(2, 1024, 1024, 1.0, 1100), (3, 500, 1024, 10.0, 1101), (2, 160, 0, 1.0, 1102),
              (1, 16, 0, 30.0, 1103), (2, 17, 17, 1.0, 1104), (2, 64 * 37, 0, 10.0, 1105)]
    return cases


@pytest.mark.parametrize("B,L,w,peak,seed", sweep_cases())
def test_sweep_parity(B, L, w, peak, seed):
    inp = make_decode_inputs(B, L, seed=seed, peak=peak)
    cache, q_recent, q, w_uv = inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda()
    c, qr, qb, wb = bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q), bf16_bits(inp.w_uv)
    m = api.num_groups(L, 16, w)
    assert m == oracle.num_groups(L, 16, w)
    cn = Canaries()
    anchor = cn.empty((B, m), torch.int32)
    o_lat = cn.empty((B, 16, 512), torch.float32)
    out = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode(cache, q_recent, q, w_uv, w=w, scale=inp.scale, out=out, o_lat=o_lat, anchor=anchor)
    mla = cn.empty((B, 16, 128), torch.float32)
    api.mla_decode_attn(cache, q, w_uv, inp.scale, out=mla)
    rep = cn.empty((B, m, 576), torch.bfloat16)
    api.lca_condense(cache, q_recent, w=w, scale=inp.scale, rep=rep)
    two = cn.empty((B, 16, 128), torch.float32)
    api.lca_decode_attn(cache, rep if m > 0 else None, q, w_uv, w=w, scale=inp.scale, out=two)
    torch.cuda.synchronize()
    cn.check("sweep")

    ol_ref, out_ref, _, nt = lca_decode_reference(c, qr, qb, wb, anchor.cpu().numpy(), inp.scale, w=w)
    compare(o_lat.cpu().numpy(), ol_ref, "fused o_lat")
    compare(out.cpu().numpy(), out_ref, "fused out")
    assert nt <= max(2, B * m // 1000)
    _, mla_ref = oracle.mla_decode(c, qb, wb, inp.scale)
    compare(mla.cpu().numpy(), mla_ref, "mla out")
    rep_bits = rep.view(torch.int16).cpu().numpy().view(np.uint16)
    _, two_ref = oracle.lca_attend_reps(c, rep_bits, qb, wb, 16, w, inp.scale)
    compare(two.cpu().numpy(), two_ref, "condense -> attend out")


def _setup(B, L, seed):
    inp = make_decode_inputs(B, L, seed=seed)
    t = dict(cache=inp.cache.cuda(), q_recent=inp.q_recent.cuda(), q=inp.q.cuda(), w_uv=inp.w_uv.cuda(),
             scale=inp.scale, B=B, L=L)
    t["ws"] = api.workspace(3, B, L)
    t["out"] = torch.empty(B, 16, 128, device="cuda")
    return t


def _run(t, stream=None):
    return api.lca_decode(t["cache"], t["q_recent"], t["q"], t["w_uv"], scale=t["scale"], out=t["out"],
                          ws=t["ws"], stream=stream)


def test_two_streams_concurrently():
    a, b = _setup(4, 20000, 71), _setup(3, 9000, 72)
    ref_a, ref_b = _run(a).clone(), _run(b).clone()
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    for _ in range(5):
        with torch.cuda.stream(s1):
            _run(a, stream=s1)
        with torch.cuda.stream(s2):
            _run(b, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(a["out"], ref_a)
    assert torch.equal(b["out"], ref_b)


def test_two_host_threads():
    a, b = _setup(2, 15000, 73), _setup(5, 4000, 74)
    ref = [_run(a).clone(), _run(b).clone()]
    torch.cuda.synchronize()
    errors = []

    def worker(t, r):
        try:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.default_stream())
            with torch.cuda.stream(s):
                for _ in range(10):
                    _run(t, stream=s)
            s.synchronize()
            if not torch.equal(t["out"], r):
                errors.append("mismatch")
        except Exception as e:  # surfaced below
            errors.append(repr(e))

    th = [threading.Thread(target=worker, args=(a, ref[0])), threading.Thread(target=worker, args=(b, ref[1]))]
    for x in th:
        x.start()
    for x in th:
        x.join(timeout=120)
    assert not errors, errors
