"""lca_decode_noalloc: the decode step for callers that cannot allocate device
memory (no cudaMalloc, no caller workspace).  It runs the same kernels with
the same scratch layout as lca_decode, so its results must be bit-identical
to lca_decode with a caller-provided workspace, call after call, although
every call reuses the library's one built-in scratch array.  The largest
batch runs first, so the later, smaller calls sit on top of stale non-zero
scratch: a call that read a slot before writing it would differ.

Kept in a file of its own that pytest collects last; it also passes when run
alone in a fresh process."""
import ctypes

import pytest
import torch

from mla_latent_space_lca_b200 import _lib, api
from mla_latent_space_lca_b200.inputs import make_decode_inputs

pytestmark = pytest.mark.gpu


def _noalloc(lib, cache, q_recent, q, w_uv, scale, out, o_lat, anchor):
    B, L, _ = cache.shape
    p = _lib.LcaParams(16, 1024, float(scale))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.lca_decode_noalloc(ctypes.c_void_p(cache.data_ptr()), ctypes.c_void_p(q_recent.data_ptr()),
                                  ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w_uv.data_ptr()), B, L, p,
                                  ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(o_lat.data_ptr()),
                                  ctypes.c_void_p(anchor.data_ptr()), stream)


def test_noalloc_matches_workspace_path_on_consecutive_calls(lcalib):
    assert torch.cuda.is_available()
    api.device_status(clear=True)
    big = make_decode_inputs(_lib.NOALLOC_MAX_BATCH, 3000, seed=32, peak=8.0)
    cases = [big, make_decode_inputs(4, 5000, seed=31), make_decode_inputs(2, 1100, seed=30), big]
    for n, inp in enumerate(cases):
        cache, q_recent, q, w_uv = (t.cuda() for t in (inp.cache, inp.q_recent, inp.q, inp.w_uv))
        B, L = inp.B, inp.L
        m = api.num_groups(L)
        out = torch.empty(B, 16, 128, device="cuda")
        o_lat = torch.empty(B, 16, 512, device="cuda")
        anchor = torch.empty(B, m, dtype=torch.int32, device="cuda")
        rc = _noalloc(lcalib, cache, q_recent, q, w_uv, inp.scale, out, o_lat, anchor)
        assert rc == _lib.LCA_OK, _lib.strerror(rc)
        ref_olat = torch.empty_like(o_lat)
        ref_anchor = torch.empty_like(anchor)
        ref = api.lca_decode(cache, q_recent, q, w_uv, scale=inp.scale, o_lat=ref_olat, anchor=ref_anchor)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all() and torch.isfinite(o_lat).all()
        assert torch.equal(out, ref), f"out, call {n}"
        assert torch.equal(o_lat, ref_olat), f"o_lat, call {n}"
        assert torch.equal(anchor, ref_anchor), f"anchor, call {n}"
    rc, detail = api.device_status(clear=True)
    assert rc == 0, f"device status {detail:#x}"


def test_noalloc_rejects_batches_beyond_its_scratch(lcalib):
    B = _lib.NOALLOC_MAX_BATCH + 1
    inp = make_decode_inputs(B, 1100, seed=33)
    cache, q_recent, q, w_uv = (t.cuda() for t in (inp.cache, inp.q_recent, inp.q, inp.w_uv))
    out = torch.empty(B, 16, 128, device="cuda")
    o_lat = torch.empty(B, 16, 512, device="cuda")
    anchor = torch.empty(B, 5, dtype=torch.int32, device="cuda")
    rc = _noalloc(lcalib, cache, q_recent, q, w_uv, inp.scale, out, o_lat, anchor)
    assert rc == _lib.LCA_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.strerror(rc)
