"""The C-ABI library loads, exports every entry point include/lca.h declares,
and rejects invalid arguments on the host before touching the GPU (these
tests run without a GPU: only argument checks are exercised)."""
import ctypes
import os
import re

import pytest

from mla_latent_space_lca_b200 import _lib
from mla_latent_space_lca_b200._lib import LcaParams

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "lca.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)) - {"sizeof"})


def test_exports_every_declared_symbol(lcalib):
    declared = header_functions()
    assert set(declared) == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lcalib, name), name


def test_num_groups(lcalib, ora):
    for L, g, w in [(4096, 16, 1024), (32768, 16, 1024), (1039, 16, 1024), (1040, 16, 1024),
                    (100, 16, 1024), (1 << 20, 16, 1024), (77, 1, 5), (1, 16, 0)]:
        assert lcalib.lca_num_groups(L, LcaParams(g, w, 0.1)) == ora.num_groups(L, g, w)
    assert lcalib.lca_num_groups(100, LcaParams(0, 1, 0.1)) == 0


def test_workspace_bytes(lcalib):
    p = LcaParams(16, 1024, 0.07)
    for op in range(4):
        n = lcalib.lca_workspace_bytes(op, 32, 32768, 0, p)
        assert n > 0 and n % 256 == 0
    assert lcalib.lca_workspace_bytes(0, 0, 32768, 0, p) == 0
    assert lcalib.lca_workspace_bytes(99, 1, 10, 0, p) == 0


def test_strerror(lcalib):
    for s in range(0, -8, -1):
        assert _lib.strerror(s)
    assert "unknown" in _lib.strerror(-100)


# fake, never-dereferenced device addresses: argument checks fail first
A = 0x7F0000000000


def call_decode(lcalib, **kw):
    args = dict(cache=A, q_recent=A, q=A, w_uv=A, B=2, L=4096, p=LcaParams(16, 1024, 0.07),
                out=A, o_lat=None, anchor=None, ws=A, ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return lcalib.lca_decode(args["cache"], args["q_recent"], args["q"], args["w_uv"], args["B"],
                             args["L"], args["p"], args["out"], args["o_lat"], args["anchor"],
                             args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(cache=None), _lib.LCA_ERR_INVALID_ARG),
    (dict(out=None), _lib.LCA_ERR_INVALID_ARG),
    (dict(q_recent=None), _lib.LCA_ERR_INVALID_ARG),
    (dict(B=0), _lib.LCA_ERR_INVALID_ARG),
    (dict(L=0), _lib.LCA_ERR_INVALID_ARG),
    (dict(L=1 << 31), _lib.LCA_ERR_INVALID_ARG),
    (dict(p=LcaParams(16, -1, 0.07)), _lib.LCA_ERR_INVALID_ARG),
    (dict(p=LcaParams(16, 1024, 0.0)), _lib.LCA_ERR_INVALID_ARG),
    (dict(p=LcaParams(16, 1024, float("nan"))), _lib.LCA_ERR_INVALID_ARG),
    (dict(p=LcaParams(8, 1024, 0.07)), _lib.LCA_ERR_UNSUPPORTED),
    (dict(p=LcaParams(16, 1024, 0.07, 3)), _lib.LCA_ERR_INVALID_ARG),
    (dict(p=LcaParams(16, 1024, 0.07, _lib.VARIANT_SPARSE)), _lib.LCA_ERR_UNSUPPORTED),
    (dict(p=LcaParams(16, 1024, 0.07, _lib.VARIANT_POOL_POSITION)), _lib.LCA_ERR_UNSUPPORTED),
    (dict(cache=A + 8), _lib.LCA_ERR_MISALIGNED),
    (dict(o_lat=A + 4), _lib.LCA_ERR_MISALIGNED),
    (dict(anchor=A + 2), _lib.LCA_ERR_MISALIGNED),
    (dict(ws=None), _lib.LCA_ERR_WORKSPACE),
    (dict(ws_bytes=1024), _lib.LCA_ERR_WORKSPACE),
    (dict(ws=A + 64), _lib.LCA_ERR_MISALIGNED),
])
def test_decode_rejects_bad_arguments(lcalib, kw, status):
    assert call_decode(lcalib, **kw) == status


def test_other_entry_points_reject_bad_arguments(lcalib):
    p = LcaParams(16, 1024, 0.07)
    big = 1 << 30
    assert lcalib.mla_decode_attn(None, A, A, 1, 10, 0.1, A, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.mla_decode_attn(A, A, A, 1, 10, -1.0, A, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.mla_decode_attn(A, A, A, 1, 10, 0.1, A, None, A, 10, None) == _lib.LCA_ERR_WORKSPACE
    assert lcalib.lca_condense(A, A, 1, 4096, LcaParams(4, 1024, 0.1), A, None, None, A, big, None) == _lib.LCA_ERR_UNSUPPORTED
    assert lcalib.lca_condense(A, A, 1, 4096, p, None, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_condense(A, A, 1, 4096, p, A + 2, None, None, A, big, None) == _lib.LCA_ERR_MISALIGNED
    assert lcalib.lca_decode_attn(A, None, A, A, 1, 4096, p, A, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_decode_attn(A, A, A, A, 1, 4096, p, A, None, A, 16, None) == _lib.LCA_ERR_WORKSPACE
    # stored representatives: capacity below m, j0 past m
    assert lcalib.lca_condense_append(A, A, 1, 4096, p, 0, A, 100, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_condense_append(A, A, 1, 4096, p, 193, A, 192, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_decode_stored(A, A, 100, A, A, 1, 4096, p, A, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    # ablation variants: the no-alloc decode condenses on the fly, so it
    # refuses them (prefill accepts them); an unknown variant is refused
    pv = LcaParams(16, 1024, 0.07, _lib.VARIANT_SPARSE)
    assert lcalib.lca_decode_noalloc(A, A, A, A, 1, 4096, pv, A, None, None, None) == _lib.LCA_ERR_UNSUPPORTED
    bad = LcaParams(16, 1024, 0.07, 3)
    assert lcalib.lca_prefill_block(A, A, A, 1, 4096, 0, 4096, bad, A, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    # prefill size limits: L beyond 2^27, and 2^31 blocks over the batch
    assert lcalib.lca_prefill_block(A, A, A, 1, (1 << 27) + 16, 0, 16, p, A, None, None, A, big, None) == _lib.LCA_ERR_UNSUPPORTED
    assert lcalib.lca_prefill_block(A, A, A, 1 << 8, 1 << 27, 0, 1 << 27, p, A, None, None, A, big, None) == _lib.LCA_ERR_UNSUPPORTED
    # prefill range checks: unaligned start, past the end
    assert lcalib.lca_prefill_block(A, A, A, 1, 4096, 8, 16, p, A, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_prefill_block(A, A, A, 1, 4096, 4080, 32, p, A, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG


def test_varlen_rejects_bad_arguments(lcalib):
    p = LcaParams(16, 1024, 0.07)
    big = 1 << 30

    def call(**kw):
        a = dict(cache=A, lens=A, q_recent=A, q=A, w_uv=A, B=2, L=4096, p=p, out=A, ws_bytes=big)
        a.update(kw)
        return lcalib.lca_decode_varlen(a["cache"], a["lens"], a["q_recent"], a["q"], a["w_uv"], a["B"], a["L"],
                                        a["p"], a["out"], None, None, A, a["ws_bytes"], None)
    assert call(lens=None) == _lib.LCA_ERR_INVALID_ARG
    assert call(q_recent=None) == _lib.LCA_ERR_INVALID_ARG
    assert call(lens=A + 2) == _lib.LCA_ERR_MISALIGNED
    assert call(p=LcaParams(8, 1024, 0.07)) == _lib.LCA_ERR_UNSUPPORTED
    assert call(p=LcaParams(16, 1024, 0.07, _lib.VARIANT_SPARSE)) == _lib.LCA_ERR_UNSUPPORTED
    assert call(B=1 << 17, L=1 << 20) == _lib.LCA_ERR_UNSUPPORTED     # tile offsets past 2^31
    assert call(ws_bytes=16) == _lib.LCA_ERR_WORKSPACE
    if not __import__("torch").cuda.is_available():
        assert call() == _lib.LCA_ERR_NO_DEVICE
        assert call(q_recent=None, p=LcaParams(1, 0, 0.07)) == _lib.LCA_ERR_NO_DEVICE


def test_cache_pitch_is_checked(lcalib):
    big = 1 << 30
    bad = [LcaParams(16, 1024, 0.07, 0, 4000),          # pitch below L = 4096
           LcaParams(16, 1024, 0.07, 0, -1),            # negative
           LcaParams(16, 1024, 0.07, 0, 1 << 39)]       # B * pitch beyond 2^40
    for p in bad:
        assert call_decode(lcalib, p=p) == _lib.LCA_ERR_INVALID_ARG
        assert lcalib.lca_condense(A, A, 2, 4096, p, A, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
        assert lcalib.lca_decode_attn(A, A, A, A, 2, 4096, p, A, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
        assert lcalib.lca_prefill_block(A, A, A, 2, 4096, 0, 16, p, A, None, None, A, big, None) == _lib.LCA_ERR_INVALID_ARG
    assert lcalib.lca_workspace_bytes(3, 2, 4096, 0, LcaParams(16, 1024, 0.07, 0, -5)) == 0
    if not __import__("torch").cuda.is_available():
        # a valid pitch gets as far as the device check
        assert call_decode(lcalib, p=LcaParams(16, 1024, 0.07, 0, 5000)) == _lib.LCA_ERR_NO_DEVICE
        assert call_decode(lcalib, p=LcaParams(1, 0, 0.07, 0, 5000)) == _lib.LCA_ERR_NO_DEVICE


def test_shard_entry_points_reject_bad_arguments(lcalib):
    p = LcaParams(16, 1024, 0.07)
    big = 1 << 30
    L = 4096 + 21            # m = 193 groups: history rows 0 .. 3087

    def shard(row0, Ls, **kw):
        a = dict(cache=A, q_recent=A, q=A, B=1, L=L, p=p, part=A, ws_bytes=big)
        a.update(kw)
        return lcalib.lca_decode_shard(a["cache"], a["q_recent"], a["q"], a["B"], a["L"], row0, Ls,
                                       a["p"], a["part"], None, A, a["ws_bytes"], None)
    INV = _lib.LCA_ERR_INVALID_ARG
    assert shard(8, 16) == INV                      # not at a group boundary
    assert shard(0, 24) == INV                      # ends inside a group
    assert shard(3088 - 16, 32) == INV              # runs into the window without reaching L
    assert shard(3104, L - 3104) == INV             # starts inside the window
    assert shard(0, L + 16) == INV                  # past the end
    assert shard(0, 0) == INV                       # empty
    assert shard(0, 16, q_recent=None) == INV       # groups need the summary query
    assert shard(0, 16, part=None) == INV
    assert shard(0, 16, part=A + 4) == _lib.LCA_ERR_MISALIGNED
    assert shard(0, 16, ws_bytes=16) == _lib.LCA_ERR_WORKSPACE
    assert shard(0, 16, p=LcaParams(8, 1024, 0.07)) == _lib.LCA_ERR_UNSUPPORTED
    assert lcalib.lca_combine_shards(A, 0, 1, A, A, None, None) == INV
    assert lcalib.lca_combine_shards(None, 2, 1, A, A, None, None) == INV
    assert lcalib.lca_combine_shards(A, 2, 1, A, A + 8, None, None) == _lib.LCA_ERR_MISALIGNED
    if not __import__("torch").cuda.is_available():
        # a valid window-only last shard needs no summary query and gets as far as the device
        assert shard(3088, L - 3088, q_recent=None) == _lib.LCA_ERR_NO_DEVICE


def test_valid_call_without_gpu_reports_no_device(lcalib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call_decode(lcalib) == _lib.LCA_ERR_NO_DEVICE


def test_binding_functions_reference_only_defined_globals():
    """Every global name the Python binding's functions load exists (the
    binding cannot reach a GPU here, so a misspelt or missing name would
    otherwise only show on a device)."""
    import builtins
    import dis
    import types

    from mla_latent_space_lca_b200 import api, split_blocks, split_l

    def code_objects(co):
        yield co
        for c in co.co_consts:
            if isinstance(c, types.CodeType):
                yield from code_objects(c)

    missing = []
    for mod in (api, _lib, split_l, split_blocks):
        for name, fn in vars(mod).items():
            if not isinstance(fn, types.FunctionType) or fn.__module__ != mod.__name__:
                continue
            for co in code_objects(fn.__code__):
                for ins in dis.get_instructions(co):
                    if ins.opname == "LOAD_GLOBAL":
                        g = ins.argval
                        if g not in vars(mod) and not hasattr(builtins, g):
                            missing.append(f"{mod.__name__}.{name}: {g}")
    assert not missing, missing


def test_append_token_rejects_bad_arguments(lcalib):
    f = lcalib.lca_append_token
    ok = dict(rows=A, cache=A, B=2, pitch=100, pos=99, q=A, ring=A, g=16, slot=15, q_dst=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["rows"], a["cache"], a["B"], a["pitch"], a["pos"], a["q"], a["ring"], a["g"], a["slot"],
                 a["q_dst"], None)

    inval = _lib.LCA_ERR_INVALID_ARG
    # valid arguments on the fake address: no device on a host without a GPU;
    # with one, the address is refused by the pointer check before any launch
    nodev = inval if __import__("torch").cuda.is_available() else _lib.LCA_ERR_NO_DEVICE
    assert call(rows=None) == inval
    assert call(cache=None) == inval
    assert call(B=0) == inval
    assert call(pos=100) == inval and call(pos=-1) == inval
    assert call(q=None) == inval                      # q and ring come together
    assert call(slot=16) == inval and call(slot=-1) == inval and call(g=0) == inval
    assert call(pitch=1 << 40, pos=0) == inval        # B * pitch must stay below 2^40
    assert call(rows=A + 8) == _lib.LCA_ERR_MISALIGNED
    assert call(ring=A + 4) == _lib.LCA_ERR_MISALIGNED
    assert call(q_dst=A + 4) == _lib.LCA_ERR_MISALIGNED
    assert call(q=None, ring=None, g=0, slot=0, q_dst=A) == inval   # a second copy of no query
    # the second copy of q: valid arguments
    assert call(q_dst=A) == nodev
    # rows only (no ring): valid arguments
    assert call(q=None, ring=None, g=0, slot=0) == nodev
