"""Failure detection without a GPU fault: a kernel whose bounded wait can
never be satisfied must give up after the library's wait limit, report
LCA_ERR_DEVICE_TIMEOUT with its kernel id and wait site in the device status
word, and leave the context usable for the next call."""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_space_lca_b200 import _lib, api
from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    assert torch.cuda.is_available()
    api.device_status(clear=True)
    assert _lib.lib().lca_selftest_wait_timeout(None) == _lib.LCA_OK
    rc, detail = api.device_status(clear=True)
    assert rc == _lib.LCA_ERR_DEVICE_TIMEOUT
    assert detail & 0xFF == 1                  # error class: wait timeout
    assert (detail >> 8) & 0xFF == 8           # kernel id of the self-test
    assert (detail >> 16) & 0xFF == 1          # wait site
    # the status word is clear again and the next real call is correct
    rc, detail = api.device_status(clear=False)
    assert rc == _lib.LCA_OK and detail == 0
    inp = make_decode_inputs(2, 2048 + 21, seed=71)
    out = api.lca_decode(inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda(),
                         scale=inp.scale)
    torch.cuda.synchronize()
    _, ref, _ = oracle.lca_decode(bf16_bits(inp.cache), bf16_bits(inp.q_recent), bf16_bits(inp.q),
                                  bf16_bits(inp.w_uv), 16, 1024, inp.scale)
    got = out.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() <= 2e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-2
    assert api.device_status(clear=True)[0] == _lib.LCA_OK
