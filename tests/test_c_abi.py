"""The C ABI used from C: tests/c_abi/decode_from_c.c drives liblca_b200.so
with plain cudaMalloc'd pointers, sizes the workspace with
lca_workspace_bytes, checks two rejected calls and runs one lca_decode step.

On CPU the program must compile and link against include/lca.h and the
library. On a GPU its output must equal the Python binding's on the same
inputs, bit for bit: the same kernels with the same arguments."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "c_abi"))
from c_abi_build import build  # noqa: E402


def test_c_consumer_compiles_and_links():
    exe = build()
    assert os.access(exe, os.X_OK)


@pytest.mark.gpu
def test_c_consumer_matches_python_binding():
    from mla_latent_space_lca_b200 import api
    from mla_latent_space_lca_b200.inputs import bf16_bits, make_decode_inputs
    exe = build()
    B, L = 3, 5000
    inp = make_decode_inputs(B, L, seed=111, peak=10.0)
    d = os.path.join(HERE, "c_abi", "_build", "io")
    os.makedirs(d, exist_ok=True)
    for name, t in (("cache", inp.cache), ("q_recent", inp.q_recent), ("q", inp.q), ("w_uv", inp.w_uv)):
        bf16_bits(t).tofile(os.path.join(d, name + ".bin"))
    r = subprocess.run([exe, str(B), str(L), d], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    got = np.fromfile(os.path.join(d, "out.bin"), dtype=np.float32).reshape(B, 16, 128)
    ref = api.lca_decode(inp.cache.cuda(), inp.q_recent.cuda(), inp.q.cuda(), inp.w_uv.cuda(),
                         scale=inp.scale).cpu().numpy()
    torch.cuda.synchronize()
    assert np.array_equal(got, ref)
