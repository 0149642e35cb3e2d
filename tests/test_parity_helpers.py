"""Host-side checks of the GPU suites' parity helpers (no GPU): the guard
regions around output buffers catch a one-byte write on either side of the
body for every dtype the outputs use, and the near-tie rule accepts a flip
only inside its tolerance."""
import numpy as np
import pytest
import torch

from parity import NEAR_TIE, Canaries, check_anchors


@pytest.mark.parametrize("shape,dtype", [((3, 5), torch.float32), ((7,), torch.bfloat16),
                                         ((2, 3), torch.int32), ((0, 4), torch.float32)])
def test_canaries_catch_writes_outside_the_body(shape, dtype):
    for side in ("head", "tail"):
        cn = Canaries(guard_bytes=1024)
        t = cn.empty(shape, dtype, device="cpu")
        t.zero_()
        cn.check("clean")
        raw, n, _ = cn.bufs[0]
        pos = 1023 if side == "head" else 1024 + n
        raw[pos] ^= 1
        with pytest.raises(AssertionError):
            cn.check(side)


def test_unwritten_float_output_reads_nan():
    cn = Canaries(guard_bytes=256)
    t = cn.empty((4,), torch.float32, device="cpu")
    assert torch.isnan(t).all()


def test_near_tie_rule():
    score = np.zeros((1, 1, 16))
    score[0, 0, :] = np.linspace(0.0, 1.0, 16)
    score[0, 0, 14] = 1.0 - 0.5 * NEAR_TIE        # within the rule of the maximum at 15
    assert check_anchors(np.array([[14]]), np.array([[15]]), score) == (1, 1)
    score[0, 0, 14] = 1.0 - 2.0 * NEAR_TIE
    with pytest.raises(AssertionError):
        check_anchors(np.array([[14]]), np.array([[15]]), score)
    with pytest.raises(AssertionError):          # outside its group
        check_anchors(np.array([[16]]), np.array([[15]]), score)
