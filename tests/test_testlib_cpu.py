"""CPU checks of the GPU tests' helpers: the grouped token-tile numbering and the NVFP4 byte
comparison, which must reject a quantiser with a planted mistake and accept decisions that sit on a
rounding midpoint only within its stated tolerance."""
import numpy as np
import pytest

from lmoe_testlib import check_act_bytes, grouped_tiles
from oracle import nvfp4 as nv


def test_grouped_tiles_restart_at_each_expert():
    counts = np.array([3, 0, 5, 1])
    tiles, rows = grouped_tiles(counts, 2)
    # expert 0: rows 0-2 -> tiles 0, 0, 1; expert 2: rows 3-7 -> tiles 2, 2, 3, 3, 4; expert 3 -> tile 5
    assert tiles.tolist() == [0, 0, 1, 2, 2, 3, 3, 4, 5]
    assert rows.tolist() == [0, 1, 0, 0, 1, 0, 1, 0, 0]


def _bytes(v, g):
    c, s, _ = nv.quantize(v.astype(np.float32), g)
    return c, s


def test_identical_bytes_pass_and_a_wrong_tensor_scale_fails():
    v = np.random.default_rng(0).standard_normal((8, 64)).astype(np.float32)
    g = nv.tensor_scale(v)
    c, s = _bytes(v, g)
    assert check_act_bytes(v, g, c, s)["differing_blocks"] == 0
    c2, s2 = _bytes(v, np.float32(g * 2))          # planted: the quantiser used 2 g
    with pytest.raises(AssertionError):
        check_act_bytes(v, g, c2, s2)
    with pytest.raises(AssertionError):             # tolerances do not excuse it either
        check_act_bytes(v, g, c2, s2, code_tol=1e-3, scale_rtol=1e-4)


def test_a_code_flip_is_excused_only_at_a_midpoint():
    g = np.float32(1.0)
    v = np.zeros((1, 16), np.float32)
    v[0, 0] = 6.0                                    # block scale 1 (E4M3 exact)
    v[0, 1] = np.float32(1.25) * np.float32(1 + 2e-4)   # just above the 1 / 1.5 midpoint: code 1.5
    c, s = _bytes(v, g)
    flipped = c.copy()
    flipped[0, 1] = 2                                # the code of 1.0, the other side of the midpoint
    with pytest.raises(AssertionError):
        check_act_bytes(v, g, flipped, s)            # exact comparison
    check_act_bytes(v, g, flipped, s, code_tol=1e-3, scale_rtol=1e-4)
    far = c.copy()
    far[0, 0] = 6                                    # 6.0 -> code of 4.0: far from any midpoint
    with pytest.raises(AssertionError):
        check_act_bytes(v, g, far, s, code_tol=1e-3, scale_rtol=1e-4)
