"""CPU checks of the test-side packer for the prepared-weight GEMM layout (include/oq.h,
"Data formats"): byte j of each 16-byte group holds element 32g + j low and 32g + 16 + j high."""
import numpy as np

from parity import pack_w4_gemm, unpack_w4_gemm


def test_gemm_layout_hand_example():
    w = np.zeros((1, 32), dtype=np.int64)
    w[0, 0], w[0, 16], w[0, 5], w[0, 21], w[0, 31] = 1, -1, -7, 7, 3
    b = pack_w4_gemm(w)
    assert b.shape == (1, 16)
    assert b[0, 0] == 0xF1          # element 0 low, element 16 high
    assert b[0, 5] == 0x79          # element 5 (-7 -> 0x9) low, element 21 (7) high
    assert b[0, 15] == 0x30         # element 15 (0) low, element 31 (3) high


def test_gemm_layout_round_trip():
    rng = np.random.default_rng(0)
    w = rng.integers(-8, 8, (5, 96))
    assert np.array_equal(unpack_w4_gemm(pack_w4_gemm(w)), w)
