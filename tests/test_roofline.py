"""The roofline accounting on hand-counted cases."""
import numpy as np

from lora_adapter_application_b200 import roofline


def test_layer_bytes_hand_counted():
    ids = np.array([0, -1, 1, 0, 5])        # id 5 is outside N=3: no adapter
    ranks = np.array([2, 4, 8])
    # active rows: 3 -> each 2*(10) + 2*2*(6+3) = 20 + 36 = 56 bytes
    # adapters 0 and 1: 2*2*(10+6) + 2*2*(10+3) = 64 + 52 ; 2*4*16 + 2*4*13 = 128 + 104
    got = roofline.layer_bytes(ids, ranks, 3, 10, [6, 3], 2)
    assert got == 3 * 56 + (64 + 52) + (128 + 104)


def test_layer_flops_hand_counted():
    ids = np.array([0, -1, 1, 0])
    ranks = np.array([2, 4])
    # per row: 2*r*(2*10 + 9)
    assert roofline.layer_flops(ids, ranks, 2, 10, [6, 3]) == 2 * (2 + 4 + 2) * 29


def test_padding_not_counted_and_linear_in_rank():
    ids = np.zeros(7, dtype=np.int64)
    a = roofline.layer_bytes(ids, np.array([16]), 1, 4096, [4096], 2)
    b = roofline.layer_bytes(ids, np.array([128]), 1, 4096, [4096], 2)
    rows = 7 * (2 * 4096 + 4 * 4096)
    assert (b - rows) == 8 * (a - rows)
