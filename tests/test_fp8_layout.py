"""Host model of the FP8 attention's P layout (no GPU): every e4m3 byte a softmax thread
stores into tensor memory sits at the K position where veda_quantize_fp8's transposed V
tile holds the same key, so P V contracts matching keys.

The softmax thread with c = lane % 4 holds, per row, the scores of key slots 8k + 2c + {0, 1}
(16x256b load shape). It packs e4m3(P) of groups 2m and 2m + 1 into one 32-bit word, low
half first, and stores it with the 16x128b shape at column 4m + c. Four e4m3 values share
a column, lowest K index in the lowest byte, so byte e of column q is K position 4q + e. The
transposed V tile's order is include/veda.h's formula (tests/parity.py, fp8_v_key_positions).
"""
import numpy as np

import parity as P


def test_every_packed_byte_meets_its_key_in_v():
    order = P.fp8_v_key_positions()               # key slot held at each K position
    assert sorted(order.tolist()) == list(range(128))
    seen = set()
    for c in range(4):
        for m in range(8):
            column = 4 * m + c
            for half in range(2):                 # low half: group 2m; high half: group 2m + 1
                k = 2 * m + half
                for e2 in range(2):               # the pair's two keys, lower slot first
                    key = 8 * k + 2 * c + e2
                    byte = 2 * half + e2
                    pos = 4 * column + byte
                    assert order[pos] == key, (c, m, half, e2)
                    seen.add(key)
    assert seen == set(range(128))


def test_permutation_stays_inside_16_key_groups():
    order = P.fp8_v_key_positions()
    assert np.array_equal(order // 16, np.arange(128) // 16)
    # and within a group it is the same for every group
    base = order[:16]
    for m in range(8):
        assert np.array_equal(order[16 * m:16 * m + 16] - 16 * m, base)
