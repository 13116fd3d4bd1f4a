"""The test-side layout readers agree with each other: the grouped reader
with one 128-channel group reads exactly what the plain reader reads (both
only locate bytes; the layout is the one include/okv.h documents)."""
import numpy as np

from tests import gpu_helpers as H


def test_grouped_reader_with_one_group_is_the_plain_reader():
    r = np.random.default_rng(0)
    hkv, n = 3, 70
    table = r.permutation(40).astype(np.int32).reshape(2, 20)
    pages = r.integers(0, 256, size=40 * hkv * 1152, dtype=np.uint8)
    for slot in range(2):
        for h in range(hkv):
            for kind in (0, 1):
                a = H.gather_codes(pages, table, slot, h, hkv, n, kind)
                b = H.gather_codes_grouped(pages, table, slot, h, hkv, n, kind, 128)
                assert np.array_equal(a[0], b[0])
                assert np.array_equal(a[1].view(np.uint16), b[1][:, 0].view(np.uint16))
                assert np.array_equal(a[2].view(np.uint16), b[2][:, 0].view(np.uint16))


def test_grouped_reader_offsets():
    """Token t, group k of a 32-channel-group block-head: scale at 1024 + 4 (4 t + k)
    for keys, 1024 + 256 + 4 (4 t + k) for values; block-heads of 1536 bytes."""
    hkv = 1
    pages = np.zeros(2 * 1536, np.uint8)
    table = np.array([[1]], np.int32)
    for t in range(16):
        for k in range(4):
            for kind in (0, 1):
                off = 1536 + 1024 + 256 * kind + 4 * (4 * t + k)
                pages[off:off + 2] = np.array([t, 16 * kind + k], np.uint8)
    for kind in (0, 1):
        _, s16, _ = H.gather_codes_grouped(pages, table, 0, 0, hkv, 16, kind, 32)
        bits = s16.view(np.uint16)
        for t in range(16):
            for k in range(4):
                assert bits[t, k] == t | ((16 * kind + k) << 8)
