"""Rotation files (host only, no GPU): the calibrated U_K and U_V of every
layer round-trip bit for bit with their tag, and every damaged or mismatched
file is refused with the documented status."""
import ctypes
import os

import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import okv
from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O


def _rotations(seed, layers, hkv):
    rng = np.random.default_rng(seed)
    uk = np.stack([[WL.haar_orthogonal(rng) for _ in range(hkv)] for _ in range(layers)]).astype(np.float32)
    uv = np.stack([[WL.haar_orthogonal(rng) for _ in range(hkv)] for _ in range(layers)]).astype(np.float32)
    return uk, uv


def test_round_trip_bit_exact_with_tag(tmp_path):
    uk, uv = _rotations(0, 3, 2)
    path = tmp_path / "model.okvrot"
    okv.save_rotations(path, uk, uv, tag="Qwen3-8B, layers 0-2 — калибровка")
    got = okv.load_rotations(path)
    assert np.array_equal(got["U_K"].view(np.uint32), uk.view(np.uint32))
    assert np.array_equal(got["U_V"].view(np.uint32), uv.view(np.uint32))
    assert got["tag"] == "Qwen3-8B, layers 0-2 — калибровка"
    # the documented size: header, tag, two matrices per (layer, head), checksum
    assert os.path.getsize(path) == 32 + len(got["tag"].encode()) + 2 * 3 * 2 * 128 * 128 * 4 + 8
    with open(path, "rb") as f:
        assert f.read(8) == b"OKVROTS1"


def test_single_layer_and_empty_tag(tmp_path):
    uk, uv = _rotations(1, 1, 1)
    path = tmp_path / "one.okvrot"
    okv.save_rotations(path, uk[0], uv[0])
    got = okv.load_rotations(path)
    assert got["U_K"].shape == (1, 1, 128, 128) and got["tag"] == ""
    assert np.array_equal(got["U_K"], uk) and np.array_equal(got["U_V"], uv)


def test_calibrated_rotations_survive_the_file(tmp_path):
    q, k, v = WL.calibration_set(0, 0, 0, 4, 1, n=256)
    rot = okv.calibrate_rotations(q, k, v, 4, 1)
    path = tmp_path / "cal.okvrot"
    okv.save_rotations(path, rot["U_K"], rot["U_V"], tag="synthetic")
    got = okv.load_rotations(path)
    assert np.array_equal(got["U_K"][0], rot["U_K"]) and np.array_equal(got["U_V"][0], rot["U_V"])
    # and they are the rotations the oracle builds R from
    assert np.abs(O.rotation(got["U_K"][0, 0].astype(np.float64)) - O.rotation(rot["U_K"][0].astype(np.float64))).max() == 0


def _damaged(tmp_path, edit):
    uk, uv = _rotations(2, 2, 2)
    path = tmp_path / "d.okvrot"
    okv.save_rotations(path, uk, uv, tag="t")
    data = bytearray(path.read_bytes())
    path.write_bytes(bytes(edit(data)))
    return path


@pytest.mark.parametrize("what,edit", [
    ("flipped payload byte", lambda b: b[:1000] + bytes([b[1000] ^ 1]) + b[1001:]),
    ("flipped tag byte", lambda b: b[:32] + bytes([b[32] ^ 0x20]) + b[33:]),
    ("flipped checksum byte", lambda b: b[:-1] + bytes([b[-1] ^ 0x80])),
    ("truncated", lambda b: b[:-9]),
    ("trailing byte", lambda b: b + b"\0"),
    ("bad magic", lambda b: b"OKVROTX1" + b[8:]),
    ("empty", lambda b: b""),
])
def test_damaged_files_are_refused(tmp_path, what, edit):
    path = _damaged(tmp_path, edit)
    with pytest.raises(okv.OkvError) as e:
        okv.load_rotations(path)
    assert e.value.status == okv.ERR_IO, what


def test_other_version_and_shape_mismatch(tmp_path):
    path = _damaged(tmp_path, lambda b: b[:8] + (2).to_bytes(4, "little") + b[12:])
    with pytest.raises(okv.OkvError) as e:
        okv.load_rotations(path)
    assert e.value.status == okv.ERR_UNSUPPORTED
    uk, uv = _rotations(3, 2, 2)
    good = tmp_path / "g.okvrot"
    okv.save_rotations(good, uk, uv)
    lib = okv.lib()
    buf = np.empty((2, 2, 128, 128), np.float32)
    st = lib.okv_load_rotations(os.fsencode(good), 2, 4, 128, buf.ctypes.data, buf.ctypes.data, None, 0, 0)
    assert st == okv.ERR_INVALID_ARG and b"2 KV heads" in lib.okv_last_error_string()
    assert lib.okv_load_rotations(os.fsencode(tmp_path / "missing"), 2, 2, 128, buf.ctypes.data, buf.ctypes.data,
                                  None, 0, 0) == okv.ERR_IO


def test_verify_rejects_a_matrix_that_is_not_orthogonal(tmp_path):
    uk, uv = _rotations(4, 2, 2)
    uv[1, 0, 5, 7] += 1e-2  # a well-formed file (valid checksum) holding a bad rotation
    path = tmp_path / "bad.okvrot"
    okv.save_rotations(path, uk, uv)
    with pytest.raises(okv.OkvError) as e:
        okv.load_rotations(path, verify=True)
    assert e.value.status == okv.ERR_NUMERIC and "U_V 2 (layer 1, KV head 0)" in str(e.value)
    got = okv.load_rotations(path, verify=False)
    assert np.array_equal(got["U_V"], uv)


def test_save_argument_checks(tmp_path):
    lib = okv.lib()
    uk, uv = _rotations(5, 1, 1)
    p = os.fsencode(tmp_path / "x.okvrot")
    assert lib.okv_save_rotations(p, 1, 1, 64, uk.ctypes.data, uv.ctypes.data, None) == okv.ERR_UNSUPPORTED
    assert lib.okv_save_rotations(p, 0, 1, 128, uk.ctypes.data, uv.ctypes.data, None) == okv.ERR_INVALID_ARG
    assert lib.okv_save_rotations(None, 1, 1, 128, uk.ctypes.data, uv.ctypes.data, None) == okv.ERR_INVALID_ARG
    assert lib.okv_save_rotations(p, 1, 1, 128, uk.ctypes.data, uv.ctypes.data, b"x" * 5000) == okv.ERR_INVALID_ARG
    assert lib.okv_save_rotations(os.fsencode(tmp_path / "no" / "dir.okvrot"), 1, 1, 128, uk.ctypes.data,
                                  uv.ctypes.data, None) == okv.ERR_IO
