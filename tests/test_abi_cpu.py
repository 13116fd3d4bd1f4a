"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every symbol the header declares, argument validation returns the
documented statuses before any launch, and the host calibration matches the
oracle."""
import ctypes

import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import okv
from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O


def test_library_exports_every_header_symbol():
    lib = okv.lib()
    names = okv.header_functions()
    assert "okv_decode_attention" in names and len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert lib.okv_version() >= 1


def _desc(**kw):
    d = okv.CacheDesc(32, 8, 128, 128, 16, 128, 64, 4, 16, 0, 4096, 8192, 16384, 32768, 0)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_status_strings_and_sizes():
    lib = okv.lib()
    assert lib.okv_status_string(0) == b"OKV_OK"
    assert lib.okv_status_string(2) == b"OKV_ERR_UNSUPPORTED"
    assert lib.okv_pages_bytes(10, 8, 128) == 10 * 8 * 1152
    assert lib.okv_pages_bytes(10, 8, 64) == 10 * 8 * 1280
    assert lib.okv_pages_bytes(10, 8, 32) == 10 * 8 * 1536
    assert [lib.okv_block_head_bytes(g) for g in (128, 64, 32, 16, 0)] == [1152, 1280, 1536, 0, 0]
    assert lib.okv_window_bytes(3, 8) == 3 * 8 * 2 * 128 * 128 * 2
    assert lib.okv_sink_bytes(3, 8, 192) == 3 * 8 * 2 * 192 * 128 * 2
    assert lib.okv_status_string(5) == b"OKV_ERR_IO"


def test_validation_before_launch():
    lib = okv.lib()
    fake = ctypes.c_void_p(1 << 20)
    # NULL descriptor
    assert lib.okv_append_quantize(None, fake, fake, 1, fake, fake, fake, fake, 0, None, None) == okv.ERR_INVALID_ARG
    # unsupported head dim / group / window
    for field, val in (("head_dim", 64), ("group", 16), ("group", 48), ("group", 256), ("window", 64),
                       ("block_tokens", 64)):
        d = _desc(**{field: val})
        st = lib.okv_append_quantize(ctypes.byref(d), fake, fake, 1, fake, fake, fake, fake, 0, None, None)
        assert st == okv.ERR_UNSUPPORTED, field
        assert b"128" in lib.okv_last_error_string() or b"16" in lib.okv_last_error_string()
    # Hq not a multiple of Hkv
    d = _desc(num_q_heads=30)
    assert lib.okv_append_quantize(ctypes.byref(d), fake, fake, 1, fake, fake, fake, fake, 0, None, None) \
        == okv.ERR_INVALID_ARG
    # sink count: a multiple of 16 up to 1024, with a 16-byte aligned buffer
    for ns in (8, 1040, -16):
        d = _desc(num_sink=ns, sink_rows=1 << 16)
        assert lib.okv_append_quantize(ctypes.byref(d), fake, fake, 1, fake, fake, fake, fake, 0, None, None) \
            == okv.ERR_UNSUPPORTED, ns
    for rows in (None, (1 << 16) + 8):
        d = _desc(num_sink=32, sink_rows=rows)
        assert lib.okv_decode_attention(ctypes.byref(d), fake, 4, fake, fake, fake, fake, fake, 1 << 30, None) \
            == okv.ERR_INVALID_ARG
        assert b"sink_rows" in lib.okv_last_error_string()
    # misaligned pages
    d = _desc(pages=4097)
    assert lib.okv_append_quantize(ctypes.byref(d), fake, fake, 1, fake, fake, fake, fake, 0, None, None) \
        == okv.ERR_INVALID_ARG
    # T = 0 and B = 0 are no-ops
    d = _desc()
    assert lib.okv_append_quantize(ctypes.byref(d), None, None, 0, None, None, None, None, 0, None, None) == okv.OK
    assert lib.okv_decode_attention(ctypes.byref(d), None, 0, None, None, None, None, None, 0, None) == okv.OK
    # unknown flags, negative T
    assert lib.okv_append_quantize(ctypes.byref(d), fake, fake, 1, fake, fake, fake, fake, 8, None, None) \
        == okv.ERR_INVALID_ARG
    assert lib.okv_append_quantize(ctypes.byref(d), fake, fake, -1, fake, fake, fake, fake, 0, None, None) \
        == okv.ERR_INVALID_ARG
    # pre-rotated input must be 16-byte aligned
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.okv_append_quantize(ctypes.byref(d), odd, fake, 1, fake, fake, fake, fake, okv.PRE_ROTATED,
                                   None, None) == okv.ERR_INVALID_ARG
    # workspace too small / misaligned
    need = lib.okv_decode_workspace_bytes(ctypes.byref(d), 4)
    assert need > 0
    ws = ctypes.c_void_p(1 << 24)
    assert lib.okv_decode_attention(ctypes.byref(d), fake, 4, fake, fake, fake, fake, ws, need - 1, None) \
        == okv.ERR_INVALID_ARG
    assert b"workspace" in lib.okv_last_error_string()
    assert lib.okv_decode_attention(ctypes.byref(d), fake, 4, fake, fake, fake, fake,
                                    ctypes.c_void_p((1 << 24) + 16), need, None) == okv.ERR_INVALID_ARG
    # group size outside {1,2,4,8,16}
    d3 = _desc(num_q_heads=24)
    assert lib.okv_decode_attention(ctypes.byref(d3), fake, 4, fake, fake, fake, fake, ws, 1 << 30, None) \
        == okv.ERR_UNSUPPORTED
    # dequantize argument checks
    assert lib.okv_dequantize(ctypes.byref(d), 1, fake, fake, fake, 16, 2, 0, 0, fake, None) == okv.ERR_INVALID_ARG
    assert lib.okv_dequantize(ctypes.byref(d), 1, fake, fake, fake, 0, 0, 0, 0, fake, None) == okv.OK
    # staged rotation image: size, a buffer to build into, 16-byte alignment
    assert lib.okv_r_image_bytes(8) == 8 * 2 * 3 * 128 * 128 * 2
    assert lib.okv_r_image_bytes(-1) == 0
    assert lib.okv_build_r_image(ctypes.byref(d), None) == okv.ERR_INVALID_ARG
    assert b"r_image" in lib.okv_last_error_string()
    d4 = _desc()
    d4.r_image = (1 << 22) + 8
    assert lib.okv_build_r_image(ctypes.byref(d4), None) == okv.ERR_INVALID_ARG
    assert lib.okv_append_quantize(ctypes.byref(d4), fake, fake, 1, fake, fake, fake, fake, 0, None, None) \
        == okv.ERR_INVALID_ARG
    assert b"r_image" in lib.okv_last_error_string()


def test_calibrate_validation():
    lib = okv.lib()
    x = np.zeros((4, 2, 128), np.float32)
    p = x.ctypes.data_as(ctypes.c_void_p)
    assert lib.okv_calibrate_rotations(p, 4, p, p, 4, 2, 2, 64, None, None, None, None) == okv.ERR_UNSUPPORTED
    assert lib.okv_calibrate_rotations(p, 4, p, p, 4, 3, 2, 128, None, None, None, None) == okv.ERR_INVALID_ARG
    assert lib.okv_calibrate_rotations(None, 4, p, p, 4, 2, 2, 128, None, None, None, None) == okv.ERR_INVALID_ARG
    assert lib.okv_calibrate_rotations(p, 0, p, p, 4, 2, 2, 128, None, None, None, None) == okv.ERR_INVALID_ARG


def _match_columns(u_lib, u_ref, lam):
    """Compare eigenvector matrices column by column where the eigenvalue is
    well separated, and by projector where eigenvalues cluster."""
    d = u_ref.shape[0]
    j = 0
    while j < d:
        k = j + 1
        while k < d and abs(lam[k] - lam[k - 1]) <= 1e-9 * abs(lam[0]):
            k += 1
        if k - j == 1:
            assert np.abs(u_lib[:, j] - u_ref[:, j]).max() < 2e-5, j
        else:
            pa = u_lib[:, j:k] @ u_lib[:, j:k].T
            pb = u_ref[:, j:k] @ u_ref[:, j:k].T
            assert np.abs(pa - pb).max() < 2e-5
        j = k


@pytest.mark.parametrize("hq,hkv,n", [(4, 1, 4096), (8, 2, 1024)])
def test_calibration_matches_oracle(hq, hkv, n):
    q, k, v = WL.calibration_set(0, 0, 0, hq, hkv, n=n)
    got = okv.calibrate_rotations(q, k, v, hq, hkv)
    ref = O.calibrate(q, k, v, hq, hkv)
    for h in range(hkv):
        for kind in ("K", "V"):
            u = got["U_" + kind][h].astype(np.float64)
            assert np.abs(u.T @ u - np.eye(128)).max() < 1e-5
            _match_columns(u, ref["U_" + kind][h], ref["lam_" + kind][h])
            r = got["R_" + kind][h].astype(np.float64)
            assert np.abs(r - ref["R_" + kind][h]).max() < 2e-5


def test_prepared_step_call_checks_its_inputs_on_the_host():
    torch = pytest.importorskip("torch")
    k = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    i32 = torch.zeros(2, dtype=torch.int32)
    q = torch.zeros((2, 32, 128), dtype=torch.bfloat16)
    table = torch.zeros((2, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        okv.DecodeStepCall(None, k, k, i32, i32, i32, q, i32, table, i32)
    with pytest.raises(TypeError, match="bfloat16"):
        okv.DecodeStepCall(None, k.float(), k, i32, i32, i32, q, i32, table, i32)
