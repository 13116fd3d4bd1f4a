"""The allocation-free decode entry point.

It serves callers that cannot allocate device memory (a plugin given only its
tensors by an engine that owns all device memory, or code that must not call
cudaMalloc because it can synchronise the device).  Its output must match the
workspace entry point's within the decode tolerance, call after call, and a
batch too large for its static scratch must be refused before anything runs.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from tests import gpu_helpers as H

TOL = 2e-3


def test_noalloc_rejects_batch_beyond_static_scratch():
    from int2_kv_cache_rotate_b200 import okv
    lib = okv.lib()
    d = okv.CacheDesc(32, 8, 128, 128, 16, 128, 64, 4, 16, 0, 4096, 8192, 16384, 32768, 0)
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 14  # rotated queries alone would need 32 MiB
    st = lib.okv_decode_attention_noalloc(ctypes.byref(d), fake, big, fake, fake, fake, fake, None)
    assert st == okv.ERR_INVALID_ARG
    assert b"scratch" in lib.okv_last_error_string()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    from int2_kv_cache_rotate_b200 import okv

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()

    seed, hq, hkv = 21, 32, 8
    lens = [3000, 129, 1, 777]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    cache = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv)
    slots, pos = lay.flat()
    k = np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, 0, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    v = np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, 1, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    okv.append_quantize(cache, dev(k), dev(v), dev(slots), dev(pos), dev(lay.table), dev(np.array(lens, np.int32)),
                        pre_rotated=True)
    seq, table = dev(np.arange(len(lens), dtype=np.int32)), dev(lay.table)
    for call in range(2):
        # a different query and shorter contexts on the second call: nothing may leak between calls
        q = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=call) for h in range(hkv)], 1)
        q = dev(q.reshape(len(lens), hq, 128)).to(torch.bfloat16)
        cl = dev(np.array(lens, np.int32) - call * np.array([100, 0, 0, 7], np.int32))
        ref = okv.decode_attention(cache, q, seq, table, cl)
        got = okv.decode_attention_noalloc(cache, q, seq, table, cl)
        torch.cuda.synchronize()
        err = H.rel_err_rows(got.cpu().numpy(), ref.cpu().numpy())
        assert err.max() <= TOL, (call, err.max())
    assert cache.device_status() == 0
