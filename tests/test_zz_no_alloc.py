"""The allocation-free decode entry point.

It serves callers that cannot allocate device memory (a plugin given only its
tensors by an engine that owns all device memory, or code that must not call
cudaMalloc because it can synchronise the device).  It runs the same kernels
as the workspace entry point on the same inputs, so its output must be
bit-identical to that entry point's, call after call, and within the decode
tolerance of the oracle.  The largest batch whose scratch fits the static
array must run; one sequence more must be refused before anything runs.
This file is collected last on purpose."""
import ctypes
import re

import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H

TOL = 2e-3


def _scratch_bytes() -> int:
    """OKV_NOALLOC_SCRATCH_BYTES as include/okv.h defines it."""
    from int2_kv_cache_rotate_b200 import okv
    m = re.search(r"#define OKV_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(okv.HEADER).read())
    return int(m.group(1)) << int(m.group(2))


def test_scratch_size_is_read_from_the_header():
    assert _scratch_bytes() == 8 << 20


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
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    slots, pos = lay.flat()
    zk = [np.stack([WL.sample_rotated(seed, 0, 0, h, n, 0, extra=b) for h in range(hkv)], 1)
          for b, n in enumerate(lens)]
    zv = [np.stack([WL.sample_rotated(seed, 0, 0, h, n, 1, extra=b) for h in range(hkv)], 1)
          for b, n in enumerate(lens)]
    for b in range(len(lens)):
        oc.append(b, 0, zk[b], zv[b], pre_rotated=True)
    okv.append_quantize(cache, dev(np.concatenate(zk)), dev(np.concatenate(zv)), dev(slots), dev(pos),
                        dev(lay.table), dev(np.array(lens, np.int32)), pre_rotated=True)
    seq, table = dev(np.arange(len(lens), dtype=np.int32)), dev(lay.table)
    for call in range(2):
        # a different query and shorter contexts on the second call: nothing may leak between calls
        qh = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=call) for h in range(hkv)], 1)
        qh = qh.reshape(len(lens), hq, 128)
        cl = np.array(lens, np.int32) - call * np.array([100, 0, 0, 7], np.int32)
        q = dev(qh).to(torch.bfloat16)
        ref = okv.decode_attention(cache, q, seq, table, dev(cl))
        got = okv.decode_attention_noalloc(cache, q, seq, table, dev(cl))
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (call, (got - ref).abs().max().item())
        if call == 0:
            want = O.decode(oc, qh, np.arange(len(lens)), cl, hq)
            err = H.rel_err_rows(got.cpu().numpy(), want)
            assert err.max() <= TOL, err.max()
    assert cache.device_status() == 0


@pytest.mark.gpu
def test_noalloc_largest_batch_runs_and_one_more_is_refused():
    """The scratch a batch needs grows with the SM count (one split-K partial
    per CTA), so the largest batch is found from okv_decode_workspace_bytes on
    this device, as a caller would."""
    import torch
    from int2_kv_cache_rotate_b200 import okv

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()

    seed, hq, hkv = 22, 32, 8
    probe = okv.Cache(hq, hkv, 1, 1, 1, *H.rotations(seed, hkv))
    bmax = 1
    while okv.decode_workspace_bytes(probe, bmax + 1) <= _scratch_bytes():
        bmax += 1
    assert 1 < bmax < 1000
    lens = [1 + (37 * b) % 300 for b in range(bmax + 1)]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    cache = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv)
    slots, pos = lay.flat()
    zk = np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, 0, extra=b) for h in range(hkv)], 1)
                         for b, n in enumerate(lens)])
    zv = np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, 1, extra=b) for h in range(hkv)], 1)
                         for b, n in enumerate(lens)])
    okv.append_quantize(cache, dev(zk), dev(zv), dev(slots), dev(pos), dev(lay.table), dev(np.array(lens, np.int32)),
                        pre_rotated=True)
    qh = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv) for h in range(hkv)], 1)
    q = dev(qh.reshape(len(lens), hq, 128)).to(torch.bfloat16)
    seq, table, cl = dev(np.arange(len(lens), dtype=np.int32)), dev(lay.table), dev(np.array(lens, np.int32))
    got = okv.decode_attention_noalloc(cache, q[:bmax], seq[:bmax], table, cl[:bmax])
    ref = okv.decode_attention(cache, q[:bmax], seq[:bmax], table, cl[:bmax])
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    out = torch.full((bmax + 1, hq, 128), 7.0, dtype=torch.float32, device="cuda")
    with pytest.raises(okv.OkvError) as exc:
        okv.decode_attention_noalloc(cache, q, seq, table, cl, out=out)
    assert exc.value.status == okv.ERR_INVALID_ARG and "scratch" in str(exc.value)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # refused before anything ran
    assert cache.device_status() == 0
