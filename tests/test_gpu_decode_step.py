"""okv_decode_step (append this step's tokens, then decode, in one call) must
leave exactly the cache bytes and produce exactly the outputs of
okv_append_quantize followed by okv_decode_attention: the fused launch runs
the same per-tile append and per-head query rotation."""
import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from tests import gpu_helpers as H

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _d(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("hq,hkv,n_new", [(32, 8, 1), (16, 4, 3), (32, 8, 31), (8, 2, 200), (32, 8, 0)])
def test_decode_step_equals_append_then_decode(hq, hkv, n_new):
    from int2_kv_cache_rotate_b200 import okv
    seed = 51
    base = [1500, 700, 129, 1]
    B = len(base)
    lens = [n + n_new for n in base]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    caches = [okv.Cache(hq, hkv, lay.num_blocks, B, lay.mbps, uk, uv) for _ in range(2)]
    # history through the pre-rotated path, identical in both caches
    slots = np.concatenate([np.full(n, b, np.int32) for b, n in enumerate(base)])
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in base])
    z = {kind: np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], 1)
                               for b, n in enumerate(base)]) for kind in (0, 1)}
    for c in caches:
        okv.append_quantize(c, _d(z[0]), _d(z[1]), _d(slots), _d(pos), _d(lay.table), _d(np.array(lens, np.int32)),
                            pre_rotated=True)
    # this step: n_new bf16 tokens per sequence, then one query per sequence
    new_slot = np.repeat(np.arange(B, dtype=np.int32), n_new)
    new_pos = np.concatenate([np.arange(n, n + n_new, dtype=np.int32) for n in base]) if n_new else \
        np.zeros(0, np.int32)
    k = np.concatenate([np.stack([WL.sample_keys(seed, 0, 0, h, n_new, extra=10 + b) for h in range(hkv)], 1)
                        for b in range(B)]) if n_new else np.zeros((0, hkv, 128), np.float32)
    v = np.concatenate([np.stack([WL.sample_values(seed, 0, 0, h, n_new, extra=10 + b) for h in range(hkv)], 1)
                        for b in range(B)]) if n_new else np.zeros((0, hkv, 128), np.float32)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, B, hq // hkv, extra=2) for h in range(hkv)], 1).reshape(B, hq, 128)
    kd, vd, qd = _d(k).to(torch.bfloat16), _d(v).to(torch.bfloat16), _d(q).to(torch.bfloat16)
    table, lens_d, seq = _d(lay.table), _d(np.array(lens, np.int32)), _d(np.arange(B, dtype=np.int32))
    if n_new:
        okv.append_quantize(caches[0], kd, vd, _d(new_slot), _d(new_pos), table, lens_d)
    ref = okv.decode_attention(caches[0], qd, seq, table, lens_d)
    got = okv.decode_step(caches[1], kd, vd, _d(new_slot), _d(new_pos), lens_d, qd, seq, table, lens_d)
    torch.cuda.synchronize()
    assert torch.equal(caches[0].pages, caches[1].pages)
    assert torch.equal(caches[0].ring, caches[1].ring)
    assert torch.equal(ref, got)
    assert caches[1].device_status() == 0


@pytest.mark.parametrize("graph", [False, True])
def test_prepared_call_equals_decode_step_over_several_steps(graph):
    """DecodeStepCall (arguments marshalled once, inputs refilled in place;
    eager, or replayed from a CUDA graph after its first call) leaves the same
    cache bytes and outputs as okv.decode_step, step by step."""
    from int2_kv_cache_rotate_b200 import okv
    seed, hq, hkv = 52, 32, 8
    base = [900, 300, 130]
    B, steps = len(base), 4
    lay = H.Layout(seed, [n + steps for n in base])
    uk, uv = H.rotations(seed, hkv)
    caches = [okv.Cache(hq, hkv, lay.num_blocks, B, lay.mbps, uk, uv, num_sink=32) for _ in range(2)]
    slots = np.concatenate([np.full(n, b, np.int32) for b, n in enumerate(base)])
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in base])
    z = {kind: np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], 1)
                               for b, n in enumerate(base)]) for kind in (0, 1)}
    for c in caches:
        okv.append_quantize(c, _d(z[0]), _d(z[1]), _d(slots), _d(pos), _d(lay.table), _d(np.array(base, np.int32)),
                            pre_rotated=True)
    table, seq = _d(lay.table), _d(np.arange(B, dtype=np.int32))
    kd = torch.empty((B, hkv, 128), dtype=torch.bfloat16, device="cuda")
    vd, qd = torch.empty_like(kd), torch.empty((B, hq, 128), dtype=torch.bfloat16, device="cuda")
    pd, ld = torch.empty(B, dtype=torch.int32, device="cuda"), torch.empty(B, dtype=torch.int32, device="cuda")
    call = okv.DecodeStepCall(caches[1], kd, vd, seq, pd, ld, qd, seq, table, ld, graph=graph)
    for i in range(steps):
        k = np.stack([np.stack([WL.sample_keys(seed, 0, 0, h, 1, extra=20 + 10 * i + b)[0] for h in range(hkv)])
                      for b in range(B)])
        v = np.stack([np.stack([WL.sample_values(seed, 0, 0, h, 1, extra=20 + 10 * i + b)[0] for h in range(hkv)])
                      for b in range(B)])
        q = np.stack([WL.sample_queries(seed, 0, 0, h, B, hq // hkv, extra=30 + i) for h in range(hkv)], 1)
        q = q.reshape(B, hq, 128)
        p = np.array(base, np.int32) + i
        kd.copy_(_d(k).to(torch.bfloat16)), vd.copy_(_d(v).to(torch.bfloat16)), qd.copy_(_d(q).to(torch.bfloat16))
        pd.copy_(_d(p)), ld.copy_(_d(p + 1))
        ref = okv.decode_step(caches[0], kd, vd, seq, pd, ld, qd, seq, table, ld).clone()
        got = call()
        torch.cuda.synchronize()
        assert torch.equal(ref, got), i
    assert torch.equal(caches[0].pages, caches[1].pages) and torch.equal(caches[0].ring, caches[1].ring)
    assert torch.equal(caches[0].sink, caches[1].sink)
    assert caches[1].device_status() == 0
