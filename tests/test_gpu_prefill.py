"""Chunked-prefill attention over the INT2 cache against the oracle.

A prefill chunk's T tokens are appended first; its queries then attend
causally to the sequence as the cache holds it (sink rows and the last W
positions fp16, the rest INT2).  The CUDA path (query rotation, tensor-core
attention, un-rotation) through the C ABI is compared with O.prefill on the
same seeded inputs, per (token, head) row at the 2e-3 tolerance of decode:
GQA group sizes 1, 4 and 8; chunks at the end of long histories, whole
sequences as one chunk, ragged chunk and context lengths; sinks; 64- and
32-channel quantisation groups; and a one-token chunk, which must equal
decode.  The pages make the compressed cache serve paged attention and
prefix caching (aiforradalom.hu, "OSCAR: figyelem-tudatos és bevetésre
kész"), where prefill chunks read the INT2 history.
"""
import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3


def _okv():
    from int2_kv_cache_rotate_b200 import okv
    return okv


def _t(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _case(seed, hq, hkv, L, T, group=128, sinks=0, checked=None, scale=1.0, vscale=1.0, tokens=None):
    """One sequence of L tokens (pre-rotated fill, identical on both sides);
    the last T are the chunk.  Returns (got, {hk: want}) for the checked KV heads."""
    okv = _okv()
    lay = H.Layout(seed, [L])
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, 1, lay.mbps, uk, uv, group=group, num_sink=sinks)
    zk = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 0, scale=scale) for h in range(hkv)], 1)
    zv = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 1, scale=vscale) for h in range(hkv)], 1)
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(zk), _t(zv), _t(slots), _t(pos), _t(lay.table), _t(np.array([L], np.int32)),
                        pre_rotated=True)
    G = hq // hkv
    q = np.stack([WL.sample_queries(seed, 0, 0, h, T, G, extra=9) for h in range(hkv)], 1).reshape(T, hq, 128)
    got = okv.prefill_attention(gc, _t(q, torch.bfloat16), 0, L, _t(lay.table)).cpu().numpy()
    assert gc.device_status() == 0
    want = {}
    for hk in (checked if checked is not None else range(hkv)):
        oc = O.Cache(1, uk[hk:hk + 1].astype(np.float64), uv[hk:hk + 1].astype(np.float64), group=group,
                     sinks=sinks)
        oc.append(0, 0, zk[:, hk:hk + 1], zv[:, hk:hk + 1], pre_rotated=True)
        want[hk] = O.prefill(oc, q[:, hk * G:(hk + 1) * G], 0, L, G, tokens=tokens)
    if tokens is not None:
        got = got[list(tokens)]
        want = {hk: w[list(tokens)] for hk, w in want.items()}
    return got, want, G


def _check(got, want, G):
    for hk, w in want.items():
        err = H.rel_err_rows(got[:, hk * G:(hk + 1) * G], w)
        assert err.max() <= TOL, (hk, err.max(), np.unravel_index(err.argmax(), err.shape))


@pytest.mark.parametrize("hq,hkv,L,T", [
    (4, 1, 2048, 300),     # the tiny single-layer shape; chunk ends the sequence
    (4, 1, 700, 700),      # the whole sequence as one chunk (INT2 and window inside the chunk)
    (32, 8, 3000, 77),     # 8B-class heads, ragged chunk
    (64, 8, 1500, 33),     # G = 8
    (8, 8, 1000, 129),     # G = 1
    (16, 4, 45, 45),       # shorter than the window: all fp16
])
def test_prefill_parity(hq, hkv, L, T):
    got, want, G = _case(51, hq, hkv, L, T, checked=[0, hkv - 1])
    _check(got, want, G)


@pytest.mark.parametrize("group", [64, 32])
def test_prefill_grouped(group):
    got, want, G = _case(52, 32, 8, 2500, 200, group=group, checked=[0, 5])
    _check(got, want, G)


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("hq,hkv,L,T,sinks,scale,vscale", [
    (8, 8, 700, 130, 32, 1.0, 1.0),       # G = 1, sinks, a ragged last tile
    (64, 8, 1300, 40, 0, 1.0, 1.0),       # G = 8
    (8, 2, 1200, 64, 0, 30.0, 1.0),       # peaked rows
    (8, 2, 1500, 100, 0, 1.0, 8000.0),    # value scales near the top of fp16
    (16, 4, 90, 90, 0, 1.0, 1.0),         # shorter than the window: all fp16
])
def test_prefill_grouped_shapes(group, hq, hkv, L, T, sinks, scale, vscale):
    got, want, G = _case(60 + hq + T, hq, hkv, L, T, group=group, sinks=sinks, scale=scale, vscale=vscale,
                         checked=[0, hkv - 1])
    _check(got, want, G)


def test_prefill_grouped_benchmark_shape_sampled():
    """32-channel groups at the prefill benchmark's shape (1,024 tokens ending
    32,768, 32 / 8 heads), sampled chunk tokens."""
    got, want, G = _case(61, 32, 8, 32768, 1024, group=32, checked=[3], tokens=[0, 511, 1023])
    _check(got, want, G)


def test_prefill_with_sinks():
    got, want, G = _case(53, 8, 2, 1000, 150, sinks=192)
    _check(got, want, G)


def test_prefill_large_logits():
    """Rotated keys in the hundreds: peaked softmax rows."""
    got, want, G = _case(54, 8, 2, 1200, 64, scale=30.0)
    _check(got, want, G)


@pytest.mark.parametrize("vscale", [300.0, 8000.0])
def test_prefill_large_value_scales(vscale):
    """Value scales near the top of fp16: the weight the value MMA takes
    (p times the value scale, fp16 hi + lo) must stay in range, so the
    tensor-core kernel re-bases its running maximum more often."""
    got, want, G = _case(57, 8, 2, 1500, 100, vscale=vscale)
    _check(got, want, G)


def test_prefill_many_ctas():
    """8,192-token context, 256-token chunk at the 32 / 8 head shape: eight
    128-row tiles per KV head, 128 key chunks each."""
    got, want, G = _case(58, 32, 8, 8192, 256, checked=[0, 7])
    _check(got, want, G)


def test_prefill_benchmark_shape_sampled():
    """The prefill benchmark's shape: a 1,024-token chunk ending a 32,768-token
    sequence, 32 query / 8 KV heads; sampled chunk tokens of two KV heads."""
    got, want, G = _case(59, 32, 8, 32768, 1024, checked=[0, 5], tokens=[0, 1, 255, 640, 1022, 1023])
    _check(got, want, G)


def test_prefill_one_token_equals_decode():
    okv = _okv()
    seed, hq, hkv, L = 55, 32, 8, 3000
    lay = H.Layout(seed, [L])
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, 1, lay.mbps, uk, uv)
    zk = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 0) for h in range(hkv)], 1)
    zv = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 1) for h in range(hkv)], 1)
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(zk), _t(zv), _t(slots), _t(pos), _t(lay.table), _t(np.array([L], np.int32)),
                        pre_rotated=True)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, 1, 4, extra=3) for h in range(hkv)], 1).reshape(1, hq, 128)
    qd = _t(q, torch.bfloat16)
    pf = okv.prefill_attention(gc, qd, 0, L, _t(lay.table)).cpu().numpy()
    dc = okv.decode_attention(gc, qd, _t(np.zeros(1, np.int32)), _t(lay.table), _t(np.array([L], np.int32)))
    assert H.rel_err_rows(pf, dc.cpu().numpy()).max() <= TOL


def test_prefill_rejects_bad_arguments():
    okv = _okv()
    lay = H.Layout(56, [100])
    uk, uv = H.rotations(56, 1)
    gc = okv.Cache(4, 1, lay.num_blocks, 1, lay.mbps, uk, uv)
    q = torch.zeros((10, 4, 128), dtype=torch.bfloat16, device="cuda")
    tb = _t(lay.table)
    for slot, L in ((1, 100), (-1, 100), (0, 5), (0, lay.mbps * 16 + 1)):
        with pytest.raises(okv.OkvError) as e:
            okv.prefill_attention(gc, q, slot, L, tb)
        assert e.value.status == okv.ERR_INVALID_ARG
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(okv.OkvError):
        okv.prefill_attention(gc, q, 0, 100, tb, ws=small)


def test_prefill_bad_block_is_flagged_and_skipped():
    """A block id outside the pool in the middle of the INT2 history: the
    kernel raises OKV_DEV_BAD_BLOCK and attends as if those 16 positions were
    absent (the oracle's attention over the remaining positions)."""
    okv = _okv()
    seed, hq, hkv, L, T = 60, 8, 2, 2000, 100
    lay = H.Layout(seed, [L])
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, 1, lay.mbps, uk, uv)
    zk = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 0) for h in range(hkv)], 1)
    zv = np.stack([WL.sample_rotated(seed, 0, 0, h, L, 1) for h in range(hkv)], 1)
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(zk), _t(zv), _t(slots), _t(pos), _t(lay.table), _t(np.array([L], np.int32)),
                        pre_rotated=True)
    torch.cuda.synchronize()
    assert gc.device_status() == 0
    table = lay.table.copy()
    bad = 10                                   # positions 160 .. 175, INT2 for every row of the chunk
    table[0, bad] = lay.num_blocks + 3
    G = hq // hkv
    q = np.stack([WL.sample_queries(seed, 0, 0, h, T, G, extra=9) for h in range(hkv)], 1).reshape(T, hq, 128)
    got = okv.prefill_attention(gc, _t(q, torch.bfloat16), 0, L, _t(table)).cpu().numpy()
    assert gc.device_status() & okv.DEV_BAD_BLOCK
    assert np.all(np.isfinite(got))
    first = L - T
    keep = np.ones(L, bool)
    keep[16 * bad:16 * bad + 16] = False
    for hk in range(hkv):
        oc = O.Cache(1, uk[hk:hk + 1].astype(np.float64), uv[hk:hk + 1].astype(np.float64))
        oc.append(0, 0, zk[:, hk:hk + 1], zv[:, hk:hk + 1], pre_rotated=True)
        kx, vx = oc.values(0, 0, 0, L), oc.values(0, 1, 0, L)
        for i in (0, 50, T - 1):
            vis = np.zeros(L, bool)
            vis[:first + i + 1] = True
            sel = vis & keep
            for h in range(hk * G, (hk + 1) * G):
                qr = q[i, h].astype(np.float64) @ oc.r[0][0]
                want = O.attend(qr, kx[sel], vx[sel]) @ oc.r[1][0].T
                err = np.abs(got[i, h] - want).max() / np.abs(want).max()
                assert err <= TOL, (hk, i, h, err)
