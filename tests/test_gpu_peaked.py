"""Decode parity on peaked attention over a long INT2 history.

One INT2-position key per checked (sequence, KV head) is aligned with the
first query head of its group, so that its logit sits `gap` nats (6 to 12)
above an otherwise flat context; the first 5 or about 40,000 positions
before it.  This is the shape of an attention sink or a retrieval token with
a long tail behind it (the pages keep sink tokens 16-bit, but with no sinks
configured such a token lives in INT2: encorp.ai, "KV cache compression е
инфраструктурно решение…", section "OSCAR има значение…").  In the split-K
kernel the dominant token sets the running maximum of its range, and every
later token of that range is weighted against it: the tail's weights must
keep their precision, and the outputs must stay within 2e-3 of the oracle.

Workloads: the decode benchmark (4 x 100,000 tokens, 32 query / 8 KV heads,
no sinks, one fused one-token append per sequence, then decode, in the
benchmark's launch configuration) and a 70B-class layer (1 x 131,072 tokens,
64 / 8 heads, G = 8).
"""
import math

import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H
from tests.test_gpu_fullsize import _Pool, _check, _d, _fill, _okv, _oracle_head, _queries

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GAPS = (6.0, 8.0, 10.0, 12.0)


def _plant(zk, pos, q_rot, gap):
    """Overwrite rotated key `pos` with a multiple of q_rot whose INT2
    dequantised logit q_rot . k / sqrt(d) is `gap` (to within 1e-3)."""
    direction = q_rot / np.linalg.norm(q_rot)
    alpha = gap * math.sqrt(128) / np.linalg.norm(q_rot)
    for _ in range(6):
        row = (alpha * direction).astype(np.float32)
        c, s, m = O.quantize(row[None])
        logit = O.dequantize(c, s, m)[0].astype(np.float64) @ q_rot / math.sqrt(128)
        alpha *= gap / logit
    zk[pos] = row
    return logit


def _dominant_share(oc, q_rot, length, pos):
    kx = oc.values(0, 0, 0, length)
    lg = kx @ q_rot / math.sqrt(128)
    w = np.exp(lg - lg.max())
    return w[pos] / w.sum(), lg[pos] - np.median(lg)


@pytest.mark.parametrize("where", ["range-start", "mid-range"])
def test_peaked_decode_100k_bench_step(where):
    okv = _okv()
    seed, cfg = 40 if where == "range-start" else 41, 2
    wl = WL.config(cfg)
    B, hq, hkv, L0 = wl.batch, wl.hq, wl.hkv, wl.ctx[0]
    G = hq // hkv
    plan = [((0, 0), GAPS[0]), ((1, 3), GAPS[1]), ((2, 5), GAPS[2]), ((3, 7), GAPS[3])]
    pos_of = {bh: (5 if where == "range-start" else 40_017 + 1_111 * bh[0]) for bh, _ in plan}
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, [L0] * B, extra_tokens=1 + 16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv)
    table_d = _d(table)
    q = _queries(seed, cfg, 0, hkv, B, G, extra=60)
    host = {}
    for (b, h), gap in plan:
        zk = WL.sample_rotated(seed, cfg, 0, h, L0, 0, extra=b)
        zv = WL.sample_rotated(seed, cfg, 0, h, L0, 1, extra=b)
        q_rot = q[b, h * G].astype(np.float64) @ O.rotation(uk[h].astype(np.float64))
        _plant(zk, pos_of[(b, h)], q_rot, gap)
        host[(b, h, 0)], host[(b, h, 1)] = zk, zv
    sampled = [bh for bh, _ in plan]
    _fill(cache, table_d, [L0] * B, [L0] * B, sampled, host, _Pool(hkv, seed))
    # the benchmark's step: one bf16 token appended per sequence, then decode
    knew = np.stack([np.stack([WL.sample_keys(seed, cfg, 0, h, 1, extra=200 + b)[0] for h in range(hkv)])
                     for b in range(B)])
    vnew = np.stack([np.stack([WL.sample_values(seed, cfg, 0, h, 1, extra=200 + b)[0] for h in range(hkv)])
                     for b in range(B)])
    pos = np.full(B, L0, np.int32)
    lens = pos + 1
    seq = _d(np.arange(B, dtype=np.int32))
    ws = okv.workspace(cache, B)
    out = okv.decode_step(cache, _d(knew).to(torch.bfloat16), _d(vnew).to(torch.bfloat16), seq, _d(pos), _d(lens),
                          _d(q).to(torch.bfloat16), seq, table_d, _d(lens), ws=ws)
    got = out.cpu().numpy()
    for (b, h), gap in plan:
        oc = _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)])
        oc.append(0, L0, knew[b, h][None, None], vnew[b, h][None, None])
        want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [int(lens[b])], G)
        share, lift = _dominant_share(oc, q[b, h * G].astype(np.float64) @ oc.r[0][0], int(lens[b]),
                                      pos_of[(b, h)])
        assert abs(lift - gap) < 0.2, (gap, lift)  # the planted token sits where it should
        expect = math.exp(gap) / (math.exp(gap) + L0 * 1.1)
        assert 0.5 * expect < share < 2.0 * expect, (gap, share, expect)
        _check(got[b:b + 1, h * G:(h + 1) * G], want, (where, b, h, gap))
    assert cache.device_status() == 0


def test_peaked_decode_70b_layer_131k():
    """G = 8 (two score n-tiles per warp), 131,072 tokens, one sequence:
    dominant tokens at the start of the history and in the middle of it."""
    okv = _okv()
    seed, cfg = 42, 3
    wl = WL.config(cfg)
    hq, hkv, L = wl.hq, wl.hkv, wl.ctx[0]
    G = hq // hkv
    plan = [((0, 0), 8.0, 5), ((0, 5), 10.0, 70_001), ((0, 2), 6.0, 9), ((0, 7), 12.0, 99_999)]
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, [L], extra_tokens=16)
    cache = okv.Cache(hq, hkv, nb, 1, table.shape[1], uk, uv)
    table_d = _d(table)
    q = _queries(seed, cfg, 0, hkv, 1, G, extra=61)
    host = {}
    for (b, h), gap, p in plan:
        zk = WL.sample_rotated(seed, cfg, 0, h, L, 0, extra=b)
        zv = WL.sample_rotated(seed, cfg, 0, h, L, 1, extra=b)
        # a different query head of the group in each case (the second n-tile too)
        hh = h * G + (h % G)
        q_rot = q[0, hh].astype(np.float64) @ O.rotation(uk[h].astype(np.float64))
        _plant(zk, p, q_rot, gap)
        host[(b, h, 0)], host[(b, h, 1)] = zk, zv
    _fill(cache, table_d, [L], [L], [bh for bh, _, _ in plan], host, _Pool(hkv, seed))
    lens = np.array([L], np.int32)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.zeros(1, np.int32)), table_d,
                               _d(lens)).cpu().numpy()
    for (b, h), gap, p in plan:
        oc = _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)])
        want = O.decode(oc, q[:, h * G:(h + 1) * G], [0], [L], G)
        _, lift = _dominant_share(oc, q[0, h * G + (h % G)].astype(np.float64) @ oc.r[0][0], L, p)
        assert abs(lift - gap) < 0.2, (gap, lift)
        _check(got[:, h * G:(h + 1) * G], want, (h, gap, p))
    assert cache.device_status() == 0
