"""Quantisation groups smaller than the head: 64 and 32 channels.

With one 128-channel group per vector the bit-reversal permutation cannot
change the codes (min and max do not depend on the order); with smaller
groups it decides which channels share a scale, which is what the pages
introduce it for (gen-hub.ru, "Together AI открывает OSCAR…", section "Что
придумали в Together AI").  The CUDA path through the C ABI against the
oracle's per-group quantiser and decode, on the same seeded inputs:

* pre-rotated append: codes, per-group fp16 scales and minima, fp16 window
  rows bit-exact (generator vectors plus the quantiser's edge cases);
* fused rotate+quantise on all three append kernels: codes, scales and
  minima bit-exact against the oracle's quantiser on the kernel's own fp32
  rotation;
* gather/dequantise bit-exact;
* decode within 2e-3 on the tiny single-layer workload (4 query heads on 1
  KV head, 2048 tokens) and at the decode benchmark's head shape (32 / 8) at
  100,000 tokens;
* the tensor-core split-K kernel's grouped layouts (per-group score MMAs and
  value m-tiles) at every head grouping it takes (G = 1, 2, 4 on 8, 2 or 1 KV
  heads, so that one warp or several serve a head; G = 8 and 16 as two and
  four CTAs per range of four query heads each), with and without sinks,
  over lengths that end inside a block, at a block edge, inside and past the
  fp16 window;
* a peaked case: one INT2 key 10 nats above a flat 30,000-token context, at
  the start and in the middle of a split, so that the per-group P' of the
  tail behind it keeps its precision.
"""
import math
import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3
GROUPS = (64, 32)


def _okv():
    from int2_kv_cache_rotate_b200 import okv
    return okv


def _t(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _fill_pre_rotated(seed, hq, hkv, lens, group, special=False):
    okv = _okv()
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv, group=group)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), group=group)
    zs = {0: [], 1: []}
    for kind in (0, 1):
        for b, n in enumerate(lens):
            z = np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], axis=1) \
                if n else np.zeros((0, hkv, 128), np.float32)
            if special and n:
                sp = H.special_vectors()
                m = min(n, sp.shape[0])
                z[:m, 0, :] = sp[:m]
                # the same rows with their halves swapped: each group sees other extremes
                m2 = min(n - m, sp.shape[0])
                if m2 > 0:
                    z[m:m + m2, 0, :] = np.roll(sp[:m2], 64, axis=1)
            zs[kind].append(z)
    for b, n in enumerate(lens):
        if n:
            oc.append(b, 0, zs[0][b], zs[1][b], pre_rotated=True)
    slots, pos = lay.flat()
    k = np.concatenate([z for z in zs[0] if len(z)], axis=0)
    v = np.concatenate([z for z in zs[1] if len(z)], axis=0)
    okv.append_quantize(gc, _t(k), _t(v), _t(slots), _t(pos), _t(lay.table), _t(np.array(lens, np.int32)),
                        pre_rotated=True)
    torch.cuda.synchronize()
    return gc, oc, lay


@pytest.mark.parametrize("group", GROUPS)
def test_grouped_append_pre_rotated_bit_exact(group):
    lens = [1, 5, 127, 128, 129, 300, 2048]
    hkv = 2
    gc, oc, lay = _fill_pre_rotated(41, 4, hkv, lens, group, special=True)
    assert gc.block_head_bytes == 1024 + 128 * (128 // group)
    assert gc.device_status() == 0
    pages = gc.pages.cpu().numpy()
    ring = gc.ring.cpu().numpy()
    for b, n in enumerate(lens):
        for h in range(hkv):
            for kind in (0, 1):
                packed, s16, m16 = H.gather_codes_grouped(pages, lay.table, b, h, hkv, n, kind, group)
                st = oc.seqs[(b, kind, h)]
                assert np.array_equal(packed, O.pack(st["codes"][:n])), (b, h, kind)
                assert np.array_equal(s16.view(np.uint16), st["s16"][:n].view(np.uint16)), (b, h, kind)
                assert np.array_equal(m16.view(np.uint16), st["m16"][:n].view(np.uint16)), (b, h, kind)
                for p in range(max(0, n - 128), n):
                    assert np.array_equal(ring[b, h, kind, p % 128].view(np.uint16), st["z16"][p].view(np.uint16))


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("lens,misalign", [
    ([30, 7], False),     # 37 tokens: CUDA-core kernel
    ([700, 45], False),   # 745 tokens: tcgen05 kernel, ragged last tile
    ([700, 45], True),    # not 16-byte aligned: the mma.sync tensor-core kernel
])
def test_grouped_fused_rotation_codes_bit_exact(group, lens, misalign):
    okv = _okv()
    seed, hq, hkv = 43, 8, 2
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv, group=group)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), group=group)
    k = [np.stack([WL.sample_keys(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1) for b, n in enumerate(lens)]
    v = [np.stack([WL.sample_values(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1) for b, n in enumerate(lens)]
    slots, pos = lay.flat()
    rot = torch.zeros((len(slots), 2, hkv, 128), dtype=torch.float32, device="cuda")
    kd, vd = _t(np.concatenate(k), torch.bfloat16), _t(np.concatenate(v), torch.bfloat16)
    if misalign:
        kd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), kd.flatten()])[2:].view(kd.shape)
        vd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), vd.flatten()])[2:].view(vd.shape)
        assert kd.data_ptr() % 16 == 4
    okv.append_quantize(gc, kd, vd, _t(slots), _t(pos), _t(lay.table), _t(np.array(lens, np.int32)), rotated_out=rot)
    rot = rot.cpu().numpy()
    pages = gc.pages.cpu().numpy()
    assert gc.device_status() == 0
    off = 0
    for b, n in enumerate(lens):
        for h in range(hkv):
            for kind, x in ((0, k[b]), (1, v[b])):
                zg = rot[off:off + n, kind, h, :]
                z64 = x[:, h, :].astype(np.float64) @ oc.r[kind][h]
                assert (np.abs(zg - z64).max(axis=1) / np.abs(z64).max(axis=1)).max() < 1e-5
                c_self, s_self, m_self = O.quantize(zg, group)
                packed, s16, m16 = H.gather_codes_grouped(pages, lay.table, b, h, hkv, n, kind, group)
                assert np.array_equal(O.unpack(packed), c_self), (b, h, kind)
                assert np.array_equal(s16.view(np.uint16), s_self.view(np.uint16)), (b, h, kind)
                assert np.array_equal(m16.view(np.uint16), m_self.view(np.uint16)), (b, h, kind)
        off += n


@pytest.mark.parametrize("group", GROUPS)
def test_grouped_dequantize_bit_exact(group):
    okv = _okv()
    lens = [300, 17, 0, 144]
    hkv = 2
    gc, oc, lay = _fill_pre_rotated(44, 4, hkv, lens, group)
    args = (_t(np.arange(len(lens), dtype=np.int32)), _t(lay.table), _t(np.array(lens, np.int32)))
    for which in (0, 1):
        rot = okv.dequantize(gc, *args, 320, which, basis=0, source=0).cpu().numpy()
        win = okv.dequantize(gc, *args, 320, which, basis=0, source=1).cpu().numpy()
        for b, n in enumerate(lens):
            for h in range(hkv):
                if n == 0:
                    continue
                st = oc.seqs[(b, which, h)]
                want = O.dequantize(st["codes"][:n], st["s16"][:n], st["m16"][:n], group)
                assert np.array_equal(rot[b, h, :n], want)
                assert np.array_equal(win[b, h, :n], oc.values(b, which, h, n).astype(np.float32))


@pytest.mark.parametrize("group", GROUPS)
def test_grouped_decode_tiny_workload(group):
    """1 sequence, 4 query heads on 1 KV head, 2048 tokens."""
    okv = _okv()
    seed, hq, hkv, n = 45, 4, 1, 2048
    gc, oc, lay = _fill_pre_rotated(seed, hq, hkv, [n], group)
    q = WL.sample_queries(seed, 0, 0, 0, 1, hq).reshape(1, hq, 128)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(np.zeros(1, np.int32)), _t(lay.table),
                               _t(np.array([n], np.int32))).cpu().numpy()
    want = O.decode(oc, q, [0], [n], hq)
    assert H.rel_err_rows(got, want).max() <= TOL
    assert gc.device_status() == 0


@pytest.mark.parametrize("group", GROUPS)
def test_grouped_decode_100k_bench_heads(group):
    """The decode benchmark's head shape (32 query / 8 KV heads) at 100,000
    tokens, two sequences; sampled (sequence, KV head) pairs get host data,
    the rest device random numbers (heads never mix)."""
    from tests.test_gpu_fullsize import _Pool, _d, _queries
    okv = _okv()
    seed, cfg, B, hq, hkv, L = 46, 2, 2, 32, 8, 100_000
    G = hq // hkv
    sampled = [(0, 0), (1, 5)]
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, [L] * B, extra_tokens=16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv, group=group)
    table_d = _d(table)
    host = {(b, h, kind): WL.sample_rotated(seed, cfg, 0, h, L, kind, extra=b) for (b, h) in sampled for kind in (0, 1)}
    pool = _Pool(hkv, seed)
    lens_d = _d(np.full(B, L, np.int32))
    for b in range(B):
        for p0 in range(0, L, pool.k.shape[0]):
            m = min(pool.k.shape[0], L - p0)
            k, v = pool.k[:m].clone(), pool.v[:m].clone()
            for (bb, h) in sampled:
                if bb == b:
                    k[:, h] = _d(host[(b, h, 0)][p0:p0 + m])
                    v[:, h] = _d(host[(b, h, 1)][p0:p0 + m])
            okv.append_quantize(cache, k, v, torch.full((m,), b, dtype=torch.int32, device="cuda"),
                                torch.arange(p0, p0 + m, dtype=torch.int32, device="cuda"), table_d, lens_d,
                                pre_rotated=True)
    q = _queries(seed, cfg, 0, hkv, B, G, extra=4)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.arange(B, dtype=np.int32)), table_d,
                               lens_d).cpu().numpy()
    for (b, h) in sampled:
        oc = O.Cache(1, uk[h:h + 1].astype(np.float64), uv[h:h + 1].astype(np.float64), group=group)
        oc.append(0, 0, host[(b, h, 0)][:, None, :], host[(b, h, 1)][:, None, :], pre_rotated=True)
        want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [L], G)
        assert H.rel_err_rows(got[b:b + 1, h * G:(h + 1) * G], want).max() <= TOL, (b, h)
    assert cache.device_status() == 0


def _fill_groups_sinks(seed, hq, hkv, lens, group, nsink, plant=None):
    """GPU and oracle caches (group, sinks) from the same fp32 rotated vectors;
    plant(b, h, zk) may edit the rotated keys first."""
    okv = _okv()
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv, num_sink=nsink, group=group)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), sinks=nsink, group=group)
    zs = {kind: [np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], axis=1)
                 for b, n in enumerate(lens)] for kind in (0, 1)}
    if plant is not None:
        for b in range(len(lens)):
            for h in range(hkv):
                plant(b, h, zs[0][b][:, h], uk)
    for b, n in enumerate(lens):
        if n:
            oc.append(b, 0, zs[0][b], zs[1][b], pre_rotated=True)
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(np.concatenate(zs[0])), _t(np.concatenate(zs[1])), _t(slots), _t(pos),
                        _t(lay.table), _t(np.array(lens, np.int32)), pre_rotated=True)
    torch.cuda.synchronize()
    return gc, oc, lay


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("hq,hkv,nsink,lens", [
    (32, 8, 0, [1, 15, 16, 17, 100, 128, 129, 143, 300, 2000, 5003]),
    (16, 8, 16, [1, 16, 17, 144, 145, 400, 3000]),       # G = 2
    (8, 8, 32, [31, 33, 160, 161, 1000, 4100]),          # G = 1
    (8, 2, 0, [0, 47, 129, 900, 6000]),                  # G = 4, 4 warps per KV head (merged)
    (4, 1, 48, [49, 176, 177, 2500]),                    # G = 4, 8 warps per KV head
    (64, 8, 0, [1, 17, 129, 300, 4000]),                 # G = 8: two CTAs per range, four heads each
    (16, 2, 16, [16, 33, 145, 2000]),                    # G = 8 on 2 KV heads (merged), sinks
    (32, 2, 0, [5, 129, 1500]),                          # G = 16: four CTAs per range
])
def test_grouped_decode_tensor_core_shapes(group, hq, hkv, nsink, lens):
    okv = _okv()
    seed = 70 + nsink + hq
    gc, oc, lay = _fill_groups_sinks(seed, hq, hkv, lens, group, nsink)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=9) for h in range(hkv)], 1)
    q = q.reshape(len(lens), hq, 128)
    seq = np.arange(len(lens), dtype=np.int32)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), _t(lay.table),
                               _t(np.array(lens, np.int32))).cpu().numpy()
    assert gc.device_status() == 0
    live = [i for i, n in enumerate(lens) if n > 0]
    want = O.decode(oc, q[live], seq[live], [lens[i] for i in live], hq)
    err = H.rel_err_rows(got[live], want)
    assert err.max() <= TOL, (err.max(), np.unravel_index(err.argmax(), err.shape))


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("where", [5, 17_011])
def test_grouped_decode_peaked_tail(group, where):
    """One INT2 key per (sequence, KV head), aligned with the first query head
    of the group, 10 nats above an otherwise flat context of 30,000 tokens."""
    okv = _okv()
    seed, hq, hkv, L, gap = 90 + where % 7, 32, 8, 30_000, 10.0
    G = hq // hkv
    lens = [L, L]
    q = np.stack([WL.sample_queries(seed, 0, 0, h, 2, G, extra=11) for h in range(hkv)], 1).reshape(2, hq, 128)

    def plant(b, h, zk, uk):
        q_rot = q[b, h * G].astype(np.float64) @ O.rotation(uk[h].astype(np.float64))
        direction = q_rot / np.linalg.norm(q_rot)
        alpha = gap * math.sqrt(128) / np.linalg.norm(q_rot)
        for _ in range(6):
            row = (alpha * direction).astype(np.float32)
            c, s_, m_ = O.quantize(row[None], group)
            logit = O.dequantize(c, s_, m_, group)[0].astype(np.float64) @ q_rot / math.sqrt(128)
            alpha *= gap / logit
        zk[where] = row

    gc, oc, lay = _fill_groups_sinks(seed, hq, hkv, lens, group, 0, plant=plant)
    seq = np.arange(2, dtype=np.int32)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), _t(lay.table),
                               _t(np.array(lens, np.int32))).cpu().numpy()
    assert gc.device_status() == 0
    want = O.decode(oc, q, seq, lens, hq)
    err = H.rel_err_rows(got, want)
    assert err.max() <= TOL, (err.max(), np.unravel_index(err.argmax(), err.shape))
