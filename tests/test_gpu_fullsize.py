"""Parity at the full workload sizes, in the launch configuration the
benchmark uses, on sampled outputs the oracle computes one by one.

Every (sequence, KV head) pair that is checked gets host-seeded rotated
vectors (the oracle's inputs) through the pre-rotated append; every other
head is filled with device random numbers, and its outputs are not read.
Heads never mix in attention, so the sampled outputs depend on the host data
alone.  The bench-shaped step (a fused bf16 append of one token per
sequence, then decode) runs exactly as the benchmark runs it.

Workloads (seeded, synthetic; shapes from the pages' evaluation settings):
* 4 sequences x 100,000 tokens, 32 query / 8 KV heads (the decode benchmark),
  without sinks and with 192 sink tokens;
* 2 sequences at 1, 2 and 4 KV heads, long enough that every split-K CTA
  streams about ten ring stages;
* 8 sequences x 32,768 tokens, 32 / 8 heads (an 8B-class layer);
* 80 layers x 131,072 tokens, 64 / 8 heads (a 70B-class model, G = 8),
  one workspace reused across all 80 layer launches;
* 64 sequences with log-uniform lengths in [1K, 64K], 32 / 8 heads, plus one
  8192-token fused prefill chunk (the tensor-core append).
"""
import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-3
CHUNK = 32768


def _okv():
    from int2_kv_cache_rotate_b200 import okv
    return okv


def _d(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


class _Pool:
    """Device random rows for the heads whose outputs are not checked."""

    def __init__(self, hkv, seed):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        self.k = torch.randn((CHUNK, hkv, 128), generator=g, device="cuda")
        self.v = torch.randn((CHUNK, hkv, 128), generator=g, device="cuda")


def _fill(cache, table_d, lens, fill_lens, sampled, host, pool):
    """Pre-rotated fill of positions [0, fill_lens[b]) of every sequence;
    slot lengths are `lens` (the window covers the last 128 of those)."""
    okv = _okv()
    lens_d = _d(np.asarray(lens, np.int32))
    for b, n in enumerate(fill_lens):
        for p0 in range(0, n, CHUNK):
            m = min(CHUNK, n - p0)
            k, v = pool.k[:m].clone(), pool.v[:m].clone()
            for (bb, h) in sampled:
                if bb == b:
                    k[:, h] = _d(host[(b, h, 0)][p0:p0 + m])
                    v[:, h] = _d(host[(b, h, 1)][p0:p0 + m])
            okv.append_quantize(cache, k, v, torch.full((m,), b, dtype=torch.int32, device="cuda"),
                                torch.arange(p0, p0 + m, dtype=torch.int32, device="cuda"), table_d, lens_d,
                                pre_rotated=True)


def _oracle_head(uk, uv, h, zk, zv, sinks=0):
    oc = O.Cache(1, uk[h:h + 1].astype(np.float64), uv[h:h + 1].astype(np.float64), sinks=sinks)
    oc.append(0, 0, zk[:, None, :], zv[:, None, :], pre_rotated=True)
    return oc


def _queries(seed, cfg, layer, hkv, B, G, extra):
    q = np.stack([WL.sample_queries(seed, cfg, layer, h, B, G, extra=extra) for h in range(hkv)], 1)
    return q.reshape(B, hkv * G, 128)


def _check(got, want, what):
    err = H.rel_err_rows(got, want)
    assert err.max() <= TOL, (what, err.max())
    return err.max()


@pytest.mark.parametrize("sinks", [0, 192])
def test_fullsize_decode_100k_bench_step(sinks):
    """4 x 100,000 tokens: prefill, then two benchmark steps through
    okv_decode_step (one-token bf16 append per sequence and decode over the
    grown context, the call the benchmark times); without sinks, and with the
    192 sink tokens that keep 0.24 % of a 128K context 16-bit."""
    okv = _okv()
    seed, cfg = 5 + sinks, 2
    wl = WL.config(cfg)
    B, hq, hkv, L0 = wl.batch, wl.hq, wl.hkv, wl.ctx[0]
    G = hq // hkv
    steps = 2
    sampled = [(0, 0), (1, 3), (2, 5), (3, 7)]
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, [L0] * B, extra_tokens=steps + 16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv, num_sink=sinks)
    table_d = _d(table)
    host = {(b, h, kind): WL.sample_rotated(seed, cfg, 0, h, L0, kind, extra=b)
            for (b, h) in sampled for kind in (0, 1)}
    _fill(cache, table_d, [L0] * B, [L0] * B, sampled, host, _Pool(hkv, seed))
    oracles = {(b, h): _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)], sinks) for (b, h) in sampled}
    ws = okv.workspace(cache, B)
    seq = _d(np.arange(B, dtype=np.int32))
    for i in range(steps):
        knew = np.stack([np.stack([WL.sample_keys(seed, cfg, 0, h, 1, extra=100 + 10 * i + b)[0]
                                   for h in range(hkv)]) for b in range(B)])
        vnew = np.stack([np.stack([WL.sample_values(seed, cfg, 0, h, 1, extra=100 + 10 * i + b)[0]
                                   for h in range(hkv)]) for b in range(B)])
        pos = np.full(B, L0 + i, np.int32)
        lens = pos + 1
        q = _queries(seed, cfg, 0, hkv, B, G, extra=50 + i)
        # the benchmark's call: append one token per sequence, then decode
        out = okv.decode_step(cache, _d(knew).to(torch.bfloat16), _d(vnew).to(torch.bfloat16), seq, _d(pos),
                              _d(lens), _d(q).to(torch.bfloat16), seq, table_d, _d(lens), ws=ws)
        got = out.cpu().numpy()
        for (b, h) in sampled:
            oc = oracles[(b, h)]
            oc.append(0, L0 + i, knew[b, h][None, None], vnew[b, h][None, None])
            want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [int(lens[b])], G)
            _check(got[b:b + 1, h * G:(h + 1) * G], want, (i, b, h))
    assert cache.device_status() == 0


@pytest.mark.parametrize("hq,hkv,L", [(4, 1, 400_000), (8, 2, 200_000), (16, 4, 100_000)])
def test_long_ranges_every_kv_head_count(hq, hkv, L):
    """With fewer KV heads a ring stage holds more blocks (16 / Hkv), so the
    split-K producer's batches, its prologue split at block-id window
    boundaries and its window refills take other paths than at 8 KV heads.
    Two sequences sized so that every CTA streams about ten stages."""
    okv = _okv()
    seed, cfg, B = 9, 2, 2
    G = hq // hkv
    sampled = [(0, 0), (1, hkv - 1)]
    uk, uv = H.rotations(seed + hkv, hkv)
    table, nb = WL.block_table(seed + hkv, cfg, [L] * B, extra_tokens=16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv)
    table_d = _d(table)
    host = {(b, h, kind): WL.sample_rotated(seed + hkv, cfg, 0, h, L, kind, extra=b)
            for (b, h) in sampled for kind in (0, 1)}
    _fill(cache, table_d, [L] * B, [L] * B, sampled, host, _Pool(hkv, seed))
    q = _queries(seed + hkv, cfg, 0, hkv, B, G, extra=3)
    lens = np.full(B, L, np.int32)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.arange(B, dtype=np.int32)), table_d,
                               _d(lens)).cpu().numpy()
    for (b, h) in sampled:
        oc = _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)])
        want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [L], G)
        _check(got[b:b + 1, h * G:(h + 1) * G], want, (hkv, b, h))
    assert cache.device_status() == 0


def test_fullsize_decode_8b_layer_32k():
    okv = _okv()
    seed, cfg = 6, 1
    wl = WL.config(cfg)
    B, hq, hkv, L = wl.batch, wl.hq, wl.hkv, wl.ctx[0]
    G = hq // hkv
    sampled = [(0, 0), (3, 4), (7, 7), (5, 2)]
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, [L] * B, extra_tokens=16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv)
    table_d = _d(table)
    host = {(b, h, kind): WL.sample_rotated(seed, cfg, 0, h, L, kind, extra=b)
            for (b, h) in sampled for kind in (0, 1)}
    _fill(cache, table_d, [L] * B, [L] * B, sampled, host, _Pool(hkv, seed))
    q = _queries(seed, cfg, 0, hkv, B, G, extra=1)
    lens = np.full(B, L, np.int32)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.arange(B, dtype=np.int32)), table_d,
                               _d(lens)).cpu().numpy()
    for (b, h) in sampled:
        oc = _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)])
        want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [L], G)
        _check(got[b:b + 1, h * G:(h + 1) * G], want, (b, h))
    assert cache.device_status() == 0


def test_fullsize_70b_shape_80_layers_131k():
    """80 layer caches, G = 8; one decode launch per layer on one stream with
    one shared workspace, as a model's decode step issues them."""
    okv = _okv()
    seed, cfg = 7, 3
    wl = WL.config(cfg)
    B, hq, hkv, L, layers = wl.batch, wl.hq, wl.hkv, wl.ctx[0], wl.layers
    G = hq // hkv
    checked = {0: 0, 37: 5, 79: 7}  # layer -> KV head
    pool = _Pool(hkv, seed)
    caches, rots, hosts = [], [], {}
    table, nb = WL.block_table(seed, cfg, [L], extra_tokens=16)
    table_d = _d(table)
    for layer in range(layers):
        uk, uv = H.rotations(seed + 1000 * layer, hkv)
        c = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv)
        sampled = [(0, checked[layer])] if layer in checked else []
        host = {(0, h, kind): WL.sample_rotated(seed, cfg, layer, h, L, kind) for (_, h) in sampled for kind in (0, 1)}
        _fill(c, table_d, [L], [L], sampled, host, pool)
        caches.append(c)
        rots.append((uk, uv))
        hosts.update({(layer,) + key: val for key, val in host.items()})
    ws = okv.workspace(caches[0], B)
    seq, lens_d = _d(np.zeros(1, np.int32)), _d(np.array([L], np.int32))
    qs = [_queries(seed, cfg, layer, hkv, B, G, extra=2) for layer in range(layers)]
    outs = [okv.decode_attention(caches[layer], _d(qs[layer]).to(torch.bfloat16), seq, table_d, lens_d, ws=ws)
            for layer in range(layers)]
    torch.cuda.synchronize()
    for layer, h in checked.items():
        uk, uv = rots[layer]
        oc = _oracle_head(uk, uv, h, hosts[(layer, 0, h, 0)], hosts[(layer, 0, h, 1)])
        want = O.decode(oc, qs[layer][:, h * G:(h + 1) * G], [0], [L], G)
        _check(outs[layer].cpu().numpy()[:, h * G:(h + 1) * G], want, (layer, h))
    for c in caches:
        assert c.device_status() == 0


def test_fullsize_mixed_64_sequences():
    okv = _okv()
    seed, cfg = 8, 4
    wl = WL.config(cfg, seed=seed)
    B, hq, hkv = wl.batch, wl.hq, wl.hkv
    lens = [int(x) for x in wl.ctx]
    G = hq // hkv
    order = np.argsort(lens)
    sampled = [(int(order[0]), 1), (int(order[-1]), 6), (int(order[B // 2]), 3), (17, 0)]
    uk, uv = H.rotations(seed, hkv)
    table, nb = WL.block_table(seed, cfg, lens, extra_tokens=16)
    cache = okv.Cache(hq, hkv, nb, B, table.shape[1], uk, uv)
    table_d = _d(table)
    host = {(b, h, kind): WL.sample_rotated(seed, cfg, 0, h, lens[b], kind, extra=b)
            for (b, h) in sampled for kind in (0, 1)}
    _fill(cache, table_d, lens, lens, sampled, host, _Pool(hkv, seed))
    q = _queries(seed, cfg, 0, hkv, B, G, extra=3)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.arange(B, dtype=np.int32)), table_d,
                               _d(np.asarray(lens, np.int32))).cpu().numpy()
    for (b, h) in sampled:
        oc = _oracle_head(uk, uv, h, host[(b, h, 0)], host[(b, h, 1)])
        want = O.decode(oc, q[b:b + 1, h * G:(h + 1) * G], [0], [lens[b]], G)
        _check(got[b:b + 1, h * G:(h + 1) * G], want, (b, h, lens[b]))
    assert cache.device_status() == 0


def test_fullsize_prefill_chunk_8192_fused():
    """One 8192-token bf16 prefill chunk (all 8 KV heads, K and V) through the
    fused rotate+quantise kernel: sampled tokens' rotation within 1e-5 of the
    fp64 oracle, and their codes equal to the oracle's except where the
    oracle shows the decision within rounding distance of a midpoint."""
    okv = _okv()
    seed, cfg = 9, 4
    n, hq, hkv = 8192, 32, 8
    table, nb = WL.block_table(seed, cfg, [n])
    r = np.random.default_rng(np.random.SeedSequence([seed, 77]))
    uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    uv = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    cache = okv.Cache(hq, hkv, nb, 1, table.shape[1], uk, uv)
    k = np.stack([WL.sample_keys(seed, cfg, 0, h, n) for h in range(hkv)], 1)
    v = np.stack([WL.sample_values(seed, cfg, 0, h, n) for h in range(hkv)], 1)
    rot = torch.zeros((n, 2, hkv, 128), dtype=torch.float32, device="cuda")
    okv.append_quantize(cache, _d(k).to(torch.bfloat16), _d(v).to(torch.bfloat16), _d(np.zeros(n, np.int32)),
                        _d(np.arange(n, dtype=np.int32)), _d(table), _d(np.array([n], np.int32)), rotated_out=rot)
    rot = rot.cpu().numpy()
    pages = cache.pages.cpu().numpy()
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    tok = np.unique(np.concatenate([np.arange(0, n, 97), [n - 1]]))
    for h in range(hkv):
        for kind, x in ((0, k), (1, v)):
            z64 = x[tok, h, :].astype(np.float64) @ oc.r[kind][h]
            zg = rot[tok, kind, h, :]
            err = np.abs(zg - z64).max(axis=1) / np.abs(z64).max(axis=1)
            assert err.max() < 1e-5, (h, kind, err.max())
            packed, s16, m16 = H.gather_codes(pages, table, 0, h, hkv, n, kind)
            c_gpu = O.unpack(packed[tok])
            # the GPU's own fp32 rotated values decide its codes bit-exactly
            c_self, s_self, m_self = O.quantize(zg)
            assert np.array_equal(c_gpu, c_self)
            assert np.array_equal(s16[tok].view(np.uint16), s_self.view(np.uint16))
            assert np.array_equal(m16[tok].view(np.uint16), m_self.view(np.uint16))
            # against the fp64 rotation: equal except at ambiguous decisions
            c_ref, _, _ = O.quantize(z64.astype(np.float32))
            amb = H.ambiguity_bound(z64, 2e-5)
            assert not np.any((c_gpu != c_ref) & ~amb)
    assert cache.device_status() == 0
