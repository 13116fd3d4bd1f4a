"""Attention-sink tokens on the GPU against the oracle.

The first S positions of every sequence are kept in fp16 as well as in INT2,
and decode reads them from fp16 (the pages keep sink and recent tokens
16-bit; S is a cache parameter).  Checks:

* append: the sink rows hold fp16(z) of exactly the positions below S, bit
  for bit, through the CUDA-core append, the tcgen05 prefill append (16-byte
  aligned K/V) and the mma.sync append (K/V off that alignment);
* decode: within 2e-3 of the oracle for lengths on both sides of S, S + 16,
  S + W and where the sink rows and the window overlap, on the tensor-core
  split-K kernel (G = 4 and 8, 8 and 2 KV heads) and the CUDA-core one (G = 16);
* the fused decode step appending tokens below, at and above S;
* gather/dequantise "as decode reads it": bit-exact with the oracle's view.
"""
import copy

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


def _fill(seed, hq, hkv, lens, nsink):
    """GPU and oracle caches with `nsink` sinks, filled from the same fp32 rotated vectors."""
    okv = _okv()
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv, num_sink=nsink)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), sinks=nsink)
    zs = {kind: [np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], axis=1)
                 for b, n in enumerate(lens)] for kind in (0, 1)}
    for b, n in enumerate(lens):
        oc.append(b, 0, zs[0][b], zs[1][b], pre_rotated=True)
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(np.concatenate(zs[0])), _t(np.concatenate(zs[1])), _t(slots), _t(pos),
                        _t(lay.table), _t(np.array(lens, np.int32)), pre_rotated=True)
    torch.cuda.synchronize()
    return gc, oc, lay


@pytest.mark.parametrize("hq,hkv,nsink,lens", [
    (32, 8, 16, [1, 15, 16, 17, 100, 143, 144, 145, 300, 2000]),
    (32, 8, 192, [1, 100, 191, 192, 193, 319, 320, 321, 400, 3000]),
    (64, 8, 64, [50, 192, 193, 1500]),
    (8, 2, 48, [47, 48, 49, 176, 177, 900]),
    (16, 1, 32, [20, 160, 161, 700]),
])
def test_decode_parity_with_sinks(hq, hkv, nsink, lens):
    okv = _okv()
    seed = 31 + nsink
    gc, oc, lay = _fill(seed, hq, hkv, lens, nsink)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=7) for h in range(hkv)], 1)
    q = q.reshape(len(lens), hq, 128)
    seq = np.arange(len(lens), dtype=np.int32)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), _t(lay.table),
                               _t(np.array(lens, np.int32))).cpu().numpy()
    want = O.decode(oc, q, seq, lens, hq)
    assert gc.device_status() == 0
    err = H.rel_err_rows(got, want)
    assert err.max() <= TOL, (err.max(), np.unravel_index(err.argmax(), err.shape))
    # the sinks matter: the oracle reading the same cache without them is farther off
    if max(lens) > nsink + O.W:
        plain = copy.copy(oc)
        plain.sinks = 0
        b = int(np.argmax(lens))
        err_plain = H.rel_err_rows(got[b:b + 1], O.decode(plain, q[b:b + 1], [b], [lens[b]], hq)).max()
        assert err_plain > max(3 * err[b].max(), TOL), (err_plain, err[b].max())


@pytest.mark.parametrize("n_tok,misalign", [(40, False), (300, False), (300, True)])
def test_append_writes_sink_rows_bit_exact(n_tok, misalign):
    """bf16 K/V through the rotating append: the sink rows of positions below
    S equal the fp16 (saturating, round-to-nearest) of the rotated vector the
    quantiser saw; rows at or above the sequence length stay untouched."""
    okv = _okv()
    seed, hq, hkv, nsink = 43, 8, 2, 64
    lens = [n_tok, 37]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv, num_sink=nsink)
    k = np.concatenate([np.stack([WL.sample_keys(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    v = np.concatenate([np.stack([WL.sample_values(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    kd, vd = _t(k, torch.bfloat16), _t(v, torch.bfloat16)
    if misalign:  # same values 4 bytes past a 16-byte boundary: the mma.sync append
        kd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), kd.flatten()])[2:].view(kd.shape)
        vd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), vd.flatten()])[2:].view(vd.shape)
    slots, pos = lay.flat()
    rot = torch.zeros((len(slots), 2, hkv, 128), dtype=torch.float32, device="cuda")
    okv.append_quantize(gc, kd, vd, _t(slots), _t(pos), _t(lay.table), _t(np.array(lens, np.int32)),
                        rotated_out=rot)
    torch.cuda.synchronize()
    assert gc.device_status() == 0
    rot = rot.cpu().numpy()
    sink = gc.sink.cpu().numpy()
    off = 0
    for b, n in enumerate(lens):
        m = min(n, nsink)
        for kind in (0, 1):
            for h in range(hkv):
                want = O.fp16_saturate(rot[off:off + m, kind, h, :])
                assert np.array_equal(sink[b, h, kind, :m].view(np.uint16), want.view(np.uint16)), (b, kind, h)
                assert not np.any(sink[b, h, kind, m:])
        off += n


def test_decode_step_across_the_sink_boundary():
    """The fused step (one bf16 token per sequence, then decode) with new
    positions just below, at and above S: the appended token lands in the sink
    rows exactly when its position is below S."""
    okv = _okv()
    seed, hq, hkv, nsink = 44, 32, 8, 32
    lens0 = [30, 31, 32, 200]
    steps = 3
    lay = H.Layout(seed, [n + steps for n in lens0])
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, lay.num_blocks, len(lens0), lay.mbps, uk, uv, num_sink=nsink)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), sinks=nsink)
    for b, n in enumerate(lens0):
        zk = np.stack([WL.sample_rotated(seed, 0, 0, h, n, 0, extra=b) for h in range(hkv)], 1)
        zv = np.stack([WL.sample_rotated(seed, 0, 0, h, n, 1, extra=b) for h in range(hkv)], 1)
        oc.append(b, 0, zk, zv, pre_rotated=True)
        okv.append_quantize(gc, _t(zk), _t(zv), _t(np.full(n, b, np.int32)), _t(np.arange(n, dtype=np.int32)),
                            _t(lay.table), _t(np.array(lens0, np.int32)), pre_rotated=True)
    ws = okv.workspace(gc, len(lens0))
    seq = _t(np.arange(len(lens0), dtype=np.int32))
    table = _t(lay.table)
    B = len(lens0)
    for i in range(steps):
        knew = np.stack([np.stack([WL.sample_keys(seed, 0, 0, h, 1, extra=100 + 10 * i + b)[0] for h in range(hkv)])
                         for b in range(B)])
        vnew = np.stack([np.stack([WL.sample_values(seed, 0, 0, h, 1, extra=100 + 10 * i + b)[0] for h in range(hkv)])
                         for b in range(B)])
        pos = np.array(lens0, np.int32) + i
        lens = pos + 1
        q = np.stack([WL.sample_queries(seed, 0, 0, h, B, hq // hkv, extra=20 + i) for h in range(hkv)], 1)
        q = q.reshape(B, hq, 128)
        got = okv.decode_step(gc, _t(knew, torch.bfloat16), _t(vnew, torch.bfloat16), seq, _t(pos), _t(lens),
                              _t(q, torch.bfloat16), seq, table, _t(lens), ws=ws).cpu().numpy()
        for b in range(B):
            oc.append(b, int(pos[b]), knew[b][None], vnew[b][None])
        want = O.decode(oc, q, np.arange(B), lens, hq)
        assert gc.device_status() == 0
        assert H.rel_err_rows(got, want).max() <= TOL, i


def test_dequantize_as_decode_reads_it_with_sinks():
    okv = _okv()
    lens = [300, 17, 70, 200]
    hkv, nsink = 2, 64
    gc, oc, lay = _fill(45, 4, hkv, lens, nsink)
    max_ctx = 320
    args = (_t(np.arange(len(lens), dtype=np.int32)), _t(lay.table), _t(np.array(lens, np.int32)))
    for which in (0, 1):
        rot = okv.dequantize(gc, *args, max_ctx, which, basis=0, source=0).cpu().numpy()
        seen = okv.dequantize(gc, *args, max_ctx, which, basis=0, source=1).cpu().numpy()
        for b, n in enumerate(lens):
            for h in range(hkv):
                st = oc.seqs[(b, which, h)]
                assert np.array_equal(rot[b, h, :n], O.dequantize(st["codes"][:n], st["s16"][:n], st["m16"][:n]))
                assert np.array_equal(seen[b, h, :n], oc.values(b, which, h, n).astype(np.float32))
                assert np.all(seen[b, h, n:] == 0)


@pytest.mark.parametrize("nsink", [0, 32])
def test_prefix_shared_pages(nsink):
    """Two sequences share the physical INT2 blocks of a common prefix (their
    block tables point at the same blocks), as a prefix cache forks a prompt;
    each then appends its own suffix into its own blocks.  The prefix is
    appended once; the fork's sink rows (per-sequence fp16) are filled by
    appending its first S tokens again, which rewrites identical codes into
    the shared blocks.  Both decode within 2e-3 of the oracle, and the shared
    blocks are left unchanged by the suffixes."""
    okv = _okv()
    seed, hq, hkv = 46, 32, 8
    prefix, suffix = 1024, [600, 300]  # prefix: 64 whole blocks
    G = hq // hkv
    lens = [prefix + s for s in suffix]
    nblk = [(n + 15) // 16 for n in lens]
    shared = prefix // 16
    rng = np.random.default_rng(seed)
    perm = rng.permutation(shared + sum(n - shared for n in nblk) + 3).astype(np.int32)
    table = np.full((2, max(nblk)), -1, np.int32)
    table[:, :shared] = perm[:shared]
    off = shared
    for b, n in enumerate(nblk):
        table[b, shared:n] = perm[off:off + n - shared]
        off += n - shared
    uk, uv = H.rotations(seed, hkv)
    gc = okv.Cache(hq, hkv, len(perm), 2, table.shape[1], uk, uv, num_sink=nsink)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64), sinks=nsink)
    zp = {kind: np.stack([WL.sample_rotated(seed, 0, 0, h, prefix, kind) for h in range(hkv)], 1) for kind in (0, 1)}
    zs = {(b, kind): np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=1 + b) for h in range(hkv)], 1)
          for b, n in enumerate(suffix) for kind in (0, 1)}
    lens_d, table_d = _t(np.array(lens, np.int32)), _t(table)

    def app(slot, p0, zk, zv):
        n = zk.shape[0]
        okv.append_quantize(gc, _t(zk), _t(zv), _t(np.full(n, slot, np.int32)),
                            _t(np.arange(p0, p0 + n, dtype=np.int32)), table_d, lens_d, pre_rotated=True)

    app(0, 0, zp[0], zp[1])                      # the prefix, once, through sequence 0
    if nsink:
        app(1, 0, zp[0][:nsink], zp[1][:nsink])  # the fork's own sink rows
    torch.cuda.synchronize()
    shared_before = gc.pages.view(len(perm), hkv * 1152)[torch.from_numpy(table[0, :shared]).long().cuda()].clone()
    for b in range(2):
        app(b, prefix, zs[(b, 0)], zs[(b, 1)])
        oc.append(b, 0, zp[0], zp[1], pre_rotated=True)
        oc.append(b, prefix, zs[(b, 0)], zs[(b, 1)], pre_rotated=True)
    torch.cuda.synchronize()
    shared_after = gc.pages.view(len(perm), hkv * 1152)[torch.from_numpy(table[0, :shared]).long().cuda()]
    assert torch.equal(shared_before, shared_after)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, 2, G, extra=9) for h in range(hkv)], 1).reshape(2, hq, 128)
    seq = np.arange(2, dtype=np.int32)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), table_d, lens_d).cpu().numpy()
    want = O.decode(oc, q, seq, lens, hq)
    assert gc.device_status() == 0
    assert H.rel_err_rows(got, want).max() <= TOL
