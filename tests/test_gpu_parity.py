"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

* quantiser, packing, paged placement and the fp16 window: bit-exact, with the
  rotated fp32 values handed to both sides (pre-rotated flag);
* fused rotate+quantise (all three append kernels): rotation within 1e-5 of
  the fp64 oracle; codes, scales and minima bit-exact against the oracle's
  quantiser fed the kernel's own fp32 rotation (nothing excused); against the
  oracle's own fp64 rotation the codes may differ only where the oracle shows
  the decision within rounding distance of a midpoint (reported as a rate);
* gather/dequantise: bit-exact in the rotated basis;
* decode attention: per (b, head) max |o - o_ref| / max |o_ref| <= 2e-3.
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


def _okv():
    from int2_kv_cache_rotate_b200 import okv
    return okv


def _t(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _gpu_cache(hq, hkv, lay: H.Layout, uk, uv, slots=None):
    okv = _okv()
    return okv.Cache(hq, hkv, lay.num_blocks, slots or len(lay.lens), lay.mbps, uk, uv)


def _fill_pre_rotated(seed, hq, hkv, lens, special=False, scale=1.0):
    """Both caches filled from the same fp32 rotated vectors."""
    okv = _okv()
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = _gpu_cache(hq, hkv, lay, uk, uv)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    zs = {}
    for kind in (0, 1):
        per_seq = []
        for b, n in enumerate(lens):
            z = np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b, scale=scale) for h in range(hkv)],
                         axis=1) if n else np.zeros((0, hkv, 128), np.float32)
            if special and n:
                sp = H.special_vectors()
                m = min(n, sp.shape[0])
                z[:m, 0, :] = sp[:m]
            per_seq.append(z)
        zs[kind] = per_seq
    for b, n in enumerate(lens):
        if n:
            oc.append(b, 0, zs[0][b], zs[1][b], pre_rotated=True)
    slots, pos = lay.flat()
    if len(slots):
        k = np.concatenate([z for z in zs[0] if len(z)], axis=0)
        v = np.concatenate([z for z in zs[1] if len(z)], axis=0)
        okv.append_quantize(gc, _t(k), _t(v), _t(slots), _t(pos), _t(lay.table), _t(np.array(lens, np.int32)),
                            pre_rotated=True)
    torch.cuda.synchronize()
    return gc, oc, lay, zs


@pytest.mark.parametrize("lens", [[2048], [1, 5, 127, 128, 129, 130, 143, 144, 145, 300]])
def test_append_pre_rotated_bit_exact(lens):
    hkv = 2
    gc, oc, lay, zs = _fill_pre_rotated(1, 4, hkv, lens, special=True)
    assert gc.device_status() == 0
    pages = gc.pages.cpu().numpy()
    ring = gc.ring.cpu().numpy()
    for b, n in enumerate(lens):
        for h in range(hkv):
            for kind in (0, 1):
                packed, s16, m16 = H.gather_codes(pages, lay.table, b, h, hkv, n, kind)
                st = oc.seqs[(b, kind, h)]
                assert np.array_equal(packed, O.pack(st["codes"][:n])), (b, h, kind)
                assert np.array_equal(s16.view(np.uint16), st["s16"][:n].view(np.uint16))
                assert np.array_equal(m16.view(np.uint16), st["m16"][:n].view(np.uint16))
                # window ring: the last min(n, W) positions, bit-exact fp16
                for p in range(max(0, n - 128), n):
                    row = ring[b, h, kind, p % 128]
                    assert np.array_equal(row.view(np.uint16), st["z16"][p].view(np.uint16)), (b, h, kind, p)


def test_quantizer_rounding_midpoints_bit_exact():
    """Groups built so that codes are decided by the last bit of the fp32
    division and by ties to even: the kernels' code decisions must match the
    oracle's division-based quantiser exactly."""
    okv = _okv()
    n = 3000
    rows = H.rounding_boundary_vectors(31, n)
    lay = H.Layout(31, [n])
    uk, uv = H.rotations(31, 1)
    gc = _gpu_cache(4, 1, lay, uk, uv)
    k, v = rows[:, None, :], rows[::-1].copy()[:, None, :]
    slots, pos = lay.flat()
    okv.append_quantize(gc, _t(k), _t(v), _t(slots), _t(pos), _t(lay.table), _t(np.array([n], np.int32)),
                        pre_rotated=True)
    pages = gc.pages.cpu().numpy()
    for kind, z in ((0, k[:, 0]), (1, v[:, 0])):
        c_ref, s_ref, m_ref = O.quantize(z)
        packed, s16, m16 = H.gather_codes(pages, lay.table, 0, 0, 1, n, kind)
        assert np.array_equal(s16.view(np.uint16), s_ref.view(np.uint16))
        assert np.array_equal(m16.view(np.uint16), m_ref.view(np.uint16))
        bad = np.argwhere(O.unpack(packed) != c_ref)
        assert len(bad) == 0, (kind, bad[:5])
    assert gc.device_status() == 0


def test_dequantize_bit_exact_and_original_basis():
    okv = _okv()
    lens = [300, 17, 0, 144]
    hkv = 2
    gc, oc, lay, zs = _fill_pre_rotated(2, 4, hkv, lens)
    max_ctx = 320
    args = (_t(np.arange(len(lens), dtype=np.int32)), _t(lay.table), _t(np.array(lens, np.int32)))
    for which in (0, 1):
        rot = okv.dequantize(gc, *args, max_ctx, which, basis=0, source=0).cpu().numpy()
        win = okv.dequantize(gc, *args, max_ctx, which, basis=0, source=1).cpu().numpy()
        orig = okv.dequantize(gc, *args, max_ctx, which, basis=1, source=0).cpu().numpy()
        for b, n in enumerate(lens):
            for h in range(hkv):
                assert np.all(rot[b, h, n:] == 0) and np.all(win[b, h, n:] == 0) and np.all(orig[b, h, n:] == 0)
                if n == 0:
                    continue
                st = oc.seqs[(b, which, h)]
                want = O.dequantize(st["codes"][:n], st["s16"][:n], st["m16"][:n])
                assert np.array_equal(rot[b, h, :n], want)
                want_w = oc.values(b, which, h, n).astype(np.float32)
                assert np.array_equal(win[b, h, :n], want_w)
                back = want.astype(np.float64) @ oc.r[which][h].T
                assert np.abs(orig[b, h, :n] - back).max() <= 1e-5 * np.abs(back).max()


@pytest.mark.parametrize("lens,misalign", [
    ([700, 45], False),   # 745 tokens: tcgen05 kernel, 6 tiles, ragged last tile
    ([60, 45], False),    # 105 tokens: CUDA-core kernel
    ([1], False),         # one token: CUDA-core kernel, a single-token tile
    ([37], False),        # CUDA-core kernel, ragged tile
    ([127], False),       # the longest run the CUDA-core kernel takes
    ([128], False),       # exactly the tensor-core threshold: one tile
    ([700, 45], True),    # K/V not 16-byte aligned: the mma.sync tensor-core kernel
])
def test_append_fused_rotation_and_codes(lens, misalign):
    okv = _okv()
    seed, hq, hkv = 3, 8, 2
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    gc = _gpu_cache(hq, hkv, lay, uk, uv)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    k = [np.stack([WL.sample_keys(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1) for b, n in enumerate(lens)]
    v = [np.stack([WL.sample_values(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1) for b, n in enumerate(lens)]
    slots, pos = lay.flat()
    kk, vv = np.concatenate(k), np.concatenate(v)
    rot = torch.zeros((len(slots), 2, hkv, 128), dtype=torch.float32, device="cuda")
    kd, vd = _t(kk, torch.bfloat16), _t(vv, torch.bfloat16)
    if misalign:  # same values at an address 4 bytes past a 16-byte boundary
        kd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), kd.flatten()])[2:].view(kd.shape)
        vd = torch.cat([torch.zeros(2, dtype=torch.bfloat16, device="cuda"), vd.flatten()])[2:].view(vd.shape)
        assert kd.data_ptr() % 16 == 4 and vd.data_ptr() % 16 == 4
    okv.append_quantize(gc, kd, vd, _t(slots), _t(pos), _t(lay.table), _t(np.array(lens, np.int32)), rotated_out=rot)
    rot = rot.cpu().numpy()
    pages = gc.pages.cpu().numpy()
    off = 0
    n_amb = n_mismatch = 0
    for b, n in enumerate(lens):
        for h in range(hkv):
            for kind, x in ((0, k[b]), (1, v[b])):
                z64 = x[:, h, :].astype(np.float64) @ oc.r[kind][h]
                zg = rot[off:off + n, kind, h, :]
                err = np.abs(zg - z64).max(axis=1) / np.abs(z64).max(axis=1)
                assert err.max() < 1e-5, err.max()
                packed, s16, m16 = H.gather_codes(pages, lay.table, b, h, hkv, n, kind)
                c_gpu = O.unpack(packed)
                # the gate: the oracle's quantiser on the kernel's own fp32 rotation, bit for bit
                c_self, s_self, m_self = O.quantize(zg)
                assert np.array_equal(c_gpu, c_self), (b, h, kind, np.argwhere(c_gpu != c_self)[:5])
                assert np.array_equal(s16.view(np.uint16), s_self.view(np.uint16)), (b, h, kind)
                assert np.array_equal(m16.view(np.uint16), m_self.view(np.uint16)), (b, h, kind)
                # against the fp64 rotation: equal except at ambiguous decisions (a reported rate)
                amb = H.ambiguity_bound(z64, 2e-5)
                c_ref, s_ref, m_ref = O.quantize(z64.astype(np.float32))
                bad = c_gpu != c_ref
                assert not np.any(bad & ~amb), np.argwhere(bad & ~amb)[:5]
                assert np.all(np.abs(c_gpu.astype(int) - c_ref.astype(int)) <= 1)
                srow = (s16.view(np.uint16) != s_ref.view(np.uint16)) | (m16.view(np.uint16) != m_ref.view(np.uint16))
                assert not np.any(srow & ~amb.all(axis=1))
                n_amb += int(amb.sum())
                n_mismatch += int(bad.sum())
        off += n
    print(f"ambiguous codes {n_amb}, differing codes {n_mismatch}")


def _decode_case(seed, hq, hkv, lens, scale=1.0):
    okv = _okv()
    gc, oc, lay, _ = _fill_pre_rotated(seed, hq, hkv, lens, scale=scale)
    q = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=7) for h in range(hkv)], 1)
    q = q.reshape(len(lens), hq, 128)
    seq = np.arange(len(lens), dtype=np.int32)
    out = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), _t(lay.table), _t(np.array(lens, np.int32)))
    got = out.cpu().numpy()
    want = O.decode(oc, q, seq, lens, hq)
    assert gc.device_status() == 0
    return got, want


@pytest.mark.parametrize("hq,hkv,lens", [
    (4, 1, [2048]),
    (32, 8, [1000, 3001, 129, 17]),
    (8, 8, [900, 128]),
    (16, 8, [1, 2, 130, 777]),
    (64, 8, [1500]),
    (16, 1, [640]),
])
def test_decode_parity(hq, hkv, lens):
    got, want = _decode_case(11, hq, hkv, lens)
    err = H.rel_err_rows(got, want)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0)
    assert err.max() <= TOL, (err.max(), np.unravel_index(err.argmax(), err.shape))


def test_decode_edge_lengths_and_empty():
    lens = [0, 1, 127, 128, 129, 143, 144, 145, 160, 161]
    got, want = _decode_case(12, 8, 2, lens)
    assert np.all(got[0] == 0)
    assert H.rel_err_rows(got, want).max() <= TOL


def test_decode_large_values():
    # rotated magnitudes in the hundreds: logits far from 0, peaked softmax
    got, want = _decode_case(13, 8, 2, [1200, 333], scale=30.0)
    assert H.rel_err_rows(got, want).max() <= TOL


def test_decode_deterministic_and_workspace_reuse():
    okv = _okv()
    lens = [1000, 2000]
    gc, oc, lay, _ = _fill_pre_rotated(14, 8, 2, lens)
    q = _t(WL.to_bf16_exact(np.random.default_rng(0).standard_normal((2, 8, 128)).astype(np.float32)),
           torch.bfloat16)
    ws = okv.workspace(gc, 2)
    a = okv.decode_attention(gc, q, _t(np.arange(2, dtype=np.int32)), _t(lay.table), _t(np.array(lens, np.int32)),
                             ws=ws).clone()
    b = okv.decode_attention(gc, q, _t(np.arange(2, dtype=np.int32)), _t(lay.table), _t(np.array(lens, np.int32)),
                             ws=ws)
    assert torch.equal(a, b)


def test_end_to_end_calibrated_fused_path():
    """Tiny workload end to end: oracle calibration, bf16 K/V through the
    fused rotate+quantise kernel, decode.  The kernel's rotation is checked
    against the oracle's fp64 rotation (1e-5), its codes bit for bit against
    the oracle's quantiser on that same fp32 rotation, and the decode against
    the oracle's decode of the cache those codes form, at a plain 2e-3."""
    okv = _okv()
    seed, hq, hkv, n = 0, 4, 1, 2048
    qc, kc, vc = WL.calibration_set(seed, 0, 0, hq, hkv, n=2048)
    cal = O.calibrate(qc, kc, vc, hq, hkv)
    uk, uv = cal["U_K"].astype(np.float32), cal["U_V"].astype(np.float32)
    lay = H.Layout(seed, [n])
    gc = _gpu_cache(hq, hkv, lay, uk, uv)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    k = WL.sample_keys(seed, 0, 0, 0, n)[:, None, :]
    v = WL.sample_values(seed, 0, 0, 0, n)[:, None, :]
    slots, pos = lay.flat()
    rot = torch.zeros((n, 2, hkv, 128), dtype=torch.float32, device="cuda")
    okv.append_quantize(gc, _t(k, torch.bfloat16), _t(v, torch.bfloat16), _t(slots), _t(pos), _t(lay.table),
                        _t(np.array([n], np.int32)), rotated_out=rot)
    rot = rot.cpu().numpy()
    zk, zv = rot[:, 0], rot[:, 1]
    for kind, x, zg in ((0, k, zk), (1, v, zv)):
        z64 = x[:, 0].astype(np.float64) @ oc.r[kind][0]
        assert (np.abs(zg[:, 0] - z64).max(axis=1) / np.abs(z64).max(axis=1)).max() < 1e-5
    oc.append(0, 0, zk, zv, pre_rotated=True)
    pages = gc.pages.cpu().numpy()
    for kind in (0, 1):
        packed, s16, m16 = H.gather_codes(pages, lay.table, 0, 0, hkv, n, kind)
        st = oc.seqs[(0, kind, 0)]
        assert np.array_equal(O.unpack(packed), st["codes"][:n])
        assert np.array_equal(s16.view(np.uint16), st["s16"][:n].view(np.uint16))
        assert np.array_equal(m16.view(np.uint16), st["m16"][:n].view(np.uint16))
    q = WL.sample_queries(seed, 0, 0, 0, 1, hq).reshape(1, hq, 128)
    got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(np.zeros(1, np.int32)), _t(lay.table),
                               _t(np.array([n], np.int32))).cpu().numpy()
    want = O.decode(oc, q, [0], [n], hq)
    err = H.rel_err_rows(got, want)
    assert err.max() <= TOL, err
    # for the record: the distance to the oracle's own fp64-rotated cache
    o64 = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    o64.append(0, 0, k, v)
    print(f"decode vs the fp64-rotated oracle cache: {H.rel_err_rows(got, O.decode(o64, q, [0], [n], hq)).max():.2e}")


def test_decode_partial_last_block_with_live_tail():
    """The last INT2 block is only partly inside the context while its other
    slots hold real tokens (the cache was filled further than the decode
    length), and entries so short that a split streams a single block."""
    okv = _okv()
    fill = [3000, 129, 1, 777]
    dec = [2900, 129, 1, 770]
    gc, oc, lay, zs = _fill_pre_rotated(21, 32, 8, fill)
    q = np.stack([WL.sample_queries(21, 0, 0, h, len(fill), 4, extra=3) for h in range(8)], 1).reshape(len(fill), 32, 128)
    seq = np.arange(len(fill), dtype=np.int32)
    for _ in range(3):
        got = okv.decode_attention(gc, _t(q, torch.bfloat16), _t(seq), _t(lay.table),
                                   _t(np.array(dec, np.int32))).cpu().numpy()
        assert np.isfinite(got).all()
    # the oracle sees the same cache as the kernels: positions < decode length,
    # the window ring rows holding whatever was appended last
    for b in range(len(fill)):
        assert oc.seqs[(b, 0, 0)]["set"][:dec[b]].all()


@pytest.mark.parametrize("group", [128, 32])
def test_staged_rotation_image_matches_in_kernel_staging(group):
    """The tcgen05 append copying R from the cache's staged image writes the
    same bytes (codes, scales, window rows) and the same rotated fp32 values
    as the append staging R from U itself; after U changes, rebuilding the
    image matches a fresh cache."""
    okv = _okv()
    seed, hq, hkv, n = 57, 32, 8, 1000
    lay = H.Layout(seed, [n])
    uk, uv = H.rotations(seed, hkv)
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randn((n, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((n, hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    slots, pos = lay.flat()
    args = (_t(slots), _t(pos), _t(lay.table), _t(np.array([n], np.int32)))

    def run(c):
        rot = torch.empty((n, 2, hkv, 128), dtype=torch.float32, device="cuda")
        okv.append_quantize(c, k, v, *args, rotated_out=rot)
        torch.cuda.synchronize()
        assert c.device_status() == 0
        return c.pages.clone(), c.ring.clone(), rot

    mk = lambda u1, u2, stage: okv.Cache(hq, hkv, lay.num_blocks, 1, lay.mbps, u1, u2, group=group, stage_r=stage)
    with_image, without = run(mk(uk, uv, True)), run(mk(uk, uv, False))
    for a, b in zip(with_image, without):
        assert torch.equal(a, b)
    # the rotation itself against the fp64 oracle
    want = np.einsum("thc,hcd->thd", k.float().cpu().numpy().astype(np.float64),
                     np.stack([O.rotation(uk[h].astype(np.float64)) for h in range(hkv)]))
    got = with_image[2][:, 0].cpu().numpy()
    assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max()
    # new rotations: rebuild the image of an existing cache
    uk2, uv2 = H.rotations(seed + 1, hkv)
    c = mk(uk, uv, True)
    c.u_k.copy_(torch.from_numpy(uk2))
    c.u_v.copy_(torch.from_numpy(uv2))
    c.rebuild_r_image()
    for a, b in zip(run(c), run(mk(uk2, uv2, True))):
        assert torch.equal(a, b)
