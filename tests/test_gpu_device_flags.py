"""Conditions only the device can see (a block id outside the pool, a bad
sequence slot, a position past the block table or past the slot's length, a
decode length beyond the table) are skipped by the kernels and reported in the
cache's status word; everything else in the same call is still computed
exactly.  Every case here is caught by a kernel's own bounds check: nothing
reads or writes outside its buffers."""
import numpy as np
import pytest

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _okv():
    from int2_kv_cache_rotate_b200 import okv
    return okv


def _d(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("n_tok", [40, 300])  # CUDA-core kernel / tcgen05 kernel
def test_append_flags_bad_block_slot_and_position(n_tok):
    okv = _okv()
    seed, hq, hkv = 41, 8, 2
    lens = [n_tok, n_tok]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    cache = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv)
    table = lay.table.copy()
    table[1, 1] = lay.num_blocks + 5          # positions 16..31 of sequence 1: block outside the pool
    slots, pos = lay.flat()
    slots, pos = slots.copy(), pos.copy()
    slots[3] = 7                                # sequence slot outside the cache
    pos[5] = n_tok + 3                          # position past the slot's length
    k = np.concatenate([np.stack([WL.sample_keys(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    v = np.concatenate([np.stack([WL.sample_values(seed, 0, 0, h, n, extra=b) for h in range(hkv)], 1)
                        for b, n in enumerate(lens)])
    rot = torch.zeros((len(slots), 2, hkv, 128), dtype=torch.float32, device="cuda")
    okv.append_quantize(cache, _d(k).to(torch.bfloat16), _d(v).to(torch.bfloat16), _d(slots), _d(pos), _d(table),
                        _d(np.array(lens, np.int32)), rotated_out=rot)
    torch.cuda.synchronize()
    st = cache.device_status()
    assert st & okv.DEV_BAD_BLOCK and st & okv.DEV_BAD_SLOT and st & okv.DEV_BAD_POS, st
    # every token with a valid destination was written, bit-exactly from its own rotation:
    # sequence 0 position p holds token p (p not 3 or 5), sequence 1 position p token n + p
    # (p outside the missing block 16..31)
    rot = rot.cpu().numpy()
    pages = cache.pages.cpu().numpy()
    checks = [(0, np.array([p for p in range(n_tok) if p not in (3, 5)]), 0),
              (1, np.array([p for p in range(n_tok) if not 16 <= p < 32]), n_tok)]
    for b, p_sel, tok0 in checks:
        t_sel = p_sel + tok0
        for h in range(hkv):
            for kind in (0, 1):
                packed, s16, m16 = H.gather_codes(pages, lay.table, b, h, hkv, n_tok, kind)
                c_ref, s_ref, m_ref = O.quantize(rot[t_sel, kind, h, :])
                assert np.array_equal(O.unpack(packed[p_sel]), c_ref), (b, h, kind)
                assert np.array_equal(s16[p_sel].view(np.uint16), s_ref.view(np.uint16))
                assert np.array_equal(m16[p_sel].view(np.uint16), m_ref.view(np.uint16))


def test_decode_flags_bad_block_and_length_keep_other_entries_exact():
    okv = _okv()
    seed, hq, hkv = 42, 32, 8
    lens = [2000, 1500, 900]
    lay = H.Layout(seed, lens)
    uk, uv = H.rotations(seed, hkv)
    cache = okv.Cache(hq, hkv, lay.num_blocks, len(lens), lay.mbps, uk, uv)
    oc = O.Cache(hkv, uk.astype(np.float64), uv.astype(np.float64))
    slots, pos = lay.flat()
    z = {kind: np.concatenate([np.stack([WL.sample_rotated(seed, 0, 0, h, n, kind, extra=b) for h in range(hkv)], 1)
                               for b, n in enumerate(lens)]) for kind in (0, 1)}
    okv.append_quantize(cache, _d(z[0]), _d(z[1]), _d(slots), _d(pos), _d(lay.table), _d(np.array(lens, np.int32)),
                        pre_rotated=True)
    off = 0
    for b, n in enumerate(lens):
        oc.append(b, 0, z[0][off:off + n], z[1][off:off + n], pre_rotated=True)
        off += n
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    table = lay.table.copy()
    table[1, 3] = -7                                   # an INT2 block of entry 1 outside the pool
    dec_lens = np.array(lens, np.int32)
    dec_lens[2] = lay.mbps * 16 + 100                  # entry 2: a length beyond its block table
    q = np.stack([WL.sample_queries(seed, 0, 0, h, len(lens), hq // hkv, extra=1) for h in range(hkv)], 1)
    q = q.reshape(len(lens), hq, 128)
    got = okv.decode_attention(cache, _d(q).to(torch.bfloat16), _d(np.arange(len(lens), dtype=np.int32)), _d(table),
                               _d(dec_lens)).cpu().numpy()
    st = cache.device_status()
    assert st & okv.DEV_BAD_BLOCK and st & okv.DEV_BAD_POS, st
    want = O.decode(oc, q[:1], [0], [lens[0]], hq)
    assert H.rel_err_rows(got[:1], want).max() <= 2e-3
    assert np.all(np.isfinite(got))
