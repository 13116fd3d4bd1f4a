"""Test-side helpers: build caches on both sides from the same seeded inputs,
and read the library's physical block layout back into canonical arrays.

The layout reader encodes only where bytes live (documented in
include/okv.h); it does no arithmetic of the method."""
from __future__ import annotations

import numpy as np

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O

D = 128


def rel_err_rows(got, want):
    """Per (b, h) row: max_i |got - want| / max_i |want| (rows with want == 0 use 1)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.abs(want).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return np.abs(got - want).max(axis=-1) / den


def read_block_head(pages: np.ndarray, blk: int, h: int, hkv: int):
    base = (blk * hkv + h) * 1152
    return pages[base:base + 1152]


def gather_codes(pages: np.ndarray, table: np.ndarray, slot: int, h: int, hkv: int, n: int, kind: int):
    """Canonical packed code bytes [n, 32], fp16 scale and min [n] for positions 0..n-1."""
    pos = np.arange(n)
    blk = table[slot, pos // 16].astype(np.int64)
    t = pos % 16
    base = (blk * hkv + h) * 1152
    b = np.arange(32)
    if kind == 0:
        off = base[:, None] + t[:, None] * 32 + b[None, :]
        sm_off = base + 1024 + 4 * t
    else:
        off = base[:, None] + 512 + ((b[None, :] >> 2) * 4 + (t[:, None] >> 2)) * 16 + (b[None, :] & 3) * 4 \
            + (t[:, None] & 3)
        sm_off = base + 1088 + 4 * t
    packed = pages[off]
    s_bits = pages[sm_off].astype(np.uint16) | (pages[sm_off + 1].astype(np.uint16) << 8)
    m_bits = pages[sm_off + 2].astype(np.uint16) | (pages[sm_off + 3].astype(np.uint16) << 8)
    return packed, s_bits.view(np.float16), m_bits.view(np.float16)


def gather_codes_grouped(pages: np.ndarray, table: np.ndarray, slot: int, h: int, hkv: int, n: int, kind: int,
                         group: int):
    """Like gather_codes for a cache with `group`-channel quantisation groups:
    packed code bytes [n, 32], fp16 scale and min [n, 128 / group]."""
    ng = D // group
    bhb = 1024 + 128 * ng
    pos = np.arange(n)
    blk = table[slot, pos // 16].astype(np.int64)
    t = pos % 16
    base = (blk * hkv + h) * bhb
    b = np.arange(32)
    if kind == 0:
        off = base[:, None] + t[:, None] * 32 + b[None, :]
    else:
        off = base[:, None] + 512 + ((b[None, :] >> 2) * 4 + (t[:, None] >> 2)) * 16 + (b[None, :] & 3) * 4 \
            + (t[:, None] & 3)
    packed = pages[off]
    k = np.arange(ng)
    sm_off = base[:, None] + 1024 + 64 * ng * kind + 4 * (t[:, None] * ng + k[None, :])
    s_bits = pages[sm_off].astype(np.uint16) | (pages[sm_off + 1].astype(np.uint16) << 8)
    m_bits = pages[sm_off + 2].astype(np.uint16) | (pages[sm_off + 3].astype(np.uint16) << 8)
    return packed, s_bits.view(np.float16), m_bits.view(np.float16)


def special_vectors() -> np.ndarray:
    """Edge-case groups for the quantiser: constant, huge range, lattice,
    ties, subnormal scale, scale that rounds to zero, min that rounds up."""
    j = np.arange(D)
    rows = []
    rows.append(np.full(D, 0.1, np.float32))
    z = np.zeros(D, np.float32); z[0], z[1] = -1e6, 1e6; rows.append(z)
    rows.append((-1.5 + 0.75 * (j % 4)).astype(np.float32))
    z = np.zeros(D, np.float32); z[:5] = [0.0, 3.0, 0.5, 1.5, 2.5]; rows.append(z)
    z = np.zeros(D, np.float32); z[1] = 1e-7; rows.append(z)
    z = np.zeros(D, np.float32); z[1] = 2e-8; rows.append(z)
    z = np.zeros(D, np.float32); z[0], z[1] = -0.3333333432674408, 1.0; rows.append(z)
    rows.append((j % 4).astype(np.float32))
    z = np.zeros(D, np.float32); z[7] = 70000.0; rows.append(z)  # window value saturates
    return np.stack(rows)


def rounding_boundary_vectors(seed: int, n: int) -> np.ndarray:
    """[n, 128] fp32 groups whose values sit within 8 fp32 ulps of each
    rounding midpoint m + (k + 1/2) s of their own quantiser, so that the
    code decision turns on the last bit of fl(fl(z - m) / s) and on ties to
    even.  s spans fp16 normals and subnormals, m sits up to 2^7 s away from
    zero on either side (so fl(z - m) rounds too).  The oracle's quantiser
    only locates s and m; the rows are then quantised afresh by both sides."""
    r = np.random.default_rng(np.random.SeedSequence([seed, 4242]))
    rows = np.empty((n, D), np.float32)
    for i in range(n):
        s_t = np.float64(np.float16(r.uniform(1.0, 2.0) * 2.0 ** int(r.integers(-24, 11))))
        if s_t == 0:
            s_t = 2.0 ** -24
        m_t = np.float32(np.float16(np.clip(r.uniform(-1.0, 1.0) * s_t * 2.0 ** int(r.integers(0, 8)),
                                            -60000.0, 60000.0)))
        row = np.full(D, m_t, np.float32)
        row[1] = np.float32(np.float64(m_t) + 3.0 * s_t)
        _, s16, m16 = O.quantize(row[None])
        s, m = np.float64(s16[0]), np.float64(m16[0])
        vals = []
        for k in range(3):
            c = np.float32(m + (k + 0.5) * s)
            up = dn = c
            vals.append(c)
            for _ in range(8):
                up = np.nextafter(up, np.float32(np.inf))
                dn = np.nextafter(dn, np.float32(-np.inf))
                vals += [up, dn]
        vals = np.array(vals, np.float32)
        row[2:2 + len(vals)] = np.clip(vals, row[0], row[1])
        rows[i] = row[r.permutation(D)]
    return rows


def rotations(seed: int, hkv: int):
    """Seeded orthogonal U_K, U_V per KV head (fp32-exact values, as float64)."""
    r = np.random.default_rng(np.random.SeedSequence([seed, 999]))
    uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    uv = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    return uk, uv


class Layout:
    """Token placement for a batch of sequences: slots, positions, block table."""

    def __init__(self, seed: int, lens, extra_blocks: int = 3):
        self.lens = [int(x) for x in lens]
        self.table, self.num_blocks = WL.block_table(seed, 0, self.lens, extra_tokens=16,
                                                     spare_blocks=extra_blocks)
        self.mbps = self.table.shape[1]

    def flat(self):
        slots = np.concatenate([np.full(n, i, np.int32) for i, n in enumerate(self.lens)]) \
            if sum(self.lens) else np.zeros(0, np.int32)
        pos = np.concatenate([np.arange(n, dtype=np.int32) for n in self.lens]) \
            if sum(self.lens) else np.zeros(0, np.int32)
        return slots, pos


def ambiguity_bound(z64: np.ndarray, eps_rel: float) -> np.ndarray:
    """For oracle-rotated vectors z64 [n, 128] (fp64), flag codes whose
    decision could flip under a relative perturbation eps_rel of z: the
    quotient (z - m)/s lies within that distance of a rounding midpoint, or
    the fp16 scale/min themselves sit next to a rounding midpoint.
    Returns a boolean array [n, 128] (a whole row is flagged in the latter case)."""
    z32 = z64.astype(np.float32)
    c, s16, m16 = O.quantize(z32)
    s = s16.astype(np.float64)[:, None]
    m = m16.astype(np.float64)[:, None]
    scale = np.abs(z64).max(axis=1, keepdims=True)
    tol = eps_rel * scale
    with np.errstate(divide="ignore", invalid="ignore"):
        qv = np.where(s > 0, (z64 - m) / s, 0.0)
        dq = np.where(s > 0, 2 * tol / s, 0.0)
    frac = qv - np.floor(qv)
    amb = (np.abs(frac - 0.5) <= dq + 1e-12) & (s > 0)
    # fp16 rounding of the scale and the min
    mn = z64.min(axis=1)
    mx = z64.max(axis=1)
    s32 = (mx - mn) / 3.0

    def near_mid(x, t):
        x16 = np.float16(np.clip(x, -65504, 65504))
        nxt = np.nextafter(x16, np.float16(np.inf))
        prv = np.nextafter(x16, np.float16(-np.inf))
        mids = np.stack([(x16.astype(np.float64) + nxt.astype(np.float64)) / 2,
                         (x16.astype(np.float64) + prv.astype(np.float64)) / 2])
        return (np.abs(mids - x[None]) <= t[None]).any(axis=0)

    row = near_mid(s32, 2 * tol[:, 0] / 3 + 1e-30) | near_mid(mn, tol[:, 0] + 1e-30)
    amb |= row[:, None]
    return amb
