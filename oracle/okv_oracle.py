"""CPU oracle for OSCAR-style INT2 KV-cache rotation, quantisation and decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library path may import or call this
module: it is used by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / reference arm of ``bench.py``.  It is plain, slow NumPy,
written from the pages' description of the method, and shares no code with
the CUDA library (the two meet only in the seeded input generators).

Pages cited (title, and the section named in each docstring):

* [GH] gen-hub.ru, "Together AI открывает OSCAR: сжатие KV-кэша до 2 бит без
  потери точности"
* [EN] encorp.ai, "KV cache compression е инфраструктурно решение, не спор за
  модела"
* [BS] bigsaas.top, "Revolução no Serviço de LLMs: Together AI Lança OSCAR
  para Contextos Extensos"
* [AF] aiforradalom.hu, "Az Apple, a Google és a NYU új technikái felezik az
  LLM-ek memóriaigényét"
* [AR] ru.arsentev.ai, "Гонка за сжатие памяти ИИ на длинном контексте"

Precision: fp64 everywhere, except the quantiser, whose fp32 steps *are* its
definition (so that integer codes can be compared bit for bit), and the fp16
scale/min and fp16 recent-window storage, which are part of the cache format.

Readings taken where the pages are silent:

* "covariance" of the queries is the uncentred second moment E[q q^T]
  (equal to the covariance for zero-mean queries), pooled over the G query
  heads that share a KV head;
* the score-weighted value covariance weights v_j v_j^T by the softmax mass
  p_ij that key j receives from every calibration query i, normalised by the
  total mass, with no causal mask;
* eigenvectors are sorted by descending eigenvalue, and each column's sign is
  fixed so that its largest-magnitude entry is positive;
* H is the Sylvester (natural-order) Hadamard matrix scaled by 1/sqrt(d); the
  bit-reversal permutation moves entry br(j) to position j;
* row-vector convention: x_rot = x R with R = U H P_br (U first, then H, then
  P_br, the order the pages give);
* quantiser: asymmetric min/max over one group of 128 channels, four levels,
  fp16 scale = (max - min)/3 and fp16 min, codes rounded half-to-even and
  clamped to [0, 3], dequantised as s*c + m;
* every token is quantised at append; the last W = 128 positions are also
  kept as fp16 rotated values and decode reads those positions from fp16;
* groups smaller than 128 channels (32, 64) follow the same rule per group,
  one fp16 scale and min each (the built format has one group per vector);
* sink tokens: the first S positions of a sequence are kept the same way and
  read from fp16.  The pages name sinks without a count; S is a cache
  parameter, 0 (no sinks) by default.  S = 192 with W = 128 keeps 320 of
  128K tokens 16-bit, the 0.24 % the pages quote.
"""
from __future__ import annotations

import math

import numpy as np

D = 128
W = 128
FP16_MAX = 65504.0


# ----------------------------------------------------------------------------
# Fixed transforms
# ----------------------------------------------------------------------------

def hadamard(d: int = D) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix, H_ij = (-1)^popcount(i & j) / sqrt(d).

    [GH] section "Что придумали в Together AI" (second step of the composite
    transform: a Hadamard that equalises channel importance); [AF] section
    "OSCAR: figyelem-tudatos és bevetésre kész"."""
    if d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d)
    parity = np.zeros((d, d), dtype=np.int64)
    x = i[:, None] & i[None, :]
    while np.any(x):
        parity ^= x & 1
        x = x >> 1
    return np.where(parity == 0, 1.0, -1.0) / math.sqrt(d)


def bit_reverse(j: int, bits: int) -> int:
    """Reverse the low ``bits`` bits of j."""
    r = 0
    for _ in range(bits):
        r = (r << 1) | (j & 1)
        j >>= 1
    return r


def bitrev_indices(d: int = D) -> np.ndarray:
    """br(j) for j in [0, d): the source index of output position j.

    [GH] section "Что придумали в Together AI" (third step: the bit-reversal
    permutation P_br that gives every quantisation group an even share of the
    importance hierarchy); [AF] section "OSCAR: figyelem-tudatos…"."""
    bits = d.bit_length() - 1
    return np.array([bit_reverse(j, bits) for j in range(d)], dtype=np.int64)


def bitrev_matrix(d: int = D) -> np.ndarray:
    """P with (y P)_j = y_{br(j)}: P[i, j] = 1 iff i = br(j)."""
    p = np.zeros((d, d))
    p[bitrev_indices(d), np.arange(d)] = 1.0
    return p


def rotation(u: np.ndarray) -> np.ndarray:
    """R = U H P_br, dense, in the row-vector convention x_rot = x R.

    [GH] section "Что придумали в Together AI": align to the importance
    directions (U), then Hadamard, then bit reversal, in that order."""
    d = u.shape[0]
    return u @ hadamard(d) @ bitrev_matrix(d)


# ----------------------------------------------------------------------------
# Offline calibration
# ----------------------------------------------------------------------------

def query_covariance(q: np.ndarray) -> np.ndarray:
    """C_Q = mean over all calibration queries of q q^T (uncentred), fp64.

    q: [N, G, d] -- the G query heads that share one KV head are pooled.
    [GH] section "Что придумали в Together AI": key error matters through the
    logits QK^T, so the error weight is the query covariance, estimated on a
    calibration set; [AF] "OSCAR: figyelem-tudatos…"; [BS] "OSCAR: Indo Além
    das Transformações de Hadamard"."""
    x = np.asarray(q, dtype=np.float64).reshape(-1, q.shape[-1])
    return (x.T @ x) / x.shape[0]


def attention_probs(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """p_ij = softmax_j(q_i . k_j / sqrt(d)) over all calibration keys (no mask), fp64.

    q: [Nq, d], k: [Nk, d] -> [Nq, Nk]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = (q @ k.T) / math.sqrt(q.shape[-1])
    s -= s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def score_weighted_value_covariance(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                                    chunk: int = 2048) -> np.ndarray:
    """C_S = sum_ij p_ij v_j v_j^T / sum_ij p_ij, fp64.

    q: [N, G, d] queries of one KV group; k, v: [Nk, d] of that KV head.
    [GH] section "Что придумали в Together AI": value error matters through
    the attention output SV, so the value covariance is weighted by the
    attention scores; [AF] "OSCAR: figyelem-tudatos…"."""
    qf = np.asarray(q, dtype=np.float64).reshape(-1, q.shape[-1])
    mass = np.zeros(k.shape[0])
    total = 0.0
    for i in range(0, qf.shape[0], chunk):
        p = attention_probs(qf[i:i + chunk], k)
        mass += p.sum(axis=0)
        total += p.sum()
    vf = np.asarray(v, dtype=np.float64)
    return (vf.T * mass) @ vf / total


def eigenbasis(c: np.ndarray):
    """Eigenvectors of a symmetric matrix as columns, sorted by descending
    eigenvalue (ties: lower eigh index first), each column's sign fixed so its
    largest-magnitude entry (first on ties) is positive.  Returns (U, lam)."""
    lam, u = np.linalg.eigh(np.asarray(c, dtype=np.float64))
    order = sorted(range(len(lam)), key=lambda i: (-lam[i], i))
    lam = lam[order]
    u = u[:, order]
    for j in range(u.shape[1]):
        a = int(np.argmax(np.abs(u[:, j])))
        if u[a, j] < 0:
            u[:, j] = -u[:, j]
    return u, lam


def calibrate(q: np.ndarray, k: np.ndarray, v: np.ndarray, hq: int, hkv: int):
    """Offline calibration for one layer.

    q: [N, hq, d]; k, v: [Nk, hkv, d].  Returns dict with U_K, U_V, R_K, R_V
    ([hkv, d, d] fp64) and the eigenvalues.  Query head h belongs to KV head
    h // (hq // hkv).  [GH] sections "Что придумали в Together AI" and
    "Открытый код — это серьёзно" (calibration runs offline, once per model);
    [BS] "Como Funciona o OSCAR?"."""
    g = hq // hkv
    d = q.shape[-1]
    out = {n: np.zeros((hkv, d, d)) for n in ("U_K", "U_V", "R_K", "R_V")}
    out["lam_K"] = np.zeros((hkv, d))
    out["lam_V"] = np.zeros((hkv, d))
    for h in range(hkv):
        qg = q[:, h * g:(h + 1) * g, :]
        uk, lk = eigenbasis(query_covariance(qg))
        uv, lv = eigenbasis(score_weighted_value_covariance(qg, k[:, h, :], v[:, h, :]))
        out["U_K"][h], out["U_V"][h] = uk, uv
        out["lam_K"][h], out["lam_V"][h] = lk, lv
        out["R_K"][h], out["R_V"][h] = rotation(uk), rotation(uv)
    return out


# ----------------------------------------------------------------------------
# INT2 group quantiser (fp32 by definition) and its storage format
# ----------------------------------------------------------------------------

def fp16_saturate(x32: np.ndarray) -> np.ndarray:
    """fp32 -> fp16, round to nearest even, saturating at +-65504."""
    x = np.clip(np.asarray(x32, dtype=np.float32), np.float32(-FP16_MAX), np.float32(FP16_MAX))
    return x.astype(np.float16)


def quantize(z32: np.ndarray, group: int = D):
    """Quantise groups of fp32 values to 2-bit codes with fp16 scale and min.

    z32: float32 [..., 128].  With group = 128 (the built format: one group
    per row) returns (codes uint8 [..., 128], s16 float16 [...], m16 float16
    [...]); with a smaller group g (a divisor of 128: the groups for which the
    pages' bit-reversal permutation spreads importance, [GH] "Что придумали…")
    s16 and m16 are [..., 128 / g], one pair per g consecutive channels.
    Steps, per group, all in IEEE fp32 with round-to-nearest-even:
      mn = min z, mx = max z; s32 = (mx - mn) / 3;
      s16 = fp16(s32), m16 = fp16(mn) (saturating); s = f32(s16), m = f32(m16);
      c = 0 if s == 0 else clamp(rint((z - m) / s), 0, 3).
    INT2 with four levels and a per-group scale/min: [BS] section "Resultados e
    Métricas de Desempenho" (2.28 bits per KV element) and the comparison
    table; [GH] section "Почему INT2 раньше не работал" (four levels)."""
    z = np.asarray(z32, dtype=np.float32)
    if z.shape[-1] != D:
        raise ValueError("vectors must have 128 channels")
    if group <= 0 or D % group != 0:
        raise ValueError("group must divide 128")
    if group != D:
        c, s16, m16 = quantize_rows(z.reshape(*z.shape[:-1], D // group, group))
        return c.reshape(z.shape), s16, m16
    return quantize_rows(z)


def quantize_rows(z: np.ndarray):
    """The rule of `quantize` applied to each row (last axis) of fp32 z."""
    z = np.asarray(z, dtype=np.float32)
    mn = z.min(axis=-1)
    mx = z.max(axis=-1)
    s32 = (mx - mn) / np.float32(3.0)
    s16 = fp16_saturate(s32)
    m16 = fp16_saturate(mn)
    s = s16.astype(np.float32)[..., None]
    m = m16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (z - m) / np.where(s == 0, np.float32(1.0), s)
    c = np.clip(np.rint(t), 0, 3)
    c = np.where(s == 0, 0, c).astype(np.uint8)
    return c, s16, m16


def pack(codes: np.ndarray) -> np.ndarray:
    """Canonical packing: channel j goes to byte j // 4, bits 2*(j % 4) .. +1."""
    c = np.asarray(codes, dtype=np.uint8)
    c4 = c.reshape(*c.shape[:-1], c.shape[-1] // 4, 4)
    return (c4[..., 0] | (c4[..., 1] << 2) | (c4[..., 2] << 4) | (c4[..., 3] << 6)).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    b = np.asarray(packed, dtype=np.uint8)
    out = np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1)
    return out.reshape(*b.shape[:-1], b.shape[-1] * 4).astype(np.uint8)


def dequantize(codes: np.ndarray, s16: np.ndarray, m16: np.ndarray, group: int = D) -> np.ndarray:
    """x_hat = s * c + m, exact in fp64 then rounded once to fp32 (per group)."""
    c = np.asarray(codes, dtype=np.float64)
    if group != D:
        c = c.reshape(*c.shape[:-1], D // group, group)
    s = np.asarray(s16, dtype=np.float64)[..., None]
    m = np.asarray(m16, dtype=np.float64)[..., None]
    return (s * c + m).reshape(np.shape(codes)).astype(np.float32)


# ----------------------------------------------------------------------------
# Cache model and decode attention
# ----------------------------------------------------------------------------

class Cache:
    """Logical (unpaged) mixed-precision KV cache for one layer.

    Every appended token is quantised to INT2; its fp16 rotated values are
    also stored, and decode reads the most recent W positions and the first
    `sinks` positions from those.
    [EN] section "OSCAR има значение…" and [AF] "OSCAR: figyelem-tudatos…"
    (recent tokens stay 16-bit, history goes to INT2, paged-cache compatible).
    """

    def __init__(self, hkv: int, u_k: np.ndarray, u_v: np.ndarray, window: int = W, sinks: int = 0,
                 group: int = D):
        self.hkv = hkv
        self.window = window
        self.sinks = sinks
        self.group = group  # channels per quantisation group (128: one per token-head)
        self.r = {0: np.stack([rotation(u) for u in u_k]), 1: np.stack([rotation(u) for u in u_v])}
        self.seqs = {}

    def _store(self, slot: int, kind: int, h: int, need: int):
        key = (slot, kind, h)
        st = self.seqs.get(key)
        if st is None or st["codes"].shape[0] < need:
            cap = max(need, 2 * (0 if st is None else st["codes"].shape[0]), 64)
            sm_shape = (cap,) if self.group == D else (cap, D // self.group)
            new = {"codes": np.zeros((cap, D), np.uint8), "s16": np.zeros(sm_shape, np.float16),
                   "m16": np.zeros(sm_shape, np.float16), "z16": np.zeros((cap, D), np.float16),
                   "set": np.zeros(cap, bool)}
            if st is not None:
                n = st["codes"].shape[0]
                for name in new:
                    new[name][:n] = st[name]
            self.seqs[key] = st = new
        return st

    def rotate(self, x: np.ndarray, kind: int, h: int) -> np.ndarray:
        """fp64 rotation x R (kind 0 = keys, 1 = values), rounded to fp32."""
        return (np.asarray(x, dtype=np.float64) @ self.r[kind][h]).astype(np.float32)

    def append(self, slot: int, pos0: int, k: np.ndarray, v: np.ndarray, pre_rotated: bool = False):
        """Append tokens k, v [n, hkv, d] at positions pos0 .. pos0 + n - 1.

        Inputs are bf16-exact float32 (rotated here in fp64, then rounded to
        fp32 for the quantiser), or fp32 values that are already rotated."""
        k = np.asarray(k).reshape(-1, self.hkv, D)
        v = np.asarray(v).reshape(-1, self.hkv, D)
        n = k.shape[0]
        for kind, x in ((0, k), (1, v)):
            for h in range(self.hkv):
                xs = np.asarray(x[:, h, :], dtype=np.float32)
                z = xs if pre_rotated else (xs.astype(np.float64) @ self.r[kind][h]).astype(np.float32)
                c, s16, m16 = quantize(z, self.group)
                st = self._store(slot, kind, h, pos0 + n)
                sl = slice(pos0, pos0 + n)
                st["codes"][sl], st["s16"][sl], st["m16"][sl] = c, s16, m16
                st["z16"][sl] = fp16_saturate(z)
                st["set"][sl] = True

    def entry(self, slot: int, kind: int, h: int, pos: int):
        st = self.seqs[(slot, kind, h)]
        return st["codes"][pos], st["s16"][pos], st["m16"][pos], st["z16"][pos]

    def values(self, slot: int, kind: int, h: int, length: int) -> np.ndarray:
        """Rotated vectors as decode sees them: the first min(length, sinks) and
        the last min(length, W) positions from fp16, the rest dequantised from
        INT2.  fp64 [length, d]."""
        st = self.seqs[(slot, kind, h)]
        if not st["set"][:length].all():
            raise ValueError("decode over positions that were never appended")
        out = st["z16"][:length].astype(np.float64)
        int2 = np.arange(length)
        int2 = int2[(int2 >= self.sinks) & (int2 < length - self.window)]
        out[int2] = dequantize(st["codes"][int2], st["s16"][int2], st["m16"][int2], self.group)
        return out


def attend(q_rot: np.ndarray, keys: np.ndarray, vals: np.ndarray) -> np.ndarray:
    """Exact softmax attention in fp64: softmax(q K^T / sqrt(d)) V for one query."""
    s = keys @ q_rot / math.sqrt(q_rot.shape[-1])
    s = s - s.max()
    p = np.exp(s)
    return (p @ vals) / p.sum()


def decode(cache: Cache, q: np.ndarray, seq_slots, context_lens, hq: int) -> np.ndarray:
    """Decode attention for one step.

    q: [B, hq, d] (bf16-exact).  Query head h reads KV head h // (hq // hkv).
    The query is rotated with R_K (so q R_K . k R_K = q . k before
    quantisation), attention runs over the cached rotated keys/values, and the
    output is brought back with R_V^T.  Empty contexts give zeros.
    Returns fp64 [B, hq, d].  [GH] section "Что придумали в Together AI";
    [AF] "OSCAR: figyelem-tudatos…" (paged attention over the mixed cache)."""
    bsz = q.shape[0]
    g = hq // cache.hkv
    out = np.zeros((bsz, hq, D))
    for b in range(bsz):
        length = int(context_lens[b])
        if length == 0:
            continue
        slot = int(seq_slots[b])
        for hk in range(cache.hkv):
            kx = cache.values(slot, 0, hk, length)
            vx = cache.values(slot, 1, hk, length)
            for h in range(hk * g, (hk + 1) * g):
                qr = np.asarray(q[b, h], dtype=np.float64) @ cache.r[0][hk]
                o_rot = attend(qr, kx, vx)
                out[b, h] = o_rot @ cache.r[1][hk].T
    return out


def prefill(cache: Cache, q: np.ndarray, slot: int, context_len: int, hq: int, tokens=None) -> np.ndarray:
    """Attention of a prefill chunk over the cache, causal.

    The chunk's T tokens have been appended, so the sequence in `slot` has
    `context_len` = L tokens and the chunk holds positions L - T .. L - 1.
    q: [T, hq, d] (bf16-exact), query i at position L - T + i.  Query i of
    head h attends to positions 0 .. L - T + i of KV head h // (hq // hkv),
    each read as the cache holds it at length L (the first `sinks` and the
    last W positions from fp16, the rest from INT2: `Cache.values`), with
    q rotated by R_K and the output brought back with R_V^T, as in `decode`.
    Returns fp64 [T, hq, d].  With T = 1 this is `decode` of that sequence.
    `tokens` (optional) lists the chunk indices i to compute; the other rows
    stay zero (a sample of a large chunk, the arithmetic unchanged).
    [AF] "OSCAR: figyelem-tudatos…" and [GH] "Что это даёт на практике"
    (the cache serves paged attention and prefix caching, so prefill chunks
    attend over the compressed history); [GH] "Что придумали в Together AI"
    (rotations of Q and of the attention output)."""
    q = np.asarray(q)
    T = q.shape[0]
    g = hq // cache.hkv
    out = np.zeros((T, hq, D))
    if T == 0:
        return out
    if context_len < T:
        raise ValueError("the chunk's tokens must already be in the cache")
    first = context_len - T
    for hk in range(cache.hkv):
        kx = cache.values(slot, 0, hk, context_len)
        vx = cache.values(slot, 1, hk, context_len)
        for h in range(hk * g, (hk + 1) * g):
            for i in (range(T) if tokens is None else tokens):
                visible = first + i + 1
                qr = np.asarray(q[i, h], dtype=np.float64) @ cache.r[0][hk]
                out[i, h] = attend(qr, kx[:visible], vx[:visible]) @ cache.r[1][hk].T
    return out


# ----------------------------------------------------------------------------
# Sizing arithmetic the pages quote
# ----------------------------------------------------------------------------

def bf16_kv_bytes_per_token(layers: int, hkv: int, d: int = D) -> int:
    """K and V, 2 bytes each, for every layer and KV head.  [EN] section
    "KV cache compression става болезнен…"; [AR] intro (0.31 MB/token)."""
    return layers * hkv * d * 2 * 2


def int2_kv_bytes_per_token(layers: int, hkv: int, d: int = D, group: int = 128) -> int:
    """2-bit codes plus an fp16 scale and fp16 min per group, for K and V."""
    return layers * hkv * 2 * (d * 2 // 8 + (d // group) * 4)


def effective_bits(frac_16bit: float, group: int = 128) -> float:
    """Average bits per KV element with a fraction of tokens kept 16-bit.
    [BS] "Resultados e Métricas de Desempenho" (2.28 bits); [EN] "OSCAR има
    значение…" (about 0.24 % of tokens stay 16-bit at 128K)."""
    int2 = 2.0 + 32.0 / group
    return (1.0 - frac_16bit) * int2 + frac_16bit * 16.0
