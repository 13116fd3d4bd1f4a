"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no arithmetic of the quantisation method: it only draws
random numbers and lays out shapes.  Both the CUDA path and the CPU oracle
receive what it produces, so it is the single source of inputs for parity.

Generative model (the same for every workload; shapes come from ``CONFIGS``):

* queries ~ N(0, Sigma), Sigma = O diag(logspace(0, -3, d)) O^T, with O a
  Haar-random orthogonal matrix drawn per (layer, KV head) and shared by the G
  query heads of that group; values are rounded to bf16;
* keys ~ N(0, 1) with four outlier channels (fixed per layer) scaled by 16,
  rounded to bf16;
* values ~ N(0, 1), rounded to bf16;
* block tables: a random permutation of the physical 16-token blocks handed
  out to the sequences in order.

Every stream is a ``numpy.random.SeedSequence([seed, config, layer, kv_head,
kind, extra])``, so a sampled (sequence, head) can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

D = 128          # head dimension
BLOCK = 16       # tokens per cache block
WINDOW = 128     # recent tokens also kept in fp16
GROUP = 128      # quantisation group (one group per token-head)
N_CALIB = 4096   # calibration queries (and keys/values) per KV head

# stream kinds
K_BASIS, K_CALIB_Q, K_CALIB_K, K_CALIB_V, K_Q, K_K, K_V, K_OUTLIER, K_BLOCKS, K_LENS, K_Z = range(11)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    ctx: tuple            # per-sequence context lengths
    layers: int = 1
    steps: int = 1        # decode steps (each appends one token per sequence)
    prefill_append: int = 0  # bf16 tokens appended per step by the prefill path

    @property
    def group_size(self) -> int:
        return self.hq // self.hkv


def _log_uniform_lens(seed: int, n: int, lo: int, hi: int) -> tuple:
    r = stream(seed, 4, 0, 0, K_LENS)
    x = np.exp(r.uniform(math.log(lo), math.log(hi), size=n))
    return tuple(int(v) for v in np.round(x))


def config(idx: int, seed: int = 0) -> Workload:
    """The five workloads: tiny, Qwen3-8B-shaped, 100K decode, Llama-3.1-70B-shaped, mixed."""
    if idx == 0:
        return Workload("tiny-b1-h4x1-L2048", 1, 4, 1, (2048,))
    if idx == 1:
        return Workload("qwen3-8b-layer-b8-L32768", 8, 32, 8, (32768,) * 8)
    if idx == 2:
        return Workload("decode-100k-b4-h32x8", 4, 32, 8, (100000,) * 4, steps=64)
    if idx == 3:
        return Workload("llama-3.1-70b-80L-b1-L131072", 1, 64, 8, (131072,), layers=80)
    if idx == 4:
        return Workload("mixed-64seq-logU1k-64k", 64, 32, 8, _log_uniform_lens(seed, 64, 1024, 65536),
                        prefill_append=8192)
    raise ValueError(idx)


def stream(seed: int, cfg: int, layer: int, kv_head: int, kind: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, cfg, layer, kv_head, kind, extra]))


def to_bf16_exact(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def haar_orthogonal(rng: np.random.Generator, d: int = D) -> np.ndarray:
    a = rng.standard_normal((d, d))
    qm, rm = np.linalg.qr(a)
    return qm * np.sign(np.diag(rm))[None, :]


def query_spectrum(d: int = D) -> np.ndarray:
    return np.logspace(0.0, -3.0, d)


def query_basis(seed: int, cfg: int, layer: int, kv_head: int) -> np.ndarray:
    return haar_orthogonal(stream(seed, cfg, layer, kv_head, K_BASIS))


def sample_queries(seed: int, cfg: int, layer: int, kv_head: int, n: int, group: int,
                   kind: int = K_Q, extra: int = 0) -> np.ndarray:
    """[n, group, D] float32 (bf16-exact) draws from N(0, O diag(spectrum) O^T)."""
    o = query_basis(seed, cfg, layer, kv_head)
    z = stream(seed, cfg, layer, kv_head, kind, extra).standard_normal((n, group, D))
    q = (z * np.sqrt(query_spectrum())) @ o.T
    return to_bf16_exact(q.astype(np.float32))


def outlier_channels(seed: int, cfg: int, layer: int) -> np.ndarray:
    return np.sort(stream(seed, cfg, layer, 0, K_OUTLIER).choice(D, size=4, replace=False))


def sample_keys(seed: int, cfg: int, layer: int, kv_head: int, n: int, kind: int = K_K,
                extra: int = 0) -> np.ndarray:
    """[n, D] float32 (bf16-exact): N(0,1) with four outlier channels x16."""
    k = stream(seed, cfg, layer, kv_head, kind, extra).standard_normal((n, D)).astype(np.float32)
    k[:, outlier_channels(seed, cfg, layer)] *= 16.0
    return to_bf16_exact(k)


def sample_values(seed: int, cfg: int, layer: int, kv_head: int, n: int, kind: int = K_V,
                  extra: int = 0) -> np.ndarray:
    """[n, D] float32 (bf16-exact): N(0,1)."""
    v = stream(seed, cfg, layer, kv_head, kind, extra).standard_normal((n, D)).astype(np.float32)
    return to_bf16_exact(v)


def sample_rotated(seed: int, cfg: int, layer: int, kv_head: int, n: int, kind: int,
                   extra: int = 0, scale: float = 1.0) -> np.ndarray:
    """[n, D] float32 stand-ins for already-rotated vectors (fed with the pre-rotated flag)."""
    r = stream(seed, cfg, layer, kv_head, K_Z, extra * 2 + kind)
    return (r.standard_normal((n, D)) * scale).astype(np.float32)


def calibration_set(seed: int, cfg: int, layer: int, hq: int, hkv: int, n: int = N_CALIB):
    """Calibration queries [n, hq, D] and keys/values [n, hkv, D] (float32, bf16-exact)."""
    g = hq // hkv
    q = np.stack([sample_queries(seed, cfg, layer, h, n, g, kind=K_CALIB_Q) for h in range(hkv)], axis=1)
    q = q.reshape(n, hq, D)
    k = np.stack([sample_keys(seed, cfg, layer, h, n, kind=K_CALIB_K) for h in range(hkv)], axis=1)
    v = np.stack([sample_values(seed, cfg, layer, h, n, kind=K_CALIB_V) for h in range(hkv)], axis=1)
    return q, k, v


def blocks_needed(ctx: int, block: int = BLOCK) -> int:
    return (ctx + block - 1) // block


def block_table(seed: int, cfg: int, lens, extra_tokens: int = 0, spare_blocks: int = 0,
                layer: int = 0):
    """Shuffled physical blocks for each sequence.

    Returns (table [n_seq, max_blocks] int32 padded with -1, num_blocks)."""
    per = [blocks_needed(int(L) + extra_tokens) for L in lens]
    total = sum(per) + spare_blocks
    perm = stream(seed, cfg, layer, 0, K_BLOCKS).permutation(total).astype(np.int32)
    width = max(per) if per else 0
    table = np.full((len(per), max(width, 1)), -1, dtype=np.int32)
    off = 0
    for i, n in enumerate(per):
        table[i, :n] = perm[off:off + n]
        off += n
    return table, total
