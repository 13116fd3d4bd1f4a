#!/usr/bin/env python
"""INT2 KV-cache decode benchmark on B200.

Workload (default, --workload 2): 4 sequences, 32 query heads / 8 KV heads,
head_dim 128, context 100000 tokens in 16-token blocks with a shuffled block
table, 128-token fp16 window, INT2 groups of 128.  One step appends one new
K/V token per sequence through the rotate-quantise kernel and runs decode
attention (query rotation, split-K attention, split combine with the value
un-rotation).  --workload 1 (8 x 32K), 3 (80 layers x 131K, G = 8) and 4 (64
log-uniform contexts plus an 8192-token prefill chunk per step) print the
same line for those workloads.

Timed region: a CUDA graph of K steps, replayed back to back at least 50
times and for at least a second, each replay bracketed by CUDA events, with a
synchronize (and a barrier under torchrun) on both sides; the median replay
gives the value.  Every workload reads more cache per step than the 126 MB L2
holds, so L2 is not flushed.  value = tokens decoded per second over all ranks
(B * K * N / max-over-ranks time).

`--impl reference` times the CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "INT2-KV decode attn achieved HBM GB/s & tokens/s at 100K ctx; append Mtok/s"
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", type=int, choices=[1, 2, 3, 4], default=2,
                    help="1: 8 x 32K (8B-class layer); 2: 4 x 100K decode (default, the headline); "
                         "3: 80 layers x 131K, G = 8; 4: 64 mixed contexts + an 8192-token prefill chunk")
    ap.add_argument("--group", type=int, choices=[32, 64, 128], default=128,
                    help="quantisation group (channels per fp16 scale/min); 128 is the headline format")
    ap.add_argument("--min-reps", type=int, default=50, help="timed replays of the K-step graph, at least")
    ap.add_argument("--min-timed-s", type=float, default=1.0, help="seconds of timed replays, at least")
    return ap.parse_args()


# ----------------------------------------------------------------- plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def job_time_ms(ms, world, dist=None, device="cpu"):
    """The job's time is its slowest rank's: the max over ranks (every rank calls this)."""
    if world == 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_units(units, world, dist=None, device="cpu"):
    """Units (decoded tokens) processed by all ranks together (every rank calls this)."""
    if world == 1:
        return int(units)
    import torch
    t = torch.tensor([int(units)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


class Clocks:
    """nvidia-smi sampler for the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measured_peak_bf16():
    """Dense bf16 tensor peak (burst: the prefill kernel is timed alone)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("decode.cu", "okv_common.cuh"):
        with open(os.path.join(ROOT, "int2_kv_cache_rotate_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload=2):
    """DRAM bytes per decode launch from the last ncu capture of this
    workload, if the kernel source is unchanged since."""
    try:
        with open(os.path.join(PROFILES, "decode_traffic.json")) as f:
            rec = json.load(f)
        if rec.get("source_hash") == kernel_source_hash() and rec.get("workload_id") == workload:
            return rec
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ workload

def workload_config(cfg=2):
    from int2_kv_cache_rotate_b200 import workloads as WL
    return WL.config(cfg)


def int2_bytes_per_token_head(group=128):
    """K and V codes (2 x 32 B) and one fp16 (scale, min) pair per group for each (8 B per group)."""
    return 64 + 8 * (128 // group)


def algorithmic_bytes(lens, hkv, group=128):
    """Cache bytes decode must read: 72 B per INT2 token-head with 128-channel
    groups (80 B with 64, 96 B with 32), 512 B per fp16 window token-head (K and V)."""
    per = int2_bytes_per_token_head(group)
    tot = 0
    for L in lens:
        n_int2 = max(0, L - 128)
        n_win = min(L, 128)
        tot += hkv * (n_int2 * per + n_win * 512)
    return tot


def append_bytes(n, hkv, window_rows):
    """Bytes a bf16 append of n tokens must move: K and V read (2 x 256 B per
    token-head), codes and scales written (72 B per token-head), fp16 window
    rows written (512 B per token-head for the rows that land in the window)."""
    return hkv * (n * (2 * 256 + 72) + window_rows * 512)


def _kv_source(torch, WL, seed, cfg, rank, hkv, dev):
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000003 * (seed + 1) + 7919 * cfg + rank)
    outl = torch.from_numpy(WL.outlier_channels(seed, cfg, 0).astype(np.int64)).to(dev)

    def kv(*shape):
        k = torch.randn((*shape, hkv, 128), generator=gen, device=dev)
        k[..., outl] *= 16.0
        v = torch.randn((*shape, hkv, 128), generator=gen, device=dev)
        return k.to(torch.bfloat16), v.to(torch.bfloat16)

    return gen, kv


def _prefill(torch, okv, cache, table_d, lens, kv, dev, slot_lens=None):
    """bf16 prefill of every sequence through the tensor-core append, in 8192-token chunks."""
    chunk = 8192
    lens_d = torch.as_tensor(np.asarray(slot_lens if slot_lens is not None else lens, np.int32), device=dev)
    for b, L in enumerate(lens):
        for p0 in range(0, int(L), chunk):
            n = min(chunk, int(L) - p0)
            k, v = kv(n)
            okv.append_quantize(cache, k, v, torch.full((n,), b, dtype=torch.int32, device=dev),
                                torch.arange(p0, p0 + n, dtype=torch.int32, device=dev), table_d, lens_d)


class _GraphCall:
    """A step's library calls, run once eagerly and then recorded in a CUDA
    graph that later calls replay (the calls allocate nothing)."""

    def __init__(self, torch, issue):
        self.torch, self.issue, self.graph = torch, issue, None

    def __call__(self):
        torch = self.torch
        if self.graph is not None:
            self.graph.replay()
            return
        self.issue()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            self.issue()
        torch.cuda.current_stream().wait_stream(cap)
        self.graph = g


class DecodeBatch:
    """Workloads 1 and 2: B sequences of one layer; a step appends one bf16
    K/V token per sequence and decodes (okv_decode_step)."""

    kernels_per_step = 3
    decode_launches_per_step = 1

    def __init__(self, cfg, seed, rank, total_steps, torch, okv, WL, group=128):
        self.group = group
        self.wl = wl = WL.config(cfg)
        self.cfg = cfg
        B, hq, hkv = wl.batch, wl.hq, wl.hkv
        L0 = wl.ctx[0]
        dev = torch.device("cuda")
        qc, kc, vc = WL.calibration_set(seed, cfg, 0, hq, hkv, n=1024)
        rot = okv.calibrate_rotations(qc, kc, vc, hq, hkv)
        table, num_blocks = WL.block_table(seed + rank, cfg, [L0] * B, extra_tokens=total_steps + 16)
        self.cache = okv.Cache(hq, hkv, num_blocks, B, table.shape[1], rot["U_K"], rot["U_V"], group=group)
        self.table = torch.from_numpy(table).to(dev)
        gen, kv = _kv_source(torch, WL, seed, cfg, rank, hkv, dev)
        _prefill(torch, okv, self.cache, self.table, [L0] * B, kv, dev)
        torch.cuda.synchronize()
        assert self.cache.device_status() == 0, self.cache.device_status()
        S = total_steps
        self.knew, self.vnew = kv(S, B)
        self.q = torch.randn((S, B, hq, 128), generator=gen, device=dev).to(torch.bfloat16)
        self.pos = (L0 + torch.arange(S, dtype=torch.int32, device=dev))[:, None].repeat(1, B).contiguous()
        self.lens = (self.pos + 1).contiguous()
        self.seq = torch.arange(B, dtype=torch.int32, device=dev)
        self.B, self.hq, self.hkv, self.L0 = B, hq, hkv, L0
        self.ws = okv.workspace(self.cache, B)
        self.out = torch.empty((B, hq, 128), dtype=torch.float32, device=dev)
        self.units_per_step = B

    def issue(self, okv, i, ev=None):
        if ev is not None:
            okv.time_next_decode_kernel(*ev[0])
        okv.decode_step(self.cache, self.knew[i], self.vnew[i], self.seq, self.pos[i], self.lens[i], self.q[i],
                        self.seq, self.table, self.lens[i], out=self.out, ws=self.ws)

    def decode_bytes(self, i):
        return [algorithmic_bytes([self.L0 + i + 1] * self.B, self.hkv, self.group)]

    def e2e_parts(self):
        return [self.knew, self.vnew, self.q, self.pos, self.lens]

    def e2e_call(self, torch, okv, views, out):
        dk, dv, dq, dpos, dlen = views
        return okv.DecodeStepCall(self.cache, dk, dv, self.seq, dpos, dlen, dq, self.seq, self.table, dlen,
                                  out=out, ws=self.ws, graph=True)

    def out_shape(self):
        return (self.B, self.hq, 128)

    def config(self):
        return {"workload": self.wl.name, "batch": self.B, "hq": self.hq, "hkv": self.hkv, "head_dim": 128,
                "context_start": self.L0, "block_tokens": 16, "window": 128, "group": self.group,
                "step": "okv_decode_step: append 1 bf16 K/V token per sequence + decode attention",
                "l2": (f"not flushed: each step reads the {self.decode_bytes(0)[0] / 1e6:.0f} MB cache, "
                       "larger than the 126 MB L2")}


class Layers:
    """Workload 3: an 80-layer model (64 query / 8 KV heads) at 131,072
    tokens, one sequence; a step is one okv_decode_step per layer."""

    kernels_per_step = 3 * 80
    decode_launches_per_step = 80

    def __init__(self, cfg, seed, rank, total_steps, torch, okv, WL, group=128):
        self.group = group
        self.wl = wl = WL.config(cfg)
        self.cfg = cfg
        B, hq, hkv, L0, NL = wl.batch, wl.hq, wl.hkv, wl.ctx[0], wl.layers
        dev = torch.device("cuda")
        table, num_blocks = WL.block_table(seed + rank, cfg, [L0] * B, extra_tokens=total_steps + 16)
        self.table = torch.from_numpy(table).to(dev)
        gen, kv = _kv_source(torch, WL, seed, cfg, rank, hkv, dev)
        self.caches = []
        for layer in range(NL):
            r = np.random.default_rng(np.random.SeedSequence([seed, cfg, layer, 31]))
            uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
            uv = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
            c = okv.Cache(hq, hkv, num_blocks, B, table.shape[1], uk, uv, group=group)
            _prefill(torch, okv, c, self.table, [L0] * B, kv, dev)
            self.caches.append(c)
        torch.cuda.synchronize()
        for c in self.caches:
            assert c.device_status() == 0, c.device_status()
        S = total_steps
        self.knew, self.vnew = kv(S, NL, B)
        self.q = torch.randn((S, NL, B, hq, 128), generator=gen, device=dev).to(torch.bfloat16)
        self.pos = (L0 + torch.arange(S, dtype=torch.int32, device=dev))[:, None].repeat(1, B).contiguous()
        self.lens = (self.pos + 1).contiguous()
        self.seq = torch.arange(B, dtype=torch.int32, device=dev)
        self.B, self.hq, self.hkv, self.L0, self.NL = B, hq, hkv, L0, NL
        self.ws = okv.workspace(self.caches[0], B)
        self.out = torch.empty((NL, B, hq, 128), dtype=torch.float32, device=dev)
        self.units_per_step = B

    def _layer_calls(self, okv, k, v, q, pos, lens, out, ev=None):
        for layer, c in enumerate(self.caches):
            if ev is not None:
                okv.time_next_decode_kernel(*ev[layer])
            okv.decode_step(c, k[layer], v[layer], self.seq, pos, lens, q[layer], self.seq, self.table, lens,
                            out=out[layer], ws=self.ws)

    def issue(self, okv, i, ev=None):
        self._layer_calls(okv, self.knew[i], self.vnew[i], self.q[i], self.pos[i], self.lens[i], self.out, ev)

    def decode_bytes(self, i):
        return [algorithmic_bytes([self.L0 + i + 1] * self.B, self.hkv, self.group)] * self.NL

    def e2e_parts(self):
        return [self.knew, self.vnew, self.q, self.pos, self.lens]

    def e2e_call(self, torch, okv, views, out):
        dk, dv, dq, dpos, dlen = views
        return _GraphCall(torch, lambda: self._layer_calls(okv, dk, dv, dq, dpos, dlen, out))

    def out_shape(self):
        return (self.NL, self.B, self.hq, 128)

    def config(self):
        return {"workload": self.wl.name, "layers": self.NL, "batch": self.B, "hq": self.hq, "hkv": self.hkv,
                "head_dim": 128, "context_start": self.L0, "block_tokens": 16, "window": 128, "group": self.group,
                "step": "80 x okv_decode_step (one per layer): append 1 bf16 K/V token + decode attention",
                "l2": (f"not flushed: each step reads {sum(self.decode_bytes(0)) / 1e9:.2f} GB of cache, "
                       "far more than the 126 MB L2")}


class Mixed:
    """Workload 4: 64 sequences with log-uniform contexts in [1K, 64K] (32 /
    8 heads); a step decodes one token per sequence (okv_decode_step) and
    appends an 8192-token bf16 prefill chunk of another sequence
    (okv_append_quantize, the tensor-core path).  Step i writes the chunk at
    positions [8192 i, 8192 (i + 1)) of the prefill sequence."""

    CHUNK = 8192
    kernels_per_step = 3 + 1
    decode_launches_per_step = 1

    def __init__(self, cfg, seed, rank, total_steps, torch, okv, WL, group=128):
        self.group = group
        self.wl = wl = WL.config(cfg, seed=seed)
        self.cfg = cfg
        B, hq, hkv = wl.batch, wl.hq, wl.hkv
        lens0 = [int(x) for x in wl.ctx]
        dev = torch.device("cuda")
        qc, kc, vc = WL.calibration_set(seed, cfg, 0, hq, hkv, n=1024)
        rot = okv.calibrate_rotations(qc, kc, vc, hq, hkv)
        S = total_steps
        pre_len = S * self.CHUNK
        table, num_blocks = WL.block_table(seed + rank, cfg, lens0 + [pre_len - total_steps - 16],
                                           extra_tokens=total_steps + 16)
        self.cache = okv.Cache(hq, hkv, num_blocks, B + 1, table.shape[1], rot["U_K"], rot["U_V"], group=group)
        self.table = torch.from_numpy(table).to(dev)
        gen, kv = _kv_source(torch, WL, seed, cfg, rank, hkv, dev)
        _prefill(torch, okv, self.cache, self.table, lens0, kv, dev, slot_lens=lens0 + [0])
        torch.cuda.synchronize()
        assert self.cache.device_status() == 0, self.cache.device_status()
        self.knew, self.vnew = kv(S, B)
        self.q = torch.randn((S, B, hq, 128), generator=gen, device=dev).to(torch.bfloat16)
        l0 = torch.as_tensor(np.asarray(lens0, np.int32), device=dev)
        self.pos = (l0[None, :] + torch.arange(S, dtype=torch.int32, device=dev)[:, None]).contiguous()
        # slot lengths after step i: the decoded sequences grow by one, the
        # prefill sequence by one chunk
        self.slot_lens = torch.cat([self.pos + 1, ((torch.arange(S, dtype=torch.int32, device=dev) + 1)
                                                   * self.CHUNK)[:, None]], dim=1).contiguous()
        self.pk, self.pv = kv(S, self.CHUNK)
        self.ppos = (torch.arange(S, dtype=torch.int32, device=dev)[:, None] * self.CHUNK
                     + torch.arange(self.CHUNK, dtype=torch.int32, device=dev)[None, :]).contiguous()
        self.pslot = torch.full((self.CHUNK,), B, dtype=torch.int32, device=dev)
        self.seq = torch.arange(B, dtype=torch.int32, device=dev)
        self.B, self.hq, self.hkv, self.lens0 = B, hq, hkv, lens0
        self.ws = okv.workspace(self.cache, B)
        self.out = torch.empty((B, hq, 128), dtype=torch.float32, device=dev)
        self.units_per_step = B

    def _calls(self, okv, k, v, q, pos, slot_lens, pk, pv, ppos, out, ev=None):
        lens = slot_lens[:self.B]
        if ev is not None:
            okv.time_next_decode_kernel(*ev[0])
        okv.decode_step(self.cache, k, v, self.seq, pos, slot_lens, q, self.seq, self.table, lens, out=out,
                        ws=self.ws)
        okv.append_quantize(self.cache, pk, pv, self.pslot, ppos, self.table, slot_lens)

    def issue(self, okv, i, ev=None):
        self._calls(okv, self.knew[i], self.vnew[i], self.q[i], self.pos[i], self.slot_lens[i], self.pk[i],
                    self.pv[i], self.ppos[i], self.out, ev)

    def decode_bytes(self, i):
        return [algorithmic_bytes([L + i + 1 for L in self.lens0], self.hkv, self.group)]

    def e2e_parts(self):
        return [self.knew, self.vnew, self.q, self.pos, self.slot_lens, self.pk, self.pv, self.ppos]

    def e2e_call(self, torch, okv, views, out):
        dk, dv, dq, dpos, dsl, dpk, dpv, dpp = views
        return _GraphCall(torch, lambda: self._calls(okv, dk, dv, dq, dpos, dsl, dpk, dpv, dpp, out))

    def out_shape(self):
        return (self.B, self.hq, 128)

    def config(self):
        return {"workload": self.wl.name, "batch": self.B, "hq": self.hq, "hkv": self.hkv, "head_dim": 128,
                "contexts": "log-uniform in [1024, 65536], seeded", "context_total": int(sum(self.lens0)),
                "prefill_append_tokens": self.CHUNK, "block_tokens": 16, "window": 128, "group": self.group,
                "step": ("okv_decode_step (1 bf16 token per sequence + decode) and okv_append_quantize of an "
                         "8192-token bf16 prefill chunk"),
                "l2": (f"not flushed: each step reads {self.decode_bytes(0)[0] / 1e6:.0f} MB of cache and "
                       f"{append_bytes(self.CHUNK, self.hkv, 0) / 1e6:.0f} MB of prefill, more than the 126 MB L2")}


BUILDERS = {1: DecodeBatch, 2: DecodeBatch, 3: Layers, 4: Mixed}


L2_FLUSH_BYTES = 256 << 20  # > the 126 MB L2


def timed_launches(torch, fn, reps=50):
    """Device time (us) of each of `reps` calls of fn, L2 flushed before each:
    a 256 MB buffer is written first (outside the timed span); the GPU is busy
    with it while the host enqueues the events and the call, so the span holds
    the call's kernels only."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    ev = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) * 1e3 for e0, e1 in ev]


def prefill_append_rate(torch, okv, WL, seed):
    """Mtok/s of an 8192-token bf16 append (all 8 KV heads, K and V): median
    of 50 launches, L2 flushed before each."""
    n, hkv, hq = 8192, 8, 32
    table, nb = WL.block_table(seed, 4, [n])
    r = np.random.default_rng(seed)
    uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    cache = okv.Cache(hq, hkv, nb, 1, table.shape[1], uk, uk)
    dev = torch.device("cuda")
    k = torch.randn((n, hkv, 128), device=dev).to(torch.bfloat16)
    v = torch.randn((n, hkv, 128), device=dev).to(torch.bfloat16)
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    lens = torch.tensor([n], dtype=torch.int32, device=dev)
    td = torch.from_numpy(table).to(dev)
    for _ in range(3):
        okv.append_quantize(cache, k, v, seq, pos, td, lens)
    torch.cuda.synchronize()
    us = statistics.median(timed_launches(torch, lambda: okv.append_quantize(cache, k, v, seq, pos, td, lens)))
    moved = append_bytes(n, hkv, 128)
    peak, src = measured_peak_hbm()
    return {"tokens": n, "us": round(us, 2), "mtok_s": round(n / us, 3), "gbs": round(moved / us / 1e3, 1),
            "bytes": moved, "frac_hbm": round(moved / us / 1e3 / peak, 4), "peak_source": src,
            "timing": "median of 50 launches, L2 flushed before each"}


def prefill_attention_rate(torch, okv, WL, seed, L=32768, T=1024, group=128):
    """Chunked-prefill attention: a T-token chunk at the end of an L-token
    sequence (32 query / 8 KV heads) attends causally over the cache; median
    of 50 calls (query rotation, attention, un-rotation), L2 flushed before
    each.  flops counts the causal score and value products (2 x 2 x 128 per
    visible (query head, key) pair); the tensor cores run twice that (hi and
    lo fp16 halves of the query and of p s)."""
    hq, hkv = 32, 8
    table, nb = WL.block_table(seed, 1, [L], extra_tokens=16)
    r = np.random.default_rng(seed + 5)
    uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
    cache = okv.Cache(hq, hkv, nb, 1, table.shape[1], uk, uk, group=group)
    dev = torch.device("cuda")
    td = torch.from_numpy(table).to(dev)
    gen, kv = _kv_source(torch, WL, seed, 1, 0, hkv, dev)
    _prefill(torch, okv, cache, td, [L], kv, dev)
    q = torch.randn((T, hq, 128), generator=gen, device=dev).to(torch.bfloat16)
    ws = torch.empty(okv.prefill_workspace_bytes(cache, T), dtype=torch.uint8, device=dev)
    out = torch.empty((T, hq, 128), dtype=torch.float32, device=dev)
    for _ in range(3):
        okv.prefill_attention(cache, q, 0, L, td, out=out, ws=ws)
    torch.cuda.synchronize()
    us = statistics.median(timed_launches(torch, lambda: okv.prefill_attention(cache, q, 0, L, td, out=out, ws=ws)))
    visible = sum(L - T + i + 1 for i in range(T))
    flops = 4 * 128 * hq * visible
    peak, src = measured_peak_bf16()
    tflops = flops / us / 1e6
    return {"context": L, "chunk_tokens": T, "hq": hq, "hkv": hkv, "group": group,
            "kernel": "tcgen05", "us": round(us, 1),
            "tflops": round(tflops, 1), "flops": flops,
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tflops / peak, 4), "peak_source": src,
                         "note": "useful flops; f16 and bf16 share the dense tensor rate; the kernel issues "
                                 "2x these flops (hi + lo halves)"},
            "timing": "median of 50 calls, L2 flushed before each"}


# ---------------------------------------------------------------- oracle arm

def oracle_unit(seed, cfg, L, g, group=128):
    """Oracle cache for one (sequence, KV head) unit at L tokens."""
    from int2_kv_cache_rotate_b200 import workloads as WL
    from oracle import okv_oracle as O
    r = np.random.default_rng(np.random.SeedSequence([seed, 77]))
    cache = O.Cache(1, WL.haar_orthogonal(r)[None], WL.haar_orthogonal(r)[None], group=group)
    k = WL.sample_keys(seed, cfg, 0, 0, L, extra=0)[:, None, :]
    v = WL.sample_values(seed, cfg, 0, 0, L, extra=0)[:, None, :]
    cache.append(0, 0, k, v)
    return {"cache": cache, "L": L, "g": g, "cfg": cfg}


def oracle_unit_step(unit, i, seed):
    """One decode step of the sampled unit: append one token, attend with its G query heads."""
    from int2_kv_cache_rotate_b200 import workloads as WL
    from oracle import okv_oracle as O
    g, L, cfg = unit["g"], unit["L"], unit["cfg"]
    pos = L + i
    kn = WL.sample_keys(seed, cfg, 0, 0, 1, extra=100 + i)[:, None, :]
    vn = WL.sample_values(seed, cfg, 0, 0, 1, extra=100 + i)[:, None, :]
    q = WL.sample_queries(seed, cfg, 0, 0, 1, g, extra=100 + i)
    t0 = time.perf_counter()
    unit["cache"].append(0, pos, kn, vn)
    O.decode(unit["cache"], q, [0], [pos + 1], g)
    return time.perf_counter() - t0


def oracle_append_seconds_per_token_head(seed, n=256):
    """Oracle append (fp64 rotation + quantiser) of n bf16 tokens of one KV head, K and V; seconds per token-head."""
    from int2_kv_cache_rotate_b200 import workloads as WL
    from oracle import okv_oracle as O
    r = np.random.default_rng(np.random.SeedSequence([seed, 78]))
    cache = O.Cache(1, WL.haar_orthogonal(r)[None], WL.haar_orthogonal(r)[None])
    k = WL.sample_keys(seed, 4, 0, 0, n, extra=1)[:, None, :]
    v = WL.sample_values(seed, 4, 0, 0, n, extra=1)[:, None, :]
    t0 = time.perf_counter()
    cache.append(0, 0, k, v)
    return (time.perf_counter() - t0) / n


class OracleSample:
    """The oracle on a bounded sample of a workload, scaled to the full step.

    Decode cost is taken as proportional to context length: one (sequence,
    KV head) unit is timed at a stated length and scaled by the workload's
    total token-heads (over layers and KV heads).  Workload 4 adds the oracle
    append of the step's 8192-token chunk, timed on 256 tokens of one head."""

    def __init__(self, cfg, seed, group=128):
        wl = workload_config(cfg) if cfg != 4 else __import__(
            "int2_kv_cache_rotate_b200.workloads", fromlist=["config"]).config(4, seed=seed)
        self.cfg, self.wl, self.seed = cfg, wl, seed
        lens = [int(x) for x in wl.ctx]
        self.L = int(statistics.median(lens))
        self.g = wl.hq // wl.hkv
        self.scale = sum(lens) * wl.hkv * wl.layers / self.L  # token-heads of a step / the unit's tokens
        self.unit = oracle_unit(seed, cfg, self.L, self.g, group)
        self.app_tokens = wl.prefill_append * wl.hkv  # token-heads appended by the prefill chunk

    def step_seconds(self, i):
        """Returns (scaled step seconds, the sampled unit's own seconds)."""
        t = oracle_unit_step(self.unit, i, self.seed)
        total = t * self.scale
        if self.app_tokens:
            total += oracle_append_seconds_per_token_head(self.seed + i) * self.app_tokens
        return total, t

    def sample_text(self, reps):
        txt = (f"one decode step (1-token append + attention of its {self.g} query heads) of one (sequence, KV "
               f"head) unit at {self.L} tokens, NumPy fp64, median of {reps}; scaled x{self.scale:.0f} to the "
               f"step's token-heads")
        if self.app_tokens:
            txt += f"; plus the oracle append of 256 tokens of one head, scaled to {self.app_tokens} token-heads"
        return txt


def cpu_baseline(cfg, seed, steps=3, group=128):
    cores = len(os.sched_getaffinity(0))
    o = OracleSample(cfg, seed, group)
    ts = [o.step_seconds(i)[0] for i in range(steps)]
    step_s = statistics.median(ts)
    out = {"value": round(o.wl.batch / step_s, 6), "unit": "tok/s", "cores": cores, "kind": "oracle",
           "sample": o.sample_text(steps)}
    if o.app_tokens:
        out["append_mtok_s"] = round(1.0 / oracle_append_seconds_per_token_head(seed) / o.wl.hkv / 1e6, 6)
    return out


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    cfg = getattr(args, "workload", 2)
    group = getattr(args, "group", 128)
    cores = len(os.sched_getaffinity(0))
    o = OracleSample(cfg, args.seed, group)
    for i in range(args.warmup):
        o.step_seconds(i)
    res = [o.step_seconds(args.warmup + i) for i in range(args.steps)]
    per_step = sum(r[0] for r in res) / len(res)
    per_unit = sum(r[1] for r in res) / len(res)
    value = o.wl.batch / per_step
    cfgblock = dict(reference_config_block(o.wl, cfg), group=group)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfgblock,
        "measured": {"unit_ms_per_step": round(per_unit * 1e3, 3), "unit_tokens": o.L,
                     "scaled_by": round(o.scale, 3),
                     "note": "ms_per_step is unit_ms_per_step x scaled_by (plus the sampled append, workload 4)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": o.sample_text(args.steps)},
        "e2e": {"value": round(value, 6), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def reference_config_block(wl, cfg):
    return {"workload": wl.name, "batch": wl.batch, "hq": wl.hq, "hkv": wl.hkv, "head_dim": 128,
            "context_start": int(wl.ctx[0]) if cfg != 4 else None, "layers": wl.layers, "block_tokens": 16,
            "window": 128, "group": 128,
            "timed_as": ("NumPy fp64 oracle on the host cores, wall clock per step; each step one (sequence, KV "
                         "head) unit, scaled to the step's token-heads")}


# ------------------------------------------------------------------ our arm

def timed_replays(torch, graph, min_reps, min_s, max_reps=4000):
    """Replay a K-step graph at least min_reps times and for at least min_s
    seconds, each replay bracketed by CUDA events; returns the per-replay ms."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    est = max(e0.elapsed_time(e1), 1e-3)
    reps = int(min(max_reps, max(min_reps, math.ceil(min_s * 1e3 / est))))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_e2e(w, base, steps, torch, okv, world, dist):
    """End to end through the public calls, as a serving loop runs them: each
    step's inputs packed in pinned host memory and sent with one host-to-device
    copy into one of two staging buffers; the step's calls (replayed from a
    CUDA graph after their first run) read that buffer's views; the output is
    read back to pinned host memory.  The copies run on a copy stream, so that
    step i + 1's inputs and step i's output move while the GPU computes;
    events keep each buffer from being reused before the step that reads it
    has finished."""
    parts = w.e2e_parts()  # each [steps][...]
    sizes = [x[0].numel() * x.element_size() for x in parts]
    offs = []
    off = 0
    for sz in sizes:
        offs.append(off)
        off = (off + sz + 255) // 256 * 256
    step_bytes = off
    # pinned host rows for steps base - 1 .. base + steps - 1 (row r is step base - 1 + r)
    rows = steps + 1
    host_rows = torch.zeros((rows, step_bytes), dtype=torch.uint8).pin_memory()
    for j, x in enumerate(parts):
        host_rows[:, offs[j]:offs[j] + sizes[j]] = \
            x[base - 1:base + steps].cpu().contiguous().view(rows, -1).view(torch.uint8)

    class _Rows:
        def __getitem__(self, i):
            return host_rows[i - (base - 1)]

    host = _Rows()
    hout = torch.empty((2, *w.out_shape()), dtype=torch.float32).pin_memory()
    devs, outs, calls = [], [], []
    for slot in range(2):
        dev = torch.empty(step_bytes, dtype=torch.uint8, device="cuda")
        views = [dev[offs[j]:offs[j] + sizes[j]].view(x.dtype).view(x[0].shape) for j, x in enumerate(parts)]
        o = torch.empty(w.out_shape(), dtype=torch.float32, device="cuda")
        devs.append(dev)
        outs.append(o)
        calls.append(w.e2e_call(torch, okv, views, o))
    # first call of each (eager, then recorded): step base - 1 again, which the
    # timed graphs already ran (same tokens, same positions: the same bytes)
    for slot in range(2):
        devs[slot].copy_(host[base - 1], non_blocking=True)
        calls[slot]()
    torch.cuda.synchronize()
    main, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    inputs_in, step_done, output_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    copy.wait_stream(main)

    def upload(i):
        slot = i % 2
        with torch.cuda.stream(copy):
            if i - 2 >= base:
                copy.wait_event(step_done[slot])  # step i - 2 no longer reads this buffer
            devs[slot].copy_(host[i], non_blocking=True)
            inputs_in[slot].record(copy)

    upload(base)
    for i in range(base, base + steps):
        slot = i % 2
        if i + 1 < base + steps:
            upload(i + 1)
        main.wait_event(inputs_in[slot])
        if i - 2 >= base:
            main.wait_event(output_out[slot])  # step i - 2's output has left this buffer
        calls[slot]()
        step_done[slot].record(main)
        with torch.cuda.stream(copy):
            copy.wait_event(step_done[slot])
            hout[slot].copy_(outs[slot], non_blocking=True)
            output_out[slot].record(copy)
    main.wait_stream(copy)
    e1.record(main)
    torch.cuda.synchronize()
    e_ms = job_time_ms(e0.elapsed_time(e1), world, dist, "cuda")
    e_units = job_units(w.units_per_step * steps, world, dist, "cuda")
    return {"value": round(e_units / (e_ms * 1e-3), 2), "unit": "tok/s",
            "h2d_bytes_per_step": int(sum(sizes)), "d2h_bytes_per_step": int(hout[0].numel() * 4),
            "ms_per_step": round(e_ms / steps, 4),
            "timed_as": "one step at a time, as a serving loop: one packed host-to-device copy of the step's "
                        "inputs and one device-to-host copy of its output on a copy stream (double-buffered, "
                        "overlapping the neighbouring steps' kernels), the step's library calls replayed from a "
                        "CUDA graph"}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from int2_kv_cache_rotate_b200 import okv
    from int2_kv_cache_rotate_b200 import workloads as WL

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    K, W = args.steps, args.warmup
    e2e_steps = 0 if args.no_e2e else K
    total = W + K + e2e_steps + 1
    w = BUILDERS[args.workload](args.workload, args.seed, rank, total, torch, okv, WL, group=args.group)
    # eager pre-warm (idempotent with graph step 0: same tokens, same positions)
    w.issue(okv, 0)
    torch.cuda.synchronize()

    nd = w.decode_launches_per_step
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nd)]
           for _ in range(K)]
    for row in evs:
        for a, b in row:
            a.record()
            b.record()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    # g_time: the K timed steps as a user runs them; g_kern: the same steps with
    # events around each split-K kernel (the library then launches that kernel
    # and the combine without overlapping their neighbours), for the roofline
    g_warm, g_time, g_kern = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=cap):
        for i in range(W):
            w.issue(okv, i)
    with torch.cuda.graph(g_time, stream=cap):
        for i in range(K):
            w.issue(okv, W + i)
    with torch.cuda.graph(g_kern, stream=cap):
        for i in range(K):
            w.issue(okv, W + i, ev=evs[i])
    g_warm.replay()
    torch.cuda.synchronize()
    kern_reps = 5
    dec_us = []
    for _ in range(kern_reps):
        g_kern.replay()
        torch.cuda.synchronize()
        dec_us.append(statistics.mean(a.elapsed_time(b) * 1e3 for row in evs for a, b in row))
    if world > 1:
        dist.barrier()
    clocks = Clocks(local)
    clocks.start()
    torch.cuda.synchronize()
    reps_ms = timed_replays(torch, g_time, args.min_reps, args.min_timed_s)
    clk = clocks.stop()
    ms = job_time_ms(statistics.median(reps_ms), world, dist, "cuda")
    units = job_units(w.units_per_step * K, world, dist, "cuda")
    if world > 1:
        dist.barrier()
    for c in getattr(w, "caches", [getattr(w, "cache", None)]):
        assert c.device_status() == 0, c.device_status()

    e2e = run_e2e(w, W + K, e2e_steps, torch, okv, world, dist) if e2e_steps else None
    append_rate = prefill_append_rate(torch, okv, WL, args.seed) if rank == 0 else None
    prefill_rate = (prefill_attention_rate(torch, okv, WL, args.seed, group=args.group)
                    if rank == 0 and args.workload == 2 else None)

    if rank == 0:
        alg = statistics.mean(statistics.mean(w.decode_bytes(W + i)) for i in range(K))
        dec_mean = statistics.median(dec_us)
        achieved = alg / (dec_mean * 1e-6) / 1e9
        peak, peak_src = measured_peak_hbm()
        tr = recorded_traffic(args.workload) if args.group == 128 else None  # captured: the group-128 kernel
        line = {
            "metric": METRIC,
            "value": round(units / (ms * 1e-3), 2),
            "unit": "tok/s",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "s8/u8-mma+f32", "data": "synthetic",
            "config": dict(w.config(), timed_as=(
                f"CUDA graph of K steps replayed {len(reps_ms)} times back to back, each replay bracketed by CUDA "
                f"events; value from the median replay; split-K kernel time from a second graph of the same "
                f"steps with events around each split-K kernel (median of {kern_reps} replays)")),
            "timing": {"reps": len(reps_ms), "replay_ms_median": round(statistics.median(reps_ms), 4),
                       "replay_ms_min": round(min(reps_ms), 4), "replay_ms_max": round(max(reps_ms), 4),
                       "timed_region_s": round(sum(reps_ms) / 1e3, 3)},
            "hbm_gbs": round(achieved, 1),
            "decode_kernel_us": round(dec_mean, 3),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_source": peak_src,
                         "traffic": (tr["bytes_per_launch"] if tr else None),
                         "kernel": ("split-K INT2 decode attention" if args.group == 128 else
                                    "split-K INT2 decode attention, per-group scales"),
                         "int2_bytes_per_token_head": int2_bytes_per_token_head(args.group),
                         "algorithmic_bytes_per_launch": int(alg)},
            "append_prefill": append_rate,
            "prefill_attention": prefill_rate,
            "e2e": e2e,
            "gpu_launches": w.kernels_per_step * K * len(reps_ms),
            "clocks": clk,
        }
        if args.workload == 4:
            step_app = append_bytes(Mixed.CHUNK, w.hkv, 128)
            line["append_in_step"] = {"tokens_per_step": Mixed.CHUNK,
                                      "mtok_s_at_step_rate": round(Mixed.CHUNK * K / (ms * 1e3), 3),
                                      "bytes_per_step": step_app}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args.workload, args.seed, group=args.group)
            if append_rate is not None:
                # the oracle's append beside the GPU's: fp64 rotation + quantiser, 256 tokens of one head
                append_rate["cpu_baseline_mtok_s"] = round(
                    1.0 / oracle_append_seconds_per_token_head(args.seed) / 8 / 1e6, 6)
        print(json.dumps(line), flush=True)
    del g_warm, g_time, g_kern
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
