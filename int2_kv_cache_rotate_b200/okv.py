"""Thin ctypes binding over ``libokv.so`` (argument marshalling only).

Every step of the hot path runs in the library's CUDA kernels; this module
checks dtypes/devices/shapes of torch tensors, passes raw pointers and the
current CUDA stream, and turns non-OK statuses into ``OkvError``.  Nothing
here computes any part of the method.  If the library is missing the first
call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# OKV_LIBRARY names another in-tree build of the same library (the short-wait
# test build); by default the binding loads libokv.so
LIB_PATH = os.environ.get("OKV_LIBRARY") or os.path.join(_HERE, "libokv.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "okv.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_NUMERIC, ERR_IO = range(6)
DEV_BAD_BLOCK, DEV_BAD_POS, DEV_BAD_SLOT, DEV_TIMEOUT = 1, 2, 4, 8
PRE_ROTATED = 1
HEAD_DIM, BLOCK_TOKENS, WINDOW, BLOCK_HEAD_BYTES = 128, 16, 128, 1152


class OkvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status}: {msg}")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("group", ctypes.c_int32),
        ("block_tokens", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("num_seq_slots", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("num_sink", ctypes.c_int32),
        ("pages", ctypes.c_void_p),
        ("window_ring", ctypes.c_void_p),
        ("u_k", ctypes.c_void_p),
        ("u_v", ctypes.c_void_p),
        ("status_word", ctypes.c_void_p),
        ("sink_rows", ctypes.c_void_p),
        ("r_image", ctypes.c_void_p),
    ]


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32
_SZ = ctypes.c_size_t
_DESC = ctypes.POINTER(CacheDesc)

_SIGNATURES = {
    "okv_calibrate_rotations": (_I32, [_P, _I64, _P, _P, _I64, _I32, _I32, _I32, _P, _P, _P, _P]),
    "okv_pages_bytes": (_SZ, [_I32, _I32, _I32]),
    "okv_block_head_bytes": (_SZ, [_I32]),
    "okv_window_bytes": (_SZ, [_I32, _I32]),
    "okv_sink_bytes": (_SZ, [_I32, _I32, _I32]),
    "okv_r_image_bytes": (_SZ, [_I32]),
    "okv_build_r_image": (_I32, [_DESC, _P]),
    "okv_append_quantize": (_I32, [_DESC, _P, _P, _I32, _P, _P, _P, _P, _U32, _P, _P]),
    "okv_decode_workspace_bytes": (_SZ, [_DESC, _I32]),
    "okv_decode_attention": (_I32, [_DESC, _P, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "okv_dequantize": (_I32, [_DESC, _I32, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P]),
    "okv_status_string": (ctypes.c_char_p, [_I32]),
    "okv_last_error_string": (ctypes.c_char_p, []),
    "okv_version": (_I32, []),
    "okv_time_next_decode_kernel": (_I32, [_P, _P]),
    "okv_decode_attention_noalloc": (_I32, [_DESC, _P, _I32, _P, _P, _P, _P, _P]),
    "okv_prefill_workspace_bytes": (_SZ, [_DESC, _I32]),
    "okv_prefill_attention": (_I32, [_DESC, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "okv_decode_step": (_I32, [_DESC, _P, _P, _I32, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "okv_save_rotations": (_I32, [ctypes.c_char_p, _I32, _I32, _I32, _P, _P, ctypes.c_char_p]),
    "okv_rotations_file_shape": (_I32, [ctypes.c_char_p, _P, _P, _P, _P]),
    "okv_load_rotations": (_I32, [ctypes.c_char_p, _I32, _I32, _I32, _P, _P, _P, _SZ, _I32]),
}


def lib() -> ctypes.CDLL:
    """Load ``libokv.so`` (built in-tree); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OkvError(-1, f"{LIB_PATH} is missing: run `python -m int2_kv_cache_rotate_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def header_functions() -> list:
    """Names of the functions ``include/okv.h`` declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(okv_[a-z0-9_]+)\s*\(", text)))


def _check(status: int):
    if status != OK:
        msg = lib().okv_last_error_string().decode()
        raise OkvError(status, msg)


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, dtype, name, device=True):
    import torch
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ---------------------------------------------------------------- calibration

def calibrate_rotations(q: np.ndarray, k: np.ndarray, v: np.ndarray, hq: int, hkv: int) -> dict:
    """Host fp64 calibration.  q [nq, hq, 128], k/v [nk, hkv, 128] (float32)."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = {n: np.zeros((hkv, HEAD_DIM, HEAD_DIM), np.float32) for n in ("R_K", "R_V", "U_K", "U_V")}
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().okv_calibrate_rotations(p(q), q.shape[0], p(k), p(v), k.shape[0], hq, hkv, q.shape[-1],
                                         p(out["R_K"]), p(out["R_V"]), p(out["U_K"]), p(out["U_V"])))
    return out


# ---------------------------------------------------------------------- cache

class Cache:
    """Device buffers of one layer's INT2 cache plus its C descriptor.

    Memory comes from torch (the caller's allocator); the library only
    receives pointers."""

    def __init__(self, hq: int, hkv: int, num_blocks: int, num_seq_slots: int, max_blocks_per_seq: int,
                 u_k, u_v, device="cuda", num_sink: int = 0, group: int = HEAD_DIM, stage_r: bool = True):
        import torch
        self.hq, self.hkv, self.num_sink, self.group = hq, hkv, num_sink, group
        self.num_blocks, self.num_seq_slots, self.max_blocks_per_seq = num_blocks, num_seq_slots, max_blocks_per_seq
        self.block_head_bytes = int(lib().okv_block_head_bytes(group))
        nbytes = lib().okv_pages_bytes(num_blocks, hkv, group)
        self.pages = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.ring = torch.zeros((num_seq_slots, hkv, 2, WINDOW, HEAD_DIM), dtype=torch.float16, device=device)
        self.u_k = torch.as_tensor(np.asarray(u_k, dtype=np.float32)).to(device).contiguous()
        self.u_v = torch.as_tensor(np.asarray(u_v, dtype=np.float32)).to(device).contiguous()
        self.status = torch.zeros(4, dtype=torch.int32, device=device)
        # first num_sink positions of every sequence, fp16 (sink tokens)
        self.sink = torch.zeros((num_seq_slots, hkv, 2, max(num_sink, 0), HEAD_DIM), dtype=torch.float16,
                                device=device)
        # the prefill append's staged R of every (KV head, K|V), built once from U
        self.r_image = torch.empty(max(int(lib().okv_r_image_bytes(hkv)), 16), dtype=torch.uint8, device=device) \
            if stage_r else None
        self.desc = CacheDesc(hq, hkv, HEAD_DIM, group, BLOCK_TOKENS, WINDOW, num_blocks, num_seq_slots,
                              max_blocks_per_seq, num_sink, self.pages.data_ptr(), self.ring.data_ptr(),
                              self.u_k.data_ptr(), self.u_v.data_ptr(), self.status.data_ptr(),
                              self.sink.data_ptr() if num_sink > 0 else None,
                              self.r_image.data_ptr() if stage_r else None)
        if stage_r:
            self.rebuild_r_image()

    def rebuild_r_image(self, stream=None):
        """Stage R from u_k, u_v into the image buffer again (after changing them)."""
        _check(lib().okv_build_r_image(ctypes.byref(self.desc), _stream(stream)))

    def device_status(self) -> int:
        return int(self.status[0].item())

    def clear_status(self):
        self.status.zero_()


def save_rotations(path, u_k, u_v, tag: str = "") -> None:
    """Write U_K and U_V (host fp32 [layers][Hkv][128][128], or [Hkv][128][128]
    for one layer) to a rotations file."""
    uk = np.ascontiguousarray(u_k, dtype=np.float32)
    uv = np.ascontiguousarray(u_v, dtype=np.float32)
    if uk.ndim == 3:
        uk, uv = uk[None], uv[None]
    if uk.ndim != 4 or uv.shape != uk.shape or uk.shape[2] != uk.shape[3]:
        raise ValueError(f"u_k {uk.shape} and u_v {uv.shape} must both be [layers][Hkv][d][d]")
    layers, hkv, d, _ = uk.shape
    _check(lib().okv_save_rotations(os.fsencode(path), layers, hkv, d, uk.ctypes.data, uv.ctypes.data,
                                    tag.encode("utf-8")))


def load_rotations(path, verify: bool = True) -> dict:
    """Read a rotations file: {"U_K", "U_V": fp32 [layers][Hkv][d][d], "tag": str}."""
    p = os.fsencode(path)
    layers, hkv, d, tag_len = (ctypes.c_int32() for _ in range(4))
    _check(lib().okv_rotations_file_shape(p, ctypes.byref(layers), ctypes.byref(hkv), ctypes.byref(d),
                                          ctypes.byref(tag_len)))
    shape = (layers.value, hkv.value, d.value, d.value)
    uk, uv = np.empty(shape, np.float32), np.empty(shape, np.float32)
    tag = ctypes.create_string_buffer(tag_len.value + 1)
    _check(lib().okv_load_rotations(p, layers.value, hkv.value, d.value, uk.ctypes.data, uv.ctypes.data, tag,
                                    tag_len.value + 1, int(verify)))
    return {"U_K": uk, "U_V": uv, "tag": tag.value.decode("utf-8")}


def append_quantize(cache: Cache, k, v, seq_slot, pos, block_table, slot_lens, pre_rotated=False,
                    rotated_out=None, stream=None):
    import torch
    dt = torch.float32 if pre_rotated else torch.bfloat16
    _need(k, dt, "k"), _need(v, dt, "v")
    for name, t in (("seq_slot", seq_slot), ("pos", pos), ("block_table", block_table), ("slot_lens", slot_lens)):
        _need(t, torch.int32, name)
    if rotated_out is not None:
        _need(rotated_out, torch.float32, "rotated_out")
    T = k.shape[0] if k.dim() > 0 else 0
    _check(lib().okv_append_quantize(ctypes.byref(cache.desc), _ptr(k), _ptr(v), T, _ptr(seq_slot), _ptr(pos),
                                     _ptr(block_table), _ptr(slot_lens), PRE_ROTATED if pre_rotated else 0,
                                     _ptr(rotated_out), _stream(stream)))


def decode_workspace_bytes(cache: Cache, batch: int) -> int:
    return int(lib().okv_decode_workspace_bytes(ctypes.byref(cache.desc), batch))


def workspace(cache: Cache, batch: int):
    import torch
    return torch.empty(max(decode_workspace_bytes(cache, batch), 256), dtype=torch.uint8, device="cuda")


def decode_attention(cache: Cache, q, seq_slot, block_table, context_lens, out=None, ws=None, stream=None):
    import torch
    _need(q, torch.bfloat16, "q")
    for name, t in (("seq_slot", seq_slot), ("block_table", block_table), ("context_lens", context_lens)):
        _need(t, torch.int32, name)
    batch = q.shape[0]
    if out is None:
        out = torch.empty((batch, cache.hq, HEAD_DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out")
    if ws is None:
        ws = workspace(cache, batch)
    _check(lib().okv_decode_attention(ctypes.byref(cache.desc), _ptr(q), batch, _ptr(seq_slot), _ptr(block_table),
                                      _ptr(context_lens), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def decode_step(cache: Cache, k, v, new_seq_slot, new_pos, slot_lens, q, seq_slot, block_table, context_lens,
                out=None, ws=None, stream=None):
    """Append this step's bf16 tokens, then decode (one call; see okv_decode_step)."""
    import torch
    _need(k, torch.bfloat16, "k"), _need(v, torch.bfloat16, "v"), _need(q, torch.bfloat16, "q")
    for name, t in (("new_seq_slot", new_seq_slot), ("new_pos", new_pos), ("slot_lens", slot_lens),
                    ("seq_slot", seq_slot), ("block_table", block_table), ("context_lens", context_lens)):
        _need(t, torch.int32, name)
    B = q.shape[0]
    T = k.shape[0]
    if out is None:
        out = torch.empty((B, cache.hq, HEAD_DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out")
    if ws is None:
        ws = workspace(cache, B)
    _check(lib().okv_decode_step(ctypes.byref(cache.desc), _ptr(k), _ptr(v), T, _ptr(new_seq_slot), _ptr(new_pos),
                                 _ptr(slot_lens), _ptr(q), B, _ptr(seq_slot), _ptr(block_table), _ptr(context_lens),
                                 _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


class DecodeStepCall:
    """okv_decode_step prepared once for fixed buffers: the arguments are
    checked and marshalled here, and each call only invokes the library, for
    serving loops that refill the same input tensors every step.  The tensors
    must stay alive, and their shapes, for as long as the object is used.

    graph=True: the first call runs eagerly and then records the step's three
    launches in a CUDA graph; later calls replay it (one launch per step)."""

    def __init__(self, cache: Cache, k, v, new_seq_slot, new_pos, slot_lens, q, seq_slot, block_table,
                 context_lens, out=None, ws=None, stream=None, graph: bool = False):
        import torch
        _need(k, torch.bfloat16, "k"), _need(v, torch.bfloat16, "v"), _need(q, torch.bfloat16, "q")
        for name, t in (("new_seq_slot", new_seq_slot), ("new_pos", new_pos), ("slot_lens", slot_lens),
                        ("seq_slot", seq_slot), ("block_table", block_table), ("context_lens", context_lens)):
            _need(t, torch.int32, name)
        B = q.shape[0]
        if out is None:
            out = torch.empty((B, cache.hq, HEAD_DIM), dtype=torch.float32, device=q.device)
        _need(out, torch.float32, "out")
        if ws is None:
            ws = workspace(cache, B)
        self.out, self._keep = out, (cache, k, v, new_seq_slot, new_pos, slot_lens, q, seq_slot, block_table,
                                      context_lens, ws)
        self._fn = lib().okv_decode_step
        self._stream = stream
        self._args = (ctypes.byref(cache.desc), _ptr(k), _ptr(v), k.shape[0], _ptr(new_seq_slot), _ptr(new_pos),
                      _ptr(slot_lens), _ptr(q), B, _ptr(seq_slot), _ptr(block_table), _ptr(context_lens), _ptr(out),
                      _ptr(ws), ws.numel())
        self._want_graph, self._graph = graph, None

    def __call__(self):
        import torch
        if self._graph is not None:
            if self._stream is None:
                self._graph.replay()
            else:
                with torch.cuda.stream(self._stream):
                    self._graph.replay()
            return self.out
        status = self._fn(*self._args, _stream(self._stream))
        if status != OK:
            _check(status)
        if self._want_graph:
            # record the same call (the library allocates nothing and only launches)
            cap = torch.cuda.Stream()
            cap.wait_stream(torch.cuda.current_stream() if self._stream is None else self._stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                status = self._fn(*self._args, cap.cuda_stream)
            _check(status)
            self._graph = g
        return self.out


def decode_attention_noalloc(cache: Cache, q, seq_slot, block_table, context_lens, out=None, stream=None):
    """Decode attention with the library's static scratch (no workspace, no allocation in the library)."""
    import torch
    _need(q, torch.bfloat16, "q")
    for name, t in (("seq_slot", seq_slot), ("block_table", block_table), ("context_lens", context_lens)):
        _need(t, torch.int32, name)
    batch = q.shape[0]
    if out is None:
        out = torch.empty((batch, cache.hq, HEAD_DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out")
    _check(lib().okv_decode_attention_noalloc(ctypes.byref(cache.desc), _ptr(q), batch, _ptr(seq_slot),
                                              _ptr(block_table), _ptr(context_lens), _ptr(out), _stream(stream)))
    return out


def prefill_workspace_bytes(cache: Cache, T: int) -> int:
    return int(lib().okv_prefill_workspace_bytes(ctypes.byref(cache.desc), T))


def prefill_attention(cache: Cache, q, slot: int, context_len: int, block_table, out=None, ws=None, stream=None):
    """Causal attention of a prefill chunk (q: bf16 [T, Hq, 128], already appended at positions
    context_len - T .. context_len - 1 of sequence `slot`) over the cache; returns fp32 [T, Hq, 128]."""
    import torch
    _need(q, torch.bfloat16, "q")
    _need(block_table, torch.int32, "block_table")
    T = q.shape[0]
    if out is None:
        out = torch.empty((T, cache.hq, HEAD_DIM), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, "out")
    if ws is None:
        ws = torch.empty(max(prefill_workspace_bytes(cache, T), 256), dtype=torch.uint8, device=q.device)
    _check(lib().okv_prefill_attention(ctypes.byref(cache.desc), _ptr(q), T, int(slot), int(context_len),
                                       _ptr(block_table), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def time_next_decode_kernel(start_event, stop_event):
    """Record two torch.cuda.Event objects around the next decode call's split-K kernel."""
    for e in (start_event, stop_event):
        if not e.cuda_event:  # torch creates the CUDA event lazily, on first record
            e.record()
    _check(lib().okv_time_next_decode_kernel(start_event.cuda_event, stop_event.cuda_event))


def dequantize(cache: Cache, seq_slot, block_table, context_lens, max_ctx: int, which: int, basis: int = 0,
               source: int = 0, out=None, stream=None):
    import torch
    for name, t in (("seq_slot", seq_slot), ("block_table", block_table), ("context_lens", context_lens)):
        _need(t, torch.int32, name)
    batch = seq_slot.shape[0]
    if out is None:
        out = torch.empty((batch, cache.hkv, max_ctx, HEAD_DIM), dtype=torch.float32, device="cuda")
    _need(out, torch.float32, "out")
    _check(lib().okv_dequantize(ctypes.byref(cache.desc), batch, _ptr(seq_slot), _ptr(block_table),
                                _ptr(context_lens), max_ctx, which, basis, source, _ptr(out), _stream(stream)))
    return out
