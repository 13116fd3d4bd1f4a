// C ABI entry points: argument validation, workspace planning, launches.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {

static thread_local char g_last_error[512] = "";
static thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;

void take_decode_events(cudaEvent_t* start, cudaEvent_t* stop) {
  *start = g_ev_start;
  *stop = g_ev_stop;
  g_ev_start = g_ev_stop = nullptr;
}

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

okv_status fail(okv_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

okv_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return OKV_OK;
}

int device_sm_count() {
  static std::atomic<int> cached[32];  // per device ordinal; 0 = not read yet
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 32 && (sms = cached[dev].load(std::memory_order_relaxed)) > 0) return sms;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 32) cached[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

cudaError_t set_smem_limit_once(const void* kernel, int bytes, std::atomic<uint32_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint32_t bit = (dev >= 0 && dev < 32) ? (1u << dev) : 0u;
  if (bit != 0u && (done.load(std::memory_order_acquire) & bit) != 0u) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0u) done.fetch_or(bit, std::memory_order_release);
  return e;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

okv_status validate_desc(const okv_cache_desc* d) {
  if (d == nullptr) return fail(OKV_ERR_INVALID_ARG, "desc is NULL");
  if (d->head_dim != kD || d->block_tokens != kBlock || d->window != kWin ||
      (d->group != 32 && d->group != 64 && d->group != 128))
    return fail(OKV_ERR_UNSUPPORTED, "only head_dim=128, group in {32, 64, 128}, block_tokens=16, window=128 "
                "are built (got %d, %d, %d, %d)", d->head_dim, d->group, d->block_tokens, d->window);
  if (d->num_kv_heads < 1 || d->num_q_heads < 1 || d->num_q_heads % d->num_kv_heads != 0)
    return fail(OKV_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                d->num_q_heads, d->num_kv_heads);
  if (d->num_kv_heads > 65535 || d->num_q_heads > 65535)
    return fail(OKV_ERR_INVALID_ARG, "too many heads");
  if (d->num_blocks < 0 || d->num_seq_slots < 1 || d->max_blocks_per_seq < 1)
    return fail(OKV_ERR_INVALID_ARG, "num_blocks >= 0, num_seq_slots >= 1, max_blocks_per_seq >= 1 required");
  if (d->pages == nullptr && d->num_blocks > 0) return fail(OKV_ERR_INVALID_ARG, "pages is NULL");
  if (d->window_ring == nullptr) return fail(OKV_ERR_INVALID_ARG, "window_ring is NULL");
  if (d->u_k == nullptr || d->u_v == nullptr) return fail(OKV_ERR_INVALID_ARG, "u_k/u_v is NULL");
  if (!aligned(d->r_image, 16)) return fail(OKV_ERR_INVALID_ARG, "r_image must be 16-byte aligned (or NULL)");
  if (!aligned(d->pages, 16) || !aligned(d->window_ring, 16) || !aligned(d->u_k, 16) || !aligned(d->u_v, 16))
    return fail(OKV_ERR_INVALID_ARG, "pages, window_ring, u_k and u_v must be 16-byte aligned");
  if ((long long)d->max_blocks_per_seq * kBlock > 0x3fffffffLL)
    return fail(OKV_ERR_INVALID_ARG, "max_blocks_per_seq too large");
  if (d->num_sink < 0 || d->num_sink > OKV_MAX_SINK || d->num_sink % kBlock != 0)
    return fail(OKV_ERR_UNSUPPORTED, "num_sink must be a multiple of %d in [0, %d] (got %d)", kBlock, OKV_MAX_SINK,
                d->num_sink);
  if (d->num_sink > 0 && (d->sink_rows == nullptr || !aligned(d->sink_rows, 16)))
    return fail(OKV_ERR_INVALID_ARG, "sink_rows must be a 16-byte aligned device buffer when num_sink > 0");
  return OKV_OK;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

DecodePlan make_decode_plan(int batch, int hq, int hkv, int ng) {
  DecodePlan p;
  p.batch = batch;
  p.hq = hq;
  p.hkv = hkv;
  p.g = hq / hkv;
  const int sms = device_sm_count();
  p.num_ctas = decode_ranges(sms > 0 ? sms : 148, p.g, hkv, ng);
  if (p.num_ctas > 1024) p.num_ctas = 1024;  // the combine caches one weight per split
  p.num_units = batch * hkv;
  size_t off = 0;
  p.qrot_off = off;
  off = align_up(off + (size_t)batch * hq * kD * sizeof(float), 256);
  p.qlimb_off = off;
  off = align_up(off + (size_t)batch * hq * 2 * kD, 256);
  p.qscale_off = off;
  off = align_up(off + (size_t)batch * hq * kQsStride * sizeof(float), 256);
  p.qwin_off = off;
  off = align_up(off + (size_t)batch * hq * 2 * kD * 2, 256);
  p.prefix_off = off;
  off = align_up(off + (size_t)(batch + 1) * sizeof(int32_t), 256);
  p.part_off = off;
  off = align_up(off + (size_t)(p.num_ctas + batch) * hq * kPartStride * sizeof(float), 256);
  p.total = off;
  return p;
}

}  // namespace okv

using namespace okv;

extern "C" {

int32_t okv_version(void) { return 3; }

okv_status okv_time_next_decode_kernel(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr))
    return fail(OKV_ERR_INVALID_ARG, "pass two events or two NULLs");
  g_ev_start = (cudaEvent_t)start_event;
  g_ev_stop = (cudaEvent_t)stop_event;
  return OKV_OK;
}

const char* okv_last_error_string(void) { return g_last_error; }

const char* okv_status_string(okv_status s) {
  switch (s) {
    case OKV_OK: return "OKV_OK";
    case OKV_ERR_INVALID_ARG: return "OKV_ERR_INVALID_ARG";
    case OKV_ERR_UNSUPPORTED: return "OKV_ERR_UNSUPPORTED";
    case OKV_ERR_CUDA: return "OKV_ERR_CUDA";
    case OKV_ERR_NUMERIC: return "OKV_ERR_NUMERIC";
    case OKV_ERR_IO: return "OKV_ERR_IO";
  }
  return "unknown okv_status";
}

size_t okv_block_head_bytes(int32_t group) {
  if (group != 32 && group != 64 && group != 128) return 0;
  return (size_t)block_head_bytes(kD / group);
}

size_t okv_pages_bytes(int32_t num_blocks, int32_t num_kv_heads, int32_t group) {
  if (num_blocks < 0 || num_kv_heads < 0) return 0;
  return (size_t)num_blocks * (size_t)num_kv_heads * okv_block_head_bytes(group);
}

size_t okv_r_image_bytes(int32_t num_kv_heads) {
  if (num_kv_heads < 0) return 0;
  return (size_t)num_kv_heads * 2 * kRImageBytesPerHead;
}

okv_status okv_build_r_image(const okv_cache_desc* desc, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (desc->r_image == nullptr) return fail(OKV_ERR_INVALID_ARG, "r_image is NULL");
  return launch_r_image(desc, (cudaStream_t)stream);
}

size_t okv_window_bytes(int32_t num_seq_slots, int32_t num_kv_heads) {
  if (num_seq_slots < 0 || num_kv_heads < 0) return 0;
  return (size_t)num_seq_slots * num_kv_heads * 2 * kWin * kD * sizeof(__half);
}

size_t okv_sink_bytes(int32_t num_seq_slots, int32_t num_kv_heads, int32_t num_sink) {
  if (num_seq_slots < 0 || num_kv_heads < 0 || num_sink < 0) return 0;
  return (size_t)num_seq_slots * num_kv_heads * 2 * num_sink * kD * sizeof(__half);
}

okv_status okv_append_quantize(const okv_cache_desc* desc, const void* k, const void* v, int32_t T,
                               const int32_t* seq_slot, const int32_t* pos,
                               const int32_t* block_table, const int32_t* slot_lens,
                               uint32_t flags, float* rotated_out, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (T < 0) return fail(OKV_ERR_INVALID_ARG, "T must be >= 0");
  if (flags & ~OKV_PRE_ROTATED) return fail(OKV_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (T == 0) return OKV_OK;
  if (!k || !v || !seq_slot || !pos || !block_table || !slot_lens)
    return fail(OKV_ERR_INVALID_ARG, "k, v, seq_slot, pos, block_table and slot_lens must be non-NULL");
  if (desc->num_blocks == 0) return fail(OKV_ERR_INVALID_ARG, "cache has no blocks");
  const size_t al = (flags & OKV_PRE_ROTATED) ? 16 : 2;
  if ((uintptr_t)k % al || (uintptr_t)v % al)
    return fail(OKV_ERR_INVALID_ARG, "k and v must be %zu-byte aligned", al);
  if (rotated_out && (uintptr_t)rotated_out % 16)
    return fail(OKV_ERR_INVALID_ARG, "rotated_out must be 16-byte aligned");
  return launch_append(desc, k, v, T, seq_slot, pos, block_table, slot_lens, flags, rotated_out,
                       (cudaStream_t)stream);
}

size_t okv_prefill_workspace_bytes(const okv_cache_desc* desc, int32_t T) {
  if (validate_desc(desc) != OKV_OK || T < 0) return 0;
  return prefill_workspace_bytes(T, desc->num_q_heads);
}

okv_status okv_prefill_attention(const okv_cache_desc* desc, const void* q, int32_t T, int32_t slot,
                                 int32_t context_len, const int32_t* block_table, float* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (T < 0) return fail(OKV_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return OKV_OK;
  if (!q || !block_table || !out || !workspace)
    return fail(OKV_ERR_INVALID_ARG, "q, block_table, out and workspace must be non-NULL");
  if (slot < 0 || slot >= desc->num_seq_slots)
    return fail(OKV_ERR_INVALID_ARG, "slot %d outside [0, %d)", slot, desc->num_seq_slots);
  if (context_len < T || (long long)context_len > (long long)desc->max_blocks_per_seq * kBlock)
    return fail(OKV_ERR_INVALID_ARG, "context_len %d must be in [T = %d, %lld]", context_len, T,
                (long long)desc->max_blocks_per_seq * kBlock);
  if ((long long)T * desc->num_q_heads > 0x7fffffffLL) return fail(OKV_ERR_INVALID_ARG, "T * Hq too large");
  if ((uintptr_t)q % 2 || (uintptr_t)out % 4 || (uintptr_t)workspace % 256)
    return fail(OKV_ERR_INVALID_ARG, "q must be 2-byte, out 4-byte and workspace 256-byte aligned");
  const size_t need = prefill_workspace_bytes(T, desc->num_q_heads);
  if (workspace_bytes < need)
    return fail(OKV_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  return launch_prefill(desc, q, T, slot, context_len, block_table, out, workspace, (cudaStream_t)stream);
}

size_t okv_decode_workspace_bytes(const okv_cache_desc* desc, int32_t B) {
  if (validate_desc(desc) != OKV_OK || B < 0) return 0;
  return make_decode_plan(B, desc->num_q_heads, desc->num_kv_heads, kD / desc->group).total;
}

okv_status okv_decode_attention(const okv_cache_desc* desc, const void* q, int32_t B,
                                const int32_t* seq_slot, const int32_t* block_table,
                                const int32_t* context_lens, float* out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (B < 0) return fail(OKV_ERR_INVALID_ARG, "B must be >= 0");
  if (B == 0) return OKV_OK;
  if (!q || !seq_slot || !block_table || !context_lens || !out || !workspace)
    return fail(OKV_ERR_INVALID_ARG, "q, seq_slot, block_table, context_lens, out and workspace must be non-NULL");
  const int g = desc->num_q_heads / desc->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16)
    return fail(OKV_ERR_UNSUPPORTED, "Hq/Hkv = %d not in {1,2,4,8,16}", g);
  if ((long long)B * desc->num_kv_heads * ((long long)desc->max_blocks_per_seq + kWinCost) >= 0x7fffffffLL)
    return fail(OKV_ERR_INVALID_ARG, "B * Hkv * max_blocks_per_seq too large");
  if ((uintptr_t)workspace % 256) return fail(OKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const DecodePlan plan = make_decode_plan(B, desc->num_q_heads, desc->num_kv_heads, kD / desc->group);
  if (workspace_bytes < plan.total)
    return fail(OKV_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, plan.total);
  return launch_decode(desc, q, B, seq_slot, block_table, context_lens, out, workspace, plan,
                       (cudaStream_t)stream);
}

okv_status okv_decode_step(const okv_cache_desc* desc, const void* k, const void* v, int32_t T,
                           const int32_t* new_seq_slot, const int32_t* new_pos, const int32_t* slot_lens,
                           const void* q, int32_t B, const int32_t* seq_slot, const int32_t* block_table,
                           const int32_t* context_lens, float* out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (T < 0 || B < 0) return fail(OKV_ERR_INVALID_ARG, "T and B must be >= 0");
  if (B == 0)
    return okv_append_quantize(desc, k, v, T, new_seq_slot, new_pos, block_table, slot_lens, 0, nullptr, stream);
  if (T > 0) {
    if (!k || !v || !new_seq_slot || !new_pos || !slot_lens)
      return fail(OKV_ERR_INVALID_ARG, "k, v, new_seq_slot, new_pos and slot_lens must be non-NULL");
    if (desc->num_blocks == 0) return fail(OKV_ERR_INVALID_ARG, "cache has no blocks");
    if ((uintptr_t)k % 2 || (uintptr_t)v % 2) return fail(OKV_ERR_INVALID_ARG, "k and v must be 2-byte aligned");
  }
  if (!q || !seq_slot || !block_table || !context_lens || !out || !workspace)
    return fail(OKV_ERR_INVALID_ARG, "q, seq_slot, block_table, context_lens, out and workspace must be non-NULL");
  const int g = desc->num_q_heads / desc->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16)
    return fail(OKV_ERR_UNSUPPORTED, "Hq/Hkv = %d not in {1,2,4,8,16}", g);
  if ((long long)B * desc->num_kv_heads * ((long long)desc->max_blocks_per_seq + kWinCost) >= 0x7fffffffLL)
    return fail(OKV_ERR_INVALID_ARG, "B * Hkv * max_blocks_per_seq too large");
  if ((uintptr_t)workspace % 256) return fail(OKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const DecodePlan plan = make_decode_plan(B, desc->num_q_heads, desc->num_kv_heads, kD / desc->group);
  if (workspace_bytes < plan.total)
    return fail(OKV_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, plan.total);
  const cudaStream_t s = (cudaStream_t)stream;
  if (T > kFusedAppendMaxTokens) {  // a prefill chunk: its own (tensor-core) launch, then the decode
    st = launch_append(desc, k, v, T, new_seq_slot, new_pos, block_table, slot_lens, 0, nullptr, s);
    if (st != OKV_OK) return st;
    return launch_decode(desc, q, B, seq_slot, block_table, context_lens, out, workspace, plan, s);
  }
  return launch_decode_step(desc, k, v, T, new_seq_slot, new_pos, slot_lens, q, B, seq_slot, block_table,
                            context_lens, out, workspace, plan, s);
}

okv_status okv_dequantize(const okv_cache_desc* desc, int32_t B, const int32_t* seq_slot,
                          const int32_t* block_table, const int32_t* context_lens,
                          int32_t max_ctx, int32_t which, int32_t basis, int32_t source,
                          float* out, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (B < 0 || max_ctx < 0) return fail(OKV_ERR_INVALID_ARG, "B and max_ctx must be >= 0");
  if ((which != 0 && which != 1) || (basis != 0 && basis != 1) || (source != 0 && source != 1))
    return fail(OKV_ERR_INVALID_ARG, "which, basis and source must each be 0 or 1");
  if (B == 0 || max_ctx == 0) return OKV_OK;
  if (!seq_slot || !block_table || !context_lens || !out)
    return fail(OKV_ERR_INVALID_ARG, "seq_slot, block_table, context_lens and out must be non-NULL");
  if ((uintptr_t)out % 16) return fail(OKV_ERR_INVALID_ARG, "out must be 16-byte aligned");
  if (B > 65535) return fail(OKV_ERR_INVALID_ARG, "B > 65535");
  return launch_dequant(desc, B, seq_slot, block_table, context_lens, max_ctx, which, basis, source, out,
                        (cudaStream_t)stream);
}

}  // extern "C"
