// Decode attention for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: a plugin that is
// given only the tensors it works on by an engine that owns every byte of
// device memory, or code that must not call cudaMalloc because that call can
// synchronise the whole device and stall the engine's other streams.  This
// entry point runs the same three kernels as okv_decode_attention, but its
// scratch (rotated queries, cost prefix, split-K partials) lives in one
// file-scope device array that every GPU loading the library keeps until the
// process exits.  Nothing here allocates.
#include <mutex>

#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[OKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device, with that device current.
okv_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(OKV_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(OKV_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return OKV_OK;
}

}  // namespace
}  // namespace okv

using namespace okv;

extern "C" okv_status okv_decode_attention_noalloc(const okv_cache_desc* desc, const void* q, int32_t B,
                                                   const int32_t* seq_slot, const int32_t* block_table,
                                                   const int32_t* context_lens, float* out, void* stream) {
  okv_status st = validate_desc(desc);
  if (st != OKV_OK) return st;
  if (B < 0) return fail(OKV_ERR_INVALID_ARG, "B must be >= 0");
  if (B == 0) return OKV_OK;
  if (!q || !seq_slot || !block_table || !context_lens || !out)
    return fail(OKV_ERR_INVALID_ARG, "q, seq_slot, block_table, context_lens and out must be non-NULL");
  const int g = desc->num_q_heads / desc->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16)
    return fail(OKV_ERR_UNSUPPORTED, "Hq/Hkv = %d not in {1,2,4,8,16}", g);
  if ((long long)B * desc->num_kv_heads * ((long long)desc->max_blocks_per_seq + kWinCost) >= 0x7fffffffLL)
    return fail(OKV_ERR_INVALID_ARG, "B * Hkv * max_blocks_per_seq too large");
  const DecodePlan plan = make_decode_plan(B, desc->num_q_heads, desc->num_kv_heads, kD / desc->group);
  if (plan.total > (size_t)OKV_NOALLOC_SCRATCH_BYTES)
    return fail(OKV_ERR_INVALID_ARG,
                "batch too large for the built-in scratch: needs %zu bytes, the static array holds %zu "
                "(use okv_decode_attention with a caller workspace)",
                plan.total, (size_t)OKV_NOALLOC_SCRATCH_BYTES);
  void* ws = nullptr;
  st = scratch_address(&ws);
  if (st != OKV_OK) return st;
  // Every slot the kernels read is written earlier in the same call, so the
  // previous call's contents need no clearing.
  return launch_decode(desc, q, B, seq_slot, block_table, context_lens, out, ws, plan, (cudaStream_t)stream);
}
