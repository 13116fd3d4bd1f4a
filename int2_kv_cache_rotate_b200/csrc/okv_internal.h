// Host-side declarations shared by the library's translation units.
#pragma once

#include <atomic>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "okv.h"

namespace okv {

void set_last_error(const char* fmt, ...);
okv_status fail(okv_status s, const char* fmt, ...);
okv_status check_launch(const char* what);
okv_status validate_desc(const okv_cache_desc* d);
int device_sm_count();

// Sets a kernel's dynamic shared-memory limit once per device (bit d of
// `done` records device d < 32; higher ordinals set it on every call).  The
// attribute belongs to the device's context, so a context reset would need
// it set again: the library assumes contexts live as long as the process.
cudaError_t set_smem_limit_once(const void* kernel, int bytes, std::atomic<uint32_t>& done);
// Launch with programmatic stream serialisation when `early` is set: the
// kernel may begin while its predecessor on the stream is still running (it
// calls grid_dep_wait() before reading the predecessor's outputs).
template <typename... Args>
static cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              bool early, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = early ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
// events set by okv_time_next_decode_kernel (consumed by the next decode launch)
void take_decode_events(cudaEvent_t* start, cudaEvent_t* stop);

// decode workspace layout (bytes, from the workspace base)
struct DecodePlan {
  int batch = 0;
  int hq = 0, hkv = 0, g = 0;
  int num_ctas = 0;         // split-K CTAs
  int num_units = 0;        // batch * hkv
  size_t qrot_off = 0;      // fp32 [B][Hq][128] rotated queries
  size_t qlimb_off = 0;     // int8 [B][Hq][2][128] query limbs (MMA order)
  size_t qscale_off = 0;    // fp32 [B][Hq][kQsStride] (score scale, min term, sigma, sum, group min terms)
  size_t qwin_off = 0;      // fp16 [B][Hq][2][128] scaled query hi/lo halves (window MMA)
  size_t prefix_off = 0;    // int32 [B+1] cost prefix over batch entries
  size_t part_off = 0;      // fp32 [(num_ctas + batch)][Hq][kPartStride]
  size_t total = 0;
};
constexpr int kPartStride = 132;  // o'[128], m, l, 2 spare
constexpr int kQsStride = 8;      // floats per query head in the query-scale workspace
constexpr int kWinCost = 4;       // cost of one 16-row fp16 chunk in block units (all heads)
constexpr int kFusedAppendMaxTokens = 127;  // okv_decode_step fuses appends this short with the query rotation
// split-K kernel choice and residency (decode.cu)
bool decode_uses_tensor_cores(int g, int hkv, int ng);
int decode_ranges(int sms, int g, int hkv, int ng);

DecodePlan make_decode_plan(int batch, int hq, int hkv, int ng);

// bytes of one (KV head, K|V) staged R in the cache's image buffer: three bf16
// parts x 128 x 128
constexpr size_t kRImageBytesPerHead = 3 * 128 * 128 * 2;

// launchers (return cudaGetLastError-mapped status)
okv_status launch_r_image(const okv_cache_desc* d, cudaStream_t s);
okv_status launch_append(const okv_cache_desc* d, const void* k, const void* v, int T,
                         const int32_t* seq_slot, const int32_t* pos, const int32_t* block_table,
                         const int32_t* slot_lens, uint32_t flags, float* rotated_out,
                         cudaStream_t s);
okv_status launch_decode(const okv_cache_desc* d, const void* q, int B, const int32_t* seq_slot,
                         const int32_t* block_table, const int32_t* context_lens, float* out,
                         void* ws, const DecodePlan& plan, cudaStream_t s);
okv_status launch_decode_step(const okv_cache_desc* d, const void* k, const void* v, int T, const int32_t* new_slot,
                              const int32_t* new_pos, const int32_t* slot_lens, const void* q, int B,
                              const int32_t* seq_slot, const int32_t* block_table, const int32_t* context_lens,
                              float* out, void* ws, const DecodePlan& plan, cudaStream_t s);
okv_status launch_prefill(const okv_cache_desc* d, const void* q, int T, int slot, int context_len,
                          const int32_t* block_table, float* out, void* ws, cudaStream_t s);
size_t prefill_workspace_bytes(int T, int hq);
okv_status launch_dequant(const okv_cache_desc* d, int B, const int32_t* seq_slot,
                          const int32_t* block_table, const int32_t* context_lens, int max_ctx,
                          int which, int basis, int source, float* out, cudaStream_t s);

}  // namespace okv
