// Gather/dequantise: block-table gather of the cache into dense fp32, in the
// rotated basis or brought back to the original one.
#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {
namespace {

constexpr int kUPadDq = 129;
constexpr int kTokPerCta = 32;

struct DequantArgs {
  const int32_t* seq_slot;
  const int32_t* block_table;
  const int32_t* context_lens;
  const uint8_t* pages;
  const __half* ring;
  const __half* sink;  // fp16 rows of the first nsink positions
  const float* u;  // U of `which`
  float* out;
  uint32_t* status;
  int hkv, num_blocks, num_slots, mbps, max_ctx, which, basis, source, nsink;
  int ng;  // quantisation groups per vector
};

// grid (ceil(max_ctx/32), Hkv, B), 128 threads; warp w handles tokens w, w+4, ...
// of the CTA's 32-token span; lane l produces rotated channels 4l..4l+3.
__global__ void __launch_bounds__(128) dequant_kernel(DequantArgs a) {
  extern __shared__ float us_[];  // U [128][129] when basis == 1
  const int hk = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (a.basis == 1) {
    const float* u = a.u + (size_t)hk * kD * kD;
    for (int i = threadIdx.x; i < kD * kD; i += blockDim.x) us_[(i / kD) * kUPadDq + (i % kD)] = u[i];
    __syncthreads();
  }
  int len = a.context_lens[b];
  if (len < 0 || len > a.mbps * kBlock) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && hk == 0) raise_flag(a.status, OKV_DEV_BAD_POS);
    len = len < 0 ? 0 : a.mbps * kBlock;
  }
  const int slot = a.seq_slot[b];
  const bool slot_ok = slot >= 0 && slot < a.num_slots;
  if (!slot_ok && threadIdx.x == 0 && blockIdx.x == 0 && hk == 0) raise_flag(a.status, OKV_DEV_BAD_SLOT);
  const int first_fp16 = (a.source == 1) ? max(0, len - kWin) : len;
  for (int i = warp; i < kTokPerCta; i += 4) {
    const int p = blockIdx.x * kTokPerCta + i;
    if (p >= a.max_ctx) break;
    float z[4] = {0.f, 0.f, 0.f, 0.f};
    bool have = false;
    if (p < len && slot_ok) {
      if (p >= first_fp16 || (a.source == 1 && p < a.nsink)) {
        const __half* row =
            p < a.nsink && a.source == 1
                ? a.sink + ((((size_t)slot * a.hkv + hk) * 2 + a.which) * a.nsink + p) * kD
                : a.ring + ((((size_t)slot * a.hkv + hk) * 2 + a.which) * kWin + (p % kWin)) * kD;
        const uint2 w = *reinterpret_cast<const uint2*>(row + 4 * lane);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
        z[0] = f0.x; z[1] = f0.y; z[2] = f1.x; z[3] = f1.y;
        have = true;
      } else {
        const int blk = a.block_table[(size_t)slot * a.mbps + (p >> 4)];
        if (blk >= 0 && blk < a.num_blocks) {
          const uint8_t* bp = a.pages + ((size_t)blk * a.hkv + hk) * block_head_bytes(a.ng);
          const int t = p & 15;
          const uint32_t byte = a.which == 0 ? bp[kKcOff + t * 32 + lane] : bp[v_code_offset(t, lane)];
          // channels 4 lane .. 4 lane + 3 lie in group 4 lane / group = lane ng / 32
          const uint32_t sm =
              *reinterpret_cast<const uint32_t*>(bp + sm_offset(a.ng, a.which, t, lane * a.ng / 32));
          const float s = __half2float(__ushort_as_half((unsigned short)(sm & 0xffff)));
          const float m = __half2float(__ushort_as_half((unsigned short)(sm >> 16)));
#pragma unroll
          for (int j = 0; j < 4; ++j) z[j] = fmaf(s, (float)((byte >> (2 * j)) & 3u), m);
          have = true;
        } else if (lane == 0) {
          raise_flag(a.status, OKV_DEV_BAD_BLOCK);
        }
      }
    }
    float* dst = a.out + (((size_t)b * a.hkv + hk) * a.max_ctx + p) * kD;
    if (a.basis == 0 || !have) {
      *reinterpret_cast<float4*>(dst + 4 * lane) = make_float4(z[0], z[1], z[2], z[3]);
      continue;
    }
    // back to the original basis: y_i = z_br(i), x = y H, out_c = sum_i x_i U[c][i]
    const int r = rev5(lane);
    float y[4];
    y[0] = __shfl_sync(0xffffffffu, z[0], r);
    y[1] = __shfl_sync(0xffffffffu, z[2], r);
    y[2] = __shfl_sync(0xffffffffu, z[1], r);
    y[3] = __shfl_sync(0xffffffffu, z[3], r);
    wht128_warp(y, lane);
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < kD; ++i) {
      const float xi = __shfl_sync(0xffffffffu, y[i >> 5], i & 31) * kInvSqrtD;
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = fmaf(xi, us_[(lane + 32 * j) * kUPadDq + i], o[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[lane + 32 * j] = o[j];
  }
}

}  // namespace

okv_status launch_dequant(const okv_cache_desc* d, int B, const int32_t* seq_slot,
                          const int32_t* block_table, const int32_t* context_lens, int max_ctx,
                          int which, int basis, int source, float* out, cudaStream_t s) {
  DequantArgs a;
  a.seq_slot = seq_slot;
  a.block_table = block_table;
  a.context_lens = context_lens;
  a.pages = (const uint8_t*)d->pages;
  a.ring = (const __half*)d->window_ring;
  a.sink = (const __half*)d->sink_rows;
  a.nsink = d->num_sink;
  a.u = which ? d->u_v : d->u_k;
  a.out = out;
  a.status = d->status_word;
  a.hkv = d->num_kv_heads;
  a.num_blocks = d->num_blocks;
  a.num_slots = d->num_seq_slots;
  a.mbps = d->max_blocks_per_seq;
  a.ng = kD / d->group;
  a.max_ctx = max_ctx;
  a.which = which;
  a.basis = basis;
  a.source = source;
  const size_t smem = basis == 1 ? (size_t)kD * kUPadDq * sizeof(float) : 0;
  if (smem > 0) {
    cudaError_t e = cudaFuncSetAttribute(dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "dequant smem attribute: %s", cudaGetErrorString(e));
  }
  dim3 grid((max_ctx + kTokPerCta - 1) / kTokPerCta, d->num_kv_heads, B);
  dequant_kernel<<<grid, 128, smem, s>>>(a);
  return check_launch("dequantize");
}

}  // namespace okv
