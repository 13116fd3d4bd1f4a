// Warp-level append shared by the append kernels and the fused decode-step
// kernel: rotate (U, Hadamard butterfly, bit-reversal remap), quantise to INT2
// with fp16 scale/min, pack, and write the paged cache and the fp16 rows of
// the recent-token window and of the sink tokens, for one 32-token tile of
// one (KV head, K|V).
#pragma once

#include "okv.h"
#include "okv_common.cuh"

namespace okv {

struct AppendArgs {
  const void* k;
  const void* v;
  const int32_t* seq_slot;
  const int32_t* pos;
  const int32_t* block_table;
  const int32_t* slot_lens;
  const float* u_k;
  const float* u_v;
  uint8_t* pages;
  __half* ring;
  __half* sink;  // fp16 rows of the first nsink positions
  float* rotated_out;
  uint32_t* status;
  int hkv, num_blocks, num_slots, mbps, nsink;
  int ng;   // quantisation groups per vector (128 / group)
  int bhb;  // bytes of one block-head
  const uint8_t* r_image;  // staged R of every (KV head, K|V) for the tcgen05 append, or null
};

inline AppendArgs make_append_args(const okv_cache_desc* d, const void* k, const void* v, const int32_t* seq_slot,
                                   const int32_t* pos, const int32_t* block_table, const int32_t* slot_lens,
                                   float* rotated_out) {
  AppendArgs a;
  a.k = k;
  a.v = v;
  a.seq_slot = seq_slot;
  a.pos = pos;
  a.block_table = block_table;
  a.slot_lens = slot_lens;
  a.u_k = d->u_k;
  a.u_v = d->u_v;
  a.pages = (uint8_t*)d->pages;
  a.ring = (__half*)d->window_ring;
  a.sink = (__half*)d->sink_rows;
  a.nsink = d->num_sink;
  a.rotated_out = rotated_out;
  a.status = d->status_word;
  a.hkv = d->num_kv_heads;
  a.num_blocks = d->num_blocks;
  a.num_slots = d->num_seq_slots;
  a.mbps = d->max_blocks_per_seq;
  a.ng = kD / d->group;
  a.bhb = block_head_bytes(a.ng);
  a.r_image = (const uint8_t*)d->r_image;
  return a;
}

// fp16 row of position p of (slot, KV head, K|V) in the recent-token ring
// (for p >= len - kWin) and in the sink rows (for p < nsink); null where the
// position has no such row.
__device__ __forceinline__ __half* window_row(const AppendArgs& a, int slot, int h, int kind, int p, int len) {
  return p >= len - kWin ? a.ring + ((((size_t)slot * a.hkv + h) * 2 + kind) * kWin + (p % kWin)) * kD : nullptr;
}
__device__ __forceinline__ __half* sink_row(const AppendArgs& a, int slot, int h, int kind, int p) {
  return p < a.nsink ? a.sink + ((((size_t)slot * a.hkv + h) * 2 + kind) * a.nsink + p) * kD : nullptr;
}

constexpr int kAppThreads = 256;
constexpr int kAppRound = 8;    // tokens reduced per round (one per warp)
constexpr int kAppTokens = 32;  // tokens per CTA

// Validate token t's destination and write everything for one rotated vector.
// Lane l owns pre-permutation channels l + 32a, which after P_br are rotated
// channels 4*rev5(l) + rev2(a): exactly the four codes of packed byte rev5(l).
// So the permutation costs nothing: it is the choice of which byte a lane writes.
__device__ __forceinline__ void finish_token(const AppendArgs& a, int t, int h, int kind, const float y[4],
                                             int lane) {
  const int slot = a.seq_slot[t];
  const int p = a.pos[t];
  if (slot < 0 || slot >= a.num_slots) {
    if (lane == 0) raise_flag(a.status, OKV_DEV_BAD_SLOT);
    return;
  }
  const int len = a.slot_lens[slot];
  if (p < 0 || (p >> 4) >= a.mbps || p >= len) {
    if (lane == 0) raise_flag(a.status, OKV_DEV_BAD_POS);
    return;
  }
  const int blk = a.block_table[(size_t)slot * a.mbps + (p >> 4)];
  if (blk < 0 || blk >= a.num_blocks) {
    if (lane == 0) raise_flag(a.status, OKV_DEV_BAD_BLOCK);
    return;
  }
  const int r = rev5(lane);
  if (a.rotated_out != nullptr) {
    float4 o = make_float4(y[0], y[2], y[1], y[3]);
    *reinterpret_cast<float4*>(a.rotated_out + (((size_t)t * 2 + kind) * a.hkv + h) * kD + 4 * r) = o;
  }
  const Quantized q = quantize_warp(y, a.ng);
  uint8_t* base = a.pages + ((size_t)blk * a.hkv + h) * a.bhb;
  const int s16 = p & 15;
  if (kind == 0) {
    base[kKcOff + s16 * 32 + r] = (uint8_t)q.byte;
  } else {
    base[v_code_offset(s16, r)] = (uint8_t)q.byte;
  }
  // one lane per group (lanes 0 .. ng - 1) writes its group's scale and min
  if (lane < a.ng) *reinterpret_cast<uint32_t*>(base + sm_offset(a.ng, kind, s16, r * a.ng / 32)) = q.sm;
  __half* wrow = window_row(a, slot, h, kind, p, len);
  __half* srow = sink_row(a, slot, h, kind, p);
  if (wrow != nullptr || srow != nullptr) {
    __half2 lo = __halves2half2(fp16_sat(y[0]), fp16_sat(y[2]));
    __half2 hi = __halves2half2(fp16_sat(y[1]), fp16_sat(y[3]));
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&lo);
    w.y = *reinterpret_cast<uint32_t*>(&hi);
    if (wrow != nullptr) *reinterpret_cast<uint2*>(wrow + 4 * r) = w;
    if (srow != nullptr) *reinterpret_cast<uint2*>(srow + 4 * r) = w;
  }
}

// One CTA per (32-token tile, KV head, K|V), 8 warps.  U stays in registers
// for the whole tile (warp w holds rows 16w..16w+15, lane l columns
// 4l..4l+3: one round of loads); each round multiplies 8 tokens, reduces the
// 8 warps' partial sums through shared memory, and hands token i to warp i
// for the Hadamard butterfly, the bit-reversal remap and the quantiser.
template <bool kPre>
__device__ __forceinline__ void append_tile(const AppendArgs& a, int T, int tile, int h, int kind) {
  __shared__ float red[kPre ? 1 : kAppRound][8][kD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = tile * kAppTokens, t1 = min(T, t0 + kAppTokens);
  float4 u[16];
  if constexpr (!kPre) {
    const float* U = (kind ? a.u_v : a.u_k) + (size_t)h * kD * kD;
#pragma unroll
    for (int r = 0; r < 16; ++r) u[r] = __ldg(reinterpret_cast<const float4*>(U + (size_t)(16 * warp + r) * kD) + lane);
  }
  for (int r0 = t0; r0 < t1; r0 += kAppRound) {
    const int nr = min(kAppRound, t1 - r0);
    float y[4];
    if constexpr (!kPre) {
      const __nv_bfloat16* src = (const __nv_bfloat16*)(kind ? a.v : a.k);
      float xv[kAppRound];
#pragma unroll
      for (int i = 0; i < kAppRound; ++i)
        xv[i] = i < nr ? __bfloat162float(src[((size_t)(r0 + i) * a.hkv + h) * kD + 16 * warp + (lane & 15)]) : 0.f;
#pragma unroll
      for (int i = 0; i < kAppRound; ++i) {
        if (i >= nr) break;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float x = __shfl_sync(0xffffffffu, xv[i], r);
          acc.x = fmaf(x, u[r].x, acc.x);
          acc.y = fmaf(x, u[r].y, acc.y);
          acc.z = fmaf(x, u[r].z, acc.z);
          acc.w = fmaf(x, u[r].w, acc.w);
        }
        *reinterpret_cast<float4*>(&red[i][warp][4 * lane]) = acc;
      }
      __syncthreads();
      if (warp < nr) {
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) {
          float s = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) s += red[warp][w][lane + 32 * aa];
          y[aa] = s;
        }
        wht128_warp(y, lane);
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) y[aa] *= kInvSqrtD;
      }
      __syncthreads();  // red is reused by the next round
    } else {
      if (warp < nr) {
        const float* src = (const float*)(kind ? a.v : a.k) + ((size_t)(r0 + warp) * a.hkv + h) * kD;
        const float4 z4 = *reinterpret_cast<const float4*>(src + 4 * rev5(lane));
        y[0] = z4.x;  // rotated channel 4r+0 <- pre-permutation index l
        y[1] = z4.z;  // 4r+2 <- l+32
        y[2] = z4.y;  // 4r+1 <- l+64
        y[3] = z4.w;  // 4r+3 <- l+96
      }
    }
    if (warp < nr) finish_token(a, r0 + warp, h, kind, y, lane);
  }
}

}  // namespace okv
