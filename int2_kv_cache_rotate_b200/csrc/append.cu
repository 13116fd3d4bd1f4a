// Append kernels: rotate (U, Hadamard butterfly, bit-reversal remap), quantise
// to INT2 with fp16 scale/min, pack, and write the paged cache and fp16 window.
// Decode steps (a few tokens) run the CUDA-core kernel; prefill chunks of 128
// tokens or more run the tensor-core kernel.
#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {
namespace {

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
  float* rotated_out;
  uint32_t* status;
  int hkv, num_blocks, num_slots, mbps;
};

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
  const Quantized q = quantize_warp(y);
  uint8_t* base = a.pages + ((size_t)blk * a.hkv + h) * kBlockHeadBytes;
  const int s16 = p & 15;
  if (kind == 0) {
    base[kKcOff + s16 * 32 + r] = (uint8_t)q.byte;
  } else {
    base[v_code_offset(s16, r)] = (uint8_t)q.byte;
  }
  if (lane == 0) *reinterpret_cast<uint32_t*>(base + (kind ? kVsmOff : kKsmOff) + 4 * s16) = q.sm;
  if (p >= len - kWin) {
    __half* row = a.ring + ((((size_t)slot * a.hkv + h) * 2 + kind) * kWin + (p % kWin)) * kD + 4 * r;
    __half2 lo = __halves2half2(fp16_sat(y[0]), fp16_sat(y[2]));
    __half2 hi = __halves2half2(fp16_sat(y[1]), fp16_sat(y[3]));
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&lo);
    w.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(row) = w;
  }
}

// One CTA per (32-token tile, KV head, K|V), 8 warps.  U stays in registers
// for the whole tile (warp w holds rows 16w..16w+15, lane l columns
// 4l..4l+3: one round of loads); each round multiplies 8 tokens, reduces the
// 8 warps' partial sums through shared memory, and hands token i to warp i
// for the Hadamard butterfly, the bit-reversal remap and the quantiser.
template <bool kPre>
__global__ void __launch_bounds__(kAppThreads) append_kernel(AppendArgs a, int T) {
  __shared__ float red[kPre ? 1 : kAppRound][8][kD];
  const int h = blockIdx.y, kind = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = blockIdx.x * kAppTokens, t1 = min(T, t0 + kAppTokens);
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

// ---------------------------------------------------------------------------
// Tensor-core append for long token runs (prefill chunks).
//
// x = k U is a dense [T x 128] x [128 x 128] contraction, so it runs on
// mma.m16n8k16 (bf16 in, fp32 accumulate): k is exact in bf16 and U is split
// into three bf16 parts (hi + mid + lo carry 24 mantissa bits), so every
// product is exact and the sum is an fp32 sum, like the CUDA-core path.
// A CTA stages U^T (three parts, rows padded to 136 elements so the fragment
// loads do not collide in banks) once and runs 4 warps x 16 tokens per round.
// In the accumulator layout lane (g, t) holds, for tokens g and g+8, outputs
// i = 8 nt + 2t + e (nt = 0..15, e = 0..1): Hadamard index bits 0 and 3..6 are
// in registers, bits 1..2 across the four lanes of a quad (two shuffle
// stages).  Bits 5..6 are register bits too, so after the bit reversal each
// lane owns whole packed bytes: byte b collects outputs rev5(b) + 32a.
// ---------------------------------------------------------------------------
constexpr int kTcMinTokens = 128;  // below this the CUDA-core kernel wins (U staging dominates)
constexpr int kTcWarps = 4;
constexpr int kTcRound = 16 * kTcWarps;   // tokens per round
constexpr int kTcCtaTokens = 256;         // tokens per CTA (U staged once)
constexpr int kUtStride = 136;            // bf16 per U^T row in shared memory
constexpr size_t kTcSmem = (size_t)3 * kD * kUtStride * 2;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One token's rotated vector, spread over the four lanes of a quad:
// zb[q][a] = y at pre-permutation index r_q + 32a, r_q = 8 (q >> 1) + 2t + (q & 1).
// The min/max reduction runs on every lane (the quad shuffles need all of
// them); `live` then gates validation and the stores.
__device__ __forceinline__ void finish_token_tc(const AppendArgs& a, int tok, bool live, int h, int kind,
                                                const float (&zb)[8][4], int t) {
  float mn = zb[0][0], mx = zb[0][0];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      mn = fminf(mn, zb[q][aa]);
      mx = fmaxf(mx, zb[q][aa]);
    }
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  if (!live) return;
  const int slot = a.seq_slot[tok];
  const int p = a.pos[tok];
  if (slot < 0 || slot >= a.num_slots) {
    if (t == 0) raise_flag(a.status, OKV_DEV_BAD_SLOT);
    return;
  }
  const int len = a.slot_lens[slot];
  if (p < 0 || (p >> 4) >= a.mbps || p >= len) {
    if (t == 0) raise_flag(a.status, OKV_DEV_BAD_POS);
    return;
  }
  const int blk = a.block_table[(size_t)slot * a.mbps + (p >> 4)];
  if (blk < 0 || blk >= a.num_blocks) {
    if (t == 0) raise_flag(a.status, OKV_DEV_BAD_BLOCK);
    return;
  }
  // the quantiser's steps, in the same fp32 operations as quantize_warp
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
  const __half s16 = fp16_sat(s32);
  const __half m16 = fp16_sat(mn);
  const float s = __half2float(s16);
  const float m = __half2float(m16);
  uint8_t* base = a.pages + ((size_t)blk * a.hkv + h) * kBlockHeadBytes;
  const int sl = p & 15;
  const bool in_win = p >= len - kWin;
  __half* wrow = a.ring + ((((size_t)slot * a.hkv + h) * 2 + kind) * kWin + (p % kWin)) * kD;
  float* rrow = a.rotated_out ? a.rotated_out + (((size_t)tok * 2 + kind) * a.hkv + h) * kD : nullptr;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int b = rev5(8 * (q >> 1) + 2 * t + (q & 1));  // packed byte = canonical channels 4b..4b+3
    uint32_t byte = 0;
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      uint32_t c = 0;
      if (s != 0.0f) {
        const float rr = rintf(__fdiv_rn(__fsub_rn(zb[q][aa], m), s));
        c = (uint32_t)fminf(fmaxf(rr, 0.0f), 3.0f);
      }
      byte |= c << (2 * rev2(aa));
    }
    if (kind == 0) base[kKcOff + sl * 32 + b] = (uint8_t)byte;
    else base[v_code_offset(sl, b)] = (uint8_t)byte;
    // channel 4b + e holds the value at a = rev2(e): e = 0..3 <- a = 0, 2, 1, 3
    if (in_win) {
      __half2 lo = __halves2half2(fp16_sat(zb[q][0]), fp16_sat(zb[q][2]));
      __half2 hi = __halves2half2(fp16_sat(zb[q][1]), fp16_sat(zb[q][3]));
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(wrow + 4 * b) = w;
    }
    if (rrow) *reinterpret_cast<float4*>(rrow + 4 * b) = make_float4(zb[q][0], zb[q][2], zb[q][1], zb[q][3]);
  }
  if (t == 0)
    *reinterpret_cast<uint32_t*>(base + (kind ? kVsmOff : kKsmOff) + 4 * sl) =
        (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
}

__global__ void __launch_bounds__(kTcWarps * 32) append_tc_kernel(AppendArgs a, int T) {
  extern __shared__ __align__(16) unsigned char tc_smem[];
  __nv_bfloat16* ut = reinterpret_cast<__nv_bfloat16*>(tc_smem);  // [3][128][136]: U^T split in three
  const int h = blockIdx.y, kind = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = blockIdx.x * kTcCtaTokens, t1 = min(T, t0 + kTcCtaTokens);
  {
    // U^T[i][c] = U[c][i], split as U = p0 + p1 + p2 (each bf16, residuals exact in fp32);
    // a thread takes column i of two consecutive rows c, c+1 and stores bf16 pairs.
    const float* U = (kind ? a.u_v : a.u_k) + (size_t)h * kD * kD;
    for (int idx = threadIdx.x; idx < kD * kD / 2; idx += blockDim.x) {
      const int i = idx & (kD - 1), c = 2 * (idx >> 7);
      const float u0 = __ldg(U + (size_t)c * kD + i), u1 = __ldg(U + (size_t)(c + 1) * kD + i);
      const __nv_bfloat162 p0 = __floats2bfloat162_rn(u0, u1);
      const float r0 = u0 - __low2float(p0), r1 = u1 - __high2float(p0);
      const __nv_bfloat162 p1 = __floats2bfloat162_rn(r0, r1);
      const __nv_bfloat162 p2 = __floats2bfloat162_rn(r0 - __low2float(p1), r1 - __high2float(p1));
      *reinterpret_cast<__nv_bfloat162*>(ut + (0 * kD + i) * kUtStride + c) = p0;
      *reinterpret_cast<__nv_bfloat162*>(ut + (1 * kD + i) * kUtStride + c) = p1;
      *reinterpret_cast<__nv_bfloat162*>(ut + (2 * kD + i) * kUtStride + c) = p2;
    }
  }
  __syncthreads();
  const __nv_bfloat16* src = (const __nv_bfloat16*)(kind ? a.v : a.k);
  for (int r0 = t0 + 16 * warp; r0 < t1; r0 += kTcRound) {
    const int ta = r0 + g, tb = r0 + g + 8;
    const bool va = ta < t1, vb = tb < t1;
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(src + ((size_t)(va ? ta : t0) * a.hkv + h) * kD);
    const uint32_t* rb = reinterpret_cast<const uint32_t*>(src + ((size_t)(vb ? tb : t0) * a.hkv + h) * kD);
    uint32_t af[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      af[ks][0] = va ? ra[8 * ks + t] : 0u;
      af[ks][1] = vb ? rb[8 * ks + t] : 0u;
      af[ks][2] = va ? ra[8 * ks + 4 + t] : 0u;
      af[ks][3] = vb ? rb[8 * ks + 4 + t] : 0u;
    }
    float d[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
#pragma unroll
      for (int j = 0; j < 4; ++j) d[nt][j] = 0.f;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const __nv_bfloat16* urow = ut + ((size_t)part * kD + 8 * nt + g) * kUtStride + 2 * t;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(urow + 16 * ks);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(urow + 16 * ks + 8);
          mma_bf16(d[nt], af[ks], b0, b1);
        }
      }
    }
    // Walsh-Hadamard over i = 8 nt + 2t + e, for token g (regs 0,1) and g+8 (regs 2,3)
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {  // bit 0 (e)
      const float x0 = d[nt][0], x1 = d[nt][1], x2 = d[nt][2], x3 = d[nt][3];
      d[nt][0] = __fadd_rn(x0, x1);
      d[nt][1] = __fsub_rn(x0, x1);
      d[nt][2] = __fadd_rn(x2, x3);
      d[nt][3] = __fsub_rn(x2, x3);
    }
#pragma unroll
    for (int bit = 1; bit <= 2; bit <<= 1) {  // bits 1, 2 (t): across the quad
      const bool up = (t & bit) != 0;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float pv = __shfl_xor_sync(0xffffffffu, d[nt][j], bit);
          d[nt][j] = up ? __fsub_rn(pv, d[nt][j]) : __fadd_rn(d[nt][j], pv);
        }
    }
#pragma unroll
    for (int bit = 1; bit < 16; bit <<= 1) {  // bits 3..6 (nt)
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        if (nt & bit) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x0 = d[nt][j], x1 = d[nt | bit][j];
          d[nt][j] = __fadd_rn(x0, x1);
          d[nt | bit][j] = __fsub_rn(x0, x1);
        }
      }
    }
    // per token: zb[q][a] = y at r_q + 32a, r_q = 8 (q >> 1) + 2t + (q & 1): nt = (q >> 1) + 4a, e = q & 1
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float zb[8][4];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) zb[q][aa] = d[(q >> 1) + 4 * aa][2 * half + (q & 1)] * kInvSqrtD;
      finish_token_tc(a, half ? tb : ta, half ? vb : va, h, kind, zb, t);
    }
  }
}

}  // namespace

okv_status launch_append(const okv_cache_desc* d, const void* k, const void* v, int T,
                         const int32_t* seq_slot, const int32_t* pos, const int32_t* block_table,
                         const int32_t* slot_lens, uint32_t flags, float* rotated_out,
                         cudaStream_t s) {
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
  a.rotated_out = rotated_out;
  a.status = d->status_word;
  a.hkv = d->num_kv_heads;
  a.num_blocks = d->num_blocks;
  a.num_slots = d->num_seq_slots;
  a.mbps = d->max_blocks_per_seq;
  if (!(flags & OKV_PRE_ROTATED) && T >= kTcMinTokens) {
    // set on every call: the attribute belongs to the current device's context
    cudaError_t e = cudaFuncSetAttribute(append_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmem);
    if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "append smem attribute: %s", cudaGetErrorString(e));
    dim3 grid((T + kTcCtaTokens - 1) / kTcCtaTokens, d->num_kv_heads, 2);
    append_tc_kernel<<<grid, kTcWarps * 32, kTcSmem, s>>>(a, T);
    return check_launch("append (tensor cores)");
  }
  dim3 grid((T + kAppTokens - 1) / kAppTokens, d->num_kv_heads, 2);
  if (flags & OKV_PRE_ROTATED) {
    append_kernel<true><<<grid, kAppThreads, 0, s>>>(a, T);
  } else {
    append_kernel<false><<<grid, kAppThreads, 0, s>>>(a, T);
  }
  return check_launch("append");
}

}  // namespace okv
