// Shared device-side definitions of the INT2 KV-cache library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "okv.h"

namespace okv {

constexpr int kD = 128;           // head dimension
constexpr int kBlock = 16;        // tokens per block
constexpr int kWin = 128;         // fp16 window length
constexpr int kBlockHeadBytes = 1152;  // one block-head with 128-channel groups
constexpr int kKcOff = 0;         // K codes, token-major 16 x 32 B
constexpr int kVcOff = 512;       // V codes, 4-token-interleaved chunks
constexpr int kKsmOff = 1024;     // K (fp16 scale, fp16 min) per token (128-channel groups)
constexpr int kVsmOff = 1088;     // V (fp16 scale, fp16 min) per token (128-channel groups)

// Layout with ng = 128 / group quantisation groups per token-head (1, 2 or
// 4): the codes as above, then K (scale, min) pairs at 1024 + 4 (t ng + k)
// for token t, group k (channels k group .. (k + 1) group - 1), then V pairs
// at 1024 + 64 ng + 4 (t ng + k).  ng = 1 is the layout above.
__host__ __device__ __forceinline__ int block_head_bytes(int ng) { return 1024 + 128 * ng; }
__host__ __device__ __forceinline__ int sm_offset(int ng, int kind, int t, int k) {
  return 1024 + 64 * ng * kind + 4 * (t * ng + k);
}
constexpr float kInvSqrtD = 0.088388347648318440550f;  // 1/sqrt(128)
constexpr float kLog2e = 1.4426950408889634074f;

// Byte offset, inside one block-head, of canonical code byte b (channels
// 4b..4b+3) of token t in the V region.  Chunk (b>>2, t>>2) of 16 bytes holds
// bytes 4*(b>>2)..+3 of the four tokens 4*(t>>2)..+3, one 4-byte word per
// code byte, one byte per token inside the word.
__host__ __device__ __forceinline__ int v_code_offset(int t, int b) {
  return kVcOff + (((b >> 2) * 4 + (t >> 2)) << 4) + ((b & 3) << 2) + (t & 3);
}

__host__ __device__ __forceinline__ int rev5(int x) {
  return ((x & 1) << 4) | ((x & 2) << 2) | (x & 4) | ((x & 8) >> 2) | ((x & 16) >> 4);
}
// position of pre-permutation index (lane l, register a), i = l + 32a, after P_br:
// br7(32a + l) = 4*rev5(l) + rev2(a), rev2 = {0, 2, 1, 3}.
__host__ __device__ __forceinline__ int rev2(int a) { return ((a & 1) << 1) | (a >> 1); }

__device__ __forceinline__ void raise_flag(uint32_t* w, uint32_t bits) {
  if (w != nullptr) atomicOr(w, bits);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Walsh-Hadamard butterfly over 128 values held as y[a] = v[l + 32a] in lane l
// of a warp (natural/Sylvester order, unnormalised).  Lane bits use shuffles,
// register bits stay in registers.
__device__ __forceinline__ void wht128_warp(float y[4], int lane) {
#pragma unroll
  for (int b = 1; b < 32; b <<= 1) {
    const bool hi = (lane & b) != 0;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float p = __shfl_xor_sync(0xffffffffu, y[a], b);
      y[a] = hi ? __fsub_rn(p, y[a]) : __fadd_rn(y[a], p);
    }
  }
  float t0 = __fadd_rn(y[0], y[1]), t1 = __fsub_rn(y[0], y[1]);
  float t2 = __fadd_rn(y[2], y[3]), t3 = __fsub_rn(y[2], y[3]);
  y[0] = __fadd_rn(t0, t2);
  y[2] = __fsub_rn(t0, t2);
  y[1] = __fadd_rn(t1, t3);
  y[3] = __fsub_rn(t1, t3);
}

__device__ __forceinline__ __half fp16_sat(float x) {
  return __float2half_rn(fminf(fmaxf(x, -65504.0f), 65504.0f));
}

// The quantiser's code decision without a division.  With x = fl(z - m)
// and s > 0 an fp16 value, the code clamp(rint_even(fl(x / s)), 0, 3) is
//   [x > s/2] + [x >= 3s/2] + [x > 5s/2]
// exactly.  Round-to-nearest-even puts the decision points of fl(x / s) at
//   c >= 1  <=>  x / s > 1/2 + 2^-25   (a tie at 1/2 goes to the even 1/2, rint 0)
//   c >= 2  <=>  x / s >= 3/2 - 2^-24  (a tie goes to the even 3/2, rint 2)
//   c >= 3  <=>  x / s > 5/2 + 2^-23   (a tie goes to the even 5/2, rint 2)
// (half-ulps of fp32 in [1/2, 1), [1, 2), [2, 4)).  Times s, each bound is
// k s (exact: s has 11 significant bits) moved by less than one ulp of k s
// and by at least a third of one: s 2^-25 = (s/2) 2^-24, s 2^-24 =
// (3s/2) (2/3) 2^-24, s 2^-23 = (5s/2) (4/5) 2^-24.  So no fp32 number lies
// between k s and the bound, and comparing x with k s itself decides the
// same way (3s/2 is never a power of two, so its predecessor is a full ulp
// below).  Every code therefore equals the division's, bit for bit.
struct CodeThresholds {
  float h1, h2, h3;  // s/2, 3s/2, 5s/2 (exact)
};

__device__ __forceinline__ CodeThresholds code_thresholds(float s) {
  CodeThresholds t;
  t.h1 = 0.5f * s;
  t.h2 = 1.5f * s;
  t.h3 = 2.5f * s;
  return t;
}

// The code of x = fl(z - m) (only for s > 0; s = 0 gives code 0 by
// definition) is [x > s/2] + [x >= 3s/2] + [x > 5s/2].  This returns -code
// (mod 2^32) as the sum of the three decisions as all-ones / zero masks (PTX
// `set` writes 0xffffffff for true), so that w - (int2_code_neg(x, t) << k)
// adds code << k to w.
__device__ __forceinline__ uint32_t int2_code_neg(float x, const CodeThresholds& t) {
  uint32_t a, b, c;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(a) : "f"(x), "f"(t.h1));
  asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(b) : "f"(x), "f"(t.h2));
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(c) : "f"(x), "f"(t.h3));
  return a + b + c;
}

// INT2 group quantiser over the 128 values of a warp (y[a] = value at
// pre-permutation index l + 32a, i.e. rotated channel 4*rev5(l) + rev2(a)).
// With ng groups per vector (ng = 128 / group: 1, 2 or 4), the group of
// lane l's four channels is rev5(l) * ng / 32: the lanes that share
// l mod ng form one group, so the min/max reductions stop at lane distance
// ng.  All steps are IEEE fp32 round-to-nearest; returns this lane's packed
// code byte (canonical byte rev5(l)) and its group's fp16 scale/min bits.
struct Quantized {
  uint32_t byte;
  uint32_t sm;  // fp16 scale in bits 0-15, fp16 min in bits 16-31
};

__device__ __forceinline__ Quantized quantize_warp(const float y[4], int ng = 1) {
  float mn = fminf(fminf(y[0], y[1]), fminf(y[2], y[3]));
  float mx = fmaxf(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    if (o < ng) break;
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
  const __half s16 = fp16_sat(s32);
  const __half m16 = fp16_sat(mn);
  const float s = __half2float(s16);
  const float m = __half2float(m16);
  uint32_t byte = 0;
  if (s != 0.0f) {
    const CodeThresholds th = code_thresholds(s);
#pragma unroll
    for (int a = 0; a < 4; ++a) byte -= int2_code_neg(__fsub_rn(y[a], m), th) << (2 * rev2(a));
  }
  Quantized q;
  q.byte = byte;
  q.sm = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
  return q;
}

}  // namespace okv


namespace okv {

// ---------------------------------------------------------------------------
// sm_90+/sm_100 primitives: mbarrier, bulk async copy (global -> shared), and
// the legacy-path integer MMA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// One bulk copy of `bytes` (multiple of 16, both addresses 16-B aligned) from
// global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before its predecessor finishes; it must call
// grid_dep_wait() before reading anything the predecessor writes.
// grid_dep_launch() lets the successor be scheduled early.  Both are no-ops
// for ordinary launches.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// 4-byte asynchronous global -> shared copy (no register round trip), grouped
// per thread; cp_async_wait_all waits for this thread's groups.
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// wait until at most N of this thread's newest copy groups are still pending
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// L2 policy for data read exactly once (the streamed cache): evict it first,
// so that small, reused tensors (rotations, block tables) stay resident.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// L2 policy for data that another CTA reads again shortly (normal eviction)
__device__ __forceinline__ uint64_t l2_evict_normal_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// bulk_g2s with an L2 cache policy
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after 2^OKV_WAIT_LIMIT_LOG2 SM cycles (2^31 by
// default, about a second) and returns false.  A test build sets a limit of
// a few dozen cycles, so that waits run out while the work they wait for is
// still in flight and the timeout paths run.
#ifndef OKV_WAIT_LIMIT_LOG2
#define OKV_WAIT_LIMIT_LOG2 31
#endif
__device__ __forceinline__ bool mbar_wait_cycles(uint64_t* bar, uint32_t parity, long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}
// non-blocking test of a phase (try_wait may itself suspend the thread until
// the phase completes, so a short limit needs polling)
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
#if OKV_WAIT_LIMIT_LOG2 < 31
  const long long t0 = clock64();
  while (!mbar_test_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << OKV_WAIT_LIMIT_LOG2)) return false;
  }
  return true;
#else
  return mbar_wait_cycles(bar, parity, 1ll << 31);
#endif
}
// The wait of a timeout path for work this CTA already issued (bulk copies,
// MMAs), which completes on its own: always the full ~2^31-cycle limit, so
// that nothing lands in shared memory or TMEM after the CTA has moved on.
__device__ __forceinline__ bool mbar_drain_bounded(uint64_t* bar, uint32_t parity) {
  return mbar_wait_cycles(bar, parity, 1ll << 31);
}

// D[16x8] += A[16x32] (u8, row-major) * B[32x8] (s8 or u8, column-major), s32 accumulate.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8u8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

}  // namespace okv
