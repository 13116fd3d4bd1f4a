// Chunked-prefill attention over the INT2 paged cache: the T queries of a
// prefill chunk (already appended, positions L - T .. L - 1 of a sequence of
// L tokens) attend causally to the sequence's cache as it is held at length
// L -- sink rows and the last W positions from fp16, the rest from INT2.
//
// Three launches:
//   1. query rotation: q~ = q R_K, split into fp16 hi + lo halves of
//      q~ 2^-e (e per row so that the halves stay in fp16 range) and the
//      per-group sums of q~;
//   2. attention on the tcgen05 tensor cores (`prefill_umma_kernel<NG>`, NG
//      = 128 / group quantisation groups per vector): a CTA takes 128 query
//      rows (query token x query head of one KV head) and streams the key
//      positions 0 .. its last row's position in 64-token chunks.  Every
//      chunk is staged in shared memory as fp16: the 2-bit codes (0..3 are
//      exact in fp16) of INT2 positions with their per-group scale s and
//      minimum m, or the fp16 values of window and sink rows with s = 1 and
//      m = 0.  Then, per group k of channels,
//        score = s_k (q~_k . c_k) + m_k sum(q~_k)
//      with q~ . c on the tensor cores (q~ as hi + lo, so the products carry
//      about 22 bits), an online softmax per row, and
//        o' += sum_t (p_t s_{t,k}) c_t + sum_t p_t m_{t,k}
//      with p s as hi + lo fp16 operands and the codes as the other.  The
//      dense contraction runs on the tensor cores; nothing is dequantised to
//      a rounded value;
//   3. normalise and un-rotate: o = (o' / l) R_V^T per row.
#include "okv_common.cuh"
#include "okv_internal.h"
#include "umma.cuh"

namespace okv {
namespace {

constexpr int kPfRows = 128;  // query rows per attention CTA (the MMA's M)

struct PrefillArgs {
  const __nv_bfloat16* q;  // [T][Hq][128]
  const int32_t* block_table;
  const uint8_t* pages;
  const __half* ring;
  const __half* sink;
  const float* u_k;
  const float* u_v;
  uint32_t* status;
  __half* qhi;   // [T][Hq][128]: hi half of q~ 2^-e
  __half* qlo;   // [T][Hq][128]: lo half
  float* qaux;   // [T][Hq][8]: sum of q~ per group (4), 2^e, spare
  float* obuf;   // [T][Hq][132]: o' (128), l, spare
  float* out;    // [T][Hq][128]
  int T, hq, hkv, g, ng, bhb, slot, L, first, mbps, num_blocks, nsink;
};

constexpr int kQaux = 8;
constexpr int kOStride = 132;

// ---------------------------------------------------------------------------
// 1. q~ = q R_K for the chunk, and 3. o = (o' / l) R_V^T: one CTA per 64 rows
// (token, query head) of one KV head.  The CTA stages the head's U (permuted
// so that lane l's four columns l + 32 c are one 16-byte load) and the 64
// input rows in shared memory; each warp takes 8 rows at once, so that every
// U load feeds 8 rows, on the paired fp32 FMA.  The butterfly and the
// bit-reversal remap run per row in registers.
// ---------------------------------------------------------------------------
constexpr int kRtRows = 64;
constexpr size_t kRtSmem = (size_t)(kD * kD + kRtRows * kD) * sizeof(float);

// global row of row rk (0 .. T G - 1) of KV head hk: token rk / G, query head hk G + rk % G
__device__ __forceinline__ int rt_row(const PrefillArgs& a, int hk, int rk) {
  return (rk / a.g) * a.hq + hk * a.g + rk % a.g;
}

// acc[rr] = x[rr] . U for 8 rows held in xs (fp32 rows of kD), U permuted in up
__device__ __forceinline__ void rt_matvec8(const float* xs, const float* up, int lane, float2 (&acc)[8][2]) {
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) acc[rr][0] = acc[rr][1] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int i = 0; i < kD; i += 4) {
    float4 x4[8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) x4[rr] = *reinterpret_cast<const float4*>(xs + rr * kD + i);
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const float4 u = *reinterpret_cast<const float4*>(up + (i + ii) * kD + 4 * lane);
      const float2 u01 = make_float2(u.x, u.y), u23 = make_float2(u.z, u.w);
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        const float xv = ii == 0 ? x4[rr].x : ii == 1 ? x4[rr].y : ii == 2 ? x4[rr].z : x4[rr].w;
        const float2 x2 = make_float2(xv, xv);
        acc[rr][0] = __ffma2_rn(x2, u01, acc[rr][0]);
        acc[rr][1] = __ffma2_rn(x2, u23, acc[rr][1]);
      }
    }
  }
}

__global__ void __launch_bounds__(256) prefill_qrot_kernel(PrefillArgs a) {
  extern __shared__ __align__(16) float rt_[];
  float* up = rt_;             // up[i][4 l + c] = U_K[i][l + 32 c]
  float* xs = rt_ + kD * kD;   // the tile's query rows, fp32
  const int hk = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nrows = a.T * a.g;
  const int r0 = blockIdx.x * kRtRows;
  {
    // lane l gathers U_K[i][l + 32 c] (coalesced across the warp) and stores one 16-byte chunk
    // (the loads of 8 rows go out before their stores: one L2 latency per 8 rows)
    const float* U = a.u_k + (size_t)hk * kD * kD;
    const int l = threadIdx.x & 31, i0 = threadIdx.x >> 5;  // rows i0, i0 + 8, ...
#pragma unroll 1
    for (int ib = 0; ib < kD; ib += 64) {
      float4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float* ur = U + (size_t)(ib + i0 + 8 * k) * kD + l;
        v[k] = make_float4(__ldg(ur), __ldg(ur + 32), __ldg(ur + 64), __ldg(ur + 96));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) *reinterpret_cast<float4*>(up + (ib + i0 + 8 * k) * kD + 4 * l) = v[k];
    }
    uint4 qv[kRtRows * kD / 8 / 256];  // this thread's 8-element pieces of the tile's rows
#pragma unroll
    for (int k = 0; k < kRtRows * kD / 8 / 256; ++k) {
      const int idx = threadIdx.x + 256 * k, r = idx >> 4, c8 = (idx & 15) * 8;
      qv[k] = *reinterpret_cast<const uint4*>(a.q + (size_t)rt_row(a, hk, min(r0 + r, nrows - 1)) * kD + c8);
    }
#pragma unroll
    for (int k = 0; k < kRtRows * kD / 8 / 256; ++k) {
      const int idx = threadIdx.x + 256 * k, r = idx >> 4, c8 = (idx & 15) * 8;
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&qv[k]);
      const float2 f0 = __bfloat1622float2(b2[0]), f1 = __bfloat1622float2(b2[1]);
      const float2 f2 = __bfloat1622float2(b2[2]), f3 = __bfloat1622float2(b2[3]);
      *reinterpret_cast<float4*>(xs + r * kD + c8) = make_float4(f0.x, f0.y, f1.x, f1.y);
      *reinterpret_cast<float4*>(xs + r * kD + c8 + 4) = make_float4(f2.x, f2.y, f3.x, f3.y);
    }
  }
  __syncthreads();
  {
    const int rb = 8 * warp;
    float2 acc[8][2];
    rt_matvec8(xs + rb * kD, up, lane, acc);
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int rk = r0 + rb + rr;
      if (rk >= nrows) continue;  // uniform across the warp
      const int row = rt_row(a, hk, rk);
      // lane l holds x[l + 32 c] in acc[rr][c / 2].(c % 2)
      float y[4] = {acc[rr][0].x, acc[rr][0].y, acc[rr][1].x, acc[rr][1].y};
      wht128_warp(y, lane);
#pragma unroll
      for (int aa = 0; aa < 4; ++aa) y[aa] *= kInvSqrtD;
      // lane l holds rotated channels 4 r + {0, 2, 1, 3} (r = rev5(l)) in y[0..3]
      const int r = rev5(lane);
      const float zc[4] = {y[0], y[2], y[1], y[3]};
      float amax = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
      amax = warp_max(amax);
      // 2^-e with amax 2^-e in [1, 2): the hi half keeps 11 bits, the lo half the next 11
      int e = 0;
      if (amax > 0.f) e = ((__float_as_int(amax) >> 23) & 0xff) - 127;
      e = max(-100, min(100, e));
      const float down = __int_as_float((127 - e) << 23);
      uint32_t hw[2], lw[2];
#pragma unroll
      for (int f = 0; f < 4; f += 2) {
        const float x0 = zc[f] * down, x1 = zc[f + 1] * down;
        const __half2 h = __floats2half2_rn(x0, x1);
        const float2 hb = __half22float2(h);
        const __half2 l2 = __floats2half2_rn(x0 - hb.x, x1 - hb.y);
        hw[f >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        lw[f >> 1] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      *reinterpret_cast<uint2*>(a.qhi + (size_t)row * kD + 4 * r) = make_uint2(hw[0], hw[1]);
      *reinterpret_cast<uint2*>(a.qlo + (size_t)row * kD + 4 * r) = make_uint2(lw[0], lw[1]);
      // per-group sums of q~: channels 4r.. lie in group r ng / 32
      const float part = (zc[0] + zc[1]) + (zc[2] + zc[3]);
      float* aux = a.qaux + (size_t)row * kQaux;
      for (int k = 0; k < a.ng; ++k) {  // (uniform: a.ng is 1, 2 or 4)
        const float gk = warp_sum(r * a.ng / 32 == k ? part : 0.f);
        if (lane == 0) aux[k] = gk;
      }
      if (lane == 0) aux[4] = __int_as_float((127 + e) << 23);
    }
  }
}

__device__ __forceinline__ uint32_t pack_half2(float lo_elem, float hi_elem) {
  const __half2 h = __floats2half2_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// 2. attention on the tcgen05 tensor cores (NG = 1, 2 or 4 groups per
// vector; a group is both 64-channel K-blocks, one of them or half of one,
// and its scores, p s and value MMA are kept apart).  A CTA takes
// 128 query rows of one KV head (the MMA's M) and streams the key positions
// in chunks of 64 (four cache blocks), with warp roles:
//   warps 0-7  softmax: warp w serves rows 32 (w % 4) .. + 31 (TMEM lanes,
//              one row per thread) and score columns 32 (w / 4) .. + 31 of
//              the chunk.  Per chunk a thread reads its 32 scores from TMEM,
//              applies the per-token scale and minimum term and the causal
//              limit, meets its partner (the other half of the row) for the
//              row maximum, keeps the online softmax state in registers, and
//              writes p s (hi + lo fp16) into the chunk's score columns in
//              TMEM, where the value MMA reads it as its A operand;
//   warps 8-11 staging: the chunk's codes (or fp16 window / sink rows) into
//              shared memory as fp16 tiles in the MMA's K-major layout --
//              keys as [token][channel], values transposed to
//              [channel][token] -- and the per-token (scale, min) pairs;
//   warp 12    TMEM allocation; lane 0 issues the MMAs:
//              S(c) = q~hi K^T + q~lo K^T (M 128, N 64 per group, K 128
//              over the groups) into one of two TMEM score buffers (one with
//              four groups), O += (p s)hi V + (p s)lo V (M 128, N 128 / NG
//              per group, K 64) into the TMEM output.
// Both MMAs take their A operand from TMEM (q~ is staged there once; p s
// replaces the scores it came from), so shared memory holds only the key and
// value tiles and the MMAs read nothing else from it.
// Two buffers of every per-chunk tile; mbarriers hand them around:
//   k_full    staging -> MMA, softmax  (a chunk's key tile and key scales are in place)
//   v_full    staging -> MMA, softmax  (its value tile and value scales)
//   s_full    MMA -> softmax           (S(c) is in TMEM)
//   s_free    softmax -> MMA, staging  (S(c) and the key scales were read: the score
//                                       buffer and the key tile may take chunk c + 2)
//   p_full    softmax -> MMA           (p s of chunk c is in shared memory)
//   pv_done   MMA -> all               (O includes chunk c; its value tile and p s are free)
//   mx        softmax partners         (both halves of the rows posted their maximum)
// The running maximum is lazy: a row rescales O (TMEM load, scale, store)
// only when a chunk's maximum exceeds the one in use by more than tau, so p
// stays below 2^tau; tau <= 12 is chosen per chunk so that p s stays inside
// fp16 for the chunk's largest value scale.  Every wait is bounded; on a
// timeout the kernel raises OKV_DEV_TIMEOUT, waits (bounded) for the MMAs it
// issued, frees TMEM and returns.
// ---------------------------------------------------------------------------
constexpr int kUpKC = 64;        // key positions per chunk
constexpr int kUpSmxWarps = 8;   // warps 0..7
constexpr int kUpStgWarps = 4;   // warps 8..11
constexpr int kUpMmaWarp = 12;
constexpr int kUpThreads = 32 * (kUpSmxWarps + kUpStgWarps + 1);
constexpr uint32_t kUpKBytes = 2 * 8192;   // a chunk's keys: 2 K-blocks of 64 rows x 128 B
constexpr uint32_t kUpVBytes = 16384;      // a chunk's values: 128 channel rows x 64 tokens
constexpr uint32_t kUpOffK = 0;
constexpr uint32_t kUpOffV = kUpOffK + 2 * kUpKBytes;
constexpr uint32_t kUpOffMisc = kUpOffV + 2 * kUpVBytes;
struct UpMisc {
  float2 ksm[2][4 * kUpKC];         // key (scale, min) of token j, group k at j NG + k: (1, 0) fp16 rows, (0, 0) masked
  float2 vsm[2][4 * kUpKC];         // value (scale, min), the same way
  int kval[2][kUpKC];               // 1 where the token was staged (only read when a block id was bad)
  float vsmax[2][kUpStgWarps];      // largest value scale, per staging warp
  int bad[2][kUpStgWarps];          // a block id was out of range, per staging warp
  float red[2][2][128];             // per chunk parity, column half, row: the half-row maximum
  float4 fin[2][128];               // per column half, row: l and the sums p m the partner needs, at the end
  uint64_t k_full[2], v_full[2], s_full[2], s_free[2], p_full[2], pv_done[2], mx[4][2];
  uint32_t tmem_slot;
};
constexpr size_t kUpSmem = 1024 + kUpOffMisc + sizeof(UpMisc);
// TMEM columns: scores 2 x 64 NG from 0 (group k's 64 columns at 64 k; p s
// of a group then replaces its scores: per column half h of the row, hi at
// 32 h + 0..15 and lo at 32 h + 16..31 of the group's columns); O 128 from
// 128 NG; q~ hi 64 and lo 64 after O.  With four groups (32-channel groups)
// two score buffers would fill TMEM: one buffer of 256 columns, O at 256, q~
// at 384, and the score MMAs of chunk c + 1 wait for the value MMAs of c.
constexpr uint32_t kUpTmemCols = 512;
constexpr uint32_t kUpIdescS = um_idesc(64, false, false);
constexpr uint32_t kUpIdescO = um_idesc(128, false, false);
constexpr uint32_t kUpIdescO64 = um_idesc(64, false, false);
constexpr uint32_t kUpIdescO32 = um_idesc(32, false, false);
constexpr uint32_t kF16Bias2 = 0x64006400u;  // (1024, 1024) as fp16 pair: 1024 + c is exact for c < 1024

// (1024 + lo, 1024 + hi) - 1024 for two 2-bit codes already in bits 0-1 and 16-17
__device__ __forceinline__ uint32_t codes_to_half2(uint32_t x) {
  const uint32_t b = (x & 0x00030003u) | kF16Bias2, bias = kF16Bias2;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&b), *reinterpret_cast<const __half2*>(&bias));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Value codes are staged centred, as 2 c - 3 (exact in fp16), with half the
// scale: s c + m = (s / 2)(2 c - 3) + (m + 1.5 s).  The value sum then holds
// terms of both signs, and the minimum term m + 1.5 s is the centre of the
// token's range, so neither sum is a large number cancelling another.
// (1024 + 2 lo, 1024 + 2 hi) - 1027 for two codes at bits 1-2 and 17-18 of x.
constexpr uint32_t kF16Centre2 = 0x64036403u;  // (1027, 1027)
__device__ __forceinline__ uint32_t centred_to_half2(uint32_t x) {
  const uint32_t b = (x & 0x00060006u) | kF16Bias2, bias = kF16Centre2;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&b), *reinterpret_cast<const __half2*>(&bias));
  return *reinterpret_cast<const uint32_t*>(&h);
}
// codes at bits 2k, 2k + 1 (and 16 higher) moved to bits 1-2 (17-18)
template <int k>
__device__ __forceinline__ uint32_t codes_at_bit1(uint32_t x) {
  if constexpr (k == 0)
    return x << 1;
  else
    return x >> (2 * k - 1);
}

// 16 consecutive-channel codes of one word (channel 4 b + k at bits 8 b + 2 k)
// as 8 fp16 pairs of adjacent channels (centred: 2 c - 3)
template <bool kCentred>
__device__ __forceinline__ void word_to_half2x8(uint32_t w, uint32_t (&e)[8]) {
  const uint32_t ev = w & 0x33333333u;         // channels 4 b, 4 b + 2 at bits 0-1, 4-5 of byte b
  const uint32_t od = (w >> 2) & 0x33333333u;  // channels 4 b + 1, 4 b + 3
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t x = __byte_perm(ev, od, (uint32_t)(b | (b << 4) | ((4 + b) << 8) | ((4 + b) << 12)));
    if constexpr (kCentred) {
      e[2 * b] = centred_to_half2(x << 1);
      e[2 * b + 1] = centred_to_half2(x >> 3);
    } else {
      e[2 * b] = codes_to_half2(x);
      e[2 * b + 1] = codes_to_half2(x >> 4);
    }
  }
}

// 2^x by the SFU's approximate exponent (PTX ex2.approx.ftz.f32); -inf gives +0
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int NG>
__global__ void __launch_bounds__(kUpThreads, 1) prefill_umma_kernel(PrefillArgs a) {
  static_assert(NG == 1 || NG == 2 || NG == 4, "one, two or four quantisation groups per vector");
  constexpr int kSW = 64 * NG;                  // score columns per buffer
  constexpr int kSBufs = NG == 4 ? 1 : 2;       // score buffers (TMEM holds one of four groups' width)
  constexpr uint32_t kUpColO = kSBufs * kSW, kUpColQ = kSBufs * kSW + 128;
  static_assert(kUpColQ + 128 <= kUpTmemCols, "TMEM columns");
  auto sbuf = [](int b) -> uint32_t { return kSBufs == 1 ? 0u : (uint32_t)(b * kSW); };
  extern __shared__ unsigned char up_raw[];
  const uint32_t raw_u32 = smem_u32(up_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  unsigned char* gb = up_raw + (base - raw_u32);
  UpMisc& ms = *reinterpret_cast<UpMisc*>(gb + kUpOffMisc);
  const uint32_t sK = base + kUpOffK, sV = base + kUpOffV;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hk = blockIdx.y;
  const int nrows = a.T * a.g;
  const int row0 = blockIdx.x * 128;
  const int last_row = min(nrows, row0 + 128) - 1;
  const int pmax = a.first + last_row / a.g;  // last position any row of this CTA sees
  const int nch = pmax / kUpKC + 1;
  const int32_t* table = a.block_table + (size_t)a.slot * a.mbps;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.k_full[i], 32 * kUpStgWarps);
      mbar_init(&ms.v_full[i], 32 * kUpStgWarps);
      mbar_init(&ms.s_full[i], 1);
      mbar_init(&ms.s_free[i], 32 * kUpSmxWarps);
      mbar_init(&ms.p_full[i], 32 * kUpSmxWarps);
      mbar_init(&ms.pv_done[i], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&ms.mx[q][i], 64);
    }
    fence_mbar_init();
  }
  if (warp == kUpMmaWarp) um_alloc(&ms.tmem_slot, kUpTmemCols);

  // ---- softmax rows: q~ halves into the A tiles, per-row constants
  int rrow = 0, rpos = 0;
  bool rok = false;
  float qsum = 0.f, qup = 0.f;
  uint32_t qrow[64];  // this thread's half of its q~ row (fp16 pairs), until it is in TMEM
  const int quarter = warp & 3, hcol = (warp >> 2) & 1;  // softmax: lane quarter, column half
  const int rowc = 32 * quarter + lane;                    // softmax: row in the tile (TMEM lane)
  grid_dep_launch();  // the un-rotation may start staging U_V
  if (warp < kUpSmxWarps) {
    const int r = row0 + rowc;
    rok = r < nrows;
    const int rr = rok ? r : nrows - 1;
    const int rtok = rr / a.g;
    rrow = rtok * a.hq + hk * a.g + rr % a.g;
    rpos = a.first + rtok;
    {  // column half 0 takes the row's hi half of q~, half 1 the lo half (to TMEM below)
      const uint4* src = reinterpret_cast<const uint4*>((hcol ? a.qlo : a.qhi) + (size_t)rrow * kD);
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        const uint4 x = src[c16];
        qrow[4 * c16] = x.x;
        qrow[4 * c16 + 1] = x.y;
        qrow[4 * c16 + 2] = x.z;
        qrow[4 * c16 + 3] = x.w;
      }
    }
    const float* aux = a.qaux + (size_t)rrow * kQaux;
    qsum = aux[0] * (kInvSqrtD * kLog2e);
    qup = aux[4] * (kInvSqrtD * kLog2e);
  }

  // ---- staging: per-thread roles and the register-held fetch of one chunk
  const int stid = tid - 32 * kUpSmxWarps, sw = stid >> 5;
  const int ktk = 16 * sw + (lane & 15), kkb = lane >> 4;      // key token, K-block (64 channels)
  const int vtq = lane & 15, vbq = 2 * sw + (lane >> 4);       // value token quad, channel sixteen
  // What a staging thread fetched of one chunk, held in registers until it is
  // staged; two of them alternate, so that a chunk's loads are in flight two
  // chunks before its tiles are written.
  struct Fetched {
    int ksrc, vsrc[4], sbad;  // sources: 0 masked, 1 INT2, 2 fp16; sbad: a block id was out of range
    int p0;                   // first position of the chunk
    uint4 kr0;                // INT2 key codes of the token (64 channels)
    uint4 vw;                 // INT2 value codes of the quad (16 channels x 4 tokens)
    uint32_t ksmw[NG];        // the token's (scale, min) per group: key scales for kkb 0, value scales for kkb 1
  };
  Fetched fa, fb;
  // block ids of this thread's key token and value quad, looked up one chunk
  // before their codes are fetched (the table read and the code read would
  // otherwise be two dependent memory latencies per chunk)
  auto lookup = [&](int c, int& kblk, int& vblk) {
    const int pk = kUpKC * c + ktk, pv = kUpKC * c + 4 * vtq;
    kblk = (c < nch && pk <= pmax && pk < a.L) ? table[pk >> 4] : -1;
    vblk = (c < nch && pv <= pmax && pv < a.L) ? table[pv >> 4] : -1;
  };
  int kblk_n = -1, vblk_n = -1;  // block ids of the next chunk to fetch
  // the fp16 row (sink or window ring) of position p
  auto fp16_row = [&](int p, int kind) -> const __half* {
    const bool sink = p < a.nsink;
    const size_t rows = sink ? (size_t)a.nsink : (size_t)kWin;
    const size_t row = sink ? (size_t)p : (size_t)(p % kWin);
    return (sink ? a.sink : a.ring) + ((((size_t)a.slot * a.hkv + hk) * 2 + kind) * rows + row) * kD;
  };
  // key position p: 1 INT2 (block-head base in *bp), 2 fp16 (read at staging), 0 masked
  auto locate = [&](Fetched& f, int p, int blk, const uint8_t** bp) -> int {
    if (p > pmax || p >= a.L) return 0;
    if (p < a.nsink || p >= a.L - kWin) return 2;
    if (blk < 0 || blk >= a.num_blocks) {
      if (!f.sbad) raise_flag(a.status, OKV_DEV_BAD_BLOCK);
      f.sbad = 1;
      return 0;
    }
    *bp = a.pages + ((size_t)blk * a.hkv + hk) * a.bhb;
    return 1;
  };
  auto fetch = [&](Fetched& f, int c, int kblk, int vblk) {
    const int p0 = kUpKC * c;
    f.p0 = p0;
    f.sbad = 0;
    // a chunk wholly between the sink rows and the fp16 window, and below every
    // row's position, is INT2 throughout (the common case): no per-token sorting
    if (p0 >= a.nsink && p0 + kUpKC - 1 < a.L - kWin && p0 + kUpKC - 1 <= pmax) {
      const bool kok = kblk >= 0 && kblk < a.num_blocks, vok = vblk >= 0 && vblk < a.num_blocks;
      if (!(kok && vok)) {
        raise_flag(a.status, OKV_DEV_BAD_BLOCK);
        f.sbad = 1;
      }
      f.ksrc = kok ? 1 : 0;
      if (kok) {
        const uint8_t* bp = a.pages + ((size_t)kblk * a.hkv + hk) * a.bhb;
        f.kr0 = *reinterpret_cast<const uint4*>(bp + kKcOff + (ktk & 15) * 32 + 16 * kkb);
#pragma unroll
        for (int k = 0; k < NG; ++k)
          f.ksmw[k] = *reinterpret_cast<const uint32_t*>(bp + sm_offset(NG, kkb, ktk & 15, k));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) f.vsrc[i] = vok ? 1 : 0;
      if (vok)
        f.vw = *reinterpret_cast<const uint4*>(a.pages + ((size_t)vblk * a.hkv + hk) * a.bhb + kVcOff +
                                               ((vbq * 4 + (vtq & 3)) << 4));
      return;
    }
    {
      const uint8_t* bp = nullptr;
      const int p = p0 + ktk;
      f.ksrc = locate(f, p, kblk, &bp);
      if (f.ksrc == 1) {
        f.kr0 = *reinterpret_cast<const uint4*>(bp + kKcOff + (p & 15) * 32 + 16 * kkb);
#pragma unroll
        for (int k = 0; k < NG; ++k)
          f.ksmw[k] = *reinterpret_cast<const uint32_t*>(bp + sm_offset(NG, kkb, p & 15, k));
      }
    }
    {
      const uint8_t* bp = nullptr;
      bool any_int2 = false;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint8_t* bpi = nullptr;
        f.vsrc[i] = locate(f, p0 + 4 * vtq + i, vblk, &bpi);
        if (f.vsrc[i] == 1) {
          bp = bpi;
          any_int2 = true;
        }
      }
      if (any_int2) f.vw = *reinterpret_cast<const uint4*>(bp + kVcOff + ((vbq * 4 + (vtq & 3)) << 4));
    }
  };
  // (scale, min) of the fetched token: key scales for kkb 0, value scales for kkb 1
  auto token_sm = [&](const Fetched& f, int k, float& s_, float& m_) {
    s_ = m_ = 0.f;
    if (f.ksrc == 1) {
      s_ = __half2float(__ushort_as_half((unsigned short)(f.ksmw[k] & 0xffffu)));
      m_ = __half2float(__ushort_as_half((unsigned short)(f.ksmw[k] >> 16)));
    } else if (f.ksrc == 2) {
      s_ = 1.f;
    }
  };
  auto stage_k = [&](const Fetched& f, int b) {
    // keys: 8 chunks of 8 channels into row ktk of K-block kkb
    const uint32_t kdst = sK + (uint32_t)b * kUpKBytes + (uint32_t)kkb * 8192u;
    unsigned char* kg = gb + (kdst - base);
    if (f.ksrc == 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t e[8];
        const uint32_t w = i == 0 ? f.kr0.x : i == 1 ? f.kr0.y : i == 2 ? f.kr0.z : f.kr0.w;
        word_to_half2x8<false>(w, e);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          *reinterpret_cast<uint4*>(kg + um_swz((uint32_t)ktk, (uint32_t)(2 * i + hh) * 16u)) =
              make_uint4(e[4 * hh], e[4 * hh + 1], e[4 * hh + 2], e[4 * hh + 3]);
      }
    } else {
      const uint4* x = f.ksrc == 2 ? reinterpret_cast<const uint4*>(fp16_row(f.p0 + ktk, 0) + 64 * kkb) : nullptr;
#pragma unroll
      for (int jc = 0; jc < 8; ++jc)
        *reinterpret_cast<uint4*>(kg + um_swz((uint32_t)ktk, (uint32_t)jc * 16u)) =
            f.ksrc == 2 ? x[jc] : make_uint4(0, 0, 0, 0);
    }
    if (kkb == 0) {
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        float s_, m_;
        token_sm(f, k, s_, m_);
        ms.ksm[b][ktk * NG + k] = make_float2(s_, m_);
      }
      ms.kval[b][ktk] = f.ksrc != 0;
    }
    const int anybad = __any_sync(0xffffffffu, f.sbad != 0);
    if (lane == 0) ms.bad[b][sw] = anybad;
  };
  const int flip = lane >> 4;
  // lanes 16..31 write rows 16 apart from lanes 0..15 (same swizzle phase):
  // they hold and store the other token pair first, so each store covers 32 banks
  const uint32_t sel_a = flip ? 0x0302u : 0x0110u, sel_b = flip ? 0x0110u : 0x0302u;
  auto stage_v = [&](const Fetched& f, int b) {
    float vmx = 0.f;
    if (kkb == 1) {
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        float s_, m_;
        token_sm(f, k, s_, m_);
        if (f.ksrc == 1) {
          ms.vsm[b][ktk * NG + k] = make_float2(0.5f * s_, fmaf(1.5f, s_, m_));  // centred codes
          vmx = fmaxf(vmx, 0.5f * s_);
        } else {
          ms.vsm[b][ktk * NG + k] = make_float2(s_, m_);
          vmx = fmaxf(vmx, s_);
        }
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, o));
    if (lane == 0) ms.vsmax[b][sw] = vmx;
    // values: channels 16 vbq + ch, token pairs (2 vtq + s): one 32-bit word per
    // (channel, pair); pr[ch][s0] is the pair stored at position s0 ^ flip
    uint32_t pr[16][2];
    if (f.vsrc[0] == 1 && f.vsrc[1] == 1 && f.vsrc[2] == 1 && f.vsrc[3] == 1) {
      const uint32_t ws[4] = {f.vw.x, f.vw.y, f.vw.z, f.vw.w};  // word b': channels 4 b' .. + 3 of tokens 0..3
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const uint32_t x01 = __byte_perm(ws[bb], 0u, sel_a);  // the pair's two tokens in bytes 0, 2
        const uint32_t x23 = __byte_perm(ws[bb], 0u, sel_b);
        pr[4 * bb + 0][0] = centred_to_half2(codes_at_bit1<0>(x01));
        pr[4 * bb + 0][1] = centred_to_half2(codes_at_bit1<0>(x23));
        pr[4 * bb + 1][0] = centred_to_half2(codes_at_bit1<1>(x01));
        pr[4 * bb + 1][1] = centred_to_half2(codes_at_bit1<1>(x23));
        pr[4 * bb + 2][0] = centred_to_half2(codes_at_bit1<2>(x01));
        pr[4 * bb + 2][1] = centred_to_half2(codes_at_bit1<2>(x23));
        pr[4 * bb + 3][0] = centred_to_half2(codes_at_bit1<3>(x01));
        pr[4 * bb + 3][1] = centred_to_half2(codes_at_bit1<3>(x23));
      }
    } else {
      uint32_t e[4][8];  // per token: fp16 pairs of adjacent channels
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (f.vsrc[i] == 1) {
          const uint32_t sel = (uint32_t)(i | ((4 + i) << 4));
          const uint32_t t01 = __byte_perm(f.vw.x, f.vw.y, sel), t23 = __byte_perm(f.vw.z, f.vw.w, sel);
          word_to_half2x8<true>(__byte_perm(t01, t23, 0x5410u), e[i]);
        } else if (f.vsrc[i] == 2) {
          const uint4* x = reinterpret_cast<const uint4*>(fp16_row(f.p0 + 4 * vtq + i, 1) + 16 * vbq);
          const uint4 x0 = x[0], x1 = x[1];
          e[i][0] = x0.x; e[i][1] = x0.y; e[i][2] = x0.z; e[i][3] = x0.w;
          e[i][4] = x1.x; e[i][5] = x1.y; e[i][6] = x1.z; e[i][7] = x1.w;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) e[i][j] = 0u;
        }
      }
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint32_t sel = (ch & 1) ? 0x7632u : 0x5410u;
        const uint32_t t01 = __byte_perm(e[0][ch >> 1], e[1][ch >> 1], sel);
        const uint32_t t23 = __byte_perm(e[2][ch >> 1], e[3][ch >> 1], sel);
        pr[ch][0] = flip ? t23 : t01;
        pr[ch][1] = flip ? t01 : t23;
      }
    }
    unsigned char* vg = gb + (sV + (uint32_t)b * kUpVBytes - base);
#pragma unroll
    for (int ch = 0; ch < 16; ++ch)
#pragma unroll
      for (int s0 = 0; s0 < 2; ++s0)
        *reinterpret_cast<uint32_t*>(vg + um_swz((uint32_t)(16 * vbq + ch), (uint32_t)(2 * vtq + (s0 ^ flip)) * 4u)) =
            pr[ch][s0];
  };
  if (warp >= kUpSmxWarps && warp < kUpMmaWarp) {
    int kb0, vb0;
    lookup(0, kb0, vb0);
    fetch(fa, 0, kb0, vb0);
    lookup(1, kb0, vb0);
    if (1 < nch) fetch(fb, 1, kb0, vb0);
    lookup(2, kblk_n, vblk_n);
  }

  um_fence_before();
  __syncthreads();
  um_fence_after();
  const uint32_t tmem = ms.tmem_slot;
  const uint32_t tS = tmem, tO = tmem + kUpColO, tQ = tmem + kUpColQ;
  if (warp < kUpSmxWarps) {  // q~ of this warp's 32 rows: half hcol into columns 64 hcol ..
    const uint32_t ta = tQ + ((uint32_t)(32 * quarter) << 16) + 64u * (uint32_t)hcol;
    um_st16(ta, qrow);
    um_st16(ta + 16u, qrow + 16);
    um_st16(ta + 32u, qrow + 32);
    um_st16(ta + 48u, qrow + 48);
    um_wait_st();
  }
  um_fence_before();
  __syncthreads();  // q~ is in TMEM before the first score MMA
  um_fence_after();

  if (warp < kUpSmxWarps) {
    // ------------------------------------------------------------ softmax
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    float m_use = -INFINITY;
    float2 l2 = make_float2(0.f, 0.f), msum2[NG];  // two partial sums each (paired arithmetic)
#pragma unroll
    for (int k = 0; k < NG; ++k) msum2[k] = make_float2(0.f, 0.f);
    const float2 qup2 = make_float2(qup, qup), qsum2 = make_float2(qsum, qsum);
    float qsum_g[NG];  // per-group sums of q~ (log2 units)
#pragma unroll
    for (int k = 0; k < NG; ++k) qsum_g[k] = a.qaux[(size_t)rrow * kQaux + k] * (kInvSqrtD * kLog2e);
    bool alive = true;
    for (int c = 0; c < nch && alive; ++c) {
      const int b = c & 1;
      const uint32_t ph = ((uint32_t)c >> 1) & 1u;
      alive = mbar_wait_bounded(&ms.k_full[b], ph) && mbar_wait_bounded(&ms.s_full[b], ph);
      alive = __all_sync(0xffffffffu, alive);
      if (!alive) break;
      um_fence_after();
      float sv[32];
      um_ld32(tS + lane_base + sbuf(b) + (uint32_t)(32 * hcol), sv);
      if constexpr (NG == 4) {
        // x = sum over the four groups of s_k (q~_k . c_k) 2^e + m_k sum q~_k, one group's raw
        // scores at a time
        um_wait_ld();
        const float4* kk = reinterpret_cast<const float4*>(&ms.ksm[b][4 * 32 * hcol]);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float4 k4 = kk[2 * j];  // (s, m) of groups 0 and 1 of token j
          sv[j] = fmaf(k4.x * qup, sv[j], k4.y * qsum_g[0]);
        }
#pragma unroll 1
        for (int k = 1; k < 4; ++k) {
          float svk[32];
          um_ld32(tS + lane_base + sbuf(b) + (uint32_t)(64 * k + 32 * hcol), svk);
          um_wait_ld();
          const float2* k2 = &ms.ksm[b][4 * 32 * hcol + k];
          const float qg = k == 1 ? qsum_g[1] : k == 2 ? qsum_g[2] : qsum_g[3];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float2 sm = k2[4 * j];
            sv[j] = fmaf(sm.x * qup, svk[j], fmaf(sm.y, qg, sv[j]));
          }
        }
      } else if constexpr (NG == 2) {
        // x = s0 (q~0 . c0) + m0 sum q~0 + s1 (q~1 . c1) + m1 sum q~1: group 1's raw scores
        // and both groups' (scale, min) fold in here; the common code below then sees s = 1, m = 0
        float sv1[32];
        um_ld32(tS + lane_base + sbuf(b) + (uint32_t)(64 + 32 * hcol), sv1);
        um_wait_ld();
        const float4* kk = reinterpret_cast<const float4*>(&ms.ksm[b][2 * 32 * hcol]);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float4 k4 = kk[j];  // (s, m) of groups 0 and 1 of token j
          sv[j] = fmaf(k4.x * qup, sv[j], fmaf(k4.y, qsum_g[0], fmaf(k4.z * qup, sv1[j], k4.w * qsum_g[1])));
        }
      }
      um_wait_ld();
      um_fence_before();
      // scores in log2 units: s (q~ . c) 2^e / sqrt(d) + m sum(q~) / sqrt(d); columns j < lim are
      // causal and inside the sequence
      const int lim = min(rpos + 1, a.L) - kUpKC * c - 32 * hcol;
      const bool bad = (ms.bad[b][0] | ms.bad[b][1] | ms.bad[b][2] | ms.bad[b][3]) != 0;
      const float4* k4p = reinterpret_cast<const float4*>(&ms.ksm[b][32 * hcol]);
      float bm = -INFINITY;
      if constexpr (NG >= 2) {
        const int* kv = &ms.kval[b][32 * hcol];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const bool ok = j < lim && (!bad || kv[j] != 0);
          sv[j] = ok ? sv[j] : -INFINITY;
          bm = fmaxf(bm, sv[j]);
        }
      } else if (lim >= 32 && !bad) {
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float4 k4 = k4p[j2];  // (s, m) of columns 2 j2, 2 j2 + 1
          const float2 x = __ffma2_rn(__fmul2_rn(make_float2(k4.x, k4.z), qup2), make_float2(sv[2 * j2], sv[2 * j2 + 1]),
                                      __fmul2_rn(make_float2(k4.y, k4.w), qsum2));
          sv[2 * j2] = x.x;
          sv[2 * j2 + 1] = x.y;
          bm = fmaxf(bm, fmaxf(x.x, x.y));
        }
      } else {
        const int* kv = &ms.kval[b][32 * hcol];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float4 k4 = k4p[j2];
          const float2 x = __ffma2_rn(__fmul2_rn(make_float2(k4.x, k4.z), qup2), make_float2(sv[2 * j2], sv[2 * j2 + 1]),
                                      __fmul2_rn(make_float2(k4.y, k4.w), qsum2));
          const bool ok0 = 2 * j2 < lim && (!bad || kv[2 * j2] != 0);
          const bool ok1 = 2 * j2 + 1 < lim && (!bad || kv[2 * j2 + 1] != 0);
          sv[2 * j2] = ok0 ? x.x : -INFINITY;
          sv[2 * j2 + 1] = ok1 ? x.y : -INFINITY;
          bm = fmaxf(bm, fmaxf(sv[2 * j2], sv[2 * j2 + 1]));
        }
      }
      mbar_arrive(&ms.s_free[b]);  // scores and key scales read
      ms.red[b][hcol][rowc] = bm;
      mbar_arrive(&ms.mx[quarter][b]);
      // tau: p < 2^tau and p s < 2^15 for the chunk's largest value scale
      alive = mbar_wait_bounded(&ms.v_full[b], ph);
      alive = __all_sync(0xffffffffu, alive);
      if (!alive) break;
      const float vmax = fmaxf(fmaxf(ms.vsmax[b][0], ms.vsmax[b][1]), fmaxf(ms.vsmax[b][2], ms.vsmax[b][3]));
      const int ex = vmax > 0.f ? ((__float_as_int(vmax) >> 23) & 0xff) - 127 : 0;
      const float tau = (float)max(0, min(12, 14 - ex));  // (a cap of 8 rescaled more often: 64-channel groups 3.09 ms, 3.00 at 12)
      alive = mbar_wait_bounded(&ms.mx[quarter][b], ph);
      alive = __all_sync(0xffffffffu, alive);
      if (!alive) break;
      bm = fmaxf(bm, ms.red[b][hcol ^ 1][rowc]);  // the row's maximum (both halves decide alike)
      const bool need = bm > m_use + tau;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2_ftz(m_use - bm) : 1.f;  // 0 while the row has seen nothing
        if (c > 0) {
          // O must hold chunk c - 1 before it is scaled; this thread scales columns 64 hcol .. + 63
          alive = mbar_wait_bounded(&ms.pv_done[(c - 1) & 1], ((uint32_t)(c - 1) >> 1) & 1u);
          alive = __all_sync(0xffffffffu, alive);
          if (!alive) break;
          um_fence_after();
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            float ov[32];
            const uint32_t ta = tO + lane_base + (uint32_t)(64 * hcol + 32 * q);
            um_ld32(ta, ov);
            um_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            um_st32(ta, ov);
          }
          um_wait_st();
        }
        l2 = __fmul2_rn(l2, make_float2(alpha, alpha));
#pragma unroll
        for (int k = 0; k < NG; ++k) msum2[k] = __fmul2_rn(msum2[k], make_float2(alpha, alpha));
        if (need) m_use = bm;
      }
      const float mref = m_use == -INFINITY ? 0.f : m_use;
      const float2 nm2 = make_float2(-mref, -mref);
      // p s over the scores of chunk c in TMEM: columns 16 hcol .. (hi) and
      // 32 + 16 hcol .. (lo) of the chunk's buffer.  The lo columns held the
      // partner's scores, which it read before it posted its maximum; the
      // value MMA of chunk c - 2 (c - 1 with one buffer), the last reader of
      // this buffer's p s, finished before S(c) was written into it.
      um_fence_after();
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        // group k: p s_k over this thread's 32 scores of group k (p is recomputed per group)
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float2 d = __fadd2_rn(make_float2(sv[2 * j2], sv[2 * j2 + 1]), nm2);
          const float2 pp = make_float2(ex2_ftz(d.x), ex2_ftz(d.y));
          const float2 v0 = ms.vsm[b][(32 * hcol + 2 * j2) * NG + k], v1 = ms.vsm[b][(32 * hcol + 2 * j2 + 1) * NG + k];
          if (k == 0) l2 = __fadd2_rn(l2, pp);
          msum2[k] = __ffma2_rn(pp, make_float2(v0.y, v1.y), msum2[k]);
          const float2 w = __fmul2_rn(pp, make_float2(v0.x, v1.x));
          // hi: w with its low 13 mantissa bits cleared (exact in fp16 from 2^-14 up); lo: the rest
          const float2 wh = make_float2(__uint_as_float(__float_as_uint(w.x) & 0xFFFFE000u),
                                        __uint_as_float(__float_as_uint(w.y) & 0xFFFFE000u));
          const float2 wl = __fadd2_rn(w, make_float2(-wh.x, -wh.y));
          hi[j2] = pack_half2(wh.x, wh.y);
          lo[j2] = pack_half2(wl.x, wl.y);
        }
        // NG = 1: hi at 16 hcol, lo at 32 + 16 hcol (the lo columns held the partner's
        // scores, read before it posted its maximum); NG = 2: over this thread's own
        // 32 score columns of group k
        const uint32_t tp = tS + lane_base + sbuf(b) +
                            (NG == 1 ? 16u * (uint32_t)hcol : 64u * (uint32_t)k + 32u * (uint32_t)hcol);
        um_st16(tp, hi);
        um_st16(tp + (NG == 1 ? 32u : 16u), lo);
      }
      um_wait_st();
      um_fence_before();
      mbar_arrive(&ms.p_full[b]);
    }
    if (alive) {
      alive = mbar_wait_bounded(&ms.pv_done[(nch - 1) & 1], ((uint32_t)(nch - 1) >> 1) & 1u);
      alive = __all_sync(0xffffffffu, alive);
    }
    float l = 0.f, msum = 0.f, msum_b = 0.f;  // msum_b: channels 64 hcol + 32 .. with four groups
    if (alive) {
      // the two halves' sums meet: one more round of the partners' barrier
      if constexpr (NG == 4) {
        // the partner writes channels 64 (1 - hcol) ..: groups 2 (1 - hcol) and + 1
        const float2 a0 = hcol ? msum2[0] : msum2[2], a1 = hcol ? msum2[1] : msum2[3];
        ms.fin[hcol][rowc] = make_float4(l2.x + l2.y, a0.x + a0.y, a1.x + a1.y, 0.f);
      } else {
        ms.fin[hcol][rowc] = make_float4(l2.x + l2.y, msum2[0].x + msum2[0].y,
                                         NG == 2 ? msum2[NG - 1].x + msum2[NG - 1].y : 0.f, 0.f);
      }
      mbar_arrive(&ms.mx[quarter][nch & 1]);
      alive = mbar_wait_bounded(&ms.mx[quarter][nch & 1], ((uint32_t)nch >> 1) & 1u);
      alive = __all_sync(0xffffffffu, alive);
      const float4 f0 = ms.fin[0][rowc], f1 = ms.fin[1][rowc];
      l = f0.x + f1.x;
      if constexpr (NG == 4) {
        const float4 fp = hcol ? f0 : f1;  // the partner's post
        const float2 o0 = hcol ? msum2[2] : msum2[0], o1 = hcol ? msum2[3] : msum2[1];
        msum = (o0.x + o0.y) + fp.y;
        msum_b = (o1.x + o1.y) + fp.z;
      } else {
        // this thread writes channels 64 hcol ..: group hcol when NG = 2
        msum = (NG == 2 && hcol == 1) ? f0.z + f1.z : f0.y + f1.y;
        msum_b = msum;
      }
    }
    if (alive) {
      um_fence_after();
      float* dst = a.obuf + (size_t)rrow * kOStride + 64 * hcol;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        float ov[32];
        um_ld32(tO + lane_base + (uint32_t)(64 * hcol + 32 * q), ov);
        um_wait_ld();
        if (rok) {
          const float mq = q ? msum_b : msum;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + 32 * q + i) =
                make_float4(ov[i] + mq, ov[i + 1] + mq, ov[i + 2] + mq, ov[i + 3] + mq);
        }
      }
      if (rok && hcol == 0) a.obuf[(size_t)rrow * kOStride + 128] = l;
    } else if (lane == 0) {
      raise_flag(a.status, OKV_DEV_TIMEOUT);
    }
  } else if (warp < kUpMmaWarp) {
    // ------------------------------------------------------------ staging
    // chunk c from fetch slot f, then chunk c + 2's loads into the same slot
    auto run_chunk = [&](Fetched& f, int c) -> bool {
      const int b = c & 1;
      // keys once the score MMA and the softmax of chunk c - 2 are past them
      if (c >= 2 && !mbar_wait_bounded(&ms.s_free[b], ((uint32_t)(c - 2) >> 1) & 1u)) return false;
      stage_k(f, b);
      um_fence_proxy_async();
      mbar_arrive(&ms.k_full[b]);
      // values once the value MMA of chunk c - 2 is done
      if (c >= 2 && !mbar_wait_bounded(&ms.pv_done[b], ((uint32_t)(c - 2) >> 1) & 1u)) return false;
      stage_v(f, b);
      um_fence_proxy_async();
      mbar_arrive(&ms.v_full[b]);
      if (c + 2 < nch) {
        fetch(f, c + 2, kblk_n, vblk_n);
        lookup(c + 3, kblk_n, vblk_n);
      }
      return true;
    };
    for (int c = 0; c < nch; c += 2) {
      if (!run_chunk(fa, c) || (c + 1 < nch && !run_chunk(fb, c + 1))) {
        raise_flag(a.status, OKV_DEV_TIMEOUT);
        break;
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issue
    // order: S(0), S(1), then per chunk c: O += P(c) V(c) as soon as the
    // softmax of c is done, then S(c + 2) once its keys are staged.  (Issuing
    // S(c + 2) first measured slower: its wait on the keys then delays the
    // value MMA, which the staging of the next values waits for.)
    uint64_t* last_bar = nullptr;  // the latest commit: it completes after every MMA issued before it
    uint32_t last_par = 0;
    // Descriptors: a tile's base descriptor plus (byte offset >> 4) in the start
    // address field (shared addresses stay below 2^18, so the field never
    // carries), which keeps this thread's per-MMA work to an add and the MMA.
    const uint64_t dK0 = um_desc(sK), dK1 = um_desc(sK + kUpKBytes);
    const uint64_t dV0 = um_desc(sV), dV1 = um_desc(sV + kUpVBytes);
    auto issue_s = [&](int c) -> bool {
      const int b = c & 1;
      if (!mbar_wait_bounded(&ms.k_full[b], ((uint32_t)c >> 1) & 1u)) return false;
      if (c >= 2 && !mbar_wait_bounded(&ms.s_free[b], ((uint32_t)(c - 2) >> 1) & 1u)) return false;
      // one score buffer: the value MMAs of c - 1 read their p s from it
      // (waiting for their completion here measured faster than relying on
      // the issue order of this thread's MMAs)
      if (kSBufs == 1 && c >= 1 &&
          !mbar_wait_bounded(&ms.pv_done[(c - 1) & 1], ((uint32_t)(c - 1) >> 1) & 1u))
        return false;
      um_fence_after();
      const uint64_t kd = b ? dK1 : dK0;
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // q~ channels 64 kb + 16 ks .. + 15: TMEM columns 8 (4 kb + ks) of its half
            const uint32_t ta = tQ + 64u * (uint32_t)half + 8u * (uint32_t)(4 * kb + ks);
            const uint64_t bd = kd + (uint64_t)((kb * 8192 + ks * 32) >> 4);
            // NG = 2: K-block kb is group kb, into its own 64 columns; NG = 4: channels
            // 32 g .. of group g = 2 kb + ks / 2
            const uint32_t gcol = NG == 2 ? 64u * (uint32_t)kb : NG == 4 ? 64u * (uint32_t)(2 * kb + (ks >> 1)) : 0u;
            const int first = NG == 2 ? (half | ks) : NG == 4 ? (half | (ks & 1)) : (half | ks | kb);
            um_mma_ts(tS + sbuf(b) + gcol, ta, bd, kUpIdescS, first != 0 ? 1u : 0u);
          }
      um_commit(&ms.s_full[b]);
      last_bar = &ms.s_full[b];
      last_par = ((uint32_t)c >> 1) & 1u;
      return true;
    };
    auto issue_pv = [&](int c) -> bool {
      const int b = c & 1;
      if (!mbar_wait_bounded(&ms.p_full[b], ((uint32_t)c >> 1) & 1u)) return false;
      if (!mbar_wait_bounded(&ms.v_full[b], ((uint32_t)c >> 1) & 1u)) return false;
      um_fence_after();
      const uint64_t vd = b ? dV1 : dV0;
      if constexpr (NG == 1) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // tokens 16 ks .. + 15 of p s (hi or lo): TMEM columns 32 half + 8 ks of the chunk's buffer
            const uint32_t ta = tS + sbuf(b) + 32u * (uint32_t)half + 8u * (uint32_t)ks;
            const uint64_t bd = vd + (uint64_t)((ks * 32) >> 4);
            um_mma_ts(tO, ta, bd, kUpIdescO, (c > 0 || half > 0 || ks > 0) ? 1u : 0u);
          }
      } else if constexpr (NG == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              // group k (channel rows 32 k .., output columns 32 k ..), tokens 16 ks ..: p s as
              // for two groups, in the group's 64 score columns
              const uint32_t ta = tS + 64u * (uint32_t)k + 32u * (uint32_t)(ks >> 1) + 16u * (uint32_t)half +
                                  8u * (uint32_t)(ks & 1);
              const uint64_t bd = vd + (uint64_t)((k * 4096 + ks * 32) >> 4);
              um_mma_ts(tO + 32u * (uint32_t)k, ta, bd, kUpIdescO32, (c > 0 || half > 0 || ks > 0) ? 1u : 0u);
            }
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              // group k, tokens 16 ks ..: p s written by column half ks / 2 at 32 (ks / 2) +
              // 16 half + 8 (ks % 2) of the group's columns; values: channel rows 64 k ..
              const uint32_t ta = tS + sbuf(b) + 64u * (uint32_t)k + 32u * (uint32_t)(ks >> 1) +
                                  16u * (uint32_t)half + 8u * (uint32_t)(ks & 1);
              const uint64_t bd = vd + (uint64_t)((k * 8192 + ks * 32) >> 4);
              um_mma_ts(tO + 64u * (uint32_t)k, ta, bd, kUpIdescO64, (c > 0 || half > 0 || ks > 0) ? 1u : 0u);
            }
      }
      um_commit(&ms.pv_done[b]);
      last_bar = &ms.pv_done[b];
      last_par = ((uint32_t)c >> 1) & 1u;
      return true;
    };
    bool alive = issue_s(0);
    if constexpr (kSBufs == 2) {
      alive = alive && (nch < 2 || issue_s(1));
      for (int c = 0; c < nch && alive; ++c) alive = issue_pv(c) && (c + 2 >= nch || issue_s(c + 2));
    } else {
      for (int c = 0; c < nch && alive; ++c) alive = issue_pv(c) && (c + 1 >= nch || issue_s(c + 1));
    }
    if (!alive) raise_flag(a.status, OKV_DEV_TIMEOUT);
    // the MMAs already issued finish before TMEM is freed (the softmax warps may
    // have given up on them): the last commit covers them all
    if (last_bar != nullptr) mbar_drain_bounded(last_bar, last_par);
  }
  um_fence_before();
  __syncthreads();
  if (warp == kUpMmaWarp) {
    um_fence_after();
    um_dealloc(tmem, kUpTmemCols);
  }
}

// 3. o = (o' / l) R_V^T (see 1. for the tiling): un-permute, 1 / l and the
// butterfly per row in registers, the row to shared memory, then o = x U_V^T
// with U_V^T permuted: ut[i][4 l + j] = U_V[l + 32 j][i].
__global__ void __launch_bounds__(256) prefill_unrotate_kernel(PrefillArgs a) {
  extern __shared__ __align__(16) float rt_[];
  float* ut = rt_;
  float* xs = rt_ + kD * kD;
  const int hk = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nrows = a.T * a.g;
  const int r0 = blockIdx.x * kRtRows;
  {
    // lane l reads 16 bytes of rows l + 32 j (columns i0 .. i0 + 3) and stores
    // the four 16-byte chunks ut[i0 + k][4 l .. 4 l + 3]: conflict-free
    const float* U = a.u_v + (size_t)hk * kD * kD;
    float4 uu[4][4];  // all four of this thread's pieces are loaded before any is stored
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = threadIdx.x + 256 * k, l = t & 31, i0 = 4 * (t >> 5);
#pragma unroll
      for (int j = 0; j < 4; ++j) uu[k][j] = __ldg(reinterpret_cast<const float4*>(U + (size_t)(l + 32 * j) * kD + i0));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = threadIdx.x + 256 * k, l = t & 31, i0 = 4 * (t >> 5);
      const float4* u = uu[k];
      *reinterpret_cast<float4*>(ut + (i0 + 0) * kD + 4 * l) = make_float4(u[0].x, u[1].x, u[2].x, u[3].x);
      *reinterpret_cast<float4*>(ut + (i0 + 1) * kD + 4 * l) = make_float4(u[0].y, u[1].y, u[2].y, u[3].y);
      *reinterpret_cast<float4*>(ut + (i0 + 2) * kD + 4 * l) = make_float4(u[0].z, u[1].z, u[2].z, u[3].z);
      *reinterpret_cast<float4*>(ut + (i0 + 3) * kD + 4 * l) = make_float4(u[0].w, u[1].w, u[2].w, u[3].w);
    }
  }
  grid_dep_wait();  // the attention's outputs are read from here on
  // this warp's 8 rows: x = H-butterfly of the un-permuted o' / l, into xs.
  // All 8 rows' loads go out before the first butterfly.
  const int r = rev5(lane);
  float4 o4[8];
  float lr[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float* src = a.obuf + (size_t)rt_row(a, hk, min(r0 + 8 * warp + k, nrows - 1)) * kOStride;
    o4[k] = *reinterpret_cast<const float4*>(src + 4 * r);  // rotated channels 4 r .. 4 r + 3
    lr[k] = src[128];
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float inv = lr[k] > 0.f ? 1.f / lr[k] : 0.f;
    // lane l: pre-permutation channels l + 32 aa = rotated channels 4 rev5(l) + rev2(aa)
    float y[4] = {o4[k].x * inv, o4[k].z * inv, o4[k].y * inv, o4[k].w * inv};
    wht128_warp(y, lane);
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) xs[(8 * warp + k) * kD + lane + 32 * aa] = y[aa] * kInvSqrtD;
  }
  __syncthreads();  // U_V^T staged (this warp's rows need only __syncwarp, U needs the CTA)
  {
    const int rb = 8 * warp;
    float2 acc[8][2];
    rt_matvec8(xs + rb * kD, ut, lane, acc);
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int rk = r0 + rb + rr;
      if (rk < nrows) {
        float* dst = a.out + (size_t)rt_row(a, hk, rk) * kD;
        dst[lane] = acc[rr][0].x;
        dst[lane + 32] = acc[rr][0].y;
        dst[lane + 64] = acc[rr][1].x;
        dst[lane + 96] = acc[rr][1].y;
      }
    }
  }
}

}  // namespace

size_t prefill_workspace_bytes(int T, int hq) {
  const size_t rows = (size_t)T * hq;
  size_t off = 0;
  off += (rows * kD * sizeof(__half) + 255) / 256 * 256;  // qhi
  off += (rows * kD * sizeof(__half) + 255) / 256 * 256;  // qlo
  off += (rows * kQaux * sizeof(float) + 255) / 256 * 256;
  off += (rows * kOStride * sizeof(float) + 255) / 256 * 256;
  return off;
}

okv_status launch_prefill(const okv_cache_desc* d, const void* q, int T, int slot, int context_len,
                          const int32_t* block_table, float* out, void* ws, cudaStream_t s) {
  PrefillArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.block_table = block_table;
  a.pages = (const uint8_t*)d->pages;
  a.ring = (const __half*)d->window_ring;
  a.sink = (const __half*)d->sink_rows;
  a.u_k = d->u_k;
  a.u_v = d->u_v;
  a.status = d->status_word;
  const size_t rows = (size_t)T * d->num_q_heads;
  uint8_t* w = (uint8_t*)ws;
  size_t off = 0;
  a.qhi = (__half*)(w + off);
  off += (rows * kD * sizeof(__half) + 255) / 256 * 256;
  a.qlo = (__half*)(w + off);
  off += (rows * kD * sizeof(__half) + 255) / 256 * 256;
  a.qaux = (float*)(w + off);
  off += (rows * kQaux * sizeof(float) + 255) / 256 * 256;
  a.obuf = (float*)(w + off);
  a.out = out;
  a.T = T;
  a.hq = d->num_q_heads;
  a.hkv = d->num_kv_heads;
  a.g = a.hq / a.hkv;
  a.ng = kD / d->group;
  a.bhb = block_head_bytes(a.ng);
  a.slot = slot;
  a.L = context_len;
  a.first = context_len - T;
  a.mbps = d->max_blocks_per_seq;
  a.num_blocks = d->num_blocks;
  a.nsink = d->num_sink;
  static std::atomic<uint32_t> qr_attr{0}, ur_attr{0};
  cudaError_t e0 = set_smem_limit_once((const void*)prefill_qrot_kernel, (int)kRtSmem, qr_attr);
  if (e0 == cudaSuccess) e0 = set_smem_limit_once((const void*)prefill_unrotate_kernel, (int)kRtSmem, ur_attr);
  if (e0 != cudaSuccess) return fail(OKV_ERR_CUDA, "prefill rotation smem attribute: %s", cudaGetErrorString(e0));
  const dim3 rt_grid((unsigned)((T * a.g + kRtRows - 1) / kRtRows), (unsigned)a.hkv);
  prefill_qrot_kernel<<<rt_grid, 256, kRtSmem, s>>>(a);
  okv_status st = check_launch("prefill query rotation");
  if (st != OKV_OK) return st;
  const dim3 grid((unsigned)((T * a.g + kPfRows - 1) / kPfRows), (unsigned)a.hkv);
  switch (a.ng) {
    case 1: {
      static std::atomic<uint32_t> up_attr{0};
      cudaError_t e1 = set_smem_limit_once((const void*)prefill_umma_kernel<1>, (int)kUpSmem, up_attr);
      if (e1 != cudaSuccess) return fail(OKV_ERR_CUDA, "prefill attention smem attribute: %s", cudaGetErrorString(e1));
      prefill_umma_kernel<1><<<grid, kUpThreads, kUpSmem, s>>>(a);
      break;
    }
    case 2: {
      static std::atomic<uint32_t> up2_attr{0};
      cudaError_t e1 = set_smem_limit_once((const void*)prefill_umma_kernel<2>, (int)kUpSmem, up2_attr);
      if (e1 != cudaSuccess) return fail(OKV_ERR_CUDA, "prefill attention smem attribute: %s", cudaGetErrorString(e1));
      prefill_umma_kernel<2><<<grid, kUpThreads, kUpSmem, s>>>(a);
      break;
    }
    default: {
      static std::atomic<uint32_t> up4_attr{0};
      cudaError_t e1 = set_smem_limit_once((const void*)prefill_umma_kernel<4>, (int)kUpSmem, up4_attr);
      if (e1 != cudaSuccess) return fail(OKV_ERR_CUDA, "prefill attention smem attribute: %s", cudaGetErrorString(e1));
      prefill_umma_kernel<4><<<grid, kUpThreads, kUpSmem, s>>>(a);
      break;
    }
  }
  st = check_launch("prefill attention");
  if (st != OKV_OK) return st;
  // The un-rotation may start (programmatic launch) while the attention's last
  // CTAs run: it stages U_V, then waits for the attention's outputs.  Starting
  // the attention early behind the query rotation in the same way measured
  // slower with 64-channel groups (3.31 against 3.10 ms) and is not done.
  const cudaError_t e3 = launch_pdl(prefill_unrotate_kernel, rt_grid, dim3(256), kRtSmem, s, true, a);
  if (e3 != cudaSuccess) return fail(OKV_ERR_CUDA, "prefill un-rotation launch: %s", cudaGetErrorString(e3));
  return check_launch("prefill un-rotation");
}

}  // namespace okv
