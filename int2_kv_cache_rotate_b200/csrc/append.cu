// Append kernels: rotate (U, Hadamard butterfly, bit-reversal remap), quantise
// to INT2 with fp16 scale/min, pack, and write the paged cache and fp16 window.
// Decode steps (a few tokens) run the CUDA-core kernel; prefill chunks of 128
// tokens or more run the tensor-core kernel, which takes R either from the
// cache's staged image (okv_build_r_image) or stages it from U per CTA.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "append_warp.cuh"
#include "okv_common.cuh"
#include "okv_internal.h"
#include "umma.cuh"

namespace okv {
namespace {

template <bool kPre>
__global__ void __launch_bounds__(kAppThreads) append_kernel(AppendArgs a, int T) {
  append_tile<kPre>(a, T, blockIdx.x, blockIdx.y, blockIdx.z);
}

// ---------------------------------------------------------------------------
// Tensor-core append for long token runs (prefill chunks).
//
// z = k R with R = U H P_br / sqrt(128) is a dense [T x 128] x [128 x 128]
// contraction, so it runs on mma.m16n8k16 (bf16 in, fp32 accumulate).  k is
// exact in bf16; R is split into three bf16 parts (hi + mid + lo carry 24
// mantissa bits), so every product is exact and the sums are fp32 sums.
// Each CTA builds R for its (KV head, K|V) once in shared memory: a warp
// takes a row c of U, runs the Hadamard butterfly across the warp and writes
// the row of R, already split, to columns in the order below.  Folding H and
// P_br into the staged matrix removes the per-token butterfly; the column
// order makes every lane own whole code bytes.
//
// Column order: in the accumulator of n-tile nt, lane (g, t) holds columns
// 8 nt + 2t + e (e = 0, 1) for tokens g and g + 8.  Physical column
// p = 8 (2k + (f >> 1)) + 2t + (f & 1) carries rotated channel 4 (8t + k) + f,
// so lane t holds packed bytes 8t .. 8t + 7 (channels 32t .. 32t + 31) of its
// two tokens: byte k field f is d[2k + (f >> 1)][2 half + (f & 1)].
// B fragments come from the [c][p] row-major R with ldmatrix.trans; rows
// are padded to 136 elements so the eight rows of a matrix fall in distinct
// bank groups.
// ---------------------------------------------------------------------------
constexpr int kTcMinTokens = 128;  // below this the CUDA-core kernel wins (R staging or its copy dominates)
constexpr int kTcWarps = 8;
constexpr int kTcRound = 16 * kTcWarps;  // tokens per CTA round
constexpr int kRStride = 136;            // bf16 per staged row of R
constexpr size_t kTcSmem = (size_t)3 * kD * kRStride * 2;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// physical column of rotated channel j = 4b + f
__device__ __forceinline__ int tc_column(int b, int f) {
  return 8 * (2 * (b & 7) + (f >> 1)) + 2 * (b >> 3) + (f & 1);
}

// One token held by the four lanes of a quad: v[k][f] = rotated channel
// 4 (8t + k) + f, so lane t holds channels 32t .. 32t + 31, one 32-channel
// quarter.  With ng groups per vector a group is 4 / ng quarters, and the
// min/max reduction runs over that many lanes of the quad.  It runs on every
// lane (the quad shuffles need all of them); `live` then gates validation
// and the stores.
__device__ __forceinline__ void finish_token_tc(const AppendArgs& a, int tok, bool live, int h, int kind,
                                                const float (&v)[8][4], int t) {
  float mn = v[0][0], mx = v[0][0];
#pragma unroll
  for (int k = 0; k < 8; ++k)
#pragma unroll
    for (int f = 0; f < 4; ++f) {
      mn = fminf(mn, v[k][f]);
      mx = fmaxf(mx, v[k][f]);
    }
  if (a.ng < 4) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  }
  if (a.ng < 2) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  }
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
  uint32_t w[2] = {0u, 0u};
  if (s != 0.0f) {
    const CodeThresholds th = code_thresholds(s);
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int f = 0; f < 4; ++f) w[k >> 2] -= int2_code_neg(__fsub_rn(v[k][f], m), th) << (8 * (k & 3) + 2 * f);
  }
  uint8_t* base = a.pages + ((size_t)blk * a.hkv + h) * a.bhb;
  const int sl = p & 15;
  if (kind == 0) {
    *reinterpret_cast<uint2*>(base + kKcOff + sl * 32 + 8 * t) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) base[v_code_offset(sl, 8 * t + k)] = (uint8_t)(w[k >> 2] >> (8 * (k & 3)));
  }
  if ((t & (4 / a.ng - 1)) == 0)  // the first lane of each group
    *reinterpret_cast<uint32_t*>(base + sm_offset(a.ng, kind, sl, t * a.ng / 4)) =
        (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
  __half* wrow = window_row(a, slot, h, kind, p, len);
  __half* srow = sink_row(a, slot, h, kind, p);
  if (wrow != nullptr || srow != nullptr) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      __half2 h0 = __halves2half2(fp16_sat(v[k][0]), fp16_sat(v[k][1]));
      __half2 h1 = __halves2half2(fp16_sat(v[k][2]), fp16_sat(v[k][3]));
      __half2 h2 = __halves2half2(fp16_sat(v[k + 1][0]), fp16_sat(v[k + 1][1]));
      __half2 h3 = __halves2half2(fp16_sat(v[k + 1][2]), fp16_sat(v[k + 1][3]));
      uint4 q4;
      q4.x = *reinterpret_cast<uint32_t*>(&h0);
      q4.y = *reinterpret_cast<uint32_t*>(&h1);
      q4.z = *reinterpret_cast<uint32_t*>(&h2);
      q4.w = *reinterpret_cast<uint32_t*>(&h3);
      if (wrow != nullptr) *reinterpret_cast<uint4*>(wrow + 32 * t + 4 * k) = q4;
      if (srow != nullptr) *reinterpret_cast<uint4*>(srow + 32 * t + 4 * k) = q4;
    }
  }
  if (a.rotated_out != nullptr) {
    float* row = a.rotated_out + (((size_t)tok * 2 + kind) * a.hkv + h) * kD + 32 * t;
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<float4*>(row + 4 * k) = make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
  }
}

// Grid (ceil(T / tokens_per_cta), Hkv, 2); a CTA stages R once and runs
// rounds of 128 tokens (16 per warp) over its token range.
__global__ void __launch_bounds__(kTcWarps * 32, 2) append_tc_kernel(AppendArgs a, int T, int tokens_per_cta) {
  extern __shared__ __align__(16) unsigned char tc_smem[];
  __nv_bfloat16* rs = reinterpret_cast<__nv_bfloat16*>(tc_smem);  // [3][128 c][136]: R split in three
  const int h = blockIdx.y, kind = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = blockIdx.x * tokens_per_cta, t1 = min(T, t0 + tokens_per_cta);
  {
    // row c of R = (row c of U) H P_br / sqrt(128): butterfly across the warp;
    // lane l's value a is rotated channel 4 rev5(l) + rev2(a)
    const float* U = (kind ? a.u_v : a.u_k) + (size_t)h * kD * kD;
    const int b = rev5(lane);
    int col[4];
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) col[aa] = tc_column(b, rev2(aa));
    for (int c0 = warp; c0 < kD; c0 += 4 * kTcWarps) {  // rows c0 + {0, 1, 2, 3} * kTcWarps
      float y[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) y[r][aa] = __ldg(U + (size_t)(c0 + r * kTcWarps) * kD + lane + 32 * aa);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        wht128_warp(y[r], lane);
        const int c = c0 + r * kTcWarps;
#pragma unroll
        for (int aa = 0; aa < 4; ++aa) {
          const float u = y[r][aa] * kInvSqrtD;
          const __nv_bfloat16 p0 = __float2bfloat16_rn(u);
          const float r1 = u - __bfloat162float(p0);
          const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
          const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
          rs[(0 * kD + c) * kRStride + col[aa]] = p0;
          rs[(1 * kD + c) * kRStride + col[aa]] = p1;
          rs[(2 * kD + c) * kRStride + col[aa]] = p2;
        }
      }
    }
  }
  __syncthreads();
  // ldmatrix.trans row addresses: lanes 8j..8j+7 give the rows of matrix j;
  // matrices 0, 1 = k rows 0-7 / 8-15 of an n-tile (b0, b1), 2, 3 = the same
  // for the next n-tile.
  const int mrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int mcol = 8 * (lane >> 4);
  const uint32_t rs_base = smem_u32(rs) + (uint32_t)(mrow * kRStride + mcol) * 2u;
  const __nv_bfloat16* src = (const __nv_bfloat16*)(kind ? a.v : a.k);
  for (int r0 = t0 + 16 * warp; r0 < t1; r0 += kTcRound) {
    const int ta = r0 + g, tb = r0 + g + 8;
    const bool va = ta < t1, vb = tb < t1;
    const uint32_t* ra = reinterpret_cast<const uint32_t*>(src + ((size_t)(va ? ta : t0) * a.hkv + h) * kD);
    const uint32_t* rb = reinterpret_cast<const uint32_t*>(src + ((size_t)(vb ? tb : t0) * a.hkv + h) * kD);
    uint32_t af[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      af[ks][0] = va ? __ldg(ra + 8 * ks + t) : 0u;
      af[ks][1] = vb ? __ldg(rb + 8 * ks + t) : 0u;
      af[ks][2] = va ? __ldg(ra + 8 * ks + 4 + t) : 0u;
      af[ks][3] = vb ? __ldg(rb + 8 * ks + 4 + t) : 0u;
    }
    float d[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) d[nt][j] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int nt = 0; nt < 16; nt += 2) {
          uint32_t bf[4];
          ldsm_x4_trans(bf, rs_base + (uint32_t)((part * kD + 16 * ks) * kRStride + 8 * nt) * 2u);
          mma_bf16(d[nt], af[ks], bf[0], bf[1]);
          mma_bf16(d[nt + 1], af[ks], bf[2], bf[3]);
        }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[8][4];
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int f = 0; f < 4; ++f) v[k][f] = d[2 * k + (f >> 1)][2 * half + (f & 1)];
      finish_token_tc(a, half ? tb : ta, half ? vb : va, h, kind, v, t);
    }
  }
}

// ---------------------------------------------------------------------------
// tcgen05 append (prefill chunks): the same z = k R contraction on the
// 5th-generation tensor cores, accumulators in tensor memory.
//
// B = R^T (128 output channels x K = 384: R's three bf16 parts stacked along
// K, so one accumulation gives k R0 + k R1 + k R2) lives in shared memory in
// the K-major 128-byte-swizzled layout the MMA descriptors describe: part pt,
// K-block kb (64 channels) is a 16 KB region of 128 rows x 128 B; element
// (n, c) sits in row n, 16-byte chunk ((c % 64) / 8) ^ (n % 8).  A is one
// 128-token tile of k for this KV head in the same layout (two K-blocks).
//
// Roles (warp-specialised):
//   warp 8      producer: one lane loads each A tile with two TMA tensor
//               copies (channels 0-63 and 64-127, the hardware applying the
//               128-byte swizzle; rows past T are filled with zeros) into a
//               3-stage ring, completing on afull[stage]; once a tile is in,
//               it issues the 24 MMAs (M = N = 128, K = 16) into TMEM buffer
//               i & 1, committed to mma_done[i & 1];
//   warps 0-3   epilogue of even tiles, warps 4-7 of odd tiles: warp w reads
//               TMEM lanes 32 (w % 4) .. +31, one token per thread, all 128
//               columns; it frees the TMEM buffer (tmem_free) as soon as the
//               values are in registers, then quantises and stores.
// Every mbarrier wait is bounded; TMEM is freed on every path.
// ---------------------------------------------------------------------------
constexpr int kUmEpiWarps = 8;
constexpr int kUmProducer = kUmEpiWarps;             // warp index of the producer
constexpr int kUmThreads = 32 * (kUmEpiWarps + 1);
constexpr int kUmTile = 128;
constexpr int kUmStages = 3;
constexpr uint32_t kUmRegion = 16384;                 // 128 rows x 128 B
constexpr uint32_t kUmBBytes = 6 * kUmRegion;         // 3 parts x 2 K-blocks
constexpr uint32_t kUmABytes = 2 * kUmRegion;         // one tile, 2 K-blocks
constexpr uint32_t kUmCtlBytes = 80;                  // 8 barriers and the TMEM base
static_assert(8 * 8 + 4 <= kUmCtlBytes, "control region");
constexpr size_t kUmSmem = 1024 + kUmBBytes + kUmStages * kUmABytes + kUmCtlBytes;
constexpr uint32_t kUmTmemCols = 256;
// instruction descriptor: D f32, A and B bf16, both K-major, N = 128, M = 128
constexpr uint32_t kUmIdesc = um_idesc(128, true, true);

// R = U H P_br / sqrt(128) of one (KV head, K|V), split in three bf16 parts,
// written into `img` in the B-operand image above (part pt, K-block kb at
// (2 pt + kb) 16 KB; element (n, c) in row n, 16-byte chunk ((c % 64) / 8) ^
// (n % 8)).  The swizzle is computed from the row index, so the image is the
// same wherever it lies; copied to a 1024-byte aligned shared address it is
// what the MMA descriptors expect.  Warp w of 8 takes input channels 16w ..
// 16w + 15 in two batches of eight: after the butterflies a lane holds its
// four output channels for all eight input channels, which is one 16-byte
// chunk of each of those four B rows.
__device__ __forceinline__ void stage_r_parts(const float* U, unsigned char* img, int warp, int lane) {
  const int b = rev5(lane);
#pragma unroll 1
  for (int c0 = 16 * warp; c0 < 16 * warp + 16; c0 += 8) {
    float y[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int aa = 0; aa < 4; ++aa) y[r][aa] = __ldg(U + (size_t)(c0 + r) * kD + lane + 32 * aa);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      wht128_warp(y[r], lane);
#pragma unroll
      for (int aa = 0; aa < 4; ++aa) y[r][aa] *= kInvSqrtD;
    }
    const uint32_t kb = (uint32_t)c0 >> 6, cb = ((uint32_t)c0 & 63u) * 2u;
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      const uint32_t nn = (uint32_t)(4 * b + rev2(aa));  // rotated channel of these values
      uint32_t pk[3][4];
#pragma unroll
      for (int r = 0; r < 8; r += 2) {
        float u0 = y[r][aa], u1 = y[r + 1][aa];
#pragma unroll
        for (int pt = 0; pt < 3; ++pt) {
          const __nv_bfloat162 pp = __floats2bfloat162_rn(u0, u1);
          pk[pt][r >> 1] = *reinterpret_cast<const uint32_t*>(&pp);
          u0 -= __low2float(pp);
          u1 -= __high2float(pp);
        }
      }
      const uint32_t off = kb * kUmRegion + um_swz(nn, cb);
#pragma unroll
      for (int pt = 0; pt < 3; ++pt)
        *reinterpret_cast<uint4*>(img + (uint32_t)pt * 2 * kUmRegion + off) =
            make_uint4(pk[pt][0], pk[pt][1], pk[pt][2], pk[pt][3]);
    }
  }
}

// one CTA of 8 warps per (KV head, K|V): the staged R into the cache's image buffer
__global__ void __launch_bounds__(256) r_image_kernel(const float* u_k, const float* u_v, uint8_t* r_image) {
  const int h = blockIdx.x, kind = blockIdx.y;
  const float* U = (kind ? u_v : u_k) + (size_t)h * kD * kD;
  stage_r_parts(U, r_image + ((size_t)h * 2 + kind) * kUmBBytes, threadIdx.x >> 5, threadIdx.x & 31);
}

// TMA tiled load of a 3-D box at (x, y, z) into shared memory, completing on bar
__device__ __forceinline__ void um_tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                               uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
template <int NG>
__global__ void __launch_bounds__(kUmThreads, 1) append_umma_kernel(AppendArgs a, int T,
                                                                     const __grid_constant__ CUtensorMap map_k,
                                                                     const __grid_constant__ CUtensorMap map_v) {
  extern __shared__ unsigned char um_raw[];
  const uint32_t raw_u32 = smem_u32(um_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  unsigned char* gbase = um_raw + (base - raw_u32);
  const uint32_t sB = base, sA = base + kUmBBytes;
  unsigned char* ctl = gbase + kUmBBytes + kUmStages * kUmABytes;
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(ctl);  // [2], one commit
  uint64_t* tmem_free = mma_done + 2;                    // [2], 128 arrivals (an epilogue warpgroup)
  uint64_t* afull = tmem_free + 2;                       // [3], one arrival + the tile's bytes
  uint64_t* rfull = afull + kUmStages;                   // the staged R copied from the cache's image
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rfull + 1);

  const int h = blockIdx.y, kind = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_tiles_all = (T + kUmTile - 1) / kUmTile;
  const int n = n_tiles_all > (int)blockIdx.x ? (n_tiles_all - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (n == 0) return;  // before any TMEM allocation
  const CUtensorMap* map = kind ? &map_v : &map_k;  // [T][Hkv][128] bf16, boxes of 128 tokens x 64 channels
  auto tile_of = [&](int i) { return (int)blockIdx.x + i * (int)gridDim.x; };

  // producer lane 0: tile i of this KV head into stage i % 3 (both K-blocks)
  auto load_tile = [&](int i) {
    const int st = i % kUmStages;
    const uint32_t abuf = sA + (uint32_t)st * kUmABytes;
    mbar_arrive_expect_tx(&afull[st], kUmABytes);
    um_tma_load_3d(abuf, map, 0, h, tile_of(i) * kUmTile, &afull[st]);
    um_tma_load_3d(abuf + kUmRegion, map, 64, h, tile_of(i) * kUmTile, &afull[st]);
  };
  int loaded = 0, landed = 0;  // tiles whose loads were issued / waited for (producer lane 0)
  int committed = 0;            // tiles whose MMAs were committed (producer lane 0)
  const bool r_copy = a.r_image != nullptr;  // R comes from the image, else the epilogue warps stage it
  bool r_landed = false;                      // (producer lane 0)

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&mma_done[i], 1);
      mbar_init(&tmem_free[i], 128);
    }
    for (int i = 0; i < kUmStages; ++i) mbar_init(&afull[i], 1);
    mbar_init(rfull, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kUmProducer) {
    // the first tiles' loads go out while the other warps stage R (or with the copy of R)
    if (lane == 0) {
      if (r_copy) {
        mbar_arrive_expect_tx(rfull, kUmBBytes);
        bulk_g2s(gbase, a.r_image + ((size_t)h * 2 + kind) * kUmBBytes, kUmBBytes, rfull);
      }
      load_tile(0);
      if (n > 1) load_tile(1);
      loaded = min(n, 2);
    }
  } else if (!r_copy) {
    // R into B (row n = output channel, K = input channel), staged from U here
    stage_r_parts((kind ? a.u_v : a.u_k) + (size_t)h * kD * kD, gbase, warp, lane);
    um_fence_proxy_async();  // R was written by ordinary stores; the MMA reads it through the async proxy
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(kUmTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  um_fence_before();
  __syncthreads();
  um_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool alive = true;

  if (warp == kUmProducer) {
    for (int i = 0; i < n; ++i) {
      // MMAs of tile i: its loads have landed, and the epilogue of tile i - 2 has drained TMEM
      // buffer i & 1
      if (lane == 0 && alive) {
        bool ok = true;
        if (i == 0 && r_copy) {
          ok = mbar_wait_bounded(rfull, 0u);
          r_landed = ok;
        }
        ok = ok && mbar_wait_bounded(&afull[i % kUmStages], ((uint32_t)(i / kUmStages)) & 1u);
        if (ok) landed = i + 1;
        ok = ok && (i < 2 || mbar_wait_bounded(&tmem_free[i & 1], ((uint32_t)(i - 2) >> 1) & 1u));
        if (ok) {
          um_fence_after();
          const uint32_t abuf = sA + (uint32_t)(i % kUmStages) * kUmABytes;
          const uint32_t dcol = tmem + ((uint32_t)i & 1u) * 128u;
          int step = 0;
#pragma unroll
          for (int pt = 0; pt < 3; ++pt)
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = um_desc(abuf + (uint32_t)kb * kUmRegion + (uint32_t)ks * 32u);
                const uint64_t bd = um_desc(sB + (uint32_t)(2 * pt + kb) * kUmRegion + (uint32_t)ks * 32u);
                um_mma(dcol, ad, bd, kUmIdesc, step > 0 ? 1u : 0u);
                ++step;
              }
          um_commit(&mma_done[i & 1]);
          committed = i + 1;
        } else {
          alive = false;
        }
      }
      alive = __shfl_sync(0xffffffffu, alive, 0);
      // tile i + 2 goes to the stage that held tile i - 1: wait until its MMAs are done
      if (alive && i + 2 < n) {
        if (i >= 1 && !mbar_wait_bounded(&mma_done[(i - 1) & 1], ((uint32_t)(i - 1) >> 1) & 1u)) alive = false;
        alive = __all_sync(0xffffffffu, alive);
        if (alive && lane == 0) {
          load_tile(i + 2);
          loaded = i + 3;
        }
      }
      if (!alive) {
        if (lane == 0) raise_flag(a.status, OKV_DEV_TIMEOUT);
        break;
      }
    }
    // no copy may outlive the CTA and no MMA may write TMEM after it is freed:
    // after a failed wait, wait (bounded) for the loads in flight and for the
    // last commit (it completes after every MMA issued before it)
    if (lane == 0) {
      if (r_copy && !r_landed) mbar_drain_bounded(rfull, 0u);
      for (int i = landed; i < loaded; ++i)
        if (!mbar_drain_bounded(&afull[i % kUmStages], ((uint32_t)(i / kUmStages)) & 1u)) break;
      if (committed > 0)  // (the epilogue may have given up on a tile this thread completed)
        mbar_drain_bounded(&mma_done[(committed - 1) & 1], ((uint32_t)(committed - 1) >> 1) & 1u);
    }
  } else {
    const int wg = warp >> 2, q = warp & 3;
    // destination of this thread's token in tile i, fetched one tile (of this warpgroup) ahead
    auto token_of = [&](int i) { return tile_of(i) * kUmTile + 32 * q + lane; };
    int n_slot = -1, n_pos = -1;
    if (wg < n && token_of(wg) < T) {
      n_slot = a.seq_slot[token_of(wg)];
      n_pos = a.pos[token_of(wg)];
    }
    for (int i = wg; i < n; i += 2) {
      const int tok = token_of(i);
      const int slot = n_slot, p = n_pos;
      const bool slot_ok = slot >= 0 && slot < a.num_slots;
      const int len = slot_ok ? a.slot_lens[slot] : 0;
      const bool pos_ok = slot_ok && p >= 0 && (p >> 4) < a.mbps && p < len;
      const int blk = pos_ok ? a.block_table[(size_t)slot * a.mbps + (p >> 4)] : -1;
      n_slot = n_pos = -1;
      if (i + 2 < n && token_of(i + 2) < T) {
        n_slot = a.seq_slot[token_of(i + 2)];
        n_pos = a.pos[token_of(i + 2)];
      }
      if (alive && !mbar_wait_bounded(&mma_done[i & 1], ((uint32_t)i >> 1) & 1u)) alive = false;
      alive = __all_sync(0xffffffffu, alive);
      if (!alive) {
        if (lane == 0) raise_flag(a.status, OKV_DEV_TIMEOUT);
        break;
      }
      um_fence_after();
      float v[128];
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + ((uint32_t)i & 1u) * 128u;
#pragma unroll
      for (int c = 0; c < 4; ++c) um_ld32(taddr + 32u * c, v + 32 * c);
      um_wait_ld();
      um_fence_before();
      mbar_arrive(&tmem_free[i & 1]);  // the buffer may take tile i + 2's MMAs
      // `valid` gates the stores (a token past T, or a bad destination)
      bool valid = tok < T;
      if (valid && !slot_ok) {
        raise_flag(a.status, OKV_DEV_BAD_SLOT);
        valid = false;
      } else if (valid && !pos_ok) {
        raise_flag(a.status, OKV_DEV_BAD_POS);
        valid = false;
      } else if (valid && (blk < 0 || blk >= a.num_blocks)) {
        raise_flag(a.status, OKV_DEV_BAD_BLOCK);
        valid = false;
      }
      // per group (NG per vector, 128 / NG channels each): min and max, the
      // fp16 scale and minimum, and the codes
      constexpr int GW = kD / NG;
      uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // the 32 code bytes of the token
      uint32_t smg[NG];                                    // (scale, min) bits of each group
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        // eight interleaved chains, then a tree: the extremes do not depend on the order
        float mn8[8], mx8[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) mn8[r] = mx8[r] = v[GW * k + r];
#pragma unroll
        for (int j = GW * k + 8; j < GW * (k + 1); ++j) {
          mn8[j & 7] = fminf(mn8[j & 7], v[j]);
          mx8[j & 7] = fmaxf(mx8[j & 7], v[j]);
        }
#pragma unroll
        for (int r = 4; r >= 1; r >>= 1)
#pragma unroll
          for (int u = 0; u < r; ++u) {
            mn8[u] = fminf(mn8[u], mn8[u + r]);
            mx8[u] = fmaxf(mx8[u], mx8[u + r]);
          }
        const float mn = mn8[0], mx = mx8[0];
        const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
        const __half s16 = fp16_sat(s32);
        const __half m16 = fp16_sat(mn);
        const float sc = __half2float(s16);
        const float m = __half2float(m16);
        smg[k] = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(m16) << 16);
        if (sc != 0.0f) {
          const CodeThresholds th = code_thresholds(sc);
#pragma unroll
          for (int j = GW * k; j < GW * (k + 1); ++j)
            w[j >> 4] -= int2_code_neg(__fsub_rn(v[j], m), th) << (2 * (j & 15));  // += code << 2 (j % 16)
        }
      }
      uint8_t* bp = a.pages + ((size_t)(valid ? blk : 0) * a.hkv + h) * a.bhb;
      const int sl = p & 15;
      if (kind == 0) {
        if (valid) {
          uint4* kp = reinterpret_cast<uint4*>(bp + kKcOff + sl * 32);
          kp[0] = make_uint4(w[0], w[1], w[2], w[3]);
          kp[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      } else if (valid) {
        // (four tokens' bytes share a 4-byte word here; assembling the words by
        // a byte transpose across lane quads measured no faster than byte stores)
#pragma unroll
        for (int bb = 0; bb < 32; ++bb) bp[v_code_offset(sl, bb)] = (uint8_t)(w[bb >> 2] >> (8 * (bb & 3)));
      }
      if (!valid) continue;
#pragma unroll
      for (int k = 0; k < NG; ++k) *reinterpret_cast<uint32_t*>(bp + sm_offset(NG, kind, sl, k)) = smg[k];
      __half* wr = window_row(a, slot, h, kind, p, len);
      __half* sr = sink_row(a, slot, h, kind, p);
      if (wr != nullptr || sr != nullptr) {
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          const __half2 h0 = __halves2half2(fp16_sat(v[j + 0]), fp16_sat(v[j + 1]));
          const __half2 h1 = __halves2half2(fp16_sat(v[j + 2]), fp16_sat(v[j + 3]));
          const __half2 h2 = __halves2half2(fp16_sat(v[j + 4]), fp16_sat(v[j + 5]));
          const __half2 h3 = __halves2half2(fp16_sat(v[j + 6]), fp16_sat(v[j + 7]));
          uint4 q4;
          q4.x = *reinterpret_cast<const uint32_t*>(&h0);
          q4.y = *reinterpret_cast<const uint32_t*>(&h1);
          q4.z = *reinterpret_cast<const uint32_t*>(&h2);
          q4.w = *reinterpret_cast<const uint32_t*>(&h3);
          if (wr != nullptr) *reinterpret_cast<uint4*>(wr + j) = q4;
          if (sr != nullptr) *reinterpret_cast<uint4*>(sr + j) = q4;
        }
      }
      if (a.rotated_out != nullptr) {
        float* ro = a.rotated_out + (((size_t)tok * 2 + kind) * a.hkv + h) * kD;
#pragma unroll
        for (int j = 0; j < 128; j += 4) *reinterpret_cast<float4*>(ro + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
  }
  // free TMEM: every epilogue read completed (wait::ld) before this barrier
  um_fence_before();
  __syncthreads();
  if (warp == 0) {
    um_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kUmTmemCols) : "memory");
  }
}

}  // namespace

// Tensor map of the bf16 input [T][Hkv][128] for the tcgen05 append's tile
// loads: boxes of 128 tokens x 64 channels (128 bytes, the swizzle span) of one
// KV head, 128-byte swizzle, zero fill past T.  The encoder comes from the
// driver through the runtime, so the library links no driver library.
static bool encode_tile_map(CUtensorMap* m, const void* base, int hkv, int T) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (encode == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)hkv, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)hkv * kD * 2};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kUmTile};
  const cuuint32_t elem[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

okv_status launch_r_image(const okv_cache_desc* d, cudaStream_t s) {
  static_assert(kRImageBytesPerHead == kUmBBytes, "the image holds one B operand per (KV head, K|V)");
  r_image_kernel<<<dim3(d->num_kv_heads, 2), 256, 0, s>>>(d->u_k, d->u_v, (uint8_t*)d->r_image);
  return check_launch("staged-rotation image");
}

okv_status launch_append(const okv_cache_desc* d, const void* k, const void* v, int T,
                         const int32_t* seq_slot, const int32_t* pos, const int32_t* block_table,
                         const int32_t* slot_lens, uint32_t flags, float* rotated_out,
                         cudaStream_t s) {
  const AppendArgs a = make_append_args(d, k, v, seq_slot, pos, block_table, slot_lens, rotated_out);
  const bool rows16 = (((uintptr_t)k | (uintptr_t)v) & 15u) == 0;  // TMA needs 16-byte aligned bases
  CUtensorMap map_k, map_v;
  const bool maps = !(flags & OKV_PRE_ROTATED) && T >= kTcMinTokens && rows16 &&
                    encode_tile_map(&map_k, k, d->num_kv_heads, T) && encode_tile_map(&map_v, v, d->num_kv_heads, T);
  if (maps) {
    const void* kern = a.ng == 1 ? (const void*)append_umma_kernel<1>
                       : a.ng == 2 ? (const void*)append_umma_kernel<2> : (const void*)append_umma_kernel<4>;
    static std::atomic<uint32_t> attr_set[3];  // per instantiation: ng = 1, 2, 4 -> 0, 1, 2
    cudaError_t e = set_smem_limit_once(kern, (int)kUmSmem, attr_set[a.ng >> 1]);
    if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "append smem attribute: %s", cudaGetErrorString(e));
    const int pairs = 2 * d->num_kv_heads;
    const int tiles = (T + kUmTile - 1) / kUmTile;
    const int per_pair = std::max(1, std::min(tiles, device_sm_count() / pairs));
    dim3 grid(per_pair, d->num_kv_heads, 2);
    switch (a.ng) {
      case 1: append_umma_kernel<1><<<grid, kUmThreads, kUmSmem, s>>>(a, T, map_k, map_v); break;
      case 2: append_umma_kernel<2><<<grid, kUmThreads, kUmSmem, s>>>(a, T, map_k, map_v); break;
      default: append_umma_kernel<4><<<grid, kUmThreads, kUmSmem, s>>>(a, T, map_k, map_v); break;
    }
    return check_launch("append (tcgen05)");
  }
  if (!(flags & OKV_PRE_ROTATED) && T >= kTcMinTokens) {
    static std::atomic<uint32_t> attr_set{0};
    cudaError_t e = set_smem_limit_once((const void*)append_tc_kernel, (int)kTcSmem, attr_set);
    if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "append smem attribute: %s", cudaGetErrorString(e));
    // about two CTAs per SM over all (KV head, K|V) pairs; each CTA takes whole rounds
    const int pairs = 2 * d->num_kv_heads;
    const int per_pair = std::max(1, 2 * device_sm_count() / pairs);
    const int rounds = (T + kTcRound - 1) / kTcRound;
    const int tokens_per_cta = ((rounds + per_pair - 1) / per_pair) * kTcRound;
    dim3 grid((T + tokens_per_cta - 1) / tokens_per_cta, d->num_kv_heads, 2);
    append_tc_kernel<<<grid, kTcWarps * 32, kTcSmem, s>>>(a, T, tokens_per_cta);
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
