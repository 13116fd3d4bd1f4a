// Decode attention over the INT2 paged cache: query rotation, split-K
// attention with online softmax, and the split combine with the value
// un-rotation.
#include <type_traits>

#include "append_warp.cuh"
#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {

// ---------------------------------------------------------------------------
// Work partition.  A batch entry with L tokens and S sink tokens reads
// positions [0, min(S, L)) from the fp16 sink rows, [S, L - W) from INT2
// blocks (table columns S/16 on) and [max(L - W, S), L) from the fp16 window
// ring.  It costs one unit per INT2 block (every KV head of a block is one
// contiguous run) plus kWinCost per 16-row fp16 chunk (window chunks first,
// then sink chunks).  Entries are laid end to end in "cost space"; split-K
// CTA c takes the contiguous range [c*total/NC, (c+1)*total/NC).  Inside an
// entry, cost positions [0, n_chunks * kWinCost) stand for the fp16 chunks
// (chunk i belongs to the CTA holding position i * kWinCost) and the rest for
// the blocks in order.  A (entry, CTA) pair writes partial slot
// c + b (all query heads): distinct for distinct pairs because CTAs and
// entries are both contiguous.
// ---------------------------------------------------------------------------
struct UnitShape {
  int len;        // tokens in the cache
  int n_int2;     // tokens read from INT2 blocks: positions nsink .. nsink + n_int2 - 1
  int n_pages;    // INT2 blocks touched (table columns nsink/16 on)
  int win_first;  // first position read from the fp16 window ring
  int n_win;      // tokens read from the ring: positions win_first .. len - 1
  int n_wchunk;   // 16-row chunks of those
  int n_sink;     // tokens read from the sink rows: positions 0 .. n_sink - 1
  int n_schunk;   // 16-row chunks of those
  int win_cost;   // cost of all fp16 chunks
  int cost;
};

__device__ __forceinline__ UnitShape unit_shape(int len, int nsink) {
  UnitShape s;
  s.len = len;
  s.n_int2 = max(0, len - kWin - nsink);
  s.n_pages = (s.n_int2 + kBlock - 1) / kBlock;
  s.win_first = max(max(len - kWin, 0), nsink);
  s.n_win = max(0, len - s.win_first);
  s.n_wchunk = (s.n_win + kBlock - 1) / kBlock;
  s.n_sink = min(len, nsink);
  s.n_schunk = (s.n_sink + kBlock - 1) / kBlock;
  s.win_cost = (s.n_wchunk + s.n_schunk) * kWinCost;
  s.cost = s.n_pages + s.win_cost;
  return s;
}

// CTA whose range contains cost position x (x < total)
__device__ __forceinline__ int cta_of(long long x, long long total, int nc) {
  const long long num = (x + 1) * (long long)nc;
  return (int)((num + total - 1) / total) - 1;
}

__device__ __forceinline__ int clamp_len(const int32_t* context_lens, int b, int mbps, uint32_t* status,
                                         bool report) {
  int len = context_lens[b];
  const int cap = mbps * kBlock;
  if (len < 0 || len > cap) {
    if (report) raise_flag(status, OKV_DEV_BAD_POS);
    len = len < 0 ? 0 : cap;
  }
  return len;
}

// the same clamp, reading the length with a load that bypasses L1 (used before
// grid_dep_wait(), when the kernel may start ahead of its predecessor)
__device__ __forceinline__ int clamp_len_cg(const int32_t* context_lens, int b, int mbps) {
  int len = __ldcg(context_lens + b);
  const int cap = mbps * kBlock;
  if (len < 0 || len > cap) len = len < 0 ? 0 : cap;
  return len;
}

struct DecodeArgs {
  const __nv_bfloat16* q;
  const int32_t* seq_slot;
  const int32_t* block_table;
  const int32_t* context_lens;
  const float* u_k;
  const float* u_v;
  const uint8_t* pages;
  const __half* ring;
  const __half* sink;  // fp16 rows of the first nsink positions
  float* out;
  uint32_t* status;
  float* qrot;       // [B][Hq][128]
  int8_t* qlimb;     // [B][Hq][2][128]
  float* qscale;     // [B][Hq][kQsStride]: score scale, min-term scale, sigma, sum, then the
                     // min-term scale of each quantisation group (groups < 128 channels)
  __half* qwin;      // [B][Hq][2][128]: q~/sigma as fp16 hi, lo (natural channel order)
  int32_t* prefix;   // [B+1] cost prefix over batch entries
  float* part;       // [(NC + B)][Hq][kPartStride]
  int batch, hq, hkv, g, nc, num_blocks, num_slots, mbps, nsink;
  int ng;  // quantisation groups per vector (128 / group)
  int hsplit;  // split-K CTAs per cost range: each serves G / hsplit query heads of every KV head
};

// split-K CTA count actually used: with fewer cost units than CTAs only the
// first `total` take work, so every working CTA owns a non-empty range
__device__ __forceinline__ int working_ctas(const DecodeArgs& a, long long total) {
  return (int)min((long long)a.nc, total);
}

// ---------------------------------------------------------------------------
// Kernel 1: q~ = q R_K for one (b, query head) per CTA: warp w holds rows
// 16w..16w+15 of U_K (lane l columns 4l..4l+3, all loads in flight
// together), the eight warps' partial sums meet in shared memory and warp 0
// runs the butterfly.  CTA 0 also writes the cost prefix.
// Also emits the query in the two forms the split-K kernel consumes:
// signed 8-bit limbs in MMA-fragment order and fp16 hi/lo halves.
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 256;
static_assert(kPrepThreads == kAppThreads, "the fused step kernel runs append tiles and query rotations alike");

__device__ __forceinline__ void qrot_cta(const DecodeArgs& a, int cta) {
  __shared__ float red[8][kD];
  const int b = cta / a.hq, head = cta % a.hq;
  const int hk = head / a.g;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* U = a.u_k + (size_t)hk * kD * kD;
  float4 u[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) u[r] = __ldg(reinterpret_cast<const float4*>(U + (size_t)(16 * warp + r) * kD) + lane);
  const float xv = __bfloat162float(a.q[((size_t)b * a.hq + head) * kD + 16 * warp + (lane & 15)]);
  if (cta == 0) {
    // cost prefix: thread i sums its chunk of consecutive entries, then a
    // block-wide exclusive scan (warp shuffles, then the eight warp totals)
    __shared__ int warp_tot[kPrepThreads / 32];
    const int per = (a.batch + kPrepThreads - 1) / kPrepThreads;
    const int lo = threadIdx.x * per, hi = min(a.batch, lo + per);
    int own = 0;
    for (int i = lo; i < hi; ++i) own += unit_shape(clamp_len(a.context_lens, i, a.mbps, a.status, true), a.nsink).cost;
    int inc = own;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += v;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kPrepThreads / 32; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    int run = before + inc - own;
    for (int i = lo; i < hi; ++i) {
      a.prefix[i] = run;
      run += unit_shape(clamp_len(a.context_lens, i, a.mbps, a.status, false), a.nsink).cost;
    }
    if (threadIdx.x == 0) a.prefix[a.batch] = total;
  }
  {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float x = __shfl_sync(0xffffffffu, xv, r);
      acc.x = fmaf(x, u[r].x, acc.x);
      acc.y = fmaf(x, u[r].y, acc.y);
      acc.z = fmaf(x, u[r].z, acc.z);
      acc.w = fmaf(x, u[r].w, acc.w);
    }
    *reinterpret_cast<float4*>(&red[warp][4 * lane]) = acc;
  }
  __syncthreads();
  if (warp == 0) {
    float y[4];
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += red[w][lane + 32 * aa];
      y[aa] = s;
    }
    wht128_warp(y, lane);
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) y[aa] *= kInvSqrtD;
    const int r = rev5(lane);
    const size_t bh = (size_t)b * a.hq + head;
    *reinterpret_cast<float4*>(a.qrot + bh * kD + 4 * r) = make_float4(y[0], y[2], y[1], y[3]);
    // Integer limbs for the tensor-core score tiles: Q = rint(q~/sigma) in
    // [-32000, 32000] = 256*hi + lo with hi, lo signed 8-bit.  Bytes are stored
    // in MMA-fragment order, so that a lane of quad t reads its 32 bytes in one
    // go; the order follows the K-columns each score MMA gives a lane (code
    // byte b = c / 4 holds channel c in field f = c % 4):
    //   ng = 1: one MMA per field f; quad t holds bytes 8t .. 8t + 7:
    //           c = 32t + 16h + 4i + f goes to 32t + 8f + 4h + i;
    //   ng = 2: one MMA per (group k, field pair p); quad t holds bytes
    //           16k + 4t .. + 3 in fields 2p (K-columns 4t..) and 2p + 1
    //           (16 + 4t..): c = 4 (16k + 4t + i) + 2p + h goes to
    //           32t + 16k + 8p + 4h + i;
    //   ng = 4: one MMA per group k; quad t holds field t of the group's
    //           bytes 8k .. 8k + 7: c = 4 (8k + j) + t goes to 32t + 8k + j.
    const float zc[4] = {y[0], y[2], y[1], y[3]};  // rotated channels 4r + e
    float amax = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
    amax = warp_max(amax);
    const float own = (y[0] + y[1]) + (y[2] + y[3]);
    const float sum = warp_sum(own);
    const float sigma = amax > 0.f ? amax / 32000.f : 1.f;
    const float inv = amax > 0.f ? 32000.f / amax : 0.f;
    int8_t* lim = a.qlimb + bh * 2 * kD;
    __half* qw = a.qwin + bh * 2 * kD;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 4 * r + e;
      const float x = zc[e] * inv;
      const int q = max(-32000, min(32000, __float2int_rn(x)));
      const int hi = ((q + 32896) >> 8) - 128;
      const int lo = q - 256 * hi;
      const int cb = c >> 2, f = c & 3;
      const int pos = a.ng == 1   ? (c >> 5) * 32 + f * 8 + ((c >> 4) & 1) * 4 + ((c >> 2) & 3)
                      : a.ng == 2 ? ((cb >> 2) & 3) * 32 + (cb >> 4) * 16 + (f >> 1) * 8 + (f & 1) * 4 + (cb & 3)
                                  : f * 32 + cb;
      lim[pos] = (int8_t)hi;
      lim[kD + pos] = (int8_t)lo;
      const __half hx = __float2half_rn(x);
      qw[c] = hx;
      qw[kD + c] = __float2half_rn(x - __half2float(hx));
    }
    // per-group sums of q~ (a lane's four channels 4r .. 4r + 3 share a group)
    float gsum[4] = {0.f, 0.f, 0.f, 0.f};
    if (a.ng > 1) {
      const int my = (4 * r) / (kD / a.ng);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < a.ng) gsum[k] = warp_sum(k == my ? own : 0.f);
    }
    if (lane == 0) {
      float4 qs4 = make_float4(sigma * (kInvSqrtD * kLog2e), sum * (kInvSqrtD * kLog2e), sigma, sum);
      *reinterpret_cast<float4*>(a.qscale + bh * kQsStride) = qs4;
      *reinterpret_cast<float4*>(a.qscale + bh * kQsStride + 4) =
          make_float4(gsum[0] * (kInvSqrtD * kLog2e), gsum[1] * (kInvSqrtD * kLog2e), gsum[2] * (kInvSqrtD * kLog2e),
                      gsum[3] * (kInvSqrtD * kLog2e));
    }
  }
}

__global__ void __launch_bounds__(kPrepThreads) qrot_kernel(DecodeArgs a) {
  grid_dep_launch();  // the split-K kernel may start its partition and first copies now
  qrot_cta(a, blockIdx.x);
}

// One launch for the start of a decode step: CTAs [0, n_app) append the
// step's new tokens (one 32-token tile of one (KV head, K|V) each), the rest
// rotate the queries.  The two halves touch disjoint data.
__global__ void __launch_bounds__(kPrepThreads) step_prep_kernel(AppendArgs aa, int T, int n_tiles, DecodeArgs a) {
  grid_dep_launch();
  const int n_app = n_tiles * aa.hkv * 2;
  const int x = blockIdx.x;
  if (x < n_app) {
    append_tile<false>(aa, T, x % n_tiles, (x / n_tiles) % aa.hkv, x / (n_tiles * aa.hkv));
  } else {
    qrot_cta(a, x - n_app);
  }
}

// ---------------------------------------------------------------------------
// Kernel 2 (SIMT fallback, for head groupings the tensor-core kernel does not
// cover): 4 warps per CTA; a warp takes whole 16-token chunks (an INT2 block,
// or 16 window rows) of one KV head and keeps its own online-softmax state;
// warps merge through shared memory.  Lane l scores token l/2 over channels
// 64*(l&1)..+63 and accumulates output channels 4l..4l+3.
// ---------------------------------------------------------------------------
constexpr int kDecWarps = 4;

template <int G>
struct WarpState {
  float m[G], l[G], o[G][4];
};

// kWindow: fp16 rows of positions first_row + t of krow0 / vrow0: the window
// ring (kRing, row = position % W) or the sink rows (row = position);
// otherwise the INT2 block at blockp.
template <int G, bool kWindow, bool kRing = true>
__device__ __forceinline__ void simt_chunk(const DecodeArgs& a, const float* qs /*smem [G][128]*/,
                                           const uint8_t* blockp, const __half* krow0,
                                           const __half* vrow0, int win_first_row, int ntok,
                                           WarpState<G>& st, int lane) {
  const int tt = lane >> 1, half = lane & 1;
  const bool valid = tt < ntok;
  float sc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) sc[g] = 0.f;
  if (valid) {
    if constexpr (!kWindow) {
      const uint4 w = *reinterpret_cast<const uint4*>(blockp + kKcOff + tt * 32 + 16 * half);
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        // channels 64 half + 16 wi .. + 15: group (4 half + wi) ng / 8
        const uint32_t smk =
            *reinterpret_cast<const uint32_t*>(blockp + sm_offset(a.ng, 0, tt, (4 * half + wi) * a.ng / 8));
        const float s = __half2float(__ushort_as_half((unsigned short)(smk & 0xffff)));
        const float m = __half2float(__ushort_as_half((unsigned short)(smk >> 16)));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int c = 64 * half + 16 * wi + j;
          const float x = fmaf(s, (float)((words[wi] >> (2 * j)) & 3u), m);
#pragma unroll
          for (int g = 0; g < G; ++g) sc[g] = fmaf(qs[g * kD + c], x, sc[g]);
        }
      }
    } else {
      const int row = kRing ? (win_first_row + tt) % kWin : win_first_row + tt;
      const __half* kr = krow0 + (size_t)row * kD + 64 * half;
#pragma unroll 4
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 w = *reinterpret_cast<const uint4*>(kr + 8 * c8);
        const __half2* hp = reinterpret_cast<const __half2*>(&w);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(hp[j]);
          const int c = 64 * half + 8 * c8 + 2 * j;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            sc[g] = fmaf(qs[g * kD + c], f.x, sc[g]);
            sc[g] = fmaf(qs[g * kD + c + 1], f.y, sc[g]);
          }
        }
      }
    }
  }
  float p[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float v = sc[g] + __shfl_xor_sync(0xffffffffu, sc[g], 1);
    v = valid ? v * (kInvSqrtD * kLog2e) : -INFINITY;
    const float cmax = warp_max(v);
    const float mnew = fmaxf(st.m[g], cmax);
    const float alpha = (st.m[g] == -INFINITY) ? 0.f : exp2f(st.m[g] - mnew);
    p[g] = valid ? exp2f(v - mnew) : 0.f;
    const float psum = warp_sum(half ? 0.f : p[g]);
    st.l[g] = st.l[g] * alpha + psum;
    st.m[g] = mnew;
#pragma unroll
    for (int j = 0; j < 4; ++j) st.o[g][j] *= alpha;
  }
  // P V: lane owns channels 4*lane .. 4*lane+3
  for (int t = 0; t < ntok; ++t) {
    float x[4];
    if constexpr (!kWindow) {
      const uint32_t byte = blockp[v_code_offset(t, lane)];
      const uint32_t smv = *reinterpret_cast<const uint32_t*>(blockp + sm_offset(a.ng, 1, t, lane * a.ng / 32));
      const float s = __half2float(__ushort_as_half((unsigned short)(smv & 0xffff)));
      const float m = __half2float(__ushort_as_half((unsigned short)(smv >> 16)));
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = fmaf(s, (float)((byte >> (2 * j)) & 3u), m);
    } else {
      const int row = kRing ? (win_first_row + t) % kWin : win_first_row + t;
      const uint2 w = *reinterpret_cast<const uint2*>(vrow0 + (size_t)row * kD + 4 * lane);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
      x[0] = f0.x;
      x[1] = f0.y;
      x[2] = f1.x;
      x[3] = f1.y;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float pt = __shfl_sync(0xffffffffu, p[g], 2 * t);
#pragma unroll
      for (int j = 0; j < 4; ++j) st.o[g][j] = fmaf(pt, x[j], st.o[g][j]);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kDecWarps * 32) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ float smem[];
  float* qs = smem;                               // [G][128]
  float* mo = qs + G * kD;                        // [warps][G][128]
  float* ml = mo + kDecWarps * G * kD;            // [warps][G][2]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long total = a.prefix[a.batch];
  if (total == 0) return;
  const int nc = working_ctas(a, total);
  const int c = blockIdx.x;
  if (c >= nc) return;
  const long long start = (long long)c * total / nc;
  const long long end = (long long)(c + 1) * total / nc;
  int lo = 0, hi = a.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.prefix[mid] <= start) lo = mid; else hi = mid - 1;
  }
  for (int b = lo; b < a.batch && a.prefix[b] < end; ++b) {
    const UnitShape us = unit_shape(clamp_len(a.context_lens, b, a.mbps, a.status, false), a.nsink);
    if (us.cost == 0) continue;
    const int slot = a.seq_slot[b];
    const bool slot_ok = slot >= 0 && slot < a.num_slots;
    const long long pu = a.prefix[b];
    const int l0 = (int)(max(start, pu) - pu), l1 = (int)(min(end, pu + us.cost) - pu);
    for (int hk = 0; hk < a.hkv; ++hk) {
      __syncthreads();
      for (int i = threadIdx.x; i < G * kD; i += blockDim.x)
        qs[i] = a.qrot[((size_t)b * a.hq + hk * G) * kD + i];
      __syncthreads();
      WarpState<G> st;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        st.m[gg] = -INFINITY;
        st.l[gg] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) st.o[gg][j] = 0.f;
      }
      if (slot_ok) {
        {
          const __half* kbase = a.ring + (((size_t)slot * a.hkv + hk) * 2 + 0) * kWin * kD;
          const __half* vbase = a.ring + (((size_t)slot * a.hkv + hk) * 2 + 1) * kWin * kD;
          const __half* ksink = a.sink + (((size_t)slot * a.hkv + hk) * 2 + 0) * a.nsink * kD;
          const __half* vsink = a.sink + (((size_t)slot * a.hkv + hk) * 2 + 1) * a.nsink * kD;
          const int ci0 = (l0 + kWinCost - 1) / kWinCost;
          const int ci1 = min(us.n_wchunk + us.n_schunk, (l1 + kWinCost - 1) / kWinCost);
          for (int ci = ci0 + warp; ci < ci1; ci += kDecWarps) {
            if (ci < us.n_wchunk) {  // window positions win_first + 16 ci .. at ring rows pos % W
              const int ntok = min(kBlock, us.n_win - ci * kBlock);
              simt_chunk<G, true>(a, qs, nullptr, kbase, vbase, us.win_first + ci * kBlock, ntok, st, lane);
            } else {  // sink positions 16 (ci - n_wchunk) .. at sink rows pos
              const int f = (ci - us.n_wchunk) * kBlock;
              simt_chunk<G, true, false>(a, qs, nullptr, ksink, vsink, f, min(kBlock, us.n_sink - f), st, lane);
            }
          }
        }
        const int p0 = max(l0, us.win_cost) - us.win_cost;
        const int p1 = l1 - us.win_cost;
        for (int pi = p0 + warp; pi < p1; pi += kDecWarps) {
          const int blk = a.block_table[(size_t)slot * a.mbps + (a.nsink >> 4) + pi];
          if (blk < 0 || blk >= a.num_blocks) {
            if (lane == 0) raise_flag(a.status, OKV_DEV_BAD_BLOCK);
            continue;
          }
          const uint8_t* bp = a.pages + ((size_t)blk * a.hkv + hk) * block_head_bytes(a.ng);
          const int ntok = min(kBlock, us.n_int2 - pi * kBlock);
          simt_chunk<G, false>(a, qs, bp, nullptr, nullptr, 0, ntok, st, lane);
        }
      } else if (lane == 0 && warp == 0) {
        raise_flag(a.status, OKV_DEV_BAD_SLOT);
      }
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mo[(warp * G + gg) * kD + 4 * lane + j] = st.o[gg][j];
        if (lane == 0) {
          ml[(warp * G + gg) * 2 + 0] = st.m[gg];
          ml[(warp * G + gg) * 2 + 1] = st.l[gg];
        }
      }
      __syncthreads();
      float* dst = a.part + ((size_t)(c + b) * a.hq + (size_t)hk * G) * kPartStride;
      for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
        const int gg = i / kD, ch = i % kD;
        float mx = -INFINITY;
        for (int w = 0; w < kDecWarps; ++w) mx = fmaxf(mx, ml[(w * G + gg) * 2]);
        float o = 0.f, l = 0.f;
        if (mx != -INFINITY) {
          for (int w = 0; w < kDecWarps; ++w) {
            const float mw = ml[(w * G + gg) * 2];
            const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - mx);
            o = fmaf(mo[(w * G + gg) * kD + ch], sc, o);
            l = fmaf(ml[(w * G + gg) * 2 + 1], sc, l);
          }
        }
        dst[gg * kPartStride + ch] = o;
        if (ch == 0) {
          dst[gg * kPartStride + 128] = mx;
          dst[gg * kPartStride + 129] = l;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 2 (tensor cores): split-K attention for G = Hq/Hkv in {1, 2, 4, 8}
// and Hkv in {1, 2, 4, 8}.
//
// A CTA of 8 warps streams a range of blocks of one sequence for every KV
// head at once: every block is one contiguous run of Hkv x 1152 bytes, fetched
// by a single bulk copy into a 6-stage CTA ring (16 block-heads per stage,
// full/empty mbarriers; warp 0 refills two stages at a time, one lane per
// block, so that its own arithmetic is delayed by the refill latency only on
// every other step; every warp copies its share of a stage to registers and
// releases the stage before computing on it).  Warp w serves KV head w % Hkv and, per stage, two
// of its blocks.
// Per 2-block step a warp computes:
//   scores  S[32 tok x 4NT heads] = C_K (u8 codes) . Q (two s8 limbs) on
//           mma.m16n8k32, then s_t * sigma * raw + m_t * sum(q~);
//   values  O[128 ch x heads] += C_V . P', P' = round(p * s_t * lam_h) as two
//           u8 limbs, exact in int32, flushed to fp32 only when the running
//           max, the scale cap or a head's P' scale moves (or every 96 steps);
//   plus sum(p * (m_t + 1.5 s_t)) for the value minimum term.
// P' precision.  lam_h = lam0 * 2^k_h per query head.  lam0 = 65535 /
// (4 s_cap), with s_cap twice the largest value scale seen, keeps P' < 2^16
// by construction (p <= 4); k_h = 0 is the normal state.  A head whose
// largest P' stays below 2^6 for 4 steps in a row -- its tokens all sit far
// below an earlier dominant token, a sink or retrieval token with a long
// flat tail -- is flushed and boosted: k_h is set so that the last step's
// largest P' lands in [2^13, 2^14).  A boosted head whose P' would pass 16
// bits is flushed and returns to k_h = 0 before anything is stored.  A run
// of 4 low steps is rare where logits are merely spread out (single low steps
// are not), so the boost costs nothing there.  The codes are also centred:
// the 3/2 s_t part of each value goes with m_t into the fp32 sum above, and
// every flush takes 3/2 inv_h sum P' back out of that sum, so the rounding
// errors of P' meet zero-mean code offsets and do not add up over a long
// range of tokens.
// Fragment facts (PTX m16n8k32, 8-bit): lane (g = lane/4, t = lane%4) holds
// A rows g and g+8 with K-columns 4t..4t+3 and 16+4t..16+4t+3; B K-rows
// 4t..4t+3 and 16+4t..+3 of column g; D rows g, g+8, columns 2t, 2t+1.
//   K side: the 32 code bytes of a token row are the contraction; a lane
//   reads 8 of them and (w >> 2s) & 0x03030303 is one A register.  Which
//   channel sits in which K-column is absorbed by the query-limb layout.
//   V side: one 16-byte chunk per lane holds 4 tokens x 16 channels; field f
//   of word j is channel 16g + 4j + f, which is an output row, so the codes
//   are only masked (w & (3 << 2f)), leaving a known 4^f factor per output
//   row that the flush removes.
// The fp16 window (at most 128 tokens) is attended in ring order (softmax
// attention does not depend on token order), 16 rows per chunk: scores and
// P.V on mma.m16n8k16 (f16 in, f32 accumulate; query and probabilities as
// fp16 hi+lo pairs), folded into the warp's state in registers.
// ---------------------------------------------------------------------------
constexpr int kHW = 8;                             // warps per CTA
constexpr int kHStages = 6;                        // ring stages
constexpr int kIssueBatch = 2;                     // stages the producer issues at a time
static_assert(kHStages % kIssueBatch == 0 && (kIssueBatch == 1 || kIssueBatch == 2),
              "a batch of up to 16-block stages must start at a multiple of its size and fit one 32-block window");
constexpr int kSlotsPerStage = 16;                 // block-heads per stage
constexpr int kPStride = 40;                       // u16 per head row of the P' tile
constexpr int kWarpScratch = 9216;                 // ring bytes each warp may use as window scratch
constexpr uint32_t kM2 = 0x03030303u;
constexpr float kMaxSlack = 2.f;  // log2 units a score may exceed the reference max without a rescale
// P' = round(x) comes out of one FFMA: bits(x + 1.5 * 2^23) = kMagicBits + round(x)
// for 0 <= x < 2^22, and the bits grow with x beyond that.
constexpr float kMagic = 12582912.f;
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr uint32_t kPLowBits = kMagicBits + 64u;     // a head's step maximum below 2^6 is "low"
constexpr uint32_t kPHighBits = kMagicBits + 65535u; // above 16 bits: back to k_h = 0 before storing
constexpr int kLowRun = 4;                           // low steps in a row that boost a head
constexpr int kBoostExp = 13;                        // a boost puts the step maximum in [2^13, 2^14)
constexpr int kMaxBoost = 60;                        // k_h <= 60 (lam0 * 2^60 stays finite)
constexpr float kPSlack = 4.f;                       // = 2^kMaxSlack

__device__ __forceinline__ float pow2f(int k) { return __int_as_float((127 + k) << 23); }  // -126 <= k <= 127

// G query heads per KV head; NGQ quantisation groups per vector (1, or 2 / 4
// for 64- / 32-channel groups, with G <= 4)
template <int G, int NGQ>
struct HCfg {
  static constexpr int NT = G <= 4 ? 1 : G / 4;  // n-tiles of 8 columns = 4 heads x 2 limbs
  static constexpr int HP = 4 * NT;              // heads incl. padding
  static constexpr int BHB = 1024 + 128 * NGQ;   // bytes per block-head
  static constexpr int stage_bytes = kSlotsPerStage * BHB;
  // (a 10-stage ring for the one-CTA-per-SM G = 8 kernel, and a 4-stage one
  // for G = 4, measured the same as 6: the kernel is bound by its per-step
  // arithmetic, not by the bytes in flight.  The grouped layouts' larger
  // stages take 4, so that two CTAs still share an SM.)
  static constexpr int NS = NGQ == 1 ? kHStages : 4;
  static constexpr size_t ring_bytes = (size_t)NS * stage_bytes;
  // fp32 o' accumulators live in tensor memory: thread (warp w, lane l) owns
  // TMEM lane 32 (w % 4) + l, columns 16 NT (w / 4) .. +16 NT
  static constexpr uint32_t tmem_cols = 32u * NT;
  static constexpr size_t smem_bytes() {
    return ring_bytes                            // ring (reused for window scratch and merging)
           + (size_t)2 * NS * 8                  // full / empty mbarriers
           + 16                                  // TMEM base address
           + (size_t)NS * kSlotsPerStage         // tokens per block slot
           + (size_t)kHW * NGQ * HP * kPStride * 2  // P' tiles (one per quantisation group)
           + (size_t)kHW * G * 2 * 4;            // merge (m, l)
  }
};
static_assert(kHW * 8 * kD * 4 <= HCfg<4, 1>::ring_bytes && kHW * 8 * kD * 4 <= HCfg<4, 2>::ring_bytes &&
                  kHW * 8 * kD * 4 <= HCfg<4, 4>::ring_bytes,
              "merge buffer must fit the ring");
static_assert(HCfg<4, 1>::ring_bytes / kHW >= kWarpScratch && HCfg<4, 2>::ring_bytes / kHW >= kWarpScratch &&
                  HCfg<4, 4>::ring_bytes / kHW >= kWarpScratch,
              "window scratch per warp");
static_assert(HCfg<4, 2>::NS % kIssueBatch == 0 && HCfg<4, 4>::NS % kIssueBatch == 0,
              "producer batches start at multiples of their size");
static_assert(4096 + 8 * 64 + 8 * kD * 4 <= kWarpScratch, "window scratch must fit a warp's share of the ring");

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A . B with a zero accumulator
__device__ __forceinline__ void mma_u8s8_z(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

template <int G, int NGQ>
struct MmaWarpState {
  static constexpr int NT = HCfg<G, NGQ>::NT;
  float m[NT];
  float2 l[NT], msum[NT][NGQ];  // two partial sums each (paired fp32 arithmetic); the value is .x + .y
  uint32_t tacc;  // TMEM address of fp32 o' for channels 16g + 0..15 of head 4nt + t at column 16 nt + i
};

// warp-collective: 8 fp32 accumulators of every lane from / to tensor memory
__device__ __forceinline__ void tacc_load8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tacc_store8(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tacc_load(uint32_t taddr, float (&v)[16]) {
  tacc_load8(taddr, v);
  tacc_load8(taddr + 8u, v + 8);
}

__device__ __forceinline__ void tacc_store(uint32_t taddr, const float (&v)[16]) {
  tacc_store8(taddr, v);
  tacc_store8(taddr + 8u, v + 8);
}

// acci[mt] holds two output channels of the lane's head (regs 0,1 = hi, lo
// limb of the first, regs 2,3 of the second), which come from code fields
// f = 2(mt&1) and f + 1, so that the unshifted masks scaled them by 4^f.  They
// land in TMEM columns 2mt and 2mt + 1 of the lane: column i holds channel
// chan_base(g, i / 4) + i % 4.  With one group per vector, m-tile mt covers
// channels 16g + 2mt, + 1 of every lane group g; with smaller groups the lanes
// load their value codes so that every m-tile lies in one quantisation group
// (group mt / (8 / NGQ)), whose P' it multiplies.
// acci: exact int32 sums of P' c 4^f since the last flush; psum: this lane's
// sum of P' per group over the same steps (wrapping modulo 2^32, which the
// plain sum never reaches).
// Flush: o' = (o' + inv * sum P' c) * rescale in tensor memory
// (warp-collective), and msum -= 3/2 inv sum P', so that together they hold
// inv * sum P' (c - 3/2) on top of the sum of p (m + 3/2 s).  The two parts
// are each rounded to fp32 before they meet; their sum is what carries the
// P' rounding errors, and there they see zero-mean code offsets.
template <int NGQ>
__device__ __forceinline__ int chan_base(int g, int q) {
  if constexpr (NGQ == 1) return 16 * g + 4 * q;
  else if constexpr (NGQ == 2) return 64 * (q >> 1) + 16 * (g & 3) + 4 * (g >> 2) + 8 * (q & 1);
  else return 32 * q + 16 * (g & 1) + 4 * (g >> 1);
}
// quantisation group of the lane's four-channel run q (TMEM columns 4q .. 4q + 3)
template <int NGQ>
__host__ __device__ constexpr int run_group(int q) {
  return NGQ == 1 ? 0 : (NGQ == 2 ? q >> 1 : q);
}

template <int G, int NGQ>
__device__ __forceinline__ void mma_flush(MmaWarpState<G, NGQ>& st, int (&acci)[HCfg<G, NGQ>::NT][8][4],
                                          uint32_t (&psum)[HCfg<G, NGQ>::NT][NGQ], int nt, float inv,
                                          float rescale = 1.f) {
#pragma unroll
  for (int k = 0; k < NGQ; ++k) {
    st.msum[nt][k].x = fmaf(-1.5f * inv, (float)psum[nt][k], st.msum[nt][k].x);
    psum[nt][k] = 0u;
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {  // two halves of 8 channels: fewer live registers
    float v[8];
    tacc_load8(st.tacc + 16u * nt + 8u * hh, v);
#pragma unroll
    for (int mq = 0; mq < 4; ++mq) {
      const int mt = 4 * hh + mq;
      const float s0 = (mt & 1) ? inv * (1.f / 16.f) : inv;  // field 0 or 2
      const float s1 = s0 * 0.25f;                            // field 1 or 3
      v[2 * mq] = (v[2 * mq] + fmaf((float)acci[nt][mt][0], 256.f * s0, (float)acci[nt][mt][1] * s0)) * rescale;
      v[2 * mq + 1] = (v[2 * mq + 1] + fmaf((float)acci[nt][mt][2], 256.f * s1, (float)acci[nt][mt][3] * s1)) * rescale;
#pragma unroll
      for (int j = 0; j < 4; ++j) acci[nt][mt][j] = 0;
    }
    tacc_store8(st.tacc + 16u * nt + 8u * hh, v);
  }
}

template <int G, int NGQ, int HS = 1>
__global__ void __launch_bounds__(kHW * 32, (G <= 4) ? 2 : 1) decode_heads_kernel(DecodeArgs a) {
  using Cfg = HCfg<G, NGQ>;
  static_assert(NGQ == 1 || G <= 4, "grouped layouts take G <= 4 (one n-tile)");
  constexpr int NT = Cfg::NT, HP = Cfg::HP;
  constexpr int kHStages = Cfg::NS;  // ring stages of this instantiation
  constexpr int kStageBytes = Cfg::stage_bytes, BHB = Cfg::BHB;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int btq[2][32];  // producer's block ids, two 32-block windows
  unsigned char* ring = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + Cfg::ring_bytes);
  uint64_t* empty = full + kHStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(empty + kHStages);          // TMEM base (16 B)
  uint8_t* ntok = reinterpret_cast<uint8_t*>(tmem_slot + 4);                    // [S][16]
  uint16_t* pst = reinterpret_cast<uint16_t*>(ntok + kHStages * kSlotsPerStage);  // [8][NGQ][HP][40]
  float* ml = reinterpret_cast<float*>(pst + kHW * NGQ * HP * kPStride);        // [8][G][2]
  float* mo = reinterpret_cast<float*>(ring);  // [8][G][128], only while the ring is idle

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int hkv = a.hkv;                 // 1, 2, 4 or 8
  const int wph = kHW / hkv;             // warps per KV head
  const int head = warp % hkv, grp = warp / hkv;
  const int nb = 2 * wph;                // blocks per stage
  const uint32_t copy_bytes = (uint32_t)hkv * BHB;
  grid_dep_launch();  // the combine kernel may take SMs as split-K CTAs finish
  // With HS > 1 the grid holds HS CTAs per cost range: CTA range + a.nc hh
  // serves query heads G hh .. G hh + G - 1 of every KV head (G here is the
  // query heads one CTA takes; a KV head has G HS).  The CTAs of a range
  // stream the same blocks, the later ones mostly from L2.  (Built for the
  // grouped layouts at G = 8; one group per vector takes G = 8 in one CTA.)
  // first query head this CTA serves of KV head h (recomputed where used: fewer live registers)
  auto qhead0 = [&](int h) { return HS == 1 ? h * G : h * G * HS + G * ((int)blockIdx.x / a.nc); };

  // The work partition, computed here from the context lengths with loads that
  // bypass L1, so that this kernel can start (and put its first copies in
  // flight) while the query rotation is still running.  Thread i sums the costs
  // of a chunk of consecutive entries; a block-wide scan gives the total and
  // the entry holding this CTA's first cost position.
  __shared__ int part_tot[kHW], part_first[2];
  int total;
  {
    const int per = (a.batch + blockDim.x - 1) / blockDim.x;
    const int i0 = threadIdx.x * per, i1 = min(a.batch, i0 + per);
    int own = 0;
    for (int i = i0; i < i1; ++i) own += unit_shape(clamp_len_cg(a.context_lens, i, a.mbps), a.nsink).cost;
    int inc = own;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += v;
    }
    if (lane == 31) part_tot[warp] = inc;
    __syncthreads();
    int before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kHW; ++w) {
      before += w < warp ? part_tot[w] : 0;
      total += part_tot[w];
    }
    before += inc - own;
    if (total > 0) {
      const int ncw = (int)min((long long)a.nc, (long long)total);
      const int cr = HS == 1 ? (int)blockIdx.x : (int)blockIdx.x % a.nc;  // cost range
      const long long st0 = (long long)cr * total / ncw;
      if (cr < ncw && st0 >= before && st0 < before + own) {
        int pu = before;
        for (int i = i0; i < i1; ++i) {
          const int cst = unit_shape(clamp_len_cg(a.context_lens, i, a.mbps), a.nsink).cost;
          if (st0 < pu + cst) {
            part_first[0] = i;
            part_first[1] = pu;
            break;
          }
          pu += cst;
        }
      }
    }
    __syncthreads();
  }
  const int nc = (int)min((long long)a.nc, (long long)total);
  // cost range of this CTA (recomputed where used, like qhead0)
  auto crange = [&]() -> int { return HS == 1 ? (int)blockIdx.x : (int)blockIdx.x % a.nc; };
  const int c = crange();
  if (total == 0 || c >= nc) {
    grid_dep_wait();  // no CTA finishes before the query rotation has
    return;
  }
  const long long start = (long long)c * total / nc;
  const long long end = (long long)(c + 1) * total / nc;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kHStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kHW);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  uint16_t* myp = pst + warp * NGQ * HP * kPStride;  // P' tile of group k at myp + k HP kPStride
  uint32_t it = 0;    // CTA ring position (continues across batch entries)
  bool alive = true;  // cleared if a wait never completes

  bool waited = false;  // grid_dep_wait() done (the query rotation's outputs are readable)
  long long pnext = part_first[1];
  for (int b = part_first[0]; b < a.batch && pnext < end; ++b) {
    const UnitShape us = unit_shape(clamp_len_cg(a.context_lens, b, a.mbps), a.nsink);
    const long long pu = pnext;
    pnext += us.cost;
    if (us.cost == 0) continue;
    const int slot = __ldcg(a.seq_slot + b);
    const bool slot_ok = slot >= 0 && slot < a.num_slots;
    const int l0 = (int)(max(start, pu) - pu), l1 = (int)(min(end, pu + us.cost) - pu);
    const size_t bh0 = (size_t)b * a.hq + (size_t)qhead0(head);  // first query head served
    __syncthreads();  // the previous entry's window scratch / merge buffers (on the ring) are free again
    if (!slot_ok && threadIdx.x == 0) raise_flag(a.status, OKV_DEV_BAD_SLOT);

    // ---------------- INT2 blocks through the ring ----------------
    const int p0 = max(l0, us.win_cost) - us.win_cost;
    const int p1 = l1 - us.win_cost;
    const int nst = (slot_ok && alive && p1 > p0) ? (p1 - p0 + nb - 1) / nb : 0;
    // INT2 block pi of this entry is table column nsink/16 + pi
    const int32_t* trow = a.block_table + (size_t)(slot_ok ? slot : 0) * a.mbps + (a.nsink >> 4);

    // Warp 0 fills the ring in batches of stages, one lane per block (lane
    // nb * i + q takes block q of the batch's stage i).  Stage j of this entry
    // sits at ring position it + j, slot (it + j) % kHStages.  Block ids come
    // from a two-window shared buffer that async copies fill one 32-block
    // window ahead (btq[bt_buf] holds blocks bt_base .. bt_base + 31), so no
    // block-table load sits between a released stage and its refill.
    int bt_base = p0, bt_buf = 0;
    int issued = 0;  // stages of this entry whose copies went out (warp 0)
    auto bt_fill = [&](int wbase, int buf) {  // all lanes of warp 0
      const int pi = wbase + lane;
      if (pi < p1) cp_async4(&btq[buf][lane], trow + pi);
      else btq[buf][lane] = -1;
      cp_async_commit();
    };
    if (warp == 0 && nst > 0) {
      cp_async_wait_all();  // the previous entry's prefetch
      __syncwarp();
      btq[0][lane] = p0 + lane < p1 ? __ldcg(trow + p0 + lane) : -1;  // first window: loads that bypass L1
      __syncwarp();
      bt_fill(p0 + 32, 1);
    }
    // Stages first .. first + cnt - 1, whose blocks lie in one window.  With
    // wait_prev, their slots' previous contents (ring positions up to that of
    // stage first + cnt - 1 - kHStages) must first be released by every warp:
    // each warp releases positions in order, so one wait on the latest covers
    // the batch.  The block ids are read before that wait, so the two latencies overlap.
    auto issue_batch = [&](int first, int cnt, bool wait_prev) -> bool {  // all lanes of warp 0
      const int pj = p0 + first * nb;
      while (pj >= bt_base + 32) {
        bt_base += 32;
        bt_buf ^= 1;
        cp_async_wait_all();
        __syncwarp();
        bt_fill(bt_base + 32, bt_buf ^ 1);  // the window just retired takes the one after next
      }
      const int bi = lane / nb, q = lane - bi * nb;  // stage first + bi, block q
      const bool act = lane < cnt * nb;
      const int pi = pj + lane;
      const bool mine = act && pi < p1;
      int bid = mine ? btq[bt_buf][pj - bt_base + lane] : -1;
      if (mine && (bid < 0 || bid >= a.num_blocks)) {
        raise_flag(a.status, OKV_DEV_BAD_BLOCK);
        bid = -1;
      }
      bool ok = true;
      if (wait_prev && lane == 0) {
        const uint32_t last = it + (uint32_t)(first + cnt - 1);  // >= kHStages
        ok = mbar_wait_bounded(&empty[last % kHStages], (last / kHStages - 1u) & 1u);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
      const uint32_t s = (it + (uint32_t)(first + bi)) % kHStages;
      const uint32_t valid = __ballot_sync(0xffffffffu, bid >= 0);
      const uint32_t nvalid = __popc((valid >> (bi * nb)) & ((1u << nb) - 1u));  // lane bi * nb <= 31
      if (act) ntok[s * kSlotsPerStage + q] = bid >= 0 ? (uint8_t)min(kBlock, us.n_int2 - kBlock * pi) : 0;
      __syncwarp();
      // the barrier must expect every byte before any copy can complete on it
      if (act && q == 0) mbar_arrive_expect_tx(&full[s], nvalid * copy_bytes);
      __syncwarp();
      if (bid >= 0)
        bulk_g2s_hint(ring + s * kStageBytes + q * copy_bytes, a.pages + (size_t)bid * copy_bytes, copy_bytes,
                      &full[s], HS > 1 ? l2_evict_normal_policy() : l2_evict_first_policy());
        // (each block is read once, or once per CTA of its range)
      issued = max(issued, first + cnt);
      return true;
    };
    // Prologue: every slot (the ring is idle at an entry's start).  A batch
    // stops at a window boundary (nb divides 32).
    bool prod_ok = true;
    if (warp == 0) {
      const int npro = min(kHStages, nst);
      for (int first = 0; first < npro && prod_ok;) {
        const int cnt = min(npro - first, (32 - (first * nb) % 32) / nb);
        prod_ok = issue_batch(first, cnt, false);
        first += cnt;
      }
    }

    if (!waited) {  // from here on the query rotation's outputs are read
      grid_dep_wait();
      waited = true;
    }
    // ---------------- per-warp state for (b, head), loaded while the first stages are in flight ----------------
    MmaWarpState<G, NGQ> st;
    int acci[NT][8][4];
    st.tacc = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(16 * NT * (warp >> 2));
    uint32_t qb[NT][8];
    float ah[NT], bh[NT][NGQ], hbias[NT];  // bh: min-term scale of each quantisation group
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      st.m[nt] = -INFINITY;
      st.l[nt] = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < NGQ; ++k) st.msum[nt][k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acci[nt][mt][j] = 0;
      const int hcol = 4 * nt + (g >> 1);  // head of this lane's B column
      if (hcol < G) {
        const uint4* src = reinterpret_cast<const uint4*>(a.qlimb + ((bh0 + hcol) * 2 + (g & 1)) * kD + 32 * t);
        const uint4 x0 = src[0], x1 = src[1];
        qb[nt][0] = x0.x; qb[nt][1] = x0.y; qb[nt][2] = x0.z; qb[nt][3] = x0.w;
        qb[nt][4] = x1.x; qb[nt][5] = x1.y; qb[nt][6] = x1.z; qb[nt][7] = x1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qb[nt][i] = 0u;
      }
      const int hs = 4 * nt + t;  // head of this lane's score columns
      const bool ok = hs < G;
      ah[nt] = ok ? a.qscale[(bh0 + hs) * kQsStride + 0] : 0.f;
#pragma unroll
      for (int k = 0; k < NGQ; ++k) bh[nt][k] = ok ? a.qscale[(bh0 + hs) * kQsStride + (NGQ == 1 ? 1 : 4 + k)] : 0.f;
      hbias[nt] = ok ? 0.f : -INFINITY;
    }
    {
      float zero[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) zero[i] = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) tacc_store(st.tacc + 16u * nt, zero);
    }
    // P' scale: the warp's base lam0 (0 until a positive value scale is seen)
    // and, per head of this lane's score column, the boost k, lam = lam0 2^k,
    // inv = 1 / lam, the count of low steps in a row, and this lane's sum of
    // P' since the last flush
    float s_cap = 0.f, lam0 = 0.f;
    float lam[NT];
    int lrb[NT];  // (low steps in a row) << 8 | boost k
    uint32_t psum[NT][NGQ];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      lam[nt] = 0.f;
      lrb[nt] = 0;
#pragma unroll
      for (int k = 0; k < NGQ; ++k) psum[nt][k] = 0u;
    }
    // 1 / lam of n-tile nt (0 before any value scale was seen)
    auto inv_of = [&](int nt) { return (s_cap * (kPSlack / 65535.f)) * pow2f(-(lrb[nt] & 0xff)); };
    int since_flush = 0;


    int done = 0;
    uint32_t cs = it % kHStages, cph = (it / kHStages) & 1u;  // consumer stage and phase parity
    for (int j = 0; j < nst; ++j) {
      if (warp == 0) {
        // every kIssueBatch steps: the next kIssueBatch stages, into the slots
        // of stages j - kIssueBatch .. j - 1 (kIssueBatch * nb blocks from a
        // multiple of kIssueBatch * nb, which divides 32: inside one window)
        const int nf = j + kHStages - kIssueBatch;
        if (prod_ok && j >= kIssueBatch && j % kIssueBatch == 0 && nf < nst)
          prod_ok = issue_batch(nf, min(kIssueBatch, nst - nf), true);
        if (!prod_ok) {
          if (lane == 0) raise_flag(a.status, OKV_DEV_TIMEOUT);
          alive = false;
        }
      }
      const uint32_t s = cs, par = cph;
      if (++cs == (uint32_t)kHStages) {
        cs = 0;
        cph ^= 1u;
      }
      if (!__all_sync(0xffffffffu, alive && mbar_wait_bounded(&full[s], par))) {
        if (lane == 0) raise_flag(a.status, OKV_DEV_TIMEOUT);
        alive = false;
        break;
      }
      const int q0 = 2 * grp;
      const int n0 = ntok[s * kSlotsPerStage + q0], n1 = ntok[s * kSlotsPerStage + q0 + 1];
      auto step = [&](auto full_tag) {
        constexpr bool fullstep = decltype(full_tag)::value;
        const unsigned char* s0 = ring + s * kStageBytes + q0 * copy_bytes + head * BHB;
        const unsigned char* s1 = s0 + copy_bytes;

        // ---- what the scores and weights need from the stage goes to
        //      registers now; the value codes follow just before the value
        //      MMAs, after which the stage is released for the producer
        uint2 kw[2][2];
        uint32_t smk[4], smv[4];
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const unsigned char* sb = bb ? s1 : s0;
          kw[bb][0] = *reinterpret_cast<const uint2*>(sb + kKcOff + 32 * g + 8 * t);
          kw[bb][1] = *reinterpret_cast<const uint2*>(sb + kKcOff + 32 * (g + 8) + 8 * t);
          smk[2 * bb] = *reinterpret_cast<const uint32_t*>(sb + kKsmOff + 4 * g);
          smk[2 * bb + 1] = *reinterpret_cast<const uint32_t*>(sb + kKsmOff + 4 * (g + 8));
          smv[2 * bb] = *reinterpret_cast<const uint32_t*>(sb + kVsmOff + 4 * g);
          smv[2 * bb + 1] = *reinterpret_cast<const uint32_t*>(sb + kVsmOff + 4 * (g + 8));
        }

        // ---- scores: D[tok][col] for both blocks
        int dq[2][NT][4];
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const uint2 wa = kw[bb][0], wb = kw[bb][1];
#pragma unroll
          for (int sf = 0; sf < 4; ++sf) {
            uint32_t af[4];
            af[0] = (wa.x >> (2 * sf)) & kM2;
            af[1] = (wb.x >> (2 * sf)) & kM2;
            af[2] = (wa.y >> (2 * sf)) & kM2;
            af[3] = (wb.y >> (2 * sf)) & kM2;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (sf == 0) mma_u8s8_z(dq[bb][nt], af, qb[nt][0], qb[nt][1]);
              else mma_u8s8(dq[bb][nt], af, qb[nt][2 * sf], qb[nt][2 * sf + 1]);
            }
          }
        }
        // token e of this lane: block e>>1, row g + 8*(e&1)
        float sk[4], mk[4], sv[4], mc[4];
        bool tv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 k2 = __half22float2(*reinterpret_cast<const __half2*>(&smk[e]));
          const float2 v2 = __half22float2(*reinterpret_cast<const __half2*>(&smv[e]));
          tv[e] = fullstep || ((g + 8 * (e & 1)) < ((e >> 1) ? n1 : n0));
          // masked slots may hold any bits (a slot whose block was not fetched
          // keeps stale shared memory): select, never multiply, them away
          sk[e] = k2.x; mk[e] = k2.y;
          sv[e] = tv[e] ? v2.x : 0.f;
          mc[e] = tv[e] ? fmaf(1.5f, v2.x, v2.y) : 0.f;  // m + 3/2 s: the codes are centred in the flush
        }
        float smax = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        if (__any_sync(0xffffffffu, smax > s_cap)) {  // rare: raise the scale cap, flushing every head first
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 4));
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 8));
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 16));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_flush(st, acci, psum, nt, inv_of(nt));
          since_flush = 0;
          // headroom: the cap jumps to twice the new maximum, and P' leaves room
          // for p up to 2^kMaxSlack, so later small increases cost nothing
          s_cap = 2.f * smax;
          lam0 = 65535.f / (s_cap * kPSlack);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) lam[nt] = lam0 * pow2f(lrb[nt] & 0xff);
        }
        // tokens in pairs (e = 0, 1: block 0; e = 2, 3: block 1) for the
        // paired fp32 instructions
        const float2 sk01 = make_float2(sk[0], sk[1]), sk23 = make_float2(sk[2], sk[3]);
        const float2 mk01 = make_float2(mk[0], mk[1]), mk23 = make_float2(mk[2], mk[3]);
        const float2 sv01 = make_float2(sv[0], sv[1]), sv23 = make_float2(sv[2], sv[3]);
        const float2 mc01 = make_float2(mc[0], mc[1]), mc23 = make_float2(mc[2], mc[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          // x = s sigma' raw + m sum' (log2 units), taken relative to the
          // running max mref straight away: x' = x - mref
          const float mref0 = st.m[nt] == -INFINITY ? 0.f : st.m[nt];
          const float2 ah2 = make_float2(ah[nt], ah[nt]), bh2 = make_float2(bh[nt][0], bh[nt][0]);
          const float2 c2 = make_float2(hbias[nt] - mref0, hbias[nt] - mref0);  // hbias: -inf on padded heads
          const float2 raw01 = make_float2((float)(dq[0][nt][0] * 256 + dq[0][nt][1]),
                                           (float)(dq[0][nt][2] * 256 + dq[0][nt][3]));
          const float2 raw23 = make_float2((float)(dq[1][nt][0] * 256 + dq[1][nt][1]),
                                           (float)(dq[1][nt][2] * 256 + dq[1][nt][3]));
          float2 x01 = __ffma2_rn(__fmul2_rn(sk01, ah2), raw01, __ffma2_rn(mk01, bh2, c2));
          float2 x23 = __ffma2_rn(__fmul2_rn(sk23, ah2), raw23, __ffma2_rn(mk23, bh2, c2));
          if constexpr (!fullstep) {
            x01.x = tv[0] ? x01.x : -INFINITY;
            x01.y = tv[1] ? x01.y : -INFINITY;
            x23.x = tv[2] ? x23.x : -INFINITY;
            x23.y = tv[3] ? x23.y : -INFINITY;
          }
          // The reference max moves only when a score passes it by more than
          // kMaxSlack (log2 units): p <= 2^kMaxSlack, which P' has room for.
          float bm = fmaxf(fmaxf(x01.x, x01.y), fmaxf(x23.x, x23.y));  // relative to mref0
          if (__any_sync(0xffffffffu, bm > (st.m[nt] == -INFINITY ? -INFINITY : kMaxSlack))) {
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            // the whole warp flushes (the accumulators are read and written
            // warp-collectively); heads whose max did not move keep scale 1
            const float mnew = bm + mref0;
            const bool need = mnew > st.m[nt] + kMaxSlack;
            const float alpha = need ? fast_ex2(st.m[nt] - mnew) : 1.f;  // ex2(-inf) = 0 on the first step
            mma_flush(st, acci, psum, nt, inv_of(nt), alpha);
            if (need) {
              const float2 a2 = make_float2(alpha, alpha), d2 = make_float2(-bm, -bm);
              st.l[nt] = __fmul2_rn(st.l[nt], a2);
              st.msum[nt][0] = __fmul2_rn(st.msum[nt][0], a2);
              st.m[nt] = mnew;
              x01 = __fadd2_rn(x01, d2);  // now relative to the new max
              x23 = __fadd2_rn(x23, d2);
            }
          }
          const float2 p01 = make_float2(fast_ex2(x01.x), fast_ex2(x01.y));  // 0 for masked tokens
          const float2 p23 = make_float2(fast_ex2(x23.x), fast_ex2(x23.y));
          st.l[nt] = __fadd2_rn(st.l[nt], __fadd2_rn(p01, p23));
          st.msum[nt][0] = __ffma2_rn(p23, mc23, __ffma2_rn(p01, mc01, st.msum[nt][0]));
          // kMagicBits + round(p s lam)
          const float2 lam2 = make_float2(lam[nt], lam[nt]), mg2 = make_float2(kMagic, kMagic);
          float2 u01 = __ffma2_rn(p01, __fmul2_rn(sv01, lam2), mg2);
          float2 u23 = __ffma2_rn(p23, __fmul2_rn(sv23, lam2), mg2);
          uint32_t u[4] = {__float_as_uint(u01.x), __float_as_uint(u01.y), __float_as_uint(u23.x),
                           __float_as_uint(u23.y)};
          // A head whose largest P' stays below 2^6 for kLowRun steps is
          // boosted; a boosted head whose P' would pass 16 bits drops back to
          // k = 0.  Either way this n-tile is flushed first.
          const uint32_t um = max(max(u[0], u[1]), max(u[2], u[3]));
          const uint32_t big = __ballot_sync(0xffffffffu, um >= kPLowBits);
          // low steps in a row, the same in the head's 8 lanes
          lrb[nt] = ((big >> t) & 0x11111111u) == 0u ? lrb[nt] + 256 : (lrb[nt] & 0xff);
          const bool raise = (4 * nt + t < G) && lrb[nt] >= (kLowRun << 8) && (lrb[nt] & 0xff) < kMaxBoost;
          if (__any_sync(0xffffffffu, um > kPHighBits || raise)) {
            uint32_t uh = um;  // the head's step maximum (lanes of the same t)
            uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 4));
            uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 8));
            uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 16));
            const float2 y01 = __fmul2_rn(p01, sv01), y23 = __fmul2_rn(p23, sv23);  // p * s
            float ym = fmaxf(fmaxf(y01.x, y01.y), fmaxf(y23.x, y23.y));
            ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 4));
            ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 8));
            ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 16));
            mma_flush(st, acci, psum, nt, inv_of(nt));
            int k = lrb[nt] & 0xff;
            if (uh > kPHighBits) {
              k = 0;
            } else if (raise) {
              // 2^k with ym * lam0 * 2^k in [2^13, 2^14): k = 13 - floor(log2(ym * lam0))
              const float y = ym * lam0;
              const int ex = ((__float_as_int(y) >> 23) & 0xff) - 127;
              if (y > 0.f) k = max(0, min(kMaxBoost, kBoostExp - ex));
            }
            lrb[nt] = (uh > kPHighBits || raise) ? k : (lrb[nt] & ~0xff) | k;
            lam[nt] = lam0 * pow2f(k);
            const float2 l2 = make_float2(lam[nt], lam[nt]);
            u01 = __ffma2_rn(y01, l2, mg2);
            u23 = __ffma2_rn(y23, l2, mg2);
            u[0] = __float_as_uint(u01.x);
            u[1] = __float_as_uint(u01.y);
            u[2] = __float_as_uint(u23.x);
            u[3] = __float_as_uint(u23.y);
          }
          uint16_t* prow = myp + (4 * nt + t) * kPStride;
#pragma unroll
          for (int e = 0; e < 4; ++e) prow[16 * (e >> 1) + g + 8 * (e & 1)] = (uint16_t)u[e];  // P' < 2^16
          psum[nt][0] += (u[0] + u[1]) + (u[2] + u[3]) - 4u * kMagicBits;
        }
        const uint4 v0 = *reinterpret_cast<const uint4*>(s0 + kVcOff + 16 * lane);
        const uint4 v1 = *reinterpret_cast<const uint4*>(s1 + kVcOff + 16 * lane);
        __syncwarp();  // every lane has its value codes (and its P' row is written)
        if (lane == 0) mbar_arrive(&empty[s]);
        // ---- values: acci[mt] += C_V (masked, row scale 4^f) . P'
        const uint32_t va[4] = {v0.x, v0.y, v0.z, v0.w};
        const uint32_t vb[4] = {v1.x, v1.y, v1.z, v1.w};
        uint32_t pb0[NT], pb1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint16_t* prow = myp + (4 * nt + (g >> 1)) * kPStride;
          const uint2 x0 = *reinterpret_cast<const uint2*>(prow + 4 * t);
          const uint2 x1 = *reinterpret_cast<const uint2*>(prow + 16 + 4 * t);
          const uint32_t sel = (g & 1) ? 0x6420u : 0x7531u;  // odd column: low byte (lo limb)
          pb0[nt] = prmt(x0.x, x0.y, sel);
          pb1[nt] = prmt(x1.x, x1.y, sel);
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int jw = mt >> 1;
          const uint32_t m0 = kM2 << (4 * (mt & 1)), m1 = m0 << 2;
          const uint32_t af[4] = {va[jw] & m0, va[jw] & m1, vb[jw] & m0, vb[jw] & m1};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_u8u8(acci[nt][mt], af, pb0[nt], pb1[nt]);
        }
        if (++since_flush >= 96) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_flush(st, acci, psum, nt, inv_of(nt));
          since_flush = 0;
        }
      };
      // Grouped layouts (NGQ = 2 or 4 groups of 128 / NGQ channels; G <= 4,
      // one n-tile).  Scores: one MMA per (block, group, field pair) for 64-
      // channel groups, per (block, group) for 32-channel groups, each over
      // code bytes of one group only (the query limbs are stored in the
      // matching order), so that every group's raw dot product comes out
      // apart and takes its own (s, m).  Values: every m-tile lies in one
      // group and multiplies that group's P' = round(p s_tk lam).
      auto step_grouped = [&](auto full_tag) {
        constexpr bool fullstep = decltype(full_tag)::value;
        const unsigned char* s0 = ring + s * kStageBytes + q0 * copy_bytes + head * BHB;
        const unsigned char* s1 = s0 + copy_bytes;
        // token e of this lane: block e>>1, row g + 8*(e&1)
        bool tv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) tv[e] = fullstep || ((g + 8 * (e & 1)) < ((e >> 1) ? n1 : n0));
        // (scale, min) pairs of every group: K at 1024 + 4 (row NGQ + k), V at
        // 1024 + 64 NGQ + 4 (row NGQ + k).  The V pairs are read again where
        // they are used (fewer live registers).  Masked slots may hold any
        // bits (a slot whose block was not fetched keeps stale shared
        // memory): their value scales and minima read as 0.
        auto vpair = [&](int e, int k) -> uint32_t {
          const unsigned char* sb = (e >> 1) ? s1 : s0;
          const uint32_t x = *reinterpret_cast<const uint32_t*>(sb + 1024 + 64 * NGQ + 4 * ((g + 8 * (e & 1)) * NGQ + k));
          return tv[e] ? x : 0u;
        };
        __half2 hm = __float2half2_rn(0.f);  // the step's largest value scale (low halves; scales are >= 0)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const unsigned char* sb = (e >> 1) ? s1 : s0;
          const int row = g + 8 * (e & 1);
          uint32_t xv[NGQ];
          if constexpr (NGQ == 2) {
            const uint2 v2 = *reinterpret_cast<const uint2*>(sb + 1024 + 128 + 8 * row);
            xv[0] = v2.x; xv[1] = v2.y;
          } else {
            const uint4 v4 = *reinterpret_cast<const uint4*>(sb + 1024 + 256 + 16 * row);
            xv[0] = v4.x; xv[1] = v4.y; xv[2] = v4.z; xv[3] = v4.w;
          }
#pragma unroll
          for (int k = 0; k < NGQ; ++k) {
            const uint32_t x = tv[e] ? xv[k] : 0u;
            hm = __hmax2(hm, *reinterpret_cast<const __half2*>(&x));
          }
        }
        float smax = __low2float(hm);
        if (__any_sync(0xffffffffu, smax > s_cap)) {  // rare: raise the scale cap, flushing first
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 4));
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 8));
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 16));
          mma_flush(st, acci, psum, 0, inv_of(0));
          since_flush = 0;
          s_cap = 2.f * smax;
          lam0 = 65535.f / (s_cap * kPSlack);
          lam[0] = lam0 * pow2f(lrb[0] & 0xff);
        }
        // ---- scores, group by group: x = sum_k (s_tk sigma' raw_k + m_tk sum'_k), relative to mref
        const float mref0 = st.m[0] == -INFINITY ? 0.f : st.m[0];
        const float2 ah2 = make_float2(ah[0], ah[0]);
        float2 x01 = make_float2(hbias[0] - mref0, hbias[0] - mref0), x23 = x01;  // hbias: -inf on padded heads
#pragma unroll
        for (int k = 0; k < NGQ; ++k) {
          int dq[2][4];
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
            const unsigned char* kc = (bb ? s1 : s0) + kKcOff;
            if constexpr (NGQ == 2) {
              // bytes 16k + 4t .. + 3 of rows g and g + 8: field 2p at K-columns
              // 4t.., field 2p + 1 at 16 + 4t..
              const uint32_t wa = *reinterpret_cast<const uint32_t*>(kc + 32 * g + 16 * k + 4 * t);
              const uint32_t wb = *reinterpret_cast<const uint32_t*>(kc + 32 * (g + 8) + 16 * k + 4 * t);
#pragma unroll
              for (int p = 0; p < 2; ++p) {
                const uint32_t af[4] = {(wa >> (4 * p)) & kM2, (wb >> (4 * p)) & kM2, (wa >> (4 * p + 2)) & kM2,
                                        (wb >> (4 * p + 2)) & kM2};
                if (p == 0) mma_u8s8_z(dq[bb], af, qb[0][4 * k], qb[0][4 * k + 1]);
                else mma_u8s8(dq[bb], af, qb[0][4 * k + 2], qb[0][4 * k + 3]);
              }
            } else {
              // field t of bytes 8k .. 8k + 3 (K-columns 4t..) and 8k + 4 .. (16 + 4t..)
              const uint2 wa = *reinterpret_cast<const uint2*>(kc + 32 * g + 8 * k);
              const uint2 wb = *reinterpret_cast<const uint2*>(kc + 32 * (g + 8) + 8 * k);
              const int sh = 2 * t;
              const uint32_t af[4] = {(wa.x >> sh) & kM2, (wb.x >> sh) & kM2, (wa.y >> sh) & kM2, (wb.y >> sh) & kM2};
              mma_u8s8_z(dq[bb], af, qb[0][2 * k], qb[0][2 * k + 1]);
            }
          }
          float2 kf[4];  // K (scale, min) of group k for the lane's four tokens
#pragma unroll
          for (int e = 0; e < 4; ++e)
            kf[e] = __half22float2(*reinterpret_cast<const __half2*>(
                ((e >> 1) ? s1 : s0) + 1024 + 4 * ((g + 8 * (e & 1)) * NGQ + k)));
          const float2 raw01 = make_float2((float)(dq[0][0] * 256 + dq[0][1]), (float)(dq[0][2] * 256 + dq[0][3]));
          const float2 raw23 = make_float2((float)(dq[1][0] * 256 + dq[1][1]), (float)(dq[1][2] * 256 + dq[1][3]));
          const float2 bh2 = make_float2(bh[0][k], bh[0][k]);
          x01 = __ffma2_rn(__fmul2_rn(make_float2(kf[0].x, kf[1].x), ah2), raw01,
                           __ffma2_rn(make_float2(kf[0].y, kf[1].y), bh2, x01));
          x23 = __ffma2_rn(__fmul2_rn(make_float2(kf[2].x, kf[3].x), ah2), raw23,
                           __ffma2_rn(make_float2(kf[2].y, kf[3].y), bh2, x23));
        }
        if constexpr (!fullstep) {
          x01.x = tv[0] ? x01.x : -INFINITY;
          x01.y = tv[1] ? x01.y : -INFINITY;
          x23.x = tv[2] ? x23.x : -INFINITY;
          x23.y = tv[3] ? x23.y : -INFINITY;
        }
        // the reference max moves only when a score passes it by more than kMaxSlack
        float bm = fmaxf(fmaxf(x01.x, x01.y), fmaxf(x23.x, x23.y));
        if (__any_sync(0xffffffffu, bm > (st.m[0] == -INFINITY ? -INFINITY : kMaxSlack))) {
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
          const float mnew = bm + mref0;
          const bool need = mnew > st.m[0] + kMaxSlack;
          const float alpha = need ? fast_ex2(st.m[0] - mnew) : 1.f;
          mma_flush(st, acci, psum, 0, inv_of(0), alpha);
          if (need) {
            const float2 a2 = make_float2(alpha, alpha), d2 = make_float2(-bm, -bm);
            st.l[0] = __fmul2_rn(st.l[0], a2);
#pragma unroll
            for (int k = 0; k < NGQ; ++k) st.msum[0][k] = __fmul2_rn(st.msum[0][k], a2);
            st.m[0] = mnew;
            x01 = __fadd2_rn(x01, d2);
            x23 = __fadd2_rn(x23, d2);
          }
        }
        const float2 p01 = make_float2(fast_ex2(x01.x), fast_ex2(x01.y));  // 0 for masked tokens
        const float2 p23 = make_float2(fast_ex2(x23.x), fast_ex2(x23.y));
        st.l[0] = __fadd2_rn(st.l[0], __fadd2_rn(p01, p23));
        // ---- P' of every group (kMagicBits + round(p s lam)), the min terms, the step's sums of P'
        const float2 mg2 = make_float2(kMagic, kMagic);
        uint32_t um = 0u, ustep[NGQ];
        auto store_p = [&](int k, const uint32_t (&u)[4]) {
          uint16_t* prow = myp + (k * HP + t) * kPStride;
#pragma unroll
          for (int e = 0; e < 4; ++e) prow[16 * (e >> 1) + g + 8 * (e & 1)] = (uint16_t)u[e];  // P' < 2^16
          ustep[k] = (u[0] + u[1]) + (u[2] + u[3]) - 4u * kMagicBits;
        };
        {
          const float2 lam2 = make_float2(lam[0], lam[0]);
#pragma unroll
          for (int k = 0; k < NGQ; ++k) {
            float2 vf[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t x = vpair(e, k);
              vf[e] = __half22float2(*reinterpret_cast<const __half2*>(&x));
            }
            const float2 sv01 = make_float2(vf[0].x, vf[1].x), sv23 = make_float2(vf[2].x, vf[3].x);
            // m + 3/2 s: the codes are centred in the flush (0 for masked tokens)
            const float2 mc01 = make_float2(fmaf(1.5f, vf[0].x, vf[0].y), fmaf(1.5f, vf[1].x, vf[1].y));
            const float2 mc23 = make_float2(fmaf(1.5f, vf[2].x, vf[2].y), fmaf(1.5f, vf[3].x, vf[3].y));
            st.msum[0][k] = __ffma2_rn(p23, mc23, __ffma2_rn(p01, mc01, st.msum[0][k]));
            const float2 u01 = __ffma2_rn(p01, __fmul2_rn(sv01, lam2), mg2);
            const float2 u23 = __ffma2_rn(p23, __fmul2_rn(sv23, lam2), mg2);
            const uint32_t u[4] = {__float_as_uint(u01.x), __float_as_uint(u01.y), __float_as_uint(u23.x),
                                   __float_as_uint(u23.y)};
            um = max(um, max(max(u[0], u[1]), max(u[2], u[3])));
            store_p(k, u);
          }
        }
        // the boost rule of the 128-channel path, on the head's largest P' over its groups
        const uint32_t big = __ballot_sync(0xffffffffu, um >= kPLowBits);
        lrb[0] = ((big >> t) & 0x11111111u) == 0u ? lrb[0] + 256 : (lrb[0] & 0xff);
        const bool raise = (t < G) && lrb[0] >= (kLowRun << 8) && (lrb[0] & 0xff) < kMaxBoost;
        if (__any_sync(0xffffffffu, um > kPHighBits || raise)) {
          uint32_t uh = um;  // the head's step maximum (lanes of the same t)
          uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 4));
          uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 8));
          uh = max(uh, __shfl_xor_sync(0xffffffffu, uh, 16));
          float ym = 0.f;  // the head's largest p s over its groups
#pragma unroll
          for (int k = 0; k < NGQ; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float pe = (e >> 1) ? ((e & 1) ? p23.y : p23.x) : ((e & 1) ? p01.y : p01.x);
              const uint32_t x = vpair(e, k);
              ym = fmaxf(ym, pe * __low2float(*reinterpret_cast<const __half2*>(&x)));
            }
          ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 4));
          ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 8));
          ym = fmaxf(ym, __shfl_xor_sync(0xffffffffu, ym, 16));
          mma_flush(st, acci, psum, 0, inv_of(0));  // psum holds the earlier steps only
          int kb = lrb[0] & 0xff;
          if (uh > kPHighBits) {
            kb = 0;
          } else if (raise) {
            const float y = ym * lam0;
            const int ex = ((__float_as_int(y) >> 23) & 0xff) - 127;
            if (y > 0.f) kb = max(0, min(kMaxBoost, kBoostExp - ex));
          }
          lrb[0] = (uh > kPHighBits || raise) ? kb : (lrb[0] & ~0xff) | kb;
          lam[0] = lam0 * pow2f(kb);
          const float2 l2 = make_float2(lam[0], lam[0]);
#pragma unroll
          for (int k = 0; k < NGQ; ++k) {
            float sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t x = vpair(e, k);
              sv[e] = __low2float(*reinterpret_cast<const __half2*>(&x));
            }
            const float2 u01 = __ffma2_rn(__fmul2_rn(p01, make_float2(sv[0], sv[1])), l2, mg2);
            const float2 u23 = __ffma2_rn(__fmul2_rn(p23, make_float2(sv[2], sv[3])), l2, mg2);
            const uint32_t u[4] = {__float_as_uint(u01.x), __float_as_uint(u01.y), __float_as_uint(u23.x),
                                   __float_as_uint(u23.y)};
            store_p(k, u);
          }
        }
#pragma unroll
        for (int k = 0; k < NGQ; ++k) psum[0][k] += ustep[k];
        // value code words of this lane, in m-tile order: m-tile mt takes word
        // mt >> 1, fields 2 (mt & 1) and + 1.  Word (chunk c, token quad t, j)
        // sits at kVcOff + 16 (4c + t) + 4j; NGQ = 2: m-tile 4k + l reads chunk
        // 4k + (g & 3), word (g >> 2) + 2 (l >> 1); NGQ = 4: m-tile 2k + l reads
        // chunk 2k + (g & 1), word g >> 1.
        uint32_t va[4], vb[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int ch = NGQ == 2 ? 4 * (w >> 1) + (g & 3) : 2 * w + (g & 1);  // chunk row
          const int jj = NGQ == 2 ? (g >> 2) + 2 * (w & 1) : g >> 1;
          const int off = kVcOff + 16 * (4 * ch + t) + 4 * jj;
          va[w] = *reinterpret_cast<const uint32_t*>(s0 + off);
          vb[w] = *reinterpret_cast<const uint32_t*>(s1 + off);
        }
        __syncwarp();  // every lane has its value codes (and its P' rows are written)
        if (lane == 0) mbar_arrive(&empty[s]);
        uint32_t pb0[NGQ], pb1[NGQ];
        const uint32_t sel = (g & 1) ? 0x6420u : 0x7531u;  // odd column: low byte (lo limb)
#pragma unroll
        for (int k = 0; k < NGQ; ++k) {
          const uint16_t* prow = myp + (k * HP + (g >> 1)) * kPStride;
          const uint2 x0 = *reinterpret_cast<const uint2*>(prow + 4 * t);
          const uint2 x1 = *reinterpret_cast<const uint2*>(prow + 16 + 4 * t);
          pb0[k] = prmt(x0.x, x0.y, sel);
          pb1[k] = prmt(x1.x, x1.y, sel);
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int jw = mt >> 1, k = mt / (8 / NGQ);
          const uint32_t m0 = kM2 << (4 * (mt & 1)), m1 = m0 << 2;
          const uint32_t af[4] = {va[jw] & m0, va[jw] & m1, vb[jw] & m0, vb[jw] & m1};
          mma_u8u8(acci[0][mt], af, pb0[k], pb1[k]);
        }
        if (++since_flush >= 96) {
          mma_flush(st, acci, psum, 0, inv_of(0));
          since_flush = 0;
        }
      };
      if (n0 == kBlock && n1 == kBlock) {
        if constexpr (NGQ == 1) step(std::true_type{});
        else step_grouped(std::true_type{});
      } else if (n0 + n1 > 0) {
        if constexpr (NGQ == 1) step(std::false_type{});
        else step_grouped(std::false_type{});
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      __syncwarp();
      ++done;
    }
    if (!alive && warp == 0 && lane == 0) {
      // after a timeout: the copies of stages issued but not consumed land
      // before the ring is reused or the CTA exits.  A stage kHStages before
      // the last issued one completed before its slot was refilled.
      for (int j = max(0, issued - kHStages); j < issued; ++j) {
        const uint32_t pos = it + (uint32_t)j;
        if (!mbar_drain_bounded(&full[pos % kHStages], (pos / kHStages) & 1u)) break;
      }
    }
    it += (uint32_t)nst;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_flush(st, acci, psum, nt, inv_of(nt));
    __syncthreads();  // every warp is done with the ring: it becomes window scratch, then merge buffers

    // ---------------- fp16 rows: chunks ci = grp, grp + wph, ... of this warp's head ----------------
    // fp16 chunks owned by this CTA: chunk ci where l0 <= ci * kWinCost < l1.
    // Chunk ci < n_wchunk: window positions win_first + 16 ci .. (ring rows
    // pos % W); then sink positions 16 (ci - n_wchunk) .. (sink rows pos).
    const UnitShape& ws = us;
    const int ci0 = (l0 + kWinCost - 1) / kWinCost;
    const int ci1 = slot_ok ? min(ws.n_wchunk + ws.n_schunk, (l1 + kWinCost - 1) / kWinCost) : ci0;
    if (ci0 + grp < ci1) {
      const size_t kv_rows = ((size_t)slot * hkv + head) * 2;  // K rows of (slot, head); V rows follow
      unsigned char* scratch = ring + warp * kWarpScratch;
      unsigned char* tile = scratch;                                   // 16 rows x 256 B, swizzled
      float* pw = reinterpret_cast<float*>(scratch + 4096);            // [HP][16]
      float* wo = reinterpret_cast<float*>(scratch + 4096 + HP * 64);  // [G][128]
      uint32_t qh[NT][16];
      float wsc[NT], wm[NT], wl[NT];
      float wacc[NT][8][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hcol = 4 * nt + (g >> 1);
        if (hcol < G) {
          const uint4* src = reinterpret_cast<const uint4*>(a.qwin + ((bh0 + hcol) * 2 + (g & 1)) * kD + 32 * t);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 x = src[i];
            qh[nt][4 * i] = x.x; qh[nt][4 * i + 1] = x.y; qh[nt][4 * i + 2] = x.z; qh[nt][4 * i + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) qh[nt][i] = 0u;
        }
        const int hs = 4 * nt + t;
        wsc[nt] = hs < G ? a.qscale[(bh0 + hs) * kQsStride + 2] * (kInvSqrtD * kLog2e) : 0.f;
        wm[nt] = -INFINITY;
        wl[nt] = 0.f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) wacc[nt][mt][i] = 0.f;
      }
      // One 16-row fp16 chunk: rows of positions c_first + i (i < c_n) of the
      // window ring (row = position % W) or of the sink rows (row = position),
      // K rows from kr and V rows right after them.
      auto fp16_chunk = [&](auto ring_tag, const __half* kr, int c_first, int c_n) {
        constexpr bool kRing = decltype(ring_tag)::value;
        const __half* vr = kr + (size_t)(kRing ? kWin : a.nsink) * kD;
        auto row_of = [&](int i) { return kRing ? ((c_first + i) & (kWin - 1)) : c_first + i; };
        // stage the V rows (swizzled 16-byte chunks) for the transposing loads
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int q = lane + 32 * k, row = q >> 4, col = q & 15;
          uint4 x = make_uint4(0, 0, 0, 0);
          if (row < c_n)
            x = *reinterpret_cast<const uint4*>(vr + (size_t)row_of(row) * kD + 8 * col);
          *reinterpret_cast<uint4*>(tile + row * 256 + ((col ^ (row & 7)) << 4)) = x;
        }
        // scores of chunk rows g and g + 8
        uint32_t ka[16], kb[16];
        const bool va_ = g < c_n, vb_ = g + 8 < c_n;
        const uint4* ra = reinterpret_cast<const uint4*>(kr + (size_t)row_of(g) * kD + 32 * t);
        const uint4* rb = reinterpret_cast<const uint4*>(kr + (size_t)row_of(g + 8) * kD + 32 * t);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 x = va_ ? ra[i] : make_uint4(0, 0, 0, 0);
          const uint4 y = vb_ ? rb[i] : make_uint4(0, 0, 0, 0);
          ka[4 * i] = x.x; ka[4 * i + 1] = x.y; ka[4 * i + 2] = x.z; ka[4 * i + 3] = x.w;
          kb[4 * i] = y.x; kb[4 * i + 1] = y.y; kb[4 * i + 2] = y.z; kb[4 * i + 3] = y.w;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t af[4] = {ka[2 * ks], kb[2 * ks], ka[2 * ks + 1], kb[2 * ks + 1]};
            mma_f16(d, af, qh[nt][2 * ks], qh[nt][2 * ks + 1]);
          }
          const int hs = 4 * nt + t;
          const float s_a = (va_ && hs < G) ? (d[0] + d[1]) * wsc[nt] : -INFINITY;
          const float s_b = (vb_ && hs < G) ? (d[2] + d[3]) * wsc[nt] : -INFINITY;
          float bm = fmaxf(s_a, s_b);
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
          const float mnew = fmaxf(wm[nt], bm);
          const float mref = mnew == -INFINITY ? 0.f : mnew;
          const float alpha = fast_ex2(wm[nt] - mref);
          const float pa_ = fast_ex2(s_a - mref), pb_ = fast_ex2(s_b - mref);
          wl[nt] = wl[nt] * alpha + pa_ + pb_;
          wm[nt] = mnew;
          pw[(4 * nt + t) * 16 + g] = pa_;
          pw[(4 * nt + t) * 16 + g + 8] = pb_;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) wacc[nt][mt][i] *= alpha;
        }
        __syncwarp();
        // P.V: A = V^T (channels x tokens) by transposing loads, B = p as fp16 hi/lo
        uint32_t b0[NT], b1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float* prw = pw + (4 * nt + (g >> 1)) * 16;
          const float2 pa2 = *reinterpret_cast<const float2*>(prw + 2 * t);
          const float2 pb2 = *reinterpret_cast<const float2*>(prw + 2 * t + 8);
          const __half2 ha = __floats2half2_rn(pa2.x, pa2.y), hb = __floats2half2_rn(pb2.x, pb2.y);
          __half2 ra2 = ha, rb2 = hb;
          if (g & 1) {
            const float2 fa = __half22float2(ha), fb = __half22float2(hb);
            ra2 = __floats2half2_rn(pa2.x - fa.x, pa2.y - fa.y);
            rb2 = __floats2half2_rn(pb2.x - fb.x, pb2.y - fb.y);
          }
          b0[nt] = *reinterpret_cast<uint32_t*>(&ra2);
          b1[nt] = *reinterpret_cast<uint32_t*>(&rb2);
        }
        {
          const int mi = lane >> 3, ri = lane & 7;
          const int tok = ri + 8 * (mi >> 1);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int col = 2 * mt + (mi & 1);
            uint32_t af[4];
            ldmatrix_x4_trans(af, tile + tok * 256 + ((col ^ (tok & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_f16(wacc[nt][mt], af, b0[nt], b1[nt]);
          }
        }
        __syncwarp();
      };
      for (int ci = ci0 + grp; ci < ci1; ci += wph) {
        if (ci < ws.n_wchunk) {
          fp16_chunk(std::true_type{}, a.ring + kv_rows * kWin * kD, ws.win_first + 16 * ci,
                     min(16, ws.n_win - 16 * ci));
        } else {
          const int f = 16 * (ci - ws.n_wchunk);
          fp16_chunk(std::false_type{}, a.sink + kv_rows * a.nsink * kD, f, min(16, ws.n_sink - f));
        }
      }
      // window o' per (head, channel) through shared memory, then fold into the block state
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hs = 4 * nt + t;
        if (hs < G) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            wo[hs * kD + 16 * mt + g] = wacc[nt][mt][0] + wacc[nt][mt][1];
            wo[hs * kD + 16 * mt + g + 8] = wacc[nt][mt][2] + wacc[nt][mt][3];
          }
        }
      }
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hs = 4 * nt + t;
        float v[16];
        tacc_load(st.tacc + 16u * nt, v);
        if (hs < G) {
          const float M = fmaxf(st.m[nt], wm[nt]);
          const float mref = M == -INFINITY ? 0.f : M;
          const float ab = fast_ex2(st.m[nt] - mref), aw = fast_ex2(wm[nt] - mref);
          const float* src = wo + hs * kD;
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = fmaf(v[i], ab, src[chan_base<NGQ>(g, i >> 2) + (i & 3)] * aw);
          st.l[nt] = make_float2(fmaf(st.l[nt].x + st.l[nt].y, ab, wl[nt] * aw), 0.f);
#pragma unroll
          for (int k = 0; k < NGQ; ++k)
            st.msum[nt][k] = make_float2((st.msum[nt][k].x + st.msum[nt][k].y) * ab, 0.f);
          st.m[nt] = M;
        }
        tacc_store(st.tacc + 16u * nt, v);
      }
    }

    // ---------------- partial for (c, b): one warp per KV head, or merged across its warps ----------------
    float* part_b = a.part + ((size_t)(crange() + b) * a.hq + (size_t)qhead0(head)) * kPartStride;
    if (wph == 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float l = st.l[nt].x + st.l[nt].y, ms[NGQ];
#pragma unroll
        for (int k = 0; k < NGQ; ++k) ms[k] = st.msum[nt][k].x + st.msum[nt][k].y;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
          for (int k = 0; k < NGQ; ++k) ms[k] += __shfl_xor_sync(0xffffffffu, ms[k], o);
        }
        const int hs = 4 * nt + t;
        float v[16];
        tacc_load(st.tacc + 16u * nt, v);
        if (hs < G) {
          float* dst = part_b + (size_t)hs * kPartStride;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float m_ = ms[run_group<NGQ>(q)];
            *reinterpret_cast<float4*>(dst + chan_base<NGQ>(g, q)) =
                make_float4(v[4 * q] + m_, v[4 * q + 1] + m_, v[4 * q + 2] + m_, v[4 * q + 3] + m_);
          }
          if (g == 0) {
            part_b[(size_t)hs * kPartStride + 128] = st.m[nt];
            part_b[(size_t)hs * kPartStride + 129] = l;
          }
        }
      }
    } else {
      __syncthreads();  // window scratch no longer in use: the ring becomes merge buffers
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float l = st.l[nt].x + st.l[nt].y, ms[NGQ];
#pragma unroll
        for (int k = 0; k < NGQ; ++k) ms[k] = st.msum[nt][k].x + st.msum[nt][k].y;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
          for (int k = 0; k < NGQ; ++k) ms[k] += __shfl_xor_sync(0xffffffffu, ms[k], o);
        }
        const int hs = 4 * nt + t;
        float v[16];
        tacc_load(st.tacc + 16u * nt, v);
        if (hs < G) {
          float* dst = mo + ((size_t)warp * G + hs) * kD;
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[chan_base<NGQ>(g, i >> 2) + (i & 3)] = v[i] + ms[run_group<NGQ>(i >> 2)];
          if (g == 0) {
            ml[(warp * G + hs) * 2 + 0] = st.m[nt];
            ml[(warp * G + hs) * 2 + 1] = l;
          }
        }
      }
      __syncthreads();
      // thread -> (KV head, query head, channel); warps hh, hh + hkv, ... share KV head hh
      for (int i = threadIdx.x; i < hkv * G * kD; i += blockDim.x) {
        const int hh = i / (G * kD), gg = (i / kD) % G, ch = i % kD;
        float mx = -INFINITY;
        for (int k = 0; k < wph; ++k) mx = fmaxf(mx, ml[((hh + k * hkv) * G + gg) * 2]);
        float o = 0.f, l = 0.f;
        if (mx != -INFINITY) {
          for (int k = 0; k < wph; ++k) {
            const int w = hh + k * hkv;
            const float mw = ml[(w * G + gg) * 2];
            if (mw == -INFINITY) continue;
            const float sc = exp2f(mw - mx);
            o = fmaf(mo[((size_t)w * G + gg) * kD + ch], sc, o);
            l = fmaf(ml[(w * G + gg) * 2 + 1], sc, l);
          }
        }
        float* dst = a.part + ((size_t)(crange() + b) * a.hq + (size_t)qhead0(hh) + gg) * kPartStride;
        dst[ch] = o;
        if (ch == 0) {
          dst[128] = mx;
          dst[129] = l;
        }
      }
    }
  }
  if (!waited) grid_dep_wait();
  if (warp == 0) cp_async_wait_all();  // no block-id prefetch may outlive the CTA
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(*tmem_slot), "r"(Cfg::tmem_cols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Kernel 3: merge the splits of one (b, query head), normalise, undo the
// value rotation (un-permute, Hadamard, U_V^T) and write the fp32 output.
// One CTA per (b, query head) so that enough loads are in flight: before any
// reduction a CTA starts async copies of U_V into shared memory and loads the
// o' rows of the first 128 splits into registers (warp w: splits w, w+8, ...;
// lane l: channels 4l..4l+3).
// ---------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;
constexpr int kCombPre = 16;      // o' rows per warp loaded ahead of the weights
constexpr int kMaxSplits = 1024;  // >= split-K CTAs (at most 4 per SM)
constexpr size_t kCombSmem = (size_t)(kD * kD + kMaxSplits + kCombWarps * kD + kD + 2 * kCombWarps) * sizeof(float);

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

__global__ void __launch_bounds__(kCombThreads) combine_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) float csm[];
  float* us_ = csm;                        // U_V [128][128]
  float* ml = us_ + kD * kD;               // [kMaxSplits] split maxima, then weights 2^(m_c - M)
  float* wsum = ml + kMaxSplits;           // [warps][128] per-warp partial sums
  float* xs = wsum + kCombWarps * kD;      // [128] merged, normalised, un-rotated o
  float* redm = xs + kD;                   // [warps]
  float* redl = redm + kCombWarps;         // [warps]
  const int b = blockIdx.x / a.hq, head = blockIdx.x % a.hq;
  const int hk = head / a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {
    const float* U = a.u_v + (size_t)hk * kD * kD;
#pragma unroll
    for (int k = 0; k < kD * kD / 4 / kCombThreads; ++k) {
      const int i = tid + kCombThreads * k;
      cp_async16(us_ + 4 * i, U + 4 * i);
    }
    cp_async_commit();
  }
  grid_dep_wait();  // the split partials (and the cost prefix) are read from here on
  const UnitShape sh = unit_shape(clamp_len(a.context_lens, b, a.mbps, a.status, false), a.nsink);
  const long long total = a.prefix[a.batch];
  float* outp = a.out + ((size_t)b * a.hq + head) * kD;
  if (sh.cost == 0 || total == 0) {
    if (tid < kD) outp[tid] = 0.f;
    cp_async_wait_all();
    return;
  }
  const long long pu = a.prefix[b];
  const int nc = working_ctas(a, total);
  const int c0 = cta_of(pu, total, nc);
  const int ns = cta_of(pu + sh.cost - 1, total, nc) - c0 + 1;  // splits of this entry
  const size_t split_stride = (size_t)a.hq * kPartStride;
  const float* base = a.part + ((size_t)(c0 + b) * a.hq + head) * kPartStride;
  // o' rows of the first kCombPre splits of this warp
  float4 pre[kCombPre];
#pragma unroll
  for (int j = 0; j < kCombPre; ++j) {
    const int c = warp + kCombWarps * j;
    pre[j] = c < ns ? *reinterpret_cast<const float4*>(base + (size_t)c * split_stride + 4 * lane)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // split maxima and sums, and the global maximum
  float mx = -INFINITY;
  for (int c = tid; c < ns; c += kCombThreads) {
    const float2 m2 = *reinterpret_cast<const float2*>(base + (size_t)c * split_stride + 128);
    ml[c] = m2.x;
    wsum[c] = m2.y;  // the sums borrow the partial-sum buffer until the weights are known
    mx = fmaxf(mx, m2.x);
  }
  mx = warp_max(mx);
  if (lane == 0) redm[warp] = mx;
  __syncthreads();
  mx = redm[0];
#pragma unroll
  for (int w = 1; w < kCombWarps; ++w) mx = fmaxf(mx, redm[w]);
  float l = 0.f;
  for (int c = tid; c < ns; c += kCombThreads) {
    const float m = ml[c];
    const float w = (mx == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - mx);
    ml[c] = w;
    l = fmaf(wsum[c], w, l);
  }
  l = warp_sum(l);
  if (lane == 0) redl[warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int w = 0; w < kCombWarps; ++w) l += redl[w];
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  // weighted sum of the splits
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kCombPre; ++j) {
    const int c = warp + kCombWarps * j;
    const float w = c < ns ? ml[c] : 0.f;
    acc.x = fmaf(pre[j].x, w, acc.x);
    acc.y = fmaf(pre[j].y, w, acc.y);
    acc.z = fmaf(pre[j].z, w, acc.z);
    acc.w = fmaf(pre[j].w, w, acc.w);
  }
  for (int c0w = warp + kCombWarps * kCombPre; c0w < ns; c0w += kCombWarps * kCombPre) {
#pragma unroll
    for (int j = 0; j < kCombPre; ++j) {
      const int c = c0w + kCombWarps * j;
      pre[j] = c < ns ? *reinterpret_cast<const float4*>(base + (size_t)c * split_stride + 4 * lane)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kCombPre; ++j) {
      const int c = c0w + kCombWarps * j;
      const float w = c < ns ? ml[c] : 0.f;
      acc.x = fmaf(pre[j].x, w, acc.x);
      acc.y = fmaf(pre[j].y, w, acc.y);
      acc.z = fmaf(pre[j].z, w, acc.z);
      acc.w = fmaf(pre[j].w, w, acc.w);
    }
  }
  __syncthreads();  // every thread is done with the sums borrowed in wsum
  *reinterpret_cast<float4*>(&wsum[warp * kD + 4 * lane]) = acc;
  cp_async_wait_all();
  __syncthreads();
  // un-permute + Hadamard in warp 0: lane holds pre-permutation channels
  // l + 32a = rotated channels 4*rev5(l) + rev2(a)
  if (warp == 0) {
    const int r = rev5(lane);
    float y[4];
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      const int ch = 4 * r + rev2(aa);
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < kCombWarps; ++w) o += wsum[w * kD + ch];
      y[aa] = o * inv_l;
    }
    wht128_warp(y, lane);
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) xs[lane + 32 * aa] = y[aa] * kInvSqrtD;
  }
  __syncthreads();
  // o_c = sum_i x_i U_V[c][i]: warp w, channels 16w..16w+15; lane l inputs 4l..4l+3
  const float4 xv = *reinterpret_cast<const float4*>(&xs[4 * lane]);
  float part[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const float4 u = *reinterpret_cast<const float4*>(us_ + (16 * warp + r) * kD + 4 * lane);
    part[r] = fmaf(xv.x, u.x, fmaf(xv.y, u.y, fmaf(xv.z, u.z, xv.w * u.w)));
  }
  // transpose-reduce: after the four halving steps lane l holds the partial of
  // channel 16w + (l & 15) summed over 16 lanes; one more step finishes it
#pragma unroll
  for (int step = 8; step >= 1; step >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int r = 0; r < step; ++r) {
      const float send = upper ? part[r] : part[r + step];
      const float keep = upper ? part[r + step] : part[r];
      part[r] = keep + __shfl_xor_sync(0xffffffffu, send, step);
    }
  }
  const float o = part[0] + __shfl_xor_sync(0xffffffffu, part[0], 16);
  if (lane < 16) outp[16 * warp + lane] = o;
}

template <int G>
static okv_status launch_decode_simt(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)(G * kD + kDecWarps * G * kD + kDecWarps * G * 2) * sizeof(float);
  static std::atomic<uint32_t> attr_set{0};
  cudaError_t e = set_smem_limit_once((const void*)decode_simt_kernel<G>, (int)smem, attr_set);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "decode smem attribute: %s", cudaGetErrorString(e));
  decode_simt_kernel<G><<<a.nc, kDecWarps * 32, smem, s>>>(a);
  return check_launch("decode");
}


template <int G, int NGQ = 1, int HS = 1>
static okv_status launch_decode_heads(const DecodeArgs& a, cudaStream_t s, bool early) {
  if (a.hsplit != HS || HS * G != a.g)
    return fail(OKV_ERR_UNSUPPORTED, "split-K head split %d x %d != %d", a.hsplit, G, a.g);
  const size_t smem = HCfg<G, NGQ>::smem_bytes();
  static std::atomic<uint32_t> attr_set{0};
  cudaError_t e = set_smem_limit_once((const void*)decode_heads_kernel<G, NGQ, HS>, (int)smem, attr_set);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "decode smem attribute: %s", cudaGetErrorString(e));
  e = launch_pdl(decode_heads_kernel<G, NGQ, HS>, dim3(a.nc * HS), dim3(kHW * 32), smem, s, early, a);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return check_launch("decode");
}

bool decode_uses_tensor_cores(int g, int hkv, int ng) {
  const bool hkv_ok = hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8;
  return hkv_ok && (ng == 1 || ng == 2 || ng == 4) && (g == 1 || g == 2 || g == 4 || g == 8 || g == 16);
}

// split-K cost ranges for a device of `sms` SMs: two CTAs per SM for the
// tensor-core kernel (one at G = 8 with one group per vector, whose CTA holds
// both n-tiles), with a range split over two (G = 8 grouped) or four (G = 16)
// CTAs of four query heads; four CTAs per SM for the CUDA-core kernel
int decode_ranges(int sms, int g, int hkv, int ng) {
  if (!decode_uses_tensor_cores(g, hkv, ng)) return 4 * sms;
  if (g <= 4) return 2 * sms;
  if (g == 8) return sms;
  return sms / 2;  // g = 16
}

static DecodeArgs make_decode_args(const okv_cache_desc* d, const void* q, int B, const int32_t* seq_slot,
                                   const int32_t* block_table, const int32_t* context_lens, float* out, void* ws,
                                   const DecodePlan& plan) {
  DecodeArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.seq_slot = seq_slot;
  a.block_table = block_table;
  a.context_lens = context_lens;
  a.u_k = d->u_k;
  a.u_v = d->u_v;
  a.pages = (const uint8_t*)d->pages;
  a.ring = (const __half*)d->window_ring;
  a.sink = (const __half*)d->sink_rows;
  a.nsink = d->num_sink;
  a.out = out;
  a.status = d->status_word;
  uint8_t* w = (uint8_t*)ws;
  a.qrot = (float*)(w + plan.qrot_off);
  a.qlimb = (int8_t*)(w + plan.qlimb_off);
  a.qscale = (float*)(w + plan.qscale_off);
  a.qwin = (__half*)(w + plan.qwin_off);
  a.prefix = (int32_t*)(w + plan.prefix_off);
  a.part = (float*)(w + plan.part_off);
  a.batch = B;
  a.hq = d->num_q_heads;
  a.hkv = d->num_kv_heads;
  a.g = plan.g;
  a.nc = plan.num_ctas;
  a.num_blocks = d->num_blocks;
  a.num_slots = d->num_seq_slots;
  a.mbps = d->max_blocks_per_seq;
  a.ng = kD / d->group;
  // grouped layouts at G = 8, and every layout at G = 16: two or four CTAs per
  // cost range, four query heads each
  a.hsplit = a.g == 16 ? 4 : (a.ng > 1 && a.g == 8) ? 2 : 1;
  return a;
}

// split-K attention and the combine, after the queries have been rotated
static okv_status launch_decode_tail(const DecodeArgs& a, int B, cudaStream_t s) {
  okv_status st = OKV_OK;
  cudaEvent_t ev0, ev1;
  take_decode_events(&ev0, &ev1);
  // inside a stream capture the events become external event nodes of the
  // graph, so that each replay records them; outside one they are recorded
  // as usual
  unsigned ev_flags = cudaEventRecordDefault;
  if (ev0 != nullptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return fail(OKV_ERR_CUDA, "cudaStreamIsCapturing failed");
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
  }
  if (ev0 != nullptr && cudaEventRecordWithFlags(ev0, s, ev_flags) != cudaSuccess)
    return fail(OKV_ERR_CUDA, "cudaEventRecord failed");
  // Early (programmatic) launches overlap each kernel's start with its
  // predecessor; they are left out when the split-K kernel is being timed, so
  // that the events bracket it alone.
  const bool early = ev0 == nullptr;
  const bool tc = decode_uses_tensor_cores(a.g, a.hkv, a.ng);
  if (tc && a.ng == 2) {
    switch (a.g) {
      case 1: st = launch_decode_heads<1, 2>(a, s, early); break;
      case 2: st = launch_decode_heads<2, 2>(a, s, early); break;
      case 4: st = launch_decode_heads<4, 2>(a, s, early); break;
      case 8: st = launch_decode_heads<4, 2, 2>(a, s, early); break;  // G = 8 as two halves
      default: st = launch_decode_heads<4, 2, 4>(a, s, early); break;  // G = 16 as four quarters
    }
  } else if (tc && a.ng == 4) {
    switch (a.g) {
      case 1: st = launch_decode_heads<1, 4>(a, s, early); break;
      case 2: st = launch_decode_heads<2, 4>(a, s, early); break;
      case 4: st = launch_decode_heads<4, 4>(a, s, early); break;
      case 8: st = launch_decode_heads<4, 4, 2>(a, s, early); break;  // G = 8 as two halves
      default: st = launch_decode_heads<4, 4, 4>(a, s, early); break;  // G = 16 as four quarters
    }
  } else if (tc) {
    switch (a.g) {
      case 1: st = launch_decode_heads<1>(a, s, early); break;
      case 2: st = launch_decode_heads<2>(a, s, early); break;
      case 4: st = launch_decode_heads<4>(a, s, early); break;
      case 8: st = launch_decode_heads<8>(a, s, early); break;
      default: st = launch_decode_heads<4, 1, 4>(a, s, early); break;  // G = 16 as four quarters
    }
  } else {
    switch (a.g) {
      case 1: st = launch_decode_simt<1>(a, s); break;
      case 2: st = launch_decode_simt<2>(a, s); break;
      case 4: st = launch_decode_simt<4>(a, s); break;
      case 8: st = launch_decode_simt<8>(a, s); break;
      case 16: st = launch_decode_simt<16>(a, s); break;
      default: return fail(OKV_ERR_UNSUPPORTED, "group size %d (Hq/Hkv) not in {1,2,4,8,16}", a.g);
    }
  }
  if (st != OKV_OK) return st;
  if (ev1 != nullptr && cudaEventRecordWithFlags(ev1, s, ev_flags) != cudaSuccess)
    return fail(OKV_ERR_CUDA, "cudaEventRecord failed");
  static std::atomic<uint32_t> attr_set{0};
  cudaError_t e = set_smem_limit_once((const void*)combine_kernel, (int)kCombSmem, attr_set);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "combine smem attribute: %s", cudaGetErrorString(e));
  e = launch_pdl(combine_kernel, dim3(B * a.hq), dim3(kCombThreads), kCombSmem, s, early && tc, a);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  return check_launch("combine");
}

okv_status launch_decode(const okv_cache_desc* d, const void* q, int B, const int32_t* seq_slot,
                         const int32_t* block_table, const int32_t* context_lens, float* out,
                         void* ws, const DecodePlan& plan, cudaStream_t s) {
  const DecodeArgs a = make_decode_args(d, q, B, seq_slot, block_table, context_lens, out, ws, plan);
  qrot_kernel<<<B * a.hq, kPrepThreads, 0, s>>>(a);
  const okv_status st = check_launch("query rotation");
  if (st != OKV_OK) return st;
  return launch_decode_tail(a, B, s);
}

okv_status launch_decode_step(const okv_cache_desc* d, const void* k, const void* v, int T, const int32_t* new_slot,
                              const int32_t* new_pos, const int32_t* slot_lens, const void* q, int B,
                              const int32_t* seq_slot, const int32_t* block_table, const int32_t* context_lens,
                              float* out, void* ws, const DecodePlan& plan, cudaStream_t s) {
  const DecodeArgs a = make_decode_args(d, q, B, seq_slot, block_table, context_lens, out, ws, plan);
  const AppendArgs aa = make_append_args(d, k, v, new_slot, new_pos, block_table, slot_lens, nullptr);
  const int n_tiles = (T + kAppTokens - 1) / kAppTokens;
  const long long ctas = (long long)n_tiles * d->num_kv_heads * 2 + (long long)B * a.hq;
  step_prep_kernel<<<(unsigned)ctas, kPrepThreads, 0, s>>>(aa, T, n_tiles, a);
  const okv_status st = check_launch("decode step (append + query rotation)");
  if (st != OKV_OK) return st;
  return launch_decode_tail(a, B, s);
}

}  // namespace okv
