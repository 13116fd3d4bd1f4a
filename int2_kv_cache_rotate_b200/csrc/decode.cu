// Decode attention over the INT2 paged cache: query rotation, split-K
// attention with online softmax, and the split combine with the value
// un-rotation.
#include "okv_common.cuh"
#include "okv_internal.h"

namespace okv {

// ---------------------------------------------------------------------------
// Work partition.  Unit u = (batch entry b, KV head hk).  With L tokens in the
// cache, the unit costs ceil(max(L-W,0)/16) INT2 blocks plus kWinCost for its
// fp16 window (if L > 0).  Units are laid end to end in "cost space"; split-K
// CTA c takes the contiguous range [c*total/NC, (c+1)*total/NC).  Inside a
// unit, cost positions [0, kWinCost) stand for the window and the rest for the
// blocks in order.  A (unit, CTA) pair writes partial slot c + u: distinct
// for distinct pairs because CTAs and units are both contiguous.
// ---------------------------------------------------------------------------
struct UnitShape {
  int len;      // tokens in the cache
  int n_int2;   // tokens read from INT2 blocks
  int n_pages;  // INT2 blocks touched
  int n_win;    // tokens read from the fp16 window
  int win_cost;
  int cost;
};

__device__ __forceinline__ UnitShape unit_shape(int len) {
  UnitShape s;
  s.len = len;
  s.n_int2 = len > kWin ? len - kWin : 0;
  s.n_pages = (s.n_int2 + kBlock - 1) / kBlock;
  s.n_win = len < kWin ? len : kWin;
  s.win_cost = len > 0 ? kWinCost : 0;
  s.cost = s.n_pages + s.win_cost;
  return s;
}

// first CTA whose range contains cost position x (x < total)
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

struct DecodeArgs {
  const __nv_bfloat16* q;
  const int32_t* seq_slot;
  const int32_t* block_table;
  const int32_t* context_lens;
  const float* u_k;
  const float* u_v;
  const uint8_t* pages;
  const __half* ring;
  float* out;
  uint32_t* status;
  float* qrot;       // [B][Hq][128]
  int8_t* qlimb;     // [B][Hq][2][128]
  float* qscale;     // [B][Hq][4]
  int32_t* prefix;   // [B+1] cost prefix over batch entries (units of b are consecutive)
  float* part;       // [(NC + NU)][G][kPartStride]
  int batch, hq, hkv, g, nc, num_blocks, num_slots, mbps;
};

// ---------------------------------------------------------------------------
// Kernel 1: q~ = q R_K for every (b, query head), plus the cost prefix.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) qrot_kernel(DecodeArgs a) {
  __shared__ float red[4][kD];
  const int b = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (b == 0 && h == 0) {
    // cost prefix over batch entries: thread-serial chunks + one pass over chunk sums
    __shared__ int chunk_sum[128];
    const int per = (a.batch + 127) / 128;
    const int lo = threadIdx.x * per, hi = min(a.batch, lo + per);
    int s = 0;
    for (int i = lo; i < hi; ++i)
      s += a.hkv * unit_shape(clamp_len(a.context_lens, i, a.mbps, a.status, true)).cost;
    chunk_sum[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      int run = 0;
      for (int i = 0; i < 128; ++i) {
        const int c = chunk_sum[i];
        chunk_sum[i] = run;
        run += c;
      }
      a.prefix[a.batch] = run;
    }
    __syncthreads();
    int run = chunk_sum[threadIdx.x];
    for (int i = lo; i < hi; ++i) {
      a.prefix[i] = run;
      run += a.hkv * unit_shape(clamp_len(a.context_lens, i, a.mbps, a.status, false)).cost;
    }
    __syncthreads();
  }
  float y[4];
  const __nv_bfloat16* src = a.q + ((size_t)b * a.hq + h) * kD;
  rotate_cta(src, a.u_k + (size_t)(h / a.g) * kD * kD, red, y);
  if (warp != 0) return;
  const int r = rev5(lane);
  float* dst = a.qrot + ((size_t)b * a.hq + h) * kD + 4 * r;
  *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[2], y[1], y[3]);
}

// ---------------------------------------------------------------------------
// Kernel 2 (SIMT): split-K attention.  4 warps per CTA; a warp takes whole
// 16-token chunks (an INT2 block, or 16 window rows) and keeps its own
// online-softmax state; warps merge through shared memory at unit end.
// Lane l scores token l/2 over channels 64*(l&1)..+63 and accumulates the
// output channels 4l..4l+3 (canonical code byte l).
// ---------------------------------------------------------------------------
constexpr int kDecWarps = 4;

template <int G>
struct WarpState {
  float m[G], l[G], o[G][4];
};

template <int G, bool kWindow>
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
      const uint32_t smk = *reinterpret_cast<const uint32_t*>(blockp + kKsmOff + 4 * tt);
      const float s = __half2float(__ushort_as_half((unsigned short)(smk & 0xffff)));
      const float m = __half2float(__ushort_as_half((unsigned short)(smk >> 16)));
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int c = 64 * half + 16 * wi + j;
          const float x = fmaf(s, (float)((words[wi] >> (2 * j)) & 3u), m);
#pragma unroll
          for (int g = 0; g < G; ++g) sc[g] = fmaf(qs[g * kD + c], x, sc[g]);
        }
      }
    } else {
      const int row = (win_first_row + tt) % kWin;
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
      const uint32_t smv = *reinterpret_cast<const uint32_t*>(blockp + kVsmOff + 4 * t);
      const float s = __half2float(__ushort_as_half((unsigned short)(smv & 0xffff)));
      const float m = __half2float(__ushort_as_half((unsigned short)(smv >> 16)));
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = fmaf(s, (float)((byte >> (2 * j)) & 3u), m);
    } else {
      const int row = (win_first_row + t) % kWin;
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
  // with fewer cost units than CTAs, only the first `total` CTAs take work, so
  // that every working CTA owns a non-empty range
  const int nc = (int)min((long long)a.nc, total);
  const int c = blockIdx.x;
  if (c >= nc) return;
  const long long start = (long long)c * total / nc;
  const long long end = (long long)(c + 1) * total / nc;
  // first batch entry whose units reach past `start`
  int lo = 0, hi = a.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.prefix[mid] <= start) lo = mid; else hi = mid - 1;
  }
  int b = lo;
  for (; b < a.batch && a.prefix[b] < end; ++b) {
    const UnitShape us = unit_shape(clamp_len(a.context_lens, b, a.mbps, a.status, false));
    if (us.cost == 0) continue;
    const int slot = a.seq_slot[b];
    const bool slot_ok = slot >= 0 && slot < a.num_slots;
    for (int hk = 0; hk < a.hkv; ++hk) {
      const long long pu = a.prefix[b] + (long long)hk * us.cost;
      if (pu + us.cost <= start) continue;
      if (pu >= end) break;
      const int u = b * a.hkv + hk;
      const int l0 = (int)(max(start, pu) - pu), l1 = (int)(min(end, pu + us.cost) - pu);
      // rotated queries of this unit into shared memory
      __syncthreads();
      for (int i = threadIdx.x; i < G * kD; i += blockDim.x)
        qs[i] = a.qrot[((size_t)b * a.hq + hk * G) * kD + i];
      __syncthreads();
      WarpState<G> st;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        st.m[g] = -INFINITY;
        st.l[g] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) st.o[g][j] = 0.f;
      }
      if (slot_ok) {
        // window part
        if (l0 == 0 && us.win_cost > 0) {
          const __half* kbase = a.ring + (((size_t)slot * a.hkv + hk) * 2 + 0) * kWin * kD;
          const __half* vbase = a.ring + (((size_t)slot * a.hkv + hk) * 2 + 1) * kWin * kD;
          const int first = us.len - us.n_win;
          const int nchunk = (us.n_win + kBlock - 1) / kBlock;
          for (int ci = warp; ci < nchunk; ci += kDecWarps) {
            const int ntok = min(kBlock, us.n_win - ci * kBlock);
            simt_chunk<G, true>(a, qs, nullptr, kbase, vbase, first + ci * kBlock, ntok, st, lane);
          }
        }
        // INT2 blocks
        const int p0 = max(l0, us.win_cost) - us.win_cost;
        const int p1 = l1 - us.win_cost;
        for (int pi = p0 + warp; pi < p1; pi += kDecWarps) {
          int blk = a.block_table[(size_t)slot * a.mbps + pi];
          if (blk < 0 || blk >= a.num_blocks) {
            if (lane == 0) raise_flag(a.status, OKV_DEV_BAD_BLOCK);
            continue;
          }
          const uint8_t* bp = a.pages + ((size_t)blk * a.hkv + hk) * kBlockHeadBytes;
          const int ntok = min(kBlock, us.n_int2 - pi * kBlock);
          simt_chunk<G, false>(a, qs, bp, nullptr, nullptr, 0, ntok, st, lane);
        }
      } else if (lane == 0 && warp == 0) {
        raise_flag(a.status, OKV_DEV_BAD_SLOT);
      }
      // merge the warps' states
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mo[(warp * G + g) * kD + 4 * lane + j] = st.o[g][j];
        if (lane == 0) {
          ml[(warp * G + g) * 2 + 0] = st.m[g];
          ml[(warp * G + g) * 2 + 1] = st.l[g];
        }
      }
      __syncthreads();
      float* dst = a.part + ((size_t)(c + u) * G) * kPartStride;
      for (int i = threadIdx.x; i < G * kD; i += blockDim.x) {
        const int g = i / kD, ch = i % kD;
        float mx = -INFINITY;
        for (int w = 0; w < kDecWarps; ++w) mx = fmaxf(mx, ml[(w * G + g) * 2]);
        float o = 0.f, l = 0.f;
        if (mx != -INFINITY) {
          for (int w = 0; w < kDecWarps; ++w) {
            const float mw = ml[(w * G + g) * 2];
            const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - mx);
            o = fmaf(mo[(w * G + g) * kD + ch], sc, o);
            l = fmaf(ml[(w * G + g) * 2 + 1], sc, l);
          }
        }
        dst[g * kPartStride + ch] = o;
        if (ch == 0) {
          dst[g * kPartStride + 128] = mx;
          dst[g * kPartStride + 129] = l;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 3: merge the splits of each unit, normalise, undo the value rotation
// (un-permute, Hadamard, U_V^T) and write fp32 outputs.  One CTA per unit.
// ---------------------------------------------------------------------------
constexpr int kUPad = 129;

__global__ void __launch_bounds__(128) combine_kernel(DecodeArgs a) {
  extern __shared__ float smem[];
  float* us_ = smem;                 // U_V [128][129]
  float* xs = us_ + kD * kUPad;      // [G][128]
  const int u = blockIdx.x;
  const int b = u / a.hkv, hk = u % a.hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.g;
  const float* uv = a.u_v + (size_t)hk * kD * kD;
  for (int i = tid; i < kD * kD; i += blockDim.x) us_[(i / kD) * kUPad + (i % kD)] = uv[i];
  const UnitShape sh = unit_shape(clamp_len(a.context_lens, b, a.mbps, a.status, false));
  const long long total = a.prefix[a.batch];
  float* outp = a.out + ((size_t)b * a.hq + hk * G) * kD;
  if (sh.cost == 0 || total == 0) {
    for (int i = tid; i < G * kD; i += blockDim.x) outp[i] = 0.f;
    return;
  }
  const long long pu = a.prefix[b] + (long long)hk * sh.cost;
  const int nc = (int)min((long long)a.nc, total);
  const int c0 = cta_of(pu, total, nc);
  const int c1 = cta_of(pu + sh.cost - 1, total, nc);
  // merge splits: thread = channel
  for (int g = 0; g < G; ++g) {
    float mx = -INFINITY;
    for (int c = c0; c <= c1; ++c) mx = fmaxf(mx, a.part[((size_t)(c + u) * G + g) * kPartStride + 128]);
    float o = 0.f, l = 0.f;
    if (mx != -INFINITY) {
      for (int c = c0; c <= c1; ++c) {
        const float* src = a.part + ((size_t)(c + u) * G + g) * kPartStride;
        const float mw = src[128];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - mx);
        o = fmaf(src[tid], sc, o);
        l = fmaf(src[129], sc, l);
      }
    }
    xs[g * kD + tid] = (l > 0.f) ? o / l : 0.f;
  }
  __syncthreads();
  // un-permute + Hadamard, one warp per head: lane holds pre-permutation
  // channels l + 32a = rotated channels 4*rev5(l) + rev2(a)
  for (int g = warp; g < G; g += 4) {
    const int r = rev5(lane);
    float y[4];
    y[0] = xs[g * kD + 4 * r + 0];
    y[1] = xs[g * kD + 4 * r + 2];
    y[2] = xs[g * kD + 4 * r + 1];
    y[3] = xs[g * kD + 4 * r + 3];
    __syncwarp();
    wht128_warp(y, lane);
#pragma unroll
    for (int j = 0; j < 4; ++j) xs[g * kD + lane + 32 * j] = y[j] * kInvSqrtD;
  }
  __syncthreads();
  // o_c = sum_i x_i U_V[c][i]: thread = output channel c
  for (int g = 0; g < G; ++g) {
    float acc = 0.f;
    const float* xr = xs + g * kD;
#pragma unroll 8
    for (int i = 0; i < kD; ++i) acc = fmaf(xr[i], us_[tid * kUPad + i], acc);
    outp[g * kD + tid] = acc;
  }
}

template <int G>
static okv_status launch_decode_g(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)(G * kD + kDecWarps * G * kD + kDecWarps * G * 2) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "decode smem attribute: %s", cudaGetErrorString(e));
  decode_simt_kernel<G><<<a.nc, kDecWarps * 32, smem, s>>>(a);
  return check_launch("decode");
}

okv_status launch_decode(const okv_cache_desc* d, const void* q, int B, const int32_t* seq_slot,
                         const int32_t* block_table, const int32_t* context_lens, float* out,
                         void* ws, const DecodePlan& plan, cudaStream_t s) {
  DecodeArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.seq_slot = seq_slot;
  a.block_table = block_table;
  a.context_lens = context_lens;
  a.u_k = d->u_k;
  a.u_v = d->u_v;
  a.pages = (const uint8_t*)d->pages;
  a.ring = (const __half*)d->window_ring;
  a.out = out;
  a.status = d->status_word;
  uint8_t* w = (uint8_t*)ws;
  a.qrot = (float*)(w + plan.qrot_off);
  a.qlimb = (int8_t*)(w + plan.qlimb_off);
  a.qscale = (float*)(w + plan.qscale_off);
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

  qrot_kernel<<<dim3(B, a.hq), 128, 0, s>>>(a);
  okv_status st = check_launch("query rotation");
  if (st != OKV_OK) return st;
  cudaEvent_t ev0, ev1;
  take_decode_events(&ev0, &ev1);
  if (ev0 != nullptr && cudaEventRecordWithFlags(ev0, s, cudaEventRecordExternal) != cudaSuccess)
    return fail(OKV_ERR_CUDA, "cudaEventRecord failed");
  switch (a.g) {
    case 1: st = launch_decode_g<1>(a, s); break;
    case 2: st = launch_decode_g<2>(a, s); break;
    case 4: st = launch_decode_g<4>(a, s); break;
    case 8: st = launch_decode_g<8>(a, s); break;
    case 16: st = launch_decode_g<16>(a, s); break;
    default: return fail(OKV_ERR_UNSUPPORTED, "group size %d (Hq/Hkv) not in {1,2,4,8,16}", a.g);
  }
  if (st != OKV_OK) return st;
  if (ev1 != nullptr && cudaEventRecordWithFlags(ev1, s, cudaEventRecordExternal) != cudaSuccess)
    return fail(OKV_ERR_CUDA, "cudaEventRecord failed");
  const size_t csmem = (size_t)(kD * kUPad + a.g * kD) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem);
  if (e != cudaSuccess) return fail(OKV_ERR_CUDA, "combine smem attribute: %s", cudaGetErrorString(e));
  combine_kernel<<<plan.num_units, 128, csmem, s>>>(a);
  return check_launch("combine");
}

}  // namespace okv
