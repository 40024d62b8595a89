// Feature preparation of the linear branch ("VDA-Prep"), B200 (sm_100a).
//
// Video DeltaNet, Section 2.3: the linear branch applies a separable short
// convolution to K and V (a depthwise 5 x 5 spatial filter over the latent
// grid and a five-tap temporal filter over frames), then SiLU, and L2
// normalisation to Q and K; Section 5 fuses this with the frame-major layout
// conversion.  Inputs are the projections of the interior video tokens,
// [B, T, U, H, d] bf16 (token u = y * Wl + x); outputs are [B, H, T, U, d]
// bf16.  Filters are per head and channel: ws [H, d, 5, 5], wt [H, d, 5]
// (float32), cross-correlations with zero padding 2 on every side.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace vda {
namespace prep {

// Packed fp32 pair FMA (one instruction for two lanes of arithmetic).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t f2_to_bf2(float2 v) {
  __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

constexpr int kThreads = 512;
constexpr int kMaxNxt = 8;   // grid columns per thread

// 16-B asynchronous global -> shared copy (L1 bypassed) and its groups
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Geometry of k_prep_kv: thread = (channel pair, column slice); NS slices of
// NXT grid columns each; the staged rows carry two zero columns on each side
// (x = -2 .. NS * NXT + 1), so the spatial filter needs no bounds checks.
__host__ __device__ constexpr int kv_slices(int D) { return kThreads / (D / 2); }
__host__ __device__ constexpr int kv_cols_per_thread(int Wl, int D) { return (Wl + kv_slices(D) - 1) / kv_slices(D); }
__host__ __device__ constexpr size_t kv_stage_bytes(int Wl, int D) {
  return (size_t)5 * (kv_slices(D) * kv_cols_per_thread(Wl, D) + 4) * D * 2;
}
// Shared memory: nst staging buffers of rows y-2..y+2 (bf16 pairs), the ring
// of the last five frames' spatial results (bf16 pairs) and the fp32 output
// row of the L2 normalisation.
__host__ __device__ constexpr size_t kv_smem_bytes(int Wl, int D, int nst) {
  return (size_t)nst * kv_stage_bytes(Wl, D) + (size_t)5 * Wl * D * 2 + (size_t)Wl * D * 4;
}

// One CTA per (grid row y, batch-head, tensor K or V).  It walks the frames:
// the rows y-2..y+2 of a frame arrive by cp.async one frame ahead (two
// staging buffers when they fit, else one, refilled once the spatial filter
// has read it); the spatial filter of row y goes into a five-frame ring, and,
// two frames behind, the temporal filter, SiLU and (K only) the L2
// normalisation of output frame t.  Thread = (channel pair cp, column slice
// xs): channel pairs use packed fp32 FMAs, and each thread keeps its NXT
// columns' accumulators and the 5-tap window of one staged row in registers.
template <int D, int NXT>
__global__ void __launch_bounds__(kThreads, 1)
k_prep_kv(const __nv_bfloat16* __restrict__ kin, const __nv_bfloat16* __restrict__ vin,
          const float* __restrict__ wk_s, const float* __restrict__ wk_t,
          const float* __restrict__ wv_s, const float* __restrict__ wv_t,
          __nv_bfloat16* __restrict__ kout, __nv_bfloat16* __restrict__ vout,
          int H, int T, int Hl, int Wl, float eps, int nst) {
  constexpr int NP = D / 2;              // channel pairs
  constexpr int NS = kThreads / NP;      // column slices
  constexpr int WS = NS * NXT + 4;       // staged columns
  constexpr int V8 = D / 8;              // 16-B chunks per token
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const size_t stage_words = (size_t)5 * WS * NP;
  uint32_t* stage0 = reinterpret_cast<uint32_t*>(smem_raw);                  // [nst][5][WS][NP]
  uint32_t* ring = stage0 + (size_t)nst * stage_words;                       // [5][Wl][NP]
  float* tile = reinterpret_cast<float*>(ring + (size_t)5 * Wl * NP);        // [Wl][D]

  const int y = blockIdx.x, bh = blockIdx.y, isv = blockIdx.z;
  const int b = bh / H, h = bh - (bh / H) * H;
  const __nv_bfloat16* in = isv ? vin : kin;
  __nv_bfloat16* out = isv ? vout : kout;
  const float* ws = (isv ? wv_s : wk_s) + (size_t)h * D * 25;
  const float* wt = (isv ? wv_t : wk_t) + (size_t)h * D * 5;
  const int U = Hl * Wl;
  const int tid = threadIdx.x, cp = tid % NP, xs = tid / NP;
  const int c0 = 2 * cp;
  const int xb = xs * NXT;

  float2 wsp[25], wtp[5];
#pragma unroll
  for (int q = 0; q < 25; ++q) wsp[q] = make_float2(__ldg(ws + (size_t)c0 * 25 + q), __ldg(ws + (size_t)(c0 + 1) * 25 + q));
#pragma unroll
  for (int s = 0; s < 5; ++s) wtp[s] = make_float2(__ldg(wt + (size_t)c0 * 5 + s), __ldg(wt + (size_t)(c0 + 1) * 5 + s));

  // padding columns and rows outside the grid are never loaded: zero them once
  for (size_t e = tid; e < (size_t)nst * stage_words; e += kThreads) stage0[e] = 0u;
  __syncthreads();

  const size_t tok_stride = (size_t)H * D;   // elements between consecutive tokens of the input
  auto issue = [&](int f) {   // rows y-2..y+2 of frame f -> staging buffer f % nst
    uint32_t* st = stage0 + (size_t)(f % nst) * stage_words;
    const __nv_bfloat16* fbase = in + ((size_t)b * T + f) * U * tok_stride + (size_t)h * D;
#pragma unroll 1
    for (int r = 0; r < 5; ++r) {
      const int row = y + r - 2;
      if (row < 0 || row >= Hl) continue;   // stays zero
      const __nv_bfloat16* rbase = fbase + (size_t)row * Wl * tok_stride;
      uint32_t* srow = st + ((size_t)r * WS + 2) * NP;
      for (int e = tid; e < Wl * V8; e += kThreads) {
        const int v8 = e & (V8 - 1), x = e / V8;   // V8 is a power of two
        cp_async16(srow + (size_t)x * NP + v8 * 4, rbase + (size_t)x * tok_stride + v8 * 8);
      }
    }
    cp_async_commit();
  };
  issue(0);
  if (nst == 2 && T > 1) issue(1);

  for (int f = 0; f < T + 2; ++f) {
    if (f < T) {   // this frame's rows have landed (the next frame's may still be in flight)
      if (nst == 2 && f + 1 < T) cp_async_wait<1>();
      else cp_async_wait<0>();
    }
    __syncthreads();   // ... for every thread; the previous frame's ring and tile reads are done
    uint32_t* ring_t = ring + (size_t)(f % 5) * Wl * NP;
    if (f < T) {
      const uint32_t* st = stage0 + (size_t)(f % nst) * stage_words + cp;
      float2 acc[NXT];
#pragma unroll
      for (int i = 0; i < NXT; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int dy = 0; dy < 5; ++dy) {
        const int row = y + dy - 2;
        if (row < 0 || row >= Hl) continue;   // a zero row
        const uint32_t* srow = st + (size_t)dy * WS * NP + (size_t)xb * NP;
        float2 win[NXT + 4];
#pragma unroll
        for (int q = 0; q < NXT + 4; ++q) win[q] = bf2_to_f2(srow[(size_t)q * NP]);
#pragma unroll
        for (int i = 0; i < NXT; ++i) {
          float2 a = acc[i];
#pragma unroll
          for (int dx = 0; dx < 5; ++dx) a = ffma2(wsp[dy * 5 + dx], win[i + dx], a);
          acc[i] = a;
        }
      }
#pragma unroll
      for (int i = 0; i < NXT; ++i)
        if (xb + i < Wl) ring_t[(size_t)(xb + i) * NP + cp] = f2_to_bf2(acc[i]);
    } else {
      // frames past the clip contribute zero (temporal zero padding)
#pragma unroll
      for (int i = 0; i < NXT; ++i)
        if (xb + i < Wl) ring_t[(size_t)(xb + i) * NP + cp] = 0u;
    }
    __syncthreads();   // ring slot written; this frame's staging buffer has been read
    if (f + nst < T) issue(f + nst);
    if (f < 2) continue;
    // temporal filter, SiLU of output frame tout = f - 2
    const int tout = f - 2;
#pragma unroll
    for (int i = 0; i < NXT; ++i) {
      const int x = xb + i;
      if (x >= Wl) continue;
      float2 o = make_float2(0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int fr = tout + s - 2;
        if (fr < 0) continue;   // frames before the clip: zero padding
        o = ffma2(wtp[s], bf2_to_f2(ring[((size_t)(fr % 5) * Wl + x) * NP + cp]), o);
      }
      o.x = silu(o.x);
      o.y = silu(o.y);
      if (isv) {
        const size_t orow = (((size_t)bh * T + tout) * U + (size_t)y * Wl + x) * D;
        reinterpret_cast<uint32_t*>(out + orow)[cp] = f2_to_bf2(o);
      } else {
        reinterpret_cast<float2*>(tile + (size_t)x * D)[cp] = o;
      }
    }
    if (!isv) {   // L2 normalisation of each token of the row, one warp per token
      __syncthreads();
      const int warp = tid >> 5, lane = tid & 31;
      constexpr int PER = D / 32 > 0 ? D / 32 : 1;
      for (int x = warp; x < Wl; x += kThreads / 32) {
        float vals[PER];
        float ss = 0.f;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
          const int c = lane * PER + p;
          vals[p] = c < D ? tile[(size_t)x * D + c] : 0.f;
          ss = fmaf(vals[p], vals[p], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float sc = rsqrtf(ss + eps);
        const size_t orow = (((size_t)bh * T + tout) * U + (size_t)y * Wl + x) * D;
        if constexpr (PER == 4) {
          const uint2 w2 = make_uint2(f2_to_bf2(make_float2(vals[0] * sc, vals[1] * sc)),
                                      f2_to_bf2(make_float2(vals[2] * sc, vals[3] * sc)));
          reinterpret_cast<uint2*>(out + orow)[lane] = w2;
        } else {
#pragma unroll
          for (int p = 0; p < PER; ++p) {
            const int c = lane * PER + p;
            if (c < D) out[orow + c] = __float2bfloat16_rn(vals[p] * sc);
          }
        }
      }
    }
  }
}

// Q: L2 normalisation and the layout change, one warp per (token, head).
template <int D>
__global__ void __launch_bounds__(256)
k_prep_q(const __nv_bfloat16* __restrict__ qin, __nv_bfloat16* __restrict__ qout,
         int B, int H, int T, int U, float eps) {
  constexpr int PER = D / 32 > 0 ? D / 32 : 1;
  const size_t w = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const size_t ntok = (size_t)B * T * U;
  if (w >= ntok * H) return;
  const size_t tok = w / H;            // (b, t, u) in input order
  const int h = (int)(w - tok * H);
  const size_t b = tok / ((size_t)T * U), tu = tok - b * ((size_t)T * U);
  const __nv_bfloat16* src = qin + (tok * H + h) * D;
  float vals[PER];
  float ss = 0.f;
  if constexpr (PER == 4) {
    const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(src) + lane);
    const float2 a = bf2_to_f2(w2.x), b2 = bf2_to_f2(w2.y);
    vals[0] = a.x; vals[1] = a.y; vals[2] = b2.x; vals[3] = b2.y;
#pragma unroll
    for (int p = 0; p < 4; ++p) ss = fmaf(vals[p], vals[p], ss);
  } else {
#pragma unroll
    for (int p = 0; p < PER; ++p) {
      const int c = lane * PER + p;
      vals[p] = c < D ? __bfloat162float(src[c]) : 0.f;
      ss = fmaf(vals[p], vals[p], ss);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float sc = rsqrtf(ss + eps);
  __nv_bfloat16* dst = qout + ((b * H + h) * ((size_t)T * U) + tu) * D;
  if constexpr (PER == 4) {
    reinterpret_cast<uint2*>(dst)[lane] = make_uint2(f2_to_bf2(make_float2(vals[0] * sc, vals[1] * sc)),
                                                     f2_to_bf2(make_float2(vals[2] * sc, vals[3] * sc)));
  } else {
#pragma unroll
    for (int p = 0; p < PER; ++p) {
      const int c = lane * PER + p;
      if (c < D) dst[c] = __float2bfloat16_rn(vals[p] * sc);
    }
  }
}

}  // namespace prep
}  // namespace vda
