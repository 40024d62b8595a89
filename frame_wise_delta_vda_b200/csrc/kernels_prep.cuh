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

constexpr int kThreads = 256;
constexpr int kMaxWc = 16;   // grid columns per thread

// Shared memory of k_prep_kv: staged input rows (bf16) and the ring of the
// last five frames' spatial results (bf16 pairs); the output row for the L2
// reduction (fp32) reuses the staging area once the spatial filter is done.
// 20 bytes per column and channel, so two CTAs fit on an SM.
__host__ __device__ constexpr size_t kv_smem_bytes(int Wl, int D) {
  return (size_t)Wl * D * (5 * 2 + 5 * 2);
}

// One CTA per (grid row y, batch-head, tensor K or V).  It walks the frames:
// for each input frame it stages rows y-2..y+2, computes the spatial filter
// for row y into a five-frame ring, and, two frames behind, the temporal
// filter, SiLU and (K only) the L2 normalisation of output frame t.  Thread =
// (channel pair cp, column slice xs): channel pairs use packed fp32 FMAs.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
k_prep_kv(const __nv_bfloat16* __restrict__ kin, const __nv_bfloat16* __restrict__ vin,
          const float* __restrict__ wk_s, const float* __restrict__ wk_t,
          const float* __restrict__ wv_s, const float* __restrict__ wv_t,
          __nv_bfloat16* __restrict__ kout, __nv_bfloat16* __restrict__ vout,
          int H, int T, int Hl, int Wl, float eps) {
  constexpr int NP = D / 2;              // channel pairs
  constexpr int NS = kThreads / NP;      // column slices
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem_raw);                      // [5][Wl][NP] bf16 pairs
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem_raw + (size_t)5 * Wl * D * 2);  // [5][Wl][NP] bf16 pairs
  float* tile = reinterpret_cast<float*>(smem_raw);                                // [Wl][D], over the stage

  const int y = blockIdx.x, bh = blockIdx.y, isv = blockIdx.z;
  const int Hn = H;
  const int b = bh / Hn, h = bh - (bh / Hn) * Hn;
  const __nv_bfloat16* in = isv ? vin : kin;
  __nv_bfloat16* out = isv ? vout : kout;
  const float* ws = (isv ? wv_s : wk_s) + (size_t)h * D * 25;
  const float* wt = (isv ? wv_t : wk_t) + (size_t)h * D * 5;
  const int U = Hl * Wl;
  const int tid = threadIdx.x, cp = tid % NP, xs = tid / NP;
  const int c0 = 2 * cp;
  const int Wc = (Wl + NS - 1) / NS;
  const int xb = xs * Wc, nx = max(0, min(Wc, Wl - xb));

  float2 wsp[25], wtp[5];
#pragma unroll
  for (int q = 0; q < 25; ++q) wsp[q] = make_float2(__ldg(ws + (size_t)c0 * 25 + q), __ldg(ws + (size_t)(c0 + 1) * 25 + q));
#pragma unroll
  for (int s = 0; s < 5; ++s) wtp[s] = make_float2(__ldg(wt + (size_t)c0 * 5 + s), __ldg(wt + (size_t)(c0 + 1) * 5 + s));

  const size_t tok_stride = (size_t)Hn * D;   // elements between consecutive tokens of the input
  for (int tin = 0; tin < T + 2; ++tin) {
    __syncthreads();   // the previous frame's stage and ring reads are done
    if (tin < T) {
      // stage rows y-2..y+2 of frame tin (zero outside the grid): 16-B vectors
      constexpr int V8 = D / 8;
      const size_t frame_tok = ((size_t)b * T + tin) * U;
      for (int e = tid; e < Wl * V8; e += kThreads) {
        const int v8 = e % V8, x = e / V8;   // V8 is a power of two
#pragma unroll
        for (int r = 0; r < 5; ++r) {
          const int row = y + r - 2;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (row >= 0 && row < Hl) {
            const size_t tok = frame_tok + (size_t)row * Wl + x;
            val = __ldg(reinterpret_cast<const uint4*>(in + tok * tok_stride + (size_t)h * D) + v8);
          }
          reinterpret_cast<uint4*>(stage)[((size_t)r * Wl + x) * V8 + v8] = val;
        }
      }
    }
    __syncthreads();
    // spatial filter of row y for this thread's columns and channel pair
    uint32_t* ring_t = ring + (size_t)(tin % 5) * Wl * NP;
    if (tin < T) {
      float2 acc[kMaxWc];
#pragma unroll
      for (int xi = 0; xi < kMaxWc; ++xi) acc[xi] = make_float2(0.f, 0.f);
#pragma unroll
      for (int dy = 0; dy < 5; ++dy) {
        const int row = y + dy - 2;
        if (row < 0 || row >= Hl) continue;
        const uint32_t* srow = stage + (size_t)dy * Wl * NP + cp;
        auto at = [&](int x) -> float2 {
          return (x >= 0 && x < Wl) ? bf2_to_f2(srow[(size_t)x * NP]) : make_float2(0.f, 0.f);
        };
        float2 w0 = at(xb - 2), w1 = at(xb - 1), w2 = at(xb), w3 = at(xb + 1), w4 = at(xb + 2);
#pragma unroll
        for (int xi = 0; xi < kMaxWc; ++xi) {
          if (xi < nx) {
            float2 a = acc[xi];
            a = ffma2(wsp[dy * 5 + 0], w0, a);
            a = ffma2(wsp[dy * 5 + 1], w1, a);
            a = ffma2(wsp[dy * 5 + 2], w2, a);
            a = ffma2(wsp[dy * 5 + 3], w3, a);
            a = ffma2(wsp[dy * 5 + 4], w4, a);
            acc[xi] = a;
            w0 = w1; w1 = w2; w2 = w3; w3 = w4;
            w4 = at(xb + xi + 3);
          }
        }
      }
#pragma unroll
      for (int xi = 0; xi < kMaxWc; ++xi)
        if (xi < nx) ring_t[(size_t)(xb + xi) * NP + cp] = f2_to_bf2(acc[xi]);
    } else {
      // frames past the clip contribute zero (temporal zero padding)
#pragma unroll
      for (int xi = 0; xi < kMaxWc; ++xi)
        if (xi < nx) ring_t[(size_t)(xb + xi) * NP + cp] = 0u;
    }
    __syncthreads();
    if (tin < 2) continue;
    // temporal filter, SiLU of output frame tout = tin - 2
    const int tout = tin - 2;
#pragma unroll
    for (int xi = 0; xi < kMaxWc; ++xi) {
      if (xi >= nx) continue;
      const int x = xb + xi;
      float2 o = make_float2(0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int f = tout + s - 2;
        if (f < 0) continue;   // frames before the clip: zero padding
        o = ffma2(wtp[s], bf2_to_f2(ring[((size_t)(f % 5) * Wl + x) * NP + cp]), o);
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
