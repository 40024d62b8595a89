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
// Shared memory: nst staging buffers of rows y-2..y+2 (bf16 pairs), the
// head's spatial filter taps (fp32, [25][d]) and the fp32 output row of the
// L2 normalisation.
__host__ __device__ constexpr size_t kv_smem_bytes(int Wl, int D, int nst) {
  return (size_t)nst * kv_stage_bytes(Wl, D) + (size_t)25 * D * 4 + (size_t)Wl * D * 4;
}

// One CTA per (grid row y, batch-head, tensor K or V).  It walks the frames:
// the rows y-2..y+2 of a frame arrive by cp.async one frame ahead (two
// staging buffers when they fit, else one, refilled once the spatial filter
// has read it).  Thread = (channel pair cp, column slice xs): it computes the
// spatial 5 x 5 filter of row y for its NXT columns with packed fp32 FMAs and
// a register window, and, since the same thread produces every frame of its
// columns, it keeps the temporal filter's five running sums in registers:
// frame f adds tap 4 - j to the sum of output frame f - 2 + j, and output
// frame f - 2 is complete after frame f (then SiLU, and for K the L2
// normalisation over the token's channels, one warp per token).
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
  uint32_t* stage0 = reinterpret_cast<uint32_t*>(smem_raw);                        // [nst][5][WS][NP]
  float2* wsm = reinterpret_cast<float2*>(stage0 + (size_t)nst * stage_words);    // [25][NP]
  float* tile = reinterpret_cast<float*>(wsm + (size_t)25 * NP);                 // [Wl][D]

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

  float2 wtp[5];
#pragma unroll
  for (int s = 0; s < 5; ++s) wtp[s] = make_float2(__ldg(wt + (size_t)c0 * 5 + s), __ldg(wt + (size_t)(c0 + 1) * 5 + s));
  // the spatial taps of this head, [tap][channel pair]
  for (int e = tid; e < 25 * NP; e += kThreads) {
    const int q = e / NP, p2 = e - q * NP;
    wsm[e] = make_float2(__ldg(ws + (size_t)(2 * p2) * 25 + q), __ldg(ws + (size_t)(2 * p2 + 1) * 25 + q));
  }
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

  float2 tacc[5][NXT];   // running sums of output frames f - 2 .. f + 2
#pragma unroll
  for (int j = 0; j < 5; ++j)
#pragma unroll
    for (int i = 0; i < NXT; ++i) tacc[j][i] = make_float2(0.f, 0.f);

  for (int f = 0; f < T + 2; ++f) {
    if (f < T) cp_async_wait<0>();   // this frame's rows have landed (this thread's copies)
    __syncthreads();   // ... every thread's; the previous frame's staging and tile reads are done
    if (nst == 2 && f + 1 < T) issue(f + 1);   // into the buffer frame f - 1 used
    if (f < T) {
      const uint32_t* st = stage0 + (size_t)(f % nst) * stage_words + cp;
      float2 acc[NXT];
#pragma unroll
      for (int i = 0; i < NXT; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int dy = 0; dy < 5; ++dy) {
        const int row = y + dy - 2;
        if (row < 0 || row >= Hl) continue;   // a zero row
        float2 w5[5];
#pragma unroll
        for (int dx = 0; dx < 5; ++dx) w5[dx] = wsm[(dy * 5 + dx) * NP + cp];
        const uint32_t* srow = st + (size_t)dy * WS * NP + (size_t)xb * NP;
        float2 win[NXT + 4];
#pragma unroll
        for (int q = 0; q < NXT + 4; ++q) win[q] = bf2_to_f2(srow[(size_t)q * NP]);
#pragma unroll
        for (int i = 0; i < NXT; ++i) {
          float2 a = acc[i];
#pragma unroll
          for (int dx = 0; dx < 5; ++dx) a = ffma2(w5[dx], win[i + dx], a);
          acc[i] = a;
        }
      }
      // frame f is tap 4 - j of output frame f - 2 + j
#pragma unroll
      for (int j = 0; j < 5; ++j)
#pragma unroll
        for (int i = 0; i < NXT; ++i) tacc[j][i] = ffma2(wtp[4 - j], acc[i], tacc[j][i]);
      if (nst == 1) {   // refill the only staging buffer once every thread has read it
        __syncthreads();
        if (f + 1 < T) issue(f + 1);
      }
    }
    if (f >= 2) {   // output frame tout = f - 2 is complete: SiLU
      const int tout = f - 2;
#pragma unroll
      for (int i = 0; i < NXT; ++i) {
        const int x = xb + i;
        if (x >= Wl) continue;
        float2 o = tacc[0][i];
        o.x = silu(o.x);
        o.y = silu(o.y);
        if (isv) {
          const size_t orow = (((size_t)bh * T + tout) * U + (size_t)y * Wl + x) * D;
          reinterpret_cast<uint32_t*>(out + orow)[cp] = f2_to_bf2(o);
        } else {
          reinterpret_cast<float2*>(tile + (size_t)x * D)[cp] = o;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < NXT; ++i) tacc[j][i] = tacc[j + 1][i];
#pragma unroll
    for (int i = 0; i < NXT; ++i) tacc[4][i] = make_float2(0.f, 0.f);
    if (!isv && f >= 2) {   // L2 normalisation of each token of the row, one warp per token
      const int tout = f - 2;
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
