// kernels_simt.cuh - FP32 SIMT kernels of the VDA path.
//
// These serve the float32-I/O specialisation and the head dims 16 and 32;
// bf16 at d = 128 and d = 64 uses the tcgen05 kernels.  The small-matrix
// inverse here is the FP32 path for every size but d = 128 with bf16.
//
// Paper: "Video DeltaNet" (arXiv 2609.20744): Eq. 3b (frame statistics),
// Eq. 5 / Appendix A.1 (M_t = (I + A_t)^{-1}, S_t = (S_{t-1} + B_t) M_t),
// Appendix A.3 (boundary gather), Eq. 1a/1c (readout, RMSNorm, gate).
#pragma once

#include "common.cuh"

namespace vda {

// ---------------------------------------------------------------------------
// Frame statistics (Eq. 3b), one CTA per frame-head:
//   A = K^T Diag(beta) K  [d x d],   B = V^T Diag(beta) K  [d x d]
// computed together as O = [K | V]^T (Diag(beta) K), O in R^{2d x d}.
// 256 threads; thread (tr, tj) owns rows r = i*32 + tr and columns
// c = jj*8 + tj of O.  Tokens are staged 32 at a time in shared memory.
// ---------------------------------------------------------------------------
template <int D, typename TIn>
__global__ void __launch_bounds__(256)
k_stats_simt(const TIn* __restrict__ K, const TIn* __restrict__ V,
             const float* __restrict__ beta, int U,
             float* __restrict__ A_out, float* __restrict__ B_out) {
  constexpr int TU = 32;
  constexpr int RR = D / 16;  // rows per thread (2D rows over 32 row-threads)
  constexpr int RJ = D / 8;   // columns per thread (D columns over 8 column-threads)
  __shared__ float sX[TU][2 * D];
  __shared__ float sBK[TU][D];

  const size_t fh = blockIdx.x;
  const TIn* Kf = K + fh * (size_t)U * D;
  const TIn* Vf = V + fh * (size_t)U * D;
  const float* bf = beta + fh * (size_t)U;
  const int tid = threadIdx.x;
  const int tj = tid & 7, tr = tid >> 3;

  float acc[RR][RJ];
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RJ; ++j) acc[i][j] = 0.f;

  for (int u0 = 0; u0 < U; u0 += TU) {
    for (int e = tid; e < TU * D; e += 256) {
      const int u = e / D, c = e - (e / D) * D;
      float kx = 0.f, vx = 0.f, b = 0.f;
      if (u0 + u < U) {
        kx = to_f32(Kf[(size_t)(u0 + u) * D + c]);
        vx = to_f32(Vf[(size_t)(u0 + u) * D + c]);
        b = bf[u0 + u];
      }
      sX[u][c] = kx;
      sX[u][D + c] = vx;
      sBK[u][c] = b * kx;
    }
    __syncthreads();
#pragma unroll 4
    for (int u = 0; u < TU; ++u) {
      float x[RR], y[RJ];
#pragma unroll
      for (int i = 0; i < RR; ++i) x[i] = sX[u][i * 32 + tr];
#pragma unroll
      for (int j = 0; j < RJ; ++j) y[j] = sBK[u][j * 8 + tj];
#pragma unroll
      for (int i = 0; i < RR; ++i)
#pragma unroll
        for (int j = 0; j < RJ; ++j) acc[i][j] = fmaf(x[i], y[j], acc[i][j]);
    }
    __syncthreads();
  }

  float* Af = A_out + fh * (size_t)D * D;
  float* Bf = B_out + fh * (size_t)D * D;
#pragma unroll
  for (int i = 0; i < RR; ++i) {
    const int r = i * 32 + tr;
#pragma unroll
    for (int j = 0; j < RJ; ++j) {
      const int c = j * 8 + tj;
      if (r < D) Af[(size_t)r * D + c] = acc[i][j];
      else Bf[(size_t)(r - D) * D + c] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// M = (I + A)^{-1} in place, one CTA per frame-head (Eq. 5; Appendix A.1).
// I + A is symmetric positive definite with eigenvalues >= 1, so Gauss-Jordan
// elimination without pivoting is stable (every pivot is >= 1).  The matrix
// lives in registers: 16 x 16 threads, each holding a (D/16) x (D/16) block;
// the pivot row and column are broadcast through double-buffered shared
// memory, one barrier per elimination step.
// With `img` (d = 64, the tensor-core scan) M is also written as that scan's
// operand image: element (j, k) = M[k][j] in row k of 64 bf16 (128 B, 128-B
// swizzle), hi part then lo part (8 KB each) per frame-head.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
k_gj_inverse(float* __restrict__ AM, uint8_t* __restrict__ img) {
  constexpr int BS = D / 16;
  __shared__ float s_row[2][D];
  __shared__ float s_col[2][D];

  float* Mx = AM + (size_t)blockIdx.x * D * D;
  const int tid = threadIdx.x;
  const int bi = tid >> 4, bj = tid & 15;
  const int r0 = bi * BS, c0 = bj * BS;

  float a[BS][BS];
#pragma unroll
  for (int i = 0; i < BS; ++i)
#pragma unroll
    for (int j = 0; j < BS; ++j)
      a[i][j] = Mx[(size_t)(r0 + i) * D + c0 + j] + ((r0 + i) == (c0 + j) ? 1.f : 0.f);

  for (int kb = 0; kb < 16; ++kb) {
#pragma unroll
    for (int kk = 0; kk < BS; ++kk) {
      const int k = kb * BS + kk;
      const int buf = k & 1;
      if (bi == kb) {
#pragma unroll
        for (int j = 0; j < BS; ++j) s_row[buf][c0 + j] = a[kk][j];
      }
      if (bj == kb) {
#pragma unroll
        for (int i = 0; i < BS; ++i) s_col[buf][r0 + i] = a[i][kk];
      }
      __syncthreads();
      const float pinv = 1.0f / s_row[buf][k];
      float c[BS], rs[BS];
#pragma unroll
      for (int i = 0; i < BS; ++i) c[i] = s_col[buf][r0 + i];
#pragma unroll
      for (int j = 0; j < BS; ++j) rs[j] = s_row[buf][c0 + j] * pinv;
#pragma unroll
      for (int i = 0; i < BS; ++i)
#pragma unroll
        for (int j = 0; j < BS; ++j) a[i][j] = fmaf(-c[i], rs[j], a[i][j]);
      if (bi == kb) {
#pragma unroll
        for (int j = 0; j < BS; ++j) a[kk][j] = rs[j];
      }
      if (bj == kb) {
#pragma unroll
        for (int i = 0; i < BS; ++i) a[i][kk] = -c[i] * pinv;
      }
      if (bi == kb && bj == kb) a[kk][kk] = pinv;
    }
  }
#pragma unroll
  for (int i = 0; i < BS; ++i)
#pragma unroll
    for (int j = 0; j < BS; ++j) Mx[(size_t)(r0 + i) * D + c0 + j] = a[i][j];
  if constexpr (D == 64) {
    if (img) {   // row k = r0 + i holds M[k][c0 .. c0 + 3]: 8 contiguous bytes of one 16-B chunk
      uint8_t* dst = img + (size_t)blockIdx.x * 16384;
#pragma unroll
      for (int i = 0; i < BS; ++i) {
        const uint32_t k = (uint32_t)(r0 + i);
        const uint32_t off = k * 128u + (((((uint32_t)c0 >> 3) ^ (k & 7u)) & 7u) << 4) + (((uint32_t)c0 & 7u) << 1);
        __nv_bfloat162 h01 = __floats2bfloat162_rn(a[i][0], a[i][1]), h23 = __floats2bfloat162_rn(a[i][2], a[i][3]);
        const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
        __nv_bfloat162 l01 = __floats2bfloat162_rn(a[i][0] - f01.x, a[i][1] - f01.y);
        __nv_bfloat162 l23 = __floats2bfloat162_rn(a[i][2] - f23.x, a[i][3] - f23.y);
        *reinterpret_cast<uint2*>(dst + off) =
            make_uint2(*reinterpret_cast<uint32_t*>(&h01), *reinterpret_cast<uint32_t*>(&h23));
        *reinterpret_cast<uint2*>(dst + 8192 + off) =
            make_uint2(*reinterpret_cast<uint32_t*>(&l01), *reinterpret_cast<uint32_t*>(&l23));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Bidirectional scan (Section 2.2; Eq. 5, with the decay of Eq. 2 when alpha
// is given), SIMT:
//   forward  P_t = (P_{t-1} Diag(alpha_t) + B_t) M_t  for t = 0..T-1 from S0_fwd
//   reverse  R_t = (R_{t+1} Diag(alpha_t) + B_t) M_t  for t = T-1..0 from S0_rev
// (alpha NULL: no decay)
// Right-multiplication acts on each row of S independently, so a chain
// (b, h, dir) is split over CTAs by blocks of RB rows with no communication.
// Thread j owns column j of its rows.  Chunk-boundary states are written to
// states [2][BH][NC+1][D][D]: fwd[j] after frames [0, jC), rev[j] after
// frames [jC, T).
// ---------------------------------------------------------------------------
template <int D, int RB>
__global__ void __launch_bounds__(D)
k_scan_simt(const float* __restrict__ M, const float* __restrict__ Bm,
            const float* __restrict__ S0f, const float* __restrict__ S0r,
            const float* __restrict__ alpha, float* __restrict__ states, int BH, int T, int chunk, int NC) {
  __shared__ float sX[RB][D];
  const int bh = blockIdx.x, dir = blockIdx.y, r0 = blockIdx.z * RB, j = threadIdx.x;
  const size_t DD = (size_t)D * D;
  const float* S0 = dir == 0 ? S0f : S0r;
  float* st = states + ((size_t)dir * BH + bh) * (size_t)(NC + 1) * DD;

  float s[RB];
#pragma unroll
  for (int i = 0; i < RB; ++i)
    s[i] = S0 ? S0[(size_t)bh * DD + (size_t)(r0 + i) * D + j] : 0.f;
  {
    const int j0 = dir == 0 ? 0 : NC;
#pragma unroll
    for (int i = 0; i < RB; ++i) st[(size_t)j0 * DD + (size_t)(r0 + i) * D + j] = s[i];
  }

  for (int step = 0; step < T; ++step) {
    const int t = dir == 0 ? step : T - 1 - step;
    const float* Bt = Bm + ((size_t)bh * T + t) * DD;
    const float* Mt = M + ((size_t)bh * T + t) * DD;
    if (alpha) {   // S_bar = S Diag(alpha_t): thread j holds key column j (Eq. 2)
      const float a = __ldg(alpha + ((size_t)bh * T + t) * D + j);
#pragma unroll
      for (int i = 0; i < RB; ++i) sX[i][j] = fmaf(s[i], a, Bt[(size_t)(r0 + i) * D + j]);
    } else {
#pragma unroll
      for (int i = 0; i < RB; ++i) sX[i][j] = s[i] + Bt[(size_t)(r0 + i) * D + j];
    }
    __syncthreads();
    float acc[RB];
#pragma unroll
    for (int i = 0; i < RB; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < D; ++kk) {
      const float m = __ldg(Mt + (size_t)kk * D + j);
#pragma unroll
      for (int i = 0; i < RB; ++i) acc[i] = fmaf(sX[i][kk], m, acc[i]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RB; ++i) s[i] = acc[i];

    int jb = -1;
    if (dir == 0) {
      if ((t + 1) % chunk == 0 || t == T - 1) jb = (t + chunk) / chunk;
    } else if (t % chunk == 0) {
      jb = t / chunk;
    }
    if (jb >= 0) {
#pragma unroll
      for (int i = 0; i < RB; ++i) st[(size_t)jb * DD + (size_t)(r0 + i) * D + j] = s[i];
    }
  }
}

// ---------------------------------------------------------------------------
// Decay bridge of Appendix A.3 (Eq. A.4): for query frame t in chunk c with
// window [l, h] (chunks c-w .. c+w clipped to the clip),
//   bridge[b,h,t][0][k] = prod_{r=l..t} alpha_r[k]   (applied to P_{l-1})
//   bridge[b,h,t][1][k] = prod_{r=t..h} alpha_r[k]   (applied to R_{h+1})
// One thread per (b, h, t, k).
// ---------------------------------------------------------------------------
__global__ void k_decay_bridge(const float* __restrict__ alpha, int BH, int T, int D, int chunk,
                               int window_chunks, float* __restrict__ bridge) {
  const size_t n = (size_t)BH * T * D;
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const int k = (int)(idx % (size_t)D);
  const size_t ft = idx / (size_t)D;
  const int t = (int)(ft % (size_t)T);
  const size_t bh = ft / (size_t)T;
  const int c = t / chunk;
  const int lo = max(0, (c - window_chunks) * chunk);
  const int hi = min(T - 1, (c + window_chunks + 1) * chunk - 1);
  const float* a = alpha + bh * (size_t)T * D + k;
  float pl = 1.f, pr = 1.f;
  for (int r = lo; r <= t; ++r) pl *= __ldg(a + (size_t)r * D);
  for (int r = t; r <= hi; ++r) pr *= __ldg(a + (size_t)r * D);
  bridge[(ft * 2) * D + k] = pl;
  bridge[(ft * 2 + 1) * D + k] = pr;
}

// ---------------------------------------------------------------------------
// Readout (Appendix A.3 gather + Eq. 1a + Eq. 1c), SIMT.  One CTA column per
// (b, h, chunk c), or per (b, h, frame t) with the decay bridge; gridDim.y
// CTAs split the unit's tokens.  The CTA builds
//   S~ = fwd[max(0, c - w)] + rev[min(NC, c + w + 1)]
// (with the bridge: fwd[..] Diag(bridge[t][0]) + rev[..] Diag(bridge[t][1]))
// transposed, in shared memory, then each warp takes groups of tokens:
// G = min(D, 32) lanes per token slot, lane li of a slot computes outputs
// i = li + G*m; NT tokens per slot share every S~ load.
//   y = sigmoid(g) * w * o / sqrt(mean(o^2) + eps)
// ---------------------------------------------------------------------------
template <int D, typename TIo>
struct ReadoutSimtCfg {
  static constexpr int G = D < 32 ? D : 32;
  static constexpr int SP = 32 / G;     // token slots per warp
  static constexpr int NT = 4;          // tokens per slot per iteration
  static constexpr int PER = D / G;     // outputs per lane
  static constexpr int WARPS = 8;
  static constexpr int TOK_PER_WARP = SP * NT;
  static constexpr size_t smem_bytes() {
    return (size_t)D * D * sizeof(float) + (size_t)WARPS * TOK_PER_WARP * D * sizeof(float);
  }
};

template <int D, typename TIo>
__global__ void __launch_bounds__(256)
k_readout_simt(const TIo* __restrict__ Q, const TIo* __restrict__ Gt,
               const float* __restrict__ w, const float* __restrict__ states,
               const float* __restrict__ bridge, TIo* __restrict__ out, int BH, int T, int U, int chunk,
               int NC, int window_chunks, float eps) {
  using Cfg = ReadoutSimtCfg<D, TIo>;
  extern __shared__ float smem[];
  float* sT = smem;                                       // [D][D], sT[k][i] = S~[i][k]
  float* sQ = smem + (size_t)D * D;                       // [WARPS][TOK_PER_WARP][D]

  // unit = one chunk, or one frame with the decay bridge (its read state
  // changes from frame to frame)
  const int NU = bridge ? T : NC;
  const int bh = blockIdx.x / NU, u = blockIdx.x - (blockIdx.x / NU) * NU;
  const int c = bridge ? u / chunk : u;
  const size_t DD = (size_t)D * D;
  const int jf = max(0, c - window_chunks);
  const int jr = min(NC, c + window_chunks + 1);
  const float* Sf = states + ((size_t)0 * BH + bh) * (size_t)(NC + 1) * DD + (size_t)jf * DD;
  const float* Sr = states + ((size_t)1 * BH + bh) * (size_t)(NC + 1) * DD + (size_t)jr * DD;
  if (bridge) {
    const float* al = bridge + (((size_t)bh * T + u) * 2) * D;
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
      const int i = e / D, k = e - (e / D) * D;
      sT[(size_t)k * D + i] = fmaf(Sf[e], al[k], Sr[e] * al[D + k]);
    }
  } else {
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
      const int i = e / D, k = e - (e / D) * D;
      sT[(size_t)k * D + i] = Sf[e] + Sr[e];
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = lane / Cfg::G, li = lane - (lane / Cfg::G) * Cfg::G;
  float* myQ = sQ + (size_t)warp * Cfg::TOK_PER_WARP * D;

  const int f0 = bridge ? u : c * chunk, f1 = bridge ? u + 1 : min(T, (c + 1) * chunk);
  const size_t tok0 = ((size_t)bh * T + f0) * U;          // first token row of the chunk
  const int ntok = (f1 - f0) * U;
  float wv[Cfg::PER];
#pragma unroll
  for (int m = 0; m < Cfg::PER; ++m) wv[m] = w[li + Cfg::G * m];

  const int groups = (ntok + Cfg::TOK_PER_WARP - 1) / Cfg::TOK_PER_WARP;
  for (int gidx = blockIdx.y * Cfg::WARPS + warp; gidx < groups; gidx += gridDim.y * Cfg::WARPS) {
    const int t0 = gidx * Cfg::TOK_PER_WARP;
    // stage the group's queries: token (slot, n) is t0 + slot*NT + n
    for (int e = lane; e < Cfg::TOK_PER_WARP * D; e += 32) {
      const int tt = e / D;
      const int tok = t0 + tt;
      myQ[e] = tok < ntok ? to_f32(Q[(tok0 + tok) * D + (e - tt * D)]) : 0.f;
    }
    __syncwarp();
    float acc[Cfg::NT][Cfg::PER];
#pragma unroll
    for (int n = 0; n < Cfg::NT; ++n)
#pragma unroll
      for (int m = 0; m < Cfg::PER; ++m) acc[n][m] = 0.f;
    const float* qs = myQ + (size_t)slot * Cfg::NT * D;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      float sv[Cfg::PER];
#pragma unroll
      for (int m = 0; m < Cfg::PER; ++m) sv[m] = sT[(size_t)k * D + li + Cfg::G * m];
#pragma unroll
      for (int n = 0; n < Cfg::NT; ++n) {
        const float qk = qs[n * D + k];
#pragma unroll
        for (int m = 0; m < Cfg::PER; ++m) acc[n][m] = fmaf(sv[m], qk, acc[n][m]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int n = 0; n < Cfg::NT; ++n) {
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < Cfg::PER; ++m) ss = fmaf(acc[n][m], acc[n][m], ss);
#pragma unroll
      for (int off = Cfg::G / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off, Cfg::G);
      const float rinv = rsqrtf(ss / (float)D + eps);
      const int tok = t0 + slot * Cfg::NT + n;
      if (tok < ntok) {
        const size_t row = (tok0 + tok) * D;
#pragma unroll
        for (int m = 0; m < Cfg::PER; ++m) {
          const int i = li + Cfg::G * m;
          const float g = to_f32(Gt[row + i]);
          out[row + i] = from_f32<TIo>(acc[n][m] * rinv * wv[m] * sigmoidf_accurate(g));
        }
      }
    }
  }
}

}  // namespace vda
