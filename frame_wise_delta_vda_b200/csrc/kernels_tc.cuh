// kernels_tc.cuh - sm_100a tensor-core kernels of the VDA path for d = 128
// and d = 64 with bf16 I/O: TMA-fed tcgen05 MMAs accumulating in TMEM.
//
// Paper: "Video DeltaNet" (arXiv 2609.20744).
//   k_stats_tc    Eq. 3b: A_t = K^T Diag(beta) K, B_t = V^T Diag(beta) K
//   k_inverse_tc  Eq. 5 / Appendix A.1: M_t = (I + A_t)^{-1} by a block sweep
//                 on the tensor cores, written as the bf16 hi/lo operand image
//                 the scan feeds to the tensor cores
//   k_scan_tc     Section 2.2 + Eq. 5: S_t = (S_{t-1} + B_t) M_t, both
//                 directions, fp32 state, 3-product bf16 hi/lo split MMAs;
//                 per-frame chains or the chunk-wise form of Section 5
//   k_readout_tc  Appendix A.3 (Eq. A.4) gather, Eq. 1a readout o = S~ q,
//                 Eq. 1c RMSNorm + sigmoid gate, bf16 store (d = 128, 64)
//   k_stats64_tc, k_scan64_tc  the d = 64 Gram kernel and scans (the inverse
//                 at d = 64 is the FP32 Gauss-Jordan kernel of kernels_simt.cuh)
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <utility>

#include "common.cuh"
#include "kernels_simt.cuh"
#include "tc_ptx.cuh"
#include "vda.h"

namespace vda {
namespace tc {

using namespace vda::ptx;

constexpr int kD = 128;
constexpr size_t kDD = (size_t)kD * kD;
constexpr uint32_t kImgHalf = 32768;   // one bf16 128x128 operand image
constexpr uint32_t kImgBytes = 65536;  // hi + lo images
// A_t is symmetric, so the Gram kernel stores its upper block triangle only:
// 16 x 16 blocks (br, bc) with br <= bc, block (br, bc) at
// (bc (bc + 1) / 2 + br) * 256 floats, element (r, c) of a block at c * 16 + r.
constexpr size_t kATri = 36 * 256;      // floats per frame-head
__host__ __device__ constexpr size_t atri_block(int br, int bc) { return (size_t)((bc * (bc + 1)) / 2 + br) * 256; }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ===========================================================================
// k_stats_tc: per frame-head, with tokens on the MMA's K dimension,
//   D[128 x 256] = (beta K)_hi^T [K | V]  +  (beta K)_lo^T [K | V]
// so D[:, 0:128] = A and D[:, 128:256] = B^T with beta*K split into bf16
// hi + lo: ~16 significant bits, which the correlated-key workload needs in
// B, and which keeps A symmetric to ~2^-16 for the symmetric-sweep inverse.  Both operands are MN-major: a TMA box of
// 64 channels x 64 tokens lands as 64 rows of 128 B with the 128-B swizzle.
//
// Persistent CTAs (one per SM) walk frame-heads fh = blockIdx.x + i*grid.
// Warps: 0-3 epilogue (TMEM -> A (upper block triangle) and B, fp32,
//        coalesced; optionally the full A for the debug output),
//        4-11 scale (beta*K hi/lo), 12 TMA producer, 13 MMA issuer + TMEM
//        owner.  Two TMEM accumulators: the epilogue of one frame-head
//        overlaps the MMAs of the next.
// Load stage s holds K0 K1 V0 V1 (TMA, 4 x 8 KB; four stages keep 128 KB of
// loads in flight); scaled buffer b holds H0 H1 (hi), L0 L1 (lo) (4 x 8 KB,
// two buffers: they live only from the scaling to the MMAs).
// TMEM: two 256-column accumulators (512 columns), so the epilogue of one
// frame-head overlaps the MMAs of the next.
// ===========================================================================
struct StatsCfg {
  static constexpr int UT = 64;
  static constexpr int NST = 4;                      // load stages
  static constexpr int NSC = 2;                      // scaled buffers
  static constexpr uint32_t BLK = UT * 128;          // 8192
  static constexpr uint32_t STAGE = 4 * BLK;         // K0 K1 V0 V1
  static constexpr uint32_t SCBUF = 4 * BLK;         // H0 H1 L0 L1
  static constexpr uint32_t OFF_SC = NST * STAGE;
  static constexpr uint32_t OFF_L = 2 * BLK;         // lo half within a scaled buffer
  static constexpr int NSCALE = 256;                 // scale threads: 64 rows x 4 column quarters
  static constexpr int WARP_PROD = 4 + NSCALE / 32;  // TMA producer
  static constexpr int WARP_MMA = WARP_PROD + 1;     // MMA issuer + TMEM owner
  static constexpr int THREADS = 32 * (WARP_MMA + 1);
  static constexpr uint32_t BAR_OFF = OFF_SC + NSC * SCBUF;
  static constexpr int NBAR = 2 * NST + 2 * NSC + 5;
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};

// byte offset of element (r, k), k < 16, in a K-major no-swizzle image
__device__ __forceinline__ uint32_t kimg16(uint32_t r, uint32_t k) {
  return (r >> 3) * 256u + (k >> 3) * 128u + (r & 7u) * 16u + (k & 7u) * 2u;
}

// 16 fp32 values -> bf16 hi and lo rows of two no-swizzle images
__device__ __forceinline__ void store_row16_hilo(uint32_t img_hi, uint32_t img_lo, uint32_t r, const float (&x)[16]) {
#pragma unroll
  for (int kc = 0; kc < 2; ++kc) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float h0, l0, h1, l1;
      split_bf16(x[8 * kc + 2 * q], h0, l0);
      split_bf16(x[8 * kc + 2 * q + 1], h1, l1);
      hw[q] = pack_bf16(h0, h1);
      lw[q] = pack_bf16(l0, l1);
    }
    const uint32_t off = kimg16(r, 8u * kc);
    st_shared_v4(img_hi + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
    st_shared_v4(img_lo + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
  }
}

__device__ __forceinline__ uint32_t mimg_offset(int j, int k) {
  return (uint32_t)(j >> 6) * 16384u + sw128_offset((uint32_t)k, (uint32_t)(j & 63));
}

// 8 fp32 values -> one 16-B chunk of the bf16 hi image and of the lo image
__device__ __forceinline__ void store_img_chunk(uint8_t* img, uint32_t off, const float (&x)[8]) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float h0, l0, h1, l1;
    split_bf16(x[2 * q], h0, l0);
    split_bf16(x[2 * q + 1], h1, l1);
    hw[q] = pack_bf16(h0, h1);
    lw[q] = pack_bf16(l0, l1);
  }
  *reinterpret_cast<uint4*>(img + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *reinterpret_cast<uint4*>(img + kImgHalf + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

__global__ void __launch_bounds__(StatsCfg::THREADS, 1)
k_stats_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
           const float* __restrict__ beta, int U, int FH, float* __restrict__ A_out,
           float* __restrict__ B_out, float* __restrict__ A_full) {
  using C = StatsCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
  // barrier indices
  const int FULL = 0, EMPTY = C::NST, SCALED = 2 * C::NST, SEMPTY = 2 * C::NST + C::NSC,
            TFULL = 2 * C::NST + 2 * C::NSC, TEMPTY = TFULL + 2, DRAIN = TFULL + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(BAR(FULL + s), 1);
      mbar_init(BAR(EMPTY + s), 1);
    }
    for (int b = 0; b < C::NSC; ++b) {
      mbar_init(BAR(SCALED + b), C::NSCALE);
      mbar_init(BAR(SEMPTY + b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(TFULL + b), 1);
      mbar_init(BAR(TEMPTY + b), 128);
    }
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched after the previous grid with programmatic serialisation: the
  // prologue above overlapped its tail; its results are visible from here.
  // Only then may the next grid start, so that every CTA of this one is
  // resident before a CTA of the next can take an SM
  grid_wait_prerequisites();
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const int nt = (U + C::UT - 1) / C::UT;
  int last_it[C::NST];   // producer: last iteration issued on each stage
  for (int s = 0; s < C::NST; ++s) last_it[s] = -1;

  if (warp == C::WARP_PROD) {
    // ---------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int fh = blockIdx.x; ok && fh < FH; fh += gridDim.x) {
        for (int tile = 0; tile < nt; ++tile, ++it) {
          const uint32_t s = it % C::NST, ph = (it / C::NST) & 1u;
          if (!mbar_wait(BAR(EMPTY + s), ph ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(BAR(FULL + s), 4 * C::BLK);
          const uint32_t st = sbase + s * C::STAGE;
          tma_load_3d(st + 0 * C::BLK, &tmK, 0, tile * C::UT, fh, BAR(FULL + s));
          tma_load_3d(st + 1 * C::BLK, &tmK, 64, tile * C::UT, fh, BAR(FULL + s));
          tma_load_3d(st + 2 * C::BLK, &tmV, 0, tile * C::UT, fh, BAR(FULL + s));
          tma_load_3d(st + 3 * C::BLK, &tmV, 64, tile * C::UT, fh, BAR(FULL + s));
          last_it[s] = (int)it;
        }
      }
    }
  } else if (warp == C::WARP_MMA) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdN256 = idesc_bf16(128, 256, 1, 1);
      uint32_t it = 0, lf = 0;
      bool ok = true;
      for (int fh = blockIdx.x; ok && fh < FH; fh += gridDim.x, ++lf) {
        const uint32_t buf = lf & 1u, bph = (lf >> 1) & 1u;
        if (!mbar_wait(BAR(TEMPTY + buf), bph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * 256u;
        for (int tile = 0; tile < nt; ++tile, ++it) {
          const uint32_t s = it % C::NST;
          const uint32_t b = it % C::NSC, bph2 = (it / C::NSC) & 1u;
          // the scale warps waited for the load of stage s before scaling into b
          if (!mbar_wait(BAR(SCALED + b), bph2, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + s * C::STAGE;
          const uint32_t sc = sbase + C::OFF_SC + b * C::SCBUF;
#pragma unroll
          for (int ks = 0; ks < C::UT / 16; ++ks) {
            const uint32_t ko = (uint32_t)ks * 2048u;
            mma_bf16_ss(d, desc_sw128(sc + ko, C::BLK, 1024),
                        desc_sw128(st + ko, C::BLK, 1024), kIdN256, (tile | ks) != 0);
            mma_bf16_ss(d, desc_sw128(sc + C::OFF_L + ko, C::BLK, 1024),
                        desc_sw128(st + ko, C::BLK, 1024), kIdN256, 1u);
          }
          mma_commit(BAR(EMPTY + s));
          mma_commit(BAR(SEMPTY + b));
        }
        if (!ok) break;
        mma_commit(BAR(TFULL + buf));
      }
      // every issued MMA must finish before TMEM is released
      mma_commit(BAR(DRAIN));
      mbar_wait_drain(BAR(DRAIN), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- beta * K, split into bf16 hi + lo (same swizzled position):
    // thread = (row r, quarter qt) of the 64 x 128 tile; 4 chunks of 8 channels
    const int st_id = tid - 128;
    const int r = st_id & 63, qt = st_id >> 6, hb = qt >> 1;
    auto beta_at = [&](int f, int tl) -> float {
      const int u = tl * C::UT + r;
      return (f < FH && u < U) ? __ldg(beta + (size_t)f * U + u) : 0.f;
    };
    uint32_t it = 0;
    int fh = blockIdx.x, tile = 0;
    float b_next = beta_at(fh, 0);
    while (fh < FH) {
      const float b = b_next;
      int nfh = fh, ntile = tile + 1;
      if (ntile == nt) { ntile = 0; nfh += gridDim.x; }
      b_next = beta_at(nfh, ntile);
      const uint32_t s = it % C::NST, ph = (it / C::NST) & 1u;
      const uint32_t sb = it % C::NSC, sph = (it / C::NSC) & 1u;
      if (!mbar_wait(BAR(FULL + s), ph, abort_flag)) break;
      if (!mbar_wait(BAR(SEMPTY + sb), sph ^ 1u, abort_flag)) break;
      const uint32_t ksrc = sbase + s * C::STAGE + hb * C::BLK + (uint32_t)r * 128u;
      const uint32_t hdst = sbase + C::OFF_SC + sb * C::SCBUF + hb * C::BLK + (uint32_t)r * 128u;
      const uint32_t ldst = hdst + C::OFF_L;
      // the loads first: the shared-memory accesses are ordered asm statements,
      // so this order is what lets the arithmetic overlap them
      uint32_t pos[4];
      uint4 kvs[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        pos[c] = (uint32_t)((4 * (qt & 1) + c + r) & 7) * 16u;   // rotated across rows: conflict-free
        kvs[c] = ld_shared_v4(ksrc + pos[c]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t w[4] = {kvs[c].x, kvs[c].y, kvs[c].z, kvs[c].w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x0 = __uint_as_float(w[q] << 16) * b;
          const float x1 = __uint_as_float(w[q] & 0xFFFF0000u) * b;
          hw[q] = pack_bf16(x0, x1);   // hi = rn(x)
          const float h0 = __uint_as_float(hw[q] << 16), h1 = __uint_as_float(hw[q] & 0xFFFF0000u);
          lw[q] = pack_bf16(x0 - h0, x1 - h1);   // lo = rn(x - hi)
        }
        st_shared_v4(hdst + pos[c], make_uint4(hw[0], hw[1], hw[2], hw[3]));
        st_shared_v4(ldst + pos[c], make_uint4(lw[0], lw[1], lw[2], lw[3]));
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(SCALED + sb));
      ++it;
      fh = nfh;
      tile = ntile;
    }
  } else {
    // ---------------- epilogue: TMEM lane i = row i of D; column c of D goes to
    // element (i, c) of A's block (i / 16, c / 16) when that block is in the
    // upper triangle (16 lanes store 64 contiguous bytes), or B[c - 128][i]
    // (32 lanes store 128 contiguous bytes)
    const int i = warp * 32 + lane;
    const int br = i >> 4;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    uint32_t lf = 0;
    for (int fh = blockIdx.x; fh < FH; fh += gridDim.x, ++lf) {
      const uint32_t buf = lf & 1u, bph = (lf >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(TFULL + buf), bph, abort_flag))) break;
      tc_fence_after();
      const uint32_t tA = tmem + buf * 256u;
      float* At = A_out + (size_t)fh * kATri + (i & 15);
      float* Bf = B_out + (size_t)fh * kDD;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) {
        uint32_t v0[32];
        tmem_ld32(lb + tA + 32u * q, v0);
        tmem_wait_ld();
        if (q == 7) {
          tc_fence_before();
          mbar_arrive(BAR(TEMPTY + buf));
        }
        if (q < 4) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int bc = 2 * q + hb;
            if (bc >= br) {
              float* dst = At + atri_block(br, bc);
#pragma unroll
              for (int c = 0; c < 16; ++c) dst[16 * c] = __uint_as_float(v0[16 * hb + c]);
            }
          }
          if (A_full) {   // debug output: the full matrix
            float* dst = A_full + (size_t)fh * kDD + (size_t)(32 * q) * kD + i;
#pragma unroll
            for (int c = 0; c < 32; ++c) dst[(size_t)c * kD] = __uint_as_float(v0[c]);
          }
        } else {
          float* dst = Bf + (size_t)(32 * (q - 4)) * kD + i;
#pragma unroll
          for (int c = 0; c < 32; ++c) dst[(size_t)c * kD] = __uint_as_float(v0[c]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (warp == C::WARP_PROD && lane == 0 && *abort_flag) {  // let issued copies land before the CTA exits
    for (int s = 0; s < C::NST; ++s)
      if (last_it[s] >= 0) mbar_wait_drain(BAR(FULL + s), ((uint32_t)last_it[s] / C::NST) & 1u);
  }
}

// ===========================================================================
// k_stats64_tc: the Gram kernel for d = 64.  With 64 channels the roles of
// the operands swap so that the MMA keeps M = 128: tokens on the K dimension,
//   D[128 x 64] = [K | V]^T (beta K)_hi + [K | V]^T (beta K)_lo
// so D[0:64, :] = A and D[64:128, :] = B (rows n of B, columns j).  Both
// operands are MN-major 64-channel TMA boxes (64 tokens x 128 B, 128-B
// swizzle); [K | V] is two boxes 8 KB apart (the M dimension's two 64-blocks).
// Warps: 0-3 epilogue (TMEM lane i < 64: A row i; lane 64 + n: B row n),
// 4-7 scale (beta K -> bf16 hi + lo), 8 TMA producer, 9 MMA issuer.  Four
// load stages (K, V: 16 KB), two scaled buffers (hi, lo: 16 KB), two
// 64-column TMEM accumulators.  Out: A [64][64] (symmetric, stored by
// columns), B^T [64][64] (B^T[j][n] = B[n][j], the layout the d = 64 scan
// reads), optionally B [n][j] for the debug output.
// ===========================================================================
struct Stats64Cfg {
  static constexpr int UT = 64;
  static constexpr int NST = 4;                      // load stages
  static constexpr int NSC = 2;                      // scaled buffers
  static constexpr uint32_t BLK = UT * 128;          // 8192: 64 tokens x 64 channels
  static constexpr uint32_t STAGE = 2 * BLK;         // K, V
  static constexpr uint32_t SCBUF = 2 * BLK;         // hi, lo
  static constexpr uint32_t OFF_SC = NST * STAGE;
  static constexpr int NSCALE = 128;                 // 64 rows x 2 halves of the 128-B row
  static constexpr int WARP_PROD = 4 + NSCALE / 32;
  static constexpr int WARP_MMA = WARP_PROD + 1;
  static constexpr int THREADS = 32 * (WARP_MMA + 1);
  static constexpr uint32_t BAR_OFF = OFF_SC + NSC * SCBUF;
  static constexpr int NBAR = 2 * NST + 2 * NSC + 5;
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};

__global__ void __launch_bounds__(Stats64Cfg::THREADS, 1)
k_stats64_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
             const float* __restrict__ beta, int U, int FH, float* __restrict__ A_out, float* __restrict__ Bt_out,
             float* __restrict__ B_full) {
  using C = Stats64Cfg;
  constexpr int D = 64;
  constexpr size_t DD = 64 * 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
  const int FULL = 0, EMPTY = C::NST, SCALED = 2 * C::NST, SEMPTY = 2 * C::NST + C::NSC,
            TFULL = 2 * C::NST + 2 * C::NSC, TEMPTY = TFULL + 2, DRAIN = TFULL + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(BAR(FULL + s), 1);
      mbar_init(BAR(EMPTY + s), 1);
    }
    for (int b = 0; b < C::NSC; ++b) {
      mbar_init(BAR(SCALED + b), C::NSCALE);
      mbar_init(BAR(SEMPTY + b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(TFULL + b), 1);
      mbar_init(BAR(TEMPTY + b), 128);
    }
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_wait_prerequisites();   // (see k_stats_tc)
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const int nt = (U + C::UT - 1) / C::UT;
  int last_it[C::NST];
  for (int s = 0; s < C::NST; ++s) last_it[s] = -1;

  if (warp == C::WARP_PROD) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int fh = blockIdx.x; ok && fh < FH; fh += gridDim.x) {
        for (int tile = 0; tile < nt; ++tile, ++it) {
          const uint32_t s = it % C::NST, ph = (it / C::NST) & 1u;
          if (!mbar_wait(BAR(EMPTY + s), ph ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(BAR(FULL + s), 2 * C::BLK);
          const uint32_t st = sbase + s * C::STAGE;
          tma_load_3d(st, &tmK, 0, tile * C::UT, fh, BAR(FULL + s));
          tma_load_3d(st + C::BLK, &tmV, 0, tile * C::UT, fh, BAR(FULL + s));
          last_it[s] = (int)it;
        }
      }
    }
  } else if (warp == C::WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, 64, 1, 1);   // A = [K | V], B = beta K, both MN-major
      uint32_t it = 0, lf = 0;
      bool ok = true;
      for (int fh = blockIdx.x; ok && fh < FH; fh += gridDim.x, ++lf) {
        const uint32_t buf = lf & 1u, bph = (lf >> 1) & 1u;
        if (!mbar_wait(BAR(TEMPTY + buf), bph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * 64u;
        for (int tile = 0; tile < nt; ++tile, ++it) {
          const uint32_t s = it % C::NST;
          const uint32_t b = it % C::NSC, bph2 = (it / C::NSC) & 1u;
          if (!mbar_wait(BAR(SCALED + b), bph2, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + s * C::STAGE;
          const uint32_t sc = sbase + C::OFF_SC + b * C::SCBUF;
#pragma unroll
          for (int ks = 0; ks < C::UT / 16; ++ks) {
            const uint32_t ko = (uint32_t)ks * 2048u;
            const uint64_t a = desc_sw128(st + ko, C::BLK, 1024);
            mma_bf16_ss(d, a, desc_sw128(sc + ko, C::BLK, 1024), kId, (tile | ks) != 0);
            mma_bf16_ss(d, a, desc_sw128(sc + C::BLK + ko, C::BLK, 1024), kId, 1u);
          }
          mma_commit(BAR(EMPTY + s));
          mma_commit(BAR(SEMPTY + b));
        }
        if (!ok) break;
        mma_commit(BAR(TFULL + buf));
      }
      mma_commit(BAR(DRAIN));
      mbar_wait_drain(BAR(DRAIN), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- beta * K -> bf16 hi + lo in the same swizzled position:
    // thread = (token row r, half qt of the row's eight 16-B chunks)
    const int st_id = tid - 128;
    const int r = st_id & 63, qt = st_id >> 6;
    auto beta_at = [&](int f, int tl) -> float {
      const int u = tl * C::UT + r;
      return (f < FH && u < U) ? __ldg(beta + (size_t)f * U + u) : 0.f;
    };
    uint32_t it = 0;
    int fh = blockIdx.x, tile = 0;
    float b_next = beta_at(fh, 0);
    while (fh < FH) {
      const float b = b_next;
      int nfh = fh, ntile = tile + 1;
      if (ntile == nt) { ntile = 0; nfh += gridDim.x; }
      b_next = beta_at(nfh, ntile);
      const uint32_t s = it % C::NST, ph = (it / C::NST) & 1u;
      const uint32_t sb = it % C::NSC, sph = (it / C::NSC) & 1u;
      if (!mbar_wait(BAR(FULL + s), ph, abort_flag)) break;
      if (!mbar_wait(BAR(SEMPTY + sb), sph ^ 1u, abort_flag)) break;
      const uint32_t ksrc = sbase + s * C::STAGE + (uint32_t)r * 128u;
      const uint32_t hdst = sbase + C::OFF_SC + sb * C::SCBUF + (uint32_t)r * 128u;
      const uint32_t ldst = hdst + C::BLK;
      uint32_t pos[4];
      uint4 kvs[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        pos[c] = (uint32_t)((4 * qt + c + r) & 7) * 16u;   // rotated across rows: conflict-free
        kvs[c] = ld_shared_v4(ksrc + pos[c]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t w[4] = {kvs[c].x, kvs[c].y, kvs[c].z, kvs[c].w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x0 = __uint_as_float(w[q] << 16) * b;
          const float x1 = __uint_as_float(w[q] & 0xFFFF0000u) * b;
          hw[q] = pack_bf16(x0, x1);
          const float h0 = __uint_as_float(hw[q] << 16), h1 = __uint_as_float(hw[q] & 0xFFFF0000u);
          lw[q] = pack_bf16(x0 - h0, x1 - h1);
        }
        st_shared_v4(hdst + pos[c], make_uint4(hw[0], hw[1], hw[2], hw[3]));
        st_shared_v4(ldst + pos[c], make_uint4(lw[0], lw[1], lw[2], lw[3]));
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(SCALED + sb));
      ++it;
      fh = nfh;
      tile = ntile;
    }
  } else {
    // ---------------- epilogue: TMEM lane i; i < 64: A row i, stored as A[c][i]
    // (A is symmetric; 32 lanes store 128 contiguous bytes); i = 64 + n: B row
    // n, stored as B^T[j][n]
    const int i = warp * 32 + lane;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    uint32_t lf = 0;
    for (int fh = blockIdx.x; fh < FH; fh += gridDim.x, ++lf) {
      const uint32_t buf = lf & 1u, bph = (lf >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(TFULL + buf), bph, abort_flag))) break;
      tc_fence_after();
      const uint32_t tA = tmem + buf * 64u;
      uint32_t v0[32], v1[32];
      tmem_ld32(lb + tA, v0);
      tmem_ld32(lb + tA + 32u, v1);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(TEMPTY + buf));
      float* dst = (i < D ? A_out : Bt_out) + (size_t)fh * DD + (i & 63);
#pragma unroll
      for (int c = 0; c < 32; ++c) dst[(size_t)c * D] = __uint_as_float(v0[c]);
#pragma unroll
      for (int c = 0; c < 32; ++c) dst[(size_t)(32 + c) * D] = __uint_as_float(v1[c]);
      if (B_full && i >= D) {   // debug output: B[n][j]
        float* bf = B_full + (size_t)fh * DD + (size_t)(i - D) * D;
#pragma unroll
        for (int c = 0; c < 32; ++c) bf[c] = __uint_as_float(v0[c]);
#pragma unroll
        for (int c = 0; c < 32; ++c) bf[32 + c] = __uint_as_float(v1[c]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (warp == C::WARP_PROD && lane == 0 && *abort_flag) {
    for (int s = 0; s < C::NST; ++s)
      if (last_it[s] >= 0) mbar_wait_drain(BAR(FULL + s), ((uint32_t)last_it[s] / C::NST) & 1u);
  }
}

// ===========================================================================
// k_inverse_tc: M = (I + A)^{-1} for every frame-head, by a block sweep of the
// symmetric positive definite I + A held in TMEM, with every product on the
// tensor cores.  Sweeping every index of a symmetric matrix ends at its
// negative inverse.  Sweeping a pivot block P of 16 indices, with
// C = (I + A)[:, P] and G = -P^{-1}, maps
//   A_ij -> A_ij + (C G)_i C_j^T   (i, j outside P; the Schur complement)
//   A_iP -> -(C G)_i,   A_PP -> G,   A_Pj -> -(C G)_j^T.
// TMEM holds T = the current matrix minus the identity on the indices not
// swept yet.  One block step:
//   1. Y = the panel T[:, P] with its P rows replaced by -e_i (then C G = Y G
//      outside P, and -G on P);  X = Y G by MMA into T's P columns.
//   2. T's P rows and P columns are cleared (TMEM stores), then by MMA
//      T += X Y^T  (Schur complement outside P; -X in the P columns;
//                   -G C_j^T in the P rows; G in the P block).
// No term cancels in floating point: every entry is a sum of products of the
// size of the result.  Operands go to the tensor cores as bf16 splits in three
// parts (h, m, l; bf16 x 3 holds an fp32 value exactly): X = Y G and the
// update X Y^T each take the six products down to 2^-24 (hh, hm, mh, hl, lh,
// mm).  This keeps the swept matrix symmetric to ~1e-5; with fewer products
// the asymmetry between the P rows and the P columns compounds through the
// scan.  Every pivot block of an SPD matrix's Schur complement is SPD, so no
// pivoting is needed.
// The 16 x 16 sweep that gives G is the sequential part, so it runs one block
// ahead: once X is known, the warp owning the next block Q brings A_QQ up to
// date in fp32 (A_QQ + X_Q C_Q^T) and sweeps it while the tensor cores apply
// the update.  Four warpgroups per CTA work on four matrices at once (own
// TMEM columns, shared-memory workspace, named barriers, completion barriers).
// In: A (fp32, upper block triangle, from k_stats_tc).  Out: the scan's M operand image
// (element (j, k) = M[k][j], MN-major, 128-B swizzle, bf16 hi / lo halves)
// and optionally M in fp32.
// ===========================================================================
struct InvCfg {
  static constexpr int GROUPS = 4;
  static constexpr int THREADS = 128 * GROUPS;
  static constexpr uint32_t TCOLS = 128;      // TMEM columns per group: the matrix
  static constexpr uint32_t SW_BYTES = 30720;  // per-group workspace (see SW_* below)
  static constexpr uint32_t BAR_OFF = GROUPS * SW_BYTES;
  static constexpr int NBAR = 2 * GROUPS;      // per group: update done, X done
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};
// per-group workspace: K-major no-swizzle operand images (rows of 16 bf16,
// 4 KB for 128 rows, 512 B for 16) and the fp32 exchange buffer
constexpr uint32_t SW_YH = 0, SW_YM = 4096, SW_YL = 8192;         // Y in three parts (P rows: -e, 0, 0)
constexpr uint32_t SW_XH = 12288, SW_XM = 16384, SW_XL = 20480;   // X in three parts
constexpr uint32_t SW_GI = 24576;                                 // G in three parts, 3 x 512 B
constexpr uint32_t SW_CQ = 26624;   // next block's rows of C, transposed, [2 steps][2 segments][16][16]

// Pivot block swept at step s: the order 0,2,4,6,1,3,5,7 rotated by rot.  The
// sweep's result does not depend on the order up to rounding; this one puts
// consecutive blocks in different warps (a block's TMEM lanes belong to warp
// block / 2, i.e. to a fixed sub-partition), and rotating it by the matrix
// index spreads the pivot warps of the groups over the sub-partitions while
// keeping each matrix's arithmetic independent of which group sweeps it.
__device__ __forceinline__ int inv_block(int s, int rot) {
  const int j = (s + rot) & 7;
  return j < 4 ? 2 * j : 2 * j - 7;
}

// In-place sweep of a symmetric 16 x 16 block by one warp.  On entry the
// block's rows are in the 16-lane segment `sel` (row r = lane & 15, all 16
// columns in x); on exit every lane holds row r, columns [8h, 8h + 8) of
// -P^{-1} in g (h = lane >> 4), so both segments share the arithmetic.  The
// pivot row and the pivot column element come from the owning lanes by
// shuffles.
__device__ __forceinline__ void sweep16(const float (&x)[16], int sel, int lane, float (&g)[8]) {
  const int r = lane & 15, h = lane >> 4;
  const int src = r + 16 * sel;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float a = __shfl_sync(0xffffffffu, x[t], src);
    const float b = __shfl_sync(0xffffffffu, x[8 + t], src);
    g[t] = h ? b : a;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int kh = k >> 3, kk = k & 7;
    float col[8];   // row k at this lane's columns
#pragma unroll
    for (int t = 0; t < 8; ++t) col[t] = __shfl_sync(0xffffffffu, g[t], k + 16 * h);
    const float akk = __shfl_sync(0xffffffffu, g[kk], k + 16 * kh);   // pivot
    const float ark = __shfl_sync(0xffffffffu, g[kk], r + 16 * kh);   // this row's column k
    const float pinv = rcp_approx(akk);
    const bool me = r == k;
    const float f = ark * pinv;
#pragma unroll
    for (int t = 0; t < 8; ++t) g[t] = me ? col[t] * pinv : fmaf(-f, col[t], g[t]);
    if (h == kh) g[kk] = me ? -pinv : f;
  }
}

// x = h + m + l exactly with bf16 h = rn(x), m = rn(x - h), l = x - h - m
// (24 significant bits in three 8-bit parts; exact for normal values).
__device__ __forceinline__ void split3_bf16(float x, float& h, float& m, float& l) {
  h = __bfloat162float(__float2bfloat16_rn(x));
  const float r = x - h;
  m = __bfloat162float(__float2bfloat16_rn(r));
  l = r - m;
}

// 16 fp32 values -> rows r of three no-swizzle K-major images (parts h, m, l)
__device__ __forceinline__ void store_row16_split3(uint32_t ih, uint32_t im, uint32_t il, uint32_t r,
                                                   const float (&x)[16]) {
#pragma unroll
  for (int kc = 0; kc < 2; ++kc) {
    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float h0, m0, l0, h1, m1, l1;
      split3_bf16(x[8 * kc + 2 * q], h0, m0, l0);
      split3_bf16(x[8 * kc + 2 * q + 1], h1, m1, l1);
      hw[q] = pack_bf16(h0, h1);
      mw[q] = pack_bf16(m0, m1);
      lw[q] = pack_bf16(l0, l1);
    }
    const uint32_t off = kimg16(r, 8u * kc);
    st_shared_v4(ih + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
    st_shared_v4(im + off, make_uint4(mw[0], mw[1], mw[2], mw[3]));
    st_shared_v4(il + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
  }
}

// G image (the X product's B operand): lane (r, h) of the sweeping warp holds
// row r, columns [8h, 8h + 8) of G; three K-major no-swizzle parts h, m, l
__device__ __forceinline__ void store_g_image(uint32_t swb, int r, int h, const float (&gq)[8]) {
  uint32_t hw[4], mw[4], lw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float h0, m0, l0, h1, m1, l1;
    split3_bf16(gq[2 * q], h0, m0, l0);
    split3_bf16(gq[2 * q + 1], h1, m1, l1);
    hw[q] = pack_bf16(h0, h1);
    mw[q] = pack_bf16(m0, m1);
    lw[q] = pack_bf16(l0, l1);
  }
  const uint32_t off = kimg16((uint32_t)r, 8u * (uint32_t)h);
  st_shared_v4(swb + SW_GI + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
  st_shared_v4(swb + SW_GI + 512u + off, make_uint4(mw[0], mw[1], mw[2], mw[3]));
  st_shared_v4(swb + SW_GI + 1024u + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
}

// Barriers of one group (ids distinct per group): `bY` closes the Y images and
// the G images of a step, `bX` the X images and the cleared rows and columns
// of P.  The group's MMAs are issued by lane 0 of its warp grp, so the four
// groups' issuers sit on different SM sub-partitions; that warp waits at the
// barriers, the other warps only arrive, and each of their next arrivals
// follows a wait on the MMA that the barrier released.
struct InvBars {
  uint32_t bY, bX, sbar, xbar;
};

// One warpgroup sweeps the matrix in TMEM columns [tA, tA + 128); thread i =
// TMEM lane i; gw = warp index within the group, grp = group index, rot = the
// rotation of the pivot order.  Returns false if a wait gave up (the matrix is
// then garbage; the barrier sequence is still kept, so the group stays in
// step).
__device__ __forceinline__ bool sweep_inverse_tmem(uint32_t tA, uint32_t lb, uint32_t swb, const InvBars& bar,
                                                   uint32_t& sphase, uint32_t& xphase, volatile int* abort_flag,
                                                   int i, int gw, int lane, int grp, int rot) {
  constexpr uint32_t kId128 = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kId16 = idesc_bf16(128, 16, 0, 0);
  const int r = lane & 15, h = lane >> 4;
  const bool issuer_warp = gw == grp;
  const bool issuer = issuer_warp && lane == 0;
  bool ok = true;
  // G of the first pivot block (the matrix is untouched: P = its own block)
  {
    const int K0 = inv_block(0, rot);
    if (gw == (K0 >> 1)) {
      uint32_t v[16];
      tmem_ld16(lb + tA + 16u * (uint32_t)K0, v);
      tmem_wait_ld();
      const bool in0 = (i >> 4) == K0;
      float x0[16], g0[8];
#pragma unroll
      for (int t = 0; t < 16; ++t) x0[t] = __uint_as_float(v[t]) + ((in0 && r == t) ? 1.f : 0.f);
      sweep16(x0, K0 & 1, lane, g0);
      store_g_image(swb, r, h, g0);
    }
  }
#pragma unroll 1
  for (int s = 0; s < 8; ++s) {
    const int K = inv_block(s, rot);
    const uint32_t p0 = 16u * (uint32_t)K;
    const bool inP = (i >> 4) == K;
    const bool pwarp = gw == (K >> 1);
    const int Kn = inv_block(s + 1, rot);
    const bool qwarp = s < 7 && gw == (Kn >> 1);     // sweeps the next block ahead
    const bool inQ = qwarp && (i >> 4) == Kn;
    // by step parity: the sweeping warp of step s + 2 writes it only after
    // passing the X barrier of step s + 1, i.e. after this step's lookahead
    const uint32_t cqb = swb + SW_CQ + 2048u * (uint32_t)(s & 1) + 1024u * (uint32_t)h;
    if (s > 0) {   // the previous step's update is in TMEM, its operand images are free
      ok = mbar_wait(bar.sbar, sphase, abort_flag) && ok;
      sphase ^= 1u;
      tc_fence_after();
    }
    // raw panel T[:, P]; the next block's columns for its warp
    float yr[16], aq[16];
    {
      uint32_t v[16];
      tmem_ld16(lb + tA + p0, v);
      if (qwarp) {
        uint32_t w2[16];
        tmem_ld16(lb + tA + 16u * (uint32_t)Kn, w2);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 16; ++t) aq[t] = __uint_as_float(w2[t]) + ((inQ && r == t) ? 1.f : 0.f);
      } else {
        tmem_wait_ld();
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) yr[t] = __uint_as_float(v[t]);
    }
    {   // Y (P rows -e) in three parts
      float ye[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) ye[t] = inP ? (r == t ? -1.f : 0.f) : yr[t];
      store_row16_split3(swb + SW_YH, swb + SW_YM, swb + SW_YL, (uint32_t)i, ye);
    }
    if (qwarp) {   // C's rows of the next block, transposed: cq[k][r] = C[Q_r][k] (Q is outside P)
#pragma unroll
      for (int k = 0; k < 16; ++k) st_shared_f1(cqb + 64u * (uint32_t)k + 4u * (uint32_t)r, yr[k]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (issuer_warp) named_bar_sync(bar.bY, 128);
    else named_bar_arrive(bar.bY, 128);
    if (issuer) {   // X = Y G into T[:, P] (overwritten)
      tc_fence_after();
      const uint64_t a0 = desc_noswz(swb + SW_YH, 128, 256), a1 = desc_noswz(swb + SW_YM, 128, 256),
                     a2 = desc_noswz(swb + SW_YL, 128, 256);
      const uint64_t b0 = desc_noswz(swb + SW_GI, 128, 256), b1 = desc_noswz(swb + SW_GI + 512u, 128, 256),
                     b2 = desc_noswz(swb + SW_GI + 1024u, 128, 256);
      const uint32_t d = tA + p0;
      mma_bf16_ss(d, a0, b0, kId16, 0u);
      mma_bf16_ss(d, a0, b1, kId16, 1u);
      mma_bf16_ss(d, a1, b0, kId16, 1u);
      mma_bf16_ss(d, a0, b2, kId16, 1u);
      mma_bf16_ss(d, a2, b0, kId16, 1u);
      mma_bf16_ss(d, a1, b1, kId16, 1u);
      mma_commit(bar.xbar);
    }
    if (pwarp) {   // clear the P rows outside the P columns (those the X product writes)
      const uint32_t sib = 16u * (uint32_t)(K ^ 1);   // P's sibling block in this warp's chunk of 32 columns
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        if (q == (K >> 1)) {
          uint32_t v[16];
          tmem_ld16(lb + tA + sib, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) v[t] = inP ? 0u : v[t];
          tmem_st16(lb + tA + sib, v);
        } else {
          uint32_t v[32];
          tmem_ld32(lb + tA + 32u * (uint32_t)q, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = inP ? 0u : v[t];
          tmem_st32(lb + tA + 32u * (uint32_t)q, v);
        }
      }
    }
    ok = mbar_wait(bar.xbar, xphase, abort_flag) && ok;
    xphase ^= 1u;
    tc_fence_after();
    float x[16];
    {
      uint32_t v[16];
      tmem_ld16(lb + tA + p0, v);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 16; ++t) x[t] = __uint_as_float(v[t]);
      uint32_t z[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) z[t] = 0u;
      tmem_st16(lb + tA + p0, z);   // T[:, P] = 0 before the update
    }
    store_row16_split3(swb + SW_XH, swb + SW_XM, swb + SW_XL, (uint32_t)i, x);
    fence_proxy_async_smem();
    tmem_wait_st();
    tc_fence_before();
    if (issuer_warp) named_bar_sync(bar.bX, 128);
    else named_bar_arrive(bar.bX, 128);
    if (issuer) {   // T += X Y^T, six products
      tc_fence_after();
      const uint64_t yh = desc_noswz(swb + SW_YH, 128, 256), ym = desc_noswz(swb + SW_YM, 128, 256),
                     yl = desc_noswz(swb + SW_YL, 128, 256);
      const uint64_t xh = desc_noswz(swb + SW_XH, 128, 256), xm = desc_noswz(swb + SW_XM, 128, 256),
                     xl = desc_noswz(swb + SW_XL, 128, 256);
      mma_bf16_ss(tA, xh, yh, kId128, 1u);
      mma_bf16_ss(tA, xh, ym, kId128, 1u);
      mma_bf16_ss(tA, xm, yh, kId128, 1u);
      mma_bf16_ss(tA, xh, yl, kId128, 1u);
      mma_bf16_ss(tA, xl, yh, kId128, 1u);
      mma_bf16_ss(tA, xm, ym, kId128, 1u);
      mma_commit(bar.sbar);
    }
    if (qwarp) {   // next block after this step, A_QQ + X_Q C_Q^T in fp32, and its sweep
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          const float4 cv = ld_shared_f4(cqb + 64u * (uint32_t)k + 4u * t);
          aq[t] = fmaf(x[k], cv.x, aq[t]); aq[t + 1] = fmaf(x[k], cv.y, aq[t + 1]);
          aq[t + 2] = fmaf(x[k], cv.z, aq[t + 2]); aq[t + 3] = fmaf(x[k], cv.w, aq[t + 3]);
        }
      }
      float gq[8];
      sweep16(aq, Kn & 1, lane, gq);
      store_g_image(swb, r, h, gq);   // this step's X product has read the previous G
    }
  }
  ok = mbar_wait(bar.sbar, sphase, abort_flag) && ok;   // the last step's update
  sphase ^= 1u;
  tc_fence_after();
  return ok;
}

// Row i, columns [64 hh, 64 hh + 64) of a symmetric A stored as its upper
// block triangle (kATri layout): blocks at or right of the diagonal give the
// row directly (16 lanes of a row block read 64 contiguous bytes per column),
// blocks left of it give the transposed block's column, contiguous per thread.
__device__ __forceinline__ void load_a_row_half(const float* __restrict__ At, int i, int hh, float (&a)[64]) {
  const int br = i >> 4, r = i & 15;
#pragma unroll
  for (int b4 = 0; b4 < 4; ++b4) {
    const int bc = 4 * hh + b4;
    if (bc >= br) {
      const float* blk = At + atri_block(br, bc) + r;
#pragma unroll
      for (int c = 0; c < 16; ++c) a[16 * b4 + c] = __ldg(blk + 16 * c);
    } else {
      const float4* blk = reinterpret_cast<const float4*>(At + atri_block(bc, br) + 16 * r);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 x = __ldg(blk + c);
        a[16 * b4 + 4 * c] = x.x; a[16 * b4 + 4 * c + 1] = x.y;
        a[16 * b4 + 4 * c + 2] = x.z; a[16 * b4 + 4 * c + 3] = x.w;
      }
    }
  }
}

// 64 fp32 values -> TMEM lane columns [col, col + 64)
__device__ __forceinline__ void tmem_st64f(uint32_t taddr, const float (&a)[64]) {
  uint32_t w[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(a[c]);
  tmem_st32(taddr, w);
#pragma unroll
  for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(a[32 + c]);
  tmem_st32(taddr + 32u, w);
}

__global__ void __launch_bounds__(InvCfg::THREADS, 1)
k_inverse_tc(const float* __restrict__ A, int FH, uint8_t* __restrict__ Mimg, float* __restrict__ M_dbg) {
  using C = InvCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = warp >> 2, gw = warp & 3;
  const int i = gw * 32 + lane;
  if (tid == 0) {
    for (int q = 0; q < C::NBAR; ++q) mbar_init(sbase + C::BAR_OFF + 8u * q, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_wait_prerequisites();   // the Gram kernel's A is complete (see k_stats_tc)
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tA = tmem + C::TCOLS * (uint32_t)g;
  const uint32_t lb = (uint32_t)(gw * 32) << 16;
  const uint32_t swb = sbase + C::SW_BYTES * (uint32_t)g;
  const uint32_t bid = 1u + (uint32_t)g;
  const InvBars bars{bid, 5u + (uint32_t)g, sbase + C::BAR_OFF + 8u * (uint32_t)g,
                     sbase + C::BAR_OFF + 8u * (uint32_t)(C::GROUPS + g)};
  uint32_t sphase = 0, xphase = 0;

  const int mstride = gridDim.x * C::GROUPS;
  int m = blockIdx.x * C::GROUPS + g;
  if (m < FH) {   // row i of the group's first matrix -> TMEM lane i
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      float a[64];
      load_a_row_half(A + (size_t)m * kATri, i, hh, a);
      tmem_st64f(lb + tA + 64u * hh, a);
    }
  }
  for (; m < FH; m += mstride) {
    const int mnext = m + mstride;
    const bool has_next = mnext < FH;
    if (i == 0 && has_next)   // the group's next matrix: into L2 while this one is swept
      bulk_prefetch_l2(A + (size_t)mnext * kATri, (uint32_t)(kATri * sizeof(float)));
    tmem_wait_st();
    tc_fence_before();
    named_bar_sync(bid, 128);
    tc_fence_after();
    const bool ok = sweep_inverse_tmem(tA, lb, swb, bars, sphase, xphase, abort_flag, i, gw, lane, g, m & 3);
    // M = -(swept matrix): row i -> operand image row i (k index), debug copy.
    // The next matrix's row i replaces each 64-column half once it has been
    // read (this thread's own TMEM lane), so its loads overlap these stores.
    uint8_t* img = Mimg + (size_t)m * kImgBytes;
    const float* An = A + (size_t)(has_next ? mnext : m) * kATri;
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      float an[64];
      if (has_next) load_a_row_half(An, i, hh, an);
#pragma unroll 1
      for (int q = 4 * hh; q < 4 * hh + 4; ++q) {   // 16-column slices
        uint32_t v[16];
        tmem_ld16(lb + tA + 16u * q, v);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = -__uint_as_float(v[8 * cc + e]);
          store_img_chunk(img, mimg_offset(16 * q + 8 * cc, i), x);
        }
        if (M_dbg) {
          float* md = M_dbg + (size_t)m * kDD + (size_t)i * kD + 16 * q;
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) md[c2] = -__uint_as_float(v[c2]);
        }
      }
      if (has_next) tmem_st64f(lb + tA + 64u * hh, an);
    }
    tc_fence_before();
    const bool all_ok = named_bar_and(bid, 128, ok);
    tc_fence_after();
    if (!all_ok) break;
  }
  if (gw == g && lane == 0) {   // the group's own tensor-core work completes before TMEM is released
    mma_commit(bars.sbar);
    mbar_wait_drain(bars.sbar, sphase);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// k_scan_tc: one CTA per chain (b, h, direction); S in R^{128 x 128} fp32.
// Step t: X = S Diag(alpha_t) + B_t (fp32; Eq. 2, alpha = 1 without decay),
// then S <- X M_t computed on the tensor cores as
//   D[j][n] = sum_k M[k][j] X[n][k]  with  M = Mh + Ml,  X = Xh + Xl  (bf16)
//   D = Mh Xh + Mh Xl + Ml Xh        (the dropped Ml Xl term is ~2^-16 rel.)
// Right-multiplication acts on each row of S independently, so the 128 rows
// run as two independent 64-row halves that ping-pong: while the tensor pipe
// works on one half, the state warps rebuild the other half's operand, and
// the pipe always has the next half queued.  TMEM: half h in columns
// 64h .. 64h+63; lane j holds column j of S.
// Warps 0-7: state; warps 4h .. 4h+3 own half h (thread j = TMEM lane j of
// its quarter): read S from TMEM, store boundary states, add B_{t+1}
// (prefetched into registers), write the X hi/lo image.  The image is
// MN-major (element (k, n) of the MMA's B operand, n contiguous, 128-B
// swizzle, one 16 KB image per half and per hi/lo): thread j holds k = j for
// all 64 n of its half, so it writes eight 16-B chunks per hi/lo image.  The
// two halves' operand rebuilds run on separate warps.
// Warp 8: bulk-copies the M image of the coming steps (two stages).
// Warp 9: MMA issuer, TMEM owner.
// Boundary states: fwd[j] after frames [0, jC), rev[j] after [jC, T).
//
// The same kernel body runs the chunk-wise form of the scans (Section 5,
// "Chunk-wise scans"; Appendix A.1): frame t acts on a state as the affine map
// S -> S (Diag(alpha_t) M_t) + B_t M_t, so the frames of chunk c compose, in
// the direction's order, into S -> S P_c + J_c.
//   kScanCompose: one CTA per (b, h, chunk, direction, part) runs the chunk's
//     frames from S = 0 with the B_t (part J: gives J_c) or from S = I
//     without them (part P: gives P_c).  The four CTAs of a chunk are
//     neighbours and share its M images and B through L2.  J_c is stored in
//     fp32, P_c as the M operand image (bf16 hi / lo).
//   kScanChunks: one CTA per chain runs the NC chunk maps,
//     S <- S P_c + J_c, and stores every boundary state.
// The sequential chain shrinks from T steps to C + NC steps at about twice
// the tensor-core work (the P_c products), which pays when few chains run.
// ===========================================================================
enum ScanMode { kScanFrames = 0, kScanCompose = 1, kScanChunks = 2 };

struct ScanArgs {
  const uint8_t* Mimg;   // frames, compose: M images [BH][T]; chunks: P_c images [2][BH][NC]
  const float* Bm;       // frames, compose: B_t [BH][T]; chunks: J_c [2][BH][NC] (fp32, [n][j])
  const float* S0f;      // [BH][d][d] or null (frames, chunks)
  const float* S0r;
  const float* alpha;    // [BH][T][d] or null (frames, compose)
  float* states;         // frames, chunks: boundary states [2][BH][NC + 1]
  float* Jout;           // compose: J_c [2][BH][NC]
  uint8_t* Pout;         // compose: P_c images [2][BH][NC]
  int BH, T, chunk, NC;
};

struct ScanCfg {
  static constexpr int THREADS = 320;
  static constexpr int PREFETCH = 1;                       // steps of L2 prefetch lead (1 measured best)
  static constexpr int WARP_PROD = 8;
  static constexpr int WARP_MMA = 9;
  static constexpr uint32_t OFF_M = 0;                    // 2 stages x 64 KB
  static constexpr uint32_t OFF_X = 2 * kImgBytes;        // [half][hi/lo] x 16 KB
  static constexpr uint32_t XIMG = 16384;                 // 128 k-rows x 64 n bf16
  static constexpr uint32_t BAR_OFF = 3 * kImgBytes;
  static constexpr int NBAR = 2 + 2 + 2 + 2 + 1;           // mfull[2], mempty[2], xfull[2], dfull[2], drain
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};

// 8 fp32 values -> one 16-B chunk of the hi image and one of the lo image
__device__ __forceinline__ void st_chunk_hilo(uint32_t hi_addr, uint32_t lo_addr, const float (&x)[8]) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    hw[q] = pack_bf16(x[2 * q], x[2 * q + 1]);   // hi = rn(x)
    const float h0 = __uint_as_float(hw[q] << 16), h1 = __uint_as_float(hw[q] & 0xFFFF0000u);
    lw[q] = pack_bf16(x[2 * q] - h0, x[2 * q + 1] - h1);   // lo = rn(x - hi)
  }
  st_shared_v4(hi_addr, make_uint4(hw[0], hw[1], hw[2], hw[3]));
  st_shared_v4(lo_addr, make_uint4(lw[0], lw[1], lw[2], lw[3]));
}

// element (n, k) of a 128-row K-major operand image: k-block (k / 64) of
// 128 rows x 128 B, 128-B swizzle
__device__ __forceinline__ uint32_t ximg_offset(int n, int k) {
  return (uint32_t)(k >> 6) * 16384u + sw128_offset((uint32_t)n, (uint32_t)(k & 63));
}

template <int MODE>
__global__ void __launch_bounds__(ScanCfg::THREADS, 1) k_scan_tc(const ScanArgs sa) {
  using C = ScanCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
  const int MFULL = 0, MEMPTY = 2, XFULL = 4, DFULL = 6, DRAIN = 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // composing: the four CTAs of a chunk (2 directions x 2 parts) are
  // neighbours and share the chunk's M images and B through L2
  const int dir = MODE == kScanCompose ? (int)((blockIdx.x >> 1) & 1u) : (int)blockIdx.y;
  const int T = sa.T, NC = sa.NC, BH = sa.BH;
  // chain (b, h) and, when composing, the chunk, its first frame, the part
  // (0: J, 1: P) and the step count L
  int bh, cc = 0, c0 = 0, part = 0, L;
  if (MODE == kScanCompose) {
    const int u = blockIdx.x;
    part = u & 1;
    bh = (u >> 2) / NC;
    cc = (u >> 2) % NC;
    c0 = cc * sa.chunk;
    L = min(sa.chunk, T - c0);
  } else {
    bh = blockIdx.x;
    L = MODE == kScanFrames ? T : NC;
  }
  const bool withB = !(MODE == kScanCompose && part == 1);
  // operand index of step i: a frame (frames, compose) or a chunk map (chunks)
  auto src_of = [&](int i) -> size_t {
    if (MODE == kScanFrames) return (size_t)bh * T + (dir == 0 ? i : T - 1 - i);
    if (MODE == kScanCompose) return (size_t)bh * T + c0 + (dir == 0 ? i : L - 1 - i);
    return ((size_t)dir * BH + bh) * NC + (dir == 0 ? i : NC - 1 - i);
  };
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(MFULL + s), 1);
      mbar_init(BAR(MEMPTY + s), 1);
      mbar_init(BAR(XFULL + s), 128);
      mbar_init(BAR(DFULL + s), 1);
    }
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_wait_prerequisites();   // the operand images and B are complete (see k_stats_tc)
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  int last_i[2] = {-1, -1};   // producer: last step issued on each stage

  if (warp == C::WARP_PROD) {
    // ---------------- operand image producer
    if (lane == 0) {
      for (int i = 0; i < L; ++i) {
        const uint32_t s = (uint32_t)i & 1u, ph = ((uint32_t)i >> 1) & 1u;
        if (!mbar_wait(BAR(MEMPTY + s), ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(BAR(MFULL + s), kImgBytes);
        const uint8_t* src = sa.Mimg + src_of(i) * kImgBytes;
        const uint32_t dst = sbase + C::OFF_M + s * kImgBytes;
        if (i + C::PREFETCH < L) {   // warm L2 with the image and B of a later step
          const size_t fa = src_of(i + C::PREFETCH);
          bulk_prefetch_l2(sa.Mimg + fa * kImgBytes, kImgBytes);
          if (withB) bulk_prefetch_l2(sa.Bm + fa * kDD, (uint32_t)(kDD * sizeof(float)));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) bulk_load(dst + q * 16384u, src + q * 16384u, 16384u, BAR(MFULL + s));
        last_i[s] = i;
      }
    }
  } else if (warp == C::WARP_MMA) {
    // ---------------- MMA issuer: step i = half 0, then half 1
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, 64, 1, 1);   // A (M image) and B (X half) MN-major
      bool ok = true;
      for (int i = 0; ok && i < L; ++i) {
        const uint32_t s = (uint32_t)i & 1u, ph = ((uint32_t)i >> 1) & 1u;
        if (!mbar_wait(BAR(MFULL + s), ph, abort_flag)) break;
        const uint32_t mh = sbase + C::OFF_M + s * kImgBytes, ml = mh + kImgHalf;
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(BAR(XFULL + h), (uint32_t)i & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xh = sbase + C::OFF_X + (uint32_t)h * 2u * C::XIMG, xl = xh + C::XIMG;
          const uint32_t d = tmem + 64u * (uint32_t)h;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (uint32_t)ks * 2048u;                                  // 16 k-rows
            const uint64_t a_h = desc_sw128(mh + ko, 16384, 1024), a_l = desc_sw128(ml + ko, 16384, 1024);
            const uint64_t b_h = desc_sw128(xh + ko, 16384, 1024), b_l = desc_sw128(xl + ko, 16384, 1024);
            mma_bf16_ss(d, a_h, b_h, kId, ks != 0);
            mma_bf16_ss(d, a_h, b_l, kId, 1u);
            mma_bf16_ss(d, a_l, b_h, kId, 1u);
          }
          mma_commit(BAR(DFULL + h));
        }
        if (ok) mma_commit(BAR(MEMPTY + s));
      }
      mma_commit(BAR(DRAIN));
      mbar_wait_drain(BAR(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ---------------- state warps: half h = warp / 4, thread j owns column j of S
    const int h = warp >> 2, q = warp & 3;
    const int j = q * 32 + lane;
    const float* S0 = dir == 0 ? sa.S0f : sa.S0r;
    float* st = MODE == kScanCompose ? nullptr
                                     : sa.states + ((size_t)dir * BH + bh) * (size_t)(NC + 1) * kDD;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + 64u * (uint32_t)h;
    // X image: row k = j, 16-B chunk c (n2 = 8c .. 8c+7) at ((c ^ (j & 7)) << 4)
    const uint32_t xbase = sbase + C::OFF_X + (uint32_t)h * 2u * C::XIMG;
    const uint32_t xrow = xbase + (uint32_t)j * 128u;
    const uint32_t jsw = (uint32_t)(j & 7);
    float bnext[64];

    // initial state (stored as the first boundary) and X_0 = S0 Diag(alpha) + B
    {
      const int j0 = dir == 0 ? 0 : NC;
      const float* B0 = sa.Bm + src_of(0) * kDD + (size_t)(64 * h) * kD + j;
      // decay of the first frame on key column j (Eq. 2); 1 without decay
      const float a0 = (MODE != kScanChunks && sa.alpha) ? __ldg(sa.alpha + src_of(0) * kD + j) : 1.f;
#pragma unroll 2
      for (int c = 0; c < 8; ++c) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int n = 64 * h + 8 * c + e;
          float s0;
          if (MODE == kScanCompose) {
            s0 = (part == 1 && n == j) ? 1.f : 0.f;
          } else {
            s0 = S0 ? __ldg(S0 + (size_t)bh * kDD + (size_t)n * kD + j) : 0.f;
            st[(size_t)j0 * kDD + (size_t)n * kD + j] = s0;
          }
          if (MODE == kScanChunks) x[e] = s0;
          else x[e] = fmaf(s0, a0, withB ? __ldg(B0 + (size_t)(8 * c + e) * kD) : 0.f);
        }
        const uint32_t o = xrow + (((uint32_t)c ^ jsw) << 4);
        st_chunk_hilo(o, o + C::XIMG, x);
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(XFULL + h));
    }
    for (int i = 0; i < L; ++i) {
      const bool more = i + 1 < L;
      int jb = -1;   // boundary state reached after this step
      if (MODE == kScanFrames) {
        const int t = dir == 0 ? i : T - 1 - i;
        if (dir == 0) {
          if ((t + 1) % sa.chunk == 0 || t == T - 1) jb = (t + sa.chunk) / sa.chunk;
        } else if (t % sa.chunk == 0) {
          jb = t / sa.chunk;
        }
      } else if (MODE == kScanChunks) {
        const int c = dir == 0 ? i : NC - 1 - i;
        jb = dir == 0 ? c + 1 : c;
      }
      float anext = 1.f;   // decay of the next frame on key column j (Eq. 2)
      // B of the next frame, or this chunk's J: 32 lanes read 128 contiguous bytes per row
      const bool loadB = MODE == kScanChunks || (more && withB);
      if (loadB) {
        const size_t si = MODE == kScanChunks ? src_of(i) : src_of(i + 1);
        const float* Bn = sa.Bm + si * kDD + (size_t)(64 * h) * kD + j;
#pragma unroll
        for (int n2 = 0; n2 < 64; ++n2) bnext[n2] = __ldg(Bn + (size_t)n2 * kD);
      }
      if (MODE != kScanChunks && more && sa.alpha) anext = __ldg(sa.alpha + src_of(i + 1) * kD + j);
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(DFULL + h), (uint32_t)i & 1u, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t v[16];
        tmem_ld16(trow + cb * 16, v);
        tmem_wait_ld();
        float y[16];   // the state after this step
#pragma unroll
        for (int c = 0; c < 16; ++c)
          y[c] = MODE == kScanChunks ? __uint_as_float(v[c]) + bnext[cb * 16 + c] : __uint_as_float(v[c]);
        if (MODE != kScanCompose && jb >= 0) {
#pragma unroll
          for (int c = 0; c < 16; ++c) st[(size_t)jb * kDD + (size_t)(64 * h + cb * 16 + c) * kD + j] = y[c];
        }
        if (MODE == kScanCompose && !more) {
          const size_t co = ((size_t)dir * BH + bh) * NC + cc;
          if (part == 0) {   // J_c, fp32 [n][j]
            float* jo = sa.Jout + co * kDD + (size_t)(64 * h + cb * 16) * kD + j;
#pragma unroll
            for (int c = 0; c < 16; ++c) jo[(size_t)c * kD] = y[c];
          } else {   // P_c as the operand image (element (j, n) = P[n][j]), this half's rows, in its X area
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int nl = cb * 16 + c;   // row within the half
              const float hi = __bfloat162float(__float2bfloat16_rn(y[c]));
              const uint32_t off = (uint32_t)(j >> 6) * 8192u + sw128_offset((uint32_t)nl, (uint32_t)(j & 63));
              st_shared_u16(xbase + off, __bfloat16_as_ushort(__float2bfloat16_rn(y[c])));
              st_shared_u16(xbase + 16384u + off, __bfloat16_as_ushort(__float2bfloat16_rn(y[c] - hi)));
            }
          }
        }
        if (more) {
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = 8 * q2 + e;
              x[e] = MODE == kScanChunks ? y[c]
                                         : fmaf(y[c], anext, withB ? bnext[cb * 16 + c] : 0.f);
            }
            const uint32_t c8 = (uint32_t)(2 * cb + q2);
            const uint32_t o = xrow + ((c8 ^ jsw) << 4);
            st_chunk_hilo(o, o + C::XIMG, x);
          }
        }
      }
      if (more) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(XFULL + h));
      }
    }
    if (MODE == kScanCompose && part == 1) {
      // this half's rows of the P_c image: 4 pieces of 8 KB (hi / lo x two
      // 64-column blocks) -> global, 16 B per thread per copy
      named_bar_sync(1u + (uint32_t)h, 128);
      uint8_t* img = sa.Pout + (((size_t)dir * BH + bh) * NC + cc) * kImgBytes;
      const int t = q * 32 + lane;
#pragma unroll 4
      for (int k2 = 0; k2 < 16; ++k2) {
        const uint32_t o = 16u * (uint32_t)(t + 128 * k2);
        const uint32_t piece = o >> 13, within = o & 8191u;
        const uint4 val = ld_shared_v4(xbase + o);
        *reinterpret_cast<uint4*>(img + (size_t)(piece >> 1) * kImgHalf + (size_t)(piece & 1u) * 16384u +
                                  8192u * (uint32_t)h + within) = val;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (warp == C::WARP_PROD && lane == 0 && *abort_flag) {  // let issued copies land before the CTA exits
    for (int s = 0; s < 2; ++s)
      if (last_i[s] >= 0) mbar_wait_drain(BAR(MFULL + s), ((uint32_t)last_i[s] >> 1) & 1u);
  }
}

// ===========================================================================
// k_scan64_tc: the scans for d = 64.  One CTA runs both chains of a (b, h):
// chain 0 forward, chain 1 reverse, in lockstep.  A 64 x 64 update would
// give the MMA M = 64, so the two chains share one M = 128, N = 128 MMA:
//   D[j'][n'] = sum_k A[j'][k] X[n'][k],   A = [M_fwd^T ; M_rev^T] (j' = 64 c + j),
//                                          X = [X_fwd ; X_rev]     (n' = 64 c + n)
// of which the diagonal blocks D[64c + j][64c + n] = (X_c M_c)[n][j] are the
// two chains' new states (the off-diagonal blocks are not read).  Operands
// are bf16 hi / lo (3 products), k = 0..63 in four steps of 16.
// Warps 0-3: state (warp w: chain w / 2, thread j = (w & 1) * 32 + lane owns
// column j of its chain's S = TMEM lane 64 c + j); warp 4: bulk copies of
// the two chains' M images (two stages); warp 5: MMA issuer.
// Operand images (d = 64): 64 rows of 128 B, 128-B swizzle, 8 KB each; M
// image element (j, k) = M[k][j] in row k; X image element (n, k) in row k.
// In: M images [BH][T] (hi 8 KB, lo 8 KB), B^T [BH][T][64][64].
// Out: boundary states [2][BH][NC + 1][64][64] as for d = 128.
// ===========================================================================
struct Scan64Cfg {
  static constexpr int THREADS = 192;
  static constexpr int PREFETCH = 3;
  static constexpr int WARP_PROD = 4;
  static constexpr int WARP_MMA = 5;
  static constexpr uint32_t IMG = 8192;                 // one 64 x 64 bf16 image
  static constexpr uint32_t MST = 4 * IMG;              // stage: hi c0, hi c1, lo c0, lo c1
  static constexpr uint32_t OFF_M = 0;                  // 2 stages
  static constexpr uint32_t OFF_X = 2 * MST;            // hi c0, hi c1, lo c0, lo c1
  static constexpr uint32_t BAR_OFF = OFF_X + 4 * IMG;
  static constexpr int NBAR = 2 + 2 + 1 + 1 + 1;         // mfull[2], mempty[2], xfull, dfull, drain
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};
constexpr uint32_t kImg64Bytes = 2 * Scan64Cfg::IMG;    // hi + lo image of one 64 x 64 matrix

__global__ void __launch_bounds__(Scan64Cfg::THREADS, 1)
k_scan64_tc(const uint8_t* __restrict__ Mimg, const float* __restrict__ Bt, const float* __restrict__ S0f,
            const float* __restrict__ S0r, const float* __restrict__ alpha, float* __restrict__ states, int BH,
            int T, int chunk, int NC) {
  using C = Scan64Cfg;
  constexpr int D = 64;
  constexpr size_t DD = 64 * 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
  const int MFULL = 0, MEMPTY = 2, XFULL = 4, DFULL = 5, DRAIN = 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  auto frame_of = [&](int c, int i) { return c == 0 ? i : T - 1 - i; };
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(MFULL + s), 1);
      mbar_init(BAR(MEMPTY + s), 1);
    }
    mbar_init(BAR(XFULL), 128);
    mbar_init(BAR(DFULL), 1);
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_wait_prerequisites();   // the M images and B^T are complete
  grid_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  int last_i[2] = {-1, -1};

  if (warp == C::WARP_PROD) {
    if (lane == 0) {
      for (int i = 0; i < T; ++i) {
        const uint32_t s = (uint32_t)i & 1u, ph = ((uint32_t)i >> 1) & 1u;
        if (!mbar_wait(BAR(MEMPTY + s), ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(BAR(MFULL + s), 4 * C::IMG);
        const uint32_t dst = sbase + C::OFF_M + s * C::MST;
        for (int c = 0; c < 2; ++c) {
          const uint8_t* src = Mimg + ((size_t)bh * T + frame_of(c, i)) * kImg64Bytes;
          bulk_load(dst + (uint32_t)c * C::IMG, src, C::IMG, BAR(MFULL + s));                 // hi
          bulk_load(dst + 2u * C::IMG + (uint32_t)c * C::IMG, src + C::IMG, C::IMG, BAR(MFULL + s));  // lo
          if (i + C::PREFETCH < T) {
            const size_t fa = (size_t)bh * T + frame_of(c, i + C::PREFETCH);
            bulk_prefetch_l2(Mimg + fa * kImg64Bytes, kImg64Bytes);
            bulk_prefetch_l2(Bt + fa * DD, (uint32_t)(DD * sizeof(float)));
          }
        }
        last_i[s] = i;
      }
    }
  } else if (warp == C::WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, 128, 1, 1);   // both MN-major
      for (int i = 0; i < T; ++i) {
        const uint32_t s = (uint32_t)i & 1u, ph = ((uint32_t)i >> 1) & 1u;
        if (!mbar_wait(BAR(MFULL + s), ph, abort_flag)) break;
        if (!mbar_wait(BAR(XFULL), (uint32_t)i & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t mh = sbase + C::OFF_M + s * C::MST, ml = mh + 2u * C::IMG;
        const uint32_t xh = sbase + C::OFF_X, xl = xh + 2u * C::IMG;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t ko = (uint32_t)ks * 2048u;   // 16 k-rows
          const uint64_t a_h = desc_sw128(mh + ko, C::IMG, 1024), a_l = desc_sw128(ml + ko, C::IMG, 1024);
          const uint64_t b_h = desc_sw128(xh + ko, C::IMG, 1024), b_l = desc_sw128(xl + ko, C::IMG, 1024);
          mma_bf16_ss(tmem, a_h, b_h, kId, ks != 0);
          mma_bf16_ss(tmem, a_h, b_l, kId, 1u);
          mma_bf16_ss(tmem, a_l, b_h, kId, 1u);
        }
        mma_commit(BAR(DFULL));
        mma_commit(BAR(MEMPTY + s));
      }
      mma_commit(BAR(DRAIN));
      mbar_wait_drain(BAR(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ---------------- state warps
    const int c = warp >> 1;                 // chain: 0 forward, 1 reverse
    const int j = (warp & 1) * 32 + lane;    // column j of the chain's S
    const float* S0 = c == 0 ? S0f : S0r;
    float* st = states + ((size_t)c * BH + bh) * (size_t)(NC + 1) * DD;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + 64u * (uint32_t)c;
    const uint32_t xrow = sbase + C::OFF_X + (uint32_t)c * C::IMG + (uint32_t)j * 128u;
    const uint32_t jsw = (uint32_t)(j & 7);
    float bnext[64];
    auto load_b = [&](int fr) {   // B[n][j] = B^T[j][n], n = 0..63: one contiguous row
      const float4* src = reinterpret_cast<const float4*>(Bt + ((size_t)bh * T + fr) * DD + (size_t)j * D);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 v = __ldg(src + q);
        bnext[4 * q] = v.x; bnext[4 * q + 1] = v.y; bnext[4 * q + 2] = v.z; bnext[4 * q + 3] = v.w;
      }
    };
    {   // initial state: the first boundary, X_0 = S0 Diag(alpha) + B
      const int j0 = c == 0 ? 0 : NC;
      const int f0 = frame_of(c, 0);
      load_b(f0);
      const float a0 = alpha ? __ldg(alpha + ((size_t)bh * T + f0) * D + j) : 1.f;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int n = 8 * cc + e;
          const float s0 = S0 ? __ldg(S0 + (size_t)bh * DD + (size_t)n * D + j) : 0.f;
          st[(size_t)j0 * DD + (size_t)n * D + j] = s0;
          x[e] = fmaf(s0, a0, bnext[n]);
        }
        const uint32_t o = xrow + (((uint32_t)cc ^ jsw) << 4);
        st_chunk_hilo(o, o + 2u * C::IMG, x);
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(XFULL));
    }
    for (int i = 0; i < T; ++i) {
      const bool more = i + 1 < T;
      const int t = frame_of(c, i);
      int jb = -1;
      if (c == 0) {
        if ((t + 1) % chunk == 0 || t == T - 1) jb = (t + chunk) / chunk;
      } else if (t % chunk == 0) {
        jb = t / chunk;
      }
      float anext = 1.f;
      if (more) {
        load_b(frame_of(c, i + 1));
        if (alpha) anext = __ldg(alpha + ((size_t)bh * T + frame_of(c, i + 1)) * D + j);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(DFULL), (uint32_t)i & 1u, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t v[16];
        tmem_ld16(trow + cb * 16, v);
        tmem_wait_ld();
        if (jb >= 0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) st[(size_t)jb * DD + (size_t)(cb * 16 + e) * D + j] = __uint_as_float(v[e]);
        }
        if (more) {
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = fmaf(__uint_as_float(v[8 * q2 + e]), anext, bnext[cb * 16 + 8 * q2 + e]);
            const uint32_t c8 = (uint32_t)(2 * cb + q2);
            const uint32_t o = xrow + ((c8 ^ jsw) << 4);
            st_chunk_hilo(o, o + 2u * C::IMG, x);
          }
        }
      }
      if (more) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(XFULL));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (warp == C::WARP_PROD && lane == 0 && *abort_flag) {
    for (int s = 0; s < 2; ++s)
      if (last_i[s] >= 0) mbar_wait_drain(BAR(MFULL + s), ((uint32_t)last_i[s] >> 1) & 1u);
  }
}

// ===========================================================================
// k_readout_tc: out = sigmoid(g) * w * o / sqrt(mean(o^2) + eps), o = S~ q.
// Work = 128-token tiles of each (b, h, chunk)'s contiguous token range; a
// persistent CTA takes a contiguous run of tiles.  Per tile the MMA computes
//   D[tok][i] = sum_k Q[tok][k] S~[i][k]     (S~ split into bf16 hi + lo)
// with Q from TMA (K-major, 128-B swizzle) and the S~ image in shared memory,
// built by the epilogue warps whenever the run enters a new (b, h, chunk):
//   S~ = fwd[max(0, c - w)] + rev[min(NC, c + w + 1)]   (Appendix A.3)
// TMEM lane = token row: two epilogue warps share a row quarter (the warps
// e and e + 4 reach the same TMEM lanes), each sums the squares of the whole
// row, in the same order, and writes one 64-column half.  Gates come through
// TMA as well; each output replaces its gate in the gate stage, and the gate
// producer sends the tile out by TMA (the partial tile at a chunk end is
// stored row by row instead).  The gate is sigmoid(g) = (1 + tanh(g/2)) / 2
// with the hardware tanh (one XU instruction per element), and the factor
// 1/2 is folded into the RMSNorm weight held in shared memory.
// Warps 0-7: epilogue + S~ builder; warp 8: Q producer; warp 9: MMA issuer;
// warp 10: gate producer (separate producers keep Q loads running ahead of
// the epilogue's release of gate stages).
// ===========================================================================
template <int D>   // d_k = d_v = 128 or 64
struct ReadoutCfgT {
  static constexpr int NEPI = 256;                             // epilogue threads (warps 0-7)
  static constexpr int WARP_Q = 8, WARP_MMA = 9, WARP_G = 10;
  static constexpr int THREADS = 352;
  static constexpr int TILE = 128;
  static constexpr int NB = D / 64;                            // 64-channel boxes of a tile
  static constexpr int HALF = D / 2;                           // output columns per epilogue thread
  static constexpr uint32_t BOX_BYTES = TILE * 128;            // 128 rows x 64 bf16
  static constexpr uint32_t TILE_BYTES = NB * BOX_BYTES;       // 128 rows x D bf16
  static constexpr uint32_t SIMG = D * D * 2;                  // one bf16 S~ image (hi or lo)
  static constexpr uint32_t OFF_S = 0;                         // S~ hi + lo
  static constexpr uint32_t OFF_Q = 2 * SIMG;                  // 2 Q stages
  static constexpr int NG = 2;                                  // gate stages (also hold the output)
  static constexpr uint32_t OFF_G = OFF_Q + 2 * TILE_BYTES;     // NG gate stages
  static constexpr uint32_t OFF_W = OFF_G + NG * TILE_BYTES;    // D floats
  static constexpr uint32_t BAR_OFF = OFF_W + 512;
  // qfull[2], qempty[2], gfull[NG], gout[NG], tfull[2], tempty[2], sready, drain
  static constexpr int NBAR = 10 + 2 * NG;
  static constexpr size_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
};
using ReadoutCfg = ReadoutCfgT<128>;

struct ReadoutGeom {
  int BH, T, U, chunk, NC, window;
  int unit;        // frames per unit of equal read state: chunk, or 1 with the decay bridge
  int frame_out;   // output map is [frames][U][128]: every tile of a one-frame unit leaves by TMA
  int NU;          // units per head
  int tpc;         // tiles of a full unit
  int tlast;       // tiles of the last unit
  int tph;         // tiles per head
  long long total; // tiles over all heads
};

// tile index -> (bh, unit u, first row of the tile relative to the unit, rows of the unit)
__device__ __forceinline__ void tile_coords(const ReadoutGeom& g, long long gt, int& bh, int& u, int& tr, int& rows) {
  bh = (int)(gt / g.tph);
  int rem = (int)(gt - (long long)bh * g.tph);
  u = rem / g.tpc;
  if (u > g.NU - 1) u = g.NU - 1;
  tr = (rem - u * g.tpc) * ReadoutCfg::TILE;
  const int f0 = u * g.unit;
  const int f1 = min(g.T, f0 + g.unit);
  rows = (f1 - f0) * g.U;
}

template <int D>
__global__ void __launch_bounds__(ReadoutCfgT<D>::THREADS, 1)
k_readout_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
             const __grid_constant__ CUtensorMap tmO,
             const float* __restrict__ w, const float* __restrict__ states, const float* __restrict__ bridge,
             __nv_bfloat16* __restrict__ out, ReadoutGeom g, float eps) {
  using C = ReadoutCfgT<D>;
  constexpr size_t DD = (size_t)D * D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
  const int QFULL = 0, QEMPTY = 2, GFULL = 4, GOUT = 4 + C::NG, TFULL = 4 + 2 * C::NG, TEMPTY = TFULL + 2,
            SREADY = TFULL + 4, DRAIN = TFULL + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sw = reinterpret_cast<float*>(smem + C::OFF_W);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // contiguous run of tiles of this CTA
  const long long t_begin = g.total * blockIdx.x / gridDim.x;
  const long long t_end = g.total * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(QFULL + s), 1);
      mbar_init(BAR(QEMPTY + s), 1);
      mbar_init(BAR(TFULL + s), 1);
      mbar_init(BAR(TEMPTY + s), C::NEPI);
    }
    for (int s = 0; s < C::NG; ++s) {
      mbar_init(BAR(GFULL + s), 1);
      mbar_init(BAR(GOUT + s), C::NEPI);
    }
    mbar_init(BAR(SREADY), C::NEPI);
    mbar_init(BAR(DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 2 * D);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  grid_wait_prerequisites();   // boundary states are complete (see k_stats_tc)
  grid_launch_dependents();
  if (tid < D) sw[tid] = 0.5f * w[tid];
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long tokens_per_head = (long long)g.T * g.U;
  int last_q[2] = {-1, -1}, last_g[C::NG];   // producer: last tile issued per stage
  for (int q = 0; q < C::NG; ++q) last_g[q] = -1;

  if (warp == C::WARP_Q || warp == C::WARP_G) {
    // ---------------- TMA producers: Q tiles; gate tiles,
    // which also sends each output tile out of the gate stage it replaced
    if (lane == 0) {
      const bool is_q = warp == C::WARP_Q;
      const CUtensorMap* map = is_q ? &tmQ : &tmG;
      const uint32_t base = sbase + (is_q ? C::OFF_Q : C::OFF_G);
      int* last = is_q ? last_q : last_g;
      const int ns = is_q ? 2 : C::NG;
      // output tile of tile index gt (stage s) -> global, when it is a full tile
      auto store_out = [&](long long gt, uint32_t s) {
        int bh, c, tr, rows;
        tile_coords(g, gt, bh, c, tr, rows);
        const uint32_t src = base + s * C::TILE_BYTES;
        if (g.frame_out) {   // rows past the frame's U are outside the map: not written
          const int fh = bh * g.T + c;
#pragma unroll
          for (int bx = 0; bx < C::NB; ++bx) tma_store_3d(&tmO, src + bx * C::BOX_BYTES, 64 * bx, tr, fh);
          bulk_commit_group();
        } else if (tr + C::TILE <= rows) {
          const int row0 = (int)((long long)bh * tokens_per_head + (long long)c * g.unit * g.U + tr);
#pragma unroll
          for (int bx = 0; bx < C::NB; ++bx) tma_store_2d(&tmO, src + bx * C::BOX_BYTES, 64 * bx, row0);
          bulk_commit_group();
        }
      };
      bool ok = true;
      int k = 0;
      for (long long gt = t_begin; gt < t_end; ++gt, ++k) {
        int bh, c, tr, rows;
        tile_coords(g, gt, bh, c, tr, rows);
        const int row0 = (int)((long long)bh * tokens_per_head + (long long)c * g.unit * g.U + tr);
        const uint32_t s = (uint32_t)(k % ns), ph = (uint32_t)(k / ns) & 1u;
        if (is_q) {
          if (!mbar_wait(BAR(QEMPTY + s), ph ^ 1u, abort_flag)) { ok = false; break; }
        } else if (k >= C::NG) {   // the stage holds tile k-NG's output: send it, let the copy read it
          if (!mbar_wait(BAR(GOUT + s), ph ^ 1u, abort_flag)) { ok = false; break; }
          store_out(gt - C::NG, s);
          bulk_wait_read_all();
        }
        const int FULLB = is_q ? QFULL : GFULL;
        mbar_arrive_expect_tx(BAR(FULLB + s), C::TILE_BYTES);
        const uint32_t dst = base + s * C::TILE_BYTES;
#pragma unroll
        for (int bx = 0; bx < C::NB; ++bx) tma_load_2d(dst + bx * C::BOX_BYTES, map, 64 * bx, row0, BAR(FULLB + s));
        last[s] = k;
      }
      if (!is_q && ok) {   // the last NG output tiles
        const int n = k;
        for (int kk = max(0, n - C::NG); kk < n; ++kk) {
          const uint32_t s = (uint32_t)(kk % C::NG), ph = (uint32_t)(kk / C::NG) & 1u;
          if (!mbar_wait(BAR(GOUT + s), ph, abort_flag)) break;
          store_out(t_begin + kk, s);
        }
      }
      if (!is_q) bulk_wait_all();   // output copies complete before the CTA retires
    }
  } else if (warp == C::WARP_MMA) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16(128, D, 0, 0);   // both K-major
      const uint32_t sh = sbase + C::OFF_S, sl = sh + C::SIMG;
      int k = 0, npair = 0, prev_bh = -1, prev_c = -1;
      for (long long gt = t_begin; gt < t_end; ++gt, ++k) {
        int bh, c, tr, rows;
        tile_coords(g, gt, bh, c, tr, rows);
        if (bh != prev_bh || c != prev_c) {
          if (!mbar_wait(BAR(SREADY), (uint32_t)npair & 1u, abort_flag)) break;
          ++npair;
          prev_bh = bh;
          prev_c = c;
        }
        const uint32_t s = (uint32_t)k & 1u, ph = ((uint32_t)k >> 1) & 1u;
        if (!mbar_wait(BAR(QFULL + s), ph, abort_flag)) break;
        if (!mbar_wait(BAR(TEMPTY + s), ph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t q = sbase + C::OFF_Q + s * C::TILE_BYTES;
        const uint32_t d = tmem + s * (uint32_t)D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          // k-block ks / 4 of 64 channels: a 16 KB box of Q, a (D x 128 B) block of S~
          const uint32_t kc = (uint32_t)(ks & 3) * 32u;
          const uint64_t a = desc_sw128(q + (uint32_t)(ks >> 2) * C::BOX_BYTES + kc, 16, 1024);
          const uint32_t so = (uint32_t)(ks >> 2) * (uint32_t)(D * 128) + kc;
          mma_bf16_ss(d, a, desc_sw128(sh + so, 16, 1024), kId, ks != 0);
          mma_bf16_ss(d, a, desc_sw128(sl + so, 16, 1024), kId, 1u);
        }
        mma_commit(BAR(QEMPTY + s));
        mma_commit(BAR(TFULL + s));
      }
      mma_commit(BAR(DRAIN));
      mbar_wait_drain(BAR(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue + S~ builder: thread = (token row r, column half ch)
    const int r = (warp & 3) * 32 + lane, ch = warp >> 2;
    const uint32_t trow_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t simg_s = sbase + C::OFF_S;
    const uint32_t sw_s = sbase + C::OFF_W + (uint32_t)(C::HALF * 4) * (uint32_t)ch;   // w/2 of this half
    int k = 0, prev_bh = -1, prev_c = -1;
    const size_t sdir = (size_t)g.BH * (size_t)(g.NC + 1) * DD;
    for (long long gt = t_begin; gt < t_end; ++gt, ++k) {
      int bh, c, tr, rows;
      tile_coords(g, gt, bh, c, tr, rows);
      if (bh != prev_bh || c != prev_c) {
        // build S~ = fwd[max(0, c-w)] + rev[min(NC, c+w+1)] (chunk c of this unit),
        // with the decay bridge fwd Diag(bl) + rev Diag(br) of frame u (Eq. A.4):
        // row i = r (rows below D), this half's columns
        const int cc_ = (c * g.unit) / g.chunk;
        const int jf = max(0, cc_ - g.window), jr = min(g.NC, cc_ + g.window + 1);
        const int rs = r < D ? r : 0;
        const float* bl = bridge ? bridge + (((size_t)bh * g.T + c) * 2) * D + C::HALF * ch : nullptr;
        const float* Sf =
            states + (size_t)bh * (size_t)(g.NC + 1) * DD + (size_t)jf * DD + (size_t)rs * D + C::HALF * ch;
        const float* Sr = states + sdir + (size_t)bh * (size_t)(g.NC + 1) * DD + (size_t)jr * DD +
                          (size_t)rs * D + C::HALF * ch;
#pragma unroll 4
        for (int cc = 0; cc < C::HALF / 8; ++cc) {
          if (r >= D) break;
          const float4 f0 = __ldg(reinterpret_cast<const float4*>(Sf + cc * 8));
          const float4 f1 = __ldg(reinterpret_cast<const float4*>(Sf + cc * 8 + 4));
          const float4 r0v = __ldg(reinterpret_cast<const float4*>(Sr + cc * 8));
          const float4 r1v = __ldg(reinterpret_cast<const float4*>(Sr + cc * 8 + 4));
          float x[8] = {f0.x + r0v.x, f0.y + r0v.y, f0.z + r0v.z, f0.w + r0v.w,
                        f1.x + r1v.x, f1.y + r1v.y, f1.z + r1v.z, f1.w + r1v.w};
          if (bl) {
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(bl + cc * 8));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(bl + cc * 8 + 4));
            const float4 b0 = __ldg(reinterpret_cast<const float4*>(bl + D + cc * 8));
            const float4 b1 = __ldg(reinterpret_cast<const float4*>(bl + D + cc * 8 + 4));
            x[0] = fmaf(f0.x, a0.x, r0v.x * b0.x); x[1] = fmaf(f0.y, a0.y, r0v.y * b0.y);
            x[2] = fmaf(f0.z, a0.z, r0v.z * b0.z); x[3] = fmaf(f0.w, a0.w, r0v.w * b0.w);
            x[4] = fmaf(f1.x, a1.x, r1v.x * b1.x); x[5] = fmaf(f1.y, a1.y, r1v.y * b1.y);
            x[6] = fmaf(f1.z, a1.z, r1v.z * b1.z); x[7] = fmaf(f1.w, a1.w, r1v.w * b1.w);
          }
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float h0, l0, h1, l1;
            split_bf16(x[2 * q], h0, l0);
            split_bf16(x[2 * q + 1], h1, l1);
            hw[q] = pack_bf16(h0, h1);
            lw[q] = pack_bf16(l0, l1);
          }
          // row i = r, columns k: k-block k / 64 of D rows x 128 B, 128-B swizzle
          const uint32_t kk = (uint32_t)(C::HALF * ch + cc * 8);
          const uint32_t off = (kk >> 6) * (uint32_t)(D * 128) + sw128_offset((uint32_t)r, kk & 63u);
          st_shared_v4(simg_s + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
          st_shared_v4(simg_s + C::SIMG + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
        }
        fence_proxy_async_smem();
        mbar_arrive(BAR(SREADY));
        prev_bh = bh;
        prev_c = c;
      }
      const uint32_t s = (uint32_t)k & 1u, ph = ((uint32_t)k >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(TFULL + s), ph, abort_flag))) break;
      tc_fence_after();
      // sum of squares over the whole row (both halves, fixed order); keep this half
      float o[C::HALF];
      float ss = 0.f;
      const uint32_t trow = trow_base + s * (uint32_t)D;
#pragma unroll
      for (int j2 = 0; j2 < 2; ++j2) {
#pragma unroll
        for (int j3 = 0; j3 < C::HALF / 32; ++j3) {
          uint32_t v0[32];
          tmem_ld32(trow + (uint32_t)(C::HALF * j2 + 32 * j3), v0);
          tmem_wait_ld();
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            const float a0 = __uint_as_float(v0[c2]);
            ss = fmaf(a0, a0, ss);
          }
          if (j2 == ch) {
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) o[32 * j3 + c2] = __uint_as_float(v0[c2]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(TEMPTY + s));
      const float rinv = rsqrtf(ss * (1.0f / D) + eps);
      const uint32_t sg = (uint32_t)(k % C::NG), phg = (uint32_t)(k / C::NG) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(GFULL + sg), phg, abort_flag))) break;
      const uint32_t gt_s = sbase + C::OFF_G + sg * C::TILE_BYTES;
      const bool valid = tr + r < rows;
      // a tile inside its chunk leaves by TMA from the gate stage (y replaces
      // g in place); the chunk's last, partial tile by per-row stores
      const bool tma_out = g.frame_out || tr + C::TILE <= rows;
      __nv_bfloat16* orow =
          out + ((size_t)bh * tokens_per_head + (size_t)c * g.unit * g.U + tr + r) * D + C::HALF * ch;
#pragma unroll
      for (int cb = 0; cb < C::HALF / 32; ++cb) {   // 4 chunks of 8 columns at a time, loads first
        uint4 gv[4];
        float4 wv[8];
        uint32_t off[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int cc = 4 * cb + q4;
          const uint32_t col = (uint32_t)(C::HALF * ch + cc * 8);   // column of the tile: box col / 64
          off[q4] = (col >> 6) * C::BOX_BYTES + sw128_offset((uint32_t)r, col & 63u);
          gv[q4] = ld_shared_v4(gt_s + off[q4]);
          wv[2 * q4] = ld_shared_f4(sw_s + (uint32_t)cc * 32u);
          wv[2 * q4 + 1] = ld_shared_f4(sw_s + (uint32_t)cc * 32u + 16u);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int cc = 4 * cb + q4;
          const float wh[8] = {wv[2 * q4].x, wv[2 * q4].y, wv[2 * q4].z, wv[2 * q4].w,
                               wv[2 * q4 + 1].x, wv[2 * q4 + 1].y, wv[2 * q4 + 1].z, wv[2 * q4 + 1].w};
          const uint32_t gw[4] = {gv[q4].x, gv[q4].y, gv[q4].z, gv[q4].w};
          uint32_t yw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i0 = cc * 8 + 2 * q;
            const float g0 = __uint_as_float(gw[q] << 16), g1 = __uint_as_float(gw[q] & 0xFFFF0000u);
            // y = w * o * rinv * sigmoid(g),  sigmoid(g) = (1 + tanh(g / 2)) / 2, w/2 in wh
            const float a0 = o[i0] * rinv * wh[2 * q], a1 = o[i0 + 1] * rinv * wh[2 * q + 1];
            const float y0 = fmaf(a0, tanh_approx(0.5f * g0), a0);
            const float y1 = fmaf(a1, tanh_approx(0.5f * g1), a1);
            yw[q] = pack_bf16(y0, y1);
          }
          if (tma_out) st_shared_v4(gt_s + off[q4], make_uint4(yw[0], yw[1], yw[2], yw[3]));
          else if (valid) *reinterpret_cast<uint4*>(orow + cc * 8) = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        }
      }
      if (tma_out) fence_proxy_async_smem();
      mbar_arrive(BAR(GOUT + sg));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * D);
  }
  if ((warp == C::WARP_Q || warp == C::WARP_G) && lane == 0 && *abort_flag) {  // let issued copies land
    const int* last = warp == C::WARP_Q ? last_q : last_g;
    const int FULLB = warp == C::WARP_Q ? QFULL : GFULL;
    const int ns = warp == C::WARP_Q ? 2 : C::NG;
    for (int s = 0; s < ns; ++s)
      if (last[s] >= 0) mbar_wait_drain(BAR(FULLB + s), (uint32_t)(last[s] / ns) & 1u);
  }
}

// ===========================================================================
// host side
// ===========================================================================
}  // namespace tc

// With VDA_DEBUG_SYNC=1 in the environment, every stage is followed by a
// stream synchronisation and a check of the device error word, and a failing
// stage is named on stderr (a debugging aid; off by default).
inline bool debug_sync_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("VDA_DEBUG_SYNC");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

inline int debug_check(const char* stage, cudaStream_t s) {
  if (!debug_sync_enabled()) return VDA_OK;
  const cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "vda: stage %s failed: %s\n", stage, cudaGetErrorString(e));
    return VDA_ERR_CUDA;
  }
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) == cudaSuccess && word != 0) {
    fprintf(stderr, "vda: stage %s gave up a bounded wait (device error word %u)\n", stage, word);
    return VDA_ERR_TIMEOUT;
  }
  return VDA_OK;
}

// Status of the launch just made; names the kernel and the CUDA error on
// stderr in debug mode.
inline int launch_status(const char* kernel) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return VDA_OK;
  if (debug_sync_enabled()) fprintf(stderr, "vda: launch of %s failed: %s\n", kernel, cudaGetErrorString(e));
  return VDA_ERR_CUDA;
}

namespace tc {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor [outer][mid][128] with a box of 64 x box_mid x 1, 128-B swizzle
// bf16 tensors with `width` (64 or 128) channels per row, 64-channel boxes
inline bool encode_bf16_3d(CUtensorMap* m, const void* base, uint64_t mid, uint64_t outer, uint32_t box_mid,
                           uint32_t width = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {width, mid, outer};
  cuuint64_t strides[2] = {2ull * width, mid * 2ull * width};
  cuuint32_t box[3] = {64, box_mid, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 matrix [rows][128] with a box of 64 x box_rows, 128-B swizzle
inline bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows,
                           uint32_t width = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {width, rows};
  cuuint64_t strides[1] = {2ull * width};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialisation: the kernel's CTAs may start
// while the previous grid on the stream finishes; each of the four kernels
// waits for that grid (griddepcontrol.wait) before reading what it wrote.
template <typename... Params, typename... Args>
inline int launch_pdl(const char* name, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    cudaGetLastError();   // reported through the status instead
    if (debug_sync_enabled()) fprintf(stderr, "vda: launch of %s failed: %s\n", name, cudaGetErrorString(e));
    return VDA_ERR_CUDA;
  }
  return launch_status(name);
}

inline int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// frame statistics for FH frame-heads of U tokens (K, V: [FH][U][128] bf16)
// Statistics for FH frame-heads of U tokens (K, V: [FH][U][128] bf16):
// A [FH][d_k][d_k] and B [FH][d_v][d_k], fp32.
inline int launch_stats(const void* K, const void* V, const float* beta, int U, size_t FH, float* A, float* B,
                        float* A_full, cudaStream_t s) {
  CUtensorMap tmK, tmV;
  if (!encode_bf16_3d(&tmK, K, (uint64_t)U, FH, 64) || !encode_bf16_3d(&tmV, V, (uint64_t)U, FH, 64))
    return VDA_ERR_CUDA;
  if (cudaFuncSetAttribute(k_stats_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StatsCfg::SMEM) !=
      cudaSuccess)
    return launch_status("k_stats_tc (shared-memory attribute)");
  // as many rounds as num_sms CTAs need, over as few CTAs as keep that count:
  // every CTA then takes the same number of frame-heads (2880 = 144 x 20 at
  // full size) instead of a last, partial round on part of the SMs
  const size_t sms = (size_t)num_sms();
  const size_t rounds = (FH + sms - 1) / sms;
  const int grid = (int)((FH + rounds - 1) / rounds);
  return launch_pdl("k_stats_tc", k_stats_tc, dim3(grid), dim3(StatsCfg::THREADS), StatsCfg::SMEM, s, tmK, tmV, beta,
                    U, (int)FH, A, B, A_full);
}

// M = (I + A)^{-1} images (and optional fp32 copy) for FH matrices
inline int launch_inverse(const float* A, size_t FH, uint8_t* Mimg, float* M_dbg, cudaStream_t s) {
  if (cudaFuncSetAttribute(k_inverse_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)InvCfg::SMEM) !=
      cudaSuccess)
    return launch_status("k_inverse_tc (shared-memory attribute)");
  const size_t per_cta = (size_t)InvCfg::GROUPS;
  const int grid = (int)std::min<size_t>((FH + per_cta - 1) / per_cta, (size_t)num_sms());
  return launch_pdl("k_inverse_tc", k_inverse_tc, dim3(grid), dim3(InvCfg::THREADS), InvCfg::SMEM, s, A, (int)FH,
                    Mimg, M_dbg);
}

template <int MODE>
inline int launch_scan_mode(const ScanArgs& sa, dim3 grid, cudaStream_t s) {
  if (cudaFuncSetAttribute(k_scan_tc<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ScanCfg::SMEM) !=
      cudaSuccess)
    return VDA_ERR_CUDA;
  const char* name = MODE == kScanFrames ? "k_scan_tc<frames>"
                                         : (MODE == kScanCompose ? "k_scan_tc<compose>" : "k_scan_tc<chunks>");
  return launch_pdl(name, k_scan_tc<MODE>, grid, dim3(ScanCfg::THREADS), ScanCfg::SMEM, s, sa);
}

// Per-frame scans: one CTA per (b, h, direction), T steps.
inline int launch_scan(const uint8_t* Mimg, const float* Bm, const float* S0f, const float* S0r,
                       const float* alpha, float* states, size_t BH, int T, int chunk, int NC, int ndir,
                       cudaStream_t s) {
  const ScanArgs sa{Mimg, Bm, S0f, S0r, alpha, states, nullptr, nullptr, (int)BH, T, chunk, NC};
  return launch_scan_mode<kScanFrames>(sa, dim3((unsigned)BH, (unsigned)ndir), s);
}

// Bytes of the chunk maps of the chunk-wise scans: J_c (fp32) and the P_c
// operand image for every (direction, b, h, chunk).
inline size_t chunk_maps_bytes(size_t BH, int NC) {
  return 2 * BH * (size_t)NC * (kDD * sizeof(float) + kImgBytes);
}

// Chunk-wise scans: compose every chunk's maps (2 x 2 x BH x NC CTAs of at
// most `chunk` steps), then scan the NC maps per chain.  `maps` holds
// chunk_maps_bytes(BH, NC) bytes, 256-B aligned.
template <typename Timer>
inline int launch_scan_chunked(const uint8_t* Mimg, const float* Bm, const float* S0f, const float* S0r,
                               const float* alpha, float* states, char* maps, size_t BH, int T, int chunk,
                               int NC, cudaStream_t s, Timer& timer) {
  float* J = reinterpret_cast<float*>(maps);
  uint8_t* P = reinterpret_cast<uint8_t*>(maps + 2 * BH * (size_t)NC * kDD * sizeof(float));
  const ScanArgs comp{Mimg, Bm, nullptr, nullptr, alpha, nullptr, J, P, (int)BH, T, chunk, NC};
  int rc = launch_scan_mode<kScanCompose>(comp, dim3((unsigned)(4 * BH * (size_t)NC)), s);
  if (rc != VDA_OK) return rc;
  timer.end(2, s);
  timer.begin(2, s);
  const ScanArgs chains{P, J, S0f, S0r, nullptr, states, nullptr, nullptr, (int)BH, T, chunk, NC};
  return launch_scan_mode<kScanChunks>(chains, dim3((unsigned)BH, 2u), s);
}

template <int D>
inline int launch_readout(const void* Q, const void* G, const float* w, const float* states, const float* bridge,
                          void* out, size_t BH, int T, int U, int chunk, int NC, int window, float eps,
                          cudaStream_t s) {
  ReadoutGeom g{};
  g.BH = (int)BH; g.T = T; g.U = U; g.chunk = chunk; g.NC = NC; g.window = window;
  // with the decay bridge the read state changes every frame: one unit per frame,
  // and the output map is 3-D by frame so that TMA clips each frame's last tile
  g.unit = bridge ? 1 : chunk;
  g.frame_out = bridge ? 1 : 0;
  g.NU = (T + g.unit - 1) / g.unit;
  const long long rows_full = (long long)std::min(T, g.unit) * U;
  const long long rows_last = (long long)(T - (g.NU - 1) * g.unit) * U;
  g.tpc = (int)((rows_full + ReadoutCfg::TILE - 1) / ReadoutCfg::TILE);
  g.tlast = (int)((rows_last + ReadoutCfg::TILE - 1) / ReadoutCfg::TILE);
  g.tph = (g.NU - 1) * g.tpc + g.tlast;
  g.total = (long long)BH * g.tph;
  const uint64_t rows = (uint64_t)BH * T * U;
  CUtensorMap tmQ, tmG, tmO;
  using RC = ReadoutCfgT<D>;
  const bool okO = g.frame_out ? encode_bf16_3d(&tmO, out, (uint64_t)U, (uint64_t)BH * T, RC::TILE, D)
                               : encode_bf16_2d(&tmO, out, rows, RC::TILE, D);
  if (!encode_bf16_2d(&tmQ, Q, rows, RC::TILE, D) || !encode_bf16_2d(&tmG, G, rows, RC::TILE, D) || !okO)
    return VDA_ERR_CUDA;
  if (cudaFuncSetAttribute(k_readout_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RC::SMEM) !=
      cudaSuccess)
    return VDA_ERR_CUDA;
  const int grid = (int)std::min<long long>(g.total, (long long)num_sms());
  return launch_pdl("k_readout_tc", k_readout_tc<D>, dim3(grid), dim3(RC::THREADS), RC::SMEM, s, tmQ,
                    tmG, tmO, w, states, bridge, static_cast<__nv_bfloat16*>(out), g, eps);
}

}  // namespace tc

// ---------------------------------------------------------------------------
// path selection and the staged launch used by vda.cu
inline bool tc_path_supported(int d, int dtype) { return (d == 128 || d == 64) && dtype == VDA_BF16; }

// extra workspace of the tensor-core path: the M hi/lo operand images
// (64 KB per frame-head), next to A
inline size_t tc_extra_workspace_bytes(bool tc, size_t FH, int d) {
  if (!tc) return 0;
  return FH * (size_t)(d == 64 ? tc::kImg64Bytes : tc::kImgBytes);
}

// Scan form of the tensor-core path.  Automatic choice: the chunk-wise scans
// when their composition CTAs (4 per (b, h) and chunk) fill the GPU in at
// most two waves (few (b, h) pairs: the per-frame chains would leave most SMs
// idle for T steps), else the per-frame scans.
inline bool use_chunk_scan(int form, size_t BH, int T, int chunk, int NC, int sms) {
  if (form == VDA_SCAN_FRAMES) return false;
  if (form == VDA_SCAN_CHUNKS) return true;
  return chunk > 1 && T > chunk && 4 * BH * (size_t)NC <= 2 * (size_t)sms;
}

// Kernel launches of one forward on the tensor-core path (without the decay
// bridge): the chunk-wise scans take two.
inline int tc_launches_per_forward(int d, int form, size_t BH, int T, int chunk, int NC) {
  if (d != 128) return 4;   // d = 64: Gram, inverse, paired-chain scans, readout
  return use_chunk_scan(form, BH, T, chunk, NC, tc::num_sms()) ? 5 : 4;
}

// The launch schedule on the caller's stream: Gram kernel, inverse, scan,
// decay bridge (with a decay gate), readout.  Timer hooks begin(stage, stream)
// / end(stage, stream) bracket each launch (stage 0 stats, 1 inverse, 2 scan,
// 3 readout).
template <typename Timer>
int launch_tc(size_t BH, int T, int U, int chunk, int NC, int window, const vda_args& a, char* ws_AM,
              char* ws_B, char* ws_states, char* ws_img, char* ws_bridge, char* ws_maps, cudaStream_t s,
              float* stats_out, Timer& timer) {
  const size_t FH = BH * (size_t)T;
  const size_t fdd = FH * tc::kDD;
  float* A = reinterpret_cast<float*>(ws_AM);
  float* Bt = reinterpret_cast<float*>(ws_B);
  float* st = reinterpret_cast<float*>(ws_states);
  uint8_t* img = reinterpret_cast<uint8_t*>(ws_img);
  int rc;
  timer.begin(0, s);
  if ((rc = tc::launch_stats(a.k, a.v, a.beta, U, FH, A, Bt, stats_out, s)) != VDA_OK) return rc;
  timer.end(0, s);
  if ((rc = debug_check("stats", s)) != VDA_OK) return rc;
  if (stats_out &&   // (the Gram kernel wrote the full A there)
      cudaMemcpyAsync(stats_out + fdd, Bt, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VDA_ERR_CUDA;
  timer.begin(1, s);
  if ((rc = tc::launch_inverse(A, FH, img, stats_out ? stats_out + 2 * fdd : nullptr, s)) != VDA_OK) return rc;
  timer.end(1, s);
  if ((rc = debug_check("inverse", s)) != VDA_OK) return rc;
  timer.begin(2, s);
  if (use_chunk_scan(a.scan_form, BH, T, chunk, NC, tc::num_sms()))
    rc = tc::launch_scan_chunked(img, Bt, a.S0_fwd, a.S0_rev, a.alpha, st, ws_maps, BH, T, chunk, NC, s, timer);
  else
    rc = tc::launch_scan(img, Bt, a.S0_fwd, a.S0_rev, a.alpha, st, BH, T, chunk, NC, 2, s);
  if (rc != VDA_OK) return rc;
  timer.end(2, s);
  if ((rc = debug_check("scan", s)) != VDA_OK) return rc;
  float* bridge = nullptr;
  if (a.alpha) {   // products of the decay bridge (Eq. A.4), one per (b, h, frame, key channel)
    bridge = reinterpret_cast<float*>(ws_bridge);
    const size_t n = FH * (size_t)tc::kD;
    k_decay_bridge<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.alpha, (int)BH, T, tc::kD, chunk, window, bridge);
    if ((rc = launch_status("k_decay_bridge")) != VDA_OK) return rc;
  }
  const float eps = a.eps > 0.f ? a.eps : 1e-6f;
  timer.begin(3, s);
  if ((rc = tc::launch_readout<128>(a.q, a.gate, a.rms_weight, st, bridge, a.out, BH, T, U, chunk, NC, window, eps,
                               s)) != VDA_OK)
    return rc;
  timer.end(3, s);
  return debug_check("readout", s);
}

// The d = 64 schedule: Gram kernel (operands swapped, M = 128), the FP32
// Gauss-Jordan inverse (which also writes the scan's operand image), the
// paired-chain scans, decay bridge (with a decay gate), readout.
template <typename Timer>
int launch_tc64(size_t BH, int T, int U, int chunk, int NC, int window, const vda_args& a, char* ws_AM,
                char* ws_B, char* ws_states, char* ws_img, char* ws_bridge, cudaStream_t s, float* stats_out,
                Timer& timer) {
  constexpr int D = 64;
  const size_t FH = BH * (size_t)T;
  const size_t fdd = FH * (size_t)D * D;
  float* AM = reinterpret_cast<float*>(ws_AM);
  float* Bt = reinterpret_cast<float*>(ws_B);
  float* st = reinterpret_cast<float*>(ws_states);
  uint8_t* img = reinterpret_cast<uint8_t*>(ws_img);
  int rc;
  {
    CUtensorMap tmK, tmV;
    if (!tc::encode_bf16_3d(&tmK, a.k, (uint64_t)U, FH, 64, D) || !tc::encode_bf16_3d(&tmV, a.v, (uint64_t)U, FH, 64, D))
      return VDA_ERR_CUDA;
    if (cudaFuncSetAttribute(tc::k_stats64_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::Stats64Cfg::SMEM) != cudaSuccess)
      return launch_status("k_stats64_tc (shared-memory attribute)");
    const size_t sms = (size_t)tc::num_sms();
    const size_t rounds = (FH + sms - 1) / sms;
    const int grid = (int)((FH + rounds - 1) / rounds);
    timer.begin(0, s);
    rc = tc::launch_pdl("k_stats64_tc", tc::k_stats64_tc, dim3(grid), dim3(tc::Stats64Cfg::THREADS),
                        tc::Stats64Cfg::SMEM, s, tmK, tmV, a.beta, U, (int)FH, AM, Bt,
                        stats_out ? stats_out + fdd : nullptr);
    if (rc != VDA_OK) return rc;
    timer.end(0, s);
  }
  if ((rc = debug_check("stats", s)) != VDA_OK) return rc;
  if (stats_out && cudaMemcpyAsync(stats_out, AM, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VDA_ERR_CUDA;
  timer.begin(1, s);
  k_gj_inverse<D><<<(unsigned)FH, 256, 0, s>>>(AM, img);
  if ((rc = launch_status("k_gj_inverse")) != VDA_OK) return rc;
  timer.end(1, s);
  if ((rc = debug_check("inverse", s)) != VDA_OK) return rc;
  if (stats_out &&
      cudaMemcpyAsync(stats_out + 2 * fdd, AM, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VDA_ERR_CUDA;
  if (cudaFuncSetAttribute(tc::k_scan64_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tc::Scan64Cfg::SMEM) != cudaSuccess)
    return VDA_ERR_CUDA;
  timer.begin(2, s);
  rc = tc::launch_pdl("k_scan64_tc", tc::k_scan64_tc, dim3((unsigned)BH), dim3(tc::Scan64Cfg::THREADS),
                      tc::Scan64Cfg::SMEM, s, (const uint8_t*)img, (const float*)Bt, a.S0_fwd, a.S0_rev, a.alpha,
                      st, (int)BH, T, chunk, NC);
  if (rc != VDA_OK) return rc;
  timer.end(2, s);
  if ((rc = debug_check("scan", s)) != VDA_OK) return rc;
  float* bridge = nullptr;
  if (a.alpha) {
    bridge = reinterpret_cast<float*>(ws_bridge);
    const size_t n = FH * (size_t)D;
    k_decay_bridge<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.alpha, (int)BH, T, D, chunk, window, bridge);
    if ((rc = launch_status("k_decay_bridge")) != VDA_OK) return rc;
  }
  const float eps = a.eps > 0.f ? a.eps : 1e-6f;
  timer.begin(3, s);
  if ((rc = tc::launch_readout<D>(a.q, a.gate, a.rms_weight, st, bridge, a.out, BH, T, U, chunk, NC, window, eps,
                                  s)) != VDA_OK)
    return rc;
  timer.end(3, s);
  return debug_check("readout", s);
}

// text state on the tensor-core kernels: stats over one frame of L tokens per
// (b, h), inverse, one forward scan step from the zero state
inline int tc_text_state(size_t BH, int L, const void* k, const void* v, const float* beta, char* ws_AM,
                         char* ws_B, char* ws_states, char* ws_img, cudaStream_t s) {
  float* A = reinterpret_cast<float*>(ws_AM);
  float* Bt = reinterpret_cast<float*>(ws_B);
  uint8_t* img = reinterpret_cast<uint8_t*>(ws_img);
  int rc;
  if ((rc = tc::launch_stats(k, v, beta, L, BH, A, Bt, nullptr, s)) != VDA_OK) return rc;
  if ((rc = tc::launch_inverse(A, BH, img, nullptr, s)) != VDA_OK) return rc;
  return tc::launch_scan(img, Bt, nullptr, nullptr, nullptr, reinterpret_cast<float*>(ws_states), BH, 1, 1, 1, 1,
                         s);
}

}  // namespace vda
