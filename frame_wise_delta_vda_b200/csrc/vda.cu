// vda.cu - C ABI of the bidirectional Video Delta Attention branch (see
// include/vda.h for the contract).  Validates arguments, plans the device
// workspace and enqueues the kernels on the caller's stream.
//
// Paper: "Video DeltaNet" (arXiv 2609.20744), Algorithm 1 steps 3-7:
//   stats (Eq. 3b) -> M_t = (I + A_t)^{-1} (Eq. 5, Appendix A.1) ->
//   forward + reverse scans (Section 2.2) -> boundary gather (Appendix A.3,
//   Eq. A.4) -> readout, RMSNorm, sigmoid gate (Eq. 1a, 1c).

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "vda.h"
#include "common.cuh"
#include "kernels_simt.cuh"
#include "kernels_tc.cuh"
#include "kernels_prep.cuh"

namespace {

using vda::ReadoutSimtCfg;

constexpr size_t kAlign = 256;
constexpr int kStages = 4;  // stats, inverse, scan, readout

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Plan {
  int B, H, T, U, d, chunk, window, NC, dtype;
  size_t BH, FH;
  bool tc;               // tensor-core (tcgen05) kernels
  size_t off_AM, off_B, off_states, off_bridge, off_maps, total;
};

int check_sizes(int B, int H, int T, int U, int d_k, int d_v, int chunk, int window, int dtype) {
  if (B < 1 || H < 1 || T < 1 || U < 1 || d_k < 1 || d_v < 1 || chunk < 1 || window < 0)
    return VDA_ERR_INVALID_ARGUMENT;
  if (dtype != VDA_BF16 && dtype != VDA_F32) return VDA_ERR_INVALID_ARGUMENT;
  if (d_k != d_v) return VDA_ERR_UNSUPPORTED;
  if (d_k != 16 && d_k != 32 && d_k != 64 && d_k != 128) return VDA_ERR_UNSUPPORTED;
  // element counts must stay well inside 63 bits and grid limits
  const double elems = (double)B * H * T * U * d_k;
  if (elems > 4.0e12) return VDA_ERR_UNSUPPORTED;
  if ((double)B * H * T > 2.0e9) return VDA_ERR_UNSUPPORTED;
  return VDA_OK;
}

Plan make_plan(int B, int H, int T, int U, int d, int chunk, int window, int dtype) {
  Plan p{};
  p.B = B; p.H = H; p.T = T; p.U = U; p.d = d; p.chunk = chunk; p.window = window;
  p.dtype = dtype;
  p.NC = (T + chunk - 1) / chunk;
  p.BH = (size_t)B * H;
  p.FH = p.BH * T;
  p.tc = vda::tc_path_supported(d, dtype);
  const size_t dd = (size_t)d * d * sizeof(float);
  size_t off = 0;
  p.off_AM = off;     off = align_up(off + p.FH * dd);
  p.off_B = off;      off = align_up(off + p.FH * dd);
  p.off_states = off; off = align_up(off + 2 * p.BH * (size_t)(p.NC + 1) * dd);
  p.off_bridge = off; off = align_up(off + 2 * p.FH * (size_t)d * sizeof(float));   // decay bridge products
  // chunk maps of the chunk-wise scans (tensor-core path): in A's region,
  // which the scans no longer need, when they fit there
  p.off_maps = p.off_AM;
  if (p.tc && d == 128) {
    const size_t maps = vda::tc::chunk_maps_bytes(p.BH, p.NC);
    if (maps > p.FH * dd) {
      p.off_maps = off;
      off = align_up(off + maps);
    }
  }
  p.total = off + vda::tc_extra_workspace_bytes(p.tc, p.FH, d);
  return p;
}

// ----------------------------------------------------------------------------
// per-stage timing (vda_timing_enable / vda_timing_read): events just before
// and just after each kernel launch, on the launch's stream
constexpr int kMaxMarks = 16;   // timed launches per forward
struct Timing {
  std::mutex mu;
  int max_calls = 0;
  int calls = 0;
  std::vector<cudaEvent_t> ev;     // 2 * kMaxMarks per call: begin, end of each launch
  std::vector<signed char> stage;  // kMaxMarks per call: the launch's stage, -1 when unused
  std::vector<char> done;          // 1 once every event of the call's slot was recorded
} g_timing;

int timing_begin_call() {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (g_timing.max_calls <= 0 || g_timing.calls >= g_timing.max_calls) return -1;
  return g_timing.calls++;
}

// The timer one forward call hands to its launch schedule.
struct CallTimer {
  int slot = -1;
  int n = 0;
  void begin(int st, cudaStream_t s) {
    if (slot < 0 || n >= kMaxMarks) return;
    g_timing.stage[(size_t)slot * kMaxMarks + n] = (signed char)st;
    cudaEventRecord(g_timing.ev[((size_t)slot * kMaxMarks + n) * 2], s);
  }
  void end(int, cudaStream_t s) {
    if (slot < 0 || n >= kMaxMarks) return;
    cudaEventRecord(g_timing.ev[((size_t)slot * kMaxMarks + n) * 2 + 1], s);
    ++n;
  }
};

// a forward that returns early leaves its slot incomplete: vda_timing_read skips it
void timing_end_call(int call_slot) {
  if (call_slot < 0) return;
  std::lock_guard<std::mutex> lk(g_timing.mu);
  g_timing.done[(size_t)call_slot] = 1;
}

void timing_reset_locked() {
  for (cudaEvent_t e : g_timing.ev)
    if (e) cudaEventDestroy(e);
  g_timing.ev.clear();
  g_timing.stage.clear();
  g_timing.done.clear();
  g_timing.calls = 0;
  g_timing.max_calls = 0;
}

// ----------------------------------------------------------------------------
template <int D, typename TIo>
int launch_simt(const Plan& p, const vda_args& a, char* ws, cudaStream_t s, CallTimer& tm,
                float* stats_out) {
  float* AM = reinterpret_cast<float*>(ws + p.off_AM);
  float* Bm = reinterpret_cast<float*>(ws + p.off_B);
  float* st = reinterpret_cast<float*>(ws + p.off_states);
  const size_t fdd = p.FH * (size_t)D * D;
  float* bridge = a.alpha ? reinterpret_cast<float*>(ws + p.off_bridge) : nullptr;

  tm.begin(0, s);
  vda::k_stats_simt<D, TIo><<<(unsigned)p.FH, 256, 0, s>>>(
      static_cast<const TIo*>(a.k), static_cast<const TIo*>(a.v), a.beta, p.U, AM, Bm);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  tm.end(0, s);
  if (stats_out) {
    if (cudaMemcpyAsync(stats_out, AM, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(stats_out + fdd, Bm, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return VDA_ERR_CUDA;
  }
  tm.begin(1, s);
  vda::k_gj_inverse<D><<<(unsigned)p.FH, 256, 0, s>>>(AM, nullptr);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  tm.end(1, s);
  if (stats_out) {
    if (cudaMemcpyAsync(stats_out + 2 * fdd, AM, fdd * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return VDA_ERR_CUDA;
  }
  tm.begin(2, s);
  constexpr int RB = 16;
  dim3 gs((unsigned)p.BH, 2, D / RB);
  vda::k_scan_simt<D, RB><<<gs, D, 0, s>>>(AM, Bm, a.S0_fwd, a.S0_rev, a.alpha, st, (int)p.BH, p.T,
                                           p.chunk, p.NC);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  tm.end(2, s);
  if (bridge) {
    const size_t n = p.FH * (size_t)D;
    vda::k_decay_bridge<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.alpha, (int)p.BH, p.T, D, p.chunk, p.window,
                                                                    bridge);
    if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  }

  using Cfg = ReadoutSimtCfg<D, TIo>;
  const size_t smem = Cfg::smem_bytes();
  if (cudaFuncSetAttribute(vda::k_readout_simt<D, TIo>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return VDA_ERR_CUDA;
  // tokens are taken per chunk, or per frame when the decay bridge makes the
  // read state differ from frame to frame
  const size_t pairs = p.BH * (size_t)(bridge ? p.T : p.NC);
  const long long tok_chunk = (long long)(bridge ? 1 : std::min(p.T, p.chunk)) * p.U;
  const long long per_cta = (long long)Cfg::WARPS * Cfg::TOK_PER_WARP * 4;
  int splits = (int)std::min<long long>((tok_chunk + per_cta - 1) / per_cta,
                                        std::max<long long>(1, 1184 / (long long)pairs));
  splits = std::max(1, std::min(splits, 65535));
  dim3 gr((unsigned)pairs, (unsigned)splits);
  const float eps = a.eps > 0.f ? a.eps : 1e-6f;
  tm.begin(3, s);
  vda::k_readout_simt<D, TIo><<<gr, 256, smem, s>>>(
      static_cast<const TIo*>(a.q), static_cast<const TIo*>(a.gate), a.rms_weight, st, bridge,
      static_cast<TIo*>(a.out), (int)p.BH, p.T, p.U, p.chunk, p.NC, p.window, eps);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  tm.end(3, s);
  return VDA_OK;
}

template <typename TIo>
int dispatch_simt(const Plan& p, const vda_args& a, char* ws, cudaStream_t s, CallTimer& tm, float* so) {
  switch (p.d) {
    case 16: return launch_simt<16, TIo>(p, a, ws, s, tm, so);
    case 32: return launch_simt<32, TIo>(p, a, ws, s, tm, so);
    case 64: return launch_simt<64, TIo>(p, a, ws, s, tm, so);
    case 128: return launch_simt<128, TIo>(p, a, ws, s, tm, so);
  }
  return VDA_ERR_UNSUPPORTED;
}

int validate_args(const vda_args* a) {
  if (!a) return VDA_ERR_INVALID_ARGUMENT;
  int rc = check_sizes(a->B, a->H, a->T, a->U, a->d_k, a->d_v, a->chunk, a->window_chunks, a->dtype);
  if (rc != VDA_OK) return rc;
  const void* req[] = {a->q, a->k, a->v, a->beta, a->gate, a->rms_weight, a->out};
  for (const void* ptr : req)
    if (!ptr || !aligned16(ptr)) return VDA_ERR_INVALID_ARGUMENT;
  if ((a->S0_fwd && !aligned16(a->S0_fwd)) || (a->S0_rev && !aligned16(a->S0_rev)) ||
      (a->alpha && !aligned16(a->alpha)))
    return VDA_ERR_INVALID_ARGUMENT;
  if (a->scan_form < VDA_SCAN_AUTO || a->scan_form > VDA_SCAN_CHUNKS) return VDA_ERR_INVALID_ARGUMENT;
  // the chunk-wise scans launch one CTA per (b, h, chunk, direction, part)
  if (a->scan_form == VDA_SCAN_CHUNKS &&
      4.0 * a->B * a->H * (double)((a->T + a->chunk - 1) / a->chunk) > 2147483647.0)
    return VDA_ERR_UNSUPPORTED;
  return VDA_OK;
}

int forward_impl(const vda_args& a, char* ws, const Plan& p, float* states_out, float* stats_out) {
  cudaStream_t s = static_cast<cudaStream_t>(a.stream);
  CallTimer tm;
  tm.slot = timing_begin_call();
  int rc;
  if (p.tc && p.d == 64) {
    rc = vda::launch_tc64(p.BH, p.T, p.U, p.chunk, p.NC, p.window, a, ws + p.off_AM, ws + p.off_B,
                          ws + p.off_states, ws + p.total - vda::tc_extra_workspace_bytes(true, p.FH, p.d),
                          ws + p.off_bridge, s, stats_out, tm);
  } else if (p.tc) {
    rc = vda::launch_tc(p.BH, p.T, p.U, p.chunk, p.NC, p.window, a, ws + p.off_AM, ws + p.off_B,
                        ws + p.off_states, ws + p.total - vda::tc_extra_workspace_bytes(true, p.FH, p.d),
                        ws + p.off_bridge, ws + p.off_maps, s, stats_out, tm);
  } else if (p.dtype == VDA_BF16) {
    rc = dispatch_simt<__nv_bfloat16>(p, a, ws, s, tm, stats_out);
  } else {
    rc = dispatch_simt<float>(p, a, ws, s, tm, stats_out);
  }
  if (rc != VDA_OK) return rc;
  timing_end_call(tm.slot);
  if (states_out) {
    const size_t bytes = 2 * p.BH * (size_t)(p.NC + 1) * p.d * p.d * sizeof(float);
    if (cudaMemcpyAsync(states_out, ws + p.off_states, bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return VDA_ERR_CUDA;
  }
  return VDA_OK;
}

int forward_alloc(const vda_args& a) {
  int rc = validate_args(&a);
  if (rc != VDA_OK) return rc;
  const Plan p = make_plan(a.B, a.H, a.T, a.U, a.d_k, a.chunk, a.window_chunks, a.dtype);
  cudaStream_t s = static_cast<cudaStream_t>(a.stream);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, p.total, s) != cudaSuccess) return VDA_ERR_CUDA;
  rc = forward_impl(a, static_cast<char*>(ws), p, nullptr, nullptr);
  if (cudaFreeAsync(ws, s) != cudaSuccess && rc == VDA_OK) rc = VDA_ERR_CUDA;
  return rc;
}

template <int D, typename TIo>
int text_state_simt(const Plan& p, const void* k, const void* v, const float* beta, char* ws,
                    cudaStream_t s) {
  float* AM = reinterpret_cast<float*>(ws + p.off_AM);
  float* Bm = reinterpret_cast<float*>(ws + p.off_B);
  float* st = reinterpret_cast<float*>(ws + p.off_states);
  vda::k_stats_simt<D, TIo><<<(unsigned)p.FH, 256, 0, s>>>(static_cast<const TIo*>(k),
                                                           static_cast<const TIo*>(v), beta, p.U, AM, Bm);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  vda::k_gj_inverse<D><<<(unsigned)p.FH, 256, 0, s>>>(AM, nullptr);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  dim3 gs((unsigned)p.BH, 1, D / 16);
  vda::k_scan_simt<D, 16><<<gs, D, 0, s>>>(AM, Bm, nullptr, nullptr, nullptr, st, (int)p.BH, 1, 1, p.NC);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  return VDA_OK;
}

template <typename TIo>
int text_state_dispatch(const Plan& p, const void* k, const void* v, const float* beta, char* ws,
                        cudaStream_t s) {
  switch (p.d) {
    case 16: return text_state_simt<16, TIo>(p, k, v, beta, ws, s);
    case 32: return text_state_simt<32, TIo>(p, k, v, beta, ws, s);
    case 64: return text_state_simt<64, TIo>(p, k, v, beta, ws, s);
    case 128: return text_state_simt<128, TIo>(p, k, v, beta, ws, s);
  }
  return VDA_ERR_UNSUPPORTED;
}

int text_state_impl(const Plan& p, const void* k, const void* v, const float* beta, char* ws,
                    cudaStream_t s) {
  if (p.tc && p.d == 128)
    return vda::tc_text_state(p.BH, p.U, k, v, beta, ws + p.off_AM, ws + p.off_B, ws + p.off_states,
                              ws + p.total - vda::tc_extra_workspace_bytes(true, p.FH, p.d), s);
  return p.dtype == VDA_BF16 ? text_state_dispatch<__nv_bfloat16>(p, k, v, beta, ws, s)
                             : text_state_dispatch<float>(p, k, v, beta, ws, s);
}

// ----------------------------------------------------------------------------
// host-buffer executor resources (one set per device)
struct HostPipe {
  bool init = false;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t in_done[2], comp_done[2], out_done[2];
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

struct HostLayout {
  int HG, groups;            // heads per group, number of groups
  size_t in_elem;            // bytes per element of q/k/v/gate/out
  size_t sz_qk, sz_v, sz_beta, sz_s0, sz_w, sz_alpha;
  size_t slot_off_q, slot_off_k, slot_off_v, slot_off_g, slot_off_beta, slot_off_s0f, slot_off_s0r,
      slot_off_alpha, slot_off_out, slot_off_ws, slot_bytes;
  size_t ws_bytes;
  size_t total;
};

HostLayout host_layout(int B, int H, int T, int U, int d, int chunk, int dtype) {
  HostLayout L{};
  const size_t BH = (size_t)B * H;
  const int target_groups = 8;
  L.HG = (int)std::max<size_t>(1, (BH + target_groups - 1) / target_groups);
  L.groups = (int)((BH + L.HG - 1) / L.HG);
  L.in_elem = dtype == VDA_BF16 ? 2 : 4;
  const size_t tok = (size_t)L.HG * T * U;
  L.sz_qk = tok * d * L.in_elem;
  L.sz_v = L.sz_qk;
  L.sz_beta = tok * sizeof(float);
  L.sz_s0 = (size_t)L.HG * d * d * sizeof(float);
  L.sz_w = (size_t)d * sizeof(float);
  L.sz_alpha = (size_t)L.HG * T * d * sizeof(float);
  const Plan p = make_plan(1, L.HG, T, U, d, chunk, 0, dtype);
  L.ws_bytes = p.total;
  size_t off = 0;
  L.slot_off_q = off;    off = align_up(off + L.sz_qk);
  L.slot_off_k = off;    off = align_up(off + L.sz_qk);
  L.slot_off_v = off;    off = align_up(off + L.sz_v);
  L.slot_off_g = off;    off = align_up(off + L.sz_v);
  L.slot_off_beta = off; off = align_up(off + L.sz_beta);
  L.slot_off_s0f = off;  off = align_up(off + L.sz_s0);
  L.slot_off_s0r = off;  off = align_up(off + L.sz_s0);
  L.slot_off_alpha = off; off = align_up(off + L.sz_alpha);
  L.slot_off_out = off;  off = align_up(off + L.sz_v);
  L.slot_off_ws = off;   off = align_up(off + L.ws_bytes);
  L.slot_bytes = off;
  L.total = align_up(L.sz_w) + 2 * L.slot_bytes;
  return L;
}

// ----------------------------------------------------------------------------
// Scratch of vda_forward_noalloc: one fixed array in this module, so that the
// entry point never allocates.  Its address is a device address only on the
// device side; host code must obtain the device pointer with
// cudaGetSymbolAddress (the symbol itself is a host-side stand-in).
static __device__ __align__(256) unsigned char g_noalloc_scratch[VDA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  Looked up on
// every call (the lookup allocates nothing): an address cached per device
// number would go stale after cudaDeviceReset, or belong to another context
// when a host runs the library under a non-primary context.
int noalloc_scratch(char** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return VDA_ERR_CUDA;
  *out = static_cast<char*>(ptr);
  return VDA_OK;
}

}  // namespace

// ============================================================================
namespace {
template <int D, int NXT>
int launch_prep_kv(const vda_prep_args& a, int nst, cudaStream_t s, float eps) {
  using namespace vda::prep;
  const size_t smem = kv_smem_bytes(a.Wl, D, nst);
  if (cudaFuncSetAttribute(k_prep_kv<D, NXT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return VDA_ERR_CUDA;
  k_prep_kv<D, NXT><<<dim3((unsigned)a.Hl, (unsigned)(a.B * a.H), 2), kThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(a.k_in), static_cast<const __nv_bfloat16*>(a.v_in), a.wk_s, a.wk_t, a.wv_s,
      a.wv_t, static_cast<__nv_bfloat16*>(a.k_out), static_cast<__nv_bfloat16*>(a.v_out), a.H, a.T, a.Hl, a.Wl, eps,
      nst);
  return cudaGetLastError() == cudaSuccess ? VDA_OK : VDA_ERR_CUDA;
}

template <int D>
int launch_prep(const vda_prep_args& a, int nst) {
  using namespace vda::prep;
  cudaStream_t s = static_cast<cudaStream_t>(a.stream);
  const float eps = a.eps > 0.f ? a.eps : 1e-6f;
  int rc = VDA_ERR_UNSUPPORTED;
  switch (kv_cols_per_thread(a.Wl, D)) {
    case 1: rc = launch_prep_kv<D, 1>(a, nst, s, eps); break;
    case 2: rc = launch_prep_kv<D, 2>(a, nst, s, eps); break;
    case 3: rc = launch_prep_kv<D, 3>(a, nst, s, eps); break;
    case 4: rc = launch_prep_kv<D, 4>(a, nst, s, eps); break;
    case 5: rc = launch_prep_kv<D, 5>(a, nst, s, eps); break;
    case 6: rc = launch_prep_kv<D, 6>(a, nst, s, eps); break;
    case 7: rc = launch_prep_kv<D, 7>(a, nst, s, eps); break;
    case 8: rc = launch_prep_kv<D, 8>(a, nst, s, eps); break;
  }
  if (rc != VDA_OK) return rc;
  const size_t warps = (size_t)a.B * a.T * a.Hl * a.Wl * a.H;
  const size_t blocks = (warps * 32 + 255) / 256;
  k_prep_q<D><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.q_in),
                                               static_cast<__nv_bfloat16*>(a.q_out), a.B, a.H, a.T,
                                               a.Hl * a.Wl, eps);
  if (cudaGetLastError() != cudaSuccess) return VDA_ERR_CUDA;
  return VDA_OK;
}
}  // namespace

extern "C" {

int vda_prep(const vda_prep_args* a) {
  if (!a) return VDA_ERR_INVALID_ARGUMENT;
  if (a->B < 1 || a->H < 1 || a->T < 1 || a->Hl < 1 || a->Wl < 1 || a->d < 1) return VDA_ERR_INVALID_ARGUMENT;
  const void* req[] = {a->q_in, a->k_in, a->v_in, a->wk_s, a->wk_t, a->wv_s, a->wv_t, a->q_out, a->k_out, a->v_out};
  for (const void* ptr : req)
    if (!ptr || !aligned16(ptr)) return VDA_ERR_INVALID_ARGUMENT;
  const int d = a->d;
  if (d != 16 && d != 32 && d != 64 && d != 128) return VDA_ERR_UNSUPPORTED;
  if (vda::prep::kv_cols_per_thread(a->Wl, d) > vda::prep::kMaxNxt) return VDA_ERR_UNSUPPORTED;
  int dev = 0, max_smem = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return VDA_ERR_CUDA;
  // two staging buffers (the next frame's rows load during this frame's
  // filters) when they fit, else one
  const int nst = vda::prep::kv_smem_bytes(a->Wl, d, 2) <= (size_t)max_smem ? 2 : 1;
  if (vda::prep::kv_smem_bytes(a->Wl, d, nst) > (size_t)max_smem) return VDA_ERR_UNSUPPORTED;
  if ((double)a->B * a->H * a->T * a->Hl * a->Wl * d > 4.0e12 || (double)a->B * a->H > 65535.0 || a->Hl > 2147483647)
    return VDA_ERR_UNSUPPORTED;
  switch (d) {
    case 16: return launch_prep<16>(*a, nst);
    case 32: return launch_prep<32>(*a, nst);
    case 64: return launch_prep<64>(*a, nst);
    default: return launch_prep<128>(*a, nst);
  }
}

const char* vda_status_string(int status) {
  switch (status) {
    case VDA_OK: return "VDA_OK";
    case VDA_ERR_INVALID_ARGUMENT: return "VDA_ERR_INVALID_ARGUMENT";
    case VDA_ERR_UNSUPPORTED: return "VDA_ERR_UNSUPPORTED";
    case VDA_ERR_WORKSPACE: return "VDA_ERR_WORKSPACE";
    case VDA_ERR_CUDA: return "VDA_ERR_CUDA";
    case VDA_ERR_TIMEOUT: return "VDA_ERR_TIMEOUT";
  }
  return "VDA_ERR_UNKNOWN";
}

size_t vda_workspace_bytes(int B, int H, int T, int U, int d_k, int d_v, int chunk, int dtype) {
  if (check_sizes(B, H, T, U, d_k, d_v, chunk, 0, dtype) != VDA_OK) return 0;
  return make_plan(B, H, T, U, d_k, chunk, 0, dtype).total;
}

int vda_launches_per_forward(int B, int H, int T, int U, int d_k, int d_v, int chunk, int dtype) {
  if (check_sizes(B, H, T, U, d_k, d_v, chunk, 0, dtype) != VDA_OK) return 0;
  const Plan p = make_plan(B, H, T, U, d_k, chunk, 0, dtype);
  return p.tc ? vda::tc_launches_per_forward(p.d, VDA_SCAN_AUTO, p.BH, p.T, p.chunk, p.NC) : 4;
}

int vda_forward_ex(const vda_args* args, void* workspace, size_t workspace_bytes,
                   float* states_out, float* stats_out) {
  int rc = validate_args(args);
  if (rc != VDA_OK) return rc;
  if ((states_out && !aligned16(states_out)) || (stats_out && !aligned16(stats_out)))
    return VDA_ERR_INVALID_ARGUMENT;
  const Plan p = make_plan(args->B, args->H, args->T, args->U, args->d_k, args->chunk,
                           args->window_chunks, args->dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < p.total)
    return VDA_ERR_WORKSPACE;
  return forward_impl(*args, static_cast<char*>(workspace), p, states_out, stats_out);
}

int vda_forward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* beta,
                const uint16_t* gate, const float* rms_weight, const float* S0_fwd,
                const float* S0_rev, int B, int H, int T, int U, int d_k, int d_v, int chunk,
                int window_chunks, uint16_t* out, void* stream) {
  vda_args a{};
  a.dtype = VDA_BF16;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.gate = gate; a.rms_weight = rms_weight;
  a.S0_fwd = S0_fwd; a.S0_rev = S0_rev; a.out = out;
  a.B = B; a.H = H; a.T = T; a.U = U; a.d_k = d_k; a.d_v = d_v;
  a.chunk = chunk; a.window_chunks = window_chunks; a.eps = 1e-6f; a.stream = stream;
  return forward_alloc(a);
}

int vda_forward_f32(const float* q, const float* k, const float* v, const float* beta,
                    const float* gate, const float* rms_weight, const float* S0_fwd,
                    const float* S0_rev, int B, int H, int T, int U, int d_k, int d_v, int chunk,
                    int window_chunks, float* out, void* stream) {
  vda_args a{};
  a.dtype = VDA_F32;
  a.q = q; a.k = k; a.v = v; a.beta = beta; a.gate = gate; a.rms_weight = rms_weight;
  a.S0_fwd = S0_fwd; a.S0_rev = S0_rev; a.out = out;
  a.B = B; a.H = H; a.T = T; a.U = U; a.d_k = d_k; a.d_v = d_v;
  a.chunk = chunk; a.window_chunks = window_chunks; a.eps = 1e-6f; a.stream = stream;
  return forward_alloc(a);
}

size_t vda_text_state_workspace_bytes(int B, int H, int L, int d_k, int d_v, int dtype) {
  if (check_sizes(B, H, 1, L, d_k, d_v, 1, 0, dtype) != VDA_OK) return 0;
  return make_plan(B, H, 1, L, d_k, 1, 0, dtype).total;
}

int vda_text_state(int dtype, const void* k_text, const void* v_text, const float* beta_text,
                   int B, int H, int L, int d_k, int d_v, float* S_out, void* workspace,
                   size_t workspace_bytes, void* stream) {
  int rc = check_sizes(B, H, 1, L, d_k, d_v, 1, 0, dtype);
  if (rc != VDA_OK) return rc;
  if (!k_text || !v_text || !beta_text || !S_out || !aligned16(k_text) || !aligned16(v_text) ||
      !aligned16(beta_text) || !aligned16(S_out))
    return VDA_ERR_INVALID_ARGUMENT;
  const Plan p = make_plan(B, H, 1, L, d_k, 1, 0, dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < p.total)
    return VDA_ERR_WORKSPACE;
  // One frame of L tokens per (b, h): stats -> inverse -> one scan step from
  // the zero state.  The readout is not needed, so only those three run.
  rc = text_state_impl(p, k_text, v_text, beta_text, static_cast<char*>(workspace),
                       static_cast<cudaStream_t>(stream));
  if (rc != VDA_OK) return rc;
  // forward state after the single frame sits at states[0][bh][1]
  const size_t dd = (size_t)d_k * d_k * sizeof(float);
  if (cudaMemcpy2DAsync(S_out, dd, static_cast<char*>(workspace) + p.off_states + dd, 2 * dd, dd,
                        p.BH, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return VDA_ERR_CUDA;
  return VDA_OK;
}

size_t vda_forward_host_bytes(int B, int H, int T, int U, int d_k, int d_v, int chunk, int dtype) {
  if (check_sizes(B, H, T, U, d_k, d_v, chunk, 0, dtype) != VDA_OK) return 0;
  return host_layout(B, H, T, U, d_k, chunk, dtype).total;
}

int vda_forward_host(const vda_args* ha, void* device_buffer, size_t device_bytes) {
  if (!ha) return VDA_ERR_INVALID_ARGUMENT;
  int rc = check_sizes(ha->B, ha->H, ha->T, ha->U, ha->d_k, ha->d_v, ha->chunk, ha->window_chunks,
                       ha->dtype);
  if (rc != VDA_OK) return rc;
  const void* req[] = {ha->q, ha->k, ha->v, ha->beta, ha->gate, ha->rms_weight, ha->out};
  for (const void* ptr : req)
    if (!ptr) return VDA_ERR_INVALID_ARGUMENT;
  const HostLayout L = host_layout(ha->B, ha->H, ha->T, ha->U, ha->d_k, ha->chunk, ha->dtype);
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) % kAlign) != 0 ||
      device_bytes < L.total)
    return VDA_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return VDA_ERR_CUDA;
  HostPipe* P;
  {
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    P = &g_pipe[dev];
    if (!P->init) {
      bool ok = cudaStreamCreateWithFlags(&P->h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&P->comp, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&P->d2h, cudaStreamNonBlocking) == cudaSuccess;
      for (int i = 0; ok && i < 2; ++i)
        ok = cudaEventCreateWithFlags(&P->in_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&P->comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&P->out_done[i], cudaEventDisableTiming) == cudaSuccess;
      if (!ok) return VDA_ERR_CUDA;
      P->init = true;
    }
  }
  char* base = static_cast<char*>(device_buffer);
  float* d_w = reinterpret_cast<float*>(base);
  char* slots = base + align_up(L.sz_w);
  const size_t BH = (size_t)ha->B * ha->H;
  const size_t per_head_tok = (size_t)ha->T * ha->U;
  const int d = ha->d_k;
  // the scan form the whole problem would take, so that every head group
  // computes what vda_forward_ex computes for all heads at once
  int scan_form = ha->scan_form;
  if (scan_form == VDA_SCAN_AUTO)
    scan_form = vda::use_chunk_scan(VDA_SCAN_AUTO, BH, ha->T, ha->chunk, (ha->T + ha->chunk - 1) / ha->chunk,
                                    vda::tc::num_sms())
                    ? VDA_SCAN_CHUNKS
                    : VDA_SCAN_FRAMES;
#define VDA_CK(x) do { if ((x) != cudaSuccess) return VDA_ERR_CUDA; } while (0)
  // the copy / compute pipeline; on an error it returns at once, with copies
  // possibly still queued on the three streams
  auto run_groups = [&]() -> int {
  VDA_CK(cudaMemcpyAsync(d_w, ha->rms_weight, L.sz_w, cudaMemcpyHostToDevice, P->h2d));
  for (int g = 0; g < L.groups; ++g) {
    const int sl = g & 1;
    char* S = slots + (size_t)sl * L.slot_bytes;
    const size_t h0 = (size_t)g * L.HG;
    const int nh = (int)std::min<size_t>(L.HG, BH - h0);
    const size_t tokb = (size_t)nh * per_head_tok;
    const size_t eb = tokb * d * L.in_elem;
    const size_t off_e = h0 * per_head_tok * d * L.in_elem;
    // the slot's inputs are free once group g-2 finished computing
    if (g >= 2) VDA_CK(cudaStreamWaitEvent(P->h2d, P->comp_done[sl], 0));
    VDA_CK(cudaMemcpyAsync(S + L.slot_off_q, static_cast<const char*>(ha->q) + off_e, eb, cudaMemcpyHostToDevice, P->h2d));
    VDA_CK(cudaMemcpyAsync(S + L.slot_off_k, static_cast<const char*>(ha->k) + off_e, eb, cudaMemcpyHostToDevice, P->h2d));
    VDA_CK(cudaMemcpyAsync(S + L.slot_off_v, static_cast<const char*>(ha->v) + off_e, eb, cudaMemcpyHostToDevice, P->h2d));
    VDA_CK(cudaMemcpyAsync(S + L.slot_off_g, static_cast<const char*>(ha->gate) + off_e, eb, cudaMemcpyHostToDevice, P->h2d));
    VDA_CK(cudaMemcpyAsync(S + L.slot_off_beta, ha->beta + h0 * per_head_tok, tokb * sizeof(float),
                           cudaMemcpyHostToDevice, P->h2d));
    const size_t s0b = (size_t)nh * d * d * sizeof(float);
    if (ha->S0_fwd)
      VDA_CK(cudaMemcpyAsync(S + L.slot_off_s0f, ha->S0_fwd + h0 * d * d, s0b, cudaMemcpyHostToDevice, P->h2d));
    if (ha->S0_rev)
      VDA_CK(cudaMemcpyAsync(S + L.slot_off_s0r, ha->S0_rev + h0 * d * d, s0b, cudaMemcpyHostToDevice, P->h2d));
    if (ha->alpha)
      VDA_CK(cudaMemcpyAsync(S + L.slot_off_alpha, ha->alpha + h0 * (size_t)ha->T * d,
                             (size_t)nh * ha->T * d * sizeof(float), cudaMemcpyHostToDevice, P->h2d));
    VDA_CK(cudaEventRecord(P->in_done[sl], P->h2d));

    VDA_CK(cudaStreamWaitEvent(P->comp, P->in_done[sl], 0));
    if (g >= 2) VDA_CK(cudaStreamWaitEvent(P->comp, P->out_done[sl], 0));
    vda_args a = *ha;
    a.B = 1; a.H = nh;
    a.scan_form = scan_form;
    a.q = S + L.slot_off_q; a.k = S + L.slot_off_k; a.v = S + L.slot_off_v; a.gate = S + L.slot_off_g;
    a.beta = reinterpret_cast<const float*>(S + L.slot_off_beta);
    a.rms_weight = d_w;
    a.S0_fwd = ha->S0_fwd ? reinterpret_cast<const float*>(S + L.slot_off_s0f) : nullptr;
    a.S0_rev = ha->S0_rev ? reinterpret_cast<const float*>(S + L.slot_off_s0r) : nullptr;
    a.alpha = ha->alpha ? reinterpret_cast<const float*>(S + L.slot_off_alpha) : nullptr;
    a.out = S + L.slot_off_out;
    a.stream = P->comp;
    const Plan p = make_plan(1, nh, a.T, a.U, d, a.chunk, a.window_chunks, a.dtype);
    const int frc = forward_impl(a, S + L.slot_off_ws, p, nullptr, nullptr);
    if (frc != VDA_OK) return frc;
    VDA_CK(cudaEventRecord(P->comp_done[sl], P->comp));

    VDA_CK(cudaStreamWaitEvent(P->d2h, P->comp_done[sl], 0));
    VDA_CK(cudaMemcpyAsync(static_cast<char*>(ha->out) + off_e, S + L.slot_off_out, eb,
                           cudaMemcpyDeviceToHost, P->d2h));
    VDA_CK(cudaEventRecord(P->out_done[sl], P->d2h));
  }
  VDA_CK(cudaStreamSynchronize(P->d2h));
  VDA_CK(cudaStreamSynchronize(P->comp));
  return VDA_OK;
  };
#undef VDA_CK
  rc = run_groups();
  if (rc != VDA_OK) {
    // the call is synchronous: no queued copy may read or write the caller's
    // host buffers after it returns, so drain every stream (their status is
    // not needed: the first error is the one reported)
    cudaStreamSynchronize(P->h2d);
    cudaStreamSynchronize(P->comp);
    cudaStreamSynchronize(P->d2h);
  }
  return rc;
}

int vda_forward_noalloc(const vda_args* args) {
  int rc = validate_args(args);
  if (rc != VDA_OK) return rc;
  const Plan p = make_plan(args->B, args->H, args->T, args->U, args->d_k, args->chunk,
                           args->window_chunks, args->dtype);
  if (p.total > VDA_NOALLOC_SCRATCH_BYTES) return VDA_ERR_WORKSPACE;
  char* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != VDA_OK) return rc;
  return forward_impl(*args, scratch, p, nullptr, nullptr);
}

int vda_selftest_wait_timeout(int max_polls, void* stream) {
  if (max_polls < 1 || max_polls > 1000000) return VDA_ERR_INVALID_ARGUMENT;
  vda::k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((long long)max_polls);
  return cudaGetLastError() == cudaSuccess ? VDA_OK : VDA_ERR_CUDA;
}

int vda_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return VDA_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, vda::g_device_error, sizeof(word)) != cudaSuccess) return VDA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemcpyToSymbol(vda::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return VDA_ERR_CUDA;
    return VDA_ERR_TIMEOUT;
  }
  return VDA_OK;
}

int vda_timing_enable(int max_calls) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  timing_reset_locked();
  if (max_calls <= 0) return VDA_OK;
  g_timing.ev.assign((size_t)max_calls * kMaxMarks * 2, nullptr);
  g_timing.stage.assign((size_t)max_calls * kMaxMarks, (signed char)-1);
  g_timing.done.assign((size_t)max_calls, 0);
  for (auto& e : g_timing.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      timing_reset_locked();
      return VDA_ERR_CUDA;
    }
  g_timing.max_calls = max_calls;
  return VDA_OK;
}

int vda_timing_read(float* stage_ms, int n_stages, int* calls) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (!stage_ms || n_stages < 1) return VDA_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < n_stages; ++i) stage_ms[i] = 0.f;
  int rc = VDA_OK, complete = 0;
  for (int c = 0; c < g_timing.calls && rc == VDA_OK; ++c) {
    if (!g_timing.done[(size_t)c]) continue;   // a forward that failed part-way
    for (int n = 0; n < kMaxMarks && rc == VDA_OK; ++n) {
      const int st = g_timing.stage[(size_t)c * kMaxMarks + n];
      if (st < 0) break;
      cudaEvent_t* e = &g_timing.ev[((size_t)c * kMaxMarks + n) * 2];
      float ms = 0.f;
      if (cudaEventSynchronize(e[1]) != cudaSuccess || cudaEventElapsedTime(&ms, e[0], e[1]) != cudaSuccess) {
        rc = VDA_ERR_CUDA;
        break;
      }
      if (st < n_stages) stage_ms[st] += ms;
    }
    ++complete;
  }
  if (calls) *calls = complete;
  // events are released and timing is switched off whatever happened above
  timing_reset_locked();
  return rc;
}

}  // extern "C"
