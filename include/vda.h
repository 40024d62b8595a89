/*
 * vda.h - C ABI of the B200 (sm_100a) bidirectional Video Delta Attention branch.
 *
 * Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
 * Generation" (arXiv 2609.20744).  The library computes the linear branch of
 * one hybrid attention block (Algorithm 1, steps 3-7; shown here with the
 * decay gate fixed to 1, see "Decay" below for the general form):
 *
 *   for every batch b, head h and interior latent frame t:
 *     A_t = K_t^T Diag(beta_t) K_t,  B_t = V_t^T Diag(beta_t) K_t     (Eq. 3b)
 *     forward scan  P_t = (P_{t-1} + B_t)(I + A_t)^{-1}, P_{-1} = S0_fwd (Eq. 5)
 *     reverse scan  R_t = (R_{t+1} + B_t)(I + A_t)^{-1}, R_T  = S0_rev
 *     query chunk c reads  S~_c = P_{l-1} + R_{h+1}  just outside its local
 *     window [l, h] (Appendix A.3, Eq. A.4; a side without distant frames reads
 *     its initial state), o = S~_c q                                   (Eq. 1a)
 *     out = sigmoid(gate) * w * o / sqrt(mean_{d_v}(o^2) + eps)        (Eq. 1c)
 *
 * Conventions shared by every entry point
 *   - Layouts are contiguous and row-major:
 *       q, k      [B, H, T, U, d_k]      v, gate, out  [B, H, T, U, d_v]
 *       beta      [B, H, T, U]  float32 (write gates, >= 0)
 *       rms_weight[d_v]         float32, shared by all heads
 *       S0_fwd, S0_rev [B, H, d_v, d_k] float32; the state maps keys to
 *                 values, o = S q.  NULL means the zero state.
 *     T counts interior frames only: the caller has already removed the two
 *     boundary anchor frames (Algorithm 1, step 2).
 *   - Chunks tile the interior frame index from 0: chunk c holds frames
 *     [c*chunk, (c+1)*chunk); the last chunk may be shorter.  The local window
 *     of chunk c is chunks c-window_chunks .. c+window_chunks clipped to the
 *     clip; a window covering the whole clip yields
 *     RMSNorm((S0_fwd + S0_rev) q) * sigmoid(gate), which is 0 for zero S0.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - All pointers except those documented as host pointers are device
 *     pointers owned by the caller; the library never frees them and keeps no
 *     reference after the call returns.  Device pointers must be 16-byte
 *     aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and the call returns without synchronising,
 *     except where stated.
 *   - Decay (Eq. 2 and Appendix A.3, Eq. A.4): with vda_args.alpha set, both
 *     scans decay the entering state channel-wise before each frame update,
 *       P_t = (P_{t-1} Diag(alpha_t) + B_t)(I + A_t)^{-1}   (and R_t alike,
 *       with the frame's own alpha_t),
 *     and query frame t reads the bridged states
 *       S~_t = P_{l-1} Diag(prod_{r=l..t} alpha_r) + R_{h+1} Diag(prod_{r=t..h} alpha_r)
 *     (a side without distant frames bridges its initial state).  alpha is
 *     [B, H, T, d_k] float32 with values in [0, 1].  vda_forward and
 *     vda_forward_f32 have no decay (alpha = 1); vda_forward_ex,
 *     vda_forward_host and vda_forward_noalloc take it from vda_args.
 *   - Supported sizes: d_k == d_v in {16, 32, 64, 128}; chunk >= 1;
 *     window_chunks >= 0; B, H, T, U >= 1.  d = 128 and d = 64 with bf16 I/O
 *     run on the tcgen05 tensor-core kernels (at d = 64 with the FP32
 *     Gauss-Jordan inverse); the other sizes run on SIMT kernels.
 *   - Errors: every argument is validated before any launch; no exception
 *     crosses the ABI.  See vda_status.
 */
#ifndef VDA_H
#define VDA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VDA_API __attribute__((visibility("default")))
#else
#define VDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vda_status {
  VDA_OK = 0,
  VDA_ERR_INVALID_ARGUMENT = 1, /* NULL required pointer, size <= 0, misaligned pointer */
  VDA_ERR_UNSUPPORTED = 2,      /* valid but unsupported sizes (d_k != d_v, d not in the list) */
  VDA_ERR_WORKSPACE = 3,        /* caller workspace smaller than vda_workspace_bytes() */
  VDA_ERR_CUDA = 4,             /* a CUDA runtime call or kernel launch failed */
  VDA_ERR_TIMEOUT = 5           /* a kernel gave up waiting on a barrier (see vda_device_status) */
} vda_status;

typedef enum vda_dtype {
  VDA_BF16 = 0, /* q, k, v, gate, out (and text tokens) are bfloat16 */
  VDA_F32 = 1   /* ... are float32 */
} vda_dtype;

/* How the forward and reverse scans of Section 2.2 run on the tensor-core
 * path at d = 128 (bf16); the other paths always scan frame by frame.  Both give
 * the same boundary states up to rounding.
 *   VDA_SCAN_FRAMES: one sequential chain of T frame updates per (b, h,
 *     direction), S <- (S Diag(alpha_t) + B_t) M_t.
 *   VDA_SCAN_CHUNKS: the chunk-wise scan of Section 5 ("Chunk-wise scans",
 *     Appendix A.1): every chunk's frames are first composed, in parallel,
 *     into one affine map S -> S P_c + J_c, then each chain runs its NC maps.
 *     About twice the tensor-core work on a chain of chunk + NC steps; it pays
 *     when few (b, h) pairs share the GPU.
 *   VDA_SCAN_AUTO: the library picks by the number of (b, h) pairs.
 * VDA_SCAN_CHUNKS with more than 2^31 - 1 composition CTAs (4 B H NC) returns
 * VDA_ERR_UNSUPPORTED. */
typedef enum vda_scan_form {
  VDA_SCAN_AUTO = 0,
  VDA_SCAN_FRAMES = 1,
  VDA_SCAN_CHUNKS = 2
} vda_scan_form;

/* Full argument block of vda_forward_ex. */
typedef struct vda_args {
  int dtype;                  /* vda_dtype of q, k, v, gate, out */
  const void* q;              /* [B,H,T,U,d_k] */
  const void* k;              /* [B,H,T,U,d_k] */
  const void* v;              /* [B,H,T,U,d_v] */
  const float* beta;          /* [B,H,T,U] */
  const void* gate;           /* [B,H,T,U,d_v] sigmoid-gate logits */
  const float* rms_weight;    /* [d_v] */
  const float* S0_fwd;        /* [B,H,d_v,d_k] or NULL */
  const float* S0_rev;        /* [B,H,d_v,d_k] or NULL */
  void* out;                  /* [B,H,T,U,d_v] */
  int B, H, T, U, d_k, d_v;
  int chunk;                  /* frames per chunk (the paper: 5) */
  int window_chunks;          /* window radius in chunks (the paper: 1) */
  float eps;                  /* RMSNorm epsilon; <= 0 selects 1e-6 */
  void* stream;               /* cudaStream_t */
  const float* alpha;         /* [B,H,T,d_k] decay gates in [0,1] (Eq. 2), or NULL: no decay */
  int scan_form;              /* vda_scan_form; 0 (zero-initialised args) = VDA_SCAN_AUTO */
} vda_args;

/* Bidirectional VDA forward, bf16 I/O.  Takes its workspace stream-ordered
 * (cudaMallocAsync / cudaFreeAsync on `stream`).  Returns vda_status. */
VDA_API int vda_forward(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const float* beta, const uint16_t* gate, const float* rms_weight,
                const float* S0_fwd, const float* S0_rev,
                int B, int H, int T, int U, int d_k, int d_v,
                int chunk, int window_chunks, uint16_t* out, void* stream);

/* Same as vda_forward with float32 q, k, v, gate and out. */
VDA_API int vda_forward_f32(const float* q, const float* k, const float* v,
                    const float* beta, const float* gate, const float* rms_weight,
                    const float* S0_fwd, const float* S0_rev,
                    int B, int H, int T, int U, int d_k, int d_v,
                    int chunk, int window_chunks, float* out, void* stream);

/* Bytes of device workspace vda_forward_ex needs for these sizes (0 when the
 * sizes are invalid).  The workspace holds the per-frame statistics and
 * transitions and the chunk-boundary states, all float32. */
VDA_API size_t vda_workspace_bytes(int B, int H, int T, int U, int d_k, int d_v,
                           int chunk, int dtype);

/* Forward with a caller-supplied device workspace (>= vda_workspace_bytes,
 * 256-byte aligned) and optional debug outputs:
 *   states_out [2, B, H, NC+1, d_v, d_k] float32, NC = ceil(T / chunk):
 *     states_out[0,b,h,j] = state after absorbing frames [0, j*chunk) forward
 *                           from S0_fwd (j = 0 is S0_fwd, j = NC the final P);
 *     states_out[1,b,h,j] = state after absorbing frames [j*chunk, T) in
 *                           reverse from S0_rev (j = NC is S0_rev).
 *   stats_out  [3, B, H, T, d, d] float32: A_t, B_t and M_t = (I + A_t)^{-1}.
 * Either may be NULL.  Resuming: passing states_out[0,b,h,NC] of one call as
 * S0_fwd of a call on the following frames continues the forward scan. */
VDA_API int vda_forward_ex(const vda_args* args, void* workspace, size_t workspace_bytes,
                   float* states_out, float* stats_out);

/* Text state of Eq. (1b) for one prompt per (b, h): one frame-wise update of
 * the zero state with the L prompt tokens treated as one frame,
 *   S_out = B'(I + A')^{-1},  A' = K'^T Diag(beta') K',  B' = V'^T Diag(beta') K'.
 * k_text [B,H,L,d_k], v_text [B,H,L,d_v] (dtype), beta_text [B,H,L] float32
 * (pass the halved gates to obtain S_T/2 for both scans), S_out [B,H,d_v,d_k]
 * float32.  Workspace: vda_text_state_workspace_bytes(), device, 256-byte
 * aligned. */
VDA_API size_t vda_text_state_workspace_bytes(int B, int H, int L, int d_k, int d_v, int dtype);
VDA_API int vda_text_state(int dtype, const void* k_text, const void* v_text, const float* beta_text,
                   int B, int H, int L, int d_k, int d_v, float* S_out,
                   void* workspace, size_t workspace_bytes, void* stream);

/* End-to-end forward from HOST buffers: every array of `args` (q, k, v, beta,
 * gate, rms_weight, S0_fwd, S0_rev, out) is a host pointer (page-locked for
 * overlap); the call copies the inputs to the device, runs the forward and
 * copies `out` back, pipelining groups of heads over two streams (copy and
 * compute) so that transfers overlap the kernels.  Every group takes the
 * scan form the whole problem takes, so `out` equals vda_forward_ex's bit for
 * bit.  `device_buffer` is caller device memory of at least
 * vda_forward_host_bytes() bytes (256-byte aligned).  Synchronous: returns
 * when `out` is complete on the host. */
VDA_API size_t vda_forward_host_bytes(int B, int H, int T, int U, int d_k, int d_v,
                              int chunk, int dtype);
VDA_API int vda_forward_host(const vda_args* host_args, void* device_buffer, size_t device_bytes);

/* Forward without any allocation, for callers that cannot allocate device
 * memory: host frameworks that own all device memory through their own
 * allocator and have no way to hand this library a workspace, plugins loaded
 * into such hosts, and fixed-footprint serving or real-time loops whose
 * policy forbids allocator calls once they are running (a cudaMalloc there
 * can block, fail under memory pressure, or synchronise the device).  Same
 * arguments and result as vda_forward_ex with no workspace and no debug
 * outputs; the scratch (statistics, transitions and chunk-boundary states)
 * lives in one fixed array of VDA_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.
 *   - Returns VDA_ERR_WORKSPACE when the sizes need more scratch than that
 *     (vda_workspace_bytes() > VDA_NOALLOC_SCRATCH_BYTES); nothing is launched.
 *   - Every call looks up the array's device address in the current context
 *     with the CUDA runtime (cudaGetSymbolAddress; no allocation), so the
 *     address is never stale after cudaDeviceReset or under another context.
 *     The first lookup in a context may load the library's device code; make
 *     the first call on each device before any stream capture begins.
 *   - Calls share the one array: two calls whose work overlaps on the GPU
 *     (different streams, or different host threads, without ordering between
 *     them) race and corrupt each other's results.  Every scratch word is
 *     written before it is read in each call, so nothing left by an earlier
 *     call leaks into a later one.
 * The paper has no counterpart to this entry point; it is a deployment aid. */
#define VDA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
VDA_API int vda_forward_noalloc(const vda_args* args);

/* Synchronises `stream`, then reads and clears the library's device error
 * word for the current device: returns VDA_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last call, VDA_ERR_CUDA on a CUDA error, else VDA_OK. */
VDA_API int vda_device_status(void* stream);

/* Failure-detection self test: launches one kernel that waits, with a bounded
 * poll, on a device flag that nothing sets.  After max_polls polls (1 ..
 * 1000000, about 0.1 us each) it gives up, records a wait time-out in the
 * device error word and returns normally, so the context stays usable; the
 * next vda_device_status(stream) returns VDA_ERR_TIMEOUT and clears it.
 * No compute path calls this; it exists to test failure detection without
 * a GPU fault.  Returns vda_status. */
VDA_API int vda_selftest_wait_timeout(int max_polls, void* stream);

/* Per-stage device timing for profiling.  vda_timing_enable(n) makes the next
 * n forward calls record a CUDA event just before and just after each kernel
 * launch, on the launch's stream; vda_timing_read(ms, 4, &calls) synchronises
 * on the recorded events and writes, per stage (stats, inverse, scan,
 * readout), the milliseconds summed over that stage's launches and calls, and
 * the number of calls recorded, then disables timing and releases the events.
 * vda_timing_enable(0) disables it. */
VDA_API int vda_timing_enable(int max_calls);
VDA_API int vda_timing_read(float* stage_ms, int n_stages, int* calls);

/* Number of kernel launches one vda_forward_ex call with these sizes makes
 * without a decay gate and with scan_form VDA_SCAN_AUTO on the current device
 * (the chunk-wise scans take two launches); with vda_args.alpha set the call
 * makes one more (the bridge products of Eq. A.4). */
VDA_API int vda_launches_per_forward(int B, int H, int T, int U, int d_k, int d_v, int chunk, int dtype);

/* ---------------------------------------------------------------------------
 * Feature preparation of the linear branch (Section 2.3; the fused "VDA-Prep"
 * step of Section 5), the step ahead of vda_forward:
 *   q' = L2(q),  k' = L2(SiLU(conv(k))),  v' = SiLU(conv(v))
 * conv = a depthwise 5 x 5 spatial filter over the Hl x Wl latent grid then a
 * depthwise five-tap temporal filter over the interior frames, both
 * cross-correlations with zero padding 2 on every side; L2(x) =
 * x / sqrt(sum(x^2) + eps) over the head dimension.
 *   q_in, k_in, v_in  [B, T, U, H, d] bf16 (the projections of the interior
 *                     video tokens, heads inner; token u = y * Wl + x)
 *   wk_s, wv_s        [H, d, 5, 5] float32, wk_t, wv_t [H, d, 5] float32
 *   q_out, k_out, v_out [B, H, T, U, d] bf16 (the layout vda_forward reads)
 * Supported: bf16, d in {16, 32, 64, 128}, at most 8 grid columns per
 * thread slice (Wl <= 8 * 1024 / d) and the staged rows, the spatial taps and
 * one fp32 output row (about 5 (Wl + 4) * 2 d + 100 d + 4 d Wl bytes) within
 * the device's shared memory (Wl <= 64 at d = 128).  Inputs and outputs must
 * not overlap.
 * Returns vda_status. */
typedef struct vda_prep_args {
  const void* q_in;
  const void* k_in;
  const void* v_in;
  const float* wk_s;
  const float* wk_t;
  const float* wv_s;
  const float* wv_t;
  void* q_out;
  void* k_out;
  void* v_out;
  int B, H, T, Hl, Wl, d;
  float eps;                  /* L2 epsilon; <= 0 selects 1e-6 */
  void* stream;               /* cudaStream_t */
} vda_prep_args;

VDA_API int vda_prep(const vda_prep_args* args);

/* Human-readable name of a vda_status value. */
VDA_API const char* vda_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* VDA_H */
