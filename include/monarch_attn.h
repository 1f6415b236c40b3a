/*
 * monarch_attn.h -- C ABI of the B200 (sm_100a) Monarch video-attention forward
 * (and the backward of its one-step form).
 *
 * Operation (MonarchRT: Efficient Attention for Real-Time Video Generation;
 * gist.science explainer §2 "Methodology", §2.A "Block Alignment", §2.B "Tiled
 * Monarch Parameterization", §2.C "Finetuning and Efficient Implementation"):
 * per (batch, head) the attention matrix over a T x H x W token grid is
 * constrained to Monarch form M = P blockdiag(L) P^T blockdiag(R), with
 *   tile     c1 = (t*(H/tile_h) + y/tile_h)*(W/tile_w) + x/tile_w
 *   position c2 = (y % tile_h)*tile_w + x % tile_w,
 *   M[(a1,a2),(c1,c2)] = L_{a2}[a1,c1] * R_{c1}[a2,c2],
 * where L and R come from `iters` rounds of alternating refinement (each an
 * R step then an L step):
 *   R step: q~[c1,a2] = sum_a1 L q / sum_a1 L;  R_{c1}[a2,:] = softmax_c2(s q~.k)
 *           h[c1,a2] = entropy of R_{c1}[a2,:]
 *   L step: k~[c1,a2] = sum_c2 R k;  L_{a2}[a1,:] = softmax_c1(s q.k~ + h)
 *   output: z = sum_c2 R v;  y[a1,a2] = sum_c1 L z;  out = y in grid order,
 * s = 1/sqrt(d).  The first R step starts from L = block identity; with a KV
 * cache (kv_len > T*H*W) the query tiles align with the last T key frames and
 * cached key tiles start from the mean query of their position.  The query
 * chunk is the newest chunk, so chunk-causal attention masks no key.  M is
 * never materialised.
 *
 * Layouts: q and out are contiguous [B, heads, T*H*W, d]; k and v are
 * contiguous [B, heads, kv_len, d]; tokens in grid order n = (t*H + y)*W + x.
 * kv_len == T*H*W is self-attention; kv_len = Tk*H*W with Tk > T is a KV-cache
 * step whose queries are the last T of the Tk key frames.
 *
 * dtype: MONARCH_F32, MONARCH_BF16 or MONARCH_F16 for q, k, v.  out_dtype:
 * MONARCH_F32 or dtype.  With bf16/f16 inputs an f32 output keeps the result
 * within 2e-2 of the output RMS of the exact (fp64) answer on peaked video
 * attention, which rounding the output to bf16 alone can exceed.
 * Arithmetic: fp32 accumulation and fp32 softmax statistics; tensor-core
 * contractions take f16 operands, with computed operands split into an f16
 * high part and an f16 low part (two products) where one rounding would cost
 * accuracy; f32 inputs use fp32 CUDA-core arithmetic throughout.
 *
 * Ownership: the caller owns q, k, v, out (device memory, 16-byte aligned).
 * The library never keeps a pointer past the call's stream work.
 * monarch_attn_fwd allocates its workspace stream-ordered on `stream` from a
 * per-device memory pool owned by the library that keeps freed memory for the
 * next call (cudaMallocFromPoolAsync / cudaFreeAsync); monarch_attn_fwd_ws
 * uses a caller buffer
 * of at least monarch_attn_workspace_bytes(...) bytes instead.
 *
 * Behaviour: asynchronous on `stream` (no host synchronisation, except in
 * monarch_attn_fwd_host); returns MONARCH_OK or a negative status, with a
 * message in monarch_attn_last_error() (thread-local).  Arguments are
 * validated on the host before any launch; kernels never trap.
 */
#ifndef MONARCH_ATTN_H
#define MONARCH_ATTN_H

#include <stddef.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  MONARCH_OK = 0,
  MONARCH_EINVAL = -1,      /* bad shape, null or misaligned pointer, bad dtype */
  MONARCH_ENOMEM = -2,      /* workspace allocation failed or buffer too small */
  MONARCH_ECUDA = -3,       /* a CUDA runtime call or launch failed */
  MONARCH_EUNSUPPORTED = -4 /* valid but outside the built kernels' limits */
};

enum { MONARCH_F32 = 0, MONARCH_BF16 = 1, MONARCH_F16 = 2 };

/* Forward.  q, k, v, out: device pointers (layouts above).  B, heads >= 1;
 * T, H, W >= 1; d in {64, 128}; tile_h | H, tile_w | W, tile_h*tile_w <= 64;
 * iters >= 1; kv_len a multiple of H*W and >= T*H*W.  stream may be 0. */
int monarch_attn_fwd(const void* q, const void* k, const void* v, void* out,
                     int B, int heads, int T, int H, int W, int d,
                     int tile_h, int tile_w, int iters, long kv_len,
                     int dtype, int out_dtype, cudaStream_t stream);

/* monarch_attn_fwd with the frame-chunk causal mask used when training over
 * the whole sequence (MonarchRT explainers, gist.science §1
 * "auto-regressive generation"): frames form chunks of chunk_frames from
 * frame 0, and a query of chunk i attends only to keys of chunks <= i.  In
 * the Monarch form this restricts the support of the factor L: the R step
 * (inside one tile, one frame) is unchanged, the L step's softmax runs over
 * the visible key tiles and the column pass over the queries that see a key
 * tile.  chunk_frames = 0, or >= T, is the bidirectional call.
 * Arguments, layout, ownership and errors as monarch_attn_fwd, plus:
 * MONARCH_EINVAL for chunk_frames < 0; MONARCH_EUNSUPPORTED for
 * chunk_frames > 0 with a KV cache (kv_len > T*H*W: the query chunk is then
 * the newest and sees every key, so call monarch_attn_fwd). */
int monarch_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                        int B, int heads, int T, int H, int W, int d,
                        int tile_h, int tile_w, int iters, long kv_len, int chunk_frames,
                        int dtype, int out_dtype, cudaStream_t stream);

/* Bytes of workspace the forward needs for these arguments (0 on invalid
 * arguments, with the reason in monarch_attn_last_error()). */
size_t monarch_attn_workspace_bytes(int B, int heads, int T, int H, int W, int d,
                                    int tile_h, int tile_w, int iters, long kv_len,
                                    int dtype);

/* Same as monarch_attn_fwd with a caller-owned device workspace of
 * workspace_bytes >= monarch_attn_workspace_bytes(...); nothing is allocated.
 * The workspace must not be used by other work while the call's stream work
 * runs. */
int monarch_attn_fwd_ws(const void* q, const void* k, const void* v, void* out,
                        int B, int heads, int T, int H, int W, int d,
                        int tile_h, int tile_w, int iters, long kv_len,
                        int dtype, int out_dtype, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* Backward of the one-step forward (iters = 1, self-attention: kv_len =
 * T*H*W), with the frame-chunk causal mask of monarch_attn_fwd_ex when
 * chunk_frames > 0.  One refinement step after finetuning is the regime the
 * method trains and runs in (MonarchRT explainers §2.C, "Finetuning and
 * Efficient Implementation"); the gradients are those of
 * sum(dy * out) for out = monarch_attn_fwd(q, k, v, ..., iters = 1):
 *   L step:  dS = L (dy.z - dy.y),  dq = s dS k~,  dk~ = s dS^T q,
 *            dz = L^T dy,  dh = colsum(dS)
 *   R step:  dSr = R (dk~ k^T + dz v^T - dh ln R - rowsum(R .)),
 *            dk = R^T dk~ + s dSr^T q,  dv = R^T dz,  dq += s dSr k.
 * q, k, v: [B, heads, T*H*W, d] in `dtype`; dy, dq, dk, dv: [B, heads,
 * T*H*W, d] in `grad_dtype` (MONARCH_F32 or dtype), all caller-owned device
 * memory, 16-byte aligned; dq, dk, dv are overwritten.  The forward factors
 * are recomputed (nothing is kept from the forward call).  Arithmetic: f32
 * inputs run fp32 CUDA-core kernels (gradients within 1e-3 of the RMS of the
 * exact ones); bf16/f16 inputs run tensor-core kernels that carry every
 * computed operand as f16 hi + lo planes with fp32 accumulation (within
 * 2e-2 of the RMS, plus one rounding of the stored gradient).  The second
 * uses about 3.2 GB of workspace at 24 heads of 32760 tokens.
 * Workspace: allocated stream-ordered from the library's pool,
 * monarch_attn_bwd_workspace_bytes(...) bytes.  Asynchronous on `stream`;
 * returns MONARCH_OK or a negative status (MONARCH_EINVAL for the checks of
 * monarch_attn_fwd and a bad grad_dtype, MONARCH_EUNSUPPORTED as there). */
int monarch_attn_bwd(const void* q, const void* k, const void* v, const void* dy,
                     void* dq, void* dk, void* dv,
                     int B, int heads, int T, int H, int W, int d,
                     int tile_h, int tile_w, int chunk_frames,
                     int dtype, int grad_dtype, cudaStream_t stream);

/* Saved-state training pair (bf16 / f16 inputs).  monarch_attn_fwd_train is
 * the one-step forward of monarch_attn_bwd's setting (iters = 1,
 * self-attention, chunk_frames as in monarch_attn_fwd_ex) with an f32 output
 * `out` [B, heads, T*H*W, d] and, in `lse`, the base-2 log-sum-exp of every
 * row of the factor L: f32, [B*heads][tile_h*tile_w][b1q_pad] with b1q =
 * T*(H/tile_h)*(W/tile_w) query tiles and b1q_pad = b1q rounded up to a
 * multiple of 4, monarch_attn_lse_bytes(...) bytes, caller-owned.
 * monarch_attn_bwd_saved takes that out and lse and returns the gradients of
 * monarch_attn_bwd without recomputing the output pass (the same values).
 * Both are asynchronous on `stream`; f32 inputs return MONARCH_EUNSUPPORTED
 * (use monarch_attn_bwd); other errors as monarch_attn_bwd. */
size_t monarch_attn_lse_bytes(int B, int heads, int T, int H, int W, int d, int tile_h, int tile_w);

int monarch_attn_fwd_train(const void* q, const void* k, const void* v, float* out, float* lse,
                           int B, int heads, int T, int H, int W, int d,
                           int tile_h, int tile_w, int chunk_frames, int dtype, cudaStream_t stream);

int monarch_attn_bwd_saved(const void* q, const void* k, const void* v, const float* out,
                           const float* lse, const void* dy, void* dq, void* dk, void* dv,
                           int B, int heads, int T, int H, int W, int d,
                           int tile_h, int tile_w, int chunk_frames,
                           int dtype, int grad_dtype, cudaStream_t stream);

/* Bytes of workspace monarch_attn_bwd takes for these arguments (0 on
 * invalid arguments). */
size_t monarch_attn_bwd_workspace_bytes(int B, int heads, int T, int H, int W, int d,
                                        int tile_h, int tile_w, int chunk_frames,
                                        int dtype, int grad_dtype);

/* End-to-end variant on HOST buffers: copies q, k, v host->device, runs the
 * forward and copies out device->host, then synchronises `stream` before
 * returning (so `out` is ready).  The (batch, head) units are split into
 * groups whose copies overlap: about 10 MB of input each (at most 8 such
 * groups), the first and last ones smaller (1, 2, 4 ... units) so that the
 * copy-out starts early and the last group's tail is short.  Copies in run
 * on a library-owned stream, each group's forward on `stream` after its
 * inputs have landed (with the R-step grouping of the one-call forward, so
 * the result has the same bits), its copy out on a second library-owned
 * stream (one pair of non-blocking streams per device, kept for the
 * process).  Device buffers are allocated stream-ordered and freed before
 * return.  Pinned host memory gives asynchronous, overlapping copies;
 * pageable memory works but is slower. */
int monarch_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                          void* out_host, int B, int heads, int T, int H, int W, int d,
                          int tile_h, int tile_w, int iters, long kv_len,
                          int dtype, int out_dtype, cudaStream_t stream);

/* monarch_attn_fwd_host with the frame-chunk causal mask of
 * monarch_attn_fwd_ex (chunk_frames as there). */
int monarch_attn_fwd_host_ex(const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, int B, int heads, int T, int H, int W, int d,
                             int tile_h, int tile_w, int iters, long kv_len, int chunk_frames,
                             int dtype, int out_dtype, cudaStream_t stream);

/* Allocation-free forward (no counterpart in the paper: an interface for
 * callers that cannot allocate device memory while they run, such as a
 * real-time generation loop that must never stall or fail on an allocation,
 * or a host application that owns all device memory).  Same arguments and
 * result as monarch_attn_fwd, but the workspace comes from a fixed 128 MiB
 * array in device memory that the library holds on every device it is
 * loaded on until the process exits; no cudaMalloc / cudaMallocAsync /
 * cudaFree is called.  Problems whose workspace
 * (monarch_attn_workspace_bytes) exceeds 128 MiB are rejected with
 * MONARCH_ENOMEM and a message.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  The address is kept for
 * the life of the process: after cudaDeviceReset on a device this entry point
 * must not be called there again in the same process.  All calls on a device
 * share the one array and it keeps the last call's contents (every value is
 * written before it is read, so nothing needs clearing): calls whose GPU work
 * overlaps (different streams, or different host threads) race on it and
 * must be serialised by the caller. */
int monarch_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                             int B, int heads, int T, int H, int W, int d,
                             int tile_h, int tile_w, int iters, long kv_len,
                             int dtype, int out_dtype, cudaStream_t stream);

/* Byte offsets, inside a workspace, of the intermediates left by the last
 * iteration (for inspection in tests), each [B*heads][b2][b1k][d] per plane
 * with b2 = tile_h*tile_w positions and b1k = kv_len/(H*W) * (H/tile_h) *
 * (W/tile_w) key tiles: [0] k~ (f32 for f32 inputs; otherwise an f16 high
 * plane followed by an f16 low plane, k~ = high + low), [1] z (same types),
 * [2] q~ of the last R step with iters >= 2 (f32 for f32 inputs; otherwise a
 * high and a low plane of the input type), [3] h [B*heads][b2][b1k_pad]
 * (f32; in nats for f32 inputs, in bits, i.e. base-2 entropy, for bf16/f16
 * inputs), [4] row log2-sum-exp of the last non-final L step
 * [B*heads][b2][b1q_pad] (f32, base-2 logits s*log2(e)*q.k~ + log2(e)*h),
 * [5] KV-init mean query [B*heads][b2][d] (f32 for f32 inputs; otherwise a
 * high and a low plane of the input type), [6] queries in block-major
 * order [B*heads][b2][b1q][d] (f16 for bf16/f16 inputs; absent for f32).
 * b1k_pad and b1q_pad are b1k and b1q rounded up to a multiple of 4.
 * Returns the total bytes, 0 on invalid arguments. */
size_t monarch_attn_workspace_layout(int B, int heads, int T, int H, int W, int d,
                                     int tile_h, int tile_w, int iters, long kv_len,
                                     int dtype, size_t offsets[7]);

/* Instrumentation.  Kernel phases of one forward: */
enum {
  MONARCH_PHASE_QBAR = 0,   /* mean query per position (KV-cache init)        */
  MONARCH_PHASE_R_STEP = 1, /* R step: per-tile softmax, entropy, k~ (and z)  */
  MONARCH_PHASE_L_LSE = 2,  /* L step LSE pass of a non-final iteration      */
  MONARCH_PHASE_L_OUT = 3,  /* final L step fused with y = L z and the store  */
  MONARCH_PHASE_L_COL = 4,  /* column pass q~ = L^T q / L^T 1                 */
  /* backward (monarch_attn_bwd; its R-step recompute counts as R_STEP): */
  MONARCH_PHASE_BWD_PREP = 5, /* row LSE and D = dy . y of the L step          */
  MONARCH_PHASE_BWD_DQ = 6,   /* L-step part of dq, per query row               */
  MONARCH_PHASE_BWD_DKV = 7,  /* dk~, dz, dh per key column                      */
  MONARCH_PHASE_BWD_R = 8,    /* R-step backward per tile: dk, dv, dq finished */
  /* one refinement step (iters = 1, bf16/f16) as one kernel, R step and output
   * pass together; used when the environment variable MONARCH_ONESTEP_KERNEL
   * is "1" at the call (the default runs the two kernels, which is faster on
   * B200; both give the same values bit for bit) */
  MONARCH_PHASE_ONESTEP = 9,
  /* a non-final L step with at most 256 query and 256 key tiles: the LSE
   * pass and the column pass in one kernel, operands kept on chip */
  MONARCH_PHASE_L_LSECOL = 10,
  MONARCH_NUM_PHASES = 11
};

/* Number of kernels this process has launched through the library (host
 * counter, always on). */
unsigned long long monarch_attn_launch_count(void);

/* on != 0: record a CUDA event pair on the launching stream around every
 * kernel launch from now on (adds a few microseconds per launch); 0: stop.
 * Returns MONARCH_OK. */
int monarch_attn_profile_enable(int on);

/* Waits for the recorded events and adds, per phase p < n, the total kernel
 * milliseconds to ms[p] and the launch count to launches[p] (either pointer
 * may be null), accumulated since the last reset; reset != 0 clears the
 * totals afterwards.  Returns MONARCH_OK or MONARCH_ECUDA. */
int monarch_attn_profile_read(double* ms, unsigned long long* launches, int n, int reset);

/* Device error word of the current device: 0 when no kernel of this library
 * has reported a problem; 1 when a bounded wait inside a kernel gave up (the
 * kernel then skipped its remaining work and its output is invalid).
 * Synchronous (reads device memory); reset != 0 clears the word.  Returns -1
 * if the word cannot be read. */
int monarch_attn_device_error(int reset);

/* Thread-local message of the last failing call ("" if none). */
const char* monarch_attn_last_error(void);

/* ABI version (major*100 + minor): 1.02 adds the backward (monarch_attn_bwd),
 * the training pair and monarch_attn_fwd_host_ex to the forward of 1.00; 1.03
 * adds MONARCH_PHASE_ONESTEP (one refinement step as one kernel, on request)
 * and MONARCH_PHASE_L_LSECOL. */
int monarch_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MONARCH_ATTN_H */
