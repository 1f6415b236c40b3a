// Host side of the Monarch video-attention forward: argument validation,
// geometry, workspace layout and the launch sequence of one call.  Every
// step of the computation runs in this library's kernels.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cmath>
#include <chrono>
#include <cstdlib>
#include <mutex>
#include <atomic>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "monarch_attn.h"
#include "common.cuh"
#include "kernels_simt.cuh"
#include "kernels_tc.cuh"
#include "kernels_rtc.cuh"
#include "kernels_l.cuh"
#include "kernels_onestep.cuh"
#include "kernels_lsecol.cuh"
#include "kernels_bwd.cuh"
#include "kernels_bwd_tc.cuh"

using namespace monarch;

namespace {

constexpr int kMaxDevices = 64;   // device ordinals with per-device state

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MONARCH_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---- instrumentation: launch counter and optional per-phase event timing ----
std::atomic<unsigned long long> g_launches{0};

struct Profiler {
  std::mutex mu;
  bool on = false;
  struct Rec { int phase; cudaEvent_t a, b; };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  double ms[MONARCH_NUM_PHASES] = {};
  unsigned long long n[MONARCH_NUM_PHASES] = {};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Profiler g_prof;

// MONARCH_DEBUG_SYNC=1: synchronise after every launch and report the phase,
// the time and the device error word on stderr (debugging aid).
bool debug_sync() {
  static const bool on = [] {
    const char* e = getenv("MONARCH_DEBUG_SYNC");
    return e && e[0] == '1';
  }();
  return on;
}

int read_device_error(int reset);

// MONARCH_ONESTEP_KERNEL=1 (read at every call): run one refinement step
// (bf16 / f16) as the single kernel onestep_tc instead of the R-step kernel
// followed by the output-pass kernel.  Both compute the same values bit for
// bit; the two kernels are the faster of the two on B200 and the default.
bool onestep_fused() {
  const char* e = getenv("MONARCH_ONESTEP_KERNEL");
  return e && e[0] == '1';
}

// Launches one kernel through `f`, counting it and, when profiling is on,
// bracketing it with events on its stream.
template <typename F>
void launch(int phase, cudaStream_t st, F&& f) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (debug_sync()) {
    static const char* names[] = {"qbar", "r_step", "l_lse", "l_out", "l_col",
                                  "bwd_prep", "bwd_dq", "bwd_dkv", "bwd_r", "onestep", "l_lsecol"};
    fprintf(stderr, "[monarch] launch %s ...\n", names[phase]);
    auto t0 = std::chrono::steady_clock::now();
    f();
    cudaError_t e = cudaStreamSynchronize(st);
    const double ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
    fprintf(stderr, "[monarch]   %s done: %.3f ms, %s, device error word %d\n", names[phase], ms,
            cudaGetErrorString(e), read_device_error(0));
    return;
  }
  if (!g_prof.on) {
    f();
    return;
  }
  std::lock_guard<std::mutex> lk(g_prof.mu);
  cudaEvent_t a = g_prof.get(), b = g_prof.get();
  cudaEventRecord(a, st);
  f();
  cudaEventRecord(b, st);
  g_prof.pending.push_back({phase, a, b});
}

int read_device_error(int reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ptx::g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (reset) {
    const int z = 0;
    cudaMemcpyToSymbol(ptx::g_device_error, &z, sizeof(int));
  }
  return v;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t elem_size(int dtype) { return dtype == MONARCH_F32 ? 4 : 2; }

constexpr int kRegions = 7;  // k~, z, q~, h, lse, mean query, block-major q

struct Plan {
  Geo g;
  int dtype;
  int out_dtype;
  int iters;
  bool kv;
  size_t off[kRegions];
  size_t counters;   // int [1 + BH]: the ticket and per-head R-item counts of onestep_tc
  size_t total;
  // key tiles per R-step CTA; 0: chosen for this plan's geometry.  A call that
  // runs its units in groups sets the whole call's choice: the stacking of
  // key tiles sets the order of the MMAs' sums, so every group then computes
  // the bits of the one-call forward.
  int r_group = 0;
};

constexpr int kMaxB2 = 64;

int make_plan(int B, int heads, int T, int H, int W, int d, int th, int tw, int iters,
              long kv_len, int dtype, int out_dtype, Plan* p, int chunk_frames = 0) {
  if (B < 1 || heads < 1 || T < 1 || H < 1 || W < 1)
    return fail(MONARCH_EINVAL, "B, heads, T, H, W must be >= 1 (got %d %d %d %d %d)", B, heads, T, H, W);
  if (d != 64 && d != 128) return fail(MONARCH_EINVAL, "head_dim d must be 64 or 128 (got %d)", d);
  if (th < 1 || tw < 1 || H % th || W % tw)
    return fail(MONARCH_EINVAL, "tile %dx%d must divide the %dx%d frame", th, tw, H, W);
  if (iters < 1) return fail(MONARCH_EINVAL, "iters must be >= 1 (got %d)", iters);
  if (dtype != MONARCH_F32 && dtype != MONARCH_BF16 && dtype != MONARCH_F16)
    return fail(MONARCH_EINVAL, "unknown dtype %d", dtype);
  if (out_dtype != dtype && out_dtype != MONARCH_F32)
    return fail(MONARCH_EINVAL, "out_dtype %d must be MONARCH_F32 or the input dtype %d", out_dtype, dtype);
  const long long hw = (long long)H * W;
  const long long nq = (long long)T * hw;
  if (kv_len < nq || kv_len % hw)
    return fail(MONARCH_EINVAL, "kv_len %ld must be a multiple of H*W=%lld and >= T*H*W=%lld", kv_len, hw, nq);
  if (th * tw > kMaxB2)
    return fail(MONARCH_EUNSUPPORTED, "tile_h*tile_w = %d exceeds the supported %d positions per tile", th * tw, kMaxB2);
  const long long Tk = kv_len / hw;
  const long long BH = (long long)B * heads;
  if (BH * (long long)kv_len * d >= (1LL << 40) || Tk * (H / th) * (W / tw) >= (1LL << 30) || BH > 65535)
    return fail(MONARCH_EUNSUPPORTED, "problem too large");
  Geo& g = p->g;
  g.BH = (int)BH;
  g.T = T;
  g.Tk = (int)Tk;
  g.H = H;
  g.W = W;
  g.d = d;
  g.th = th;
  g.tw = tw;
  g.ntx = W / tw;
  g.P = (H / th) * (W / tw);
  g.b2 = th * tw;
  g.b1q = T * g.P;
  g.b1k = g.Tk * g.P;
  g.off = (g.Tk - T) * g.P;
  g.b1k_pad = (g.b1k + 3) & ~3;
  g.b1q_pad = (g.b1q + 3) & ~3;
  g.Nq = nq;
  g.Nk = kv_len;
  g.sl2 = (float)(1.0 / std::sqrt((double)d) * 1.4426950408889634);
  if (chunk_frames < 0) return fail(MONARCH_EINVAL, "chunk_frames must be >= 0 (got %d)", chunk_frames);
  if (chunk_frames > 0 && g.Tk != T)
    return fail(MONARCH_EUNSUPPORTED,
                "the frame-chunk causal mask is for self-attention (kv_len == T*H*W); with a KV cache the "
                "query chunk is the newest and sees every key");
  g.cq = (chunk_frames > 0 && chunk_frames < T) ? chunk_frames * g.P : 0;   // C >= T: one chunk, no mask
  g.pk = 1;
  g.pb1q = g.b1q;
  g.pb1k = g.b1k;
  p->dtype = dtype;
  p->out_dtype = out_dtype;
  p->iters = iters;
  p->kv = g.Tk != T;
  const size_t big = (size_t)BH * g.b2 * g.b1k * d * 4;  // fp32, or two 16-bit planes
  size_t sizes[kRegions] = {big,
                            big,
                            big,
                            (size_t)BH * g.b2 * g.b1k_pad * 4,
                            (size_t)BH * g.b2 * g.b1q_pad * 4,
                            (size_t)BH * g.b2 * d * 4,
                            dtype == MONARCH_F32 ? 0 : (size_t)BH * g.b2 * g.b1q * d * 2};
  size_t o = 0;
  for (int i = 0; i < kRegions; ++i) {
    p->off[i] = o;
    o += align256(sizes[i]);
  }
  p->counters = o;
  o += align256((size_t)(1 + BH) * sizeof(int));
  p->total = o;
  return MONARCH_OK;
}

int check_ptr(const void* ptr, const char* name) {
  if (!ptr) return fail(MONARCH_EINVAL, "%s is null", name);
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return fail(MONARCH_EINVAL, "%s is not 16-byte aligned", name);
  return MONARCH_OK;
}

// ---- tensor-core path (bf16 / f16 inputs) -------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// Tiled tensor map with a 128-byte swizzle (rank 2 or 3, 16-bit or 32-bit
// elements); zero fill outside the tensor.
int make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int rank, const cuuint64_t* dims,
             const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swz) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MONARCH_ECUDA, "cuTensorMapEncodeTiled is not available");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, dt, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MONARCH_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MONARCH_OK;
}

// Launch with programmatic stream serialization: the kernel may begin its
// set-up while the previous kernel on the stream finishes; it waits
// (griddepcontrol.wait) before touching global memory.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Runs `set` (a call site's shared-memory limits) once per device: a function
// attribute belongs to the current device's context.  Ordinals outside the
// table are set on every call.
template <typename F>
cudaError_t once_per_device(std::atomic<bool> (&done)[kMaxDevices], F&& set) {
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e = set();
  if (e == cudaSuccess && cached) done[dev].store(true, std::memory_order_release);
  return e;
}

// Key tiles per R-step CTA.  At most floor(128 / r8) fit the 128 MMA rows;
// fewer give more, shorter CTAs.  Two CTAs run per SM, so the launch takes
// ceil(CTAs / (2 * SMs)) rounds of CTAs whose time grows with G plus a fixed
// part (loads, the MMA and softmax chain, the epilogue).  The group size with
// the fewest rounds x (G + kRFixed) is taken.  Measured on B200 with 6 x 4
// tiles, a CTA takes about (G + 3.7) times the time of one tile's share.
int r_step_group(const Geo& g, int sm_count) {
  constexpr double kRFixed = 3.5;   // fixed part of a CTA's time, in tiles
  const int gmax = kRtcRows / ((g.b2 + 7) & ~7);
  int best = gmax;
  double best_t = 1e300;
  for (int G = gmax; G >= 1; --G) {
    const long long ctas = (long long)((g.b1k + G - 1) / G) * g.BH;
    const long long rounds = (ctas + 2LL * sm_count - 1) / (2LL * sm_count);
    const double t = (double)rounds * (G + kRFixed);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = G;
    }
  }
  return best;
}

int sm_count_of_device() {
  static std::atomic<int> n[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = n[dev].load(std::memory_order_relaxed);
  if (!v) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 1;
    n[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Geometry of the L-step kernels.  On small self-attention grids (one
// position's problem is b1 x b1 with b1 a multiple of 4 that divides 128) the
// L step stacks pk = 128 / b1 positions of a head in one 128-row block, each
// row seeing only its own position's keys (row_keys / col_queries): one CTA
// then does pk positions' work, where each would otherwise fill a 128-row
// tensor-core tile with b1 rows.  Positions are contiguous in every
// position-major buffer ([BH][b2][b1][d] and the padded h and LSE rows, whose
// padding is zero when b1 is a multiple of 4), so the stacked geometry views
// the same memory.
Geo stacked_geometry(const Geo& g) {
  Geo s = g;
  const int b1 = g.b1q;
  if (g.Tk != g.T || g.b1k != b1 || b1 % 4 || b1 >= kTile || kTile % b1) return s;
  const int pk = kTile / b1;
  if (g.b2 % pk) return s;
  s.pk = pk;
  s.pb1q = s.pb1k = b1;
  s.b2 = g.b2 / pk;
  s.b1q = s.b1k = s.b1q_pad = s.b1k_pad = kTile;
  return s;
}

// Tensor maps of the L-step kernels (block-major q copy, k~ and z planes, h,
// row LSE) for geometry g, which may stack positions (stacked_geometry).
template <int D>
int tc_l_maps(const Geo& g, const Work& w, const __half* kt_hi, const __half* z_hi, tc::Maps& maps) {
  int rc;
  {
    const cuuint64_t rows = (cuuint64_t)g.BH * g.b2;
    cuuint32_t box3[3] = {64, (cuuint32_t)tc::kBlk, 1};
    cuuint64_t dq3[3] = {(cuuint64_t)D, (cuuint64_t)g.b1q, rows};
    cuuint64_t sq3[2] = {(cuuint64_t)D * 2, (cuuint64_t)g.b1q * D * 2};
    cuuint64_t dk3[3] = {(cuuint64_t)D, (cuuint64_t)g.b1k, 2 * rows};
    cuuint64_t sk3[2] = {(cuuint64_t)D * 2, (cuuint64_t)g.b1k * D * 2};
    cuuint32_t box2[2] = {(cuuint32_t)tc::kBlk, 1};
    cuuint64_t dh2[2] = {(cuuint64_t)g.b1k_pad, rows};
    cuuint64_t sh2[1] = {(cuuint64_t)g.b1k_pad * 4};
    cuuint64_t dl2[2] = {(cuuint64_t)g.b1q_pad, rows};
    cuuint64_t sl2[1] = {(cuuint64_t)g.b1q_pad * 4};
    // the L step computes in f16: q (block-major copy) and the k~ planes are f16
    if ((rc = make_map(&maps.qb, w.qb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dq3, sq3, box3,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&maps.kt, kt_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dk3, sk3, box3,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&maps.z, z_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dk3, sk3, box3,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&maps.h, w.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dh2, sh2, box2, CU_TENSOR_MAP_SWIZZLE_NONE)) ||
        (rc = make_map(&maps.lse, w.lse, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dl2, sl2, box2,
                       CU_TENSOR_MAP_SWIZZLE_NONE)))
      return rc;
  }
  return MONARCH_OK;
}

// Workspace views and tensor maps of the tensor-core forward (shared by the
// forward and the backward's recompute).
template <typename TQ, int D>
int tc_prepare(const Geo& g, const TQ* q, const TQ* k, const TQ* v, const Work& w, TcPlanes<TQ>& planes,
               tc::Maps& maps, RtcMaps& rmaps, int G) {
  planes.kt_hi = reinterpret_cast<__half*>(w.kt);
  planes.z_hi = reinterpret_cast<__half*>(w.z);
  planes.plane = (long long)g.BH * g.b2 * g.b1k * D;
  const CUtensorMapDataType dq =
      TcType<TQ>::kBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  int rc;
  if ((rc = tc_l_maps<D>(g, w, planes.kt_hi, planes.z_hi, maps))) return rc;
  // R-step maps: the key / value / query grids as (d, W, H, frames) with one
  // tile per box, and the q~ planes as (d, b1k, 2*BH*b2) with one key tile per box
  {
    cuuint32_t box4[4] = {64, (cuuint32_t)g.tw, (cuuint32_t)g.th, 1};
    cuuint64_t dk4[4] = {(cuuint64_t)D, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.BH * g.Tk};
    cuuint64_t dq4[4] = {(cuuint64_t)D, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.BH * g.T};
    cuuint64_t s4[3] = {(cuuint64_t)D * 2, (cuuint64_t)g.W * D * 2, (cuuint64_t)g.H * g.W * D * 2};
    cuuint32_t boxt[3] = {64, 1, (cuuint32_t)g.b2};
    cuuint64_t dt3[3] = {(cuuint64_t)D, (cuuint64_t)g.b1k, 2 * (cuuint64_t)g.BH * g.b2};
    cuuint64_t st3[2] = {(cuuint64_t)D * 2, (cuuint64_t)g.b1k * D * 2};
    // the mean-query planes of the KV-init step: [2][BH][b2][d], one "tile"
    cuuint64_t dm3[3] = {(cuuint64_t)D, 1, 2 * (cuuint64_t)g.BH * g.b2};
    cuuint64_t sm3[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2};
    if ((rc = make_map(&rmaps.q, q, dq, 4, dq4, s4, box4, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.k, k, dq, 4, dk4, s4, box4, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.v, v, dq, 4, dk4, s4, box4, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.qt, w.qt, dq, 3, dt3, st3, boxt, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.qm, w.qbar, dq, 3, dm3, sm3, boxt, CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
    // R-step stores of all G tiles of an item in one box per (plane, d half):
    // dims (d, position, tile, plane*BH + head), the position stride above the
    // tile stride, so the box's shared-memory rows are tile-major (tile g at
    // rows [g b2, (g + 1) b2))
    cuuint32_t boxg[4] = {64, (cuuint32_t)g.b2, (cuuint32_t)G, 1};
    cuuint64_t dg4[4] = {(cuuint64_t)D, (cuuint64_t)g.b2, (cuuint64_t)g.b1k, 2 * (cuuint64_t)g.BH};
    cuuint64_t sg4[3] = {(cuuint64_t)g.b1k * D * 2, (cuuint64_t)D * 2, (cuuint64_t)g.b2 * g.b1k * D * 2};
    cuuint64_t dgq[4] = {(cuuint64_t)D, (cuuint64_t)g.b2, (cuuint64_t)g.b1q, (cuuint64_t)g.BH};
    cuuint64_t sgq[3] = {(cuuint64_t)g.b1q * D * 2, (cuuint64_t)D * 2, (cuuint64_t)g.b2 * g.b1q * D * 2};
    if ((rc = make_map(&rmaps.kt, planes.kt_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, dg4, sg4, boxg,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.z, planes.z_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, dg4, sg4, boxg,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&rmaps.qbg, w.qb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, dgq, sgq, boxg,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
    cuuint64_t db3[3] = {(cuuint64_t)D, (cuuint64_t)g.b1q, (cuuint64_t)g.BH * g.b2};
    cuuint64_t sb3[2] = {(cuuint64_t)D * 2, (cuuint64_t)g.b1q * D * 2};
    if ((rc = make_map(&rmaps.qb, w.qb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, db3, sb3, boxt,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
  }
  return MONARCH_OK;
}

template <typename TQ, typename TO, int D>
int run_tc(const Plan& p, const TQ* q, const TQ* k, const TQ* v, TO* out, char* ws, cudaStream_t st) {
  const Geo& g = p.g;
  Work w;
  w.kt = reinterpret_cast<float*>(ws + p.off[0]);
  w.z = reinterpret_cast<float*>(ws + p.off[1]);
  w.qt = reinterpret_cast<float*>(ws + p.off[2]);
  w.h = reinterpret_cast<float*>(ws + p.off[3]);
  w.lse = reinterpret_cast<float*>(ws + p.off[4]);
  w.qbar = reinterpret_cast<float*>(ws + p.off[5]);
  w.qb = ws + p.off[6];
  TcPlanes<TQ> planes;
  tc::Maps maps;
  RtcMaps rmaps;
  int rc;
  const int r_group = p.r_group ? p.r_group : r_step_group(g, sm_count_of_device());   // key tiles per R-step CTA
  if ((rc = tc_prepare<TQ, D>(g, q, k, v, w, planes, maps, rmaps, r_group))) return rc;

  constexpr size_t smem_lse = tc::lse_smem<D>();
  constexpr size_t smem_out = tc::row_smem<D, true>();
  constexpr size_t smem_col = tc::col_smem<D>();
  constexpr size_t smem_r = rtc_smem<D>();
  constexpr size_t smem_lc = tc::LsecolLayout<D>::smem();
  // at most 256 query and 256 key tiles: a non-final L step is one kernel
  // (l_lsecol) that keeps its operands on chip for both of its passes
  const bool small_l = g.b1q <= 2 * kTile && g.b1k <= 2 * kTile;

  static std::atomic<bool> attrs_set[kMaxDevices];
  {
    const cudaError_t e = once_per_device(attrs_set, [&] {
      cudaError_t r;
      if ((r = allow_smem(tc::l_lse<D>, smem_lse)) != cudaSuccess ||
          (r = allow_smem(tc::l_row<__half, TO, D, true>, smem_out)) != cudaSuccess ||
          (r = allow_smem(tc::l_col<TQ, D>, smem_col)) != cudaSuccess ||
          (r = allow_smem(tc::l_lsecol<TQ, D>, smem_lc)) != cudaSuccess ||
          (r = allow_smem(r_step_tc5<TQ, D>, smem_r)) != cudaSuccess)
        return r;
      return cudaSuccess;
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  }
  const dim3 grid_q((g.b1q + 2 * kTile - 1) / (2 * kTile), g.b2, g.BH);  // two 128-row tiles per CTA
  // persistent column pass: one CTA per SM over (head, position, 256 key tiles) items
  const int sm_count = sm_count_of_device();
  const long long col_items = (long long)g.BH * g.b2 * ((g.b1k + 2 * kTile - 1) / (2 * kTile));
  const dim3 grid_k((unsigned)std::min<long long>(col_items, sm_count));
  const dim3 grid_r((g.b1k + r_group - 1) / r_group, g.BH);
  if (p.iters == 1 && onestep_fused()) {
    // one refinement step: the R step and the output pass in one kernel
    constexpr size_t smem_one = onestep_smem<D>();
    static std::atomic<bool> one_set[kMaxDevices];
    cudaError_t e = once_per_device(one_set, [&] { return allow_smem(onestep_tc<TQ, TO, D>, smem_one); });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(onestep)");
    int* counters = reinterpret_cast<int*>(ws + p.counters);
    if ((e = cudaMemsetAsync(counters, 0, (size_t)(1 + g.BH) * sizeof(int), st)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync(counters)");
    if (p.kv)
      launch(MONARCH_PHASE_QBAR, st, [&] {
        launch_pdl(qbar_kernel<TQ>, dim3(g.b2, g.BH), dim3(kQbarThreads), 0, st, q, w.qbar, g);
      });
    const long long n_r = (long long)grid_r.x * g.BH;
    const long long n_l = (long long)grid_q.x * grid_q.y * grid_q.z;
    // launched in plain stream order (after the counters are zeroed)
    launch(MONARCH_PHASE_ONESTEP, st, [&] {
      onestep_tc<TQ, TO, D><<<(unsigned)((n_r + 1) / 2 + n_l), tc::kThreads, smem_one, st>>>(
          rmaps, maps, q, w, planes, out, g, p.kv ? (int)QT_KVINIT : (int)QT_IDENTITY, r_group, counters);
    });
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return MONARCH_OK;
  }
  // the L-step kernels below run on the stacked geometry when it applies
  const Geo gl = stacked_geometry(g);
  if (gl.pk > 1 && (rc = tc_l_maps<D>(gl, w, planes.kt_hi, planes.z_hi, maps))) return rc;
  const dim3 grid_ql((gl.b1q + 2 * kTile - 1) / (2 * kTile), gl.b2, gl.BH);
  for (int it = 0; it < p.iters; ++it) {
    const int final_step = it == p.iters - 1;
    int mode = QT_BUFFER;
    if (it == 0) {
      mode = p.kv ? QT_KVINIT : QT_IDENTITY;
      if (p.kv)
        launch(MONARCH_PHASE_QBAR, st, [&] {
          launch_pdl(qbar_kernel<TQ>, dim3(g.b2, g.BH), dim3(kQbarThreads), 0, st, q, w.qbar, g);
        });
    } else if (!small_l) {
      launch(MONARCH_PHASE_L_COL, st, [&] {
        launch_pdl(tc::l_col<TQ, D>, grid_k, dim3(tc::kThreads), smem_col, st, maps, (const float*)w.h,
                   reinterpret_cast<TQ*>(w.qt), g);
      });
    }
    launch(MONARCH_PHASE_R_STEP, st, [&] {
      launch_pdl(r_step_tc5<TQ, D>, grid_r, dim3(kRtcThreads), smem_r, st, rmaps, q, w, planes, g, mode, final_step,
                 r_group);
    });
    if (final_step) {
      launch(MONARCH_PHASE_L_OUT, st, [&] {
        launch_pdl(tc::l_row<__half, TO, D, true>, grid_ql, dim3(tc::kThreads), smem_out, st, out, maps, w.lse, gl);
      });
    } else if (small_l) {
      launch(MONARCH_PHASE_L_LSECOL, st, [&] {
        launch_pdl(tc::l_lsecol<TQ, D>, dim3(gl.b2, gl.BH), dim3(tc::kThreads), smem_lc, st, maps, w.lse,
                   reinterpret_cast<TQ*>(w.qt), gl);
      });
    } else {
      launch(MONARCH_PHASE_L_LSE, st, [&] {
        launch_pdl(tc::l_lse<D>, grid_q, dim3(tc::kThreads), smem_lse, st, maps, w.lse, g);
      });
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MONARCH_OK;
}

template <typename T, typename TO>
int run(const Plan& p, const T* q, const T* k, const T* v, TO* out, char* ws, cudaStream_t st) {
  const Geo& g = p.g;
  Work w;
  w.kt = reinterpret_cast<float*>(ws + p.off[0]);
  w.z = reinterpret_cast<float*>(ws + p.off[1]);
  w.qt = reinterpret_cast<float*>(ws + p.off[2]);
  w.h = reinterpret_cast<float*>(ws + p.off[3]);
  w.lse = reinterpret_cast<float*>(ws + p.off[4]);
  w.qbar = reinterpret_cast<float*>(ws + p.off[5]);
  w.qb = ws + p.off[6];

  const size_t r_smem = (size_t)(3 * g.b2 * g.d + g.b2 * (g.b2 + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(r_step_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)r_smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(r_step)");
  constexpr int kRows = 16;
  for (int it = 0; it < p.iters; ++it) {
    const int final_step = it == p.iters - 1;
    int mode = QT_BUFFER;
    if (it == 0) {
      mode = p.kv ? QT_KVINIT : QT_IDENTITY;
      if (p.kv)
        launch(MONARCH_PHASE_QBAR, st, [&] { qbar_kernel<T><<<dim3(g.b2, g.BH), kQbarThreads, 0, st>>>(q, w.qbar, g); });
    } else {
      dim3 grid((g.b1k + kRows - 1) / kRows, g.b2, g.BH);
      launch(MONARCH_PHASE_L_COL, st, [&] {
        if (g.d == 128) l_col_simt<T, 128><<<grid, 32 * kRows, 0, st>>>(q, w, g);
        else l_col_simt<T, 64><<<grid, 32 * kRows, 0, st>>>(q, w, g);
      });
    }
    launch(MONARCH_PHASE_R_STEP, st, [&] {
      r_step_simt<T><<<dim3(g.b1k, g.BH), 128, r_smem, st>>>(q, k, v, w, g, mode, final_step);
    });
    dim3 grid((g.b1q + kRows - 1) / kRows, g.b2, g.BH);
    launch(final_step ? MONARCH_PHASE_L_OUT : MONARCH_PHASE_L_LSE, st, [&] {
      if (g.d == 128) l_row_simt<T, TO, 128><<<grid, 32 * kRows, 0, st>>>(q, out, w, g, final_step);
      else l_row_simt<T, TO, 64><<<grid, 32 * kRows, 0, st>>>(q, out, w, g, final_step);
    });
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MONARCH_OK;
}

template <typename T, typename TO>
int run_any(const Plan& p, const T* q, const T* k, const T* v, TO* out, char* w, cudaStream_t st) {
  if constexpr (sizeof(T) == 4) {
    return run<T, TO>(p, q, k, v, out, w, st);
  } else {
    if (p.g.d == 128) return run_tc<T, TO, 128>(p, q, k, v, out, w, st);
    return run_tc<T, TO, 64>(p, q, k, v, out, w, st);
  }
}

template <typename T>
int dispatch_out(const Plan& p, const void* q, const void* k, const void* v, void* out, char* w,
                 cudaStream_t st) {
  if (p.out_dtype == MONARCH_F32)
    return run_any<T, float>(p, (const T*)q, (const T*)k, (const T*)v, (float*)out, w, st);
  return run_any<T, T>(p, (const T*)q, (const T*)k, (const T*)v, (T*)out, w, st);
}

int dispatch(const Plan& p, const void* q, const void* k, const void* v, void* out, void* ws,
             cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  switch (p.dtype) {
    case MONARCH_F32: return dispatch_out<float>(p, q, k, v, out, w, st);
    case MONARCH_BF16: return dispatch_out<__nv_bfloat16>(p, q, k, v, out, w, st);
    default: return dispatch_out<__half>(p, q, k, v, out, w, st);
  }
}

// ---- backward (one-step forward, self-attention) -------------------------
constexpr int kBwdRegions = 9;  // f32 path: k~, z, h, lse, D, dqL, dk~, dz, dh
constexpr int kBwdTcRegions = 8;  // tensor-core path, after the forward's regions: y, dy planes, D, amax, dqL, dk~, dz, dh

struct BwdPlan {
  Plan fwd;   // geometry and validation of the forward it differentiates
  int grad_dtype;
  bool tc;    // bf16 / f16 inputs: tensor-core L-step backward
  size_t off[kBwdRegions];
  size_t toff[kBwdTcRegions];
  size_t total;
};

int make_bwd_plan(int B, int heads, int T, int H, int W, int d, int th, int tw, int chunk_frames, int dtype,
                  int grad_dtype, BwdPlan* bp) {
  const long kv = (long)T * H * W;
  int rc = make_plan(B, heads, T, H, W, d, th, tw, 1, kv, dtype, dtype, &bp->fwd, chunk_frames);
  if (rc) return rc;
  if (grad_dtype != dtype && grad_dtype != MONARCH_F32)
    return fail(MONARCH_EINVAL, "grad_dtype %d must be MONARCH_F32 or the input dtype %d", grad_dtype, dtype);
  bp->grad_dtype = grad_dtype;
  bp->tc = dtype != MONARCH_F32;
  const Geo& g = bp->fwd.g;
  const size_t big = (size_t)g.BH * g.b2 * g.b1k * d * 4;
  const size_t col = (size_t)g.BH * g.b2 * g.b1k_pad * 4;
  const size_t row = (size_t)g.BH * g.b2 * g.b1q_pad * 4;
  size_t o = 0;
  if (bp->tc) {
    const size_t sizes[kBwdTcRegions] = {(size_t)g.BH * g.Nq * d * 4, (size_t)2 * g.BH * g.b2 * g.b1q * d * 2, row,
                                         (size_t)g.BH * 4, big, big, big, col};
    o = bp->fwd.total;
    for (int i = 0; i < kBwdTcRegions; ++i) {
      bp->toff[i] = o;
      o += align256(sizes[i]);
    }
  } else {
    const size_t sizes[kBwdRegions] = {big, big, col, row, row, big, big, big, col};
    for (int i = 0; i < kBwdRegions; ++i) {
      bp->off[i] = o;
      o += align256(sizes[i]);
    }
  }
  bp->total = o;
  return MONARCH_OK;
}

template <typename T, typename TG, int D>
void launch_l_bwd(const Geo& g, const T* q, const TG* dy, const Work& w, const BwdWork& bw, cudaStream_t st) {
  constexpr int kRows = 16;
  const dim3 rgrid((g.b1q + kRows - 1) / kRows, g.b2, g.BH);
  const dim3 cgrid((g.b1k + kRows - 1) / kRows, g.b2, g.BH);
  launch(MONARCH_PHASE_BWD_PREP, st, [&] { l_bwd_prep_simt<T, TG, D><<<rgrid, 32 * kRows, 0, st>>>(q, dy, w, bw, g); });
  launch(MONARCH_PHASE_BWD_DQ, st, [&] { l_bwd_dq_simt<T, TG, D><<<rgrid, 32 * kRows, 0, st>>>(q, dy, w, bw, g); });
  launch(MONARCH_PHASE_BWD_DKV, st, [&] { l_bwd_dkv_simt<T, TG, D><<<cgrid, 32 * kRows, 0, st>>>(q, dy, w, bw, g); });
}

// Recomputes the forward's R step (k~, z, h), then runs the L-step backward
// passes and the per-tile R-step backward, which writes dq, dk, dv.
template <typename T, typename TG>
int run_bwd(const BwdPlan& bp, const T* q, const T* k, const T* v, const TG* dy, TG* dq, TG* dk, TG* dv,
            char* ws, cudaStream_t st) {
  const Geo& g = bp.fwd.g;
  Work w = {};
  w.kt = reinterpret_cast<float*>(ws + bp.off[0]);
  w.z = reinterpret_cast<float*>(ws + bp.off[1]);
  w.h = reinterpret_cast<float*>(ws + bp.off[2]);
  w.lse = reinterpret_cast<float*>(ws + bp.off[3]);
  BwdWork bw;
  bw.dd = reinterpret_cast<float*>(ws + bp.off[4]);
  bw.dqL = reinterpret_cast<float*>(ws + bp.off[5]);
  bw.dkt = reinterpret_cast<float*>(ws + bp.off[6]);
  bw.dz = reinterpret_cast<float*>(ws + bp.off[7]);
  bw.dh = reinterpret_cast<float*>(ws + bp.off[8]);

  const size_t r_smem = (size_t)(3 * g.b2 * g.d + g.b2 * (g.b2 + 1)) * sizeof(float);
  cudaError_t e = allow_smem(r_step_simt<T>, r_smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(r_step)");
  const size_t rb_smem = r_bwd_smem_bytes(g.b2, g.d);
  if ((e = allow_smem(r_bwd_simt<T, TG, 128>, r_bwd_smem_bytes(kMaxB2, 128))) != cudaSuccess ||
      (e = allow_smem(r_bwd_simt<T, TG, 64>, r_bwd_smem_bytes(kMaxB2, 64))) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(r_bwd)");
  launch(MONARCH_PHASE_R_STEP, st, [&] {
    r_step_simt<T><<<dim3(g.b1k, g.BH), 128, r_smem, st>>>(q, k, v, w, g, QT_IDENTITY, 1);
  });
  if (g.d == 128) launch_l_bwd<T, TG, 128>(g, q, dy, w, bw, st);
  else launch_l_bwd<T, TG, 64>(g, q, dy, w, bw, st);
  launch(MONARCH_PHASE_BWD_R, st, [&] {
    if (g.d == 128) r_bwd_simt<T, TG, 128><<<dim3(g.b1k, g.BH), 256, rb_smem, st>>>(q, k, v, dq, dk, dv, bw, g);
    else r_bwd_simt<T, TG, 64><<<dim3(g.b1k, g.BH), 256, rb_smem, st>>>(q, k, v, dq, dk, dv, bw, g);
  });
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MONARCH_OK;
}

// Tensor-core backward (bf16 / f16 inputs): the forward's R step and output
// pass recompute k~, z, h, y and the row LSE; dy becomes scaled f16
// hi/lo planes with D = sigma dy . y; the two tensor-core L-step kernels give
// dk~, dz, dh and the L-step dq; the per-tile R-step backward finishes.
// saved_out / saved_lse: the output (f32) and row LSE written by the one-step
// training forward; when given, the output pass is not recomputed.
template <typename TQ, typename TG, int D>
int run_bwd_tc(const BwdPlan& bp, const TQ* q, const TQ* k, const TQ* v, const TG* dy, TG* dq, TG* dk, TG* dv,
               char* ws, cudaStream_t st, const float* saved_out = nullptr, const float* saved_lse = nullptr) {
  const Plan& p = bp.fwd;
  const Geo& g = p.g;
  const bool saved = saved_out != nullptr;
  Work w;
  w.kt = reinterpret_cast<float*>(ws + p.off[0]);
  w.z = reinterpret_cast<float*>(ws + p.off[1]);
  w.qt = reinterpret_cast<float*>(ws + p.off[2]);
  w.h = reinterpret_cast<float*>(ws + p.off[3]);
  w.lse = saved ? const_cast<float*>(saved_lse) : reinterpret_cast<float*>(ws + p.off[4]);   // read only when saved
  w.qbar = reinterpret_cast<float*>(ws + p.off[5]);
  w.qb = ws + p.off[6];
  const float* y = saved ? saved_out : reinterpret_cast<const float*>(ws + bp.toff[0]);
  __half* dyp = reinterpret_cast<__half*>(ws + bp.toff[1]);
  float* ddv = reinterpret_cast<float*>(ws + bp.toff[2]);
  unsigned* amax = reinterpret_cast<unsigned*>(ws + bp.toff[3]);
  BwdWork bw;
  bw.dd = ddv;
  bw.dqL = reinterpret_cast<float*>(ws + bp.toff[4]);
  bw.dkt = reinterpret_cast<float*>(ws + bp.toff[5]);
  bw.dz = reinterpret_cast<float*>(ws + bp.toff[6]);
  bw.dh = reinterpret_cast<float*>(ws + bp.toff[7]);

  TcPlanes<TQ> planes;
  tc::Maps maps;
  RtcMaps rmaps;
  int rc;
  const int r_group = r_step_group(g, sm_count_of_device());
  if ((rc = tc_prepare<TQ, D>(g, q, k, v, w, planes, maps, rmaps, r_group))) return rc;
  tcb::BwdMaps bmaps;
  {
    const cuuint64_t rows = (cuuint64_t)g.BH * g.b2;
    cuuint32_t box3[3] = {64, 64, 1};
    cuuint64_t dy3[3] = {(cuuint64_t)D, (cuuint64_t)g.b1q, 2 * rows};
    cuuint64_t sy3[2] = {(cuuint64_t)D * 2, (cuuint64_t)g.b1q * D * 2};
    cuuint32_t box2[2] = {64, 1};
    cuuint64_t dd2[2] = {(cuuint64_t)g.b1q_pad, rows};
    cuuint64_t sd2[1] = {(cuuint64_t)g.b1q_pad * 4};
    if ((rc = make_map(&bmaps.dy, dyp, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dy3, sy3, box3,
                       CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (rc = make_map(&bmaps.dd, ddv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dd2, sd2, box2,
                       CU_TENSOR_MAP_SWIZZLE_NONE)))
      return rc;
  }
  constexpr size_t smem_out = tc::row_smem<D, true>();
  constexpr size_t smem_r = rtc_smem<D>();
  constexpr size_t smem_kv = tcb::kv_smem<D>();
  constexpr size_t smem_q = tcb::q_smem<D>();
  static_assert(smem_kv <= (size_t)tc::kMaxSmem && smem_q <= (size_t)tc::kMaxSmem, "backward shared memory");
  const size_t rb_smem = r_bwd_smem_bytes(g.b2, D);
  static std::atomic<bool> attrs_set[kMaxDevices];
  {
    const cudaError_t e = once_per_device(attrs_set, [&] {
      cudaError_t r;
      if ((r = allow_smem(tc::l_row<__half, float, D, true, true>, smem_out)) != cudaSuccess ||
          (r = allow_smem(r_step_tc5<TQ, D>, smem_r)) != cudaSuccess ||
          (r = allow_smem(tcb::l_bwd_kv<D>, smem_kv)) != cudaSuccess ||
          (r = allow_smem(tcb::l_bwd_q<D>, smem_q)) != cudaSuccess ||
          (r = allow_smem(r_bwd_simt<TQ, TG, D>, r_bwd_smem_bytes(kMaxB2, D))) != cudaSuccess)
        return r;
      return cudaSuccess;
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  }
  const dim3 grid_q((g.b1q + 2 * kTile - 1) / (2 * kTile), g.b2, g.BH);
  const dim3 grid_r((g.b1k + r_group - 1) / r_group, g.BH);
  launch(MONARCH_PHASE_R_STEP, st, [&] {
    launch_pdl(r_step_tc5<TQ, D>, grid_r, dim3(kRtcThreads), smem_r, st, rmaps, q, w, planes, g, (int)QT_IDENTITY, 1,
               r_group);
  });
  // the output pass gives y and the row LSE of the same (hi + lo) scores
  if (!saved)
    launch(MONARCH_PHASE_L_OUT, st, [&] {
      launch_pdl(tc::l_row<__half, float, D, true, true>, grid_q, dim3(tc::kThreads), smem_out, st,
                 const_cast<float*>(y), maps, w.lse, g);
    });
  cudaError_t e = cudaMemsetAsync(amax, 0, (size_t)g.BH * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  launch(MONARCH_PHASE_BWD_PREP, st, [&] {
    // about 8 blocks of 256 threads per SM over all heads, each striding through its head
    const long long n = g.Nq * D;
    const long long per_head = std::max<long long>(1, std::min<long long>((n + 4095) / 4096,
                                                                         (8LL * sm_count_of_device() + g.BH - 1) / g.BH));
    tcb::dy_amax<TG><<<dim3((unsigned)per_head, g.BH), 256, 0, st>>>(dy, amax, g);
  });
  launch(MONARCH_PHASE_BWD_PREP, st, [&] {
    tcb::dy_planes<TG, D><<<dim3((unsigned)((g.Nq + 7) / 8), g.BH), 256, 0, st>>>(dy, y, amax, dyp, ddv, g);
  });
  launch(MONARCH_PHASE_BWD_DKV, st, [&] {
    launch_pdl(tcb::l_bwd_kv<D>, dim3((g.b1k + tcb::kBlk - 1) / tcb::kBlk, g.b2, g.BH), dim3(tcb::kThreads), smem_kv,
               st, maps, bmaps, (const float*)w.h, (const unsigned*)amax, bw.dkt, bw.dz, bw.dh, g);
  });
  launch(MONARCH_PHASE_BWD_DQ, st, [&] {
    launch_pdl(tcb::l_bwd_q<D>, dim3((g.b1q + tcb::kBlk - 1) / tcb::kBlk, g.b2, g.BH), dim3(tcb::kThreads), smem_q,
               st, maps, bmaps, (const float*)w.lse, (const float*)ddv, (const unsigned*)amax, bw.dqL, g);
  });
  launch(MONARCH_PHASE_BWD_R, st, [&] {
    r_bwd_simt<TQ, TG, D><<<dim3(g.b1k, g.BH), 256, rb_smem, st>>>(q, k, v, dq, dk, dv, bw, g);
  });
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MONARCH_OK;
}

// One-step training forward (bf16 / f16): the R step, then the output pass
// writing the f32 output and the row LSE that monarch_attn_bwd_saved reads.
template <typename TQ, int D>
int run_fwd_train_tc(const Plan& p, const TQ* q, const TQ* k, const TQ* v, float* out, float* lse, char* ws,
                     cudaStream_t st) {
  const Geo& g = p.g;
  Work w;
  w.kt = reinterpret_cast<float*>(ws + p.off[0]);
  w.z = reinterpret_cast<float*>(ws + p.off[1]);
  w.qt = reinterpret_cast<float*>(ws + p.off[2]);
  w.h = reinterpret_cast<float*>(ws + p.off[3]);
  w.lse = lse;
  w.qbar = reinterpret_cast<float*>(ws + p.off[5]);
  w.qb = ws + p.off[6];
  TcPlanes<TQ> planes;
  tc::Maps maps;
  RtcMaps rmaps;
  int rc;
  const int r_group = r_step_group(g, sm_count_of_device());
  if ((rc = tc_prepare<TQ, D>(g, q, k, v, w, planes, maps, rmaps, r_group))) return rc;
  constexpr size_t smem_out = tc::row_smem<D, true>();
  constexpr size_t smem_r = rtc_smem<D>();
  static std::atomic<bool> attrs_set[kMaxDevices];
  {
    const cudaError_t e = once_per_device(attrs_set, [&] {
      cudaError_t r;
      if ((r = allow_smem(tc::l_row<__half, float, D, true, true>, smem_out)) != cudaSuccess ||
          (r = allow_smem(r_step_tc5<TQ, D>, smem_r)) != cudaSuccess)
        return r;
      return cudaSuccess;
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  }
  const dim3 grid_q((g.b1q + 2 * kTile - 1) / (2 * kTile), g.b2, g.BH);
  const dim3 grid_r((g.b1k + r_group - 1) / r_group, g.BH);
  launch(MONARCH_PHASE_R_STEP, st, [&] {
    launch_pdl(r_step_tc5<TQ, D>, grid_r, dim3(kRtcThreads), smem_r, st, rmaps, q, w, planes, g, (int)QT_IDENTITY, 1,
               r_group);
  });
  launch(MONARCH_PHASE_L_OUT, st, [&] {
    launch_pdl(tc::l_row<__half, float, D, true, true>, grid_q, dim3(tc::kThreads), smem_out, st, out, maps, lse, g);
  });
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MONARCH_OK;
}

// Saved-state backward: the bf16 / f16 tensor-core path with y and the LSE
// from monarch_attn_fwd_train.
template <typename T>
int dispatch_bwd_saved(const BwdPlan& bp, const void* q, const void* k, const void* v, const float* out,
                       const float* lse, const void* dy, void* dq, void* dk, void* dv, char* ws, cudaStream_t st) {
  const T *qq = (const T*)q, *kk = (const T*)k, *vv = (const T*)v;
  if (bp.fwd.g.d == 128) {
    if (bp.grad_dtype == MONARCH_F32)
      return run_bwd_tc<T, float, 128>(bp, qq, kk, vv, (const float*)dy, (float*)dq, (float*)dk, (float*)dv, ws, st,
                                       out, lse);
    return run_bwd_tc<T, T, 128>(bp, qq, kk, vv, (const T*)dy, (T*)dq, (T*)dk, (T*)dv, ws, st, out, lse);
  }
  if (bp.grad_dtype == MONARCH_F32)
    return run_bwd_tc<T, float, 64>(bp, qq, kk, vv, (const float*)dy, (float*)dq, (float*)dk, (float*)dv, ws, st,
                                    out, lse);
  return run_bwd_tc<T, T, 64>(bp, qq, kk, vv, (const T*)dy, (T*)dq, (T*)dk, (T*)dv, ws, st, out, lse);
}

template <typename T>
int dispatch_bwd_grad(const BwdPlan& bp, const void* q, const void* k, const void* v, const void* dy, void* dq,
                      void* dk, void* dv, char* ws, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {
    if (bp.fwd.g.d == 128) {
      if (bp.grad_dtype == MONARCH_F32)
        return run_bwd_tc<T, float, 128>(bp, (const T*)q, (const T*)k, (const T*)v, (const float*)dy, (float*)dq,
                                         (float*)dk, (float*)dv, ws, st);
      return run_bwd_tc<T, T, 128>(bp, (const T*)q, (const T*)k, (const T*)v, (const T*)dy, (T*)dq, (T*)dk, (T*)dv,
                                   ws, st);
    }
    if (bp.grad_dtype == MONARCH_F32)
      return run_bwd_tc<T, float, 64>(bp, (const T*)q, (const T*)k, (const T*)v, (const float*)dy, (float*)dq,
                                      (float*)dk, (float*)dv, ws, st);
    return run_bwd_tc<T, T, 64>(bp, (const T*)q, (const T*)k, (const T*)v, (const T*)dy, (T*)dq, (T*)dk, (T*)dv, ws,
                                st);
  } else {
    if (bp.grad_dtype == MONARCH_F32)
      return run_bwd<T, float>(bp, (const T*)q, (const T*)k, (const T*)v, (const float*)dy, (float*)dq, (float*)dk,
                               (float*)dv, ws, st);
    return run_bwd<T, T>(bp, (const T*)q, (const T*)k, (const T*)v, (const T*)dy, (T*)dq, (T*)dk, (T*)dv, ws, st);
  }
}

int dispatch_bwd(const BwdPlan& bp, const void* q, const void* k, const void* v, const void* dy, void* dq,
                 void* dk, void* dv, void* ws, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  switch (bp.fwd.dtype) {
    case MONARCH_F32: return dispatch_bwd_grad<float>(bp, q, k, v, dy, dq, dk, dv, w, st);
    case MONARCH_BF16: return dispatch_bwd_grad<__nv_bfloat16>(bp, q, k, v, dy, dq, dk, dv, w, st);
    default: return dispatch_bwd_grad<__half>(bp, q, k, v, dy, dq, dk, dv, w, st);
  }
}

// Stream-ordered workspace comes from a per-device pool owned by the library
// that keeps freed memory (release threshold = max), so repeated calls reuse
// it without returning memory to the driver between calls.
int workspace_pool(cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MONARCH_EUNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess)
      return cuda_fail(e, "cudaMemPoolSetAttribute");
    pools[dev] = pool;
  }
  *out = pools[dev];
  return MONARCH_OK;
}

// Copy streams of the host-buffer entry point, one pair per device, created
// on first use (non-blocking) and kept for the life of the process.
constexpr int kHostGroups = 16;  // most groups one host-buffer call splits its units into

// Unit counts of the groups of a host-buffer call.  Groups hold about 10 MB
// of input each (at most 8 of them; one group below 10 MB).  With two or more,
// the first and the last groups ramp (1, 2, 4, 8 units while smaller than the
// others): the copy-out starts sooner, runs beside more of the copy-in, and
// the forward and copy-out of the last group, which nothing overlaps, are
// short.  Measured on B200 (full_32760, 24 heads): 1, 2, 3 x 6, 2, 1 took
// 14.4 ms against 15.0 ms for 3 x 8; the 4680-token grid is bound by the host
// link either way.
int host_groups(long long U, long long in_bytes, long long* sizes) {
  int ng = (int)std::max<long long>(1, std::min<long long>({in_bytes / (10LL << 20), U, 8LL}));
  const long long gs = (U + ng - 1) / ng;
  ng = (int)((U + gs - 1) / gs);
  if (ng == 1) {
    sizes[0] = U;
    return 1;
  }
  long long ramp[4];
  int nr = 0;
  long long left = U;
  for (long long r = 1; r < gs && nr < 4 && left >= 2 * r + gs; r *= 2) {
    ramp[nr++] = r;
    left -= 2 * r;
  }
  int n = 0;
  for (int i = 0; i < nr; ++i) sizes[n++] = ramp[i];
  while (left > 0) {
    const long long t = std::min(gs, left);
    sizes[n++] = t;
    left -= t;
  }
  for (int i = nr - 1; i >= 0; --i) sizes[n++] = ramp[i];
  return n;
}

struct HostStreams {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev[2 * kHostGroups + 3] = {};   // per group: inputs landed, forward done; + 3
};

// One host-buffer call at a time per device: the call holds this lock until
// its copies are done, since the events above are shared.
std::mutex g_host_call_mu[kMaxDevices];

int host_streams(HostStreams* hs, int* dev_out) {
  static std::mutex mu;
  static HostStreams per_dev[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MONARCH_EUNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  HostStreams& s = per_dev[dev];
  if (!s.in) {
    HostStreams n;
    bool good = cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& x : n.ev) good = good && cudaEventCreateWithFlags(&x, cudaEventDisableTiming) == cudaSuccess;
    if (!good) {
      e = cudaGetLastError();
      if (n.in) cudaStreamDestroy(n.in);
      if (n.out) cudaStreamDestroy(n.out);
      for (auto& x : n.ev)
        if (x) cudaEventDestroy(x);
      return cuda_fail(e, "creating the copy streams");
    }
    s = n;
  }
  *hs = s;
  *dev_out = dev;
  return MONARCH_OK;
}

int check_io(const void* q, const void* k, const void* v, const void* out) {
  int rc;
  if ((rc = check_ptr(q, "q")) || (rc = check_ptr(k, "k")) || (rc = check_ptr(v, "v")) ||
      (rc = check_ptr(out, "out")))
    return rc;
  return MONARCH_OK;
}

}  // namespace

extern "C" {

int monarch_attn_version(void) { return 103; }

unsigned long long monarch_attn_launch_count(void) { return g_launches.load(); }

int monarch_attn_device_error(int reset) { return read_device_error(reset); }

int monarch_attn_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.on = on != 0;
  return MONARCH_OK;
}

int monarch_attn_profile_read(double* ms, unsigned long long* launches, int n, int reset) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  int rc = MONARCH_OK;
  for (auto& r : g_prof.pending) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess && rc == MONARCH_OK) rc = cuda_fail(e, "profile events");
    g_prof.ms[r.phase] += t;
    g_prof.n[r.phase] += 1;
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.pending.clear();
  for (int p = 0; p < n && p < MONARCH_NUM_PHASES; ++p) {
    if (ms) ms[p] = g_prof.ms[p];
    if (launches) launches[p] = g_prof.n[p];
  }
  if (reset)
    for (int p = 0; p < MONARCH_NUM_PHASES; ++p) g_prof.ms[p] = 0, g_prof.n[p] = 0;
  return rc;
}

const char* monarch_attn_last_error(void) { return g_err.c_str(); }

size_t monarch_attn_workspace_layout(int B, int heads, int T, int H, int W, int d, int tile_h,
                                     int tile_w, int iters, long kv_len, int dtype,
                                     size_t offsets[7]) {
  Plan p;
  if (make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, dtype, &p) != MONARCH_OK) return 0;
  if (offsets)
    for (int i = 0; i < kRegions; ++i) offsets[i] = p.off[i];
  return p.total;
}

size_t monarch_attn_workspace_bytes(int B, int heads, int T, int H, int W, int d, int tile_h,
                                    int tile_w, int iters, long kv_len, int dtype) {
  return monarch_attn_workspace_layout(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype,
                                       nullptr);
}

int monarch_attn_fwd_ws(const void* q, const void* k, const void* v, void* out, int B, int heads,
                        int T, int H, int W, int d, int tile_h, int tile_w, int iters, long kv_len,
                        int dtype, int out_dtype, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &p);
  if (rc) return rc;
  if ((rc = check_io(q, k, v, out))) return rc;
  if ((rc = check_ptr(workspace, "workspace"))) return rc;
  if (workspace_bytes < p.total)
    return fail(MONARCH_ENOMEM, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes, p.total);
  return dispatch(p, q, k, v, out, workspace, stream);
}

int monarch_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int heads,
                     int T, int H, int W, int d, int tile_h, int tile_w, int iters, long kv_len,
                     int dtype, int out_dtype, cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &p);
  if (rc) return rc;
  if ((rc = check_io(q, k, v, out))) return rc;
  void* ws = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, p.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", p.total, cudaGetErrorString(e));
  }
  rc = dispatch(p, q, k, v, out, ws, stream);
  e = cudaFreeAsync(ws, stream);
  if (rc == MONARCH_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

int monarch_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int heads,
                        int T, int H, int W, int d, int tile_h, int tile_w, int iters, long kv_len,
                        int chunk_frames, int dtype, int out_dtype, cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &p, chunk_frames);
  if (rc) return rc;
  if ((rc = check_io(q, k, v, out))) return rc;
  void* ws = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, p.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", p.total, cudaGetErrorString(e));
  }
  rc = dispatch(p, q, k, v, out, ws, stream);
  e = cudaFreeAsync(ws, stream);
  if (rc == MONARCH_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

size_t monarch_attn_bwd_workspace_bytes(int B, int heads, int T, int H, int W, int d, int tile_h, int tile_w,
                                        int chunk_frames, int dtype, int grad_dtype) {
  BwdPlan bp;
  if (make_bwd_plan(B, heads, T, H, W, d, tile_h, tile_w, chunk_frames, dtype, grad_dtype, &bp) != MONARCH_OK)
    return 0;
  return bp.total;
}

int monarch_attn_bwd(const void* q, const void* k, const void* v, const void* dy, void* dq, void* dk, void* dv,
                     int B, int heads, int T, int H, int W, int d, int tile_h, int tile_w, int chunk_frames,
                     int dtype, int grad_dtype, cudaStream_t stream) {
  g_err.clear();
  BwdPlan bp;
  int rc = make_bwd_plan(B, heads, T, H, W, d, tile_h, tile_w, chunk_frames, dtype, grad_dtype, &bp);
  if (rc) return rc;
  if ((rc = check_ptr(q, "q")) || (rc = check_ptr(k, "k")) || (rc = check_ptr(v, "v")) ||
      (rc = check_ptr(dy, "dy")) || (rc = check_ptr(dq, "dq")) || (rc = check_ptr(dk, "dk")) ||
      (rc = check_ptr(dv, "dv")))
    return rc;
  void* ws = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bp.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", bp.total, cudaGetErrorString(e));
  }
  rc = dispatch_bwd(bp, q, k, v, dy, dq, dk, dv, ws, stream);
  e = cudaFreeAsync(ws, stream);
  if (rc == MONARCH_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

size_t monarch_attn_lse_bytes(int B, int heads, int T, int H, int W, int d, int tile_h, int tile_w) {
  Plan p;
  if (make_plan(B, heads, T, H, W, d, tile_h, tile_w, 1, (long)T * H * W, MONARCH_BF16, MONARCH_BF16, &p) != MONARCH_OK)
    return 0;
  return (size_t)p.g.BH * p.g.b2 * p.g.b1q_pad * 4;
}

int monarch_attn_fwd_train(const void* q, const void* k, const void* v, float* out, float* lse, int B, int heads,
                           int T, int H, int W, int d, int tile_h, int tile_w, int chunk_frames, int dtype,
                           cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, 1, (long)T * H * W, dtype, MONARCH_F32, &p, chunk_frames);
  if (rc) return rc;
  if (dtype == MONARCH_F32)
    return fail(MONARCH_EUNSUPPORTED, "the saved-state training pair is for bf16 / f16 inputs (f32: monarch_attn_bwd)");
  if ((rc = check_io(q, k, v, out)) || (rc = check_ptr(lse, "lse"))) return rc;
  void* ws = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, p.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", p.total, cudaGetErrorString(e));
  }
  char* w = static_cast<char*>(ws);
  if (dtype == MONARCH_BF16)
    rc = d == 128 ? run_fwd_train_tc<__nv_bfloat16, 128>(p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                          (const __nv_bfloat16*)v, out, lse, w, stream)
                  : run_fwd_train_tc<__nv_bfloat16, 64>(p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                         (const __nv_bfloat16*)v, out, lse, w, stream);
  else
    rc = d == 128 ? run_fwd_train_tc<__half, 128>(p, (const __half*)q, (const __half*)k, (const __half*)v, out, lse, w,
                                                   stream)
                  : run_fwd_train_tc<__half, 64>(p, (const __half*)q, (const __half*)k, (const __half*)v, out, lse, w,
                                                  stream);
  e = cudaFreeAsync(ws, stream);
  if (rc == MONARCH_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

int monarch_attn_bwd_saved(const void* q, const void* k, const void* v, const float* out, const float* lse,
                           const void* dy, void* dq, void* dk, void* dv, int B, int heads, int T, int H, int W, int d,
                           int tile_h, int tile_w, int chunk_frames, int dtype, int grad_dtype, cudaStream_t stream) {
  g_err.clear();
  BwdPlan bp;
  int rc = make_bwd_plan(B, heads, T, H, W, d, tile_h, tile_w, chunk_frames, dtype, grad_dtype, &bp);
  if (rc) return rc;
  if (dtype == MONARCH_F32)
    return fail(MONARCH_EUNSUPPORTED, "the saved-state training pair is for bf16 / f16 inputs (f32: monarch_attn_bwd)");
  if ((rc = check_ptr(q, "q")) || (rc = check_ptr(k, "k")) || (rc = check_ptr(v, "v")) ||
      (rc = check_ptr(out, "out")) || (rc = check_ptr(lse, "lse")) || (rc = check_ptr(dy, "dy")) ||
      (rc = check_ptr(dq, "dq")) || (rc = check_ptr(dk, "dk")) || (rc = check_ptr(dv, "dv")))
    return rc;
  void* ws = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bp.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", bp.total, cudaGetErrorString(e));
  }
  char* w = static_cast<char*>(ws);
  rc = dtype == MONARCH_BF16
           ? dispatch_bwd_saved<__nv_bfloat16>(bp, q, k, v, out, lse, dy, dq, dk, dv, w, stream)
           : dispatch_bwd_saved<__half>(bp, q, k, v, out, lse, dy, dq, dk, dv, w, stream);
  e = cudaFreeAsync(ws, stream);
  if (rc == MONARCH_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

int monarch_attn_fwd_host_ex(const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, int B, int heads, int T, int H, int W, int d,
                             int tile_h, int tile_w, int iters, long kv_len, int chunk_frames, int dtype,
                             int out_dtype, cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &p, chunk_frames);
  if (rc) return rc;
  if (!q_host || !k_host || !v_host || !out_host) return fail(MONARCH_EINVAL, "null host pointer");
  HostStreams hs;
  int dev = 0;
  if ((rc = host_streams(&hs, &dev))) return rc;
  std::lock_guard<std::mutex> call_lock(g_host_call_mu[dev]);
  // (batch, head) units are independent: split them into groups whose copies
  // in, compute and copies out overlap (copies in on hs.in, the forward on
  // `stream`, copies out on hs.out, ordered by events per group)
  const long long U = p.g.BH;
  const size_t es = elem_size(dtype), eo = elem_size(out_dtype);
  const size_t qu = (size_t)p.g.Nq * d * es, ku = (size_t)p.g.Nk * d * es, ou = (size_t)p.g.Nq * d * eo;
  const long long in_bytes = (long long)(U * (qu + 2 * ku));
  long long sizes[kHostGroups], starts[kHostGroups];
  const int ng = host_groups(U, in_bytes, sizes);
  for (int i = 0; i < ng; ++i) starts[i] = i ? starts[i - 1] + sizes[i - 1] : 0;
  const long long gs = *std::max_element(sizes, sizes + ng);
  Plan pg;   // the largest group (B = 1, heads = gs): its workspace serves every group
  if ((rc = make_plan(1, (int)gs, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &pg, chunk_frames)))
    return rc;
  pg.r_group = r_step_group(p.g, sm_count_of_device());
  const size_t oq = 0, ok = align256(U * qu), ov = ok + align256(U * ku), oo = ov + align256(U * ku);
  const size_t ow = oo + align256(U * ou);
  char* buf = nullptr;
  cudaMemPool_t pool;
  if ((rc = workspace_pool(&pool))) return rc;
  cudaError_t e = cudaMallocFromPoolAsync((void**)&buf, ow + pg.total, pool, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MONARCH_ENOMEM, "cudaMallocFromPoolAsync(%zu): %s", ow + pg.total, cudaGetErrorString(e));
  }
  cudaEvent_t* ev = hs.ev;   // the device's events (this call holds its lock)
  cudaEvent_t ev_alloc = ev[2 * kHostGroups], ev_in_done = ev[2 * kHostGroups + 1], ev_out_done = ev[2 * kHostGroups + 2];
  {
    cudaEventRecord(ev_alloc, stream);
    cudaStreamWaitEvent(hs.in, ev_alloc, 0);
    for (int gi = 0; gi < ng && rc == MONARCH_OK; ++gi) {
      const long long u0 = starts[gi], n = sizes[gi];
      const char* qh = static_cast<const char*>(q_host);
      const char* kh = static_cast<const char*>(k_host);
      const char* vh = static_cast<const char*>(v_host);
      if ((e = cudaMemcpyAsync(buf + oq + u0 * qu, qh + u0 * qu, n * qu, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(buf + ok + u0 * ku, kh + u0 * ku, n * ku, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(buf + ov + u0 * ku, vh + u0 * ku, n * ku, cudaMemcpyHostToDevice, hs.in)) != cudaSuccess)
        rc = cuda_fail(e, "cudaMemcpyAsync(host->device)");
      cudaEventRecord(ev[gi], hs.in);
    }
    for (int gi = 0; gi < ng && rc == MONARCH_OK; ++gi) {
      const long long u0 = starts[gi], n = sizes[gi];
      Plan pn = pg;
      if (n != gs &&
          (rc = make_plan(1, (int)n, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &pn, chunk_frames)))
        break;
      pn.r_group = pg.r_group;
      cudaStreamWaitEvent(stream, ev[gi], 0);
      rc = dispatch(pn, buf + oq + u0 * qu, buf + ok + u0 * ku, buf + ov + u0 * ku, buf + oo + u0 * ou, buf + ow,
                    stream);
      cudaEventRecord(ev[ng + gi], stream);
      cudaStreamWaitEvent(hs.out, ev[ng + gi], 0);
      if (rc == MONARCH_OK &&
          (e = cudaMemcpyAsync(static_cast<char*>(out_host) + u0 * ou, buf + oo + u0 * ou, n * ou,
                               cudaMemcpyDeviceToHost, hs.out)) != cudaSuccess)
        rc = cuda_fail(e, "cudaMemcpyAsync(device->host)");
    }
    // the caller's stream waits for every copy, then frees the buffers
    cudaEventRecord(ev_in_done, hs.in);
    cudaStreamWaitEvent(stream, ev_in_done, 0);
    cudaEventRecord(ev_out_done, hs.out);
    cudaStreamWaitEvent(stream, ev_out_done, 0);
  }
  cudaFreeAsync(buf, stream);
  e = cudaStreamSynchronize(stream);
  if (rc == MONARCH_OK && e != cudaSuccess) rc = cuda_fail(e, "cudaStreamSynchronize");
  return rc;
}

int monarch_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                          void* out_host, int B, int heads, int T, int H, int W, int d,
                          int tile_h, int tile_w, int iters, long kv_len, int dtype,
                          int out_dtype, cudaStream_t stream) {
  return monarch_attn_fwd_host_ex(q_host, k_host, v_host, out_host, B, heads, T, H, W, d, tile_h, tile_w, iters,
                                  kv_len, 0, dtype, out_dtype, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward.  Some callers cannot allocate device memory once
// they are running: a real-time generation loop that must not stall or fail
// on an allocation mid-stream, or a host application that owns every byte of
// device memory and forbids allocations from plug-ins.  This entry point takes
// its workspace from a fixed array in device memory that exists as soon as the
// library is loaded on a device (and stays until the process exits), so it
// never calls cudaMalloc, cudaMallocAsync or cudaFree.
constexpr size_t kNoAllocScratchBytes = size_t(128) << 20;  // 128 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device, with that device current, and cached.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MONARCH_EUNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MONARCH_OK;
}
}  // namespace

extern "C" int monarch_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                                        int heads, int T, int H, int W, int d, int tile_h, int tile_w,
                                        int iters, long kv_len, int dtype, int out_dtype, cudaStream_t stream) {
  g_err.clear();
  Plan p;
  int rc = make_plan(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype, out_dtype, &p);
  if (rc) return rc;
  if ((rc = check_io(q, k, v, out))) return rc;
  if (p.total > kNoAllocScratchBytes)
    return fail(MONARCH_ENOMEM,
                "problem needs %zu bytes of workspace; the allocation-free entry point has a fixed %zu-byte "
                "scratch array (use monarch_attn_fwd or monarch_attn_fwd_ws)",
                p.total, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  return dispatch(p, q, k, v, out, scratch, stream);
}
