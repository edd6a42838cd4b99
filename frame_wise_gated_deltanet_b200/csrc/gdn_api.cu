// Host side of the C ABI declared in include/gdn.h: argument validation, the cached per-GPU
// workspace, TMA descriptor encoding and kernel launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/gdn.h"
#include "bwd_chain_kernel.cuh"
#include "bwd_frame_kernel.cuh"
#include "bwd_token_kernel.cuh"
#include "chain_kernel.cuh"
#include "common.cuh"
#include "fused_kernel.cuh"
#include "la_scan_kernel.cuh"
#include "output_kernel.cuh"
#include "rope_kernel.cuh"
#include "scan_kernel.cuh"
#include "softmax_kernel.cuh"
#include "stats_kernel.cuh"
#include "step_kernel.cuh"

// Scratch of gdn_frame_forward_noalloc: a fixed 64 MiB array in device memory, reserved by the
// CUDA module on every GPU that loads this library and held until the process exits. Host code
// only sees a stand-in symbol; the device address comes from cudaGetSymbolAddress.
static constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

using gdn::Problem;

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------------ driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tiled map (dims[0] contiguous) with 128B swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
               const cuuint64_t* dims, const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims,
                  strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// q/k/v [B, T, N, H, D] bf16 -> 4-D map (D, H, N, B*T), box 64 x 1 x 128 x 1.
bool tmap_tokens(CUtensorMap* m, const void* base, const Problem& p) {
  const cuuint64_t dims[4] = {(cuuint64_t)p.D, (cuuint64_t)p.H, (cuuint64_t)p.N,
                              (cuuint64_t)p.B * p.T};
  const cuuint64_t strides[3] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.H * p.D * 2,
                                 (cuuint64_t)p.N * p.H * p.D * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box);
}

// e4m3 q/k/v [B, T, N, H, D] bytes -> 4-D map (D, H, N, B*T), box 128 x 1 x 128 x 1 (one
// 128-byte swizzled row of 128 dims per token; dims past D read as zero). D % 16 == 0.
bool tmap_tokens_f8(CUtensorMap* m, const void* base, const Problem& p) {
  const cuuint64_t dims[4] = {(cuuint64_t)p.D, (cuuint64_t)p.H, (cuuint64_t)p.N,
                              (cuuint64_t)p.B * p.T};
  const cuuint64_t strides[3] = {(cuuint64_t)p.D, (cuuint64_t)p.H * p.D,
                                 (cuuint64_t)p.N * p.H * p.D};
  const cuuint32_t box[4] = {128, 1, 128, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box);
}

// q/k/v/out [B, T, N, H, D] bf16 as flattened token rows -> 3-D map (D, H, B*T*N), box
// 64 x 1 x 128 (block-causal LA: a block's frames are consecutive rows).
bool tmap_rows(CUtensorMap* m, const void* base, const Problem& p) {
  const cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.H, (cuuint64_t)p.B * p.T * p.N};
  const cuuint64_t strides[2] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.H * p.D * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box);
}

// q/k/v/out [B, T, N, H, D] bf16 as (D, H, T*N, B): a clip's tokens as one row axis, so tiles
// span frames and rows past the clip read as zero and are not stored (softmax attention).
bool tmap_clip(CUtensorMap* m, const void* base, int B, int H, int L, int D) {
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                                 (cuuint64_t)L * H * D * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box);
}

// Token map of q, k or v in the element type of the path.
template <bool kF8>
bool tmap_in(CUtensorMap* m, const void* base, const Problem& p) {
  return kF8 ? tmap_tokens_f8(m, base, p) : tmap_tokens(m, base, p);
}

// [count, rows, D] matrices (bf16 or f32) -> 3-D map (D, rows, count), box (128 B) x DP x 1.
bool tmap_mats(CUtensorMap* m, const void* base, bool f32, int D, int rows, long count, int DP) {
  const int es = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)count};
  const cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)rows * D * es};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / es), (cuuint32_t)DP, 1};
  return make_tmap(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   base, dims, strides, box);
}

// ------------------------------------------------------------------ device info / workspace
constexpr int kMaxSegEvents = 64;  // chain segments of the backward with saved states (events)

struct DeviceState {
  int sms = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  uint64_t attr_done = 0;  // bit per kernel instantiation whose smem attribute is set
  int* step_flags = nullptr;  // hand-off words of the step kernel (persist across launches)
  long step_items = 0;
  int step_epoch = 0;
  // second stream of the backward (work that overlaps the state chains) and its fork/join events
  cudaStream_t aux = nullptr;
  // (and one per chain segment of the backward with saved states)
  cudaEvent_t ev[5 + kMaxSegEvents] = {};
  // (cos, sin) table of gdn_frame_forward_rope (kept apart from the forward's workspace)
  float2* rope_tab = nullptr;
  size_t rope_tab_bytes = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

int env_int(const char* name, int dflt, int lo, int hi);

gdn_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return GDN_ERR_CUDA;
  DeviceState& d = g_dev[*dev];
  if (d.sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return GDN_ERR_CUDA;
    // GDN_WAIT_LIMIT_MS: limit of the kernels' bounded waits (default 4000 ms)
    const int ms = env_int("GDN_WAIT_LIMIT_MS", 4000, 1, 60000);
    if (ms != 4000) {
      const unsigned long long ns = static_cast<unsigned long long>(ms) * 1000000ull;
      if (cudaMemcpyToSymbol(gdn::g_wait_limit_ns, &ns, sizeof(ns)) != cudaSuccess)
        return GDN_ERR_CUDA;
    }
    d.sms = sms;
  }
  return GDN_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// GDN_POISON_WORKSPACE=1 (testing aid, read once): every call fills the workspace bytes it will
// use with 0xFF (NaN as f32 and bf16) on its stream before its kernels run, so a kernel that reads
// workspace it did not write first produces NaN instead of a silently plausible value.
bool poison_workspace() {
  static const bool on = [] {
    const char* s = getenv("GDN_POISON_WORKSPACE");
    return s != nullptr && s[0] == '1';
  }();
  return on;
}

gdn_status poison(void* p, size_t bytes, cudaStream_t stream) {
  if (!poison_workspace() || bytes == 0) return GDN_OK;
  return cudaMemsetAsync(p, 0xFF, bytes, stream) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Grows a library-owned device buffer in stream order: the old buffer is released by
// cudaFreeAsync on `stream` (after the work already enqueued there, which includes every earlier
// call's use of it: calls on one GPU are ordered on the caller's stream) and the new one is
// taken by cudaMallocAsync from the device's default memory pool, so growing does not
// synchronise the device or other streams. Refused with GDN_ERR_NO_MEMORY while `stream` is being
// captured (the buffer outlives any graph).
gdn_status grow_buffer(void** buf, size_t* have, size_t bytes, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return GDN_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return GDN_ERR_NO_MEMORY;
  if (*buf != nullptr && cudaFreeAsync(*buf, stream) != cudaSuccess) return GDN_ERR_CUDA;
  *buf = nullptr;
  *have = 0;
  void* p = nullptr;
  if (cudaMallocAsync(&p, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_NO_MEMORY;
  }
  *buf = p;
  *have = bytes;
  return GDN_OK;
}

gdn_status get_workspace(int dev, size_t bytes, cudaStream_t stream, void** out) {
  DeviceState& d = g_dev[dev];
  if (d.ws_bytes < bytes)
    if (gdn_status s = grow_buffer(&d.ws, &d.ws_bytes, bytes, stream)) return s;
  *out = d.ws;
  return poison(d.ws, bytes, stream);
}

template <typename K>
gdn_status ensure_smem_attr(int dev, int bit, K kernel, int bytes) {
  DeviceState& d = g_dev[dev];
  if (d.attr_done & (uint64_t(1) << bit)) return GDN_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  d.attr_done |= uint64_t(1) << bit;
  return GDN_OK;
}

// ------------------------------------------------------------------ launch profiling
// When armed, every kernel launch records events[2i] before and events[2i+1] after launch i
// on the launch's stream, until the caller's array is used up.
constexpr int kMaxProfiled = 8192;
cudaEvent_t* g_prof_events = nullptr;
int g_prof_n = 0;
int g_prof_count = 0;
const char* g_prof_names[kMaxProfiled];

struct ProfiledLaunch {
  int slot = -1;
  cudaStream_t st;
  ProfiledLaunch(const char* name, cudaStream_t s) : st(s) {
    if (g_prof_events != nullptr && 2 * g_prof_count + 1 < g_prof_n &&
        g_prof_count < kMaxProfiled) {
      slot = g_prof_count++;
      g_prof_names[slot] = name;
      cudaEventRecord(g_prof_events[2 * slot], st);
    }
  }
  ~ProfiledLaunch() {
    if (slot >= 0) cudaEventRecord(g_prof_events[2 * slot + 1], st);
  }
};

// ------------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

gdn_status check_sizes(int B, int H, int T, int N, int D, int d_max) {
  if (B < 1 || H < 1 || T < 1 || N < 1 || D < 1) return GDN_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > d_max) return GDN_ERR_UNSUPPORTED;
  const double elems = double(B) * T * N * H * D;
  if (elems > 4.0e18 || double(B) * T > 2147483647.0 || double(B) * H * T > 2147483647.0)
    return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

// The key scale of a call: 0 selects the pages' 1/sqrt(D*N) (D head dim, N tokens per frame;
// gen-hub.ru SANA-WM article, "Архитектура"), any other value must be finite and > 0 and is used
// as given. Returns false for an invalid value. D and N are already validated (>= 1).
bool resolve_key_scale(float ks, int D, int N, float* out) {
  if (ks == 0.f) {
    *out = static_cast<float>(1.0 / std::sqrt(double(D) * double(N)));
    return true;
  }
  if (!(std::isfinite(ks) && ks > 0.f)) return false;
  *out = ks;
  return true;
}

gdn_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ------------------------------------------------------------------ kernel runners
// kB4: B_t in the chain's interleaved layout (forward paths) or row-major (gdn_frame_stats).
// max_ctas > 0 caps the grid (the backward runs it beside the state chain's CTAs).
template <int DP, bool kB4, bool kF8 = false, bool kRope = false>
gdn_status run_stats(int dev, const Problem& p, const void* k, const void* v, void* A, float* Bm,
                     cudaStream_t st, int max_ctas = 0) {
  using L = gdn::StatsLayout<DP, false, kF8, kRope>;
  CUtensorMap tk, tv;
  if (!tmap_in<kF8>(&tk, k, p) || !tmap_in<kF8>(&tv, v, p)) return GDN_ERR_CUDA;
  auto kern = gdn::gdn_stats_kernel<DP, false, kB4, kF8, kRope>;
  const int bit = kRope ? 40 + (DP == 128 ? 0 : 1)
                        : (kF8 ? 15 : (DP == 128 ? 0 : 1) + (kB4 ? 10 : 0));
  if (gdn_status s = ensure_smem_attr(dev, bit, kern, L::kSmemBytes)) return s;
  const long items = long(p.B) * p.T * p.H;
  const long cap = max_ctas > 0 ? max_ctas : g_dev[dev].sms;
  const int grid = static_cast<int>(items < cap ? items : cap);
  {
    ProfiledLaunch pl("gdn_stats_kernel", st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(tk, tv, static_cast<__nv_bfloat16*>(A), Bm, p,
                                                   1);
  }
  return check_launch();
}

// seg.kind 0: one CTA per (head, chunk) replaying the chunk (the plain chain when seg.nc == 1);
// seg.kind 1: a CTA pair per (head, chunk < nc - 1) composing the chunk's frame maps.
template <int DP>
gdn_status run_chain(int dev, const Problem& p, const void* A, const float* Bm,
                     const float* gamma, const float* beta, const float* s_in, void* S_ws,
                     float* s_out, const gdn::ChainSeg& seg, cudaStream_t st) {
  using L = gdn::ChainLayout<DP>;
  const long count = long(p.B) * p.H * p.T;
  CUtensorMap ta;
  if (!tmap_mats(&ta, A, false, p.D, p.D, count, DP)) return GDN_ERR_CUDA;
  auto kern = gdn::gdn_chain_kernel<DP>;
  if (gdn_status s = ensure_smem_attr(dev, DP == 128 ? 2 : 3, kern, L::kSmemBytes)) return s;
  const long bh = long(p.B) * p.H;
  const long grid = seg.kind == 0 ? bh * seg.nc : 2 * bh * (seg.nc - 1);
  if (grid < 1 || grid > 2147483647L) return GDN_ERR_INVALID_ARG;
  {
    ProfiledLaunch pl(seg.kind == 0 ? (seg.nc == 1 ? "gdn_chain_kernel" : "gdn_chain_kernel_replay")
                                    : "gdn_chain_kernel_compose",
                      st);
    kern<<<static_cast<unsigned>(grid), L::kThreads, L::kSmemBytes, st>>>(
        ta, Bm, static_cast<__nv_bfloat16*>(S_ws), gamma, beta, s_in, s_out, p, seg);
  }
  return check_launch();
}

template <int DP>
gdn_status run_scan(int dev, const Problem& p, const gdn::ChainSeg& seg, const float* s_in,
                    cudaStream_t st) {
  using L = gdn::ScanLayout<DP>;
  auto kern = gdn::gdn_scan_kernel<DP>;
  if (gdn_status s = ensure_smem_attr(dev, DP == 128 ? 13 : 14, kern, L::kSmemBytes)) return s;
  {
    ProfiledLaunch pl("gdn_scan_kernel", st);
    kern<<<p.B * p.H, L::kThreads, L::kSmemBytes, st>>>(seg.maps, seg.starts, s_in, seg.nc, p.D);
  }
  return check_launch();
}

template <int DP, bool kLA, bool kF8 = false, bool kRope = false>
gdn_status run_output(int dev, const Problem& p, const void* q, const void* S_ws, int srows,
                      void* out, int F, cudaStream_t st) {
  using L = gdn::OutputLayout<DP, kLA, 4, kF8, kRope>;
  const long count = long(p.B) * p.H * ((p.T + F - 1) / F);  // stored states (per block for LA)
  CUtensorMap tq, ts, to;
  if (kLA) {
    if (!tmap_rows(&tq, q, p) || !tmap_rows(&to, out, p)) return GDN_ERR_CUDA;
  } else if (!tmap_in<kF8>(&tq, q, p) || !tmap_tokens(&to, out, p)) {
    return GDN_ERR_CUDA;
  }
  if (kLA) {
    if (!tmap_mats(&ts, S_ws, false, p.D, srows, count, DP)) return GDN_ERR_CUDA;
  } else {
    ts = tq;  // unused: GDN states are bulk-copied from S_ws
  }
  auto kern = gdn::gdn_output_kernel<DP, kLA, kF8, kRope>;
  const int bit = kRope ? 42 + (DP == 128 ? 0 : 1) : (kF8 ? 16 : (kLA ? 6 : (DP == 128 ? 4 : 5)));
  if (gdn_status s = ensure_smem_attr(dev, bit, kern, L::kSmemBytes)) return s;
  const long items = long(p.B) * (kLA ? (p.T + F - 1) / F : p.T) * p.H;
  const int grid = static_cast<int>(items < g_dev[dev].sms ? items : g_dev[dev].sms);
  {
    ProfiledLaunch pl("gdn_output_kernel", st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(
        tq, ts, static_cast<const __nv_bfloat16*>(S_ws), to, p, F,
        static_cast<__nv_bfloat16*>(out));
  }
  return check_launch();
}

struct ForwardWs {
  void* A;
  float* B;
  void* S;
};

int padded_dim(int D) { return D <= 64 ? 64 : 128; }

// per frame-head: A_t bf16 D x D, B_t f32 D x D, S_t bf16 DP x DP (core-matrix layout)
size_t forward_ws_bytes(long count, int D) {
  const size_t m = size_t(D) * D, dp = padded_dim(D);
  return align256(count * m * 2) + align256(count * m * 4) + align256(count * dp * dp * 2);
}

ForwardWs carve_forward(void* base, long count, int D) {
  const size_t m = size_t(D) * D;
  uint8_t* p = static_cast<uint8_t*>(base);
  ForwardWs w;
  w.A = p;
  p += align256(count * m * 2);
  w.B = reinterpret_cast<float*>(p);
  p += align256(count * m * 4);
  w.S = p;
  return w;
}

// ------------------------------------------------------------------ fused forward
// 0 = choose automatically, 1 = always the three-kernel path, 2 = fused whenever it applies,
// 3 = chunked.
int g_forward_mode = 0;

// Tuning of the fused forward, read once from the environment:
//   GDN_FUSED_RING       A_t / B_t ring slots per head (default 8, 4..64)
//   GDN_FUSED_SRING      S_t ring slots per head (default 16, 8..64)
// (with the outputs' publish-order queue, rings of 8 / 16 frames measured fastest on every box
// tried; deeper rings only grow the L2 working set)
//   GDN_FUSED_STATS_PCT  share of the non-chain SMs given to the stats role (default 54, 20..80)
}  // namespace

namespace {
int env_int(const char* name, int dflt, int lo, int hi) {
  const char* s = getenv(name);
  if (s == nullptr || *s == 0) return dflt;
  const int v = atoi(s);
  return v < lo ? lo : (v > hi ? hi : v);
}
// A_t / B_t ring slots per head of the fused forward: how many frames the statistics may run
// ahead of the chain. 16 when sixteen slots of every head (bf16 A_t and f32 B_t, 6 D^2 bytes a
// slot) take at most 16 MB, so that they stay in L2 beside the streams; else 8. Measured: the
// 480p clip (12.6 MB) 5-8 % faster with 16, the 720p clip (31 MB) 10 % slower.
int fused_ring(long bh, int D) {
  static const int r = env_int("GDN_FUSED_RING", 0, 0, 64);
  if (r > 0) return r < 4 ? 4 : r;
  return 16.0 * bh * D * D * 6 <= 16e6 ? 16 : 8;
}
int fused_sring() {
  static const int r = env_int("GDN_FUSED_SRING", 16, 8, 64);
  return r;
}
// Share of the worker SMs (those left after the chains) that run the statistics role, in %:
// by default about the ratio of the two roles' per-frame times, 54 for bf16 inputs at DP = 128;
// 40 for e4m3 inputs, whose statistics read half the bytes of bf16 on the tensor core's f8f6f4
// path while the outputs still write bf16 (measured: 2.60 ms on the 720p clip against 3.03 at
// 54); 40 at DP = 64, where the chain's short frame steps leave the outputs behind (the 480p
// clip 6 % faster than at 54).
int fused_stats_pct(bool f8, int DP) {
  static const int p = env_int("GDN_FUSED_STATS_PCT", 0, 0, 80);
  return p > 0 ? p : ((f8 || DP == 64) ? 40 : 54);
}

struct FusedWs {
  void* A;
  float* B;
  void* S;
  int* flags;  // stats_flag [BH*T], out_flag [BH*T], chain_prog [BH], abort, 2 work counters,
               // ready_tail, ready_items [BH*T] (the outputs' queue)
  size_t flag_bytes;
};

// R, Rs: A_t/B_t and S_t ring slots per head (0: the tuned defaults). With R = Rs = T every
// frame keeps its own slot, and the A, B, S blocks are laid out exactly like the three-kernel
// workspace (row (b*H + h)*T + t): gdn_frame_forward_train keeps them for the backward.
size_t fused_ws_bytes(long bh, long T, int D, int R = 0, int Rs = 0) {
  const int kRing = R > 0 ? R : fused_ring(bh, D);
  const size_t m = size_t(D) * D * bh * kRing;
  const size_t dp = padded_dim(D), ms = dp * dp * bh * (Rs > 0 ? Rs : fused_sring());
  const size_t flags = sizeof(int) * (3 * bh * T + bh + 4);
  return align256(m * 2) + align256(m * 4) + align256(ms * 2) + align256(flags);
}

FusedWs carve_fused(void* base, long bh, long T, int D, int R = 0, int Rs = 0) {
  const int kRing = R > 0 ? R : fused_ring(bh, D);
  const size_t m = size_t(D) * D * bh * kRing;
  const size_t dp = padded_dim(D), ms = dp * dp * bh * (Rs > 0 ? Rs : fused_sring());
  uint8_t* p = static_cast<uint8_t*>(base);
  FusedWs w;
  w.A = p;
  p += align256(m * 2);
  w.B = reinterpret_cast<float*>(p);
  p += align256(m * 4);
  w.S = p;
  p += align256(ms * 2);
  w.flags = reinterpret_cast<int*>(p);
  w.flag_bytes = sizeof(int) * (3 * bh * T + bh + 4);
  return w;
}

// Whether the fused forward can run this problem on this GPU: every (batch, head) needs its own
// chain CTA and enough SMs must remain for the two streaming roles.
bool fused_applies(int dev, const Problem& p) {
  if (g_forward_mode == 1) return false;
  const int sms = g_dev[dev].sms;
  const long bh = long(p.B) * p.H;
  int coop = 0;
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
  if (!coop || sms - bh < 8) return false;
  if (g_forward_mode == 2) return true;
  return bh * 3 <= sms && p.T >= 4;
}

// keep_all: every frame keeps its own A_t/B_t/S_t slot (R = Rs = T) in the caller's buffer
// `kept` (fused_ws_bytes(bh, T, D, T, T) bytes) instead of the cached workspace's rings.
template <int DP, bool kF8 = false, bool kRope = false>
gdn_status run_fused(int dev, const Problem& p, const void* q, const void* k, const void* v,
                     const float* gamma, const float* beta, const float* s_in, void* out,
                     float* s_out, cudaStream_t st, void* kept = nullptr) {
  using L = gdn::FusedLayout<DP>;
  constexpr int kSmem = kRope ? L::kSmemBytesRope : L::kSmemBytes;
  const int sms = g_dev[dev].sms;
  const int bh = p.B * p.H;
  const int kRing = kept ? p.T : fused_ring(bh, p.D);
  const int kSRing = kept ? p.T : fused_sring();
  void* base = kept;
  if (!kept)
    if (gdn_status s = get_workspace(dev, fused_ws_bytes(bh, p.T, p.D), st, &base)) return s;
  FusedWs w = carve_fused(base, bh, p.T, p.D, kRing, kSRing);
  if (cudaMemsetAsync(w.flags, 0, w.flag_bytes, st) != cudaSuccess) return GDN_ERR_CUDA;
  CUtensorMap tk, tv, tq, to, ta;
  if (!tmap_in<kF8>(&tk, k, p) || !tmap_in<kF8>(&tv, v, p) || !tmap_in<kF8>(&tq, q, p) ||
      !tmap_tokens(&to, out, p) || !tmap_mats(&ta, w.A, false, p.D, p.D, long(bh) * kRing, DP))
    return GDN_ERR_CUDA;
  auto kern = gdn::gdn_fused_kernel<DP, kF8, kRope>;
  const int bit = kRope ? 44 + (DP == 128 ? 0 : 1) : (kF8 ? 17 : (DP == 128 ? 8 : 9));
  if (gdn_status s = ensure_smem_attr(dev, bit, kern, kSmem)) return s;
  // split the SMs left after the chains between the stats and output roles (fused_stats_pct)
  const int workers = sms - bh;
  int n_stats = (workers * fused_stats_pct(kF8, DP) + 50) / 100;
  if (n_stats < 1) n_stats = 1;
  if (n_stats > workers - 1) n_stats = workers - 1;
  int* f = w.flags;
  const long ft = long(bh) * p.T;
  int* abort_word = f + 2 * ft + bh;
  // GDN_TEST_WITHHOLD_FRAME (tests only): the statistics of this frame of head 0 are computed
  // but never published, so the chain's wait for them runs out and the call reports
  // GDN_ERR_TIMEOUT through gdn_sync_status
  static const int withhold = env_int("GDN_TEST_WITHHOLD_FRAME", -1, -1, 1 << 30);
  gdn::Handoff hc{f, f + ft, f + 2 * ft, abort_word, nullptr, kRing, kSRing, withhold, 0, bh};
  hc.ready_tail = abort_word + 3;
  hc.ready_items = abort_word + 4;
  gdn::Handoff hs = hc;
  hs.base = bh;
  hs.count = n_stats;
  hs.next_item = abort_word + 1;
  gdn::Handoff ho = hc;
  ho.base = bh + n_stats;
  ho.count = workers - n_stats;
  ho.next_item = abort_word + 2;
  __nv_bfloat16* a_ring = static_cast<__nv_bfloat16*>(w.A);
  float* b_ring = w.B;
  __nv_bfloat16* s_ring = static_cast<__nv_bfloat16*>(w.S);
  gdn::Problem pp = p;
  void* args[] = {&tk, &tv, &tq, &to, &ta, &a_ring, &b_ring, &s_ring,
                  const_cast<float**>(&gamma), const_cast<float**>(&beta),
                  const_cast<float**>(&s_in), &s_out, &pp, &hc, &hs, &ho};
  {
    ProfiledLaunch pl("gdn_fused_kernel", st);
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(sms),
                                    dim3(L::kThreads), args, kSmem, st) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  return check_launch();
}

// ------------------------------------------------------------------ chunked forward
// Frames are cut into chunks of L; the chain's serial path shrinks from T frame steps to
// L (composition) + ceil(T/L) - 1 (scan) + L (replay), at about three times the chain's total
// work. It pays when few (batch, head) chains run long clips, so that the chain and not HBM
// bounds the other paths.

// Costs on B200 used to choose the path and L, fitted to measurements on the 720p clip shape
// with 1..8 heads: one frame step of the standalone and of the fused chain (D <= 64 / D <= 128,
// microseconds), one inter-chunk scan step, the fill and drain of a launch, the HBM bandwidth
// the fused kernel and the streaming kernels reach, and the bandwidth the composition and replay
// launches reach while all their CTAs pull A_t / B_t at once (bytes per microsecond).
constexpr double kChainStepUs[2] = {1.6, 2.0};
constexpr double kFusedChainStepUs[2] = {1.7, 2.1};
constexpr double kScanStepUs = 2.8;
constexpr double kLaunchFillUs = 5.0;
constexpr double kFusedBytesPerUs = 5.5e6;
constexpr double kStreamBytesPerUs = 5.77e6;
constexpr double kChainSideBytesPerUs = 4.5e6;

struct ChunkPlan {
  int L = 0;
  int nc = 1;
  double us = 0;  // estimated chain-side time (composition + scan + replay)
};

ChunkPlan plan_chunks(int dev, const Problem& p, int forced_L) {
  const double tc = kChainStepUs[p.D <= 64 ? 0 : 1];
  const long bh = long(p.B) * p.H;
  const int sms = g_dev[dev].sms > 0 ? g_dev[dev].sms : 148;
  const double dd = double(p.D) * p.D, dp2 = double(padded_dim(p.D)) * padded_dim(p.D);
  // composition reads A_t (P) and A_t, B_t (C); the replay reads A_t, B_t and writes S_t
  const double compose_floor = bh * p.T * dd * 8.0 / kChainSideBytesPerUs;
  const double replay_floor = bh * p.T * (dd * 6.0 + dp2 * 2.0) / kChainSideBytesPerUs;
  auto waves = [&](long ctas) { return double((ctas + sms - 1) / sms); };
  auto cost = [&](int L) {
    const int nc = (p.T + L - 1) / L;
    const double replay = waves(bh * nc) * L * tc;
    double us = (replay > replay_floor ? replay : replay_floor) + kLaunchFillUs;
    if (nc > 1) {
      const double compose = waves(2 * bh * (nc - 1)) * L * tc;
      us += (compose > compose_floor ? compose : compose_floor) + kLaunchFillUs +
            (nc - 1) * kScanStepUs + kLaunchFillUs;
    }
    return us;
  };
  ChunkPlan best;
  if (forced_L > 0) {
    best.L = forced_L < p.T ? forced_L : p.T;
  } else {
    best.L = p.T;
    double c = cost(p.T);
    for (int L = 4; L < p.T && L <= 256; ++L) {  // gdn_workspace_bytes assumes L >= 4
      const double x = cost(L);
      if (x < c) {
        c = x;
        best.L = L;
      }
    }
  }
  best.nc = (p.T + best.L - 1) / best.L;
  best.us = cost(best.L);
  return best;
}

// GDN_CHUNK_LEN: frames per chunk of the chunked forward (0 or unset: chosen per problem)
int chunk_len_override() { return env_int("GDN_CHUNK_LEN", 0, 0, 1 << 20); }

size_t chunked_ws_bytes(long bh, long T, int D, int nc) {
  const int dp = padded_dim(D);
  return forward_ws_bytes(bh * T, D) + align256(size_t(bh) * (nc - 1) * gdn::chunk_map_bytes(dp)) +
         align256(size_t(bh) * nc * gdn::chunk_start_bytes(dp));
}

// Whether the chunked forward is expected to beat the path chosen otherwise.
bool chunked_pays(int dev, const Problem& p, bool fused) {
  if (p.T < 16) return false;
  const int dx = p.D <= 64 ? 0 : 1;
  const double bh = double(p.B) * p.H;
  const double dp2 = double(padded_dim(p.D)) * padded_dim(p.D);
  const double io = bh * p.T * (4.0 * p.N * p.D * 2);          // Q, K, V read, O written
  const double ws = bh * p.T * (6.0 * p.D * p.D + 2.0 * dp2);  // A_t, B_t written, S_t read
  double other;
  if (fused) {
    const double hbm = io / kFusedBytesPerUs, chain = p.T * kFusedChainStepUs[dx] + kLaunchFillUs;
    other = hbm > chain ? hbm : chain;
  } else {
    other = (io + ws) / kStreamBytesPerUs + p.T * kChainStepUs[dx] + 3 * kLaunchFillUs;
  }
  const ChunkPlan c = plan_chunks(dev, p, 0);
  if (c.nc < 2) return false;
  const double chunked = (io + ws) / kStreamBytesPerUs + c.us;
  return chunked < 0.9 * other;
}

template <int DP, bool kF8 = false, bool kRope = false>
gdn_status run_chunked(int dev, const Problem& p, const void* q, const void* k, const void* v,
                       const float* gamma, const float* beta, const float* s_in, void* out,
                       float* s_out, cudaStream_t st) {
  const ChunkPlan plan = plan_chunks(dev, p, chunk_len_override());
  const long bh = long(p.B) * p.H;
  void* base = nullptr;
  if (gdn_status s = get_workspace(dev, chunked_ws_bytes(bh, p.T, p.D, plan.nc), st, &base))
    return s;
  const long count = bh * p.T;
  ForwardWs w = carve_forward(base, count, p.D);
  uint8_t* maps = static_cast<uint8_t*>(base) + forward_ws_bytes(count, p.D);
  uint8_t* starts = maps + align256(size_t(bh) * (plan.nc - 1) * gdn::chunk_map_bytes(DP));
  const gdn::ChainSeg compose{plan.L, plan.nc, 1, maps, starts};
  const gdn::ChainSeg replay{plan.L, plan.nc, 0, maps, starts};
  if (gdn_status s = run_stats<DP, true, kF8, kRope>(dev, p, k, v, w.A, w.B, st)) return s;
  if (plan.nc > 1) {
    if (gdn_status s = run_chain<DP>(dev, p, w.A, w.B, gamma, beta, nullptr, nullptr, nullptr,
                                     compose, st))
      return s;
    if (gdn_status s = run_scan<DP>(dev, p, compose, s_in, st)) return s;
  }
  if (gdn_status s = run_chain<DP>(dev, p, w.A, w.B, gamma, beta, s_in, w.S, s_out, replay, st))
    return s;
  return run_output<DP, false, kF8, kRope>(dev, p, q, w.S, p.D, out, 1, st);
}

// kF8: e4m3 q, k, v (scales in p; 64 < D <= 128, checked by the caller). kRope: q and k rotated
// by the 3D RoPE of p.rope inside the statistics and output kernels.
template <bool kF8, bool kRope = false>
gdn_status forward_path(int dev, const void* q, const void* k, const void* v, const float* gamma,
                        const float* beta, const float* s_in, void* out, float* s_out,
                        const Problem& p, cudaStream_t st) {
  constexpr int kDP = 128;
  const bool fused = fused_applies(dev, p);
  if (g_forward_mode == 3 || (g_forward_mode == 0 && chunked_pays(dev, p, fused))) {
    if (!kF8 && p.D <= 64)
      return run_chunked<64, false, kRope>(dev, p, q, k, v, gamma, beta, s_in, out, s_out, st);
    return run_chunked<kDP, kF8, kRope>(dev, p, q, k, v, gamma, beta, s_in, out, s_out, st);
  }
  if (fused) {
    if (!kF8 && p.D <= 64)
      return run_fused<64, false, kRope>(dev, p, q, k, v, gamma, beta, s_in, out, s_out, st);
    return run_fused<kDP, kF8, kRope>(dev, p, q, k, v, gamma, beta, s_in, out, s_out, st);
  }
  const long count = long(p.B) * p.H * p.T;
  void* base = nullptr;
  if (gdn_status s = get_workspace(dev, forward_ws_bytes(count, p.D), st, &base)) return s;
  ForwardWs w = carve_forward(base, count, p.D);
  const gdn::ChainSeg whole{p.T, 1, 0, nullptr, nullptr};
  if (!kF8 && p.D <= 64) {
    if (gdn_status s = run_stats<64, true, false, kRope>(dev, p, k, v, w.A, w.B, st)) return s;
    if (gdn_status s = run_chain<64>(dev, p, w.A, w.B, gamma, beta, s_in, w.S, s_out, whole, st))
      return s;
    return run_output<64, false, false, kRope>(dev, p, q, w.S, p.D, out, 1, st);
  }
  if (gdn_status s = run_stats<kDP, true, kF8, kRope>(dev, p, k, v, w.A, w.B, st)) return s;
  if (gdn_status s = run_chain<kDP>(dev, p, w.A, w.B, gamma, beta, s_in, w.S, s_out, whole, st))
    return s;
  return run_output<kDP, false, kF8, kRope>(dev, p, q, w.S, p.D, out, 1, st);
}

gdn_status forward_impl(const void* q, const void* k, const void* v, const float* gamma,
                        const float* beta, const float* s_in, void* out, float* s_out,
                        const Problem& p, cudaStream_t st) {
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  if (p.k_scale != nullptr)
    return forward_path<true>(dev, q, k, v, gamma, beta, s_in, out, s_out, p, st);
  if (p.rope.tab != nullptr)
    return forward_path<false, true>(dev, q, k, v, gamma, beta, s_in, out, s_out, p, st);
  return forward_path<false>(dev, q, k, v, gamma, beta, s_in, out, s_out, p, st);
}

// Device address of g_noalloc_scratch on the current GPU, looked up once per GPU (with that GPU
// current) and cached.
void* g_noalloc_addr[kMaxDevices];

gdn_status noalloc_scratch(int dev, void** out) {
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return GDN_OK;
}

// Single-frame step (64 < D <= 128): one cooperative launch; statistics units and output units
// are taken dynamically (the workspace holds the per-item S' tiles and the hand-off flags).
gdn_status run_step(int dev, const Problem& p, const void* q, const void* k, const void* v,
                    const float* gamma, const float* beta, const float* s_in, void* out,
                    float* s_out, cudaStream_t st) {
  using L = gdn::StepLayout;
  const long items = long(p.B) * p.H;
  DeviceState& d = g_dev[dev];
  // persistent flag words: ready [items] (epochs), next_unit, done, abort; zeroed when allocated
  if (d.step_items < items || d.step_epoch >= 0x7fffff00) {
    const size_t bytes = sizeof(int) * (items + 3);
    void* buf = d.step_flags;
    size_t have = 0;
    d.step_items = 0;
    if (gdn_status s = grow_buffer(&buf, &have, bytes, st)) {
      d.step_flags = static_cast<int*>(buf);
      return s;
    }
    d.step_flags = static_cast<int*>(buf);
    if (cudaMemsetAsync(d.step_flags, 0, bytes, st) != cudaSuccess) return GDN_ERR_CUDA;
    d.step_items = items;
    d.step_epoch = 0;
  }
  void* base = nullptr;
  if (gdn_status s = get_workspace(dev, align256(size_t(items) * L::kTileBytes), st, &base))
    return s;
  int* f = d.step_flags;
  gdn::StepShared sh{f, f + d.step_items, f + d.step_items + 1, f + d.step_items + 2,
                     static_cast<uint8_t*>(base), ++d.step_epoch};
  CUtensorMap tq, tk, tv, to;
  if (!tmap_tokens(&tq, q, p) || !tmap_tokens(&tk, k, p) || !tmap_tokens(&tv, v, p) ||
      !tmap_tokens(&to, out, p))
    return GDN_ERR_CUDA;
  auto kern = gdn::gdn_step_kernel;
  if (gdn_status s = ensure_smem_attr(dev, 12, kern, L::kSmemBytes)) return s;
  const int n_tiles = (p.N + gdn::kRowsPerTile - 1) / gdn::kRowsPerTile;
  const long units = items * (1 + (n_tiles + L::kOutTiles - 1) / L::kOutTiles);
  const int grid = static_cast<int>(units < d.sms ? units : d.sms);
  gdn::Problem pp = p;
  void* args[] = {&tq, &tk, &tv, &to, const_cast<float**>(&gamma), const_cast<float**>(&beta),
                  const_cast<float**>(&s_in), &s_out, &pp, &sh};
  {
    ProfiledLaunch pl("gdn_step_kernel", st);
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid),
                                    dim3(L::kThreads), args, L::kSmemBytes, st) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  return check_launch();
}

gdn_status validate_common(const void* q, const void* k, const void* v, const void* out,
                           const float* gamma, const float* beta, const float* s_in,
                           const float* s_out, int B, int H, int T, int N, int D, float ks) {
  if (!q || !k || !v || !out || !gamma || !beta) return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  float ks_eff;
  if (!resolve_key_scale(ks, D, N, &ks_eff)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (s_in && !aligned16(s_in)) || (s_out && !aligned16(s_out)))
    return GDN_ERR_MISALIGNED;
  const size_t n = size_t(B) * T * N * H * D * 2;
  if (overlaps(out, n, q, n) || overlaps(out, n, k, n) || overlaps(out, n, v, n))
    return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}


// ------------------------------------------------------------------ backward
// Workspace of gdn_frame_backward, per frame-head: the forward's A_t (bf16 D x D), B_t (f32),
// S_t (bf16 DP x DP), E_t = dO^T Q (f32), G_t (bf16 DP x DP) and W'_t (bf16 DP x DP; before the
// per-frame kernel writes it, the same space takes the unused Q^T Q of the E statistics); per
// head the f32 G carried between segments of the backward chain.
struct BackwardWs {
  void* A;
  float* B;
  void* S;
  float* E;
  void* G;
  void* W;
  float* C;
};

size_t backward_ws_bytes(long count, int D, long bh) {
  const size_t m = size_t(D) * D, dp2 = size_t(128) * 128;
  return align256(count * m * 2) + align256(count * m * 4) + 3 * align256(count * dp2 * 2) +
         align256(count * m * 4) + align256(bh * m * 4);
}

// With the forward's A_t, B_t, S_t saved by gdn_frame_forward_train, the workspace holds only
// E_t, G_t, W'_t and the carried G.
size_t backward_saved_ws_bytes(long count, int D, long bh) {
  const size_t m = size_t(D) * D, dp2 = size_t(128) * 128;
  return align256(count * m * 4) + 2 * align256(count * dp2 * 2) + align256(bh * m * 4);
}

BackwardWs carve_backward_saved(void* base, const void* saved, long count, int D) {
  const size_t m = size_t(D) * D, dp2 = size_t(128) * 128;
  const ForwardWs f = carve_forward(const_cast<void*>(saved), count, D);
  uint8_t* p = static_cast<uint8_t*>(base);
  BackwardWs w;
  w.A = f.A;
  w.B = f.B;
  w.S = f.S;
  w.E = reinterpret_cast<float*>(p);
  p += align256(count * m * 4);
  w.G = p;
  p += align256(count * dp2 * 2);
  w.W = p;
  p += align256(count * dp2 * 2);
  w.C = reinterpret_cast<float*>(p);
  return w;
}

BackwardWs carve_backward(void* base, long count, int D) {
  const size_t m = size_t(D) * D, dp2 = size_t(128) * 128;
  uint8_t* p = static_cast<uint8_t*>(base);
  BackwardWs w;
  w.A = p;
  p += align256(count * m * 2);
  w.B = reinterpret_cast<float*>(p);
  p += align256(count * m * 4);
  w.S = p;
  p += align256(count * dp2 * 2);
  w.E = reinterpret_cast<float*>(p);
  p += align256(count * m * 4);
  w.G = p;
  p += align256(count * dp2 * 2);
  w.W = p;
  p += align256(count * dp2 * 2);
  w.C = reinterpret_cast<float*>(p);
  return w;
}

gdn_status run_bwd_chain(int dev, const Problem& p, const void* A, const float* E,
                         const float* gamma, const float* beta, const float* d_state_out,
                         void* G, float* d_state_in, float* carry, int t_lo, int t_hi,
                         cudaStream_t st) {
  using L = gdn::BwdChainLayout<128>;
  const long count = long(p.B) * p.H * p.T;
  CUtensorMap ta;
  if (!tmap_mats(&ta, A, false, p.D, p.D, count, 128)) return GDN_ERR_CUDA;
  auto kern = gdn::gdn_bwd_chain_kernel<128>;
  if (gdn_status s = ensure_smem_attr(dev, 20, kern, L::kSmemBytes)) return s;
  {
    ProfiledLaunch pl("gdn_bwd_chain_kernel", st);
    kern<<<p.B * p.H, L::kThreads, L::kSmemBytes, st>>>(ta, E, static_cast<__nv_bfloat16*>(G),
                                                        gamma, beta, d_state_out, d_state_in,
                                                        carry, t_lo, t_hi, p);
  }
  return check_launch();
}

gdn_status run_bwd_frame(int dev, const Problem& p, const BackwardWs& w, const float* state_in,
                         const float* gamma, const float* beta, float* d_gamma, float* d_beta,
                         int t_lo, int t_hi, cudaStream_t st, int max_sms = 0) {
  using L = gdn::BwdFrameLayout<128>;
  auto kern = gdn::gdn_bwd_frame_kernel<128>;
  if (gdn_status s = ensure_smem_attr(dev, 21, kern, L::kSmemBytes)) return s;
  const long items = long(p.B) * p.H * (t_hi - t_lo);
  // two CTAs of 98 KB shared memory per SM
  const long cap = 2L * (max_sms > 0 ? max_sms : g_dev[dev].sms);
  const int grid = static_cast<int>(items < cap ? items : cap);
  {
    ProfiledLaunch pl("gdn_bwd_frame_kernel", st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(
        static_cast<const __nv_bfloat16*>(w.S), static_cast<const __nv_bfloat16*>(w.G),
        static_cast<const __nv_bfloat16*>(w.A), w.B, state_in, gamma, beta,
        static_cast<__nv_bfloat16*>(w.W), d_gamma, d_beta, t_lo, t_hi, p);
  }
  return check_launch();
}

// One of the token GEMMs of the backward: out = scale * sum over terms of X_i Y_i^(T)
// (kDualV: also out2 = scale * X1 Y0^T; kDualE: out = X0 Y0 and E = X0^T X1 per frame).
template <int kTerms, bool kMN0, bool kMN1, bool kDualV = false, bool kDualE = false>
gdn_status run_bwd_token(int dev, const Problem& p, const void* x0, const void* x1,
                         const void* Y0, const void* Y1, const float* beta, void* out,
                         const char* name, int attr_bit, cudaStream_t st, int max_ctas = 0,
                         void* out2 = nullptr, int t_lo = 0, int t_hi = -1, float* E = nullptr) {
  if (t_hi < 0) t_hi = p.T;
  using L = gdn::BwdTokenLayout<128, kTerms, kDualV, kDualE>;
  CUtensorMap t0, t1, to, to2;
  if (!tmap_tokens(&t0, x0, p) || !tmap_tokens(&t1, kTerms == 2 ? x1 : x0, p) ||
      !tmap_tokens(&to, out, p) || !tmap_tokens(&to2, kDualV ? out2 : out, p))
    return GDN_ERR_CUDA;
  auto kern = gdn::gdn_bwd_token_kernel<128, kTerms, kMN0, kMN1, kDualV, kDualE>;
  if (gdn_status s = ensure_smem_attr(dev, attr_bit, kern, L::kSmemBytes)) return s;
  const long items = long(p.B) * (t_hi - t_lo) * p.H;
  const long cap = max_ctas > 0 ? max_ctas : g_dev[dev].sms;
  const int grid = static_cast<int>(items < cap ? items : cap);
  const gdn::BwdTokenArgs a{static_cast<const __nv_bfloat16*>(Y0),
                            static_cast<const __nv_bfloat16*>(Y1), beta, t_lo, t_hi, E};
  {
    ProfiledLaunch pl(name, st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(t0, t1, to, to2, a, p);
  }
  return check_launch();
}

// The whole backward (64 < D <= 128): recompute the forward's statistics and states, then the
// output statistics E_t, the backward chain, the per-frame kernel and the token passes (dq;
// dk and dv together).
//
// The two state chains run one CTA per head and leave most SMs idle, so when the heads fill at
// most a quarter of the SMs, the rest runs beside them on a second stream (fork and join through
// events, so the call stays ordered on `st` and can be captured in a graph), and the backward
// chain is launched in segments of frames, last segment first, so that the per-frame and dk/dv
// passes of a finished segment run while the chain walks the next one:
//   st:  stats(k,v) -> forward chain -> [E] chain seg 1 -> chain seg 2 -> ... -> [end]
//   aux:      [A] stats(q,dO) -> [S] dq -> [seg 1] frame, dk/dv -> [seg 2] frame, dk/dv -> ...
// Kernels on the second stream that run beside a chain get grids that leave the chains' SMs free
// (a persistent grid that waited for them would finish its last items after the chain).
gdn_status aux_stream(int dev, DeviceState** out) {
  DeviceState& d = g_dev[dev];
  if (d.aux == nullptr) {
    if (cudaStreamCreateWithFlags(&d.aux, cudaStreamNonBlocking) != cudaSuccess) return GDN_ERR_CUDA;
    for (cudaEvent_t& e : d.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return GDN_ERR_CUDA;
  }
  *out = &d;
  return GDN_OK;
}

// saved: the forward's A_t, B_t, S_t as gdn_frame_forward_train stored them, or nullptr (the
// statistics and the state chain of the forward are recomputed first).
gdn_status backward_path(int dev, const void* q, const void* k, const void* v,
                         const float* gamma, const float* beta, const float* s_in,
                         const void* d_out, const float* ds_out, void* dq, void* dk, void* dv,
                         float* d_gamma, float* d_beta, float* ds_in, const Problem& p,
                         cudaStream_t st, const void* saved = nullptr) {
  const long count = long(p.B) * p.H * p.T;
  const long bh = long(p.B) * p.H;
  void* base = nullptr;
  const size_t ws_bytes =
      saved ? backward_saved_ws_bytes(count, p.D, bh) : backward_ws_bytes(count, p.D, bh);
  if (gdn_status s = get_workspace(dev, ws_bytes, st, &base)) return s;
  const BackwardWs w =
      saved ? carve_backward_saved(base, saved, count, p.D) : carve_backward(base, count, p.D);
  const gdn::ChainSeg whole{p.T, 1, 0, nullptr, nullptr};
  Problem pe = p;  // E_t = dO^T Q: the "B" statistic of (key = q, value = dO), key scale 1
  pe.key_scale = 1.0f;
  const int sms = g_dev[dev].sms;
  const bool overlap = bh * 4 <= sms;
  DeviceState* d = nullptr;
  if (overlap)
    if (gdn_status s = aux_stream(dev, &d)) return s;
  const int side = overlap ? static_cast<int>(sms - bh) : 0;  // SMs beside the chains
  cudaStream_t sx = overlap ? d->aux : st;
  auto link = [&](cudaStream_t from, cudaStream_t to, int e) -> gdn_status {
    if (!overlap) return GDN_OK;
    if (cudaEventRecord(d->ev[e], from) != cudaSuccess) return GDN_ERR_CUDA;
    return cudaStreamWaitEvent(to, d->ev[e], 0) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  };
  // segments of the backward chain: about GDN_BWD_SEGMENT_FRAMES frames each (default 240)
  const int seg_target = env_int("GDN_BWD_SEGMENT_FRAMES", 240, 1, 1 << 20);
  const int n_seg = overlap ? std::max(1, (p.T + seg_target / 2) / seg_target) : 1;
  const int seg_len = (p.T + n_seg - 1) / n_seg;

  if (saved != nullptr) {
    // The forward's states are given: dQ_t and E_t come from one pass over dO (gdn_bwd_token_
    // kernel_dqe), run segment by segment from the clip's end, so that each segment of the
    // backward chain starts as soon as its E_t are stored:
    //   aux: [A] dqe seg 1 -> dqe seg 2 -> ... -> [seg 1] frame, dk/dv -> [seg 2] frame, dk/dv
    //   st:    [E1] chain seg 1 -> [E2] chain seg 2 -> ...                                 [end]
    // (one event per chain segment, all recorded before the aux stream waits on the first)
    const int n_s = std::min(n_seg, kMaxSegEvents);
    const int len = (p.T + n_s - 1) / n_s;
    if (gdn_status s = link(st, sx, 0)) return s;  // [A]: aux after the caller's earlier work
    // A chain segment [lo, hi) ends with G_{lo-1}, which includes E_{lo-1}: the dQ/E pass
    // before it covers frames [lo - 1, lo' - 1) (lo' the previous segment's start; T for the
    // first), so every frame is covered once and each segment's E_t are stored before it runs.
    int k_seg = 0;
    int e_hi = p.T;
    for (int hi = p.T, lo; hi > 0; hi = lo, ++k_seg) {
      lo = std::max(0, hi - len);
      const int e_lo = std::max(0, lo - 1);
      // the first segment's pass runs alone: all SMs; later ones beside the chain
      if (e_lo < e_hi)
        if (gdn_status s = run_bwd_token<2, true, false, false, true>(
                dev, p, d_out, q, w.S, nullptr, nullptr, dq, "gdn_bwd_token_kernel_dqe", 23, sx,
                k_seg == 0 ? 0 : side, nullptr, e_lo, e_hi, w.E))
          return s;
      e_hi = e_lo;
      if (gdn_status s = link(sx, st, 2)) return s;  // [E]: this segment's E_t are stored
      if (gdn_status s = run_bwd_chain(dev, p, w.A, w.E, gamma, beta, ds_out, w.G, ds_in, w.C,
                                       lo, hi, st))
        return s;
      if (overlap && cudaEventRecord(d->ev[5 + k_seg], st) != cudaSuccess) return GDN_ERR_CUDA;
    }
    k_seg = 0;
    for (int hi = p.T, lo; hi > 0; hi = lo, ++k_seg) {
      lo = std::max(0, hi - len);
      // [segment]: its G_t are stored
      if (overlap && cudaStreamWaitEvent(sx, d->ev[5 + k_seg], 0) != cudaSuccess)
        return GDN_ERR_CUDA;
      const int g = lo == 0 ? 0 : side;  // the last segment's passes run after the chain
      if (gdn_status s = run_bwd_frame(dev, p, w, s_in, gamma, beta, d_gamma, d_beta, lo, hi, sx,
                                       g))
        return s;
      if (gdn_status s = run_bwd_token<2, true, false, true>(
              dev, p, v, k, w.G, w.W, beta, dk, "gdn_bwd_token_kernel_dkdv", 25, sx, g, dv, lo, hi))
        return s;
    }
    return link(sx, st, 3);  // [end]: the call ends on `st` after everything
  }

  if (gdn_status s = run_stats<128, true>(dev, p, k, v, w.A, w.B, st)) return s;
  if (gdn_status s = link(st, sx, 0)) return s;  // [A]: aux after the forward statistics
  if (gdn_status s = run_chain<128>(dev, p, w.A, w.B, gamma, beta, s_in, w.S, nullptr, whole,
                                    st))
    return s;
  // E_t statistics beside the forward chain
  if (gdn_status s = run_stats<128, true>(dev, pe, q, d_out, w.W, w.E, sx, side)) return s;
  if (gdn_status s = link(st, sx, 1)) return s;  // [S]: dq after the forward chain
  if (gdn_status s = link(sx, st, 2)) return s;  // [E]: backward chain after E_t
  if (gdn_status s = run_bwd_token<1, true, false>(dev, p, d_out, nullptr, w.S, nullptr, nullptr,
                                                   dq, "gdn_bwd_token_kernel_dq", 22, sx, side))
    return s;
  for (int hi = p.T, lo; hi > 0; hi = lo) {
    lo = std::max(0, hi - seg_len);
    if (gdn_status s = run_bwd_chain(dev, p, w.A, w.E, gamma, beta, ds_out, w.G, ds_in, w.C, lo,
                                     hi, st))
      return s;
    if (gdn_status s = link(st, sx, 4)) return s;  // [segment]: its G_t are stored
    // the last segment's passes run after the chain: full grids
    const int g = lo == 0 ? 0 : side;
    if (gdn_status s = run_bwd_frame(dev, p, w, s_in, gamma, beta, d_gamma, d_beta, lo, hi, sx, g))
      return s;
    // dK and dV in one pass over the K tiles
    if (gdn_status s = run_bwd_token<2, true, false, true>(
            dev, p, v, k, w.G, w.W, beta, dk, "gdn_bwd_token_kernel_dkdv", 25, sx, g, dv, lo, hi))
      return s;
  }
  return link(sx, st, 3);  // [end]: the call ends on `st` after everything
}

// ------------------------------------------------------------------ host-resident clips
// gdn_frame_forward_host streams a clip held in host memory through the GPU in segments of
// frames: segment i's inputs are copied in on a copy-in stream while segment i-1 is computed on
// the caller's stream and segment i-2's output is copied out on a copy-out stream (two staging
// buffers, ordered by events). The state is carried on the device from segment to segment, so
// the frame recurrence is split exactly as a resumed clip.
struct HostPipe {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t entry, in_done[2], comp_done[2], out_done[2], fin;
  void* buf = nullptr;
  size_t bytes = 0;
  bool ready = false;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

gdn_status pipe_init(int dev, HostPipe& hp) {
  if (hp.ready) return GDN_OK;
  if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess)
    return GDN_ERR_CUDA;
  cudaEvent_t* evs[] = {&hp.entry, &hp.in_done[0], &hp.in_done[1], &hp.comp_done[0],
                        &hp.comp_done[1], &hp.out_done[0], &hp.out_done[1], &hp.fin};
  for (cudaEvent_t* e : evs)
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return GDN_ERR_CUDA;
  (void)dev;
  hp.ready = true;
  return GDN_OK;
}

// Frames per segment: GDN_HOST_SEGMENT_FRAMES, else about 256 MB of q/k/v per segment.
int host_segment_frames(const Problem& p) {
  const int forced = env_int("GDN_HOST_SEGMENT_FRAMES", 0, 0, 1 << 30);
  if (forced > 0) return forced < p.T ? forced : p.T;
  const double per_frame = 3.0 * p.B * p.N * p.H * p.D * 2;
  int f = static_cast<int>((256.0 * (1 << 20)) / per_frame);
  if (f < 1) f = 1;
  return f < p.T ? f : p.T;
}

struct SegBufs {
  uint8_t *q, *k, *v, *out;
  float *g, *b;
};

gdn_status forward_host_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const float* gamma, const float* beta, const float* s_in,
                             uint16_t* out, float* s_out, const Problem& p, cudaStream_t st) {
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& hp = g_pipe[dev];
  if (gdn_status s = pipe_init(dev, hp)) return s;
  const int F = host_segment_frames(p);
  const size_t tok = size_t(p.N) * p.H * p.D;            // elements of one frame of one batch
  const size_t seg_tok = align256(size_t(p.B) * F * tok * 2);
  const size_t seg_gb = align256(size_t(p.B) * F * p.H * 4);
  const size_t per_buf = 4 * seg_tok + 2 * seg_gb;
  const size_t state_bytes = align256(size_t(p.B) * p.H * p.D * p.D * 4);
  const size_t need = 2 * per_buf + state_bytes;
  // (a previous call's copies on the internal streams are ordered before `st`'s later work)
  if (hp.bytes < need)
    if (gdn_status s = grow_buffer(&hp.buf, &hp.bytes, need, st)) return s;
  uint8_t* base = static_cast<uint8_t*>(hp.buf);
  SegBufs sb[2];
  for (int i = 0; i < 2; ++i) {
    uint8_t* b0 = base + i * per_buf;
    sb[i].q = b0;
    sb[i].k = b0 + seg_tok;
    sb[i].v = b0 + 2 * seg_tok;
    sb[i].out = b0 + 3 * seg_tok;
    sb[i].g = reinterpret_cast<float*>(b0 + 4 * seg_tok);
    sb[i].b = reinterpret_cast<float*>(b0 + 4 * seg_tok + seg_gb);
  }
  float* dstate = reinterpret_cast<float*>(base + 2 * per_buf);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // everything earlier on the caller's stream (including a previous call's pipeline) first
  if (!ok(cudaEventRecord(hp.entry, st)) || !ok(cudaStreamWaitEvent(hp.s_in, hp.entry, 0)) ||
      !ok(cudaStreamWaitEvent(hp.s_out, hp.entry, 0)))
    return GDN_ERR_CUDA;
  if (s_in != nullptr &&
      !ok(cudaMemcpyAsync(dstate, s_in, size_t(p.B) * p.H * p.D * p.D * 4,
                          cudaMemcpyHostToDevice, st)))
    return GDN_ERR_CUDA;
  const int n_seg = (p.T + F - 1) / F;
  for (int i = 0; i < n_seg; ++i) {
    const int j = i & 1;
    const int t0 = i * F;
    const int f = p.T - t0 < F ? p.T - t0 : F;
    // copy in (after segment i-2's compute has released buffer j)
    if (i >= 2 && !ok(cudaStreamWaitEvent(hp.s_in, hp.comp_done[j], 0))) return GDN_ERR_CUDA;
    for (int b = 0; b < p.B; ++b) {
      const size_t src = (size_t(b) * p.T + t0) * tok, dst = size_t(b) * f * tok;
      const size_t n = size_t(f) * tok * 2;
      if (!ok(cudaMemcpyAsync(sb[j].q + dst * 2, q + src, n, cudaMemcpyHostToDevice, hp.s_in)) ||
          !ok(cudaMemcpyAsync(sb[j].k + dst * 2, k + src, n, cudaMemcpyHostToDevice, hp.s_in)) ||
          !ok(cudaMemcpyAsync(sb[j].v + dst * 2, v + src, n, cudaMemcpyHostToDevice, hp.s_in)))
        return GDN_ERR_CUDA;
      const size_t gsrc = (size_t(b) * p.T + t0) * p.H, gdst = size_t(b) * f * p.H;
      const size_t gn = size_t(f) * p.H * 4;
      if (!ok(cudaMemcpyAsync(sb[j].g + gdst, gamma + gsrc, gn, cudaMemcpyHostToDevice,
                              hp.s_in)) ||
          !ok(cudaMemcpyAsync(sb[j].b + gdst, beta + gsrc, gn, cudaMemcpyHostToDevice, hp.s_in)))
        return GDN_ERR_CUDA;
    }
    if (!ok(cudaEventRecord(hp.in_done[j], hp.s_in))) return GDN_ERR_CUDA;
    // compute (after the copy-in, and after segment i-2's output has left buffer j)
    if (!ok(cudaStreamWaitEvent(st, hp.in_done[j], 0))) return GDN_ERR_CUDA;
    if (i >= 2 && !ok(cudaStreamWaitEvent(st, hp.out_done[j], 0))) return GDN_ERR_CUDA;
    const Problem ps{p.B, p.H, f, p.N, p.D, p.key_scale};
    const float* sin = (i == 0 && s_in == nullptr) ? nullptr : dstate;
    if (gdn_status s = forward_impl(sb[j].q, sb[j].k, sb[j].v, sb[j].g, sb[j].b, sin, sb[j].out,
                                    dstate, ps, st))
      return s;
    if (!ok(cudaEventRecord(hp.comp_done[j], st))) return GDN_ERR_CUDA;
    // copy out
    if (!ok(cudaStreamWaitEvent(hp.s_out, hp.comp_done[j], 0))) return GDN_ERR_CUDA;
    for (int b = 0; b < p.B; ++b) {
      const size_t dst = (size_t(b) * p.T + t0) * tok, src = size_t(b) * f * tok;
      if (!ok(cudaMemcpyAsync(out + dst, sb[j].out + src * 2, size_t(f) * tok * 2,
                              cudaMemcpyDeviceToHost, hp.s_out)))
        return GDN_ERR_CUDA;
    }
    if (!ok(cudaEventRecord(hp.out_done[j], hp.s_out))) return GDN_ERR_CUDA;
  }
  if (s_out != nullptr &&
      !ok(cudaMemcpyAsync(s_out, dstate, size_t(p.B) * p.H * p.D * p.D * 4,
                          cudaMemcpyDeviceToHost, hp.s_out)))
    return GDN_ERR_CUDA;
  // the caller's stream completes only after every copy of this call
  if (!ok(cudaEventRecord(hp.fin, hp.s_out)) || !ok(cudaStreamWaitEvent(st, hp.fin, 0)) ||
      !ok(cudaStreamWaitEvent(hp.s_in, hp.fin, 0)))
    return GDN_ERR_CUDA;
  return GDN_OK;
}

// Host checks of the 3D RoPE arguments shared by gdn_rope_3d and gdn_frame_forward_rope, and
// the table's dimensions (time, row and column slices of the head dimension).
gdn_status rope_dims(int B, int T, int N, int H, int D, int grid_h, int grid_w, float base,
                     int t_offset, gdn::RopeDims* r, long* n_tab) {
  if (B < 1 || T < 1 || N < 1 || H < 1 || D < 1 || grid_h < 1 || grid_w < 1 || t_offset < 0)
    return GDN_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 1024) return GDN_ERR_UNSUPPORTED;
  if (double(grid_h) * grid_w != double(N)) return GDN_ERR_INVALID_ARG;
  if (!(std::isfinite(base) && base > 1.f)) return GDN_ERR_INVALID_ARG;
  if (double(T) + t_offset > 2147483647.0) return GDN_ERR_INVALID_ARG;
  if (double(N) * H * (D / 8) > 2147483647.0 || double(B) * T > 2147483647.0)
    return GDN_ERR_INVALID_ARG;
  r->B = B;
  r->T = T;
  r->N = N;
  r->H = H;
  r->D = D;
  r->d_h = 2 * (D / 6);
  r->d_w = r->d_h;
  r->d_t = D - 2 * r->d_h;
  // the table layout of gdn::RopeArgs: per axis, rows of whole 16-byte entry pairs indexed by
  // the absolute pair index from the axis's first pair rounded down to even
  gdn::RopeArgs& a = r->ra;
  a.tab = nullptr;
  a.grid_h = grid_h;
  a.grid_w = grid_w;
  a.pt = r->d_t / 2;
  a.ph = r->d_h / 2;
  auto even_up = [](int x) { return (x + 1) & ~1; };
  a.len_t = even_up(a.pt);
  a.j0_h = a.pt & ~1;
  a.len_h = even_up(a.pt + a.ph - a.j0_h);
  a.j0_w = (a.pt + a.ph) & ~1;
  a.len_w = even_up(a.pt + 2 * a.ph - a.j0_w);
  if (double(T) * a.len_t + double(grid_h) * a.len_h + double(grid_w) * a.len_w > 2147483647.0)
    return GDN_ERR_INVALID_ARG;
  a.off_h = T * a.len_t;
  a.off_w = a.off_h + grid_h * a.len_h;
  *n_tab = long(a.off_w) + long(grid_w) * a.len_w;
  a.n_rc = static_cast<int>(*n_tab - a.off_h);
  return GDN_OK;
}

gdn_status launch_rope_table(float2* tab, const gdn::RopeDims& r, long n_tab, int t_offset,
                             float base, cudaStream_t st) {
  ProfiledLaunch pl("gdn_rope_table_kernel", st);
  gdn::gdn_rope_table_kernel<<<static_cast<unsigned>((n_tab + 255) / 256), 256, 0, st>>>(
      tab, r, t_offset, std::log2(double(base)));
  return check_launch();
}

// The per-GPU buffer of gdn_frame_forward_rope's table, grown like the workspace.
gdn_status get_rope_table(int dev, size_t bytes, cudaStream_t stream, float2** out) {
  DeviceState& d = g_dev[dev];
  if (d.rope_tab_bytes < bytes) {
    void* buf = d.rope_tab;
    gdn_status s = grow_buffer(&buf, &d.rope_tab_bytes, bytes, stream);
    d.rope_tab = static_cast<float2*>(buf);
    if (s) return s;
  }
  *out = d.rope_tab;
  return GDN_OK;
}

// Chunk-causal softmax attention: one persistent CTA per SM over (b, h, query tile) items.
template <int DP>
gdn_status run_softmax(int dev, const void* q, const void* k, const void* v, void* out, int B,
                       int H, int T, int N, int D, int F, float scale, cudaStream_t st) {
  using L = gdn::SoftmaxLayout<DP>;
  const int Ltok = T * N;
  CUtensorMap tq, tk, tv, to;
  if (!tmap_clip(&tq, q, B, H, Ltok, D) || !tmap_clip(&tk, k, B, H, Ltok, D) ||
      !tmap_clip(&tv, v, B, H, Ltok, D) || !tmap_clip(&to, out, B, H, Ltok, D))
    return GDN_ERR_CUDA;
  auto kern = gdn::gdn_softmax_kernel<DP>;
  if (gdn_status s = ensure_smem_attr(dev, DP == 128 ? 46 : 47, kern, L::kSmemBytes)) return s;
  const long items = long(B) * H * ((Ltok + gdn::kRowsPerTile - 1) / gdn::kRowsPerTile);
  const int grid = static_cast<int>(items < g_dev[dev].sms ? items : g_dev[dev].sms);
  // scores enter the base-2 exponential as S * scale * log2(e)
  const float c = static_cast<float>(double(scale) * 1.4426950408889634);
  // (batch, head) pairs per group: their K and V (re-read by every query tile) within ~48 MB of L2
  const double kv_bytes = 2.0 * Ltok * D * 2;
  const long bh = long(B) * H;
  const int G = static_cast<int>(std::max(1L, std::min(bh, static_cast<long>(48.0e6 / kv_bytes))));
  void* ws = nullptr;  // the work counter
  if (gdn_status s = get_workspace(dev, 256, st, &ws)) return s;
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return GDN_ERR_CUDA;
  {
    ProfiledLaunch pl("gdn_softmax_kernel", st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(tq, tk, tv, to, B, H, T, N, F, c,
                                                   static_cast<int*>(ws), G);
  }
  return check_launch();
}

}  // namespace

static gdn_status backward_entry(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                 const float* gamma, const float* beta, const float* state_in,
                                 const gdn_bf16* d_out, const float* d_state_out, gdn_bf16* dq,
                                 gdn_bf16* dk, gdn_bf16* dv, float* d_gamma, float* d_beta,
                                 float* d_state_in, int B, int H, int T, int N, int D,
                                 float key_scale, gdn_stream_t stream, const void* saved) {
  if (!q || !k || !v || !gamma || !beta || !d_out || !dq || !dk || !dv || !d_gamma || !d_beta)
    return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  if (D <= 64) return GDN_ERR_UNSUPPORTED;
  if (!resolve_key_scale(key_scale, D, N, &key_scale)) return GDN_ERR_INVALID_ARG;
  const void* dev_ptrs[] = {q, k, v, gamma, beta, d_out, dq, dk, dv, d_gamma, d_beta};
  for (const void* ptr : dev_ptrs)
    if (!aligned16(ptr)) return GDN_ERR_MISALIGNED;
  if ((state_in && !aligned16(state_in)) || (d_state_out && !aligned16(d_state_out)) ||
      (d_state_in && !aligned16(d_state_in)))
    return GDN_ERR_MISALIGNED;
  // outputs must not overlap the inputs or each other (d_state_in may alias d_state_out: each
  // element is read once before it is written, by the same thread)
  const size_t n = size_t(B) * T * N * H * D * 2, ng = size_t(B) * T * H * 4,
               ns = size_t(B) * H * D * D * 4;
  const void* ins[] = {q, k, v, d_out};
  const void* outs[] = {dq, dk, dv};
  for (const void* o : outs) {
    for (const void* i : ins)
      if (overlaps(o, n, i, n)) return GDN_ERR_INVALID_ARG;
    for (const void* o2 : outs)
      if (o != o2 && overlaps(o, n, o2, n)) return GDN_ERR_INVALID_ARG;
  }
  if (overlaps(d_gamma, ng, d_beta, ng) || overlaps(d_gamma, ng, gamma, ng) ||
      overlaps(d_gamma, ng, beta, ng) || overlaps(d_beta, ng, gamma, ng) ||
      overlaps(d_beta, ng, beta, ng))
    return GDN_ERR_INVALID_ARG;
  if (d_state_in && state_in && overlaps(d_state_in, ns, state_in, ns)) return GDN_ERR_INVALID_ARG;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  const Problem p{B, H, T, N, D, key_scale};
  if (saved) {  // the saved states must not overlap any output
    const size_t sb = fused_ws_bytes(long(B) * H, T, D, T, T);
    const void* outs2[] = {dq, dk, dv};
    for (const void* o : outs2)
      if (overlaps(saved, sb, o, n)) return GDN_ERR_INVALID_ARG;
  }
  return backward_path(dev, q, k, v, gamma, beta, state_in, d_out, d_state_out, dq, dk, dv,
                       d_gamma, d_beta, d_state_in, p, reinterpret_cast<cudaStream_t>(stream),
                       saved);
}


extern "C" {

gdn_status gdn_softmax_attention(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                 gdn_bf16* out, int B, int H, int T, int N, int D,
                                 int frames_per_chunk, float scale, gdn_stream_t stream) {
  if (!q || !k || !v || !out) return GDN_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || T < 1 || N < 1 || D < 1 || frames_per_chunk < 1)
    return GDN_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 128) return GDN_ERR_UNSUPPORTED;
  if (double(T) * N >= 2147483647.0 || double(B) * H * T * N * D > 4.0e18)
    return GDN_ERR_INVALID_ARG;
  if (scale == 0.f) {
    scale = static_cast<float>(1.0 / std::sqrt(double(D)));
  } else if (!(std::isfinite(scale) && scale > 0.f)) {
    return GDN_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return GDN_ERR_MISALIGNED;
  const size_t n = size_t(B) * T * N * H * D * 2;
  if (overlaps(out, n, q, n) || overlaps(out, n, k, n) || overlaps(out, n, v, n))
    return GDN_ERR_INVALID_ARG;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int F = frames_per_chunk < T ? frames_per_chunk : T;
  if (D <= 64) return run_softmax<64>(dev, q, k, v, out, B, H, T, N, D, F, scale, st);
  return run_softmax<128>(dev, q, k, v, out, B, H, T, N, D, F, scale, st);
}


gdn_status gdn_frame_forward_rope(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                  const float* gamma, const float* beta, const float* state_in,
                                  gdn_bf16* out, float* state_out, int B, int H, int T, int N,
                                  int D, float key_scale, int grid_h, int grid_w,
                                  float rope_base, int t_offset, gdn_stream_t stream) {
  if (gdn_status s = validate_common(q, k, v, out, gamma, beta, state_in, state_out, B, H, T, N,
                                     D, key_scale))
    return s;
  resolve_key_scale(key_scale, D, N, &key_scale);  // validated above
  gdn::RopeDims r;
  long n_tab = 0;
  if (gdn_status s = rope_dims(B, T, N, H, D, grid_h, grid_w, rope_base, t_offset, &r, &n_tab))
    return s;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float2* tab = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (gdn_status s = get_rope_table(dev, align256(size_t(n_tab) * sizeof(float2)), st, &tab))
      return s;
    if (gdn_status s = launch_rope_table(tab, r, n_tab, t_offset, rope_base, st)) return s;
  }
  Problem p{B, H, T, N, D, key_scale};
  p.rope = r.ra;
  p.rope.tab = tab;
  return forward_impl(q, k, v, gamma, beta, state_in, out, state_out, p, st);
}


gdn_status gdn_frame_forward(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                             const float* gamma, const float* beta, const float* state_in,
                             gdn_bf16* out, float* state_out, int B, int H, int T, int N, int D,
                             float key_scale, gdn_stream_t stream) {
  if (gdn_status s = validate_common(q, k, v, out, gamma, beta, state_in, state_out, B, H, T, N,
                                     D, key_scale))
    return s;
  resolve_key_scale(key_scale, D, N, &key_scale);  // validated above
  const Problem p{B, H, T, N, D, key_scale};
  return forward_impl(q, k, v, gamma, beta, state_in, out, state_out, p,
                      reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_frame_forward_noalloc(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                     const float* gamma, const float* beta,
                                     const float* state_in, gdn_bf16* out, float* state_out,
                                     int B, int H, int T, int N, int D, float key_scale,
                                     gdn_stream_t stream) {
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  const long count = long(B) * H * T;
  if (forward_ws_bytes(count, D) > kNoAllocScratchBytes) return GDN_ERR_SCRATCH_LIMIT;
  if (gdn_status s = validate_common(q, k, v, out, gamma, beta, state_in, state_out, B, H, T, N,
                                     D, key_scale))
    return s;
  resolve_key_scale(key_scale, D, N, &key_scale);  // validated above
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  void* base = nullptr;
  if (gdn_status s = noalloc_scratch(dev, &base)) return s;
  // Every scratch element (A_t, B_t, S_t) is written by this call before it is read, so nothing
  // needs clearing between calls.
  if (gdn_status s = poison(base, forward_ws_bytes(count, D), reinterpret_cast<cudaStream_t>(stream)))
    return s;
  const ForwardWs w = carve_forward(base, count, D);
  const Problem p{B, H, T, N, D, key_scale};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const gdn::ChainSeg whole{T, 1, 0, nullptr, nullptr};
  if (D <= 64) {
    if (gdn_status s = run_stats<64, true>(dev, p, k, v, w.A, w.B, st)) return s;
    if (gdn_status s = run_chain<64>(dev, p, w.A, w.B, gamma, beta, state_in, w.S, state_out,
                                     whole, st))
      return s;
    return run_output<64, false>(dev, p, q, w.S, D, out, 1, st);
  }
  if (gdn_status s = run_stats<128, true>(dev, p, k, v, w.A, w.B, st)) return s;
  if (gdn_status s = run_chain<128>(dev, p, w.A, w.B, gamma, beta, state_in, w.S, state_out,
                                    whole, st))
    return s;
  return run_output<128, false>(dev, p, q, w.S, D, out, 1, st);
}

gdn_status gdn_frame_forward_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v,
                                 const float* q_scale, const float* k_scale,
                                 const float* v_scale, const float* gamma, const float* beta,
                                 const float* state_in, gdn_bf16* out, float* state_out, int B,
                                 int H, int T, int N, int D, float key_scale,
                                 gdn_stream_t stream) {
  if (!q || !k || !v || !out || !gamma || !beta || !q_scale || !k_scale || !v_scale)
    return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  if (D <= 64 || D % 16 != 0) return GDN_ERR_UNSUPPORTED;
  if (!resolve_key_scale(key_scale, D, N, &key_scale)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return GDN_ERR_MISALIGNED;
  const size_t n8 = size_t(B) * T * N * H * D, n16 = n8 * 2;
  if (overlaps(out, n16, q, n8) || overlaps(out, n16, k, n8) || overlaps(out, n16, v, n8))
    return GDN_ERR_INVALID_ARG;
  Problem p{B, H, T, N, D, key_scale};
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  return forward_impl(q, k, v, gamma, beta, state_in, out, state_out, p,
                      reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_frame_forward_host(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                  const float* gamma, const float* beta, const float* state_in,
                                  gdn_bf16* out, float* state_out, int B, int H, int T, int N,
                                  int D, float key_scale, gdn_stream_t stream) {
  if (!q || !k || !v || !out || !gamma || !beta) return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  if (!resolve_key_scale(key_scale, D, N, &key_scale)) return GDN_ERR_INVALID_ARG;
  const size_t n = size_t(B) * T * N * H * D * 2;
  if (overlaps(out, n, q, n) || overlaps(out, n, k, n) || overlaps(out, n, v, n))
    return GDN_ERR_INVALID_ARG;
  const Problem p{B, H, T, N, D, key_scale};
  return forward_host_impl(q, k, v, gamma, beta, state_in, out, state_out, p,
                           reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_frame_step(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                          const float* gamma, const float* beta, const float* state_in,
                          gdn_bf16* out, float* state_out, int B, int H, int N, int D,
                          float key_scale, gdn_stream_t stream) {
  if (gdn_status s = validate_common(q, k, v, out, gamma, beta, state_in, state_out, B, H, 1, N,
                                     D, key_scale))
    return s;
  resolve_key_scale(key_scale, D, N, &key_scale);  // validated above
  const Problem p{B, H, 1, N, D, key_scale};
  if (D > 64 && g_forward_mode != 1) {
    int dev;
    if (gdn_status s = current_device(&dev)) return s;
    std::lock_guard<std::mutex> lock(g_mu);
    return run_step(dev, p, q, k, v, gamma, beta, state_in, out, state_out,
                    reinterpret_cast<cudaStream_t>(stream));
  }
  return forward_impl(q, k, v, gamma, beta, state_in, out, state_out, p,
                      reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_frame_stats(const gdn_bf16* k, const gdn_bf16* v, gdn_bf16* A_out, float* B_out,
                           int B, int H, int T, int N, int D, float key_scale,
                           gdn_stream_t stream) {
  if (!k || !v || !A_out || !B_out) return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 128)) return s;
  if (!resolve_key_scale(key_scale, D, N, &key_scale)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(A_out) || !aligned16(B_out))
    return GDN_ERR_MISALIGNED;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  const Problem p{B, H, T, N, D, key_scale};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (D <= 64) return run_stats<64, false>(dev, p, k, v, A_out, B_out, st);
  return run_stats<128, false>(dev, p, k, v, A_out, B_out, st);
}

gdn_status gdn_block_causal_la(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                               const float* state_in, const float* z_in, gdn_bf16* out,
                               float* state_out, float* z_out, int B, int H, int T, int N, int D,
                               int frames_per_block, gdn_stream_t stream) {
  if (!q || !k || !v || !out) return GDN_ERR_INVALID_ARG;
  if (frames_per_block < 1) return GDN_ERR_INVALID_ARG;
  if (gdn_status s = check_sizes(B, H, T, N, D, 120)) return s;
  // token rows are addressed as one flattened TMA coordinate
  if (double(B) * T * N >= 2147483647.0) return GDN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GDN_ERR_MISALIGNED;
  const size_t n = size_t(B) * T * N * H * D * 2;
  if (overlaps(out, n, q, n) || overlaps(out, n, k, n) || overlaps(out, n, v, n))
    return GDN_ERR_INVALID_ARG;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Problem p{B, H, T, N, D, 1.0f};
  const int F = frames_per_block < T ? frames_per_block : T;
  const int n_blocks = (T + F - 1) / F;
  const long count = long(B) * H * n_blocks;
  const size_t per = size_t(D + 1) * D;
  void* base = nullptr;
  if (gdn_status s = get_workspace(dev, align256(count * per * 4) + align256(count * per * 2),
                                   st, &base))
    return s;
  float* Bws = static_cast<float*>(base);
  void* Sws = static_cast<uint8_t*>(base) + align256(count * per * 4);
  {
    // per-block statistics: one item per (batch, block, head)
    using L = gdn::StatsLayout<128, true>;
    CUtensorMap tk, tv;
    if (!tmap_rows(&tk, k, p) || !tmap_rows(&tv, v, p)) return GDN_ERR_CUDA;
    auto kern = gdn::gdn_stats_kernel<128, true, false>;
    if (gdn_status s = ensure_smem_attr(dev, 7, kern, L::kSmemBytes)) return s;
    const int grid = static_cast<int>(count < g_dev[dev].sms ? count : g_dev[dev].sms);
    ProfiledLaunch pl("gdn_stats_kernel_la", st);
    kern<<<grid, L::kThreads, L::kSmemBytes, st>>>(tk, tv, nullptr, Bws, p, F);
    if (gdn_status s = check_launch()) return s;
  }
  {
    dim3 grid(static_cast<unsigned>((per + 255) / 256), static_cast<unsigned>(B * H));
    ProfiledLaunch pl("gdn_la_scan_kernel", st);
    gdn::gdn_la_scan_kernel<<<grid, 256, 0, st>>>(Bws, static_cast<__nv_bfloat16*>(Sws), state_in,
                                                  z_in, state_out, z_out, n_blocks, D);
    if (gdn_status s = check_launch()) return s;
  }
  return run_output<128, true>(dev, p, q, Sws, D + 1, out, F, st);
}

gdn_status gdn_frame_backward(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                              const float* gamma, const float* beta, const float* state_in,
                              const gdn_bf16* d_out, const float* d_state_out, gdn_bf16* dq,
                              gdn_bf16* dk, gdn_bf16* dv, float* d_gamma, float* d_beta,
                              float* d_state_in, int B, int H, int T, int N, int D,
                              float key_scale, gdn_stream_t stream) {
  return backward_entry(q, k, v, gamma, beta, state_in, d_out, d_state_out, dq, dk, dv, d_gamma,
                        d_beta, d_state_in, B, H, T, N, D, key_scale, stream, nullptr);
}

size_t gdn_train_saved_bytes(int B, int H, int T, int N, int D) {
  (void)N;
  if (B < 1 || H < 1 || T < 1 || D <= 64 || D > 128) return 0;
  // the three-kernel workspace layout, followed by the fused kernel's hand-off flags
  return fused_ws_bytes(long(B) * H, T, D, T, T);
}

gdn_status gdn_frame_forward_train(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                   const float* gamma, const float* beta, const float* state_in,
                                   gdn_bf16* out, float* state_out, void* saved, int B, int H,
                                   int T, int N, int D, float key_scale, gdn_stream_t stream) {
  if (!saved) return GDN_ERR_INVALID_ARG;
  if (gdn_status s = validate_common(q, k, v, out, gamma, beta, state_in, state_out, B, H, T, N,
                                     D, key_scale))
    return s;
  if (D <= 64) return GDN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(saved) & 255) != 0) return GDN_ERR_MISALIGNED;
  resolve_key_scale(key_scale, D, N, &key_scale);  // validated above
  const long count = long(B) * H * T;
  const size_t sb = fused_ws_bytes(long(B) * H, T, D, T, T), n = size_t(B) * T * N * H * D * 2;
  const void* ins[] = {q, k, v, out};
  for (const void* x : ins)
    if (overlaps(saved, sb, x, n)) return GDN_ERR_INVALID_ARG;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  const Problem p{B, H, T, N, D, key_scale};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the fused kernel with one ring slot per frame writes A_t, B_t, S_t where the backward reads
  // them (the three-kernel workspace layout); else the three kernels write them there
  if (fused_applies(dev, p))
    return run_fused<128>(dev, p, q, k, v, gamma, beta, state_in, out, state_out, st, saved);
  const ForwardWs w = carve_forward(saved, count, D);
  const gdn::ChainSeg whole{T, 1, 0, nullptr, nullptr};
  if (gdn_status s = run_stats<128, true>(dev, p, k, v, w.A, w.B, st)) return s;
  if (gdn_status s = run_chain<128>(dev, p, w.A, w.B, gamma, beta, state_in, w.S, state_out,
                                    whole, st))
    return s;
  return run_output<128, false>(dev, p, q, w.S, D, out, 1, st);
}

gdn_status gdn_frame_backward_saved(const gdn_bf16* q, const gdn_bf16* k, const gdn_bf16* v,
                                    const float* gamma, const float* beta, const float* state_in,
                                    const void* saved, const gdn_bf16* d_out,
                                    const float* d_state_out, gdn_bf16* dq, gdn_bf16* dk,
                                    gdn_bf16* dv, float* d_gamma, float* d_beta,
                                    float* d_state_in, int B, int H, int T, int N, int D,
                                    float key_scale, gdn_stream_t stream) {
  if (!saved) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(saved) & 255) != 0) return GDN_ERR_MISALIGNED;
  return backward_entry(q, k, v, gamma, beta, state_in, d_out, d_state_out, dq, dk, dv, d_gamma,
                        d_beta, d_state_in, B, H, T, N, D, key_scale, stream, saved);
}

gdn_status gdn_rope_3d(const gdn_bf16* x, gdn_bf16* y, int B, int T, int N, int H, int D,
                       int grid_h, int grid_w, float base, int t_offset, gdn_stream_t stream) {
  if (!x || !y) return GDN_ERR_INVALID_ARG;
  gdn::RopeDims r;
  long n_tab = 0;
  if (gdn_status s = rope_dims(B, T, N, H, D, grid_h, grid_w, base, t_offset, &r, &n_tab))
    return s;
  if (!aligned16(x) || !aligned16(y)) return GDN_ERR_MISALIGNED;
  const size_t n = size_t(B) * T * N * H * D * 2;
  if (x != y && overlaps(x, n, y, n)) return GDN_ERR_INVALID_ARG;
  int dev;
  if (gdn_status s = current_device(&dev)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* base_ws = nullptr;
  if (gdn_status s = get_workspace(dev, align256(size_t(n_tab) * sizeof(float2)), st, &base_ws))
    return s;
  float2* tab = static_cast<float2*>(base_ws);
  if (gdn_status s = launch_rope_table(tab, r, n_tab, t_offset, base, st)) return s;
  r.ra.tab = tab;
  // one block row per frame of one batch element, one block per kRopeTokens of its tokens
  const long chunks = (long(N) + gdn::kRopeTokens - 1) / gdn::kRopeTokens;
  if (chunks > 65535) return GDN_ERR_INVALID_ARG;
  {
    ProfiledLaunch pl("gdn_rope_kernel", st);
    // a thread per 16-byte vector of a token (H*D/8 of them, rounded up to whole warps)
    const int per_tok = H * (D / 8);
    const int threads = std::min(gdn::kRopeMaxThreads, (per_tok + 31) / 32 * 32);
    gdn::gdn_rope_kernel<<<dim3(static_cast<unsigned>(B * T), static_cast<unsigned>(chunks)),
                           threads, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                    reinterpret_cast<__nv_bfloat16*>(y), r);
  }
  return check_launch();
}

size_t gdn_backward_workspace_bytes(int B, int H, int T, int N, int D) {
  (void)N;
  if (B < 1 || H < 1 || T < 1 || D < 1) return 0;
  return backward_ws_bytes(long(B) * H * T, D, long(B) * H);
}

size_t gdn_workspace_bytes(int B, int H, int T, int N, int D) {
  (void)N;
  if (B < 1 || H < 1 || T < 1 || D < 1) return 0;
  const size_t split = forward_ws_bytes(long(B) * H * T, D);
  const size_t fused = fused_ws_bytes(long(B) * H, T, D);
  // chunked: chunks of at least 4 frames unless GDN_CHUNK_LEN asks for shorter ones
  const int forced = chunk_len_override();
  const int min_len = forced > 0 && forced < 4 ? forced : 4;
  const size_t chunked = chunked_ws_bytes(long(B) * H, T, D, (T + min_len - 1) / min_len);
  size_t m = split > fused ? split : fused;
  return m > chunked ? m : chunked;
}

size_t gdn_la_workspace_bytes(int B, int H, int T, int D) {
  if (B < 1 || H < 1 || T < 1 || D < 1) return 0;
  // upper bound: one block per frame
  const size_t count = size_t(B) * H * T, per = size_t(D + 1) * D;
  return align256(count * per * 4) + align256(count * per * 2);
}

const char* gdn_status_string(gdn_status status) {
  switch (status) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported head dimension";
    case GDN_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case GDN_ERR_NO_MEMORY: return "workspace allocation failed";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device-side wait timed out";
    case GDN_ERR_SCRATCH_LIMIT:
      return "problem needs more than the 64 MiB fixed scratch of gdn_frame_forward_noalloc";
  }
  return "unknown status";
}

gdn_status gdn_sync_status(gdn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GDN_ERR_CUDA;
  int code = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&code, gdn::g_status, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  if (code != 0 && cudaMemcpyToSymbol(gdn::g_status, &zero, sizeof(int)) != cudaSuccess)
    return GDN_ERR_CUDA;
  return static_cast<gdn_status>(code);
}

void gdn_release_workspace(void) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& d = g_dev[dev];
  cudaDeviceSynchronize();
  if (d.ws) cudaFree(d.ws);
  d.ws = nullptr;
  d.ws_bytes = 0;
  // per-context facts cached on the host: looked up again by the next call (after a context
  // reset the old kernel attributes and the scratch address no longer hold)
  d.attr_done = 0;
  g_noalloc_addr[dev] = nullptr;
  if (d.rope_tab) cudaFree(d.rope_tab);
  d.rope_tab = nullptr;
  d.rope_tab_bytes = 0;
  {
    std::lock_guard<std::mutex> pl(g_pipe_mu);
    HostPipe& hp = g_pipe[dev];
    if (hp.ready) {
      if (hp.buf) cudaFree(hp.buf);
      cudaStreamDestroy(hp.s_in);
      cudaStreamDestroy(hp.s_out);
      cudaEvent_t evs[] = {hp.entry, hp.in_done[0], hp.in_done[1], hp.comp_done[0],
                           hp.comp_done[1], hp.out_done[0], hp.out_done[1], hp.fin};
      for (cudaEvent_t e : evs) cudaEventDestroy(e);
    }
    hp = HostPipe();
  }
  if (d.step_flags) cudaFree(d.step_flags);
  d.step_flags = nullptr;
  d.step_items = 0;
  d.step_epoch = 0;
  for (cudaEvent_t& e : d.ev) {
    if (e) cudaEventDestroy(e);
    e = nullptr;
  }
  if (d.aux) cudaStreamDestroy(d.aux);
  d.aux = nullptr;
  cudaGetLastError();  // handles of a context that was reset report errors: nothing to act on
}

int gdn_version(void) { return 100; }

int gdn_debug_checks(void) {
#ifdef GDN_DEBUG
  return 1;
#else
  return 0;
#endif
}

int gdn_debug_report(int* site, long long* value) {
  int s = 0;
  long long v = 0;
  if (cudaMemcpyFromSymbol(&s, gdn::g_debug_site, sizeof(int)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&v, gdn::g_debug_value, sizeof(long long)) != cudaSuccess)
    return -1;
  if (site) *site = s;
  if (value) *value = v;
  if (s != 0) {
    const int zero = 0;
    const long long zl = 0;
    if (cudaMemcpyToSymbol(gdn::g_debug_site, &zero, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(gdn::g_debug_value, &zl, sizeof(long long)) != cudaSuccess)
      return -1;
  }
  return s != 0 ? 1 : 0;
}

gdn_status gdn_profile_arm(void* const* events, int n) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (events == nullptr || n < 2) {
    g_prof_events = nullptr;
    g_prof_n = 0;
  } else {
    g_prof_events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
    g_prof_n = n;
  }
  g_prof_count = 0;
  return GDN_OK;
}

int gdn_profile_count(void) { return g_prof_count; }

gdn_status gdn_set_forward_mode(int mode) {
  if (mode < 0 || mode > 3) return GDN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_forward_mode = mode;
  return GDN_OK;
}

const char* gdn_profile_kernel(int i) {
  if (i < 0 || i >= g_prof_count) return "";
  return g_prof_names[i];
}

}  // extern "C"
