// Host side of libsinkattn.so: argument validation, TMA descriptors and
// launches for the C ABI declared in include/sink_attn.h.  Everything here is
// plain host logic; all attention arithmetic runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sink_attn.h"

#include "common.cuh"
#include "tma_host.cuh"
#include "fwd_kernel.cuh"
#include "fwd_pair_kernel.cuh"
#include "bwd_kernels.cuh"
#include "decode_kernel.cuh"

namespace sa {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2_exact(int x) {
  if (x <= 0 || (x & (x - 1)) != 0) return -1;
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

// Validates the sizes and fills the geometry.  T == 0 is valid (no work).
sink_attn_status check_dims(const sink_attn_dims* d, const int* cu_seqlens, bool packed, int window, float scale,
                            Geometry* geo) {
  if (!d) return SINK_ATTN_ERR_NULL;
  if (d->batch < 0 || d->max_seqlen < 0 || d->total_tokens < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
      d->head_dim <= 0)
    return SINK_ATTN_ERR_SHAPE;
  if (d->num_q_heads % d->num_kv_heads != 0) return SINK_ATTN_ERR_SHAPE;
  if (!packed && static_cast<int64_t>(d->batch) * d->max_seqlen != d->total_tokens)
    return SINK_ATTN_ERR_SHAPE;
  if (d->total_tokens > 0 && d->batch == 0) return SINK_ATTN_ERR_SHAPE;
  if (d->head_dim != kHeadDim) return SINK_ATTN_ERR_UNSUPPORTED;
  const int G = d->num_q_heads / d->num_kv_heads;
  const int gl = ilog2_exact(G);
  if (gl < 0 || G > kBlockM) return SINK_ATTN_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SINK_ATTN_ERR_UNSUPPORTED;
  // Token and element indices are formed in 32-bit ints in places.
  if (static_cast<int64_t>(d->total_tokens) * d->num_q_heads * kHeadDim >= (int64_t(1) << 40) ||
      d->total_tokens > (1 << 30))
    return SINK_ATTN_ERR_UNSUPPORTED;
  geo->T = d->total_tokens;
  geo->Hq = d->num_q_heads;
  geo->Hkv = d->num_kv_heads;
  geo->G_log2 = gl;
  geo->P_log2 = 7 - gl;
  geo->num_qblocks = (d->total_tokens + (1 << geo->P_log2) - 1) >> geo->P_log2;
  geo->batch = d->batch;
  geo->seqlen = d->max_seqlen;
  geo->cu_seqlens = cu_seqlens;
  geo->window = window > 0 ? window : 0;
  if (!packed && d->total_tokens > 0 && d->max_seqlen <= 0) return SINK_ATTN_ERR_SHAPE;
  return SINK_ATTN_OK;
}

// Checks of a forward call (both forward entry points): sizes, then (for
// T > 0) pointers and alignment.  Fills the geometry.
sink_attn_status check_fwd_args(const sink_attn_dims* d, const void* q, const void* k, const void* v,
                                const float* sinks, const int* cu_seqlens, int window, float scale, const void* out,
                                const float* lse, Geometry* geo) {
  sink_attn_status st = check_dims(d, cu_seqlens, cu_seqlens != nullptr, window, scale, geo);
  if (st != SINK_ATTN_OK || geo->T == 0) return st;
  if (!q || !k || !v || !sinks || !out || !lse) return SINK_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(sinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return SINK_ATTN_ERR_ALIGN;
  return SINK_ATTN_OK;
}

// The forward kernel sink_attn_fwd runs: two query tiles per CTA for every
// size.  Timed against one tile per CTA on B200 (interleaved CUDA-event
// runs): 21% faster on sliding-window-128 layers, where a one-tile CTA does
// only a few 64-key steps between its set-up and its epilogue, and 1-4%
// faster on full-causal layers (4k, 60k, packed documents), where both are
// bound by each warpgroup's S round trip and the exp2 unit.
int fwd_auto_kernel(const Geometry&) { return SINK_ATTN_FWD_TWO_TILES; }

// 3-D bf16 view [outer][mid][inner] with a box {box_inner, 1, box_outer}
// under the given swizzle: the pair forward's half-steps of K (32 keys x 64
// dims, 128-byte rows) and V (64 keys x 32 dims, 64-byte rows).
bool make_map_3d_box(CUtensorMap* map, const void* base, int inner, int mid, int outer, int box_inner,
                     int box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(mid),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2, static_cast<cuuint64_t>(inner) * mid * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Events registered by sink_attn_profile_events: [which][begin/end].
cudaEvent_t g_profile_events[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};


// Decode: sizes, split count and workspace layout of one call.
struct DecPlan {
  DecParams p;
  size_t o_off, m_off, l_off, total;  // workspace layout (bytes)
};

// CTAs that run at once (two per SM of a 148-SM B200), and a cap on the
// splits of one (sequence, key/value head).
constexpr int kDecTargetCtas = 296;
constexpr int kDecMaxSplit = 64;

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

sink_attn_status plan_decode(const sink_attn_decode_dims* d, int window, float scale, DecPlan* plan) {
  if (!d) return SINK_ATTN_ERR_NULL;
  if (d->batch < 0 || d->new_tokens <= 0 || d->cache_capacity <= 0 || d->max_seqlen < d->new_tokens ||
      d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0)
    return SINK_ATTN_ERR_SHAPE;
  if (d->num_q_heads % d->num_kv_heads != 0) return SINK_ATTN_ERR_SHAPE;
  if (d->head_dim != kHeadDim) return SINK_ATTN_ERR_UNSUPPORTED;
  const int G = d->num_q_heads / d->num_kv_heads;
  const int gl = ilog2_exact(G);
  if (gl < 0 || static_cast<int64_t>(G) * d->new_tokens > kDecRows) return SINK_ATTN_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SINK_ATTN_ERR_UNSUPPORTED;
  // Slot and element indices are formed in 32-bit ints in places.
  if (static_cast<int64_t>(d->batch) * d->cache_capacity > (int64_t(1) << 30) ||
      static_cast<int64_t>(d->max_seqlen) + kDecTile > (int64_t(1) << 30) ||
      static_cast<int64_t>(d->batch) * d->new_tokens * d->num_q_heads > (int64_t(1) << 30))
    return SINK_ATTN_ERR_UNSUPPORTED;
  DecParams& p = plan->p;
  p.batch = d->batch;
  p.Lq = d->new_tokens;
  p.C = d->cache_capacity;
  p.Hq = d->num_q_heads;
  p.Hkv = d->num_kv_heads;
  p.G = G;
  p.G_log2 = gl;
  p.R = G * d->new_tokens;
  p.window = window > 0 ? window : 0;
  p.scale_log2 = scale * kLog2e;
  p.seqlens = nullptr;
  p.sinks = nullptr;
  p.k_scale = p.v_scale = nullptr;
  p.o_part = p.m_part = p.l_part = nullptr;
  p.out = nullptr;
  p.lse_out = nullptr;
  // Upper bound on the 128-slot tiles one sequence scans.
  int64_t slots = std::min<int64_t>(d->cache_capacity, d->max_seqlen);
  if (p.window > 0) slots = std::min<int64_t>(slots, static_cast<int64_t>(p.window) + d->new_tokens - 1 + kDecTile);
  const int tiles = static_cast<int>((slots + kDecTile - 1) / kDecTile) + 1;
  const int64_t pairs = static_cast<int64_t>(d->batch) * d->num_kv_heads;
  // Split count: the CTAs run in waves of kDecTargetCtas, each CTA over
  // ceil(tiles / split) tiles plus about one tile's worth of fixed cost
  // (set-up, Q load, partial results); pick the split with the fewest
  // tile-times, preferring fewer splits on ties.
  int split = 1;
  if (pairs > 0) {
    int64_t best = -1;
    for (int k = 1; k <= std::min(tiles, kDecMaxSplit); ++k) {
      const int64_t waves = (pairs * k + kDecTargetCtas - 1) / kDecTargetCtas;
      const int64_t cost = waves * ((tiles + k - 1) / k + 1);
      if (best < 0 || cost < best) {
        best = cost;
        split = k;
      }
    }
  }
  p.n_split = split;
  const size_t parts = static_cast<size_t>(pairs) * split * kDecRows;
  plan->o_off = 0;
  plan->m_off = round256(parts * kHeadDim * sizeof(float));
  plan->l_off = plan->m_off + round256(parts * sizeof(float));
  plan->total = plan->l_off + round256(parts * sizeof(float));
  return SINK_ATTN_OK;
}

}  // namespace

// Self-test of the bounded waits every kernel uses, on an mbarrier that
// nothing ever completes.  Thread 0 gives up after limit_ns and raises the
// CTA's abort flag; thread 32 (another warp) waits with ten times that limit
// and must leave through the flag.  out[0], out[2]: 1 if the wait returned
// true (neither should); out[1], out[3]: microseconds each waited.
__global__ void __launch_bounds__(64) sink_attn_selftest_wait_kernel(unsigned long long limit_ns, int* out) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0 || threadIdx.x == 32) {
    const bool first = threadIdx.x == 0;
    const uint64_t t0 = global_timer_ns();
    const bool ok = first ? mbar_wait_for(&bar[0], 0, abort, &g_device_error, kDevErrTimeoutSelfTest, limit_ns)
                          : mbar_wait_for(&bar[1], 0, abort, &g_device_error, kDevErrTimeoutSelfTestAbort,
                                          10ull * limit_ns);
    const uint64_t us = (global_timer_ns() - t0) / 1000ull;
    out[first ? 0 : 2] = ok ? 1 : 0;
    out[first ? 1 : 3] = static_cast<int>(us < 0x7fffffffull ? us : 0x7fffffffull);
  }
}

}  // namespace sa

using namespace sa;

extern "C" {

const char* sink_attn_status_string(sink_attn_status s) {
  switch (s) {
    case SINK_ATTN_OK: return "ok";
    case SINK_ATTN_ERR_NULL: return "a required pointer is NULL";
    case SINK_ATTN_ERR_SHAPE: return "inconsistent sizes";
    case SINK_ATTN_ERR_ALIGN: return "a tensor is not 16-byte aligned";
    case SINK_ATTN_ERR_UNSUPPORTED: return "unsupported configuration (D must be 64, Hq/Hkv a power of two <= 128, scale > 0)";
    case SINK_ATTN_ERR_CUDA: return "CUDA call failed";
    case SINK_ATTN_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out";
    case SINK_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

sink_attn_status sink_attn_profile_events(int which, void* ev_begin, void* ev_end) {
  if (which < 0 || which > 1) return SINK_ATTN_ERR_SHAPE;
  g_profile_events[which][0] = static_cast<cudaEvent_t>(ev_begin);
  g_profile_events[which][1] = static_cast<cudaEvent_t>(ev_end);
  return SINK_ATTN_OK;
}

sink_attn_status sink_attn_selftest_wait(unsigned long long limit_ns, int* out, void* stream) {
  if (out == nullptr || (reinterpret_cast<uintptr_t>(out) & 3u) != 0) return SINK_ATTN_ERR_ALIGN;
  if (limit_ns == 0 || limit_ns > kWaitLimitNs) return SINK_ATTN_ERR_SHAPE;
  sink_attn_selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, out);
  return cudaGetLastError() == cudaSuccess ? SINK_ATTN_OK : SINK_ATTN_ERR_CUDA;
}

int sink_attn_last_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

int sink_attn_device_error(void* stream) { return sink_attn_last_device_error(stream); }

int sink_attn_fwd_launches(const sink_attn_dims* d) {
  Geometry geo;
  if (check_dims(d, nullptr, true, 0, 1.f, &geo) != SINK_ATTN_OK) return 0;
  return d->total_tokens > 0 ? 1 : 0;
}

sink_attn_status sink_attn_fwd(const sink_attn_dims* d, const void* q, const void* k, const void* v,
                               const float* sinks, const int* cu_seqlens, int window, float scale, void* out,
                               float* lse, void* stream) {
  return sink_attn_fwd_with(d, q, k, v, sinks, cu_seqlens, window, scale, out, lse, SINK_ATTN_FWD_AUTO, stream);
}

sink_attn_status sink_attn_fwd_pair(const sink_attn_dims* d, const void* q, const void* k, const void* v,
                                    const float* sinks, const int* cu_seqlens, int window, float scale, void* out,
                                    float* lse, void* stream) {
  return sink_attn_fwd_with(d, q, k, v, sinks, cu_seqlens, window, scale, out, lse, SINK_ATTN_FWD_CTA_PAIR,
                            stream);
}

int sink_attn_fwd_kernel_for(const sink_attn_dims* d, int window) {
  Geometry geo;
  if (check_dims(d, nullptr, true, window, 1.f, &geo) != SINK_ATTN_OK) return -1;
  return fwd_auto_kernel(geo);
}

sink_attn_status sink_attn_fwd_with(const sink_attn_dims* d, const void* q, const void* k, const void* v,
                                    const float* sinks, const int* cu_seqlens, int window, float scale, void* out,
                                    float* lse, int kernel, void* stream) {
  if (kernel < SINK_ATTN_FWD_AUTO || kernel > SINK_ATTN_FWD_CTA_PAIR) return SINK_ATTN_ERR_UNSUPPORTED;
  Geometry geo;
  sink_attn_status st = check_fwd_args(d, q, k, v, sinks, cu_seqlens, window, scale, out, lse, &geo);
  if (st != SINK_ATTN_OK || geo.T == 0) return st;
  if (kernel == SINK_ATTN_FWD_AUTO) kernel = fwd_auto_kernel(geo);

  const int G = 1 << geo.G_log2;
  const bool pair = kernel == SINK_ATTN_FWD_CTA_PAIR;
  CUtensorMap tq, tk, tv;
  if (!make_map_3d(&tq, q, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2)) return SINK_ATTN_ERR_CUDA;
  if (pair) {
    // Each CTA of a pair loads 32 keys x 64 dims of K and 64 keys x 32 dims
    // of V per 64-key step.
    if (!make_map_3d_box(&tk, k, kHeadDim, geo.Hkv, geo.T, kHeadDim, kHalfN / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d_box(&tv, v, kHeadDim, geo.Hkv, geo.T, kHeadDim / 2, kHalfN, CU_TENSOR_MAP_SWIZZLE_64B))
      return SINK_ATTN_ERR_CUDA;
  } else if (!make_map_3d(&tk, k, kHeadDim, geo.Hkv, geo.T, 1, kBlockN) ||
             !make_map_3d(&tv, v, kHeadDim, geo.Hkv, geo.T, 1, kBlockN)) {
    return SINK_ATTN_ERR_CUDA;
  }

  FwdParams p;
  p.geo = geo;
  p.scale_log2 = scale * kLog2e;
  p.sinks = sinks;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  // One tile: a CTA per (query tile, head g); two tiles and pairs: a CTA per
  // two query tiles, or a pair of CTAs per two query tiles.
  const int64_t units = kernel == SINK_ATTN_FWD_ONE_TILE ? geo.num_qblocks : (geo.num_qblocks + 1) / 2;
  const int64_t grid = units * geo.Hkv * (pair ? 2 : 1);
  if (grid > 0x7fffffff) return SINK_ATTN_ERR_UNSUPPORTED;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kFwdThreads, 1, 1);
  cfg.stream = st_;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaError_t e;
  if (g_profile_events[0][0]) cudaEventRecord(g_profile_events[0][0], st_);
  if (kernel == SINK_ATTN_FWD_ONE_TILE) {
    static SmemAttrOnce smem_set;
    cfg.dynamicSmemBytes = fwd_smem_bytes<1>();
    e = smem_set.ensure(sink_attn_fwd_kernel<1>, cfg.dynamicSmemBytes)
            ? cudaLaunchKernelEx(&cfg, sink_attn_fwd_kernel<1>, tq, tk, tv, p)
            : cudaErrorInvalidValue;
  } else if (kernel == SINK_ATTN_FWD_TWO_TILES) {
    static SmemAttrOnce smem_set;
    cfg.dynamicSmemBytes = fwd_smem_bytes<2>();
    e = smem_set.ensure(sink_attn_fwd_kernel<2>, cfg.dynamicSmemBytes)
            ? cudaLaunchKernelEx(&cfg, sink_attn_fwd_kernel<2>, tq, tk, tv, p)
            : cudaErrorInvalidValue;
  } else {
    static SmemAttrOnce smem_set;
    cfg.dynamicSmemBytes = kF2SmemBytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = smem_set.ensure(sink_attn_fwd_pair_kernel, cfg.dynamicSmemBytes)
            ? cudaLaunchKernelEx(&cfg, sink_attn_fwd_pair_kernel, tq, tk, tv, p)
            : cudaErrorInvalidValue;
  }
  if (g_profile_events[0][1]) cudaEventRecord(g_profile_events[0][1], st_);
  return e == cudaSuccess ? SINK_ATTN_OK : SINK_ATTN_ERR_CUDA;
}

size_t sink_attn_bwd_workspace_size(const sink_attn_dims* d) {
  Geometry geo;
  if (check_dims(d, nullptr, true, 0, 1.f, &geo) != SINK_ATTN_OK) return 0;
  return bwd_workspace_layout(geo).total;
}

int sink_attn_bwd_launches(const sink_attn_dims* d) {
  Geometry geo;
  if (check_dims(d, nullptr, true, 0, 1.f, &geo) != SINK_ATTN_OK) return 0;
  return d->total_tokens > 0 ? kBwdLaunches : 0;
}

sink_attn_status sink_attn_bwd(const sink_attn_dims* d, const void* q, const void* k, const void* v,
                               const float* sinks, const int* cu_seqlens, int window, float scale, const void* out,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv, float* dsinks,
                               void* workspace, size_t workspace_bytes, void* stream) {
  Geometry geo;
  sink_attn_status st = check_dims(d, cu_seqlens, cu_seqlens != nullptr, window, scale, &geo);
  if (st != SINK_ATTN_OK) return st;
  if (!dsinks) return SINK_ATTN_ERR_NULL;
  if (geo.T == 0) {
    // No rows: every sink gradient is an empty sum.
    return cudaMemsetAsync(dsinks, 0, sizeof(float) * geo.Hq, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SINK_ATTN_OK
               : SINK_ATTN_ERR_CUDA;
  }
  if (!q || !k || !v || !sinks || !out || !lse || !dout || !dq || !dk || !dv) return SINK_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(sinks) & 3u) || (reinterpret_cast<uintptr_t>(dsinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return SINK_ATTN_ERR_ALIGN;
  const BwdWorkspace ws = bwd_workspace_layout(geo);
  if (!workspace || workspace_bytes < ws.total) return SINK_ATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SINK_ATTN_ERR_ALIGN;
  return bwd_launch(geo, scale, q, k, v, sinks, out, lse, dout, dq, dk, dv, dsinks,
                    static_cast<uint8_t*>(workspace), ws, static_cast<cudaStream_t>(stream), g_profile_events[1][0],
                    g_profile_events[1][1]);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Backward without caller-provided workspace, for callers that cannot
// allocate device memory (see sink_attn_bwd_noalloc in sink_attn.h).  The
// scratch is this fixed array; host code must not use its name as a device
// address (it is a host-side stand-in), so its address is looked up once per
// device with cudaGetSymbolAddress and cached.
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[SINK_ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, or nullptr.
void* noalloc_scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" sink_attn_status sink_attn_bwd_noalloc(const sink_attn_dims* d, const void* q, const void* k,
                                                  const void* v, const float* sinks, const int* cu_seqlens,
                                                  int window, float scale, const void* out, const float* lse,
                                                  const void* dout, void* dq, void* dk, void* dv, float* dsinks,
                                                  void* stream) {
  Geometry geo;
  sink_attn_status st = check_dims(d, cu_seqlens, cu_seqlens != nullptr, window, scale, &geo);
  if (st != SINK_ATTN_OK) return st;
  const size_t need = bwd_workspace_layout(geo).total;
  if (need > SINK_ATTN_NOALLOC_SCRATCH_BYTES) return SINK_ATTN_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_for_current_device();
  if (scratch == nullptr) return SINK_ATTN_ERR_CUDA;
  return sink_attn_bwd(d, q, k, v, sinks, cu_seqlens, window, scale, out, lse, dout, dq, dk, dv, dsinks, scratch,
                       SINK_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" {

size_t sink_attn_decode_workspace_size(const sink_attn_decode_dims* d, int window) {
  DecPlan plan;
  if (plan_decode(d, window, 1.f, &plan) != SINK_ATTN_OK) return 0;
  return plan.total;
}

int sink_attn_decode_launches(const sink_attn_decode_dims* d, int window) {
  DecPlan plan;
  if (plan_decode(d, window, 1.f, &plan) != SINK_ATTN_OK) return 0;
  return d->batch > 0 ? (plan.p.n_split > 1 ? 3 : 2) : 0;
}

}  // extern "C"

namespace {

// mode: 0 bf16 cache; 1 e4m3 cache, fp16 MMAs; 2 e4m3 cache, FP8 PV.
sink_attn_status decode_impl(const sink_attn_decode_dims* d, const void* q, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, const int* cache_seqlens, const float* k_scale,
                             const float* v_scale, int mode, const float* sinks, int window, float scale, void* out,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  const bool e4m3 = mode != 0;
  DecPlan plan;
  sink_attn_status st = plan_decode(d, window, scale, &plan);
  if (st != SINK_ATTN_OK) return st;
  if (d->batch == 0) return SINK_ATTN_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_seqlens || !sinks || !out || !lse ||
      (e4m3 && (!k_scale || !v_scale)))
    return SINK_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(sinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    return SINK_ATTN_ERR_ALIGN;
  if (!workspace || workspace_bytes < plan.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SINK_ATTN_ERR_WORKSPACE;
  DecParams p = plan.p;
  p.seqlens = cache_seqlens;
  p.sinks = sinks;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.o_part = reinterpret_cast<float*>(ws + plan.o_off);
  p.m_part = reinterpret_cast<float*>(ws + plan.m_off);
  p.l_part = reinterpret_cast<float*>(ws + plan.l_off);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse_out = lse;

  CUtensorMap tq, tk, tv;
  if (!make_map_3d(&tq, q, kHeadDim, p.Hq, p.batch * p.Lq, p.G, p.Lq)) return SINK_ATTN_ERR_CUDA;
  if (e4m3) {
    if (!make_map_3d_u8(&tk, k_cache, kHeadDim, p.Hkv, p.batch * p.C, 1, kDecTile) ||
        !make_map_3d_u8(&tv, v_cache, kHeadDim, p.Hkv, p.batch * p.C, 1, kDecTile))
      return SINK_ATTN_ERR_CUDA;
  } else if (!make_map_3d(&tk, k_cache, kHeadDim, p.Hkv, p.batch * p.C, 1, kDecTile) ||
             !make_map_3d(&tv, v_cache, kHeadDim, p.Hkv, p.batch * p.C, 1, kDecTile)) {
    return SINK_ATTN_ERR_CUDA;
  }
  // Register arrays sized for the real query rows.
  using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, DecParams);
  static const Kern kerns[3][4] = {
      {sink_attn_decode_kernel<8, 0>, sink_attn_decode_kernel<16, 0>, sink_attn_decode_kernel<32, 0>,
       sink_attn_decode_kernel<64, 0>},
      {sink_attn_decode_kernel<8, 1>, sink_attn_decode_kernel<16, 1>, sink_attn_decode_kernel<32, 1>,
       sink_attn_decode_kernel<64, 1>},
      {sink_attn_decode_kernel<8, 2>, sink_attn_decode_kernel<16, 2>, sink_attn_decode_kernel<32, 2>,
       sink_attn_decode_kernel<64, 2>}};
  static SmemAttrOnce smem_set[3][4];
  const int vi = p.R <= 8 ? 0 : (p.R <= 16 ? 1 : (p.R <= 32 ? 2 : 3));
  const Kern kern = kerns[mode][vi];
  const size_t smem = mode == 2 ? kDecSmemBytesPv8 : (mode == 1 ? kDecSmemBytes8 : kDecSmemBytes);
  if (!smem_set[mode][vi].ensure(kern, smem)) return SINK_ATTN_ERR_CUDA;
  const long long ctas = static_cast<long long>(p.batch) * p.Hkv * p.n_split;
  if (ctas > 0x7fffffff) return SINK_ATTN_ERR_UNSUPPORTED;

  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  if (e4m3) {
    const long long chunks = 2LL * p.batch * p.Lq * p.Hkv * (kHeadDim / 16);
    sink_attn_cache_append_e4m3_kernel<<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, st_>>>(
        p, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache));
  } else {
    const long long chunks = 2LL * p.batch * p.Lq * p.Hkv * (kHeadDim * 2 / 16);
    sink_attn_cache_append_kernel<<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, st_>>>(
        p, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache));
  }
  kern<<<static_cast<unsigned>(ctas), e4m3 ? kDecThreads8 : kDecThreads, smem, st_>>>(tq, tk, tv, p);
  if (p.n_split > 1) {
    const long long rows = static_cast<long long>(p.batch) * p.Lq * p.Hq;
    sink_attn_decode_combine_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st_>>>(
        p, static_cast<__nv_bfloat16*>(out), lse);
  }
  return cudaPeekAtLastError() == cudaSuccess ? SINK_ATTN_OK : SINK_ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

sink_attn_status sink_attn_decode(const sink_attn_decode_dims* d, const void* q, const void* k_new,
                                  const void* v_new, void* k_cache, void* v_cache, const int* cache_seqlens,
                                  const float* sinks, int window, float scale, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(d, q, k_new, v_new, k_cache, v_cache, cache_seqlens, nullptr, nullptr, 0, sinks, window,
                     scale, out, lse, workspace, workspace_bytes, stream);
}

sink_attn_status sink_attn_decode_e4m3(const sink_attn_decode_dims* d, const void* q, const void* k_new,
                                       const void* v_new, void* k_cache, void* v_cache, const int* cache_seqlens,
                                       const float* k_scale, const float* v_scale, const float* sinks, int window,
                                       float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  return decode_impl(d, q, k_new, v_new, k_cache, v_cache, cache_seqlens, k_scale, v_scale, 1, sinks, window,
                     scale, out, lse, workspace, workspace_bytes, stream);
}

sink_attn_status sink_attn_decode_e4m3_f8pv(const sink_attn_decode_dims* d, const void* q, const void* k_new,
                                            const void* v_new, void* k_cache, void* v_cache,
                                            const int* cache_seqlens, const float* k_scale, const float* v_scale,
                                            const float* sinks, int window, float scale, void* out, float* lse,
                                            void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(d, q, k_new, v_new, k_cache, v_cache, cache_seqlens, k_scale, v_scale, 2, sinks, window,
                     scale, out, lse, workspace, workspace_bytes, stream);
}

}  // extern "C"
