// Backward kernels: gradients of causal GQA sink attention.
//
//   P_ij = e^{l_ij - lse_i}, P_sink,i = e^{s_h - lse_i}, D_i = dout_i . out_i
//   dS_ij = P_ij (dout_i . v_j - D_i)
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_{i,h in group} dS_ij q_i,
//   dv_j = sum_{i,h in group} P_ij dout_i,  dsinks_h = -sum_i P_sink,i D_i
//
// Three launches on the caller's stream:
//   1. bwd_preprocess: D_i (fp32, [Hq][T]), per-block partial sums of
//      -P_sink,i D_i (fixed order), and zeroes the fp32 dq accumulator.
//   2. bwd_main (tcgen05): one CTA per 128-key tile of one key/value head g.
//      It visits every query tile (the fwd's 128 rows = 128/G tokens x G
//      heads) that can see one of its keys and computes, with keys on the
//      TMEM lanes:  S^T = K Q^T, dP^T = V dO^T (MMA), P and dS (1 thread =
//      1 key), dV += P^T dO, dK += dS^T Q (MMA, A operand from TMEM: dK and
//      dV sum over all G heads of the group inside TMEM, no atomics), and
//      dQ = dS K (MMA, A operand = dS staged in shared memory) which is added
//      to the fp32 accumulator with vector atomics.
//   3. bwd_finish: dq = bf16(scale * accumulator), and dsinks_h = fixed-order
//      tree sum of the partials (bitwise reproducible).
#pragma once
#include "common.cuh"
#include "tma_host.cuh"

namespace sa {

constexpr int kBwdLaunches = 3;
constexpr int kPreThreads = 256;  // tokens per preprocess CTA (one head per CTA)
constexpr int kBwdThreads = 320;  // 10 warps
constexpr int kBwdStages = 2;
constexpr uint32_t kBwdTmemCols = 512;
constexpr uint32_t kBwdTmemS = 0;     // S^T fp32 [128 keys][128 rows]; P^T (bf16) aliases cols 0..63
constexpr uint32_t kBwdTmemDP = 128;  // dP^T fp32; dS^T (bf16) aliases cols 128..191
constexpr uint32_t kBwdTmemDV = 256;  // dV accumulator fp32 [128 keys][64]
constexpr uint32_t kBwdTmemDK = 320;  // dK accumulator
constexpr uint32_t kBwdTmemDQ = 384;  // dQ tile fp32 [128 rows][64]
constexpr int kFinishThreads = 256;

struct BwdWorkspace {
  size_t dq_acc;    // fp32 [T][Hq][D]
  size_t Dvec;      // fp32 [Hq][T]
  size_t partials;  // fp32 [Hq][num_pre_blocks]
  int num_pre_blocks;
  size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline BwdWorkspace bwd_workspace_layout(const Geometry& geo) {
  BwdWorkspace w;
  const size_t T = static_cast<size_t>(geo.T);
  w.num_pre_blocks = static_cast<int>((T + kPreThreads - 1) / kPreThreads);
  w.dq_acc = 0;
  w.Dvec = align_up(T * geo.Hq * kHeadDim * sizeof(float), 256);
  w.partials = w.Dvec + align_up(T * geo.Hq * sizeof(float), 256);
  w.total = w.partials + align_up(static_cast<size_t>(geo.Hq) * (w.num_pre_blocks > 0 ? w.num_pre_blocks : 1) *
                                      sizeof(float),
                                  256);
  return w;
}

// ------------------------------------------------------------ preprocess
struct PreParams {
  int T, Hq;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  const float* lse;
  const float* sinks;
  float* Dvec;
  float* partials;
  float* dq_acc;
  int num_pre_blocks;
};

__device__ __forceinline__ float dot8_bf16(uint4 a, uint4 b) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fx = __bfloat1622float2(x[i]);
    const float2 fy = __bfloat1622float2(y[i]);
    s = fmaf(fx.x, fy.x, s);
    s = fmaf(fx.y, fy.y, s);
  }
  return s;
}

// Grid (num_pre_blocks, Hq); thread = one token of head blockIdx.y.
__global__ void __launch_bounds__(kPreThreads) sink_attn_bwd_preprocess_kernel(const PreParams p) {
  __shared__ float warp_sums[kPreThreads / 32];
  const int h = blockIdx.y;
  const int t = blockIdx.x * kPreThreads + threadIdx.x;
  float contrib = 0.f;
  if (t < p.T) {
    const size_t row = (static_cast<size_t>(t) * p.Hq + h) * kHeadDim;
    const uint4* o = reinterpret_cast<const uint4*>(p.out + row);
    const uint4* g = reinterpret_cast<const uint4*>(p.dout + row);
    float D = 0.f;
#pragma unroll
    for (int i = 0; i < kHeadDim / 8; ++i) D += dot8_bf16(__ldg(o + i), __ldg(g + i));
    p.Dvec[static_cast<size_t>(h) * p.T + t] = D;
    const float lse = __ldg(p.lse + static_cast<size_t>(h) * p.T + t);
    const float psink = ex2_approx((__ldg(p.sinks + h) - lse) * kLog2e);  // e^{s_h - lse}; 0 for s = -inf
    contrib = -psink * D;
    float4* acc = reinterpret_cast<float4*>(p.dq_acc + row);
#pragma unroll
    for (int i = 0; i < kHeadDim / 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // Fixed-order block reduction: butterfly within each warp, then warps in
  // index order.
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) contrib += __shfl_xor_sync(0xffffffffu, contrib, off);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = contrib;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < kPreThreads / 32; ++w) s += warp_sums[w];
    p.partials[static_cast<size_t>(h) * p.num_pre_blocks + blockIdx.x] = s;
  }
}

// --------------------------------------------------------------- finish
struct FinishParams {
  size_t n_dq;  // T * Hq * D
  float scale;
  const float* dq_acc;
  __nv_bfloat16* dq;
  const float* partials;
  int num_pre_blocks;
  int Hq;
  int convert_blocks;
  float* dsinks;
};

// CTAs [0, convert_blocks): dq = bf16(scale * acc), 8 elements per thread
// per step.  CTAs [convert_blocks, convert_blocks + Hq): dsinks_h.
__global__ void __launch_bounds__(kFinishThreads) sink_attn_bwd_finish_kernel(const FinishParams p) {
  if (static_cast<int>(blockIdx.x) >= p.convert_blocks) {
    __shared__ float red[kFinishThreads];
    const int h = blockIdx.x - p.convert_blocks;
    float s = 0.f;
    for (int b = threadIdx.x; b < p.num_pre_blocks; b += kFinishThreads)
      s += p.partials[static_cast<size_t>(h) * p.num_pre_blocks + b];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int off = kFinishThreads / 2; off > 0; off >>= 1) {
      if (static_cast<int>(threadIdx.x) < off) red[threadIdx.x] += red[threadIdx.x + off];
      __syncthreads();
    }
    if (threadIdx.x == 0) p.dsinks[h] = red[0];
    return;
  }
  const size_t n8 = p.n_dq / 8;
  const size_t stride = static_cast<size_t>(p.convert_blocks) * kFinishThreads;
  for (size_t i = static_cast<size_t>(blockIdx.x) * kFinishThreads + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p.dq_acc) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(p.dq_acc) + 2 * i + 1);
    uint4 o;
    o.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    o.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    o.z = pack_bf16x2(b.x * p.scale, b.y * p.scale);
    o.w = pack_bf16x2(b.z * p.scale, b.w * p.scale);
    reinterpret_cast<uint4*>(p.dq)[i] = o;
  }
}

// ------------------------------------------------------------------ main
struct BwdParams {
  Geometry geo;
  float scale;
  float scale_log2;
  const float* lse;    // [Hq][T]
  const float* Dvec;   // [Hq][T]
  float* dq_acc;       // [T][Hq][D] fp32
  __nv_bfloat16* dk;   // [T][Hkv][D]
  __nv_bfloat16* dv;
  int num_key_tiles;
};

struct BwdAux {
  float lse2[kBlockM];  // lse * log2(e) per row (+inf for padding rows)
  float D[kBlockM];
  int lo[kBlockM];      // first allowed key per position of the tile
};

struct BwdCtl {
  uint64_t kv_full;
  uint64_t qdo_full[kBwdStages];
  uint64_t qdo_empty[kBwdStages];
  uint64_t aux_full[kBwdStages];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t dq_full;
  uint64_t dq_empty;
  uint64_t kd_full;
  uint32_t tmem_base;
  int abort;
};

// K, V, Q x2, dO x2, dS (two 16 KB halves) + aux + control.
constexpr size_t kBwdSmemBytes =
    1024 + kTileBytes * (2 + 2 * kBwdStages + 2) + sizeof(BwdAux) * kBwdStages + sizeof(BwdCtl);

__device__ __forceinline__ int doc_end(const Geometry& g, int t) {
  if (g.cu_seqlens == nullptr) return (t / g.seqlen + 1) * g.seqlen;
  int lo = 0, hi = g.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(g.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return __ldg(g.cu_seqlens + lo + 1);
}

struct BwdTile {
  int g, k0, k_last, qb0, nq;
};

__device__ __forceinline__ BwdTile bwd_tile(const Geometry& geo, int num_key_tiles) {
  BwdTile w;
  w.g = blockIdx.x % geo.Hkv;
  const int n = blockIdx.x / geo.Hkv;  // earlier keys are seen by more queries: they go first
  w.k0 = n * kBlockN;
  w.k_last = min(w.k0 + kBlockN - 1, geo.T - 1);
  int q_hi = doc_end(geo, w.k_last) - 1;
  if (geo.window > 0) q_hi = min(q_hi, w.k_last + geo.window - 1);
  w.qb0 = w.k0 >> geo.P_log2;
  w.nq = (q_hi >> geo.P_log2) - w.qb0 + 1;
  (void)num_key_tiles;
  return w;
}

// dS staged for the dQ MMA as an MN-major (rows contiguous) 128B-swizzled
// operand: two 64-row halves 16 KB apart (LBO), 8-key groups 1 KB apart
// (SBO), 128 B per key within a group, 16-byte chunks XOR-swizzled by key%8.
__device__ __forceinline__ uint32_t ds_smem_offset(int key, int chunk16) {
  const int half = chunk16 >> 3;  // rows 0-63 / 64-127
  const int c = chunk16 & 7;
  return static_cast<uint32_t>(half * 16384 + (key >> 3) * 1024 + (key & 7) * 128 + ((c ^ (key & 7)) << 4));
}

__global__ void __launch_bounds__(kBwdThreads, 1)
    sink_attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                              const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = sK + kTileBytes;
  uint8_t* sQ = sV + kTileBytes;                  // [kBwdStages]
  uint8_t* sDO = sQ + kBwdStages * kTileBytes;    // [kBwdStages]
  uint8_t* sDS = sDO + kBwdStages * kTileBytes;   // 32 KB
  BwdAux* aux = reinterpret_cast<BwdAux*>(sDS + 2 * kTileBytes);
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(aux + kBwdStages);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const Geometry& geo = p.geo;
  const BwdTile w = bwd_tile(geo, p.num_key_tiles);
  const int G = 1 << geo.G_log2;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->kv_full, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&ctl->qdo_full[s], 1);
      mbar_init(&ctl->qdo_empty[s], 1);
      mbar_init(&ctl->aux_full[s], 128);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->p_full, 128);
    mbar_init(&ctl->dq_full, 1);
    mbar_init(&ctl->dq_empty, 128);
    mbar_init(&ctl->kd_full, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl->tmem_base, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 4) {
    // ---------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&ctl->kv_full, 2 * kTileBytes);
      tma_load_3d(sK, &tm_k, &ctl->kv_full, 0, w.g, w.k0);
      tma_load_3d(sV, &tm_v, &ctl->kv_full, 0, w.g, w.k0);
      for (int i = 0; i < w.nq; ++i) {
        const int s = i % kBwdStages;
        if (i >= kBwdStages &&
            !mbar_wait(&ctl->qdo_empty[s], ((i / kBwdStages) - 1) & 1, abort, &g_device_error,
                       kDevErrTimeoutProducer))
          break;
        const int q0 = (w.qb0 + i) << geo.P_log2;
        mbar_arrive_expect_tx(&ctl->qdo_full[s], 2 * kTileBytes);
        tma_load_3d(sQ + s * kTileBytes, &tm_q, &ctl->qdo_full[s], 0, w.g << geo.G_log2, q0);
        tma_load_3d(sDO + s * kTileBytes, &tm_do, &ctl->qdo_full[s], 0, w.g << geo.G_log2, q0);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = make_idesc_bf16(kBlockN, kBlockM, 0, 0);    // M=128 keys, N=128 rows
      constexpr uint32_t idesc_acc = make_idesc_bf16(kBlockN, kHeadDim, 0, 1); // A tmem (K-major), B MN-major
      constexpr uint32_t idesc_dq = make_idesc_bf16(kBlockM, kHeadDim, 1, 1);  // A smem MN-major, B MN-major
      const uint32_t tS = tmem + kBwdTmemS, tDP = tmem + kBwdTmemDP;
      const uint32_t tDV = tmem + kBwdTmemDV, tDK = tmem + kBwdTmemDK, tDQ = tmem + kBwdTmemDQ;
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), ds_addr = smem_u32(sDS);
      bool ok = mbar_wait(&ctl->kv_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      for (int i = 0; ok && i < w.nq; ++i) {
        const int s = i % kBwdStages;
        ok = mbar_wait(&ctl->qdo_full[s], (i / kBwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + s * kTileBytes), do_addr = smem_u32(sDO + s * kTileBytes);
        // S^T = K Q^T and dP^T = V dO^T (both operands K-major over the head dim)
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_ss(tS, make_sdesc_sw128(k_addr + kk * 32, 16, 1024), make_sdesc_sw128(q_addr + kk * 32, 16, 1024),
                 idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_ss(tDP, make_sdesc_sw128(v_addr + kk * 32, 16, 1024),
                 make_sdesc_sw128(do_addr + kk * 32, 16, 1024), idesc_s, kk > 0);
        tc_commit(&ctl->s_full);
        ok = mbar_wait(&ctl->p_full, i & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q   (K = the tile's 128 query rows)
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk) {
          mma_ts(tDV, tS + kk * 8, make_sdesc_sw128(do_addr + kk * 2048, kTileBytes, 1024), idesc_acc,
                 (i > 0 || kk > 0) ? 1u : 0u);
          mma_ts(tDK, tDP + kk * 8, make_sdesc_sw128(q_addr + kk * 2048, kTileBytes, 1024), idesc_acc,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ = dS K   (M = 128 rows, K = 128 keys)
        if (i > 0) {
          ok = mbar_wait(&ctl->dq_empty, (i - 1) & 1, abort, &g_device_error, kDevErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          mma_ss(tDQ, make_sdesc_sw128(ds_addr + kk * 2048, 16384, 1024),
                 make_sdesc_sw128(k_addr + kk * 2048, kTileBytes, 1024), idesc_dq, kk > 0);
        tc_commit(&ctl->qdo_empty[s]);
        tc_commit(&ctl->dq_full);
      }
      if (ok) tc_commit(&ctl->kd_full);
    }
  } else if (warp < 4) {
    // ------------------------------------- P / dS (1 thread = 1 key = 1 lane)
    const int j = w.k0 + threadIdx.x;  // this thread's key
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base + kBwdTmemS;
    const uint32_t tDP = tmem + lane_base + kBwdTmemDP;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int i = 0; i < w.nq; ++i) {
      const int s = i % kBwdStages;
      ok = mbar_wait(&ctl->aux_full[s], (i / kBwdStages) & 1, abort, &g_device_error, kDevErrTimeoutBwd) &&
           mbar_wait(&ctl->s_full, i & 1, abort, &g_device_error, kDevErrTimeoutBwd);
      if (!ok) break;
      tc_fence_after();
      const BwdAux& a = aux[s];
      const int q0 = (w.qb0 + i) << geo.P_log2;
      const int q_last = q0 + (1 << geo.P_log2) - 1;
      // CTA-uniform: is every (key, row) pair of this block allowed?
      const bool full = (w.k0 + kBlockN - 1 < geo.T) && (q_last < geo.T) && (w.k0 + kBlockN - 1 <= q0) &&
                        (w.k0 >= a.lo[kBlockM / G - 1]);
#pragma unroll 1
      for (int c0 = 0; c0 < kBlockM; c0 += 32) {
        uint32_t sr[32], dr[32];
        __syncwarp();
        tmem_ld32(tS + c0, sr);
        tmem_ld32(tDP + c0, dr);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float pv[2], dsv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = c0 + c + u;
            float pe = ex2_approx(fmaf(__uint_as_float(sr[c + u]), sl2, -a.lse2[col]));
            if (!full) {
              const int pos = col >> geo.G_log2;
              const int tq = q0 + pos;
              if (!(j >= a.lo[pos] && j <= tq)) pe = 0.f;
            }
            pv[u] = pe;
            dsv[u] = pe * (__uint_as_float(dr[c + u]) - a.D[col]);
          }
          pk[c >> 1] = pack_bf16x2(pv[0], pv[1]);
          dk[c >> 1] = pack_bf16x2(dsv[0], dsv[1]);
        }
        __syncwarp();
        tmem_st16(tS + (c0 >> 1), pk);
        tmem_st16(tDP + (c0 >> 1), dk);
        // dS row segment -> shared memory, rows [c0, c0+32) = 4 chunks of 8
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = (c0 >> 3) + q;
          *reinterpret_cast<uint4*>(sDS + ds_smem_offset(threadIdx.x, chunk)) =
              make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
        }
      }
      // Generic-proxy shared-memory writes -> visible to the tensor core.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }
    // -------------------------------------------------- dK / dV epilogue
    if (ok) ok = mbar_wait(&ctl->kd_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    if (ok) {
      tc_fence_after();
      uint32_t r[kHeadDim];
      __syncwarp();
      tmem_ld64(tmem + lane_base + kBwdTmemDK, r);
      if (j < geo.T) {
        uint4* dst = reinterpret_cast<uint4*>(p.dk + (static_cast<size_t>(j) * geo.Hkv + w.g) * kHeadDim);
#pragma unroll
        for (int i = 0; i < kHeadDim / 8; ++i) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * p.scale, __uint_as_float(r[8 * i + 1]) * p.scale);
          v.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * p.scale, __uint_as_float(r[8 * i + 3]) * p.scale);
          v.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * p.scale, __uint_as_float(r[8 * i + 5]) * p.scale);
          v.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * p.scale, __uint_as_float(r[8 * i + 7]) * p.scale);
          dst[i] = v;
        }
      }
      __syncwarp();
      tmem_ld64(tmem + lane_base + kBwdTmemDV, r);
      if (j < geo.T) {
        uint4* dst = reinterpret_cast<uint4*>(p.dv + (static_cast<size_t>(j) * geo.Hkv + w.g) * kHeadDim);
#pragma unroll
        for (int i = 0; i < kHeadDim / 8; ++i) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]), __uint_as_float(r[8 * i + 1]));
          v.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3]));
          v.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5]));
          v.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7]));
          dst[i] = v;
        }
      }
    }
  } else {
    // ---------------------- warps 6-9: per-row aux loads + dQ accumulation
    const int r = 32 * (warp & 3) + (threadIdx.x & 31);  // TMEM lane = query row of the tile
    const uint32_t tDQ = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kBwdTmemDQ;
    const int hh = r & (G - 1);
    const int h = (w.g << geo.G_log2) + hh;
    auto load_aux = [&](int i) {
      BwdAux& a = aux[i % kBwdStages];
      const int t = ((w.qb0 + i) << geo.P_log2) + (r >> geo.G_log2);
      const bool valid = t < geo.T;
      a.lse2[r] = valid ? __ldg(p.lse + static_cast<size_t>(h) * geo.T + t) * kLog2e : INFINITY;
      a.D[r] = valid ? __ldg(p.Dvec + static_cast<size_t>(h) * geo.T + t) : 0.f;
      if (hh == 0) a.lo[r >> geo.G_log2] = valid ? first_key(geo, t) : 0x7fffffff;
      mbar_arrive(&ctl->aux_full[i % kBwdStages]);
    };
    for (int i = 0; i < kBwdStages && i < w.nq; ++i) load_aux(i);
    bool ok = true;
    for (int i = 0; i < w.nq; ++i) {
      ok = mbar_wait(&ctl->dq_full, i & 1, abort, &g_device_error, kDevErrTimeoutBwd);
      if (!ok) break;
      tc_fence_after();
      uint32_t d[kHeadDim];
      __syncwarp();
      tmem_ld64(tDQ, d);
      tc_fence_before();
      mbar_arrive(&ctl->dq_empty);
      const int t = ((w.qb0 + i) << geo.P_log2) + (r >> geo.G_log2);
      if (t < geo.T) {
        float4* dst = reinterpret_cast<float4*>(p.dq_acc + (static_cast<size_t>(t) * geo.Hq + h) * kHeadDim);
#pragma unroll
        for (int c = 0; c < kHeadDim / 4; ++c)
          atomicAdd(dst + c, make_float4(__uint_as_float(d[4 * c]), __uint_as_float(d[4 * c + 1]),
                                         __uint_as_float(d[4 * c + 2]), __uint_as_float(d[4 * c + 3])));
      }
      // Block i's aux stage is free: its P/dS pass finished before dQ_i.
      if (i + kBwdStages < w.nq) load_aux(i + kBwdStages);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// ------------------------------------------------------------------ host
inline sink_attn_status bwd_launch(const Geometry& geo, float scale, const void* q, const void* k, const void* v,
                                   const float* sinks, const void* out, const float* lse, const void* dout, void* dq,
                                   void* dk, void* dv, float* dsinks, uint8_t* ws_base, const BwdWorkspace& ws,
                                   cudaStream_t stream, cudaEvent_t ev_main_begin, cudaEvent_t ev_main_end) {
  float* dq_acc = reinterpret_cast<float*>(ws_base + ws.dq_acc);
  float* Dvec = reinterpret_cast<float*>(ws_base + ws.Dvec);
  float* partials = reinterpret_cast<float*>(ws_base + ws.partials);

  // 1. preprocess
  PreParams pp;
  pp.T = geo.T;
  pp.Hq = geo.Hq;
  pp.out = static_cast<const __nv_bfloat16*>(out);
  pp.dout = static_cast<const __nv_bfloat16*>(dout);
  pp.lse = lse;
  pp.sinks = sinks;
  pp.Dvec = Dvec;
  pp.partials = partials;
  pp.dq_acc = dq_acc;
  pp.num_pre_blocks = ws.num_pre_blocks;
  sink_attn_bwd_preprocess_kernel<<<dim3(ws.num_pre_blocks, geo.Hq), kPreThreads, 0, stream>>>(pp);
  if (cudaPeekAtLastError() != cudaSuccess) return SINK_ATTN_ERR_CUDA;

  // 2. main
  const int G = 1 << geo.G_log2;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_3d(&tq, q, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2) ||
      !make_map_3d(&tdo, dout, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2) ||
      !make_map_3d(&tk, k, kHeadDim, geo.Hkv, geo.T, 1, kBlockN) ||
      !make_map_3d(&tv, v, kHeadDim, geo.Hkv, geo.T, 1, kBlockN))
    return SINK_ATTN_ERR_CUDA;
  static int smem_set = 0;
  if (!smem_set) {
    if (cudaFuncSetAttribute(sink_attn_bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kBwdSmemBytes)) != cudaSuccess)
      return SINK_ATTN_ERR_CUDA;
    smem_set = 1;
  }
  BwdParams bp;
  bp.geo = geo;
  bp.scale = scale;
  bp.scale_log2 = scale * kLog2e;
  bp.lse = lse;
  bp.Dvec = Dvec;
  bp.dq_acc = dq_acc;
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.num_key_tiles = (geo.T + kBlockN - 1) / kBlockN;
  const int64_t grid = static_cast<int64_t>(bp.num_key_tiles) * geo.Hkv;
  if (grid > 0x7fffffff) return SINK_ATTN_ERR_UNSUPPORTED;
  if (ev_main_begin) cudaEventRecord(ev_main_begin, stream);
  sink_attn_bwd_main_kernel<<<static_cast<unsigned>(grid), kBwdThreads, kBwdSmemBytes, stream>>>(tq, tk, tv, tdo,
                                                                                                  bp);
  if (ev_main_end) cudaEventRecord(ev_main_end, stream);
  if (cudaPeekAtLastError() != cudaSuccess) return SINK_ATTN_ERR_CUDA;

  // 3. finish
  FinishParams fp;
  fp.n_dq = static_cast<size_t>(geo.T) * geo.Hq * kHeadDim;
  fp.scale = scale;
  fp.dq_acc = dq_acc;
  fp.dq = static_cast<__nv_bfloat16*>(dq);
  fp.partials = partials;
  fp.num_pre_blocks = ws.num_pre_blocks;
  fp.Hq = geo.Hq;
  const size_t want = (fp.n_dq / 8 + kFinishThreads - 1) / kFinishThreads;
  fp.convert_blocks = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
  if (fp.convert_blocks < 1) fp.convert_blocks = 1;
  fp.dsinks = dsinks;
  sink_attn_bwd_finish_kernel<<<fp.convert_blocks + geo.Hq, kFinishThreads, 0, stream>>>(fp);
  return cudaPeekAtLastError() == cudaSuccess ? SINK_ATTN_OK : SINK_ATTN_ERR_CUDA;
}

}  // namespace sa
