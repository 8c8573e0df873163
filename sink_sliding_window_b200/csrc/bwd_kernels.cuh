// Backward kernels: gradients of causal GQA sink attention.
//
//   P_ij = e^{l_ij - lse_i}, P_sink,i = e^{s_h - lse_i}, D_i = dout_i . out_i
//   dS_ij = P_ij (dout_i . v_j - D_i)
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_{i,h in group} dS_ij q_i,
//   dv_j = sum_{i,h in group} P_ij dout_i,  dsinks_h = -sum_i P_sink,i D_i
//
// Three launches on the caller's stream:
//   1. bwd_preprocess: D_i; -lse_i*log2(e) and -D_i re-laid out in
//      query-tile row order (so the main kernel fetches a tile's 128 values
//      with one bulk copy); the first allowed key of every token; per-block partial sums of
//      -P_sink,i D_i (fixed order); and zeroes the fp32 dq accumulator.
//   2. bwd_main (tcgen05): one CTA per 128-key tile of one key/value head g,
//      visiting every query tile (the forward's 128 rows = 128/G tokens x G
//      heads) that can see one of its keys.  Keys sit on the TMEM lanes:
//        S^T = K Q^T, dP^T = V dO^T          (MMA, fp32 in TMEM)
//        P = 2^(S^T*scale*log2e - lse2), dS = P (dP - D)   (8 warps)
//        dV += P^T dO, dK += dS^T Q          (MMA, A from TMEM; dV and dK sum
//                                             over the G heads inside TMEM)
//        dQ = dS K                           (MMA, A = dS in shared memory)
//      dQ tiles are reduced into the fp32 accumulator by TMA reduce-add.
//      Two S^T buffers let the tensor core compute tile i+2's S^T and tile
//      i+1's dP^T while the softmax warps work on tile i+1.
//   3. bwd_finish: dq = bf16(scale * accumulator), and dsinks_h = fixed-order
//      tree sum of the partials (bitwise reproducible).
#pragma once
#include "common.cuh"
#include "tma_host.cuh"

namespace sa {

constexpr int kBwdLaunches = 3;
constexpr int kPreThreads = 256;  // tokens per preprocess CTA (one head per CTA)
constexpr int kFinishThreads = 256;

// ---------------------------------------------------------------- workspace
struct BwdWorkspace {
  size_t dq_acc;    // fp32 [T][Hq][D]
  size_t Dvec;      // fp32 [Hq][T]
  size_t lse2_blk;  // fp32 [num_qblocks][Hkv][128]  -lse*log2(e) in tile-row order (-inf for padding rows)
  size_t D_blk;     // fp32 [num_qblocks][Hkv][128]  -D in tile-row order (0 for padding rows)
  size_t lo_blk;    // int  [num_qblocks][128]       first allowed key per token of the tile
  size_t partials;  // fp32 [Hq][num_pre_blocks]
  int num_pre_blocks;
  size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline BwdWorkspace bwd_workspace_layout(const Geometry& geo) {
  BwdWorkspace w;
  const size_t T = static_cast<size_t>(geo.T);
  const size_t T_pad = static_cast<size_t>(geo.num_qblocks) << geo.P_log2;
  w.num_pre_blocks = static_cast<int>((T_pad + kPreThreads - 1) / kPreThreads);
  size_t off = 0;
  w.dq_acc = off;
  off += align_up(T * geo.Hq * kHeadDim * sizeof(float), 256);
  w.Dvec = off;
  off += align_up(T * geo.Hq * sizeof(float), 256);
  w.lse2_blk = off;
  off += align_up(static_cast<size_t>(geo.num_qblocks) * geo.Hkv * kBlockM * sizeof(float), 256);
  w.D_blk = off;
  off += align_up(static_cast<size_t>(geo.num_qblocks) * geo.Hkv * kBlockM * sizeof(float), 256);
  w.lo_blk = off;
  off += align_up(static_cast<size_t>(geo.num_qblocks) * kBlockM * sizeof(int), 256);
  w.partials = off;
  off += align_up(static_cast<size_t>(geo.Hq) * (w.num_pre_blocks > 0 ? w.num_pre_blocks : 1) * sizeof(float), 256);
  w.total = off;
  return w;
}

// ------------------------------------------------------------ preprocess
struct PreParams {
  Geometry geo;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  const float* lse;
  const float* sinks;
  float* Dvec;
  float* lse2_blk;
  float* D_blk;
  int* lo_blk;
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

// Grid (num_pre_blocks, Hq).  Each group of 8 lanes reads one 128-byte row
// (token, head blockIdx.y) of out and dout with one 16-byte load per lane, so
// a warp-wide load covers 4 rows; a CTA covers kPreThreads tokens (padded up
// to whole query tiles).
__global__ void __launch_bounds__(kPreThreads) sink_attn_bwd_preprocess_kernel(const PreParams p) {
  __shared__ float warp_sums[kPreThreads / 32];
  const Geometry& geo = p.geo;
  const int h = blockIdx.y;
  const int t_pad = geo.num_qblocks << geo.P_log2;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;              // 16-byte piece of the row
  const int t_base = blockIdx.x * kPreThreads + (threadIdx.x >> 5) * 32;  // this warp's 32 tokens
  float contrib = 0.f;                   // valid in lanes with sub == 0
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int t = t_base + it * 4 + (lane >> 3);
    float D = 0.f;
    if (t < geo.T) {
      const size_t row = (static_cast<size_t>(t) * geo.Hq + h) * kHeadDim;
      D = dot8_bf16(__ldg(reinterpret_cast<const uint4*>(p.out + row) + sub),
                    __ldg(reinterpret_cast<const uint4*>(p.dout + row) + sub));
      float4* acc = reinterpret_cast<float4*>(p.dq_acc + row) + 2 * sub;
      acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // sum the 8 pieces of the row (fixed butterfly)
    D += __shfl_xor_sync(0xffffffffu, D, 1);
    D += __shfl_xor_sync(0xffffffffu, D, 2);
    D += __shfl_xor_sync(0xffffffffu, D, 4);
    if (sub == 0 && t < t_pad) {
      const int qb = t >> geo.P_log2;
      const int pos = t & ((1 << geo.P_log2) - 1);
      const int g = h >> geo.G_log2;
      const int r = (pos << geo.G_log2) + (h & ((1 << geo.G_log2) - 1));
      const size_t bi = (static_cast<size_t>(qb) * geo.Hkv + g) * kBlockM + r;
      if (t < geo.T) {
        const float lse = __ldg(p.lse + static_cast<size_t>(h) * geo.T + t);
        p.Dvec[static_cast<size_t>(h) * geo.T + t] = D;
        // Stored negated: the main kernel adds them with two-wide fp32 ops.
        p.D_blk[bi] = -D;
        p.lse2_blk[bi] = -(lse * kLog2e);
        const float psink = ex2_approx((__ldg(p.sinks + h) - lse) * kLog2e);  // e^{s_h - lse}; 0 for s = -inf
        contrib -= psink * D;
        if (h == 0) p.lo_blk[static_cast<size_t>(qb) * kBlockM + pos] = first_key(geo, t);
      } else {
        // padding rows of the last query tile: P = 0 and dS = 0 there
        p.D_blk[bi] = 0.f;
        p.lse2_blk[bi] = -INFINITY;
        if (h == 0) p.lo_blk[static_cast<size_t>(qb) * kBlockM + pos] = 0x7fffffff;
      }
    }
  }
  // Fixed-order block reduction: butterfly within each warp, then warps in
  // index order.
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) contrib += __shfl_xor_sync(0xffffffffu, contrib, off);
  if (lane == 0) warp_sums[threadIdx.x >> 5] = contrib;
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
constexpr int kBwdThreads = 448;    // 14 warps
constexpr int kBwdStages = 3;       // Q/dO/aux ring
constexpr int kBwdWarpProducer = 8;
constexpr int kBwdWarpMma = 9;
constexpr int kBwdWarpDq0 = 10;     // warps 10..13
constexpr uint32_t kBwdTmemCols = 512;
constexpr uint32_t kBwdTmemS0 = 0;    // S^T buffer 0: fp32 [128 keys][128 rows]; P^T bf16 in cols 0..31
constexpr uint32_t kBwdTmemS1 = 128;  //   (rows 0-63) and 64..95 (rows 64-127); the tile's dQ (fp32
                                      //   [128 rows][64]) later in cols 64..127, after the dV MMA read P^T
constexpr uint32_t kBwdTmemDP = 256;  // dP^T fp32; dS^T bf16 in cols 0..31 (rows 0-63) and 64..95 (rows 64-127)
constexpr uint32_t kBwdTmemDV = 384;  // dV accumulator fp32 [128 keys][64]
constexpr uint32_t kBwdTmemDK = 448;  // dK accumulator

struct BwdParams {
  Geometry geo;
  float scale;
  float scale_log2;
  const float* lse2_blk;
  const float* D_blk;
  const int* lo_blk;
  __nv_bfloat16* dk;   // [T][Hkv][D]
  __nv_bfloat16* dv;
};

struct BwdAux {
  float lse2[kBlockM];  // -lse*log2(e) per row of the query tile (-inf for padding rows)
  float D[kBlockM];     // -D per row
  int lo[kBlockM];      // first allowed key per token of the tile (first 128/G entries)
};

struct BwdCtl {
  uint64_t kv_full;
  uint64_t qdo_full[kBwdStages];
  uint64_t qdo_empty[kBwdStages];
  uint64_t s_full[2];
  uint64_t dp_full;
  uint64_t p_full;
  // dQ_i ready in TMEM, one barrier per tile parity: tile i+2's dQ can only
  // be committed after the dQ warps released tile i's TMEM (dq_empty), so a
  // barrier never runs two phases ahead of the dQ warps' parity wait, however
  // late the dQ warps are.
  uint64_t dq_full[2];
  uint64_t dq_empty;
  uint64_t kd_full;
  uint64_t dq_sync;       // the four dQ warps (128 threads)
  uint32_t tmem_base;
  int abort;
};

// Barrier over the threads counted by `bar` (each arrives once per use),
// with the same bounded wait as every other wait in these kernels.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, volatile int* abort, int code) {
  mbar_arrive(bar);
  const bool ok = warp_all(mbar_wait(bar, phase, abort, &g_device_error, code));
  phase ^= 1u;
  return ok;
}

// K, V, Q x3, dO x3, dS (32 KB), dQ staging (32 KB), aux x3, control.
constexpr size_t kBwdSmemBytes =
    1024 + kTileBytes * (2 + 2 * kBwdStages + 2 + 2) + sizeof(BwdAux) * kBwdStages + sizeof(BwdCtl);

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
  int g, k0, qb_last, nq;  // query tiles qb_last, qb_last-1, ..., qb_last-nq+1
};

__device__ __forceinline__ BwdTile bwd_tile(const Geometry& geo) {
  BwdTile w;
  w.g = blockIdx.x % geo.Hkv;
  int n = blockIdx.x / geo.Hkv;
  // Key tiles early in their document are seen by the most query tiles: with
  // equal-length documents hand out the first tile of every document, then
  // the second, ... (longest first).
  if (geo.cu_seqlens == nullptr && (geo.seqlen % kBlockN) == 0) {
    const int per_doc = geo.seqlen / kBlockN;
    n = (n % geo.batch) * per_doc + n / geo.batch;
  }
  w.k0 = n * kBlockN;
  const int k_last = min(w.k0 + kBlockN - 1, geo.T - 1);
  int q_hi = doc_end(geo, k_last) - 1;
  if (geo.window > 0) q_hi = min(q_hi, k_last + geo.window - 1);
  // Visit query tiles from the last one down: the key tiles of a document
  // that run at the same time then add into the same rows of the fp32 dq
  // accumulator at about the same time, and those rows stay in L2.
  const int qb0 = w.k0 >> geo.P_log2;
  w.qb_last = q_hi >> geo.P_log2;
  w.nq = w.qb_last - qb0 + 1;
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

// P^T for this thread's key over the 64 query rows [64*ch, 64*ch+64) of a
// tile: P = 2^(S^T * scale*log2e - lse2), zero outside the rows
// [r_lo, r_lo + r_span) that see the key (kMask), rounded to bf16 and packed
// in row pairs (pk[r/2] holds rows r, r+1).  The scaling runs two rows per
// instruction (a.lse2 holds -lse2).
template <bool kMask>
__device__ __forceinline__ void bwd_p_rows(uint32_t tS, const BwdAux& a, int ch, float sl2, int r_lo, int r_span,
                                           uint32_t* pk) {
  const uint64_t sl2x2 = f32x2_pack(sl2, sl2);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t sr[32];
    __syncwarp();
    tmem_ld32(tS + 32 * half, sr);
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
      const int col = 64 * ch + 32 * half + c;
      const float4 l4 = *reinterpret_cast<const float4*>(&a.lse2[col]);
      float y[4];
      f32x2_unpack(fma_f32x2(f32x2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2,
                             f32x2_pack(l4.x, l4.y)), y[0], y[1]);
      f32x2_unpack(fma_f32x2(f32x2_pack(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sl2x2,
                             f32x2_pack(l4.z, l4.w)), y[2], y[3]);
      float pe[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        pe[u] = ex2_approx(y[u]);
        if (kMask && static_cast<unsigned>(col + u - r_lo) >= static_cast<unsigned>(r_span)) pe[u] = 0.f;
      }
      pk[16 * half + c / 2] = pack_bf16x2(pe[0], pe[1]);
      pk[16 * half + c / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
    }
  }
}

__global__ void __launch_bounds__(kBwdThreads, 1)
    sink_attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                              const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;
  uint8_t* sV = sK + kTileBytes;
  uint8_t* sQ = sV + kTileBytes;                  // [kBwdStages]
  uint8_t* sDO = sQ + kBwdStages * kTileBytes;    // [kBwdStages]
  uint8_t* sDS = sDO + kBwdStages * kTileBytes;   // 32 KB
  uint8_t* sDQ = sDS + 2 * kTileBytes;            // 32 KB: two {32 fp32 x 128 rows} swizzled halves
  BwdAux* aux = reinterpret_cast<BwdAux*>(sDQ + 2 * kTileBytes);
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(aux + kBwdStages);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const Geometry& geo = p.geo;
  const BwdTile w = bwd_tile(geo);

  if (threadIdx.x == 0) {
    mbar_init(&ctl->kv_full, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&ctl->qdo_full[s], 1);
      mbar_init(&ctl->qdo_empty[s], 1);
    }
    mbar_init(&ctl->s_full[0], 1);
    mbar_init(&ctl->s_full[1], 1);
    mbar_init(&ctl->dp_full, 1);
    mbar_init(&ctl->p_full, 256);
    mbar_init(&ctl->dq_full[0], 1);
    mbar_init(&ctl->dq_full[1], 1);
    mbar_init(&ctl->dq_empty, 128);
    mbar_init(&ctl->kd_full, 1);
    mbar_init(&ctl->dq_sync, 128);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == kBwdWarpMma) {
    tmem_alloc(&ctl->tmem_base, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kBwdWarpProducer) {
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
        const int qb = w.qb_last - i;
        const int q0 = qb << geo.P_log2;
        const size_t blk = (static_cast<size_t>(qb) * geo.Hkv + w.g) * kBlockM;
        mbar_arrive_expect_tx(&ctl->qdo_full[s], 2 * kTileBytes + 3 * kBlockM * 4);
        tma_load_3d(sQ + s * kTileBytes, &tm_q, &ctl->qdo_full[s], 0, w.g << geo.G_log2, q0);
        tma_load_3d(sDO + s * kTileBytes, &tm_do, &ctl->qdo_full[s], 0, w.g << geo.G_log2, q0);
        bulk_load(aux[s].lse2, p.lse2_blk + blk, kBlockM * 4, &ctl->qdo_full[s]);
        bulk_load(aux[s].D, p.D_blk + blk, kBlockM * 4, &ctl->qdo_full[s]);
        bulk_load(aux[s].lo, p.lo_blk + static_cast<size_t>(qb) * kBlockM, kBlockM * 4, &ctl->qdo_full[s]);
      }
    }
  } else if (warp == kBwdWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = make_idesc_bf16(kBlockN, kBlockM, 0, 0);    // M=128 keys, N=128 rows
      constexpr uint32_t idesc_acc = make_idesc_bf16(kBlockN, kHeadDim, 0, 1); // A tmem (K-major), B MN-major
      constexpr uint32_t idesc_dq = make_idesc_bf16(kBlockM, kHeadDim, 1, 1);  // A smem MN-major, B MN-major
      const uint32_t tS0 = tmem + kBwdTmemS0, tS1 = tmem + kBwdTmemS1;
      const uint32_t tDP = tmem + kBwdTmemDP, tDV = tmem + kBwdTmemDV, tDK = tmem + kBwdTmemDK;
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), ds_addr = smem_u32(sDS);
      auto issue_s = [&](int i) {  // S^T_i = K Q_i^T into buffer i%2
        const uint32_t q_addr = smem_u32(sQ + (i % kBwdStages) * kTileBytes);
        const uint32_t d = (i & 1) ? tS1 : tS0;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_ss(d, make_sdesc_sw128(k_addr + kk * 32, 16, 1024), make_sdesc_sw128(q_addr + kk * 32, 16, 1024),
                 idesc_s, kk > 0);
      };
      auto issue_dp = [&](int i) {  // dP^T_i = V dO_i^T
        const uint32_t do_addr = smem_u32(sDO + (i % kBwdStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_ss(tDP, make_sdesc_sw128(v_addr + kk * 32, 16, 1024), make_sdesc_sw128(do_addr + kk * 32, 16, 1024),
                 idesc_s, kk > 0);
      };
      auto wait_q = [&](int i) {
        return mbar_wait(&ctl->qdo_full[i % kBwdStages], (i / kBwdStages) & 1, abort, &g_device_error,
                         kDevErrTimeoutMma);
      };
      bool ok = mbar_wait(&ctl->kv_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      if (ok && w.nq > 0) {
        ok = wait_q(0);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          tc_commit(&ctl->s_full[0]);
          issue_dp(0);
          tc_commit(&ctl->dp_full);
        }
      }
      if (ok && w.nq > 1) {
        ok = wait_q(1);
        if (ok) {
          tc_fence_after();
          issue_s(1);
          tc_commit(&ctl->s_full[1]);
        }
      }
      for (int i = 0; ok && i < w.nq; ++i) {
        const uint32_t tSb = (i & 1) ? tS1 : tS0;
        const int st = i % kBwdStages;
        ok = mbar_wait(&ctl->p_full, i & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + st * kTileBytes), do_addr = smem_u32(sDO + st * kTileBytes);
        // dV += P^T dO and dK += dS^T Q over the tile's 128 query rows.  P^T
        // sits in cols 0..31 (rows 0-63) and 64..95 (rows 64-127) of the S^T
        // buffer; dS^T at the same columns of the dP^T region.
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_ts(tDV, tSb + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                 make_sdesc_sw128(do_addr + kk * 2048, kTileBytes, 1024), idesc_acc, acc);
          mma_ts(tDK, tDP + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                 make_sdesc_sw128(q_addr + kk * 2048, kTileBytes, 1024), idesc_acc, acc);
        }
        // dQ_i = dS K into the upper half of this tile's S^T buffer
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          mma_ss(tSb + 64, make_sdesc_sw128(ds_addr + kk * 2048, 16384, 1024),
                 make_sdesc_sw128(k_addr + kk * 2048, kTileBytes, 1024), idesc_dq, kk > 0);
        tc_commit(&ctl->dq_full[i & 1]);
        tc_commit(&ctl->qdo_empty[st]);
        if (i + 1 < w.nq) {
          // dP^T_{i+1} (dS_i in the dP region was consumed by dK above)
          ok = wait_q(i + 1);
          if (!ok) break;
          tc_fence_after();
          issue_dp(i + 1);
          tc_commit(&ctl->dp_full);
        }
        if (i + 2 < w.nq) {
          // S^T_{i+2} reuses this buffer once dQ_i has been read out of it
          ok = mbar_wait(&ctl->dq_empty, i & 1, abort, &g_device_error, kDevErrTimeoutMma) && wait_q(i + 2);
          if (!ok) break;
          tc_fence_after();
          issue_s(i + 2);
          tc_commit(&ctl->s_full[i & 1]);
        }
      }
      if (ok) tc_commit(&ctl->kd_full);
    }
  } else if (warp < 8) {
    // -------------------- P / dS: 2 warps per TMEM lane group (one key per lane)
    const int lg = warp & 3;                 // TMEM lane group: keys 32*lg .. 32*lg+31
    const int ch = warp >> 2;                // query rows [64*ch, 64*ch+64)
    const int kl = 32 * lg + (threadIdx.x & 31);
    const int j = w.k0 + kl;                 // this thread's key
    const uint32_t lane_base = static_cast<uint32_t>(32 * lg) << 16;
    const float sl2 = p.scale_log2;
    // The tokens that see key j are j <= t <= t_max (the end of j's document
    // and, with a window, j + W - 1), so in every query tile the rows that
    // see it form one range: the mask is one unsigned compare per element.
    int t_max = -1;
    if (j < geo.T) {
      t_max = doc_end(geo, j) - 1;
      if (geo.window > 0) t_max = min(t_max, j + geo.window - 1);
    }
    const int G = 1 << geo.G_log2;
    bool ok = true;
    for (int i = 0; i < w.nq; ++i) {
      const int st = i % kBwdStages;
      const uint32_t sbuf = (i & 1) ? kBwdTmemS1 : kBwdTmemS0;
      ok = mbar_wait(&ctl->qdo_full[st], (i / kBwdStages) & 1, abort, &g_device_error, kDevErrTimeoutSoftmax) &&
           mbar_wait(&ctl->s_full[i & 1], (i >> 1) & 1, abort, &g_device_error, kDevErrTimeoutSoftmax);
      ok = warp_all(ok);
      if (!ok) break;
      tc_fence_after();
      const BwdAux& a = aux[st];
      const int q0 = (w.qb_last - i) << geo.P_log2;
      const int q_last = q0 + (1 << geo.P_log2) - 1;
      // CTA-uniform: is every (key, row) pair of this tile allowed?
      const bool full = (w.k0 + kBlockN - 1 < geo.T) && (q_last < geo.T) && (w.k0 + kBlockN - 1 <= q0) &&
                        (w.k0 >= a.lo[(kBlockM >> geo.G_log2) - 1]);
      const uint32_t tS = tmem + lane_base + sbuf + 64 * ch;
      const uint32_t tDP = tmem + lane_base + kBwdTmemDP + 64 * ch;
      uint32_t pk[32];
      // The mask test is resolved once per tile (CTA-uniform), not per element.
      if (full) {
        bwd_p_rows<false>(tS, a, ch, sl2, 0, 0, pk);
      } else {
        const int r_lo = (max(j, q0) - q0) * G;
        const int r_span = max(0, (min(t_max, q_last) - q0 + 1) * G - r_lo);
        bwd_p_rows<true>(tS, a, ch, sl2, r_lo, r_span, pk);
      }
      // P^T (bf16) of this warp's 64 rows over the first half of its own
      // S^T columns (rows 0-63 -> columns 0..31, rows 64-127 -> 64..95):
      // this warp has read them and no other warp reads them.
      __syncwarp();
      tmem_st32_nowait(tmem + lane_base + sbuf + 64 * ch, pk);
      ok = warp_all(mbar_wait(&ctl->dp_full, i & 1, abort, &g_device_error, kDevErrTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - D); dQ_{i-1} has finished reading the shared dS buffer
      // (it was issued before dP^T_i).
      uint32_t ds_all[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t dr[32];
        __syncwarp();
        tmem_ld32(tDP + 32 * half, dr);
        uint32_t* dk = ds_all + 16 * half;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const int col = 64 * ch + 32 * half + c;
          const float4 nd4 = *reinterpret_cast<const float4*>(&a.D[col]);  // -D
          // dS = P (dP - D), two rows per instruction.
          float ds[4];
          f32x2_unpack(mul_f32x2(bf16x2_to_f32x2(pk[16 * half + c / 2]),
                                 add_f32x2(f32x2_pack(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])),
                                           f32x2_pack(nd4.x, nd4.y))),
                       ds[0], ds[1]);
          f32x2_unpack(mul_f32x2(bf16x2_to_f32x2(pk[16 * half + c / 2 + 1]),
                                 add_f32x2(f32x2_pack(__uint_as_float(dr[c + 2]), __uint_as_float(dr[c + 3])),
                                           f32x2_pack(nd4.z, nd4.w))),
                       ds[2], ds[3]);
          dk[c / 2] = pack_bf16x2(ds[0], ds[1]);
          dk[c / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
        }
        // dS^T for this warp's rows -> the first 32 columns of its own dP^T
        // column range (this warp has finished reading them).
        __syncwarp();
        tmem_st16_nowait(tDP + 16 * half, dk);
        // dS -> shared memory for the dQ MMA: rows [col0, col0 + 32)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((64 * ch + 32 * half) >> 3) + q;
          *reinterpret_cast<uint4*>(sDS + ds_smem_offset(kl, chunk)) =
              make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
        }
      }
      // P^T and dS^T stores must have landed before the MMA warp reads them
      tmem_wait_st_keep32(pk);
      tmem_wait_st_keep32(ds_all);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }
    // ------------------------------------------ dK (ch 0) / dV (ch 1) epilogue
    if (ok) ok = mbar_wait(&ctl->kd_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    ok = warp_all(ok);
    if (ok) {
      tc_fence_after();
      uint32_t r[kHeadDim];
      __syncwarp();
      tmem_ld64(tmem + lane_base + (ch == 0 ? kBwdTmemDK : kBwdTmemDV), r);
      if (j < geo.T) {
        const float sc = ch == 0 ? p.scale : 1.f;
        __nv_bfloat16* base = ch == 0 ? p.dk : p.dv;
        uint4* dst = reinterpret_cast<uint4*>(base + (static_cast<size_t>(j) * geo.Hkv + w.g) * kHeadDim);
#pragma unroll
        for (int i = 0; i < kHeadDim / 8; ++i) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * sc, __uint_as_float(r[8 * i + 1]) * sc);
          v.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * sc, __uint_as_float(r[8 * i + 3]) * sc);
          v.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * sc, __uint_as_float(r[8 * i + 5]) * sc);
          v.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * sc, __uint_as_float(r[8 * i + 7]) * sc);
          dst[i] = v;
        }
      }
    }
  } else if (warp >= kBwdWarpDq0) {
    // ------------------------ warps 10-13: dQ tile -> TMA reduce-add to the accumulator
    const int lg = warp & 3;
    const int r = 32 * lg + (threadIdx.x & 31);  // TMEM lane = query row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(32 * lg) << 16;
    const bool leader = threadIdx.x == kBwdWarpDq0 * 32;
    uint32_t sync_phase = 0;
    bool ok = true;
    for (int i = 0; i < w.nq; ++i) {
      ok = warp_all(mbar_wait(&ctl->dq_full[i & 1], (i >> 1) & 1, abort, &g_device_error, kDevErrTimeoutBwd));
      if (!ok) break;
      tc_fence_after();
      uint32_t d[kHeadDim];
      __syncwarp();
      tmem_ld64(tmem + lane_base + ((i & 1) ? kBwdTmemS1 : kBwdTmemS0) + 64, d);
      tc_fence_before();
      mbar_arrive(&ctl->dq_empty);
      // the previous reduce must have finished reading the staging buffer
      if (leader) bulk_wait_group_read<0>();
      ok = group_sync(&ctl->dq_sync, sync_phase, abort, kDevErrTimeoutBwd);
      if (!ok) break;
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t off = static_cast<uint32_t>(hlf * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
          *reinterpret_cast<uint4*>(sDQ + off) = make_uint4(d[32 * hlf + 4 * c], d[32 * hlf + 4 * c + 1],
                                                            d[32 * hlf + 4 * c + 2], d[32 * hlf + 4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      ok = group_sync(&ctl->dq_sync, sync_phase, abort, kDevErrTimeoutBwd);
      if (!ok) break;
      if (leader) {
        const int q0 = (w.qb_last - i) << geo.P_log2;
        tma_reduce_add_3d(&tm_dq, sDQ, 0, w.g << geo.G_log2, q0);
        tma_reduce_add_3d(&tm_dq, sDQ + 16384, 32, w.g << geo.G_log2, q0);
        bulk_commit_group();
      }
    }
    if (leader) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdWarpMma) {
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
  float* partials = reinterpret_cast<float*>(ws_base + ws.partials);

  // 1. preprocess
  PreParams pp;
  pp.geo = geo;
  pp.out = static_cast<const __nv_bfloat16*>(out);
  pp.dout = static_cast<const __nv_bfloat16*>(dout);
  pp.lse = lse;
  pp.sinks = sinks;
  pp.Dvec = reinterpret_cast<float*>(ws_base + ws.Dvec);
  pp.lse2_blk = reinterpret_cast<float*>(ws_base + ws.lse2_blk);
  pp.D_blk = reinterpret_cast<float*>(ws_base + ws.D_blk);
  pp.lo_blk = reinterpret_cast<int*>(ws_base + ws.lo_blk);
  pp.partials = partials;
  pp.dq_acc = dq_acc;
  pp.num_pre_blocks = ws.num_pre_blocks;
  sink_attn_bwd_preprocess_kernel<<<dim3(ws.num_pre_blocks, geo.Hq), kPreThreads, 0, stream>>>(pp);
  if (cudaPeekAtLastError() != cudaSuccess) return SINK_ATTN_ERR_CUDA;

  // 2. main
  const int G = 1 << geo.G_log2;
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (!make_map_3d(&tq, q, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2) ||
      !make_map_3d(&tdo, dout, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2) ||
      !make_map_3d(&tk, k, kHeadDim, geo.Hkv, geo.T, 1, kBlockN) ||
      !make_map_3d(&tv, v, kHeadDim, geo.Hkv, geo.T, 1, kBlockN) ||
      !make_map_3d_f32(&tdq, dq_acc, kHeadDim, geo.Hq, geo.T, G, 1 << geo.P_log2))
    return SINK_ATTN_ERR_CUDA;
  static SmemAttrOnce smem_set;
  if (!smem_set.ensure(sink_attn_bwd_main_kernel, kBwdSmemBytes)) return SINK_ATTN_ERR_CUDA;
  BwdParams bp;
  bp.geo = geo;
  bp.scale = scale;
  bp.scale_log2 = scale * kLog2e;
  bp.lse2_blk = pp.lse2_blk;
  bp.D_blk = pp.D_blk;
  bp.lo_blk = pp.lo_blk;
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  const int64_t grid = static_cast<int64_t>((geo.T + kBlockN - 1) / kBlockN) * geo.Hkv;
  if (grid > 0x7fffffff) return SINK_ATTN_ERR_UNSUPPORTED;
  if (ev_main_begin) cudaEventRecord(ev_main_begin, stream);
  sink_attn_bwd_main_kernel<<<static_cast<unsigned>(grid), kBwdThreads, kBwdSmemBytes, stream>>>(tq, tk, tv, tdo,
                                                                                                  tdq, bp);
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
