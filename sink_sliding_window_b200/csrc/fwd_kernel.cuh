// Forward kernel: causal GQA attention with a per-head sink logit, sliding
// window and packed documents, on sm_100a tensor cores.
//
// Work unit: one CTA owns one query tile = (128 / G) consecutive tokens x the
// G query heads of one key/value head g, i.e. 128 MMA rows, row r <->
// (token t0 + r / G, head g*G + r % G).  Because q is [T][Hq][D], the G heads
// of a group are contiguous and a single 3-D TMA box {64, G, 128/G} lands the
// tile in exactly this row order.  Every key/value tile that is loaded serves
// all G heads of the group.
//
// Per key/value tile j (128 keys starting at kv_lo + 128 j):
//   S = Q K_j^T            tcgen05.mma, bf16 in, fp32 in TMEM (128 cols)
//   softmax (1 thread = 1 row, the row lives in that thread's TMEM lane):
//     masked logits -> running reference max m (seeded with the sink logit,
//     lazily raised), P = 2^(S*scale*log2e - m) as bf16 written back into the
//     S columns, row sum l (seeded with the sink's e^{s-m} = 1)
//   O += P V_j             tcgen05.mma with A = P from TMEM, fp32 O in TMEM
// Tiles outside the causal / window / document range are never visited; only
// the edge tiles apply an element mask.
//
// Warp roles (192 threads, 2 CTAs per SM so one CTA's softmax overlaps the
// other's MMAs): warps 0-3 softmax + epilogue, warp 4 TMA producer, warp 5
// TMEM allocator + MMA issuer.  TMEM: S/P in columns [0,128), O in [128,192).
#pragma once
#include "common.cuh"

namespace sa {

constexpr int kFwdStages = 2;
constexpr int kFwdThreads = 192;
constexpr uint32_t kFwdTmemCols = 256;
constexpr uint32_t kFwdTmemS = 0;
constexpr uint32_t kFwdTmemO = 128;
// The reference max is raised only when a tile's max exceeds it by more than
// this many powers of two; P <= 2^8 in between, which fp32 and bf16 hold
// exactly in range.  The result is the same softmax (only rounding differs).
constexpr float kRescaleLog2 = 8.0f;

struct FwdParams {
  Geometry geo;
  float scale_log2;     // scale * log2(e)
  const float* sinks;   // [Hq]
  __nv_bfloat16* out;   // [T][Hq][D]
  float* lse;           // [Hq][T]
};

struct FwdCtl {
  uint64_t q_full;
  uint64_t k_full[kFwdStages];
  uint64_t v_full[kFwdStages];
  uint64_t kv_empty[kFwdStages];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kFwdSmemBytes = 1024 /*alignment slack*/ + kTileBytes * (1 + 2 * kFwdStages) + sizeof(FwdCtl);

// Query tile handled by this CTA and its key range.
struct FwdTile {
  int g;       // key/value head
  int t0;      // first token of the tile
  int t_last;  // last valid token of the tile
  int kv_lo;   // first key any row may see
  int lo_max;  // first key the last row may see (largest over rows)
  int n_tiles; // key tiles to visit
};

__device__ __forceinline__ FwdTile fwd_tile(const Geometry& geo) {
  FwdTile w;
  w.g = blockIdx.x % geo.Hkv;
  // Later tiles see more keys under a causal mask: hand them out first.
  const int qb = geo.num_qblocks - 1 - static_cast<int>(blockIdx.x / geo.Hkv);
  w.t0 = qb << geo.P_log2;
  w.t_last = min(w.t0 + (1 << geo.P_log2) - 1, geo.T - 1);
  w.kv_lo = first_key(geo, w.t0);
  w.lo_max = first_key(geo, w.t_last);
  w.n_tiles = (w.t_last - w.kv_lo + kBlockN) / kBlockN;
  return w;
}

__device__ __forceinline__ void fwd_issue_qk(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = make_idesc_bf16(kBlockM, kBlockN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint64_t a = make_sdesc_sw128(q_addr + kk * 32, 16, 1024);
    const uint64_t b = make_sdesc_sw128(k_addr + kk * 32, 16, 1024);
    mma_ss(tmem_s, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

__device__ __forceinline__ void fwd_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr, bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(kBlockM, kHeadDim, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kBlockN / 16; ++kk) {
    const uint64_t b = make_sdesc_sw128(v_addr + kk * 2048, kTileBytes, 1024);
    mma_ts(tmem_o, tmem_p + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One key tile of one query row: mask (kMask), row max, lazily raised
// reference max, P = 2^(S*scale*log2e - m) packed to bf16 pairs in s[0..63],
// and the row sum of P.  s[] holds the row's 128 fp32 logits on entry.
struct FwdRowStep {
  bool need;    // the reference max was raised
  float alpha;  // factor applied to the running sum / O (1 when not raised)
  float m_new;  // reference max after this tile
  float sum;    // sum of this tile's P
};

template <bool kMask>
__device__ __forceinline__ FwdRowStep fwd_row_step(uint32_t* s, int c_lo, int c_hi, float sl2, float m_ref) {
  float x[kBlockN];
#pragma unroll
  for (int c = 0; c < kBlockN; ++c) {
    x[c] = __uint_as_float(s[c]);
    if (kMask) x[c] = (c < c_lo || c > c_hi) ? -INFINITY : x[c];
  }
  float mx = fmax3(x[0], x[1], x[2]);
#pragma unroll
  for (int c = 3; c < kBlockN - 1; c += 2) mx = fmax3(mx, x[c], x[c + 1]);
  mx = fmaxf(mx, x[kBlockN - 1]);
  const float mx2 = mx * sl2;
  FwdRowStep r;
  r.need = mx2 > m_ref + kRescaleLog2;
  r.alpha = r.need ? ex2_approx(m_ref - mx2) : 1.f;
  r.m_new = r.need ? mx2 : m_ref;
  const float m_use = (r.m_new == -INFINITY) ? 0.f : r.m_new;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < kBlockN / 2; ++c) {
    const float e0 = ex2_approx(fmaf(x[2 * c], sl2, -m_use));
    const float e1 = ex2_approx(fmaf(x[2 * c + 1], sl2, -m_use));
    acc[(2 * c) & 3] += e0;
    acc[(2 * c + 1) & 3] += e1;
    s[c] = pack_bf16x2(e0, e1);
  }
  r.sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  return r;
}

__global__ void __launch_bounds__(kFwdThreads, 2)
    sink_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;
  uint8_t* sV = sK + kFwdStages * kTileBytes;
  FwdCtl* ctl = reinterpret_cast<FwdCtl*>(sV + kFwdStages * kTileBytes);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const Geometry& geo = p.geo;
  const FwdTile w = fwd_tile(geo);

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->p_full, 128);
    mbar_init(&ctl->o_full, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl->tmem_base, kFwdTmemCols);
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
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&ctl->q_full, kTileBytes);
      tma_load_3d(sQ, &tm_q, &ctl->q_full, 0, w.g << geo.G_log2, w.t0);
      for (int j = 0; j < w.n_tiles; ++j) {
        const int s = j % kFwdStages;
        if (j >= kFwdStages &&
            !mbar_wait(&ctl->kv_empty[s], ((j / kFwdStages) - 1) & 1, abort, &g_device_error,
                       kDevErrTimeoutProducer))
          break;
        const int ts = w.kv_lo + j * kBlockN;
        mbar_arrive_expect_tx(&ctl->k_full[s], kTileBytes);
        tma_load_3d(sK + s * kTileBytes, &tm_k, &ctl->k_full[s], 0, w.g, ts);
        mbar_arrive_expect_tx(&ctl->v_full[s], kTileBytes);
        tma_load_3d(sV + s * kTileBytes, &tm_v, &ctl->v_full[s], 0, w.g, ts);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t tS = tmem + kFwdTmemS;
      const uint32_t tO = tmem + kFwdTmemO;
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      for (int j = 0; ok && j <= w.n_tiles; ++j) {
        if (j > 0) {
          // O += P_{j-1} V_{j-1}
          const int sp = (j - 1) % kFwdStages;
          const uint32_t php = ((j - 1) / kFwdStages) & 1;
          ok = mbar_wait(&ctl->v_full[sp], php, abort, &g_device_error, kDevErrTimeoutMma) &&
               mbar_wait(&ctl->p_full, (j - 1) & 1, abort, &g_device_error, kDevErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          fwd_issue_pv(tO, tS, smem_u32(sV + sp * kTileBytes), j > 1);
          tc_commit(&ctl->kv_empty[sp]);
        }
        if (j == w.n_tiles) break;
        // S = Q K_j^T (overwrites P_{j-1}: the PV above was issued first and
        // tcgen05 MMAs from one thread execute in order).
        const int s = j % kFwdStages;
        ok = mbar_wait(&ctl->k_full[s], (j / kFwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        fwd_issue_qk(tS, q_addr, smem_u32(sK + s * kTileBytes));
        tc_commit(&ctl->s_full);
      }
      if (ok) tc_commit(&ctl->o_full);
    }
  } else {
    // ------------------------------------------------------ softmax (1 row)
    const int r = threadIdx.x;
    const int G = 1 << geo.G_log2;
    const int t = w.t0 + (r >> geo.G_log2);
    const int h = (w.g << geo.G_log2) + (r & (G - 1));
    const bool valid = t < geo.T;
    int lo_r = 0, hi_r = -1;  // allowed keys [lo_r, hi_r]; empty for padding rows
    if (valid) {
      lo_r = first_key(geo, t);
      hi_r = t;
    }
    const float sink = __ldg(p.sinks + h);
    float m_ref = sink * kLog2e;                 // -inf when the sink is off
    float l = (sink == -INFINITY) ? 0.f : 1.f;   // e^{s - m} with m = s
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base + kFwdTmemS;
    const uint32_t tO = tmem + lane_base + kFwdTmemO;
    const float sl2 = p.scale_log2;
    bool ok = true;

    for (int j = 0; j < w.n_tiles; ++j) {
      ok = mbar_wait(&ctl->s_full, j & 1, abort, &g_device_error, kDevErrTimeoutSoftmax);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kBlockN];
      tmem_ld64(tS, sr);
      tmem_ld64(tS + 64, sr + 64);
      const int ts = w.kv_lo + j * kBlockN;
      // CTA-uniform: does any row of this tile see a masked key?  Resolved
      // once per tile, not per element.
      FwdRowStep st;
      if (ts + kBlockN - 1 > w.t0 || ts < w.lo_max)
        st = fwd_row_step<true>(sr, lo_r - ts, hi_r - ts, sl2, m_ref);
      else
        st = fwd_row_step<false>(sr, 0, 0, sl2, m_ref);
      const bool need = st.need;
      const float alpha = st.alpha;
      const float m_new = st.m_new;
      l = l * alpha + st.sum;
      uint32_t* pk = sr;  // fwd_row_step packed P (bf16 pairs) into sr[0..63]
      __syncwarp();
      tmem_st32(tS, pk);
      tmem_st32(tS + 32, pk + 32);
      // Rescale the running O (TMEM) when a row of this warp raised its
      // reference max.  O_{j-1} is complete: the S_j commit came after it.
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        uint32_t o[kHeadDim];
        tmem_ld64(tO, o);
#pragma unroll
        for (int i = 0; i < kHeadDim; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st32(tO, o);
        tmem_st32(tO + 32, o + 32);
      }
      m_ref = m_new;
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }

    // ----------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait(&ctl->o_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    if (ok) {
      tc_fence_after();
      uint32_t o[kHeadDim];
      __syncwarp();
      tmem_ld64(tO, o);
      if (valid) {
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t) * geo.Hq + h) * kHeadDim);
#pragma unroll
        for (int i = 0; i < kHeadDim / 8; ++i) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
          dst[i] = v;
        }
        p.lse[static_cast<size_t>(h) * geo.T + t] = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace sa
