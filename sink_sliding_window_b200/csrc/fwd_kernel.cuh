// Forward kernel: causal GQA attention with a per-head sink logit, sliding
// window and packed documents, on sm_100a tensor cores.
//
// Query tile: (128 / G) consecutive tokens x the G query heads of one
// key/value head g, i.e. 128 MMA rows, row r <-> (token t0 + r / G, head
// g*G + r % G).  Because q is [T][Hq][D], the G heads of a group are
// contiguous and a single 3-D TMA box {64, G, 128/G} lands the tile in
// exactly this row order.  Every key/value tile that is loaded serves all G
// heads of the group.
//
// One-tile mode (kTiles = 1): a CTA owns one query tile.  Keys are consumed
// in steps of 64 ("halves" of a 128-key K/V tile):
//   S_h = Q K_h^T          tcgen05.mma, bf16 in, fp32 in TMEM (64 columns),
//                          into S/P buffer h % 2
//   softmax (1 thread = 1 row, the row lives in that thread's TMEM lane):
//     masked logits -> running reference max m (seeded with the sink logit,
//     lazily raised), P = 2^(S*scale*log2e - m) as bf16 written back into the
//     buffer's first 32 columns, row sum l (seeded with the sink's e^{s-m}=1)
//   O += P_h V_h           tcgen05.mma with A = P from TMEM, fp32 O in TMEM
// The steps alternate between two softmax warpgroups: warpgroup b takes the
// steps h with h % 2 == b, owns S/P buffer b and its own accumulator O_b, and
// keeps its own running max and sum.  Softmax is invariant to how the keys
// are split, so the epilogue merges the two partial results exactly:
//   m = max(m_0, m_1),  l = l_0 2^{m_0 - m} + l_1 2^{m_1 - m},
//   out = (O_0 2^{m_0 - m} + O_1 2^{m_1 - m}) / l
// (the sink is counted once, in warpgroup 0's seed).  While one warpgroup
// waits for its next S, the other works on its own step; with two CTAs per
// SM, four softmax warps share each SM sub-partition's exp2 unit.  A
// warpgroup may rescale its O_b without waiting for an MMA: the commit that
// announced S_h came after the previous PV into O_b (tcgen05 MMAs of one
// thread execute in order).
// Tiles outside the causal / window / document range are never visited; only
// the edge steps apply an element mask.
//
// Two-tile mode (kTiles = 2, what sink_attn_fwd runs): the CTA owns two
// adjacent query tiles of the same head g, warpgroup b takes every step of
// tile b (its own S/P buffer, O_b, running max and sum, no merge), and one
// K/V stream over the union of the two tiles' key ranges serves both; each
// warpgroup masks its own rows.  The MMA issuer serves the warpgroups in turn
// (PV_b and S_b of the next step as soon as P_b is written), so one
// warpgroup's exponentials overlap the other's S round trip, as the
// alternating steps do in the one-tile mode.  Set-up, first loads and
// epilogue are paid once per two tiles, which matters most on sliding-window
// layers (a tile sees only 3-4 key steps there).
//
// Warp roles (320 threads, 2 CTAs per SM): warps 0-7 softmax + epilogue (two
// warpgroups), warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer.
// TMEM: S/P buffers in columns [0,64) and [64,128), O_0 in [128,192), O_1 in
// [192,256).
#pragma once
#include "common.cuh"

namespace sa {

constexpr int kFwdStages = 2;
constexpr int kFwdThreads = 320;
constexpr int kFwdProducerWarp = 8;
constexpr int kFwdMmaWarp = 9;
constexpr int kHalfN = kBlockN / 2;  // keys per softmax step
constexpr int kHalfBytes = kHalfN * kHeadDim * 2;
constexpr uint32_t kFwdTmemCols = 256;
constexpr uint32_t kFwdTmemS = 0;
constexpr uint32_t kFwdTmemO = 128;
// The reference max is raised only when a step's max exceeds it by more than
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
  uint64_t s_full[2];   // S_h computed into buffer h % 2
  uint64_t p_full[2];   // P_h written into buffer h % 2 (128 arrivals)
  uint64_t o_full;      // every MMA done (epilogue may read O_0, O_1)
  uint64_t merge;       // both warpgroups published their (m, l) (256 arrivals)
  float m_part[2][kBlockM];
  float l_part[2][kBlockM];
  uint32_t tmem_base;
  int abort;
};

// Q tiles (kTiles), then K and V stages, then the control block.
template <int kTiles>
constexpr size_t fwd_smem_bytes() {
  return 1024 /*alignment slack*/ + kTileBytes * (kTiles + 2 * kFwdStages) + sizeof(FwdCtl);
}

// Query tiles handled by this CTA (kTiles adjacent tiles of head g) and the
// key range of their common step stream.
struct FwdTile {
  int g;       // key/value head
  int t0;      // first token of the CTA's first tile
  int kv_lo;   // first key any row may see
  int n_half;  // 64-key steps to visit
  int n_tiles; // 128-key K/V tiles to load
};

// Work unit `idx` (0 .. units x Hkv - 1; a CTA's blockIdx.x in the
// non-persistent kernels).
template <int kTiles>
__device__ __forceinline__ FwdTile fwd_tile(const Geometry& geo, int idx) {
  FwdTile w;
  w.g = idx % geo.Hkv;
  // Later tiles see more keys under a causal mask: hand them out first.
  const int units = (geo.num_qblocks + kTiles - 1) / kTiles;
  const int u = units - 1 - idx / geo.Hkv;
  w.t0 = (u * kTiles) << geo.P_log2;
  // first_key is non-decreasing in t: the first row has the smallest first
  // key, the last valid token the largest key.
  const int t_end = min(w.t0 + (kTiles << geo.P_log2) - 1, geo.T - 1);
  w.kv_lo = first_key(geo, w.t0);
  w.n_half = (t_end - w.kv_lo + kHalfN) / kHalfN;
  w.n_tiles = (w.n_half + 1) / 2;
  return w;
}

// S (64 columns) = Q K^T for the 64 keys whose K rows start at k_addr.
__device__ __forceinline__ void fwd_issue_qk(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = make_idesc_bf16(kBlockM, kHalfN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint64_t a = make_sdesc_sw128(q_addr + kk * 32, 16, 1024);
    const uint64_t b = make_sdesc_sw128(k_addr + kk * 32, 16, 1024);
    mma_ss(tmem_s, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O += P V for the 64 keys whose V rows start at v_addr; P (bf16 pairs) in
// the 32 TMEM columns at tmem_p.
__device__ __forceinline__ void fwd_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr, bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(kBlockM, kHeadDim, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kHalfN / 16; ++kk) {
    const uint64_t b = make_sdesc_sw128(v_addr + kk * 2048, kTileBytes, 1024);
    mma_ts(tmem_o, tmem_p + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One 64-key step of one query row: mask (kMask), row max, lazily raised
// reference max, P = 2^(S*scale*log2e - m) packed to bf16 pairs in s[0..31],
// and the row sum of P.  s[] holds the row's 64 fp32 logits on entry.
struct FwdRowStep {
  bool need;    // the reference max was raised
  float alpha;  // factor applied to the running sum / O (1 when not raised)
  float m_new;  // reference max after this step
  float sum;    // sum of this step's P
};

template <bool kMask>
__device__ __forceinline__ FwdRowStep fwd_row_step(uint32_t* s, int c_lo, int c_hi, float sl2, float m_ref) {
  float x[kHalfN];
#pragma unroll
  for (int c = 0; c < kHalfN; ++c) {
    x[c] = __uint_as_float(s[c]);
    if (kMask) x[c] = (c < c_lo || c > c_hi) ? -INFINITY : x[c];
  }
  // Row max as four independent chains of 3-input maxima, then combined.
  float m4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m4[i] = fmax3(x[i], x[i + 4], x[i + 8]);
#pragma unroll
  for (int c = 12; c < kHalfN - 4; c += 8) {
#pragma unroll
    for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], x[c + i], x[c + 4 + i]);
  }
  const float mx = fmax3(fmaxf(m4[0], x[kHalfN - 4]), fmax3(m4[1], x[kHalfN - 3], x[kHalfN - 2]),
                         fmax3(m4[2], m4[3], x[kHalfN - 1]));
  const float mx2 = mx * sl2;
  FwdRowStep r;
  r.need = mx2 > m_ref + kRescaleLog2;
  r.alpha = r.need ? ex2_approx(m_ref - mx2) : 1.f;
  r.m_new = r.need ? mx2 : m_ref;
  const float m_use = (r.m_new == -INFINITY) ? 0.f : r.m_new;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < kHalfN / 2; ++c) {
    const float e0 = ex2_approx(fmaf(x[2 * c], sl2, -m_use));
    const float e1 = ex2_approx(fmaf(x[2 * c + 1], sl2, -m_use));
    acc[(2 * c) & 3] += e0;
    acc[(2 * c + 1) & 3] += e1;
    s[c] = pack_bf16x2(e0, e1);
  }
  r.sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  return r;
}

template <int kTiles>
__global__ void __launch_bounds__(kFwdThreads, 2)
    sink_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(kTiles == 1 || kTiles == 2, "one or two query tiles per CTA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTiles * kTileBytes;
  uint8_t* sV = sK + kFwdStages * kTileBytes;
  FwdCtl* ctl = reinterpret_cast<FwdCtl*>(sV + kFwdStages * kTileBytes);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const Geometry& geo = p.geo;
  const FwdTile w = fwd_tile<kTiles>(geo, static_cast<int>(blockIdx.x));

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->p_full[b], kBlockM);
    }
    mbar_init(&ctl->o_full, 1);
    mbar_init(&ctl->merge, 2 * kBlockM);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == kFwdMmaWarp) {
    tmem_alloc(&ctl->tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kFwdProducerWarp) {
    // ---------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&ctl->q_full, kTiles * kTileBytes);
#pragma unroll
      for (int u = 0; u < kTiles; ++u)
        tma_load_3d(sQ + u * kTileBytes, &tm_q, &ctl->q_full, 0, w.g << geo.G_log2, w.t0 + (u << geo.P_log2));
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
  } else if (warp == kFwdMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S_0, S_1, then for every step h: O_{h%2} += P_h V_h, S_{h+2}
    // into the buffer P_h just left (tcgen05 MMAs of one thread execute in
    // order, so the PV reads P_h before S_{h+2} overwrites it).
    if (kTiles == 2 && elect_one()) {
      // Two tiles: warpgroup b's steps are S_b(h) -> P_b(h) -> O_b += P_b V(h)
      // -> S_b(h+1) into the buffer P_b(h) just left (the PV, issued first,
      // reads P_b(h) before the S MMA overwrites it).  S_0(0) and S_1(0) go
      // out together; then the warpgroups are served in turn at every step.
      const uint32_t tS = tmem + kFwdTmemS;
      const uint32_t tO = tmem + kFwdTmemO;
      bool ok = mbar_wait(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutMma) &&
                mbar_wait(&ctl->k_full[0], 0, abort, &g_device_error, kDevErrTimeoutMma);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          fwd_issue_qk(tS + b * kHalfN, smem_u32(sQ + b * kTileBytes), smem_u32(sK));
          tc_commit(&ctl->s_full[b]);
        }
      }
      for (int h = 0; ok && h < w.n_half; ++h) {
        const int j = h >> 1;
        const int s = j % kFwdStages;
        const int hn = h + 1;
        const int jn = hn >> 1;
        const int sn = jn % kFwdStages;
        ok = mbar_wait(&ctl->v_full[s], (j / kFwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma) &&
             (hn >= w.n_half ||
              mbar_wait(&ctl->k_full[sn], (jn / kFwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma));
        for (int b = 0; ok && b < 2; ++b) {
          ok = mbar_wait(&ctl->p_full[b], h & 1, abort, &g_device_error, kDevErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          fwd_issue_pv(tO + b * kHeadDim, tS + b * kHalfN, smem_u32(sV + s * kTileBytes) + (h & 1) * kHalfBytes,
                       h > 0);
          if (hn < w.n_half) {
            fwd_issue_qk(tS + b * kHalfN, smem_u32(sQ + b * kTileBytes),
                         smem_u32(sK + sn * kTileBytes) + (hn & 1) * kHalfBytes);
            tc_commit(&ctl->s_full[b]);
          }
        }
        // K/V tile j is done once both warpgroups' PVs of its second step
        // (or of the last step) are.
        if (ok && ((h & 1) == 1 || h == w.n_half - 1)) tc_commit(&ctl->kv_empty[s]);
      }
      if (ok) tc_commit(&ctl->o_full);
    } else if (kTiles == 1 && elect_one()) {
      const uint32_t tS = tmem + kFwdTmemS;
      const uint32_t tO = tmem + kFwdTmemO;
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      for (int h = 0; ok && h < min(2, w.n_half); ++h) {
        ok = mbar_wait(&ctl->k_full[0], 0, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        fwd_issue_qk(tS + h * kHalfN, q_addr, smem_u32(sK) + h * kHalfBytes);
        tc_commit(&ctl->s_full[h]);
      }
      for (int h = 0; ok && h < w.n_half; ++h) {
        const int b = h & 1;
        const int j = h >> 1;
        const int s = j % kFwdStages;
        ok = mbar_wait(&ctl->v_full[s], (j / kFwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma) &&
             mbar_wait(&ctl->p_full[b], (h >> 1) & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        fwd_issue_pv(tO + b * kHeadDim, tS + b * kHalfN, smem_u32(sV + s * kTileBytes) + b * kHalfBytes, h >= 2);
        if (b == 1 || h == w.n_half - 1) tc_commit(&ctl->kv_empty[s]);
        const int h2 = h + 2;
        if (h2 < w.n_half) {
          const int j2 = h2 >> 1;
          const int s2 = j2 % kFwdStages;
          ok = mbar_wait(&ctl->k_full[s2], (j2 / kFwdStages) & 1, abort, &g_device_error, kDevErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          fwd_issue_qk(tS + b * kHalfN, q_addr, smem_u32(sK + s2 * kTileBytes) + b * kHalfBytes);
          tc_commit(&ctl->s_full[b]);
        }
      }
      if (ok) tc_commit(&ctl->o_full);
    }
  } else {
    // ------------------------------------------- softmax (1 row per thread)
    // One tile: warpgroup wg takes the steps h with h % 2 == wg.  Two tiles:
    // warpgroup wg takes every step of tile wg.
    const int wg = warp >> 2;
    const int r = threadIdx.x & (kBlockM - 1);
    const int G = 1 << geo.G_log2;
    const int tw0 = w.t0 + (kTiles == 2 ? (wg << geo.P_log2) : 0);  // first token of this warpgroup's tile
    const bool rows = tw0 < geo.T;
    const int lo_max = rows ? first_key(geo, min(tw0 + (1 << geo.P_log2) - 1, geo.T - 1)) : 0;
    const int t = tw0 + (r >> geo.G_log2);
    const int h = (w.g << geo.G_log2) + (r & (G - 1));
    const bool valid = t < geo.T;
    int lo_r = 0, hi_r = -1;  // allowed keys [lo_r, hi_r]; empty for padding rows
    if (valid) {
      lo_r = first_key(geo, t);
      hi_r = t;
    }
    const float sink = __ldg(p.sinks + h);
    // Every warpgroup takes the sink logit as its first reference max; the
    // sink's own e^{s-m} = 1 is counted once per row (one tile: by warpgroup
    // 0 only).
    float m_ref = sink * kLog2e;  // -inf when the sink is off
    float l = ((kTiles == 2 || wg == 0) && sink != -INFINITY) ? 1.f : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + kFwdTmemS + wg * kHalfN;
    const uint32_t tO = tmem + lane_base + kFwdTmemO + wg * kHeadDim;
    const float sl2 = p.scale_log2;
    bool ok = true;

    for (int hs = (kTiles == 1 ? wg : 0), i = 0; hs < w.n_half; hs += 3 - kTiles, ++i) {
      ok = warp_all(mbar_wait(&ctl->s_full[wg], i & 1, abort, &g_device_error, kDevErrTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kHalfN];
      tmem_ld64(tS, sr);
      const int ks = w.kv_lo + hs * kHalfN;
      // Uniform over the tile: does any row of this step see a masked key?
      // Resolved once per step, not per element.
      FwdRowStep st;
      if (!rows || ks + kHalfN - 1 > tw0 || ks < lo_max)
        st = fwd_row_step<true>(sr, lo_r - ks, hi_r - ks, sl2, m_ref);
      else
        st = fwd_row_step<false>(sr, 0, 0, sl2, m_ref);
      l = l * st.alpha + st.sum;
      __syncwarp();
      tmem_st32(tS, sr);  // fwd_row_step packed P (bf16 pairs) into sr[0..31]
      // Rescale this warpgroup's O when a row of the warp raised its
      // reference max.  Its previous PV is complete: it was issued before
      // the S MMA whose commit was just observed.
      if (i > 0 && __any_sync(0xffffffffu, st.need)) {
        uint32_t o[kHeadDim];
        tmem_ld64(tO, o);
#pragma unroll
        for (int c = 0; c < kHeadDim; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * st.alpha);
        tmem_st32(tO, o);
        tmem_st32(tO + 32, o + 32);
      }
      m_ref = st.m_new;
      tc_fence_before();
      mbar_arrive(&ctl->p_full[wg]);
    }

    if (ok) ok = mbar_wait(&ctl->o_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    ok = warp_all(ok);
    if constexpr (kTiles == 2) {
      // ------------------------------------------ epilogue of tile wg alone
      if (ok) {
        tc_fence_after();
        uint32_t o[kHeadDim];
        __syncwarp();
        tmem_ld64(tO, o);
        if (valid) {
          const float inv_l = l > 0.f ? 1.f / l : 0.f;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t) * geo.Hq + h) * kHeadDim);
#pragma unroll
          for (int c8 = 0; c8 < kHeadDim / 8; ++c8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * c8 + 0]) * inv_l, __uint_as_float(o[8 * c8 + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * c8 + 2]) * inv_l, __uint_as_float(o[8 * c8 + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * c8 + 4]) * inv_l, __uint_as_float(o[8 * c8 + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * c8 + 6]) * inv_l, __uint_as_float(o[8 * c8 + 7]) * inv_l);
            dst[c8] = v;
          }
          p.lse[static_cast<size_t>(h) * geo.T + t] = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
        }
      }
    } else {
      // ------------------------------------------------ merge and epilogue
      // Each warpgroup publishes its (m, l); then warpgroup b writes output
      // columns [32 b, 32 b + 32) of its rows from both accumulators.
      ctl->m_part[wg][r] = m_ref;
      ctl->l_part[wg][r] = l;
      uint32_t merge_phase = 0;
      mbar_arrive(&ctl->merge);
      if (ok) ok = mbar_wait(&ctl->merge, merge_phase, abort, &g_device_error, kDevErrTimeoutEpilogue);
      ok = warp_all(ok);
      if (ok) {
        tc_fence_after();
        const bool has1 = w.n_half >= 2;  // warpgroup 1 saw at least one step
        const float m0 = ctl->m_part[0][r], l0 = ctl->l_part[0][r];
        const float m1 = has1 ? ctl->m_part[1][r] : -INFINITY;
        const float l1 = has1 ? ctl->l_part[1][r] : 0.f;
        const float m = fmaxf(m0, m1);
        const float f0 = (m == -INFINITY) ? 0.f : ex2_approx(m0 - m);
        const float f1 = (m == -INFINITY || !has1) ? 0.f : ex2_approx(m1 - m);
        const float lt = l0 * f0 + l1 * f1;
        const uint32_t tO0 = tmem + lane_base + kFwdTmemO + wg * 32;
        uint32_t o0[32], o1[32];
        __syncwarp();
        tmem_ld32(tO0, o0);
        if (has1) tmem_ld32(tO0 + kHeadDim, o1);
        if (valid) {
          const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
          const float g0 = f0 * inv_l, g1 = f1 * inv_l;
          uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t) * geo.Hq + h) * kHeadDim + wg * 32);
  #pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float y[8];
  #pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int c = 8 * c8 + u;
              y[u] = __uint_as_float(o0[c]) * g0;
              if (has1) y[u] = fmaf(__uint_as_float(o1[c]), g1, y[u]);
            }
            uint4 v;
            v.x = pack_bf16x2(y[0], y[1]);
            v.y = pack_bf16x2(y[2], y[3]);
            v.z = pack_bf16x2(y[4], y[5]);
            v.w = pack_bf16x2(y[6], y[7]);
            dst[c8] = v;
          }
          if (wg == 0) p.lse[static_cast<size_t>(h) * geo.T + t] = lt > 0.f ? (m + __log2f(lt)) * kLn2 : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kFwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace sa
