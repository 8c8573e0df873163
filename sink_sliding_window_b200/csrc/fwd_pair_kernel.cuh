// Forward kernel on CTA pairs (tcgen05 .cta_group::2, M = 256).
//
// A cluster of two CTAs owns two adjacent query tiles of one key/value head
// g: CTA rank c holds tile 2p + c (128 rows, row r <-> token t0 + r / G, head
// g*G + r % G, as in the single-CTA forward).  Both tiles walk one stream of
// 64-key steps, the union of their key ranges; each CTA masks its own rows.
// Per step the leader CTA (rank 0) issues, for both CTAs at once,
//   S_h = Q K_h^T   M = 256 (both CTAs' Q), N = 64 keys, K = 64 head dims;
//                   CTA c supplies keys [32c, 32c + 32) of the step (B's N/2)
//   O += P_h V_h    M = 256 (P from each CTA's TMEM), N = 64 head dims,
//                   K = 64 keys; CTA c supplies head dims [32c, 32c + 32)
//                   of the step's V rows (B's N/2, MN-major, 64-byte rows)
// so each CTA loads and stores only half of every K and V step and the
// pair issues one MMA stream instead of two.  Softmax, the two alternating
// warpgroups with their own O and running max, the lazily raised reference
// max and the exact merge in the epilogue are those of the single-CTA
// forward (fwd_kernel.cuh), row for row.
//
// Synchronisation across the pair:
//   q_full, k_full[s], v_full[s]  leader's barriers; both CTAs' TMA loads
//                                 complete on them (the leader announces
//                                 both CTAs' bytes)
//   p_full[b]                     leader's barrier; one arrival per softmax
//                                 warp of either CTA (8)
//   s_full[b], kv_empty[s], o_full  each CTA's own; the leader commits to
//                                 both copies (one commit per CTA)
// A cluster barrier after initialisation and before TMEM release keeps
// either CTA from touching a barrier or TMEM the other has not set up or
// has already given back.
//
// Warp roles (320 threads, 2 CTAs per SM): warps 0-7 softmax + epilogue, warp
// 8 TMA producer, warp 9 TMEM allocator (both CTAs) and MMA issuer (leader).
#pragma once
#include "common.cuh"
#include "pair_ptx.cuh"
#include "fwd_kernel.cuh"

namespace sa {

constexpr int kF2Stages = 4;                          // 64-key steps in flight
constexpr int kF2KBytes = (kHalfN / 2) * kHeadDim * 2;  // 32 keys x 64 dims, 128 B rows (SW128)
constexpr int kF2VBytes = kHalfN * (kHeadDim / 2) * 2;  // 64 keys x 32 dims, 64 B rows (SW64)
constexpr int kF2SoftmaxWarps = 8;

struct F2Ctl {
  uint64_t q_full;
  uint64_t k_full[kF2Stages];
  uint64_t v_full[kF2Stages];
  uint64_t kv_empty[kF2Stages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint64_t merge;
  float m_part[2][kBlockM];
  float l_part[2][kBlockM];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kF2SmemBytes =
    1024 /*alignment slack*/ + kTileBytes + kF2Stages * (kF2KBytes + kF2VBytes) + sizeof(F2Ctl);

// This CTA's query tile and the pair's key range.
struct F2Tile {
  int g;       // key/value head
  int t0;      // first token of this CTA's tile (>= T: the tile has no rows)
  int lo_max;  // first key the tile's last row may see
  int kv_lo;   // first key of the pair's step stream
  int n_half;  // 64-key steps of the pair
  bool rows;   // the tile has at least one valid row
};

__device__ __forceinline__ F2Tile f2_tile(const Geometry& geo, uint32_t rank) {
  F2Tile w;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  w.g = pair % geo.Hkv;
  // Later pairs see more keys under a causal mask: hand them out first.
  const int npairs = (geo.num_qblocks + 1) >> 1;
  const int pb = npairs - 1 - pair / geo.Hkv;
  const int t_pair = (2 * pb) << geo.P_log2;
  w.t0 = t_pair + (static_cast<int>(rank) << geo.P_log2);
  w.rows = w.t0 < geo.T;
  const int t_last = min(w.t0 + (1 << geo.P_log2) - 1, geo.T - 1);
  w.lo_max = w.rows ? first_key(geo, t_last) : 0;
  // first_key is non-decreasing in t, so the pair's first row has the
  // smallest first key and the pair's last valid token the largest key.
  w.kv_lo = first_key(geo, t_pair);
  const int t_end = min(t_pair + (2 << geo.P_log2) - 1, geo.T - 1);
  w.n_half = (t_end - w.kv_lo + kHalfN) / kHalfN;
  return w;
}

// S (64 columns of each CTA's 128 rows) = Q K^T for one 64-key step; k_addr:
// this CTA's 32 keys of the step (K-major, 128 B rows).
__device__ __forceinline__ void f2_issue_qk(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = make_idesc_bf16(2 * kBlockM, kHalfN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint64_t a = make_sdesc_sw128(q_addr + kk * 32, 16, 1024);
    const uint64_t b = make_sdesc_sw128(k_addr + kk * 32, 16, 1024);
    mma_ss_pair(tmem_s, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O += P V for one 64-key step; P (bf16 pairs) in the 32 TMEM columns at
// tmem_p; v_addr: this CTA's 32 head dims of the step's 64 value rows
// (MN-major: one 64-byte row of dims per key, 64-byte swizzle).
__device__ __forceinline__ void f2_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr, bool accumulate) {
  constexpr uint32_t idesc = make_idesc_bf16(2 * kBlockM, kHeadDim, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kHalfN / 16; ++kk) {
    // 16 keys = 16 rows of 64 B; SBO = 8 rows; LBO (next 32-dim group) unused.
    const uint64_t b = make_sdesc_sw64(v_addr + kk * 1024, kF2VBytes, 512);
    mma_ts_pair(tmem_o, tmem_p + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kFwdThreads, 2)
    sink_attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;
  uint8_t* sV = sK + kF2Stages * kF2KBytes;
  F2Ctl* ctl = reinterpret_cast<F2Ctl*>(sV + kF2Stages * kF2VBytes);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  const Geometry& geo = p.geo;
  const F2Tile w = f2_tile(geo, rank);

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < kF2Stages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->p_full[b], 2 * (kF2SoftmaxWarps / 2));
    }
    mbar_init(&ctl->o_full, 1);
    mbar_init(&ctl->merge, 2 * kBlockM);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == kFwdMmaWarp) {
    tmem_alloc_pair(&ctl->tmem_base, kFwdTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kFwdProducerWarp) {
    // ---------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int dq = static_cast<int>(rank) * (kHeadDim / 2);
      const int dk = static_cast<int>(rank) * (kHalfN / 2);
      if (rank == 0) mbar_arrive_expect_tx(&ctl->q_full, 2 * kTileBytes);
      tma_load_3d_pair(sQ, &tm_q, mapa_shared(smem_u32(&ctl->q_full), 0), 0, w.g << geo.G_log2, w.t0);
      for (int h = 0; h < w.n_half; ++h) {
        const int s = h % kF2Stages;
        if (h >= kF2Stages && !mbar_wait_cl(&ctl->kv_empty[s], ((h / kF2Stages) - 1) & 1, abort, &g_device_error,
                                            kDevErrTimeoutProducer))
          break;
        const int ks = w.kv_lo + h * kHalfN;
        if (rank == 0) mbar_arrive_expect_tx(&ctl->k_full[s], 2 * kF2KBytes);
        tma_load_3d_pair(sK + s * kF2KBytes, &tm_k, mapa_shared(smem_u32(&ctl->k_full[s]), 0), 0, w.g, ks + dk);
        if (rank == 0) mbar_arrive_expect_tx(&ctl->v_full[s], 2 * kF2VBytes);
        tma_load_3d_pair(sV + s * kF2VBytes, &tm_v, mapa_shared(smem_u32(&ctl->v_full[s]), 0), dq, w.g, ks);
      }
    }
  } else if (warp == kFwdMmaWarp) {
    // ------------------------------------------------ MMA issuer (leader)
    // Order as in the single-CTA forward: S_0, S_1, then for every step h:
    // O_{h%2} += P_h V_h, S_{h+2} into the buffer P_h just left.
    if (rank == 0 && elect_one()) {
      const uint32_t tS = tmem + kFwdTmemS;
      const uint32_t tO = tmem + kFwdTmemO;
      const uint32_t q_addr = smem_u32(sQ);
      auto commit_both = [](uint64_t* bar) {
        const uint32_t a = smem_u32(bar);
        tc_commit_pair(a);
        tc_commit_pair(mapa_shared(a, 1));
      };
      bool ok = mbar_wait_cl(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      for (int h = 0; ok && h < min(2, w.n_half); ++h) {
        ok = mbar_wait_cl(&ctl->k_full[h], 0, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        f2_issue_qk(tS + h * kHalfN, q_addr, smem_u32(sK + h * kF2KBytes));
        commit_both(&ctl->s_full[h]);
      }
      for (int h = 0; ok && h < w.n_half; ++h) {
        const int b = h & 1;
        const int s = h % kF2Stages;
        ok = mbar_wait_cl(&ctl->v_full[s], (h / kF2Stages) & 1, abort, &g_device_error, kDevErrTimeoutMma) &&
             mbar_wait_cl(&ctl->p_full[b], (h >> 1) & 1, abort, &g_device_error, kDevErrTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        f2_issue_pv(tO + b * kHeadDim, tS + b * kHalfN, smem_u32(sV + s * kF2VBytes), h >= 2);
        commit_both(&ctl->kv_empty[s]);
        const int h2 = h + 2;
        if (h2 < w.n_half) {
          const int s2 = h2 % kF2Stages;
          ok = mbar_wait_cl(&ctl->k_full[s2], (h2 / kF2Stages) & 1, abort, &g_device_error, kDevErrTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          f2_issue_qk(tS + b * kHalfN, q_addr, smem_u32(sK + s2 * kF2KBytes));
          commit_both(&ctl->s_full[b]);
        }
      }
      if (ok) commit_both(&ctl->o_full);
    }
  } else {
    // ------------------------------------------- softmax (1 row per thread)
    const int wg = warp >> 2;  // steps h with h % 2 == wg
    const int r = threadIdx.x & (kBlockM - 1);
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
    float m_ref = sink * kLog2e;
    float l = (wg == 0 && sink != -INFINITY) ? 1.f : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + kFwdTmemS + wg * kHalfN;
    const uint32_t tO = tmem + lane_base + kFwdTmemO + wg * kHeadDim;
    const float sl2 = p.scale_log2;
    const uint32_t p_bar = mapa_shared(smem_u32(&ctl->p_full[wg]), 0);
    bool ok = true;

    for (int hs = wg, i = 0; hs < w.n_half; hs += 2, ++i) {
      ok = warp_all(mbar_wait_cl(&ctl->s_full[wg], i & 1, abort, &g_device_error, kDevErrTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kHalfN];
      tmem_ld64(tS, sr);
      const int ks = w.kv_lo + hs * kHalfN;
      // CTA-uniform: does any row of this tile see a masked key in this step?
      FwdRowStep st;
      if (!w.rows || ks + kHalfN - 1 > w.t0 || ks < w.lo_max)
        st = fwd_row_step<true>(sr, lo_r - ks, hi_r - ks, sl2, m_ref);
      else
        st = fwd_row_step<false>(sr, 0, 0, sl2, m_ref);
      l = l * st.alpha + st.sum;
      __syncwarp();
      tmem_st32(tS, sr);
      if (i > 0 && __any_sync(0xffffffffu, st.need)) {
        uint32_t o[kHeadDim];
        tmem_ld64(tO, o);
#pragma unroll
        for (int c = 0; c < kHeadDim; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * st.alpha);
        tmem_st32(tO, o);
        tmem_st32(tO + 32, o + 32);
      }
      m_ref = st.m_new;
      // Every lane's P (and rescaled O) stores have completed (tmem_st32
      // waits for them); one arrival per warp on the leader's barrier.
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive_cluster(p_bar);
    }

    // ------------------------------------------------ merge and epilogue
    if (ok) ok = mbar_wait_cl(&ctl->o_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    ok = warp_all(ok);
    ctl->m_part[wg][r] = m_ref;
    ctl->l_part[wg][r] = l;
    mbar_arrive(&ctl->merge);
    if (ok) ok = mbar_wait(&ctl->merge, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
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

  // Neither CTA releases TMEM or exits while the other may still signal its
  // barriers or the leader's MMAs may still write its TMEM (both waited for
  // o_full, which follows every MMA, unless a wait gave up).
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == kFwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kFwdTmemCols);
  }
}

}  // namespace sa
