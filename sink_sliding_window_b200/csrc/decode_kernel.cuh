// Decode forward: a few new query tokens per sequence attend to that
// sequence's key/value cache (sink, sliding window and causal mask as in the
// forward).  Three kernels per call: append the new keys/values to the cache,
// attend (split over the cache), combine the splits.
//
// Cache layout.  Sequence b owns `C` slots of k_cache / v_cache, each slot
// [Hkv][D]; the token at position p lives in slot p mod C.  A cache with
// C >= the sequence length is a plain linear cache; a sliding-window layer
// can keep a ring of C >= window + new_tokens - 1 slots.  Before a call the
// cache holds positions [0, L0) (the last C of them), L0 = cache_seqlens[b];
// the call writes the Lq new tokens at positions L0 .. L0+Lq-1 and their
// queries attend with the same masks as the forward: key position j is
// allowed for query position i iff j <= i and (window <= 0 or i - j < window).
//
// Attention kernel (one CTA = sequence b, key/value head g, one split of
// the cache slots).  With only G x Lq (<= 64) query rows per head group, the
// MMA roles are swapped so the keys fill the 128-row M dimension:
//   S^T = K Q^T           M = 128 keys of a slot tile, N = 64 query rows
//                         (G x Lq real, the rest zero), K = D
//   softmax over keys     one thread per key (its TMEM lane); the per-row
//                         reference max is shared by all threads (seeded
//                         with the sink logit, raised lazily: only when some
//                         key exceeds it by more than 2^8, found by an OR
//                         over the keys in the barrier hardware)
//   O^T += [V | 1]^T P^T  M = 128: rows 0..63 are the head dims (A = V read
//                         MN-major), rows 64..127 multiply P^T by a tile of
//                         ones and so accumulate the row sums l for free;
//                         B = P^T [keys][rows] written to shared memory
// Softmax is invariant to the order of the keys, so slots are visited in
// slot order; each key's position (and so its mask) follows from the slot.
// Each split writes (O, l, m) partials; the combine kernel merges them and
// adds the sink's e^{s-m} once.  With a single split (the cache of every
// (sequence, key/value head) fits one CTA's share of the grid) the attention
// kernel finishes the rows itself and the combine launch is skipped.
//
// e4m3 cache variant (kF8): the cache holds FP8 e4m3 codes with one
// dequantisation scale per key/value head (k = code * k_scale[g], likewise
// v).  Tiles arrive as bytes; the softmax threads (one slot each) widen their
// slot's K row straight into TMEM, where it is the A operand of the S^T MMA,
// and their V row into a shared-memory tile for the PV MMA.  This variant's
// MMAs run in fp16: one instruction widens two e4m3 codes to fp16, exactly;
// Q is converted from bf16 to fp16 once per CTA (saturating at +-65504) and P
// is rounded to fp16 (P <= 2^8 here, so fp16 keeps more of it than bf16).
// k_scale folds into the logit scale and v_scale into O.  Half the bytes of
// the bf16 cache cross HBM.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"

namespace sa {

constexpr int kDecThreads = 192;  // warps 0-3 softmax (one key per thread), 4 TMA producer, 5 MMA
constexpr int kDecThreads8 = 320; // e4m3 cache: + warps 6-9 widening K and V (one slot per thread)
constexpr int kDecConvWarp0 = 6;
constexpr int kDecProducerWarp = 4;
constexpr int kDecMmaWarp = 5;
constexpr int kDecRows = 64;      // MMA N: query rows per CTA (G x Lq <= 64)
constexpr int kDecTile = 128;     // slots per key tile (MMA M)
constexpr int kDecStages = 2;      // bf16 cache: K/V tile stages
constexpr int kDecStages8 = 2;     // e4m3 cache: byte-tile stages
constexpr int kDecQBytes = kDecRows * kHeadDim * 2;    // Q tile, [64][64] bf16
constexpr int kDecKvBytes = kDecTile * kHeadDim * 2;   // one K or V tile, [128][64] bf16
constexpr int kDecPBytes = kDecTile * kDecRows * 2;    // P^T tile, [128 keys][64 rows] bf16
constexpr int kDecKv8Bytes = kDecTile * kHeadDim;      // one e4m3 K or V tile, [128][64] bytes
constexpr uint32_t kDecTmemCols = 256;  // S^T buffers [0,64), [64,128); O^T [128,192)
constexpr uint32_t kDecTmemS = 0;
constexpr uint32_t kDecTmemO = 128;
constexpr uint32_t kDecTmemK = 192;  // e4m3 cache: widened K tiles, two 32-column buffers
constexpr float kDecRescaleLog2 = 8.0f;

struct DecParams {
  int batch, Lq, C, Hq, Hkv, G, R;  // R = G * Lq query rows per (sequence, kv head)
  int G_log2;                       // G is a power of two
  int window;                       // <= 0: full causal
  int n_split;                      // CTAs per (sequence, kv head)
  float scale_log2;                 // scale * log2(e)
  const int* seqlens;               // [batch] tokens in the cache before this call
  const float* k_scale;             // e4m3 cache: [Hkv] dequantisation scales (else unused)
  const float* v_scale;
  const float* sinks;               // [Hq]
  float* o_part;                    // [batch][Hkv][n_split][64 rows][64] unnormalised O
  float* m_part;                    // [batch][Hkv][n_split][64 rows] reference max (log2 units)
  float* l_part;                    // [batch][Hkv][n_split][64 rows] sum of P
  __nv_bfloat16* out;               // n_split == 1: the attention kernel writes out and lse itself
  float* lse_out;
};

struct DecCtl {
  uint64_t q_full;
  uint64_t q_conv;      // e4m3 cache: Q converted to fp16 in place (128 arrivals)
  uint64_t k_full[kDecStages8];
  uint64_t k_empty[kDecStages8];
  uint64_t v_full[kDecStages8];
  uint64_t v_empty[kDecStages8];
  uint64_t kt_full[2];  // e4m3 cache: K of tile i widened into TMEM buffer i % 2 (128 arrivals)
  uint64_t v_ready[2];  // e4m3 cache: V of tile i widened into fp16 tile i % 2, barrier i % 2
                        // (128 arrivals; split so that a converter two tiles ahead stays unambiguous)
  uint64_t s_full[2];   // S^T of tile i in TMEM buffer i % 2
  uint64_t s_free[2];   // the softmax has loaded that S^T (128 arrivals)
  uint64_t p_full;      // P^T of tile i written (128 arrivals)
  uint64_t pv_done[2];  // O^T += ... of tile i complete, barrier i % 2 (the softmax and the e4m3
                        // widening threads wait on different tiles' completions)
  uint64_t o_full;      // every MMA done
  float m_ref[kDecRows];    // reference max per query row (log2 units)
  float alpha[kDecRows];    // rescale factor of the current tile per row
  float wmax[4][kDecRows];  // per-warp tile maxima (rare path)
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kDecSmemBytes = 1024 /*alignment slack*/ + kDecQBytes + 2 * kDecStages * kDecKvBytes +
                                 kDecKvBytes /*ones*/ + kDecPBytes + sizeof(DecCtl);
constexpr size_t kDecSmemBytes8 = 1024 + kDecQBytes + 2 * kDecStages8 * kDecKv8Bytes + 2 * kDecKvBytes /*fp16 V x2*/ +
                                  kDecKvBytes /*ones*/ + kDecPBytes + sizeof(DecCtl);
// e4m3 cache with the PV product in FP8: no widened V tiles; the ones tile
// and P^T are e4m3 bytes, [128 slots][64].
constexpr int kDecP8Bytes = kDecTile * kDecRows;
constexpr size_t kDecSmemBytesPv8 =
    1024 + kDecQBytes + 2 * kDecStages8 * kDecKv8Bytes + kDecKv8Bytes /*ones*/ + kDecP8Bytes + sizeof(DecCtl);

// Slot range of one CTA: [z0, z0 + 128 n) in 128-slot tiles.
struct DecWork {
  int b, g, split;
  int L0, L;     // cache length before / after this call
  int z0;        // first slot of the first tile
  int n;         // tiles to visit (may be 0)
  bool bad;      // a needed key is no longer in the cache
};

__device__ __forceinline__ DecWork dec_work(const DecParams& p) {
  DecWork w;
  const int bg = blockIdx.x / p.n_split;
  w.split = blockIdx.x % p.n_split;
  w.b = bg / p.Hkv;
  w.g = bg % p.Hkv;
  w.L0 = __ldg(p.seqlens + w.b);
  w.L = w.L0 + p.Lq;
  if (w.L0 < 0) {  // invalid length: visit nothing, report it
    w.z0 = 0;
    w.n = 0;
    w.bad = true;
    return w;
  }
  // Oldest position any new query may see.
  const int pmin = p.window > 0 ? max(0, w.L0 - p.window + 1) : 0;
  int zlo, zhi;  // slots to scan
  if (w.L <= p.C) {
    zlo = pmin;  // no wrap: slot == position
    zhi = w.L;
    w.bad = false;
  } else {
    zlo = 0;     // wrapped ring: every slot holds one of the last C positions
    zhi = p.C;
    w.bad = pmin < w.L - p.C;
  }
  const int t_first = zlo / kDecTile;
  const int t_count = (zhi + kDecTile - 1) / kDecTile - t_first;
  const int per = (t_count + p.n_split - 1) / p.n_split;
  const int t_begin = min(t_count, w.split * per);
  w.n = min(t_count, t_begin + per) - t_begin;
  w.z0 = (t_first + t_begin) * kDecTile;
  return w;
}

// Slot of the newest token, (L - 1) mod C (one division per CTA).
__device__ __forceinline__ int dec_last_slot(int L, int C) {
  int r = (L - 1) % C;
  return r < 0 ? r + C : r;
}

// Position of the token in slot z, 0 <= z < C (negative: the slot holds no
// token yet): the largest position <= L - 1 that is congruent to z mod C.
__device__ __forceinline__ int dec_slot_pos(int z, int L, int last_slot, int C) {
  int d = last_slot - z;
  if (d < 0) d += C;
  return L - 1 - d;
}

// S^T (kN columns) = K Q^T: A = the K tile (128 slots, K-major), B = the
// first kN rows of Q (K-major).  kN = max(kR, 16), the smallest N an M = 128
// MMA of this kind takes: the operand reads and the MMA time follow the real
// query rows, not the 64 rows the tiles are laid out for.
template <int kN>
__device__ __forceinline__ void dec_issue_qk(uint32_t tmem_s, uint32_t k_addr, uint32_t q_addr) {
  constexpr uint32_t idesc = make_idesc_bf16(kDecTile, kN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint64_t a = make_sdesc_sw128(k_addr + kk * 32, 16, 1024);
    const uint64_t b = make_sdesc_sw128(q_addr + kk * 32, 16, 1024);
    mma_ss(tmem_s, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// S^T = K Q^T in fp16 with K (32 packed columns) read from TMEM.
template <int kN>
__device__ __forceinline__ void dec_issue_qk_ts(uint32_t tmem_s, uint32_t tmem_k, uint32_t q_addr) {
  constexpr uint32_t idesc = make_idesc_f16(kDecTile, kN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk) {
    const uint64_t b = make_sdesc_sw128(q_addr + kk * 32, 16, 1024);
    mma_ts(tmem_s, tmem_k + kk * 8, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// Two e4m3 codes (low byte first) -> two fp16 (low half first); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(codes & 0xFFFFu)));
  return h2;
}

// Row r of a byte tile (64 e4m3 codes) into registers, in element order.  The
// tile was written by TMA with the 64-byte swizzle: 16-byte chunk c of row r
// sits at chunk c ^ ((r >> 1) & 3), so the eight rows that one quarter-warp
// reads fall in eight different bank groups.
__device__ __forceinline__ void dec_row_load(const uint8_t* tile, int r, uint4* raw) {
  const uint4* row = reinterpret_cast<const uint4*>(tile + r * kHeadDim);
  const int swz = (r >> 1) & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) raw[q] = row[q ^ swz];
}

// 64 e4m3 codes -> 32 packed fp16 pairs (element order kept).
__device__ __forceinline__ void dec_row_widen(const uint4* raw, uint32_t* out) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w4[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      out[8 * q + 2 * u] = e4m3x2_to_f16x2(w4[u]);
      out[8 * q + 2 * u + 1] = e4m3x2_to_f16x2(w4[u] >> 16);
    }
  }
}

// Two bf16 (packed) -> two fp16 (packed), rounded to nearest, saturating.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t v) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(f.y), "f"(f.x));
  return r;
}

// O^T (+)= [V | 1]^T P^T over the 128 slots of a tile: A (M = 128) is read
// MN-major from the V tile (M rows 0..63) and the ones tile (M rows 64..127,
// reached through the descriptor's leading-byte offset); B = the first kN
// query rows of P^T [slots][64 rows], MN-major.
template <bool kF16, int kN>
__device__ __forceinline__ void dec_issue_pv(uint32_t tmem_o, uint32_t v_addr, uint32_t ones_addr, uint32_t p_addr,
                                             bool accumulate) {
  constexpr uint32_t idesc =
      kF16 ? make_idesc_f16(kDecTile, kN, 1, 1) : make_idesc_bf16(kDecTile, kN, 1, 1);
  const uint32_t lbo = ones_addr - v_addr;
#pragma unroll
  for (int kk = 0; kk < kDecTile / 16; ++kk) {
    const uint64_t a = make_sdesc_sw128(v_addr + kk * 2048, lbo, 1024);
    const uint64_t b = make_sdesc_sw128(p_addr + kk * 2048, kDecPBytes, 1024);
    mma_ss(tmem_o, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// O^T (+)= [V | 1]^T P^T in FP8 (tcgen05 kind::f8f6f4, e4m3 A and B, fp32
// accumulate, K = 32 slots per MMA): A (M = 128) read MN-major straight from
// the e4m3 V byte tile (M rows 0..63: 64 bytes per slot, 64-byte swizzle) and
// the e4m3 ones tile (M rows 64..127, through the leading-byte offset); B =
// the first kN query rows of P^T, e4m3 bytes [slots][64 rows], MN-major,
// 64-byte swizzle.
template <int kN>
__device__ __forceinline__ void dec_issue_pv_f8(uint32_t tmem_o, uint32_t v_addr, uint32_t ones_addr,
                                                uint32_t p_addr, bool accumulate) {
  constexpr uint32_t idesc = make_idesc_e4m3(kDecTile, kN, 1, 1);
  const uint32_t lbo = ones_addr - v_addr;
#pragma unroll
  for (int kk = 0; kk < kDecTile / 32; ++kk) {
    const uint64_t a = make_sdesc_sw64(v_addr + kk * 2048, lbo, 512);
    const uint64_t b = make_sdesc_sw64(p_addr + kk * 2048, kDecP8Bytes, 512);
    mma_ss_f8(tmem_o, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Two fp32 -> two e4m3 codes (low byte first), rounded to nearest even and
// saturated to +-448.
__device__ __forceinline__ uint32_t dec_f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// The 128 softmax threads (warps 0-3) on hardware barrier 1: an OR of one
// predicate over them, and a plain barrier.  Every softmax thread executes the
// same sequence of these (see the softmax loop), so none is left waiting.
__device__ __forceinline__ bool dec_group_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kDecTile)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void dec_group_sync() { named_barrier(1, kDecTile); }

// Loads / stores kN (8, 16, 32 or 64) consecutive TMEM columns of this warp's lanes.
template <int kN>
__device__ __forceinline__ void dec_tmem_ld(uint32_t taddr, uint32_t* r) {
  if constexpr (kN == 8) tmem_ld8(taddr, r);
  else if constexpr (kN == 16) tmem_ld16(taddr, r);
  else if constexpr (kN == 32) tmem_ld32(taddr, r);
  else tmem_ld64(taddr, r);
}
template <int kN>
__device__ __forceinline__ void dec_tmem_st(uint32_t taddr, const uint32_t* r) {
  if constexpr (kN == 8) {
    tmem_st8(taddr, r);
  } else if constexpr (kN == 16) {
    tmem_st16(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < kN / 32; ++c) tmem_st32(taddr + 32 * c, r + 32 * c);
  }
}

// kR: query rows handled in registers (8, 16, 32 or 64; >= G * Lq).
// kMode: 0 bf16 cache; 1 e4m3 cache (see the file comment); 2 e4m3 cache
// with the PV product in FP8 (P rounded to e4m3; V read as stored).
template <int kR, int kMode>
__global__ void __launch_bounds__(kMode ? kDecThreads8 : kDecThreads, (kMode && kR > 16) ? 1 : 2)
    sink_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  constexpr bool kF8 = kMode >= 1;
  constexpr bool kPv8 = kMode == 2;
  constexpr int kStages = kF8 ? kDecStages8 : kDecStages;
  constexpr int kTileB = kF8 ? kDecKv8Bytes : kDecKvBytes;  // bytes of one staged K or V tile
  constexpr int kThreads = kF8 ? kDecThreads8 : kDecThreads;
  constexpr int kN = kR < 16 ? 16 : kR;  // MMA N: query rows the MMAs compute
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sK = smem;                                   // stages of K tiles
  uint8_t* sV = sK + kStages * kTileB;                  // stages of V tiles
  uint8_t* sVb = sV + kStages * kTileB;                 // e4m3 cache: two widened V tiles (fp16)
  uint8_t* sOnes = sVb + ((kF8 && !kPv8) ? 2 * kDecKvBytes : 0);  // [128][64] ones
  uint8_t* sP = sOnes + (kPv8 ? kDecKv8Bytes : kDecKvBytes);      // P^T
  uint8_t* sQ = sP + (kPv8 ? kDecP8Bytes : kDecPBytes);           // Q rows (8 KB, 1024-aligned)
  DecCtl* ctl = reinterpret_cast<DecCtl*>(sQ + kDecQBytes);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const DecWork w = dec_work(p);

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_conv, kDecTile);
    mbar_init(&ctl->v_ready[0], kDecTile);
    mbar_init(&ctl->v_ready[1], kDecTile);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], kF8 ? kDecTile : 1);  // e4m3: freed by the 128 widening threads
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], (kF8 && !kPv8) ? kDecTile : 1);  // FP8 PV: released by the MMA
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->s_full[b], 1);
      mbar_init(&ctl->s_free[b], kDecTile);
      mbar_init(&ctl->kt_full[b], kDecTile);
    }
    mbar_init(&ctl->p_full, kDecTile);
    mbar_init(&ctl->pv_done[0], 1);
    mbar_init(&ctl->pv_done[1], 1);
    mbar_init(&ctl->o_full, 1);
    ctl->abort = 0;
    if (w.bad) atomicCAS(&g_device_error, 0, static_cast<int>(kDevErrDecodeCacheTooSmall));
    fence_mbar_init();
  }
  if (threadIdx.x < kDecRows) {
    float m0 = -INFINITY;
    if (threadIdx.x < p.R) m0 = __ldg(p.sinks + w.g * p.G + (threadIdx.x & (p.G - 1))) * kLog2e;
    ctl->m_ref[threadIdx.x] = m0;
    ctl->alpha[threadIdx.x] = 1.f;
  }
  // Constant operands written by the threads: the ones tile, zeroed P^T and
  // zeroed Q padding rows (the TMA fills rows [0, R)).
  {
    // 1.0 in e4m3 codes / fp16 pairs / bf16 pairs
    const uint32_t one2 = kPv8 ? 0x38383838u : (kF8 ? 0x3C003C00u : 0x3F803F80u);
    const uint4 ones = make_uint4(one2, one2, one2, one2);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    constexpr int kOnesChunks = (kPv8 ? kDecKv8Bytes : kDecKvBytes) / 16;
    constexpr int kPChunks = (kPv8 ? kDecP8Bytes : kDecPBytes) / 16;
    for (int i = threadIdx.x; i < kOnesChunks; i += kThreads) reinterpret_cast<uint4*>(sOnes)[i] = ones;
    for (int i = threadIdx.x; i < kPChunks; i += kThreads) reinterpret_cast<uint4*>(sP)[i] = zero;
    for (int i = p.R * 8 + threadIdx.x; i < kDecQBytes / 16; i += kThreads) reinterpret_cast<uint4*>(sQ)[i] = zero;
    fence_proxy_async_smem();
  }
  if (warp == kDecMmaWarp) {
    tmem_alloc(&ctl->tmem_base, kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kDecProducerWarp) {
    // ---------------------------------------------------------- TMA producer
    if (w.n > 0 && elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&ctl->q_full, p.R * kHeadDim * 2);
      tma_load_3d(sQ, &tm_q, &ctl->q_full, 0, w.g * p.G, w.b * p.Lq);
      const int row0 = w.b * p.C + w.z0;
      for (int i = 0; i < w.n; ++i) {
        const int s = i % kStages;
        const uint32_t par = ((i / kStages) - 1) & 1;
        if (i >= kStages && !mbar_wait(&ctl->k_empty[s], par, abort, &g_device_error, kDevErrTimeoutProducer))
          break;
        mbar_arrive_expect_tx(&ctl->k_full[s], kTileB);
        tma_load_3d(sK + s * kTileB, &tm_k, &ctl->k_full[s], 0, w.g, row0 + i * kDecTile);
        if (i >= kStages && !mbar_wait(&ctl->v_empty[s], par, abort, &g_device_error, kDevErrTimeoutProducer))
          break;
        mbar_arrive_expect_tx(&ctl->v_full[s], kTileB);
        tma_load_3d(sV + s * kTileB, &tm_v, &ctl->v_full[s], 0, w.g, row0 + i * kDecTile);
      }
    }
  } else if (warp == kDecMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // S^T_i, then O^T += ... for tile i - 1 (its P^T is written while S^T_i
    // is being computed).
    if (w.n > 0 && elect_one()) {
      const uint32_t tS = tmem + kDecTmemS;
      const uint32_t tO = tmem + kDecTmemO;
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t ones_addr = smem_u32(sOnes);
      const uint32_t p_addr = smem_u32(sP);
      bool ok = kF8 ? mbar_wait(&ctl->q_conv, 0, abort, &g_device_error, kDevErrTimeoutMma)
                    : mbar_wait(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutMma);
      for (int i = 0; ok && i <= w.n; ++i) {
        if (i < w.n) {
          const int b = i & 1;
          const int s = i % kStages;
          // e4m3: K_i widened into TMEM buffer b by the softmax threads.
          ok = (i < 2 || mbar_wait(&ctl->s_free[b], ((i >> 1) - 1) & 1, abort, &g_device_error, kDevErrTimeoutMma)) &&
               (kF8 ? mbar_wait(&ctl->kt_full[b], (i >> 1) & 1, abort, &g_device_error, kDevErrTimeoutMma)
                    : mbar_wait(&ctl->k_full[s], (i / kStages) & 1, abort, &g_device_error, kDevErrTimeoutMma));
          if (!ok) break;
          tc_fence_after();
          if constexpr (kF8) {
            dec_issue_qk_ts<kN>(tS + b * kDecRows, tmem + kDecTmemK + 32 * b, q_addr);
            tc_commit(&ctl->s_full[b]);
          } else {
            dec_issue_qk<kN>(tS + b * kDecRows, smem_u32(sK + s * kDecKvBytes), q_addr);
            tc_commit(&ctl->s_full[b]);
            tc_commit(&ctl->k_empty[s]);
          }
        }
        if (i >= 1) {
          const int j = i - 1;
          const int s = j % kStages;
          // e4m3: V_j widened into fp16 tile j % 2 (v_ready); FP8 PV: the
          // V bytes as loaded (the softmax threads zero empty slots' rows
          // before their P^T arrival).
          ok = mbar_wait(&ctl->p_full, j & 1, abort, &g_device_error, kDevErrTimeoutMma) &&
               ((kF8 && !kPv8)
                    ? mbar_wait(&ctl->v_ready[j & 1], (j >> 1) & 1, abort, &g_device_error, kDevErrTimeoutMma)
                    : mbar_wait(&ctl->v_full[s], (j / kStages) & 1, abort, &g_device_error, kDevErrTimeoutMma));
          if (!ok) break;
          tc_fence_after();
          if constexpr (kPv8) {
            dec_issue_pv_f8<kN>(tO, smem_u32(sV + s * kTileB), ones_addr, p_addr, j > 0);
          } else {
            dec_issue_pv<kF8, kN>(tO, kF8 ? smem_u32(sVb + (j & 1) * kDecKvBytes) : smem_u32(sV + s * kDecKvBytes),
                                  ones_addr, p_addr, j > 0);
          }
          tc_commit(&ctl->pv_done[j & 1]);
          if constexpr (!kF8 || kPv8) tc_commit(&ctl->v_empty[s]);
        }
      }
      if (ok) tc_commit(&ctl->o_full);
    }
  } else if (warp >= kDecConvWarp0) {
    // ------------------- e4m3 cache: widen K and V, one slot per thread
    if constexpr (kF8) {
      const int kl = 32 * (warp & 3) + (threadIdx.x & 31);  // slot == the TMEM lane this warp may access
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const int last_slot = dec_last_slot(w.L, p.C);
      bool ok = true;
      if (w.n > 0) {
        // Q (bf16, as loaded) -> fp16 in place: elementwise, so the swizzle
        // does not matter; the zeroed padding rows stay zero.
        ok = mbar_wait(&ctl->q_full, 0, abort, &g_device_error, kDevErrTimeoutDecode);
        if (ok) {
          uint32_t* qw = reinterpret_cast<uint32_t*>(sQ);
          for (int e = kl; e < kDecQBytes / 4; e += kDecTile) qw[e] = bf16x2_to_f16x2_sat(qw[e]);
          fence_proxy_async_smem();
          mbar_arrive(&ctl->q_conv);
        }
      }
      for (int i = 0; ok && i < w.n; ++i) {
        const int b = i & 1;
        const int s = i % kStages;
        uint32_t buf[32];
        // K_i -> TMEM buffer b, whose last reader was the S^T MMA of tile i-2.
        if (i >= 2) {
          ok = mbar_wait(&ctl->s_full[b], ((i - 2) >> 1) & 1, abort, &g_device_error, kDevErrTimeoutDecode);
          if (!ok) break;
          tc_fence_after();
        }
        ok = mbar_wait(&ctl->k_full[s], (i / kStages) & 1, abort, &g_device_error, kDevErrTimeoutDecode);
        if (!ok) break;
        uint4 raw[4];
        dec_row_load(sK + s * kTileB, kl, raw);
        dec_row_widen(raw, buf);
        tmem_st32(tmem + lane_base + kDecTmemK + 32 * b, buf);
        // Release the byte stage only after its values have been consumed
        // (a shared load may still be in flight until its result is used),
        // and order these generic reads before the next TMA write there.
        fence_proxy_async_smem();
        mbar_arrive(&ctl->k_empty[s]);
        tc_fence_before();
        mbar_arrive(&ctl->kt_full[b]);
        if constexpr (kPv8) continue;  // the FP8 PV reads the V bytes as loaded
        // V_i -> fp16 tile i % 2, whose last reader was the PV MMA of tile
        // i-2.  A slot that holds no token may hold any bits (NaN included)
        // and its V row is still multiplied by P = 0: it becomes zeros.
        if (i >= 2) {
          ok = mbar_wait(&ctl->pv_done[i & 1], ((i - 2) >> 1) & 1, abort, &g_device_error, kDevErrTimeoutDecode);
          if (!ok) break;
        }
        ok = mbar_wait(&ctl->v_full[s], (i / kStages) & 1, abort, &g_device_error, kDevErrTimeoutDecode);
        if (!ok) break;
        const int z = w.z0 + i * kDecTile + kl;
        const int pos = z < p.C ? dec_slot_pos(z, w.L, last_slot, p.C) : -1;
        if (pos >= 0) {
          dec_row_load(sV + s * kTileB, kl, raw);
          dec_row_widen(raw, buf);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) buf[c] = 0u;
        }
        uint8_t* vline = sVb + (i & 1) * kDecKvBytes + (kl >> 3) * 1024 + (kl & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(vline + ((c ^ (kl & 7)) << 4)) =
              make_uint4(buf[4 * c], buf[4 * c + 1], buf[4 * c + 2], buf[4 * c + 3]);
        fence_proxy_async_smem();  // the fp16 tile for the MMA; the byte reads before the next TMA
        mbar_arrive(&ctl->v_empty[s]);
        mbar_arrive(&ctl->v_ready[i & 1]);
      }
    }
  } else {
    // ---------------------------------------- softmax (1 key per thread)
    const int kl = threadIdx.x;  // slot within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    // e4m3: logits carry k_scale, O carries v_scale.
    const float sl2 = kF8 ? p.scale_log2 * __ldg(p.k_scale + w.g) : p.scale_log2;
    const int last_slot = dec_last_slot(w.L, p.C);
    // The reference max of each row, also kept in registers (it changes only
    // when raised, below); kR = 64 reads it from shared memory instead.
    float mreg[kR <= 32 ? kR : 1];
    if constexpr (kR <= 32) {
#pragma unroll
      for (int n = 0; n < kR; ++n) mreg[n] = ctl->m_ref[n];
    }
    auto mref = [&](int n) -> float {
      if constexpr (kR <= 32) return mreg[n];
      else return ctl->m_ref[n];
    };
    // Every softmax thread runs all w.n iterations and meets the other 127 at
    // the group barrier once per tile (three times on a raise), also after an
    // abort: then it only skips the work, so no barrier is left waiting.
    // Wait outcomes are made warp-uniform for the .sync.aligned TMEM ops.
    bool ok = true;
    for (int i = 0; i < w.n; ++i) {
      const int b = i & 1;
      // Mask: slot -> position -> the query rows that see it.  New token t
      // (position L0 + t, rows t*G .. t*G + G - 1) sees position pos iff
      // pos <= L0 + t and, with a window, L0 + t - pos < window: one range of
      // tokens, hence one range [n_lo, n_lo + n_span) of rows.
      const int z = w.z0 + i * kDecTile + kl;
      const int pos = z < p.C ? dec_slot_pos(z, w.L, last_slot, p.C) : -1;
      int n_lo = 0, n_span = 0;  // (computed before the wait for S, which it overlaps)
      if (pos >= 0) {
        const int t_lo = max(0, pos - w.L0);
        const int t_hi = p.window > 0 ? min(p.Lq, pos - w.L0 + p.window) : p.Lq;
        n_lo = t_lo * p.G;
        n_span = max(0, t_hi * p.G - n_lo);
      }
      asm volatile("" ::"r"(n_lo), "r"(n_span));
      if (ok) ok = mbar_wait(&ctl->s_full[b], (i >> 1) & 1, abort, &g_device_error, kDevErrTimeoutDecode);
      ok = __all_sync(0xffffffffu, ok);
      float x[kR];
      if (ok) {
        tc_fence_after();
        uint32_t raw[kR];
        dec_tmem_ld<kR>(tmem + lane_base + kDecTmemS + b * kDecRows, raw);
#pragma unroll
        for (int n = 0; n < kR; ++n) x[n] = __uint_as_float(raw[n]);
        tc_fence_before();
        mbar_arrive(&ctl->s_free[b]);
      } else {
#pragma unroll
        for (int n = 0; n < kR; ++n) x[n] = -INFINITY;
      }
      bool viol = false;
#pragma unroll
      for (int n = 0; n < kR; ++n) {
        const bool allowed = static_cast<unsigned>(n - n_lo) < static_cast<unsigned>(n_span);
        x[n] = allowed ? x[n] * sl2 : -INFINITY;
        viol |= x[n] > mref(n) + kDecRescaleLog2;
      }
      // Raise the reference max only when some key exceeds it by more than
      // 2^8: an OR over the 128 keys, taken in the barrier hardware.
      const bool raise = dec_group_any(viol);
      if (raise) {
#pragma unroll
        for (int n = 0; n < kR; ++n) {
          if (n < p.R) {
            float v = x[n];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if ((kl & 31) == 0) ctl->wmax[warp][n] = v;
          }
        }
        dec_group_sync();
        if (kl < p.R) {
          const float tmax = fmaxf(fmaxf(ctl->wmax[0][kl], ctl->wmax[1][kl]), fmaxf(ctl->wmax[2][kl], ctl->wmax[3][kl]));
          const float mr = ctl->m_ref[kl];
          const bool up = tmax > mr + kDecRescaleLog2;
          ctl->alpha[kl] = up ? ex2_approx(mr - tmax) : 1.f;
          if (up) ctl->m_ref[kl] = tmax;
        }
        dec_group_sync();
        if constexpr (kR <= 32) {
#pragma unroll
          for (int n = 0; n < kR; ++n) mreg[n] = ctl->m_ref[n];
        }
      }
      if (!ok) continue;
      // P^T row of this key, packed to bf16 / fp16 pairs (rows 2c, 2c+1),
      // or (FP8 PV) to e4m3 codes, four rows per word (rows 4c..4c+3).
      uint32_t pk[kR / 2];
#pragma unroll
      for (int c = 0; c < kR / 2; ++c) {
        const float m0 = mref(2 * c), m1 = mref(2 * c + 1);
        const float e0 = ex2_approx(x[2 * c] - (m0 == -INFINITY ? 0.f : m0));
        const float e1 = ex2_approx(x[2 * c + 1] - (m1 == -INFINITY ? 0.f : m1));
        if constexpr (kPv8) {
          const uint32_t codes = dec_f32x2_to_e4m3x2(e0, e1);
          pk[c / 2] = (c & 1) ? (pk[c / 2] | (codes << 16)) : codes;
        } else {
          pk[c] = kF8 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
        }
      }
      // The previous PV read P^T and wrote O^T: wait for it before both.
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&ctl->pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort,
                                               &g_device_error, kDevErrTimeoutDecode));
        if (!ok) continue;
        if (raise) {
          // O^T[lane][n] *= alpha[n]: head dims in lanes 0..63, row sums in
          // lanes 64..127, query rows in columns.
          tc_fence_after();
          uint32_t o[kR];
          dec_tmem_ld<kR>(tmem + lane_base + kDecTmemO, o);
#pragma unroll
          for (int n = 0; n < kR; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * ctl->alpha[n]);
          dec_tmem_st<kR>(tmem + lane_base + kDecTmemO, o);
        }
      }
      // A slot that holds no token (never written, or past this sequence's
      // C slots) may hold any bits, NaN included, and its V row is still
      // multiplied by P = 0: its row of the V operand is zeroed.
      if ((!kF8 || kPv8) && __any_sync(0xffffffffu, pos < 0)) {
        const int sv = i % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&ctl->v_full[sv], (i / kStages) & 1, abort, &g_device_error,
                                               kDevErrTimeoutDecode));
        if (!ok) continue;
        if (pos < 0) {
          if constexpr (kPv8) {
            // e4m3 bytes: the slot's 64-byte row (its chunks permuted within it)
            uint4* vrow = reinterpret_cast<uint4*>(sV + sv * kTileB + kl * kHeadDim);
#pragma unroll
            for (int c = 0; c < 4; ++c) vrow[c] = make_uint4(0u, 0u, 0u, 0u);
          } else {
            uint4* vrow = reinterpret_cast<uint4*>(sV + sv * kDecKvBytes + (kl >> 3) * 1024 + (kl & 7) * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      if constexpr (kPv8) {
        // P^T [slot kl][rows] in e4m3: 64 B per slot, 16-byte chunk c (rows
        // 16c..16c+15) at chunk position c ^ ((kl >> 1) & 3) (64-byte swizzle).
        uint8_t* line = sP + kl * kDecRows;
        if constexpr (kR == 8) {
          *reinterpret_cast<uint2*>(line + ((0 ^ ((kl >> 1) & 3)) << 4)) = make_uint2(pk[0], pk[1]);
        } else {
#pragma unroll
          for (int c = 0; c < kR / 16; ++c) {
            if (c * 16 < p.R)
              *reinterpret_cast<uint4*>(line + ((c ^ ((kl >> 1) & 3)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
      } else {
        // P^T [slot kl][rows]: 128 B per slot, 16-byte chunk c (rows 8c..8c+7)
        // at chunk position c ^ (kl % 8).
        uint8_t* line = sP + (kl >> 3) * 1024 + (kl & 7) * 128;
#pragma unroll
        for (int c = 0; c < kR / 8; ++c) {
          if (c * 8 < p.R)
            *reinterpret_cast<uint4*>(line + ((c ^ (kl & 7)) << 4)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }

    // ------------------------------------------------------------ partials
    const size_t cta = static_cast<size_t>(blockIdx.x);
    bool have = ok && w.n > 0;
    if (have) have = mbar_wait(&ctl->o_full, 0, abort, &g_device_error, kDevErrTimeoutEpilogue);
    have = __all_sync(0xffffffffu, have);
    if (have) tc_fence_after();
    if (p.n_split == 1) {
      // One split covers the whole cache: finish here (what the combine
      // kernel does for several splits), m = max(s, m_0),
      // l = e^{s-m} + l_0 e^{m_0-m}, out = O_0 e^{m_0-m} / l, lse = m + ln l
      // (exponents in base 2), and skip the combine launch.
      if (warp < 3) {
        uint32_t o[kR];
        if (have) {
          __syncwarp();
          dec_tmem_ld<kR>(tmem + lane_base + kDecTmemO, o);
        }
        if (kl == 64) {
          // Lane 64: the row sums -> per-row output factor and lse.
#pragma unroll
          for (int n = 0; n < kR; ++n) {
            if (n >= p.R) continue;
            const int h = (w.g << p.G_log2) + (n & (p.G - 1));
            const float s2 = __ldg(p.sinks + h) * kLog2e;
            const float m0 = (have && w.n > 0) ? ctl->m_ref[n] : -INFINITY;
            const float m = fmaxf(s2, m0);
            float l = 0.f, f = 0.f;
            if (m != -INFINITY) {
              if (s2 != -INFINITY) l = ex2_approx(s2 - m);
              if (m0 != -INFINITY) {
                f = ex2_approx(m0 - m);
                l = fmaf(__uint_as_float(o[n]), f, l);
              }
            }
            ctl->alpha[n] = l > 0.f ? f / l : 0.f;
            const int t = n >> p.G_log2;
            p.lse_out[static_cast<size_t>(h) * (p.batch * p.Lq) + w.b * p.Lq + t] =
                l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
          }
        }
        named_barrier(2, 96);  // warps 0-2: the factors are in shared memory
        if (warp < 2) {
          // Lanes 0..63: head dim kl of every query row.
          const float vs = kF8 ? __ldg(p.v_scale + w.g) : 1.f;
#pragma unroll
          for (int n = 0; n < kR; ++n) {
            if (n >= p.R) continue;
            const int h = (w.g << p.G_log2) + (n & (p.G - 1));
            const int t = n >> p.G_log2;
            const float y = have ? __uint_as_float(o[n]) * vs * ctl->alpha[n] : 0.f;
            p.out[(static_cast<size_t>(w.b * p.Lq + t) * p.Hq + h) * kHeadDim + kl] = __float2bfloat16_rn(y);
          }
        }
      }
    } else if (warp < 3) {
      uint32_t o[kR];
      if (have) {
        __syncwarp();
        dec_tmem_ld<kR>(tmem + lane_base + kDecTmemO, o);
      }
      if (warp < 2) {
        // Lanes 0..63: head dim kl of every query row.
        float* dst = p.o_part + cta * kDecRows * kHeadDim + kl;
        const float vs = kF8 ? __ldg(p.v_scale + w.g) : 1.f;
#pragma unroll
        for (int n = 0; n < kR; ++n)
          if (n < p.R) dst[n * kHeadDim] = have ? __uint_as_float(o[n]) * vs : 0.f;
      } else if (kl == 64) {
        // Lane 64: the row sums.
#pragma unroll
        for (int n = 0; n < kR; ++n)
          if (n < p.R) p.l_part[cta * kDecRows + n] = have ? __uint_as_float(o[n]) : 0.f;
      }
    }
    if (p.n_split > 1 && kl < p.R) p.m_part[cta * kDecRows + kl] = (w.n > 0) ? ctl->m_ref[kl] : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDecMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kDecTmemCols);
  }
}

// Merges the splits of every (sequence, new token, query head) and adds the
// sink: m = max(s, m_k), l = e^{s-m} + sum_k l_k e^{m_k-m},
// out = sum_k O_k e^{m_k-m} / l, lse = m + ln l (exponents in base 2 here).
// One warp per output row, two head dims per lane.
__global__ void __launch_bounds__(128) sink_attn_decode_combine_kernel(const DecParams p, __nv_bfloat16* out,
                                                                       float* lse) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);  // (b * Lq + t) * Hq + h
  const int lane = threadIdx.x & 31;
  const int total = p.batch * p.Lq * p.Hq;
  if (row >= total) return;
  const int h = row % p.Hq;
  const int bt = row / p.Hq;
  const int b = bt / p.Lq;
  const int t = bt % p.Lq;
  const int g = h >> p.G_log2;
  const int n = (t << p.G_log2) + (h & (p.G - 1));
  const size_t base = (static_cast<size_t>(b) * p.Hkv + g) * p.n_split;
  const float s2 = __ldg(p.sinks + h) * kLog2e;
  float m = s2;
  for (int k = 0; k < p.n_split; ++k) m = fmaxf(m, p.m_part[(base + k) * kDecRows + n]);
  float l = 0.f, o0 = 0.f, o1 = 0.f;
  if (m != -INFINITY) {
    if (s2 != -INFINITY) l = ex2_approx(s2 - m);
    for (int k = 0; k < p.n_split; ++k) {
      const float mk = p.m_part[(base + k) * kDecRows + n];
      if (mk == -INFINITY) continue;
      const float f = ex2_approx(mk - m);
      l = fmaf(p.l_part[(base + k) * kDecRows + n], f, l);
      const float2 v = reinterpret_cast<const float2*>(p.o_part + ((base + k) * kDecRows + n) * kHeadDim)[lane];
      o0 = fmaf(v.x, f, o0);
      o1 = fmaf(v.y, f, o1);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  reinterpret_cast<uint32_t*>(out + static_cast<size_t>(row) * kHeadDim)[lane] = pack_bf16x2(o0 * inv, o1 * inv);
  if (lane == 0) lse[static_cast<size_t>(h) * (p.batch * p.Lq) + bt] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
}

// Writes the new tokens' keys and values into their cache slots: token t of
// sequence b goes to slot (cache_seqlens[b] + t) mod C.  One thread per 16
// bytes.
__global__ void __launch_bounds__(256) sink_attn_cache_append_kernel(const DecParams p, const uint4* k_new,
                                                                     const uint4* v_new, uint4* k_cache,
                                                                     uint4* v_cache) {
  constexpr int kChunks = kHeadDim * 2 / 16;  // 16-byte chunks per [D] row
  const long long total = static_cast<long long>(p.batch) * p.Lq * p.Hkv * kChunks;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= 2 * total) return;
  const bool is_v = i >= total;
  const long long e = is_v ? i - total : i;
  const int c = static_cast<int>(e % kChunks);
  const long long r = e / kChunks;  // (b * Lq + t) * Hkv + g
  const int g = static_cast<int>(r % p.Hkv);
  const long long bt = r / p.Hkv;
  const int b = static_cast<int>(bt / p.Lq);
  const int t = static_cast<int>(bt % p.Lq);
  const int L0 = __ldg(p.seqlens + b);
  if (L0 < 0) return;  // reported by the attention kernel
  const int slot = (L0 + t) % p.C;
  const size_t dst = ((static_cast<size_t>(b) * p.C + slot) * p.Hkv + g) * kChunks + c;
  if (is_v) v_cache[dst] = v_new[e];
  else k_cache[dst] = k_new[e];
}

// Appends the new tokens to an e4m3 cache: code = e4m3(x * (1 / scale[g]))
// (round to nearest even, saturated to the largest finite code, +-448).  One
// thread per 16 codes (two 16-byte loads of bf16 input, one 16-byte store).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(256) sink_attn_cache_append_e4m3_kernel(const DecParams p, const uint4* k_new,
                                                                          const uint4* v_new, uint4* k_cache,
                                                                          uint4* v_cache) {
  constexpr int kChunks = kHeadDim / 16;  // 16-code chunks per [D] row
  const long long total = static_cast<long long>(p.batch) * p.Lq * p.Hkv * kChunks;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= 2 * total) return;
  const bool is_v = i >= total;
  const long long e = is_v ? i - total : i;
  const int c = static_cast<int>(e % kChunks);
  const long long r = e / kChunks;  // (b * Lq + t) * Hkv + g
  const int g = static_cast<int>(r % p.Hkv);
  const long long bt = r / p.Hkv;
  const int b = static_cast<int>(bt / p.Lq);
  const int t = static_cast<int>(bt % p.Lq);
  const int L0 = __ldg(p.seqlens + b);
  if (L0 < 0) return;  // reported by the attention kernel
  const int slot = (L0 + t) % p.C;
  const float inv = 1.f / __ldg((is_v ? p.v_scale : p.k_scale) + g);
  const uint4* src = (is_v ? v_new : k_new) + r * (kHeadDim / 8) + 2 * c;  // 16 bf16
  uint32_t w[8];
  const uint4 a = src[0], bq = src[1];
  const uint32_t in[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[u]));
    w[u] = f32x2_to_e4m3x2(f.x * inv, f.y * inv);
  }
  const size_t dst = ((static_cast<size_t>(b) * p.C + slot) * p.Hkv + g) * kChunks + c;
  (is_v ? v_cache : k_cache)[dst] = make_uint4(w[0] | (w[1] << 16), w[2] | (w[3] << 16), w[4] | (w[5] << 16),
                                               w[6] | (w[7] << 16));
}

}  // namespace sa
